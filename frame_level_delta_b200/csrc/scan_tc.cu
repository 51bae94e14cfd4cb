// Bidirectional scan on tcgen05 tensor cores (Video DeltaNet summary,
// onedev.kr/papers/80, section "how it works": a forward and a reverse state,
// both started at S_T/2; section "how to use": S_t = S_{t-1} M_t + C_t).
//
// One CTA per (b, h, direction) runs the recurrence frame by frame, or chunk by
// chunk over the maps the composition kernel formed (same step, same operands):
//   S <- S M_t + C_t,  S = Sh + Sl, M_t = Mh + Ml (bf16 parts, ~2^-16 relative),
//   S M_t ~= Sh Mh + Sh Ml + Sl Mh  (24 MMAs of 128x128x16, fp32 in TMEM).
// S lives in TMEM twice: as the fp32 accumulator (two buffers, alternating by
// step) and as the bf16 hi/lo A operand of the next step's MMAs. The epilogue
// (one thread per state row and column group) adds C_t, writes the readout
// states of the chunks that need this state and the hi/lo operand, 32-column
// K-chunk by K-chunk, so the next step's MMAs start on the first chunk while
// the rest are still being written. M_t's hi/lo images (the B operand, in the
// layout the solve wrote) arrive by bulk copies, double-buffered; C_t rows are
// prefetched into registers (and into L2 two steps ahead) during the MMAs.
//
// In frame mode after the sweep solve (the default path) the step is written
// as S <- (S Diag(alpha_t) + B_t) P_t, which equals S M_t + C_t: the solve then
// writes only P_t's images, and the epilogue of step t forms the next step's
// operand S Diag(alpha_{t+1}) + B_{t+1} (one FMA per element; alpha from a
// four-deep ring of bulk copies, B rows prefetched) before it splits it into
// the hi/lo A operand. The first operand is S_T/2 Diag(alpha) + B of the
// direction's first frame.
//
// In frame mode the kernel may be launched while the solve's last CTAs still
// run (programmatic dependent launch): the copy thread then acquires each
// slot's ready word before it copies that slot's M_t or lets the epilogue read
// its C_t (through a counter in shared memory), so the scan advances through
// every frame the solve has finished.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace vda {

namespace {

constexpr int D = 128;
constexpr int kThreads = 320;  // copy warp, MMA warp, eight epilogue warps
constexpr int kImg = D * D * 2;           // one bf16 operand image
constexpr int kMBuf = 2 * kImg;           // hi + lo images of one M_t
constexpr int kARing = 4;                 // pform: alpha of the frames two steps ahead
constexpr int kAOff = 2 * kMBuf;          // pform: alpha ring (kARing x D floats)
constexpr int kBarOff = kAOff + kARing * D * 4;  // barriers after the two M buffers and the alpha ring
constexpr int kSmemUsed = kBarOff + 128 + 1024;
// Launched while the solve's last CTAs run, a scan CTA must not share an SM
// with one (67 KB of shared memory each): it would wait in tcgen05.alloc for
// the solve CTA's TMEM columns instead of starting on a free SM.
constexpr int kSmemBytes = kSmemUsed > 164 * 1024 ? kSmemUsed : 164 * 1024;
// TMEM columns: two fp32 accumulators (step st uses (st & 1) * 128..), then S
// as the A operand, bf16 hi and lo pairs (state column j in column j / 2).
constexpr uint32_t kShi = 256, kSlo = 320;
constexpr uint32_t kIdesc = sm100::idesc_bf16_f32(128, 128, false, true);  // A (S, TMEM) K-major, B (M) MN-major


struct ScanArgs {
  int B, H, T, c, J;
  int chunked;        // 1: step over composed chunk maps, 0: over frames
  const float* C;     // [B,H,T-1,D,D]; slot 0 = S_T
  const uint8_t* Mi;  // [B,H,T-1] x (hi, lo) operand images
  const uint8_t* CMi; // [B,H,2,J] x (hi, lo) composed chunk transitions
  const float* CC;    // [B,H,2,J,D,D] composed chunk injections
  const uint32_t* ready;  // [B,H,T-1] slot-ready words to acquire first, or nullptr
  // Injection form. 0: the step operands are M_t = Diag(alpha_t) P_t and the
  // injections C_t = B_t P_t. 1: the operands are P_t and the epilogue forms the
  // next product's left factor S Diag(alpha_t) + B_t itself, since
  // S M_t + C_t = (S Diag(alpha_t) + B_t) P_t; C_t is never materialised.
  int pform;
  const float* Bm;     // [B,H,T-1,D,D] B_t (pform)
  const float* alpha;  // [B,H,T,D] (pform)
  float* Sf;
  float* Sr;
  uint32_t* status;
  unsigned long long wait_ns;
};

__device__ __forceinline__ void split8(const float* x, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __nv_bfloat162 hh = __floats2bfloat162_rn(x[2 * q], x[2 * q + 1]);
    const float2 hf = __bfloat1622float2(hh);
    h[q] = sm100::bf162_bits(hh);
    // x - hi is exact in fp32; one packed add for the pair.
    const float2 d = __fadd2_rn(make_float2(x[2 * q], x[2 * q + 1]), make_float2(-hf.x, -hf.y));
    l[q] = sm100::bf162_bits(__floats2bfloat162_rn(d.x, d.y));
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// 16 consecutive values of a state row as 8 hi and 8 lo bf16 pairs (lower
// column in the low half): the TMEM A-operand layout.
__device__ __forceinline__ void split16(const float* x, uint32_t (&hi)[8], uint32_t (&lo)[8]) {
  uint4 h0, l0, h1, l1;
  split8(x, h0, l0);
  split8(x + 8, h1, l1);
  hi[0] = h0.x; hi[1] = h0.y; hi[2] = h0.z; hi[3] = h0.w; hi[4] = h1.x; hi[5] = h1.y; hi[6] = h1.z; hi[7] = h1.w;
  lo[0] = l0.x; lo[1] = l0.y; lo[2] = l0.z; lo[3] = l0.w; lo[4] = l1.x; lo[5] = l1.y; lo[6] = l1.z; lo[7] = l1.w;
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          sm100::smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(sm100::smem_u32(bar))
      : "memory");
}

__global__ void __launch_bounds__(kThreads, 1) scan_tc_kernel(const ScanArgs a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = sm100::align_smem_1024(smem_raw);
  uint8_t* sM = smem;           // [2][hi, lo]
  const float* sA = reinterpret_cast<const float*>(smem + kAOff);  // [kARing][D]
  uint64_t* mfull = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* mempty = mfull + 2;
  uint64_t* tfull = mempty + 2;
  uint64_t* sready = tfull + 1;  // [4]: K-chunk q (state columns 32q..32q+31) of the next image written
  uint64_t* drain = sready + 4;
  uint64_t* afull = drain + 1;  // [kARing] pform: alpha of step st in buffer st % kARing
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(afull + kARing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // Slots whose ready word the copy thread has acquired: 1 = slot 0 (S_T), then
  // st + 2 once step st's slot is.
  uint32_t* cgot = reinterpret_cast<uint32_t*>(tmem_slot + 2);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.x, dir = blockIdx.y;
  const int c = a.c, T = a.T, J = a.J;
  const int f_first = dir == 0 ? 1 : T - 2;
  const int f_last = dir == 0 ? c * (J - 2) - 1 : 2 * c;
  const int nsteps = a.chunked ? max(0, J - 2) : max(0, dir == 0 ? f_last - f_first + 1 : f_first - f_last + 1);
  const long long slots = (long long)bh * (T - 1);
  // Step st absorbs frame f(st), or chunk m(st) (forward m = st, reverse m = J-1-st),
  // whose transition image and injection rows are:
  auto step_img = [&](int st) -> const uint8_t* {
    if (a.chunked) return a.CMi + (((long long)bh * 2 + dir) * J + (dir == 0 ? st : J - 1 - st)) * (long long)kMBuf;
    return a.Mi + (slots + (dir == 0 ? f_first + st : f_first - st)) * (long long)kMBuf;
  };
  auto step_c = [&](int st) -> const float* {
    if (a.chunked) return a.CC + (((long long)bh * 2 + dir) * J + (dir == 0 ? st : J - 1 - st)) * (long long)D * D;
    return a.C + (slots + (dir == 0 ? f_first + st : f_first - st)) * (long long)D * D;
  };
  // Frame mode with pform: B_t and alpha_t of step st's frame.
  auto step_b = [&](int st) -> const float* {
    return a.Bm + (slots + (dir == 0 ? f_first + st : f_first - st)) * (long long)D * D;
  };
  auto step_alpha = [&](int st) -> const float* {
    return a.alpha + ((long long)bh * T + (dir == 0 ? f_first + st : f_first - st)) * D;
  };

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&mfull[s], 1);
      mbar_init(&mempty[s], 1);
    }
    mbar_init(tfull, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&sready[q], 8);
    mbar_init(drain, 1);
    for (int r = 0; r < kARing; ++r) mbar_init(&afull[r], 1);
    *abort_flag = 0;
    *cgot = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);  // two accumulators and the S operand
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  int issued = 0;
  int aissued = 0;  // alpha copies issued (steps 0 .. aissued - 1)

  if (warp == 0) {
    if (lane == 0) {
      bool go = a.ready == nullptr || flag_wait_gpu(a.ready + slots, 1u, abort_flag, a.status, a.wait_ns);
      if (go) smem_release_u32(cgot, 1u);
      for (int st = 0; go && a.pform && st < 2 && st < nsteps; ++st) {  // alpha is an input: no slot to wait for
        mbar_arrive_expect_tx(&afull[st], D * 4);
        bulk_load(smem + kAOff + st * D * 4, step_alpha(st), D * 4, &afull[st]);
        aissued = st + 1;
      }
      for (int st = 0; go && st < nsteps; ++st) {
        const int s = st & 1;
        // Acquire the slot before anything reads it: ahead of the wait for the
        // buffer, so the epilogue's C_t loads find it already acquired.
        if (a.ready != nullptr) {
          const int f = dir == 0 ? f_first + st : f_first - st;
          if (!flag_wait_gpu(a.ready + slots + f, 1u, abort_flag, a.status, a.wait_ns)) break;
          fence_proxy_async_global();
        }
        smem_release_u32(cgot, (uint32_t)st + 2u);
        if (!mbar_wait(&mempty[s], ((st >> 1) & 1) ^ 1, abort_flag, a.status, a.wait_ns)) break;
        mbar_arrive_expect_tx(&mfull[s], kMBuf);
        const uint8_t* src = step_img(st);
        // alpha two steps ahead: its buffer's previous frame (st - 2) was read by
        // the epilogue before it released the operand of step st - 2, whose MMA
        // freed the image buffer waited for above.
        if (a.pform && st + 2 < nsteps) {
          const int r = (st + 2) % kARing;
          mbar_arrive_expect_tx(&afull[r], D * 4);
          bulk_load(smem + kAOff + r * D * 4, step_alpha(st + 2), D * 4, &afull[r]);
          aissued = st + 3;
        }
        // The injection rows the epilogue reads with plain loads (C_t of this
        // step, or B_t of this and the next step under pform): into L2 now.
        if (!a.pform) {
          asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(step_c(st)), "r"((uint32_t)(D * D * 4))
                       : "memory");
        } else {
          // The epilogue of step st reads B of step st + 1: fetch two steps ahead.
          for (int u = st == 0 ? 0 : st + 2; u <= st + 2 && u < nsteps; ++u)
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(step_b(u)), "r"((uint32_t)(D * D * 4))
                         : "memory");
        }
        bulk_load(sM + s * kMBuf, src, kImg, &mfull[s]);
        bulk_load(sM + s * kMBuf + kImg, src + kImg, kImg, &mfull[s]);
        issued = st + 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool run = true;
      for (int st = 0; st < nsteps && run; ++st) {
        const int s = st & 1;
        const uint32_t acc = tmem + (uint32_t)(st & 1) * 128;
        if (!mbar_wait(&mfull[s], (st >> 1) & 1, abort_flag, a.status, a.wait_ns)) break;
        const uint32_t mh = smem_u32(sM + s * kMBuf), ml = mh + kImg;
        const uint32_t as[3] = {kShi, kShi, kSlo}, bs[3] = {mh, ml, mh};
        // K-chunk by K-chunk, as soon as the epilogue has written that part of S.
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (!mbar_wait(&sready[q], st & 1, abort_flag, a.status, a.wait_ns)) {
            run = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 2 * q; kk < 2 * q + 2; ++kk)
#pragma unroll
            for (int t = 0; t < 3; ++t) {
              const uint64_t db = smem_desc_sw128(bs[t] + kk * 2048, D * 128, 1024);
              mma_f16_ts(acc, tmem + as[t] + kk * 8, db, kIdesc, (kk == 0 && t == 0) ? 0u : 1u);
            }
        }
        if (!run) break;
        mma_commit(&mempty[s]);
        mma_commit(tfull);
      }
      mma_commit(drain);
    }
  } else {
    // Eight epilogue warps: warp w serves TMEM lanes (state rows) 32 (w % 4)..
    // and the 16-column groups 2 cc + hf (cc = 0..3), so both warps of a lane
    // quadrant finish each 32-column K-chunk of the next image together and the
    // chunks reach the MMAs one after the other, as early as possible.
    const int q = warp % 4;
    const int hf = (warp - 2) / 4;
    const int i = q * 32 + lane;  // state row == TMEM lane
    constexpr int kCols = D / 2;
    auto col_of = [&](int cc) { return 16 * (2 * cc + hf); };
    const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
    float* out = dir == 0 ? a.Sf : a.Sr;
    auto store_row = [&](int j, const float* x, int col0, int n) {
      float4* d4 = reinterpret_cast<float4*>(out + ((long long)bh * J + j) * D * D);
      for (int t = 0; t < n / 4; ++t)
        d4[(col0 / 4 + t) * D + i] = make_float4(x[4 * t], x[4 * t + 1], x[4 * t + 2], x[4 * t + 3]);
    };
    // x (16 state columns col..) <- x Diag(alpha) + B, row i: a pform operand
    // (alpha from shared memory).
    auto next_operand = [&](float* x, const float* bsrc, const float* al, int col0) {
      const float4* b4 = reinterpret_cast<const float4*>(bsrc);
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float4 w = b4[(col0 / 4 + t) * D + i];
        const float4 g = reinterpret_cast<const float4*>(al + col0)[t];
        const float2 p0 = __ffma2_rn(make_float2(x[4 * t], x[4 * t + 1]), make_float2(g.x, g.y), make_float2(w.x, w.y));
        const float2 p1 =
            __ffma2_rn(make_float2(x[4 * t + 2], x[4 * t + 3]), make_float2(g.z, g.w), make_float2(w.z, w.w));
        x[4 * t] = p0.x; x[4 * t + 1] = p0.y; x[4 * t + 2] = p1.x; x[4 * t + 3] = p1.y;
      }
    };
    // Initial state S_T / 2: readout states of the chunks that see no frame of
    // this direction, and the first operand image.
    // Under pform the first operand is S_T/2 Diag(alpha) + B of the first frame:
    // its slot must be acquired too.
    bool live = smem_wait_geq(cgot, (a.pform && nsteps > 0) ? 2u : 1u, abort_flag, a.status, a.wait_ns);
    // ... and its alpha, copied with the first frame's images.
    if (live && a.pform && nsteps > 0) live = mbar_wait(&afull[0], 0, abort_flag, a.status, a.wait_ns);
    if (live) {
      const float4* st0 = reinterpret_cast<const float4*>(a.C + slots * (long long)D * D);
      float4 row[kCols / 4];  // all of this warp's columns first: one load latency
#pragma unroll
      for (int cc = 0; cc < kCols / 16; ++cc)
#pragma unroll
        for (int t = 0; t < 4; ++t) row[cc * 4 + t] = st0[(col_of(cc) / 4 + t) * D + i];
#pragma unroll
      for (int c16 = 0; c16 < kCols / 16; ++c16) {
        const int col = col_of(c16);
        float x[16];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float4 v = row[c16 * 4 + t];
          x[4 * t] = 0.5f * v.x; x[4 * t + 1] = 0.5f * v.y; x[4 * t + 2] = 0.5f * v.z; x[4 * t + 3] = 0.5f * v.w;
        }
        for (int j = 0; j < J; ++j)
          if (dir == 0 ? (c * (j - 1) - 1 <= 0) : (c * (j + 2) >= T - 1)) store_row(j, x, col, 16);
        if (a.pform && nsteps > 0) next_operand(x, step_b(0), sA, col);
        uint32_t hi[8], lo[8];
        split16(x, hi, lo);
        tmem_st8(tl + kShi + col / 2, hi);
        tmem_st8(tl + kSlo + col / 2, lo);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0)
        for (int q4 = 0; q4 < 4; ++q4) mbar_arrive(&sready[q4]);
    }
    for (int st = 0; live && st < nsteps; ++st) {
      const int f = dir == 0 ? f_first + st : f_first - st;
      // Under pform the epilogue of step st forms the operand of step st + 1.
      const bool nxt = a.pform && st + 1 < nsteps;
      if (!smem_wait_geq(cgot, (uint32_t)st + (nxt ? 3u : 2u), abort_flag, a.status, a.wait_ns)) break;
      // Prefetch this warp's columns of the injection's row i while the MMAs run:
      // C_t of this step, or B_t of the next step under pform.
      float crow[kCols];
      if (!a.pform || nxt) {
        const float4* csrc = reinterpret_cast<const float4*>(a.pform ? step_b(st + 1) : step_c(st));
#pragma unroll
        for (int cc = 0; cc < kCols / 16; ++cc)
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float4 v = csrc[(col_of(cc) / 4 + t) * D + i];
            crow[16 * cc + 4 * t] = v.x; crow[16 * cc + 4 * t + 1] = v.y;
            crow[16 * cc + 4 * t + 2] = v.z; crow[16 * cc + 4 * t + 3] = v.w;
          }
      }
      // alpha of the next step's frame, copied two steps ahead.
      if (nxt && !mbar_wait(&afull[(st + 1) % kARing], ((st + 1) / kARing) & 1, abort_flag, a.status, a.wait_ns))
        break;
      const float* anext = nxt ? sA + ((st + 1) % kARing) * D : nullptr;
      if (!mbar_wait(tfull, st & 1, abort_flag, a.status, a.wait_ns)) break;
      tc_fence_after();
      int jout = -1;
      if (a.chunked) {
        jout = dir == 0 ? st + 2 : (J - 1 - st) - 2;  // after chunk m: readout state of chunk m+2 / m-2
      } else if (dir == 0) {
        if ((f + 1) % c == 0 && (f + 1) / c + 1 < J) jout = (f + 1) / c + 1;
      } else {
        if (f % c == 0 && f / c - 2 >= 0) jout = f / c - 2;
      }
#pragma unroll
      for (int c16 = 0; c16 < kCols / 16; ++c16) {
        const int col = col_of(c16);
        // pform: this group's alpha, read while the accumulator columns load.
        float4 g[4];
        if (nxt) {
#pragma unroll
          for (int t = 0; t < 4; ++t) g[t] = reinterpret_cast<const float4*>(anext + col)[t];
        }
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(st & 1) * 128 + col, v);
        tmem_ld_wait();
        // The new state's 16 columns: the product plus C_t, or under pform the
        // product itself. A readout state is stored as it is formed (the stores
        // do not hold up the operand).
        // (Packed fp32x2 arithmetic: the epilogue's instruction issue paces the scan.)
        float x[16];
        if (!a.pform) {
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const float2 r = __fadd2_rn(make_float2(__uint_as_float(v[2 * t]), __uint_as_float(v[2 * t + 1])),
                                        make_float2(crow[c16 * 16 + 2 * t], crow[c16 * 16 + 2 * t + 1]));
            x[2 * t] = r.x;
            x[2 * t + 1] = r.y;
          }
        } else {
#pragma unroll
          for (int t = 0; t < 16; ++t) x[t] = __uint_as_float(v[t]);
        }
        if (jout >= 0) store_row(jout, x, col, 16);
        if (nxt) {  // pform: the next operand is S Diag(alpha) + B
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float* cr = crow + c16 * 16 + 4 * t;
            const float2 p0 = __ffma2_rn(make_float2(x[4 * t], x[4 * t + 1]), make_float2(g[t].x, g[t].y),
                                         make_float2(cr[0], cr[1]));
            const float2 p1 = __ffma2_rn(make_float2(x[4 * t + 2], x[4 * t + 3]), make_float2(g[t].z, g[t].w),
                                         make_float2(cr[2], cr[3]));
            x[4 * t] = p0.x; x[4 * t + 1] = p0.y; x[4 * t + 2] = p1.x; x[4 * t + 3] = p1.y;
          }
        }
        uint32_t hi[8], lo[8];
        split16(x, hi, lo);
        tmem_st8(tl + kShi + col / 2, hi);
        tmem_st8(tl + kSlo + col / 2, lo);
        // This warp's part of K-chunk col / 32 of the next operand is in TMEM: release it.
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sready[col >> 5]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      int last = -1;
      for (int st = s; st < issued; st += 2) last = st;
      if (last >= 0) mbar_wait(&mfull[s], (last >> 1) & 1, nullptr, a.status, a.wait_ns);
    }
    for (int r = 0; r < kARing; ++r) {
      int last = -1;
      for (int st = r; st < aissued; st += kARing) last = st;
      if (last >= 0) mbar_wait(&afull[r], (last / kARing) & 1, nullptr, a.status, a.wait_ns);
    }
  }
  if (warp == 1) {
    if (lane == 0) mbar_wait(drain, 0, nullptr, a.status, a.wait_ns);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool scan_tc_supported(const Problem& p) { return solve_tc_supported(p); }

cudaError_t launch_scan_tc(const Problem& p, cudaStream_t s, bool chunked) {
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(scan_tc_kernel), kSmemBytes);
  if (e != cudaSuccess) return e;
  // Composed chunks come from a kernel that ran after the whole solve: only the
  // frame scan waits on the slot-ready words, and only it overlaps the solve.
  const bool overlap = !chunked && p.ready != nullptr;
  ScanArgs a{p.B, p.H, p.T, p.c, p.J, chunked ? 1 : 0, p.C, static_cast<const uint8_t*>(p.Msplit),
             static_cast<const uint8_t*>(p.CMi), p.CC, overlap ? p.ready : nullptr,
             (!chunked && p.pform) ? 1 : 0, p.Bm, p.alpha, p.Sf, p.Sr, p.status, p.spin_limit};
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(p.B * p.H, 2);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = overlap ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, scan_tc_kernel, a);
}

}  // namespace vda
