// Bidirectional frame scan on tcgen05, each state's columns split over a
// two-CTA cluster (Video DeltaNet summary, onedev.kr/papers/80, section "how it
// works": a forward and a reverse state, both started at S_T/2; section "how to
// use": S_t = S_{t-1} M_t + C_t, here in the form S_t = (S_{t-1} Diag(alpha_t)
// + B_t) P_t with P_t = (I + A_t)^-1 from the sweep solve).
//
// One cluster of two CTAs per (b, h, direction). CTA r owns state columns
// 64 r .. 64 r + 63 and computes, per frame,
//   S_t[:, r] = L_t P_t[:, r],   L_t = S_{t-1} Diag(alpha_t) + B_t   (128 x 128),
// as 24 MMAs of 128 x 64 x 16 (L = Lh + Ll and P = Ph + Pl in bf16 parts,
// L P ~= Lh Ph + Lh Pl + Ll Ph, ~2^-16 relative; fp32 accumulator in TMEM).
// The left factor is a K-major operand in shared memory, double-buffered: the
// epilogue of step t writes its 64 columns of L_{t+1} (one 64-wide K atom,
// 32 KB as hi and lo images) and one bulk copy forwards them into the same
// place in the peer CTA, completing on the peer's barrier. Each CTA reads only
// its 64-column atom of P_t's images. Against one CTA per (b, h, direction)
// this halves the tensor time, the epilogue and the P bytes per CTA.
//
// The double buffer needs no other synchronisation: the peer writes L_{t+2}
// into this CTA's buffer only after its own step t+1 MMAs, which needed this
// CTA's half of L_{t+1}, which this CTA sent after its step t MMAs had read the
// buffer. Likewise this CTA rewrites its half of a buffer two steps after it
// sent it, and by then the copy has landed (the peer's MMAs consumed it).
//
// Launched while the solve's last CTAs still run (programmatic dependent
// launch), the copy thread acquires each slot's ready word before it copies
// that slot's P_t or lets the epilogue read its B_t (through a counter in
// shared memory), so the scan advances through every frame the solve has
// finished.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace vda {

namespace {

constexpr int D = 128;
constexpr int DH = 64;                        // state columns per CTA
constexpr int kThreads = 320;                 // copy warp, MMA warp, eight epilogue warps
constexpr int kHalfImg = D * DH * 2;          // one 64-column atom of a bf16 image (16 KB)
constexpr int kPBuf = 2 * kHalfImg;           // hi + lo atoms of P_t (32 KB)
constexpr int kLAtom = 2 * kHalfImg;          // hi + lo images of one 64-wide K atom of L
constexpr int kLBuf = 2 * kLAtom;             // both K atoms of L (64 KB)
constexpr int kARing = 4;                     // alpha of the frames two steps ahead
constexpr int kLOff = 2 * kPBuf;              // two L buffers after the two P buffers
constexpr int kAOff = kLOff + 2 * kLBuf;      // alpha ring (kARing x DH floats)
constexpr int kBarOff = kAOff + kARing * DH * 4;
constexpr int kSmemBytes = kBarOff + 256 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory");
// TMEM: two fp32 accumulators of 64 columns (step st uses (st & 1) * 64 ..).
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kIdesc = sm100::idesc_bf16_f32(128, DH, false, true);  // A (L) K-major, B (P) MN-major

struct SplitArgs {
  int B, H, T, c, J;
  const float* C;         // [B,H,T-1,D,D]; slot 0 = S_T
  const uint8_t* Mi;      // [B,H,T-1] x (hi, lo) images of P_t
  const uint32_t* ready;  // [B,H,T-1] slot-ready words to acquire first, or nullptr
  const float* Bm;        // [B,H,T-1,D,D] B_t
  const float* alpha;     // [B,H,T,D]
  float* Sf;
  float* Sr;
  uint32_t* status;
  unsigned long long wait_ns;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// This CTA's shared address `a` as the same offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          sm100::smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(sm100::smem_u32(bar))
      : "memory");
}
// Shared memory of this CTA -> shared memory of a peer CTA, completing `bytes`
// on the peer's barrier (both peer addresses from peer_addr).
__device__ __forceinline__ void bulk_to_peer(uint32_t dst_cluster, const void* src, uint32_t bytes,
                                             uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst_cluster),
      "r"(sm100::smem_u32(src)), "r"(bytes), "r"(bar_cluster)
      : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// 16 consecutive values of a row as 8 hi and 8 lo bf16 pairs (lower column in
// the low half).
__device__ __forceinline__ void split16(const float* x, uint4 (&hi)[2], uint4 (&lo)[2]) {
  uint32_t h[8], l[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const __nv_bfloat162 hh = __floats2bfloat162_rn(x[2 * q], x[2 * q + 1]);
    const float2 hf = __bfloat1622float2(hh);
    h[q] = sm100::bf162_bits(hh);
    // x - hi is exact in fp32; one packed add for the pair.
    const float2 d = __fadd2_rn(make_float2(x[2 * q], x[2 * q + 1]), make_float2(-hf.x, -hf.y));
    l[q] = sm100::bf162_bits(__floats2bfloat162_rn(d.x, d.y));
  }
  hi[0] = make_uint4(h[0], h[1], h[2], h[3]);
  hi[1] = make_uint4(h[4], h[5], h[6], h[7]);
  lo[0] = make_uint4(l[0], l[1], l[2], l[3]);
  lo[1] = make_uint4(l[4], l[5], l[6], l[7]);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1) scan_split_tc_kernel(const SplitArgs a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = sm100::align_smem_1024(smem_raw);
  uint8_t* sP = smem;  // [2][hi atom, lo atom] of P_t, this CTA's columns
  uint8_t* sL = smem + kLOff;  // [2][K atom 0, 1][hi, lo] of L
  const float* sA = reinterpret_cast<const float*>(smem + kAOff);  // [kARing][DH]
  uint64_t* mfull = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* mempty = mfull + 2;
  uint64_t* tfull = mempty + 2;
  uint64_t* sready = tfull + 1;  // [2]: K chunk q (own columns 32q..32q+31) of the next L written here
  uint64_t* lhalf = sready + 2;  // all of this CTA's half of the next L written (8 epilogue warps)
  uint64_t* lfull = lhalf + 1;   // [2]: the peer's half of L in buffer b has landed
  uint64_t* drain = lfull + 2;
  uint64_t* afull = drain + 1;   // [kARing]: alpha of step st in buffer st % kARing
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(afull + kARing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // Slots whose ready word the copy thread has acquired: 1 = slot 0 (S_T), then
  // st + 2 once step st's slot is.
  uint32_t* cgot = reinterpret_cast<uint32_t*>(tmem_slot + 2);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t r = cluster_rank(), peer = r ^ 1u;
  const int bh = blockIdx.x / 2, dir = blockIdx.y;
  const int c = a.c, T = a.T, J = a.J;
  const int f_first = dir == 0 ? 1 : T - 2;
  const int f_last = dir == 0 ? c * (J - 2) - 1 : 2 * c;
  const int nsteps = max(0, dir == 0 ? f_last - f_first + 1 : f_first - f_last + 1);
  const long long slots = (long long)bh * (T - 1);
  auto frame_of = [&](int st) { return dir == 0 ? f_first + st : f_first - st; };
  auto step_img = [&](int st) -> const uint8_t* { return a.Mi + (slots + frame_of(st)) * (long long)(2 * D * D * 2); };
  auto step_b = [&](int st) -> const float* { return a.Bm + (slots + frame_of(st)) * (long long)D * D; };
  auto step_alpha = [&](int st) -> const float* {
    return a.alpha + ((long long)bh * T + frame_of(st)) * D + DH * r;
  };

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&mfull[s], 1);
      mbar_init(&mempty[s], 1);
      mbar_init(&lfull[s], 1);
      mbar_init(&sready[s], 8);
    }
    mbar_init(tfull, 1);
    mbar_init(lhalf, 8);
    mbar_init(drain, 1);
    for (int q = 0; q < kARing; ++q) mbar_init(&afull[q], 1);
    *abort_flag = 0;
    *cgot = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  // The peer's barriers are initialised before any copy completes on them.
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  int issued = 0;
  int aissued = 0;  // alpha copies issued (steps 0 .. aissued - 1)
  bool sent = false;

  if (warp == 0) {
    if (lane == 0) {
      bool go = a.ready == nullptr || flag_wait_gpu(a.ready + slots, 1u, abort_flag, a.status, a.wait_ns);
      if (go) smem_release_u32(cgot, 1u);
      for (int st = 0; go && st < 2 && st < nsteps; ++st) {  // alpha is an input: no slot to wait for
        mbar_arrive_expect_tx(&afull[st], DH * 4);
        bulk_load(smem + kAOff + st * DH * 4, step_alpha(st), DH * 4, &afull[st]);
        aissued = st + 1;
      }
      for (int st = 0; go && st < nsteps; ++st) {
        const int s = st & 1;
        // Acquire the slot before anything reads it: ahead of the wait for the
        // buffer, so the epilogue's B_t loads find it already acquired.
        if (a.ready != nullptr) {
          if (!flag_wait_gpu(a.ready + slots + frame_of(st), 1u, abort_flag, a.status, a.wait_ns)) break;
          fence_proxy_async_global();
        }
        smem_release_u32(cgot, (uint32_t)st + 2u);
        if (!mbar_wait(&mempty[s], ((st >> 1) & 1) ^ 1, abort_flag, a.status, a.wait_ns)) break;
        mbar_arrive_expect_tx(&mfull[s], kPBuf);
        const uint8_t* src = step_img(st);
        // alpha two steps ahead: its buffer's previous frame (st - 2) was read by
        // the epilogue before it released the operand of step st - 2, whose MMAs
        // freed the image buffer waited for above.
        if (st + 2 < nsteps) {
          const int q = (st + 2) % kARing;
          mbar_arrive_expect_tx(&afull[q], DH * 4);
          bulk_load(smem + kAOff + q * DH * 4, step_alpha(st + 2), DH * 4, &afull[q]);
          aissued = st + 3;
        }
        // The epilogue of step st reads this CTA's columns of B of step st + 1
        // (column quads 16 r ..: one contiguous 32 KB range): into L2 two ahead.
        for (int u = st == 0 ? 0 : st + 2; u <= st + 2 && u < nsteps; ++u)
          asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(step_b(u) + (DH / 4) * r * D * 4),
                       "r"((uint32_t)(DH * D * 4))
                       : "memory");
        // This CTA's 64-column atom of each image.
        bulk_load(sP + s * kPBuf, src + r * kHalfImg, kHalfImg, &mfull[s]);
        bulk_load(sP + s * kPBuf + kHalfImg, src + D * D * 2 + r * kHalfImg, kHalfImg, &mfull[s]);
        issued = st + 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool run = true;
      for (int st = 0; st < nsteps && run; ++st) {
        const int s = st & 1, b = st & 1;
        const uint32_t acc = tmem + (uint32_t)(st & 1) * DH;
        if (!mbar_wait(&mfull[s], (st >> 1) & 1, abort_flag, a.status, a.wait_ns)) break;
        const uint32_t ph = smem_u32(sP + s * kPBuf), pl = ph + kHalfImg;
        const uint32_t lb = smem_u32(sL + b * kLBuf);
        // The peer's half of L_st completes this phase of lfull[b].
        mbar_arrive_expect_tx(&lfull[b], kLAtom);
        // Own K atom first (K chunk by K chunk, as the epilogue writes it), then
        // the peer's once it has landed.
        for (int h = 0; h < 2 && run; ++h) {
          const uint32_t atom = h == 0 ? r : peer;
          const uint32_t lh = lb + atom * kLAtom, ll = lh + kHalfImg;
          const uint32_t as[3] = {lh, lh, ll}, bs[3] = {ph, pl, ph};
          if (h == 1) {
            if (!mbar_wait(&lfull[b], (st >> 1) & 1, abort_flag, a.status, a.wait_ns)) {
              run = false;
              break;
            }
          }
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            if (h == 0 && !mbar_wait(&sready[q], st & 1, abort_flag, a.status, a.wait_ns)) {
              run = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 2 * q; kk < 2 * q + 2; ++kk)
#pragma unroll
              for (int t = 0; t < 3; ++t) {
                // K rows 64 atom + 16 kk .. of P: 8-row groups of 1024 bytes.
                const uint64_t da = smem_desc_sw128(as[t] + kk * 32, 16, 1024);
                const uint64_t db = smem_desc_sw128(bs[t] + (atom * 8 + kk * 2) * 1024, kHalfImg, 1024);
                mma_f16(acc, da, db, kIdesc, (h == 0 && kk == 0 && t == 0) ? 0u : 1u);
              }
          }
        }
        if (!run) break;
        mma_commit(&mempty[s]);
        mma_commit(tfull);
      }
      mma_commit(drain);
    }
  } else {
    // Eight epilogue warps: warp w serves TMEM lanes (state rows) 32 (w % 4) ..
    // and the 16-column groups 2 cc + hf (cc = 0, 1) of this CTA's 64 columns,
    // so both warps of a lane quadrant finish each 32-column K chunk together.
    const int q4 = warp % 4;
    const int hf = (warp - 2) / 4;
    const int i = q4 * 32 + lane;  // state row == TMEM lane
    auto col_of = [&](int cc) { return 16 * (2 * cc + hf); };  // local column
    const int gcol0 = DH * (int)r;                             // this CTA's first state column
    float* out = dir == 0 ? a.Sf : a.Sr;
    auto store_row = [&](int j, const float* x, int col) {
      float4* d4 = reinterpret_cast<float4*>(out + ((long long)bh * J + j) * D * D);
#pragma unroll
      for (int t = 0; t < 4; ++t)
        d4[((gcol0 + col) / 4 + t) * D + i] = make_float4(x[4 * t], x[4 * t + 1], x[4 * t + 2], x[4 * t + 3]);
    };
    // x (16 columns col..) <- x Diag(alpha) + B, row i.
    auto next_operand = [&](float* x, const float* bsrc, const float* al, int col) {
      const float4* b4 = reinterpret_cast<const float4*>(bsrc);
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float4 w = b4[((gcol0 + col) / 4 + t) * D + i];
        const float4 g = reinterpret_cast<const float4*>(al + col)[t];
        const float2 p0 = __ffma2_rn(make_float2(x[4 * t], x[4 * t + 1]), make_float2(g.x, g.y), make_float2(w.x, w.y));
        const float2 p1 =
            __ffma2_rn(make_float2(x[4 * t + 2], x[4 * t + 3]), make_float2(g.z, g.w), make_float2(w.z, w.w));
        x[4 * t] = p0.x; x[4 * t + 1] = p0.y; x[4 * t + 2] = p1.x; x[4 * t + 3] = p1.y;
      }
    };
    // 16 columns of row i of L (buffer b, this CTA's K atom) in the K-major
    // 128-byte-swizzled layout: row i at byte 128 i, 16-byte chunk k / 8 at
    // position (k / 8) ^ (i % 8).
    auto write_l = [&](int b, int col, const float* x) {
      uint4 hi[2], lo[2];
      split16(x, hi, lo);
      uint8_t* ah = sL + b * kLBuf + r * kLAtom;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int off = i * 128 + ((((col >> 3) + h) ^ (i & 7)) << 4);
        *reinterpret_cast<uint4*>(ah + off) = hi[h];
        *reinterpret_cast<uint4*>(ah + kHalfImg + off) = lo[h];
      }
    };
    // This warp's part of K chunk `kc` of L is written: make it visible to the
    // tensor cores and the bulk copy, then release it.
    auto release_chunk = [&](int kc) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sready[kc]);
    };
    // All of this CTA's half of L in buffer b is written: forward it (one
    // thread, once all eight warps have arrived).
    auto forward_half = [&](int b, int n) -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(lhalf);
      if (warp != 2) return true;
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait(lhalf, n & 1, abort_flag, a.status, a.wait_ns);
        if (ok) {
          const uint32_t src_off = kLOff + b * kLBuf + r * kLAtom;
          bulk_to_peer(peer_addr(smem_u32(smem + src_off), peer), smem + src_off, kLAtom,
                       peer_addr(smem_u32(&lfull[b]), peer));
          sent = true;
        }
      }
      return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    };
    // Initial state S_T / 2: readout states of the chunks that see no frame of
    // this direction, and the first operand L_0 = S_T/2 Diag(alpha) + B of the
    // direction's first frame (whose slot must be acquired, and its alpha copied).
    bool live = smem_wait_geq(cgot, nsteps > 0 ? 2u : 1u, abort_flag, a.status, a.wait_ns);
    if (live && nsteps > 0) live = mbar_wait(&afull[0], 0, abort_flag, a.status, a.wait_ns);
    if (live) {
      const float4* st0 = reinterpret_cast<const float4*>(a.C + slots * (long long)D * D);
      float4 row[8];  // both column groups first: one load latency
#pragma unroll
      for (int cc = 0; cc < 2; ++cc)
#pragma unroll
        for (int t = 0; t < 4; ++t) row[cc * 4 + t] = st0[((gcol0 + col_of(cc)) / 4 + t) * D + i];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int col = col_of(cc);
        float x[16];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float4 v = row[cc * 4 + t];
          x[4 * t] = 0.5f * v.x; x[4 * t + 1] = 0.5f * v.y; x[4 * t + 2] = 0.5f * v.z; x[4 * t + 3] = 0.5f * v.w;
        }
        for (int j = 0; j < J; ++j)
          if (dir == 0 ? (c * (j - 1) - 1 <= 0) : (c * (j + 2) >= T - 1)) store_row(j, x, col);
        if (nsteps > 0) {
          next_operand(x, step_b(0), sA, col);
          write_l(0, col, x);
          release_chunk(cc);
        }
      }
      if (nsteps > 0) live = forward_half(0, 0);
    }
    for (int st = 0; live && st < nsteps; ++st) {
      const int f = frame_of(st);
      // The epilogue of step st forms L_{st+1}.
      const bool nxt = st + 1 < nsteps;
      if (!smem_wait_geq(cgot, (uint32_t)st + (nxt ? 3u : 2u), abort_flag, a.status, a.wait_ns)) break;
      // Prefetch this warp's columns of B_{st+1}'s row i while the MMAs run.
      float crow[32];
      if (nxt) {
        const float4* csrc = reinterpret_cast<const float4*>(step_b(st + 1));
#pragma unroll
        for (int cc = 0; cc < 2; ++cc)
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float4 v = csrc[((gcol0 + col_of(cc)) / 4 + t) * D + i];
            crow[16 * cc + 4 * t] = v.x; crow[16 * cc + 4 * t + 1] = v.y;
            crow[16 * cc + 4 * t + 2] = v.z; crow[16 * cc + 4 * t + 3] = v.w;
          }
      }
      // alpha of the next step's frame, copied two steps ahead.
      if (nxt && !mbar_wait(&afull[(st + 1) % kARing], ((st + 1) / kARing) & 1, abort_flag, a.status, a.wait_ns))
        break;
      const float* anext = nxt ? sA + ((st + 1) % kARing) * DH : nullptr;
      if (!mbar_wait(tfull, st & 1, abort_flag, a.status, a.wait_ns)) break;
      tc_fence_after();
      int jout = -1;
      if (dir == 0) {
        if ((f + 1) % c == 0 && (f + 1) / c + 1 < J) jout = (f + 1) / c + 1;
      } else {
        if (f % c == 0 && f / c - 2 >= 0) jout = f / c - 2;
      }
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int col = col_of(cc);
        float4 g[4];
        if (nxt) {
#pragma unroll
          for (int t = 0; t < 4; ++t) g[t] = reinterpret_cast<const float4*>(anext + col)[t];
        }
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(st & 1) * DH + col, v);
        tmem_ld_wait();
        float x[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) x[t] = __uint_as_float(v[t]);
        // A readout state is stored as it is formed.
        if (jout >= 0) store_row(jout, x, col);
        if (nxt) {  // L_{st+1} = S_st Diag(alpha) + B
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float* cr = crow + cc * 16 + 4 * t;
            const float2 p0 = __ffma2_rn(make_float2(x[4 * t], x[4 * t + 1]), make_float2(g[t].x, g[t].y),
                                         make_float2(cr[0], cr[1]));
            const float2 p1 = __ffma2_rn(make_float2(x[4 * t + 2], x[4 * t + 3]), make_float2(g[t].z, g[t].w),
                                         make_float2(cr[2], cr[3]));
            x[4 * t] = p0.x; x[4 * t + 1] = p0.y; x[4 * t + 2] = p1.x; x[4 * t + 3] = p1.y;
          }
          write_l((st + 1) & 1, col, x);
          release_chunk(cc);
        }
      }
      if (nxt && !forward_half((st + 1) & 1, st + 1)) break;
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
    for (int q = 0; q < kARing; ++q) {
      int last = -1;
      for (int st = q; st < aissued; st += kARing) last = st;
      if (last >= 0) mbar_wait(&afull[q], (last / kARing) & 1, nullptr, a.status, a.wait_ns);
    }
  }
  // This CTA's copies into the peer have completed before either CTA retires.
  if (sent) bulk_wait_all();
  if (warp == 1) {
    if (lane == 0) mbar_wait(drain, 0, nullptr, a.status, a.wait_ns);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  __syncwarp();
  cluster_sync();
}

}  // namespace

bool scan_split_tc_supported(const Problem& p) { return p.D == 128 && p.pform; }

cudaError_t launch_scan_split_tc(const Problem& p, cudaStream_t s) {
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(scan_split_tc_kernel), kSmemBytes);
  if (e != cudaSuccess) return e;
  SplitArgs a{p.B, p.H, p.T, p.c, p.J, p.C, static_cast<const uint8_t*>(p.Msplit), p.ready,
              p.Bm, p.alpha, p.Sf, p.Sr, p.status, p.spin_limit};
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2 * p.B * p.H, 2);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.ready != nullptr ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, scan_split_tc_kernel, a);
}

}  // namespace vda
