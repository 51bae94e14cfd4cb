// Chunk composition for the bidirectional scan (Video DeltaNet summary,
// onedev.kr/papers/80, section "assumptions and limits", notes on the inference
// kernels: the frame maps of a VAE chunk compose into S_out = S_in M_chunk +
// J_chunk, and the shorter chunk sequence is scanned in both directions).
//
// One CTA per (chunk m, direction, b*h). The forward direction composes the
// chunk's non-anchor frames in increasing order, the reverse direction in
// decreasing order (the reverse scan absorbs later frames first):
//   (MM, JJ) <- (M_f0, C_f0);  for each next frame f: (MM, JJ) <- (MM M_f, JJ M_f + C_f).
// Only the chunks the readout states need are composed: forward m = 0..J-3,
// reverse m = 2..J-1; an empty chunk gets the identity map (I, 0).
//
// Both products are three-term split products (bf16 hi/lo, ~2^-16 relative)
// with fp32 accumulation. MM and JJ live in TMEM as the A operands (hi/lo bf16
// pairs), next to their two fp32 accumulators, so each step's epilogue (one
// thread per row) turns the accumulators into the next step's operands with
// TMEM loads and stores only. M_f, the B operand, is the hi/lo image the solve
// wrote, double-buffered in shared memory by bulk copies; C_f (fp32, column
// quads) is staged in shared memory by a bulk copy as well. The last step
// writes the composed map as a hi/lo operand image and JJ as fp32 column
// quads, exactly the operands of the chunk-level scan.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace vda {

namespace {

constexpr int D = 128;
constexpr int kThreads = 128;
constexpr int kImg = D * D * 2;   // one bf16 operand image
constexpr int kPair = 2 * kImg;   // hi + lo
constexpr int kCBytes = D * D * 4;
constexpr int kMfOff = 0;                      // two M_f buffers (hi, lo each)
constexpr int kCOff = 2 * kPair;               // C_f, fp32 column quads
constexpr int kBarOff = kCOff + kCBytes;
constexpr int kSmemBytes = kBarOff + 128 + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
// TMEM columns: accumulators of MM M_f and JJ M_f, then MM and JJ as A operands.
constexpr uint32_t kAccM = 0, kAccJ = 128, kMMh = 256, kMMl = 320, kJJh = 384, kJJl = 448;
constexpr uint32_t kIdesc = sm100::idesc_bf16_f32(128, 128, false, true);  // A K-major, B MN-major

struct ComposeArgs {
  int H, T, c, J;
  const uint8_t* Mi;  // per-frame M hi/lo images [B*H][T-1]
  const float* C;     // per-frame C [B*H][T-1][D][D] (column quads)
  uint8_t* CMi;       // [B*H][2][J] hi/lo images
  float* CC;          // [B*H][2][J][D][D] (column quads)
  uint32_t* status;
  unsigned long long wait_ns;
};

__device__ __forceinline__ uint32_t img_off(int row, int col) {
  const int atom = col >> 6, cc = col & 63;
  return (uint32_t)(atom * D * 128 + row * 128 + ((((cc >> 3) ^ (row & 7))) << 4) + (cc & 7) * 2);
}

__device__ __forceinline__ void split8(const float* x, uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __nv_bfloat162 hh = __floats2bfloat162_rn(x[2 * q], x[2 * q + 1]);
    const float2 hf = __bfloat1622float2(hh);
    h[q] = sm100::bf162_bits(hh);
    l[q] = sm100::bf162_bits(__floats2bfloat162_rn(x[2 * q] - hf.x, x[2 * q + 1] - hf.y));
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// 32 consecutive values of a row as 16 hi and 16 lo bf16 pairs (lower column
// in the low half): the TMEM A-operand layout.
__device__ __forceinline__ void split32(const float (&x)[32], uint32_t (&hi)[16], uint32_t (&lo)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 h, l;
    split8(x + 8 * q, h, l);
    hi[4 * q] = h.x; hi[4 * q + 1] = h.y; hi[4 * q + 2] = h.z; hi[4 * q + 3] = h.w;
    lo[4 * q] = l.x; lo[4 * q + 1] = l.y; lo[4 * q + 2] = l.z; lo[4 * q + 3] = l.w;
  }
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          sm100::smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(sm100::smem_u32(bar))
      : "memory");
}

// Store a split row chunk (8 values at columns col..col+7 of row `row`) into a hi/lo image pair.
__device__ __forceinline__ void put8(uint8_t* pair, int row, int col, const float* x) {
  uint4 hi, lo;
  split8(x, hi, lo);
  const uint32_t o = img_off(row, col);
  *reinterpret_cast<uint4*>(pair + o) = hi;
  *reinterpret_cast<uint4*>(pair + kImg + o) = lo;
}

__global__ void __launch_bounds__(kThreads, 1) compose_tc_kernel(const ComposeArgs a) {
  using namespace sm100;
  const int m = blockIdx.x, dir = blockIdx.y, bh = blockIdx.z;
  const int c = a.c, T = a.T, J = a.J;
  if (dir == 0 ? (m > J - 3) : (m < 2)) return;  // map not needed by any readout state
  const int lo = dir == 0 ? max(1, c * m) : c * m;
  const int hi = dir == 0 ? c * (m + 1) - 1 : min(c * (m + 1) - 1, T - 2);
  const int nf = hi >= lo ? hi - lo + 1 : 0;
  auto frame = [&](int k) { return dir == 0 ? lo + k : hi - k; };
  const long long slots = (long long)bh * (T - 1);
  const long long oc = ((long long)bh * 2 + dir) * J + m;  // output chunk index
  uint8_t* out_img = a.CMi + oc * kPair;
  float* out_c = a.CC + oc * (long long)D * D;
  const int i = threadIdx.x;  // matrix row == TMEM lane
  const int warp = threadIdx.x / 32;

  if (nf <= 1) {
    // Identity map for an empty chunk; a one-frame chunk is that frame's map.
    const float4* csrc = nf == 1 ? reinterpret_cast<const float4*>(a.C + (slots + frame(0)) * (long long)D * D) : nullptr;
    const uint8_t* msrc = nf == 1 ? a.Mi + (slots + frame(0)) * (long long)kPair : nullptr;
    for (int c8 = 0; c8 < D / 8; ++c8) {
      const uint32_t o = img_off(i, c8 * 8);
      if (nf == 1) {
        *reinterpret_cast<uint4*>(out_img + o) = *reinterpret_cast<const uint4*>(msrc + o);
        *reinterpret_cast<uint4*>(out_img + kImg + o) = *reinterpret_cast<const uint4*>(msrc + kImg + o);
      } else {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = (c8 * 8 + u == i) ? 1.f : 0.f;
        put8(out_img, i, c8 * 8, x);
      }
    }
    float4* cd = reinterpret_cast<float4*>(out_c);
    for (int t = 0; t < D / 4; ++t) cd[t * D + i] = nf == 1 ? csrc[t * D + i] : make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = sm100::align_smem_1024(smem_raw);
  uint8_t* sMf = smem + kMfOff;  // buffer s at sMf + s * kPair
  const float4* sC = reinterpret_cast<const float4*>(smem + kCOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOff);  // [2]: M_f landed in buffer s
  uint64_t* cbar = full + 2;                                     // C_f (and at first M_f0) landed
  uint64_t* mmabar = full + 3;                                   // this step's MMAs are complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(full + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto mi = [&](int k) { return a.Mi + (slots + frame(k)) * (long long)kPair; };
  auto ci = [&](int k) { return a.C + (slots + frame(k)) * (long long)D * D; };

  // Thread 0 issues every copy and MMA and counts, per barrier, the completions
  // it started and the ones it saw, so an abandoned step can be drained.
  int issued_full[2] = {0, 0}, seen_full[2] = {0, 0};
  int issued_c = 0, seen_c = 0, issued_mma = 0, seen_mma = 0;
  if (threadIdx.x == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    mbar_init(cbar, 1);
    mbar_init(mmabar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    // M_f0 (into buffer 1, read once by the threads) and C_f0; M_f1 into buffer 0.
    mbar_arrive_expect_tx(cbar, kPair + kCBytes);
    bulk_load(sMf + kPair, mi(0), kImg, cbar);
    bulk_load(sMf + kPair + kImg, mi(0) + kImg, kImg, cbar);
    bulk_load(smem + kCOff, ci(0), kCBytes, cbar);
    issued_c = 1;
    mbar_arrive_expect_tx(&full[0], kPair);
    bulk_load(sMf, mi(1), kImg, &full[0]);
    bulk_load(sMf + kImg, mi(1) + kImg, kImg, &full[0]);
    issued_full[0] = 1;
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);

  // ---------------- MM <- M_f0 (its image rows are already bf16 hi/lo pairs), JJ <- C_f0
  bool ok = mbar_wait(cbar, 0, abort_flag, a.status, a.wait_ns);
  if (threadIdx.x == 0 && ok) seen_c = 1;
  const bool started = !__syncthreads_or(!ok);
  if (started) {
    const uint8_t* m0 = sMf + kPair;
#pragma unroll 1
    for (int c32 = 0; c32 < D / 32; ++c32) {
      uint32_t mh[16], ml[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t o = img_off(i, c32 * 32 + 8 * q);
        const uint4 h = *reinterpret_cast<const uint4*>(m0 + o);
        const uint4 l = *reinterpret_cast<const uint4*>(m0 + kImg + o);
        mh[4 * q] = h.x; mh[4 * q + 1] = h.y; mh[4 * q + 2] = h.z; mh[4 * q + 3] = h.w;
        ml[4 * q] = l.x; ml[4 * q + 1] = l.y; ml[4 * q + 2] = l.z; ml[4 * q + 3] = l.w;
      }
      tmem_st16(tl + kMMh + c32 * 16, mh);
      tmem_st16(tl + kMMl + c32 * 16, ml);
      float xj[32];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 v = sC[(c32 * 8 + q) * D + i];
        xj[4 * q] = v.x; xj[4 * q + 1] = v.y; xj[4 * q + 2] = v.z; xj[4 * q + 3] = v.w;
      }
      uint32_t jh[16], jl[16];
      split32(xj, jh, jl);
      tmem_st16(tl + kJJh + c32 * 16, jh);
      tmem_st16(tl + kJJl + c32 * 16, jl);
    }
    tmem_st_wait();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && started) {
    // Buffer 1 and the C buffer are free again: M_f2 and C_f1.
    if (nf > 2) {
      mbar_arrive_expect_tx(&full[1], kPair);
      bulk_load(sMf + kPair, mi(2), kImg, &full[1]);
      bulk_load(sMf + kPair + kImg, mi(2) + kImg, kImg, &full[1]);
      issued_full[1] = 1;
    }
    mbar_arrive_expect_tx(cbar, kCBytes);
    bulk_load(smem + kCOff, ci(1), kCBytes, cbar);
    issued_c = 2;
  }

  // ---------------- steps k = 1 .. nf-1: absorb frame(k), whose map sits in buffer (k-1) & 1
#pragma unroll 1
  for (int k = 1; k < nf && started; ++k) {
    const int s = (k - 1) & 1;
    ok = true;
    if (threadIdx.x == 0) {
      ok = mbar_wait(&full[s], ((k - 1) >> 1) & 1, abort_flag, a.status, a.wait_ns);
      if (ok) {
        ++seen_full[s];
        tc_fence_after();
        const uint32_t mfh = smem_u32(sMf + s * kPair), mfl = mfh + kImg;
        const uint32_t am[3] = {kMMh, kMMh, kMMl}, aj[3] = {kJJh, kJJh, kJJl};
        const uint32_t bs[3] = {mfh, mfl, mfh};
#pragma unroll
        for (int t = 0; t < 3; ++t)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t db = smem_desc_sw128(bs[t] + kk * 2048, D * 128, 1024);
            const uint32_t acc = (t == 0 && kk == 0) ? 0u : 1u;
            mma_f16_ts(tmem + kAccM, tmem + am[t] + kk * 8, db, kIdesc, acc);
            mma_f16_ts(tmem + kAccJ, tmem + aj[t] + kk * 8, db, kIdesc, acc);
          }
        mma_commit(mmabar);
        ++issued_mma;
      }
    }
    // A failed wait in thread 0 sets the abort flag, which ends the others' waits.
    if (ok) ok = mbar_wait(mmabar, (k - 1) & 1, abort_flag, a.status, a.wait_ns);
    if (ok && threadIdx.x == 0) ++seen_mma;
    if (ok) ok = mbar_wait(cbar, k & 1, abort_flag, a.status, a.wait_ns);
    if (ok && threadIdx.x == 0) ++seen_c;
    // Every thread takes the same exit, so the block barriers below stay matched.
    if (__syncthreads_or(!ok)) break;
    tc_fence_after();
    // The MMAs are done with buffer s: the map two frames ahead goes there.
    if (threadIdx.x == 0 && k + 2 < nf) {
      mbar_arrive_expect_tx(&full[s], kPair);
      bulk_load(sMf + s * kPair, mi(k + 2), kImg, &full[s]);
      bulk_load(sMf + s * kPair + kImg, mi(k + 2) + kImg, kImg, &full[s]);
      ++issued_full[s];
    }
    const bool last = k + 1 == nf;
#pragma unroll 1
    for (int c32 = 0; c32 < D / 32; ++c32) {
      uint32_t v0[16], v1[16], w0[16], w1[16];
      tmem_ld16(tl + kAccM + c32 * 32, v0);
      tmem_ld16(tl + kAccM + c32 * 32 + 16, v1);
      tmem_ld16(tl + kAccJ + c32 * 32, w0);
      tmem_ld16(tl + kAccJ + c32 * 32 + 16, w1);
      tmem_ld_wait();
      float xm[32], xj[32];
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        xm[t] = __uint_as_float(v0[t]);
        xm[16 + t] = __uint_as_float(v1[t]);
        xj[t] = __uint_as_float(w0[t]);
        xj[16 + t] = __uint_as_float(w1[t]);
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {  // JJ M_f + C_f
        const float4 v = sC[(c32 * 8 + q) * D + i];
        xj[4 * q] += v.x; xj[4 * q + 1] += v.y; xj[4 * q + 2] += v.z; xj[4 * q + 3] += v.w;
      }
      if (last) {
        float4* cd = reinterpret_cast<float4*>(out_c);
#pragma unroll
        for (int q = 0; q < 4; ++q) put8(out_img, i, c32 * 32 + 8 * q, xm + 8 * q);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          cd[(c32 * 8 + q) * D + i] = make_float4(xj[4 * q], xj[4 * q + 1], xj[4 * q + 2], xj[4 * q + 3]);
      } else {
        uint32_t h[16], l[16];
        split32(xm, h, l);
        tmem_st16(tl + kMMh + c32 * 16, h);
        tmem_st16(tl + kMMl + c32 * 16, l);
        split32(xj, h, l);
        tmem_st16(tl + kJJh + c32 * 16, h);
        tmem_st16(tl + kJJl + c32 * 16, l);
      }
    }
    tmem_st_wait();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // Everyone is done with C_f: the next frame's C goes into the buffer.
    if (threadIdx.x == 0 && k + 1 < nf) {
      mbar_arrive_expect_tx(cbar, kCBytes);
      bulk_load(smem + kCOff, ci(k + 1), kCBytes, cbar);
      ++issued_c;
    }
  }

  // ---------------- teardown: nothing may be in flight when TMEM and smem go away
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {
    // Completions of one barrier arrive in order: waiting for the last one started covers all.
    for (int s = 0; s < 2; ++s)
      if (issued_full[s] > seen_full[s]) mbar_wait(&full[s], (issued_full[s] - 1) & 1, nullptr, a.status, a.wait_ns);
    if (issued_c > seen_c) mbar_wait(cbar, (issued_c - 1) & 1, nullptr, a.status, a.wait_ns);
    if (issued_mma > seen_mma) mbar_wait(mmabar, (issued_mma - 1) & 1, nullptr, a.status, a.wait_ns);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_compose_tc(const Problem& p, cudaStream_t s) {
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(compose_tc_kernel), kSmemBytes);
  if (e != cudaSuccess) return e;
  if (p.J < 3) return cudaSuccess;  // no readout state sees a composed chunk
  if ((long long)p.B * p.H > 65535) return cudaErrorInvalidConfiguration;
  ComposeArgs a{p.H, p.T, p.c, p.J, static_cast<const uint8_t*>(p.Msplit), p.C, static_cast<uint8_t*>(p.CMi),
                p.CC, p.status, p.spin_limit};
  dim3 grid(p.J, 2, p.B * p.H);
  compose_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(a);
  return cudaGetLastError();
}

}  // namespace vda
