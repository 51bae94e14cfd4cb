// Frame solve (Video DeltaNet summary, onedev.kr/papers/80, section "how to use":
// S_t (I + A_t) = Sbar_t + B_t, transition M_t = Diag(alpha_t)(I + A_t)^-1, with
// the inverse taken in the d_k x d_k key space; the injection is C_t = B_t (I + A_t)^-1).
//
// The Cholesky form of the solve, selected by VDA_SOLVE_CHOLESKY; the default
// path inverts I + A by the symmetric sweep (solve_tc.cu). Both give the same
// unique M_t and C_t.
//
// Per (b, h, slot), d = 128, one CTA of 256 threads, two CTAs per SM. Blocked
// right-looking Cholesky X = I + A = L L^T and the inverse W = L^-1 run together
// in one loop over 16-wide block columns kb, with X and the inverse's
// accumulator R (starting at I) held in TMEM as fp32:
//   1. read X's block column kb (one row per thread) and R's block row kb;
//   2. one warp factors the 16x16 diagonal block L_kk and inverts it;
//   3. the panel L[:, kb] = X[:, kb] L_kk^-T (independent 16-term dots per row)
//      and W's block row kb = L_kk^-1 R[kb, :] are formed on CUDA cores and
//      stored as bf16 hi/lo operand images;
//   4. tcgen05 applies both rank-16 updates, X -= Lp Lp^T and R -= Lp W[kb, :],
//      as three-term split products (error ~2^-16 relative) with fp32 accumulation.
// Then P = W^T W (tcgen05, same split), M = Diag(alpha) P (fp32 and the bf16
// hi/lo operand images the tensor-core scan loads as they are), and C = B P with
// B_t split into hi/lo in TMEM as the A operand. The text slot produces only C = S_T.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace vda {

namespace {

constexpr int D = 128;
constexpr int NB = D / 16;
constexpr int kThreads = 256;
constexpr int kImg = D * D * 2;       // one bf16 operand image (two 64-column atoms of D rows)
constexpr int kWOff = 0;              // W image (hi, lo), later the P image
constexpr int kLOff = 2 * kImg;       // current panel as a K-major image (hi, lo): one atom each
constexpr int kLPart = D * 128;       // 16 KB per part
constexpr int kRvOff = kLOff + 2 * kLPart;  // 1 / L_kk[j][j] (16 fp32)
constexpr int kLkOff = kRvOff + 1024;       // L_kk (16x16 fp32)
constexpr int kTbOff = kLkOff + 1024;       // R's block row kb (16 x D fp32)
constexpr int kBarOff = kTbOff + 16 * D * 4;
constexpr int kSmemBytes = kBarOff + 64 + 1024;
constexpr uint32_t kNegA = 1u << 13;
constexpr uint32_t kIdKK = sm100::idesc_bf16_f32(128, 128, false, false);  // A, B K-major
constexpr uint32_t kIdKM = sm100::idesc_bf16_f32(128, 128, false, true);   // A K-major, B MN-major
constexpr uint32_t kIdMM = sm100::idesc_bf16_f32(128, 128, true, true);    // A, B MN-major
constexpr uint32_t kAccX = 0, kAccR = 128, kTmemB = 128;  // TMEM columns

struct SolveArgs {
  int B, H, T;
  const float* A;
  const float* Bm;
  const float* alpha;
  float* M;
  float* C;
  uint8_t* Msplit;
  uint32_t* status;
  unsigned long long wait_ns;
};

// Byte offset of element (row, col) in a bf16 operand image with 128-byte rows of
// 64 elements, 16-byte chunks XOR-swizzled by (row % 8) and 64-column atoms of D
// rows one after the other (the 128-byte-swizzle canonical layout).
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

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  return sm100::bf162_bits(__floats2bfloat162_rn(a, b));
}

// Three-term split product: D (+/-)= Ah Bh + Ah Bl + Al Bh, K = 16 per call
// (one MMA per term) or K = 128 (eight K steps per term, MN-major operands).
__device__ __forceinline__ void mma3(uint32_t d, uint64_t ah, uint64_t al, uint64_t bh, uint64_t bl,
                                     uint32_t idesc, uint32_t acc_first) {
  sm100::mma_f16(d, ah, bh, idesc, acc_first);
  sm100::mma_f16(d, ah, bl, idesc, 1u);
  sm100::mma_f16(d, al, bh, idesc, 1u);
}

__global__ void __launch_bounds__(kThreads, 2) solve_chol_tc_kernel(const SolveArgs a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = sm100::align_smem_1024(smem_raw);
  uint8_t* wimg = smem + kWOff;
  uint8_t* limg = smem + kLOff;
  float* Rv = reinterpret_cast<float*>(smem + kRvOff);
  float* Lk = reinterpret_cast<float*>(smem + kLkOff);
  float* Tb = reinterpret_cast<float*>(smem + kTbOff);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int slot = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const long long off = (((long long)b * a.H + h) * (a.T - 1) + slot) * (long long)D * D;
  const int q = warp % 4, hc = warp / 4;
  const int ri = q * 32 + lane;  // TMEM lane / matrix row of this thread
  uint32_t phase = 0;            // parity of the next completion of `bar`
  int commits = 0;

  if (tid == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);

  // X = I + A into TMEM columns 0..127 and R = I into 128..255 (this thread: row
  // ri, columns hc*64 .. hc*64+63). All sixteen loads are issued before use.
  {
    const float4* src = reinterpret_cast<const float4*>(a.A + off);
    float4 v[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) v[t] = src[(hc * 16 + t) * D + ri];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t x[16], r[16];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int col = hc * 64 + c * 16 + 4 * t;
        const float4 w = v[c * 4 + t];
        x[4 * t] = __float_as_uint(w.x + (ri == col ? 1.f : 0.f));
        x[4 * t + 1] = __float_as_uint(w.y + (ri == col + 1 ? 1.f : 0.f));
        x[4 * t + 2] = __float_as_uint(w.z + (ri == col + 2 ? 1.f : 0.f));
        x[4 * t + 3] = __float_as_uint(w.w + (ri == col + 3 ? 1.f : 0.f));
#pragma unroll
        for (int u = 0; u < 4; ++u) r[4 * t + u] = __float_as_uint(ri == col + u ? 1.f : 0.f);
      }
      tmem_st16(tl + kAccX + hc * 64 + c * 16, x);
      tmem_st16(tl + kAccR + hc * 64 + c * 16, r);
    }
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t wbase = smem_u32(wimg), lbase = smem_u32(limg);
  for (int kb = 0; kb < NB; ++kb) {
    const int k0 = kb * 16;
    const int pw = k0 / 32, l0 = k0 % 32;  // warp and first lane holding rows k0..k0+15
    // ---- 1. block column kb of X (rows ri), block row kb of R (into Tb)
    float x[16];
    if (hc == 0) {
      uint32_t v[16];
      tmem_ld16(tl + kAccX + k0, v);
      tmem_ld_wait();
#pragma unroll
      for (int t = 0; t < 16; ++t) x[t] = __uint_as_float(v[t]);
    }
    if (q == pw) {
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t v[16];
        tmem_ld16(tl + kAccR + hc * 64 + c * 16, v);
        tmem_ld_wait();
        const int r = lane - l0;
        if (r >= 0 && r < 16) {
          float4* dst = reinterpret_cast<float4*>(Tb + r * D + hc * 64 + c * 16);
#pragma unroll
          for (int t = 0; t < 4; ++t)
            dst[t] = make_float4(__uint_as_float(v[4 * t]), __uint_as_float(v[4 * t + 1]),
                                 __uint_as_float(v[4 * t + 2]), __uint_as_float(v[4 * t + 3]));
        }
      }
    }
    // ---- 2. factor the diagonal block (warp pw, lanes l0..l0+15). Register arrays
    // are only ever indexed by constants: the current column is always g[0] and
    // the row shifts left after every pivot.
    if (warp == pw) {
      const int r = lane - l0;  // row within the block for lanes l0..l0+15
      const bool in = r >= 0 && r < 16;
      float g[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) g[c] = x[c];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float dj = __shfl_sync(0xffffffffu, g[0], l0 + j);
        const float inv = rsqrtf(dj);
        const float lrj = (r == j) ? dj * inv : g[0] * inv;  // L[r][j] for r >= j
        if (in && r >= j) Lk[r * 16 + j] = lrj;
        if (in && r == j) Rv[j] = inv;                        // 1 / L[j][j]
#pragma unroll
        for (int t = 1; t < 16; ++t) {
          const float lmj = __shfl_sync(0xffffffffu, lrj, (l0 + j + t) & 31);
          g[t - 1] = (in && j + t < 16 && r >= j + t) ? fmaf(-lrj, lmj, g[t]) : g[t];
        }
      }
      if (in) {
#pragma unroll
        for (int c = 1; c < 16; ++c)
          if (c > r) Lk[r * 16 + c] = 0.f;
      }
    }
    __syncthreads();
    if (hc == 0) {
      // ---- 3a. panel row ri: L[ri, kb] L_kk^T = X[ri, kb] by forward substitution,
      // into the K-major panel image (K columns 0..15)
      float pv[16];
      if (ri >= k0 + 16) {
#pragma unroll
        for (int c = 0; c < 16; ++c) pv[c] = 0.f;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float y = x[0] * Rv[c];
#pragma unroll
          for (int t = 0; t < 15; ++t) {
            const float l = (c + 1 + t < 16) ? Lk[(c + 1 + t) * 16 + c] : 0.f;
            x[t] = fmaf(-y, l, x[t + 1]);
          }
#pragma unroll
          for (int t = 0; t < 15; ++t) pv[t] = pv[t + 1];
          pv[15] = y;
        }
      } else if (ri >= k0) {
#pragma unroll
        for (int c = 0; c < 16; ++c) pv[c] = Lk[(ri - k0) * 16 + c];
      } else {
#pragma unroll
        for (int c = 0; c < 16; ++c) pv[c] = 0.f;
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint4 hi, lo;
        split8(pv + 8 * hh, hi, lo);
        const uint32_t o = img_off(ri, 8 * hh);
        *reinterpret_cast<uint4*>(limg + o) = hi;
        *reinterpret_cast<uint4*>(limg + kLPart + o) = lo;
      }
    } else {
      // ---- 3b. column j of W[kb, :]: L_kk W[kb, j] = R[kb, j] by forward substitution
      const int j = ri;  // column 0..127
      float z[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) z[r] = Tb[r * D + j];
      __nv_bfloat16* wh = reinterpret_cast<__nv_bfloat16*>(wimg);
      __nv_bfloat16* wl = reinterpret_cast<__nv_bfloat16*>(wimg + kImg);
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const float w = z[0] * Rv[r];
#pragma unroll
        for (int t = 0; t < 15; ++t) {
          const float l = (r + 1 + t < 16) ? Lk[(r + 1 + t) * 16 + r] : 0.f;
          z[t] = fmaf(-w, l, z[t + 1]);
        }
        const __nv_bfloat16 hb = __float2bfloat16_rn(w);
        const uint32_t o = img_off(k0 + r, j) >> 1;
        wh[o] = hb;
        wl[o] = __float2bfloat16_rn(w - __bfloat162float(hb));
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- 4. rank-16 updates on tcgen05: X -= Lp Lp^T, R -= Lp W[kb, :]
    if (kb + 1 < NB) {
      if (tid == 0 && !*abort_flag) {
        tc_fence_after();
        const uint64_t lh = smem_desc_sw128(lbase, 16, 1024), ll = smem_desc_sw128(lbase + kLPart, 16, 1024);
        const uint64_t wh = smem_desc_sw128(wbase + kb * 2048, D * 128, 1024);
        const uint64_t wl = smem_desc_sw128(wbase + kImg + kb * 2048, D * 128, 1024);
        mma3(tmem + kAccX, lh, ll, lh, ll, kIdKK | kNegA, 1u);
        mma3(tmem + kAccR, lh, ll, wh, wl, kIdKM | kNegA, 1u);
        mma_commit(bar);
      }
      ++commits;
      mbar_wait(bar, phase, abort_flag, a.status, a.wait_ns);
      phase ^= 1;
      tc_fence_after();
    }
  }

  // ---------------- P = W^T W into TMEM columns 0..127
  if (tid == 0 && !*abort_flag) {
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t dh = smem_desc_sw128(wbase + kk * 2048, D * 128, 1024);
      const uint64_t dl = smem_desc_sw128(wbase + kImg + kk * 2048, D * 128, 1024);
      mma3(tmem + kAccX, dh, dl, dh, dl, kIdMM, kk > 0 ? 1u : 0u);
    }
    mma_commit(bar);
  }
  ++commits;
  // B_t (row ri, columns hc*64..) -> TMEM columns 128.. as hi | lo bf16 pairs, while P runs.
  {
    const float4* src = reinterpret_cast<const float4*>(a.Bm + off);
    float4 v[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) v[t] = src[(hc * 16 + t) * D + ri];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint32_t ph[16], pl[16];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const float4 w = v[c * 8 + t];
        const float xs[4] = {w.x, w.y, w.z, w.w};
        float hv[4], lv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          hv[u] = __bfloat162float(__float2bfloat16_rn(xs[u]));
          lv[u] = xs[u] - hv[u];
        }
        ph[2 * t] = pack_bf16(hv[0], hv[1]);
        ph[2 * t + 1] = pack_bf16(hv[2], hv[3]);
        pl[2 * t] = pack_bf16(lv[0], lv[1]);
        pl[2 * t + 1] = pack_bf16(lv[2], lv[3]);
      }
      tmem_st16(tl + kTmemB + hc * 32 + c * 16, ph);
      tmem_st16(tl + kTmemB + 64 + hc * 32 + c * 16, pl);
    }
    tmem_st_wait();
  }
  bool ok = mbar_wait(bar, phase, abort_flag, a.status, a.wait_ns);
  phase ^= 1;
  tc_fence_after();

  // ---------------- M = Diag(alpha) P (fp32 + hi/lo images); P image over the W image
  if (ok) {
    const float al = slot > 0 ? a.alpha[(((long long)b * a.H + h) * a.T + slot) * D + ri] : 0.f;
    uint8_t* mimg = a.Msplit + off * 4;  // two D*D bf16 images per slot
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      const int j0 = hc * 64 + cc * 16;
      uint32_t v[16];
      tmem_ld16(tl + kAccX + j0, v);
      tmem_ld_wait();
      float pv[16], mv[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        pv[t] = __uint_as_float(v[t]);
        mv[t] = al * pv[t];
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint4 hi, lo;
        split8(pv + 8 * hh, hi, lo);
        const uint32_t o = img_off(ri, j0 + 8 * hh);
        *reinterpret_cast<uint4*>(wimg + o) = hi;
        *reinterpret_cast<uint4*>(wimg + kImg + o) = lo;
        if (slot > 0) {
          split8(mv + 8 * hh, hi, lo);
          *reinterpret_cast<uint4*>(mimg + o) = hi;
          *reinterpret_cast<uint4*>(mimg + kImg + o) = lo;
        }
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  // ---------------- C = B P (A operand B_t from TMEM, B operand the P image)
  if (tid == 0 && !*abort_flag) {
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t ph = smem_desc_sw128(wbase + kk * 2048, D * 128, 1024);
      const uint64_t pl = smem_desc_sw128(wbase + kImg + kk * 2048, D * 128, 1024);
      const uint32_t bh = tmem + kTmemB + kk * 8, bl = tmem + kTmemB + 64 + kk * 8;
      mma_f16_ts(tmem + kAccX, bh, ph, kIdKM, kk > 0 ? 1u : 0u);
      mma_f16_ts(tmem + kAccX, bh, pl, kIdKM, 1u);
      mma_f16_ts(tmem + kAccX, bl, ph, kIdKM, 1u);
    }
    mma_commit(bar);
  }
  ++commits;
  if (ok) ok = mbar_wait(bar, phase, abort_flag, a.status, a.wait_ns);
  phase ^= 1;
  tc_fence_after();
  if (ok) {
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      const int j0 = hc * 64 + cc * 16;
      uint32_t v[16];
      tmem_ld16(tl + kAccX + j0, v);
      tmem_ld_wait();
      float4* cd = reinterpret_cast<float4*>(a.C + off);
#pragma unroll
      for (int t = 0; t < 4; ++t)
        cd[(j0 / 4 + t) * D + ri] = make_float4(__uint_as_float(v[4 * t]), __uint_as_float(v[4 * t + 1]), __uint_as_float(v[4 * t + 2]),
                            __uint_as_float(v[4 * t + 3]));
    }
  }

  // ---------------- teardown: no MMA may still be running when TMEM is freed
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag && commits > 0) {
    // Completions arrive in order: waiting for the last committed phase covers all.
    mbar_wait(bar, phase ^ 1, nullptr, a.status, a.wait_ns);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

cudaError_t launch_solve_chol_tc(const Problem& p, cudaStream_t s) {
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(solve_chol_tc_kernel), kSmemBytes);
  if (e != cudaSuccess) return e;
  SolveArgs a{p.B, p.H, p.T, p.A, p.Bm, p.alpha, p.M, p.C, static_cast<uint8_t*>(p.Msplit), p.status,
              p.spin_limit};
  dim3 grid(p.T - 1, p.H, p.B);
  solve_chol_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(a);
  return cudaGetLastError();
}

}  // namespace vda
