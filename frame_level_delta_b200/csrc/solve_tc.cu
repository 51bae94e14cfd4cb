// Frame solve (Video DeltaNet summary, onedev.kr/papers/80, section "how to use":
// S_t (I + A_t) = Sbar_t + B_t, transition M_t = Diag(alpha_t)(I + A_t)^-1, with
// the inverse taken in the d_k x d_k key space; the injection is C_t = B_t (I + A_t)^-1).
//
// Per (b, h, slot), d = 128, one CTA of 256 threads:
//   1. X = I + A in shared memory (fp32), blocked right-looking Cholesky X = L L^T
//      (16-wide panels: one warp factors the diagonal block, one thread per row
//      solves the panel, 4x4 register tiles apply the rank-16 trailing update);
//   2. W = L^-1 in place (diagonal 16x16 blocks inverted by 8 warps in parallel,
//      then block rows top to bottom), all fp32 on CUDA cores;
//   3. P = W^T W on tcgen05 (W split into bf16 hi + lo; P = Wh'Wh + Wh'Wl + Wl'Wh,
//      fp32 accumulation in TMEM; error ~2^-16 relative);
//   4. M = Diag(alpha) P written as fp32 and as the bf16 hi/lo operand images the
//      tensor-core scan loads as they are; P kept as bf16 hi/lo operand in smem;
//   5. C = B P on tcgen05 with the same three-term split (B_t arrives by a bulk
//      copy issued at kernel start, overlapping steps 1-4).
// The text slot (slot 0) produces only C = S_T.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace vda {

namespace {

constexpr int D = 128;
constexpr int LDX = D + 4;  // padded fp32 row stride: rows stay 16-byte aligned
constexpr int NB = D / 16;
constexpr int kThreads = 256;
constexpr int kImgBytes = D * D * 2;  // one bf16 operand image (two 64-column atoms)
constexpr int kR1 = 0;                                  // X (fp32), later the P image
constexpr int kR2 = ((LDX * D * 4 + 1023) / 1024) * 1024;  // W image, later the B image
constexpr int kR3 = kR2 + 2 * kImgBytes;                // B_t (fp32) landing buffer
constexpr int kWd = kR3 + D * D * 4;                    // 8 diagonal inverses, 16x16 fp32
constexpr int kTb = kWd + NB * 256 * 4;                 // block-row temporary 16 x D fp32
constexpr int kBar = kTb + 16 * D * 4;
constexpr int kSmemBytes = kBar + 64 + 1024;
constexpr uint32_t kIdescP = sm100::idesc_bf16_f32(128, 128, true, true);   // A, B MN-major
constexpr uint32_t kIdescC = sm100::idesc_bf16_f32(128, 128, false, true);  // A K-major, B MN-major
static_assert(kR2 >= 2 * kImgBytes, "P image must fit in the X region");

struct SolveArgs {
  int B, H, T;
  const float* A;
  const float* Bm;
  const float* alpha;
  float* M;
  float* C;
  __nv_bfloat16* Msplit;
  uint32_t* status;
  unsigned long long wait_ns;
};

// Byte offset of element (row, col) in a bf16 operand image: 128-byte rows of 64
// elements, 16-byte chunks XOR-swizzled by (row % 8), 64-column atoms of `rows`
// rows stored one after the other (the 128-byte-swizzle canonical layout).
__device__ __forceinline__ uint32_t img_off(int row, int col, int rows) {
  const int atom = col >> 6, cc = col & 63;
  return (uint32_t)(atom * rows * 128 + row * 128 + ((((cc >> 3) ^ (row & 7))) << 4) + (cc & 7) * 2);
}

__device__ __forceinline__ void split8(const float* x, uint4& hi, uint4& lo) {
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&hi);
  __nv_bfloat162* l = reinterpret_cast<__nv_bfloat162*>(&lo);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __nv_bfloat162 hh = __floats2bfloat162_rn(x[2 * q], x[2 * q + 1]);
    const float2 hf = __bfloat1622float2(hh);
    h[q] = hh;
    l[q] = __floats2bfloat162_rn(x[2 * q] - hf.x, x[2 * q + 1] - hf.y);
  }
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          sm100::smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(sm100::smem_u32(bar))
      : "memory");
}

// Three-term split product D = Ah Bh + Ah Bl + Al Bh over K = 128.
// a_mn: A operand MN-major (advance 16 rows per K step) or K-major (32 bytes).
__device__ __forceinline__ void mma_split3(uint32_t dtm, uint32_t a_hi, uint32_t a_lo, bool a_mn, uint32_t b_hi,
                                           uint32_t b_lo, uint32_t idesc) {
  using namespace sm100;
  const uint32_t as[3] = {a_hi, a_hi, a_lo}, bs[3] = {b_hi, b_lo, b_hi};
#pragma unroll
  for (int t = 0; t < 3; ++t) {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t da = a_mn ? smem_desc_sw128(as[t] + kk * 2048, D * 128, 1024)
                               : smem_desc_sw128(as[t] + (kk / 4) * (D * 128) + (kk % 4) * 32, 16, 1024);
      const uint64_t db = smem_desc_sw128(bs[t] + kk * 2048, D * 128, 1024);
      mma_f16(dtm, da, db, idesc, (t == 0 && kk == 0) ? 0u : 1u);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) solve_tc_kernel(const SolveArgs a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* X = reinterpret_cast<float*>(smem + kR1);
  uint8_t* img1 = smem + kR1;  // P image (after X is consumed)
  uint8_t* img2 = smem + kR2;  // W image, then B image
  float* Bf = reinterpret_cast<float*>(smem + kR3);
  float* Wd = reinterpret_cast<float*>(smem + kWd);  // [NB][16][16]
  float* Tb = reinterpret_cast<float*>(smem + kTb);  // [16][D]
  uint64_t* bar_b = reinterpret_cast<uint64_t*>(smem + kBar);
  uint64_t* bar_p = bar_b + 1;
  uint64_t* bar_c = bar_b + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_b + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int slot = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const long long off = (((long long)b * a.H + h) * (a.T - 1) + slot) * (long long)D * D;

  if (tid == 0) {
    mbar_init(bar_b, 1);
    mbar_init(bar_p, 1);
    mbar_init(bar_c, 1);
    *abort_flag = 0;
    fence_mbar_init();
    mbar_arrive_expect_tx(bar_b, D * D * 4);
    bulk_load(Bf, a.Bm + off, D * D * 4, bar_b);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  // X = I + A
  {
    const float4* src = reinterpret_cast<const float4*>(a.A + off);
    for (int e = tid; e < D * D / 4; e += kThreads) {
      const int i = e / (D / 4), c4 = e % (D / 4);
      float4 v = src[e];
      const int j = c4 * 4;
      if (i == j) v.x += 1.f;
      if (i == j + 1) v.y += 1.f;
      if (i == j + 2) v.z += 1.f;
      if (i == j + 3) v.w += 1.f;
      *reinterpret_cast<float4*>(X + i * LDX + j) = v;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ---------------- 1. blocked Cholesky, lower, in place
  for (int kb = 0; kb < NB; ++kb) {
    const int k0 = kb * 16;
    if (warp == 0) {  // factor the 16x16 diagonal block in registers
      const int r = lane & 15;
      float x[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) x[c] = X[(k0 + r) * LDX + k0 + c];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float dj = __shfl_sync(0xffffffffu, x[j], j);
        const float ljj = sqrtf(dj);
        const float inv = 1.f / ljj;
        if (r == j) x[j] = ljj;
        else if (r > j) x[j] *= inv;
#pragma unroll
        for (int m = j + 1; m < 16; ++m) {
          const float lmj = __shfl_sync(0xffffffffu, x[j], m);
          if (r >= m) x[m] = fmaf(-x[j], lmj, x[m]);
        }
      }
      if (lane < 16) {
#pragma unroll
        for (int c = 0; c < 16; ++c)
          if (c <= r) X[(k0 + r) * LDX + k0 + c] = x[c];
      }
    }
    __syncthreads();
    const int n = D - k0 - 16;
    if (n == 0) break;
    if (tid < n) {  // panel: row i solves L_kk y = x (forward substitution)
      const int i = k0 + 16 + tid;
      float y[16];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        const float4 v = *reinterpret_cast<const float4*>(X + i * LDX + k0 + 4 * c4);
        y[4 * c4] = v.x; y[4 * c4 + 1] = v.y; y[4 * c4 + 2] = v.z; y[4 * c4 + 3] = v.w;
      }
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        float acc = y[c];
#pragma unroll
        for (int m = 0; m < c; ++m) acc = fmaf(-y[m], X[(k0 + c) * LDX + k0 + m], acc);
        y[c] = acc / X[(k0 + c) * LDX + k0 + c];
      }
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4)
        *reinterpret_cast<float4*>(X + i * LDX + k0 + 4 * c4) =
            make_float4(y[4 * c4], y[4 * c4 + 1], y[4 * c4 + 2], y[4 * c4 + 3]);
    }
    __syncthreads();
    {  // rank-16 trailing update of the lower triangle, 4x4 tiles
      const int nt = n / 4;
      const int ntiles = nt * (nt + 1) / 2;
      for (int t = tid; t < ntiles; t += kThreads) {
        int ti = (int)((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
        while ((ti + 1) * (ti + 2) / 2 <= t) ++ti;
        while (ti * (ti + 1) / 2 > t) --ti;
        const int tj = t - ti * (ti + 1) / 2;
        const int i0 = k0 + 16 + 4 * ti, j0 = k0 + 16 + 4 * tj;
        float acc[4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float4 v = *reinterpret_cast<const float4*>(X + (i0 + r) * LDX + j0);
          acc[r][0] = v.x; acc[r][1] = v.y; acc[r][2] = v.z; acc[r][3] = v.w;
        }
#pragma unroll
        for (int m4 = 0; m4 < 4; ++m4) {
          float4 li[4], lj[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            li[r] = *reinterpret_cast<const float4*>(X + (i0 + r) * LDX + k0 + 4 * m4);
            lj[r] = *reinterpret_cast<const float4*>(X + (j0 + r) * LDX + k0 + 4 * m4);
          }
#pragma unroll
          for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float s = acc[r][c];
              s = fmaf(-li[r].x, lj[c].x, s);
              s = fmaf(-li[r].y, lj[c].y, s);
              s = fmaf(-li[r].z, lj[c].z, s);
              s = fmaf(-li[r].w, lj[c].w, s);
              acc[r][c] = s;
            }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r)
          *reinterpret_cast<float4*>(X + (i0 + r) * LDX + j0) = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
      }
    }
    __syncthreads();
  }

  // ---------------- 2. W = L^-1 in place
  if (warp < NB) {  // diagonal blocks: lane c computes column c of (L_ww)^-1
    const int w0 = warp * 16, c = lane & 15;
    float wv[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float acc = (r == c) ? 1.f : 0.f;
#pragma unroll
      for (int m = 0; m < r; ++m) acc = fmaf(-X[(w0 + r) * LDX + w0 + m], wv[m], acc);
      wv[r] = acc / X[(w0 + r) * LDX + w0 + r];
    }
    if (lane < 16) {
#pragma unroll
      for (int r = 0; r < 16; ++r) Wd[warp * 256 + r * 16 + c] = wv[r];
    }
  }
  __syncthreads();
  {
    const int r = tid / 16, c = tid % 16;
    X[r * LDX + c] = Wd[r * 16 + c];
    for (int ib = 1; ib < NB; ++ib) {
      __syncthreads();
      const int row = ib * 16 + r;
      for (int jb = 0; jb < ib; ++jb) {  // T_jb = L[ib, jb..ib-1] W[jb..ib-1, jb]
        float acc = 0.f;
        for (int k = jb * 16; k < ib * 16; ++k) acc = fmaf(X[row * LDX + k], X[k * LDX + jb * 16 + c], acc);
        Tb[r * D + jb * 16 + c] = acc;
      }
      __syncthreads();
      for (int jb = 0; jb < ib; ++jb) {  // W_ib,jb = -W_ib,ib T_jb
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) acc = fmaf(Wd[ib * 256 + r * 16 + m], Tb[m * D + jb * 16 + c], acc);
        X[row * LDX + jb * 16 + c] = -acc;
      }
      X[row * LDX + ib * 16 + c] = Wd[ib * 256 + r * 16 + c];
    }
  }
  __syncthreads();

  // ---------------- 3. W image (rows k, columns i; zero above the diagonal), P = W^T W
  for (int e = tid; e < D * (D / 8); e += kThreads) {
    const int k = e / (D / 8), i0 = (e % (D / 8)) * 8;
    float x[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) x[q] = (i0 + q <= k) ? X[k * LDX + i0 + q] : 0.f;
    uint4 hi, lo;
    split8(x, hi, lo);
    const uint32_t o = img_off(k, i0, D);
    *reinterpret_cast<uint4*>(img2 + o) = hi;
    *reinterpret_cast<uint4*>(img2 + kImgBytes + o) = lo;
  }
  fence_proxy_async_smem();
  __syncthreads();
  if (tid == 0) {
    tc_fence_after();
    const uint32_t wh = smem_u32(img2), wl = wh + kImgBytes;
    mma_split3(tmem, wh, wl, true, wh, wl, kIdescP);
    mma_commit(bar_p);
  }
  bool ok = mbar_wait(bar_p, 0, abort_flag, a.status, a.wait_ns);
  tc_fence_after();

  // ---------------- 4. M = Diag(alpha) P (fp32 + hi/lo images), P image into smem
  const int q = warp % 4, half = warp / 4;
  const int i = q * 32 + lane;  // TMEM lane / matrix row of this thread
  if (ok) {
    const float al = slot > 0 ? a.alpha[(((long long)b * a.H + h) * a.T + slot) * D + i] : 0.f;
    uint8_t* mimg = reinterpret_cast<uint8_t*>(a.Msplit) + off * 4;  // 2 images of D*D bf16 per slot
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      const int j0 = half * 64 + cc * 16;
      uint32_t v[16];
      tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + j0, v);
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
        const uint32_t o = img_off(i, j0 + 8 * hh, D);
        *reinterpret_cast<uint4*>(img1 + o) = hi;
        *reinterpret_cast<uint4*>(img1 + kImgBytes + o) = lo;
        if (slot > 0) {
          split8(mv + 8 * hh, hi, lo);
          *reinterpret_cast<uint4*>(mimg + o) = hi;
          *reinterpret_cast<uint4*>(mimg + kImgBytes + o) = lo;
        }
      }
      if (slot > 0) {
        float4* md = reinterpret_cast<float4*>(a.M + off + (long long)i * D + j0);
#pragma unroll
        for (int t = 0; t < 4; ++t) md[t] = make_float4(mv[4 * t], mv[4 * t + 1], mv[4 * t + 2], mv[4 * t + 3]);
      }
    }
  }
  // ---------------- 5. C = B P: B (K-major image) from the landed fp32 copy
  if (ok) ok = mbar_wait(bar_b, 0, abort_flag, a.status, a.wait_ns);
  if (ok) {
    for (int e = tid; e < D * (D / 8); e += kThreads) {
      const int r = e / (D / 8), k0 = (e % (D / 8)) * 8;
      const float4 v0 = *reinterpret_cast<const float4*>(Bf + r * D + k0);
      const float4 v1 = *reinterpret_cast<const float4*>(Bf + r * D + k0 + 4);
      const float x[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      uint4 hi, lo;
      split8(x, hi, lo);
      const uint32_t o = img_off(r, k0, D);
      *reinterpret_cast<uint4*>(img2 + o) = hi;
      *reinterpret_cast<uint4*>(img2 + kImgBytes + o) = lo;
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && !*abort_flag) {
    tc_fence_after();
    const uint32_t bh = smem_u32(img2), bl = bh + kImgBytes;
    const uint32_t ph = smem_u32(img1), pl = ph + kImgBytes;
    mma_split3(tmem + 128, bh, bl, false, ph, pl, kIdescC);
    mma_commit(bar_c);
  }
  if (ok) ok = mbar_wait(bar_c, 0, abort_flag, a.status, a.wait_ns);
  tc_fence_after();
  if (ok) {
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      const int j0 = half * 64 + cc * 16;
      uint32_t v[16];
      tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + 128 + j0, v);
      tmem_ld_wait();
      float4* cd = reinterpret_cast<float4*>(a.C + off + (long long)i * D + j0);
#pragma unroll
      for (int t = 0; t < 4; ++t)
        cd[t] = make_float4(__uint_as_float(v[4 * t]), __uint_as_float(v[4 * t + 1]), __uint_as_float(v[4 * t + 2]),
                            __uint_as_float(v[4 * t + 3]));
    }
  }

  // ---------------- teardown
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag) {
    mbar_wait(bar_b, 0, nullptr, a.status, a.wait_ns);  // the bulk copy must have landed
    mbar_wait(bar_p, 0, nullptr, a.status, a.wait_ns);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

bool solve_tc_supported(const Problem& p) { return p.bf16 && p.D == 128; }

cudaError_t launch_solve_tc(const Problem& p, cudaStream_t s) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(solve_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  SolveArgs a{p.B, p.H, p.T, p.A, p.Bm, p.alpha, p.M, p.C, static_cast<__nv_bfloat16*>(p.Msplit), p.status,
              p.spin_limit};
  dim3 grid(p.T - 1, p.H, p.B);
  solve_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(a);
  return cudaGetLastError();
}

}  // namespace vda
