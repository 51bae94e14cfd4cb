// Frame solve (Video DeltaNet summary, onedev.kr/papers/80, section "how to use":
// S_t (I + A_t) = Sbar_t + B_t, transition M_t = Diag(alpha_t)(I + A_t)^-1, with
// the inverse taken in the d_k x d_k key space; the injection is C_t = B_t (I + A_t)^-1).
//
// Per (b, h, slot), d = 128, one CTA of 256 threads, two CTAs per SM.
//
// The inverse P = (I + A)^-1 comes from the symmetric sweep (Gauss-Jordan
// elimination without pivoting, safe here because I + A is symmetric positive
// definite with every eigenvalue >= 1). Sweeping pivot k of a symmetric X:
//   x_ij -= x_ik x_kj / x_kk  (i, j != k),  x_ik /= x_kk,  x_kj /= x_kk,  x_kk = -1 / x_kk,
// and after all 128 pivots X = -P. Each thread keeps an 8 x 8 tile of X in
// registers and applies the rank-1 update of every step to it (64 FMAs); the
// pivot row (= column, by symmetry) and its reciprocal are published through
// a double-buffered shared-memory vector by the threads that own it, with one
// block barrier per step. The loop over pivots is unrolled by 8, so the
// pivot's row and column inside a tile are compile-time register indices.
//
// Then M = Diag(alpha) P (the bf16 hi/lo operand images the tensor-core scan
// loads as they are) and C = B P on tcgen05 with B_t split
// into hi/lo in TMEM as the A operand and P as a hi/lo shared-memory image
// (three-term split product, ~2^-16 relative, fp32 accumulation). The text
// slot produces only C = S_T.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace vda {

namespace {

constexpr int D = 128;
constexpr int kThreads = 256;
constexpr int kImg = D * D * 2;            // one bf16 operand image (two 64-column atoms of D rows)
constexpr int kPOff = 0;                   // P image (hi, lo)
constexpr int kPvOff = 2 * kImg;           // pivot vectors: 2 x (D values + reciprocal), 16-byte aligned
constexpr int kPvStride = D + 4;           // floats per pivot buffer
constexpr int kBarOff = kPvOff + 2 * kPvStride * 4 + 64;
// More shared memory than the kernel uses, so that at most two CTAs share an
// SM: each holds 256 of the SM's 512 TMEM columns.
constexpr int kSmemBytes = 80 * 1024;
static_assert(kBarOff + 64 + 1024 <= kSmemBytes, "shared memory layout");
static_assert(3 * kSmemBytes > 227 * 1024, "at most two CTAs per SM");
constexpr uint32_t kIdKM = sm100::idesc_bf16_f32(128, 128, false, true);  // A K-major, B MN-major
constexpr uint32_t kAccC = 0, kTmemB = 128;  // TMEM columns: C accumulator, B_t hi (+64: lo)

struct SolveArgs {
  int B, H, T;
  uint32_t* ready;  // [B,H,T-1] slot-ready words, or nullptr
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

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// 1 / d by the hardware's approximate reciprocal plus one Newton-Raphson step
// (r <- r + r (1 - d r)), which leaves about one ulp of error. Pivots of I + A
// are >= 1, so no special cases arise.
__device__ __forceinline__ float recip(float d) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(d));
  return fmaf(r, fmaf(-d, r, 1.f), r);
}

// Publish row `row` of this thread's tile (global row 8 ti + row) as the next
// pivot vector, and, from the tile on the diagonal, the pivot's reciprocal. The
// vector is stored in two halves: entries 8t..8t+3 of tile t at float4 t, entries
// 8t+4..8t+7 at float4 D/8 + t, so that a warp's float4 reads of the 16 tiles'
// entries fall on distinct banks (consecutive 16-byte words) rather than on every
// other group of four banks.
template <int row>
__device__ __forceinline__ void publish(float* pv, const float (&x)[8][8], int ti, int tj) {
  reinterpret_cast<float4*>(pv)[tj] = make_float4(x[row][0], x[row][1], x[row][2], x[row][3]);
  reinterpret_cast<float4*>(pv + D / 2)[tj] = make_float4(x[row][4], x[row][5], x[row][6], x[row][7]);
  if (ti == tj) pv[D] = recip(x[row][row]);
}

// One sweep step, pivot k = 8 K + s (s is a compile-time constant).
template <int s>
__device__ __forceinline__ void sweep_step(float (&x)[8][8], float* pv_all, int K, int ti, int tj) {
  const float* v = pv_all + (s & 1) * kPvStride;
  float* vn = pv_all + ((s + 1) & 1) * kPvStride;
  const float4 r0 = reinterpret_cast<const float4*>(v)[ti];
  const float4 r1 = reinterpret_cast<const float4*>(v + D / 2)[ti];
  const float4 c0 = reinterpret_cast<const float4*>(v)[tj];
  const float4 c1 = reinterpret_cast<const float4*>(v + D / 2)[tj];
  const float inv = v[D];
  const float vr[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
  const float vc[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  float ur[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) ur[r] = vr[r] * inv;  // x_ik / x_kk
  // The rank-1 update as packed fp32x2 FMAs (each lane rounds exactly as fmaf).
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const float2 nu = make_float2(-ur[r], -ur[r]);
#pragma unroll
    for (int c = 0; c < 8; c += 2) {
      const float2 xv = __ffma2_rn(nu, make_float2(vc[c], vc[c + 1]), make_float2(x[r][c], x[r][c + 1]));
      x[r][c] = xv.x;
      x[r][c + 1] = xv.y;
    }
  }
  if (tj == K) {  // column k
#pragma unroll
    for (int r = 0; r < 8; ++r) x[r][s] = ur[r];
  }
  if (ti == K) {  // row k
#pragma unroll
    for (int c = 0; c < 8; ++c) x[s][c] = vc[c] * inv;
    if (tj == K) x[s][s] = -inv;
  }
  // The next pivot, k + 1, is row s + 1 of tile row K, or row 0 of tile row K + 1.
  if (s < 7) {
    if (ti == K) publish<(s + 1) & 7>(vn, x, ti, tj);
  } else {
    if (ti == K + 1) publish<0>(vn, x, ti, tj);
  }
  __syncthreads();
}

// CTA order over the n = T-1 slots of all BH heads, in the order the scans need
// them: first every head's slot 0 (S_T, read by both directions at the start),
// then key k = 1, 2, ...: slots k (forward step k-1) and n-k (reverse step k-1)
// of every head, and for even n the middle slot n/2 last. CTAs start in about
// this order, so the last wave holds the frames both scans reach last and the
// scans, launched while that wave runs, advance on everything before them.
__device__ __forceinline__ void order_slot(int cta, int BH, int n, int& bh, int& slot) {
  if (cta < BH) {
    bh = cta;
    slot = 0;
    return;
  }
  const int l = cta - BH, npairs = (n - 1) / 2;
  if (l < npairs * 2 * BH) {
    const int k = 1 + l / (2 * BH), w = l % (2 * BH);
    bh = w >> 1;
    slot = (w & 1) ? n - k : k;
  } else {
    bh = l - npairs * 2 * BH;
    slot = n / 2;
  }
}

__global__ void __launch_bounds__(kThreads, 2) solve_tc_kernel(const SolveArgs a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = sm100::align_smem_1024(smem_raw);
  uint8_t* pimg = smem + kPOff;
  float* pv = reinterpret_cast<float*>(smem + kPvOff);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  // Let the scan kernel launch as soon as every solve CTA has started (it then
  // waits on the slot-ready words, not on the end of this grid).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  int bh, slot;
  order_slot(blockIdx.x, a.B * a.H, a.T - 1, bh, slot);
  const int b = bh / a.H, h = bh % a.H;
  const long long off = ((long long)bh * (a.T - 1) + slot) * (long long)D * D;
  // TMEM-side roles: matrix row ri == TMEM lane, column half hc.
  const int q = warp % 4, hc = warp / 4;
  const int ri = q * 32 + lane;
  // Sweep roles: the 8 x 8 tile (ti, tj) of X, rows 8 ti.., columns 8 tj..
  const int ti = tid / 16, tj = tid % 16;

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

  // ---------------- X = I + A into the register tiles; publish pivot 0
  float x[8][8];
  {
    const float4* src = reinterpret_cast<const float4*>(a.A + off);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int i = 8 * ti + r;
      const float4 w0 = src[(2 * tj) * D + i], w1 = src[(2 * tj + 1) * D + i];
      x[r][0] = w0.x; x[r][1] = w0.y; x[r][2] = w0.z; x[r][3] = w0.w;
      x[r][4] = w1.x; x[r][5] = w1.y; x[r][6] = w1.z; x[r][7] = w1.w;
    }
    if (ti == tj) {
#pragma unroll
      for (int r = 0; r < 8; ++r) x[r][r] += 1.f;
    }
    if (ti == 0) publish<0>(pv, x, ti, tj);
  }
  __syncthreads();

  // ---------------- the sweep: pivots k = 8 K + s
#pragma unroll 1
  for (int K = 0; K < D / 8; ++K) {
    // B_t is needed only after the sweep: fetch it into L2 in the middle of the
    // sweep, not while the slot's A is being loaded.
    if (K == 6 && tid == 0)
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.Bm + off), "r"((uint32_t)(D * D * 4)) : "memory");
    sweep_step<0>(x, pv, K, ti, tj);
    sweep_step<1>(x, pv, K, ti, tj);
    sweep_step<2>(x, pv, K, ti, tj);
    sweep_step<3>(x, pv, K, ti, tj);
    sweep_step<4>(x, pv, K, ti, tj);
    sweep_step<5>(x, pv, K, ti, tj);
    sweep_step<6>(x, pv, K, ti, tj);
    sweep_step<7>(x, pv, K, ti, tj);
  }

  // ---------------- P = -X: the P image for C = B P; M = Diag(alpha) P as the hi/lo images
  // the tensor-core scan reads (no fp32 copy: nothing on this path reads one)
  {
    float al[8];
    if (slot > 0) {
      const float4* ap = reinterpret_cast<const float4*>(a.alpha + (((long long)b * a.H + h) * a.T + slot) * D + 8 * ti);
      const float4 a0 = ap[0], a1 = ap[1];
      al[0] = a0.x; al[1] = a0.y; al[2] = a0.z; al[3] = a0.w;
      al[4] = a1.x; al[5] = a1.y; al[6] = a1.z; al[7] = a1.w;
    }
    uint8_t* mimg = a.Msplit + off * 4;  // two D*D bf16 images per slot
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int i = 8 * ti + r;
      float pr[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) pr[c] = -x[r][c];
      const uint32_t o = img_off(i, 8 * tj);
      uint4 hi, lo;
      split8(pr, hi, lo);
      *reinterpret_cast<uint4*>(pimg + o) = hi;
      *reinterpret_cast<uint4*>(pimg + kImg + o) = lo;
      if (slot > 0) {
        float mr[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) mr[c] = al[r] * pr[c];
        split8(mr, hi, lo);
        *reinterpret_cast<uint4*>(mimg + o) = hi;
        *reinterpret_cast<uint4*>(mimg + kImg + o) = lo;
      }
    }
  }
  // ---------------- B_t (row ri, columns hc*64..) -> TMEM as hi | lo bf16 pairs (from L2:
  // prefetched during the sweep, needed only by C = B P)
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

  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();

  // ---------------- C = B P (A operand B_t from TMEM, B operand the P image)
  if (tid == 0) {
    tc_fence_after();
    const uint32_t pb = smem_u32(pimg);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t ph = smem_desc_sw128(pb + kk * 2048, D * 128, 1024);
      const uint64_t pl = smem_desc_sw128(pb + kImg + kk * 2048, D * 128, 1024);
      const uint32_t bh = tmem + kTmemB + kk * 8, bl = tmem + kTmemB + 64 + kk * 8;
      mma_f16_ts(tmem + kAccC, bh, ph, kIdKM, kk > 0 ? 1u : 0u);
      mma_f16_ts(tmem + kAccC, bh, pl, kIdKM, 1u);
      mma_f16_ts(tmem + kAccC, bl, ph, kIdKM, 1u);
    }
    mma_commit(bar);
  }
  const bool ok = mbar_wait(bar, 0, abort_flag, a.status, a.wait_ns);
  tc_fence_after();
  if (ok) {
    float4* cd = reinterpret_cast<float4*>(a.C + off);
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      const int j0 = hc * 64 + cc * 16;
      uint32_t v[16];
      tmem_ld16(tl + kAccC + j0, v);
      tmem_ld_wait();
#pragma unroll
      for (int t = 0; t < 4; ++t)
        cd[(j0 / 4 + t) * D + ri] = make_float4(__uint_as_float(v[4 * t]), __uint_as_float(v[4 * t + 1]),
                                                __uint_as_float(v[4 * t + 2]), __uint_as_float(v[4 * t + 3]));
    }
  }

  // ---------------- teardown: the MMA must be complete before TMEM is freed
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag) mbar_wait(bar, 0, nullptr, a.status, a.wait_ns);
  // Every thread's C_t and M_t stores precede the barrier above: publish the slot.
  if (tid == 0 && ok && a.ready != nullptr) {
    __threadfence();
    flag_release_gpu(a.ready + (long long)bh * (a.T - 1) + slot, 1u);
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
  SolveArgs a{p.B, p.H, p.T, p.ready, p.A, p.Bm, p.alpha, p.M, p.C, static_cast<uint8_t*>(p.Msplit), p.status,
              p.spin_limit};
  const long long n = (long long)p.B * p.H * (p.T - 1);
  solve_tc_kernel<<<(unsigned)n, kThreads, kSmemBytes, s>>>(a);
  return cudaGetLastError();
}

}  // namespace vda
