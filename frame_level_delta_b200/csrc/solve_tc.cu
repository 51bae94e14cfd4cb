// Frame solve (Video DeltaNet summary, onedev.kr/papers/80, section "how to use":
// S_t (I + A_t) = Sbar_t + B_t, transition M_t = Diag(alpha_t)(I + A_t)^-1, with
// the inverse taken in the d_k x d_k key space; the injection is C_t = B_t (I + A_t)^-1).
//
// Per (b, h, slot), d = 128, one CTA of 160 threads, three CTAs per SM.
//
// The inverse P = (I + A)^-1 comes from the symmetric sweep (Gauss-Jordan
// elimination without pivoting, safe here because I + A is symmetric positive
// definite with every eigenvalue >= 1). Sweeping pivot k of a symmetric X:
//   x_ij -= x_ik x_kj / x_kk  (i, j != k),  x_ik /= x_kk,  x_kj /= x_kk,  x_kk = -1 / x_kk,
// keeps X symmetric, and after all 128 pivots X = -P. Only the upper triangle
// is kept: its 136 8 x 8 tiles (ti <= tj) live in the registers of threads
// 0..135, which apply every step's rank-1 update to them (64 FMAs, as packed
// fp32x2 FMAs). Pivot row k (= column k) is published through a double-buffered
// shared-memory vector: its entries left of the diagonal tile come from column
// k of the tiles above it, the rest from row k of the tiles right of it, and
// the reciprocal from the diagonal tile; one block barrier per step. Half the
// registers of a full-matrix sweep let three slots share an SM, whose steps
// (each bound by the barrier -> load -> update -> publish latency) then overlap.
//
// Then M = Diag(alpha) P (the bf16 hi/lo operand images the tensor-core scan
// loads as they are), and C = B P on tcgen05 in two halves of the contraction
// index: B_t (hi/lo, K-major) and 64 rows of P (hi/lo, N-major) as shared-memory
// images, three-term split product (~2^-16 relative), fp32 accumulation in 128
// TMEM columns. The text slot produces only C = S_T.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace vda {

namespace {

constexpr int D = 128;
constexpr int kThreads = 160;               // five warps
constexpr int kTiles = 136;                 // 8 x 8 tiles with ti <= tj
constexpr int kHalf = 64 * D * 2;           // one bf16 image of 64 x 128 values (16 KB)
constexpr int kPOff = 0;                    // P rows of one half: hi, lo (N-major, two 64-column atoms)
constexpr int kBOff = 2 * kHalf;            // B_t columns of one half: hi, lo (K-major, one atom)
constexpr int kPvOff = 4 * kHalf;           // pivot vectors: 2 x (D values + reciprocal)
constexpr int kPvStride = D + 4;            // floats per pivot buffer (16-byte aligned)
constexpr int kBarOff = kPvOff + 2 * kPvStride * 4;
constexpr int kSmemBytes = kBarOff + 64 + 1024;  // + room to align the base to 1024 bytes
static_assert(3 * (kSmemBytes + 1024) <= 228 * 1024, "three CTAs per SM");
// A grid of frame slots whose scan forms the injections (P form) needs neither
// the operand images nor TMEM: only the pivot vectors and the barrier block.
constexpr int kCompactPvOff = 0;
constexpr int kCompactBarOff = 2 * kPvStride * 4;
constexpr int kCompactSmemBytes = kCompactBarOff + 64 + 1024;
constexpr uint32_t kTmemCols = 128;         // the C accumulator; three CTAs use 384 of 512
constexpr uint32_t kIdKM = sm100::idesc_bf16_f32(128, 128, false, true);  // A K-major, B MN-major

struct SolveArgs {
  int B, H, T;
  uint32_t* ready;         // [B,H,T-1] slot-ready words to raise, or nullptr
  const uint32_t* gready;  // [B,H,T-1] statistics counts to wait for, or nullptr
  const float* A;
  const float* Bm;
  const float* alpha;
  float* M;
  float* C;
  uint8_t* Msplit;
  uint32_t* status;
  unsigned long long wait_ns;
  int pform;  // frames write P_t's images and no C_t (the scan forms the injection)
  int key0;     // key index of this grid's first CTA (0, or B*H for a grid of frame slots)
  int compact;  // shared memory holds only the pivot vectors and barriers (P-form frame slots)
};

// Byte offset of element (row, col) in a bf16 image with 128-byte rows of 64
// elements, 16-byte chunks XOR-swizzled by (row % 8), and 64-column atoms of
// `rows` rows one after the other (the 128-byte-swizzle canonical layout).
__device__ __forceinline__ uint32_t img_off(int rows, int row, int col) {
  const int atom = col >> 6, cc = col & 63;
  return (uint32_t)(atom * rows * 128 + row * 128 + ((((cc >> 3) ^ (row & 7))) << 4) + (cc & 7) * 2);
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

// 1 / d by the hardware's approximate reciprocal refined with one step of
// Newton's iteration for the reciprocal (the Newton-Raphson method applied to
// f(r) = 1/r - d: r <- r + r (1 - d r), which roughly squares the relative
// error of the starting value); about one ulp of error remains. Pivots of
// I + A are >= 1, so no special cases arise. vda_selftest_recip runs this same
// function so a test can bound its error against the correctly rounded 1/d.
__device__ __forceinline__ float recip(float d) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(d));
  return fmaf(r, fmaf(-d, r, 1.f), r);
}

// The pivot vector is stored in two halves: entries 8t..8t+3 of tile t at
// float4 t, entries 8t+4..8t+7 at float4 D/8 + t, so that a warp's float4 reads
// of different tiles' entries fall on consecutive 16-byte words.
__device__ __forceinline__ void put8(float* pv, int t, float a0, float a1, float a2, float a3, float a4, float a5,
                                     float a6, float a7) {
  reinterpret_cast<float4*>(pv)[t] = make_float4(a0, a1, a2, a3);
  reinterpret_cast<float4*>(pv + D / 2)[t] = make_float4(a4, a5, a6, a7);
}
// Row `row` of tile (ti, tj) as entries 8 tj.. of the pivot vector; the
// diagonal tile adds the pivot's reciprocal.
template <int row>
__device__ __forceinline__ void publish_row(float* pv, const float (&x)[8][8], int ti, int tj) {
  put8(pv, tj, x[row][0], x[row][1], x[row][2], x[row][3], x[row][4], x[row][5], x[row][6], x[row][7]);
  if (ti == tj) pv[D] = recip(x[row][row]);
}
// Column `col` of tile (ti, tj) above the diagonal as entries 8 ti.. (symmetry).
template <int col>
__device__ __forceinline__ void publish_col(float* pv, const float (&x)[8][8], int ti) {
  put8(pv, ti, x[0][col], x[1][col], x[2][col], x[3][col], x[4][col], x[5][col], x[6][col], x[7][col]);
}

// One sweep step, pivot k = 8 K + s (s is a compile-time constant).
template <int s>
__device__ __forceinline__ void sweep_step(float (&x)[8][8], float* pv_all, int K, int ti, int tj, bool active) {
  if (active) {
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
    if (tj == K) {  // column k (the tiles above and on the diagonal)
#pragma unroll
      for (int r = 0; r < 8; ++r) x[r][s] = ur[r];
    }
    if (ti == K) {  // row k (the tiles on and right of the diagonal)
#pragma unroll
      for (int c = 0; c < 8; ++c) x[s][c] = vc[c] * inv;
      if (tj == K) x[s][s] = -inv;
    }
    // The next pivot, k + 1, is row/column n of tile row/column Kn.
    constexpr int n = (s + 1) & 7;
    const int Kn = s < 7 ? K : K + 1;
    if (tj == Kn && ti < Kn) publish_col<n>(vn, x, ti);
    if (ti == Kn) publish_row<n>(vn, x, ti, tj);
  }
  __syncthreads();
}

// Tile t of the upper triangle, row-major: (0,0..15), (1,1..15), ...
__device__ __forceinline__ void tile_of(int t, int& ti, int& tj) {
  int r = 0, n = D / 8;
  while (t >= n) {
    t -= n;
    ++r;
    --n;
  }
  ti = r;
  tj = r + t;
}

__global__ void __launch_bounds__(kThreads, 3) solve_tc_kernel(const SolveArgs a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = sm100::align_smem_1024(smem_raw);
  uint8_t* pimg = smem + kPOff;
  uint8_t* bimg = smem + kBOff;
  float* pv = reinterpret_cast<float*>(smem + (a.compact ? kCompactPvOff : kPvOff));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + (a.compact ? kCompactBarOff : kBarOff));  // [2]: the two halves' MMAs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  // CTAs start in about key order, so the last wave holds the frames both
  // scans reach last, and the scans, launched while that wave runs, advance on
  // everything before them.
  int bh, slot;
  key_slot(a.key0 + blockIdx.x, a.B * a.H, a.T - 1, bh, slot);
  const long long off = ((long long)bh * (a.T - 1) + slot) * (long long)D * D;
  const bool active = tid < kTiles;
  // C = B P on tcgen05: for every slot, or only for the text slot (S_T) when
  // the frame scan forms the frames' injections itself.
  const bool mma = !a.pform || slot == 0;
  int ti = -1, tj = -1;
  if (active) tile_of(tid, ti, tj);

  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
    // Launched while the statistics kernel finishes: wait until its four
    // epilogue warps have stored this slot's A_t and B_t (the block barrier
    // below orders every thread's loads after this acquire).
    if (a.gready != nullptr)
      flag_wait_gpu(a.gready + (long long)bh * (a.T - 1) + slot, kGramReadyCount, abort_flag, a.status, a.wait_ns);
  }
  if (warp == 0) {
    if (mma) tmem_alloc(tmem_slot, kTmemCols);
    // Also when not allocating: until a CTA gives up its permit, no other CTA
    // of the grid is placed on the SM.
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = mma ? *tmem_slot : 0u;
  // Let the scan kernel launch once every solve CTA holds its TMEM (the scan
  // then waits on the slot-ready words, not on the end of this grid, and never
  // competes with a solve CTA for TMEM columns).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---------------- X = I + A (upper tiles) into registers; publish pivot 0
  float x[8][8];
  if (active) {
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
    if (ti == 0) publish_row<0>(pv, x, ti, tj);
  }
  __syncthreads();

  // ---------------- the sweep: pivots k = 8 K + s
#pragma unroll 1
  for (int K = 0; K < D / 8; ++K) {
    // B_t is needed only after the sweep: fetch it into L2 in the middle of the
    // sweep, not while the slot's A is being loaded.
    if (K == 6 && tid == 0)
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.Bm + off), "r"((uint32_t)(D * D * 4)) : "memory");
    sweep_step<0>(x, pv, K, ti, tj, active);
    sweep_step<1>(x, pv, K, ti, tj, active);
    sweep_step<2>(x, pv, K, ti, tj, active);
    sweep_step<3>(x, pv, K, ti, tj, active);
    sweep_step<4>(x, pv, K, ti, tj, active);
    sweep_step<5>(x, pv, K, ti, tj, active);
    sweep_step<6>(x, pv, K, ti, tj, active);
    sweep_step<7>(x, pv, K, ti, tj, active);
  }

  // ---------------- P = -X; M = Diag(alpha) P as the hi/lo images the scan reads
  // (the tile and, off the diagonal, its mirror; no fp32 copy: nothing on this
  // path reads one)
  if (active) {
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int c = 0; c < 8; ++c) x[r][c] = -x[r][c];
    if (slot > 0) {
      const float* al = a.alpha + ((long long)bh * a.T + slot) * D;
      float ar[8], ac[8];
      if (a.pform) {  // the images of P itself
#pragma unroll
        for (int r = 0; r < 8; ++r) ar[r] = ac[r] = 1.f;
      } else {
        const float4 p0 = reinterpret_cast<const float4*>(al + 8 * ti)[0];
        const float4 p1 = reinterpret_cast<const float4*>(al + 8 * ti)[1];
        const float4 q0 = reinterpret_cast<const float4*>(al + 8 * tj)[0];
        const float4 q1 = reinterpret_cast<const float4*>(al + 8 * tj)[1];
        ar[0] = p0.x; ar[1] = p0.y; ar[2] = p0.z; ar[3] = p0.w; ar[4] = p1.x; ar[5] = p1.y; ar[6] = p1.z; ar[7] = p1.w;
        ac[0] = q0.x; ac[1] = q0.y; ac[2] = q0.z; ac[3] = q0.w; ac[4] = q1.x; ac[5] = q1.y; ac[6] = q1.z; ac[7] = q1.w;
      }
      uint8_t* mimg = a.Msplit + off * 4;  // two D*D bf16 images per slot
      constexpr int kImg = D * D * 2;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        float mr[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) mr[c] = ar[r] * x[r][c];
        uint4 hi, lo;
        split8(mr, hi, lo);
        const uint32_t o = img_off(D, 8 * ti + r, 8 * tj);
        *reinterpret_cast<uint4*>(mimg + o) = hi;
        *reinterpret_cast<uint4*>(mimg + kImg + o) = lo;
      }
      if (ti != tj) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float mr[8];
#pragma unroll
          for (int r = 0; r < 8; ++r) mr[r] = ac[c] * x[r][c];
          uint4 hi, lo;
          split8(mr, hi, lo);
          const uint32_t o = img_off(D, 8 * tj + c, 8 * ti);
          *reinterpret_cast<uint4*>(mimg + o) = hi;
          *reinterpret_cast<uint4*>(mimg + kImg + o) = lo;
        }
      }
    }
  }

  // ---------------- C = B P in two halves of the contraction index k
  bool ok = true;
  if (mma) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (h == 1) {
      // The first half's MMAs must have read the images before they are rewritten.
      ok = mbar_wait(&bar[0], 0, abort_flag, a.status, a.wait_ns) && ok;
      tc_fence_after();
    }
    // Rows 64 h.. of P: this tile's rows if its tile row is in the half, its
    // mirrored rows if its tile column is.
    if (active) {
      if ((ti >> 3) == h) {
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          uint4 hi, lo;
          split8(x[r], hi, lo);
          const uint32_t o = img_off(64, 8 * ti + r - 64 * h, 8 * tj);
          *reinterpret_cast<uint4*>(pimg + o) = hi;
          *reinterpret_cast<uint4*>(pimg + kHalf + o) = lo;
        }
      }
      if (ti != tj && (tj >> 3) == h) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float pc[8];
#pragma unroll
          for (int r = 0; r < 8; ++r) pc[r] = x[r][c];
          uint4 hi, lo;
          split8(pc, hi, lo);
          const uint32_t o = img_off(64, 8 * tj + c - 64 * h, 8 * ti);
          *reinterpret_cast<uint4*>(pimg + o) = hi;
          *reinterpret_cast<uint4*>(pimg + kHalf + o) = lo;
        }
      }
    }
    // Columns 64 h.. of B_t (from L2: prefetched during the sweep) as K-major
    // hi/lo images: float4 f = (column quad 16 h + f / D, row f % D).
    {
      const float4* src = reinterpret_cast<const float4*>(a.Bm + off) + (long long)(16 * h) * D;
#pragma unroll 4
      for (int f = tid; f < 16 * D; f += kThreads) {
        const float4 w = src[f];
        const int i = f % D, kq = f / D;  // row, column quad within the half
        const float xs[4] = {w.x, w.y, w.z, w.w};
        float hv[4], lv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          hv[u] = __bfloat162float(__float2bfloat16_rn(xs[u]));
          lv[u] = xs[u] - hv[u];
        }
        const uint32_t o = img_off(D, i, 4 * kq);
        *reinterpret_cast<uint2*>(bimg + o) = make_uint2(pack_bf16(hv[0], hv[1]), pack_bf16(hv[2], hv[3]));
        *reinterpret_cast<uint2*>(bimg + kHalf + o) = make_uint2(pack_bf16(lv[0], lv[1]), pack_bf16(lv[2], lv[3]));
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t pb = smem_u32(pimg), bb = smem_u32(bimg);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ph = smem_desc_sw128(pb + kk * 2048, 64 * 128, 1024);
        const uint64_t pl = smem_desc_sw128(pb + kHalf + kk * 2048, 64 * 128, 1024);
        const uint64_t dbh = smem_desc_sw128(bb + kk * 32, 16, 1024);
        const uint64_t dbl = smem_desc_sw128(bb + kHalf + kk * 32, 16, 1024);
        mma_f16(tmem, dbh, ph, kIdKM, (h > 0 || kk > 0) ? 1u : 0u);
        mma_f16(tmem, dbh, pl, kIdKM, 1u);
        mma_f16(tmem, dbl, ph, kIdKM, 1u);
      }
      mma_commit(&bar[h]);
    }
  }
  }
  if (mma) ok = mbar_wait(&bar[1], 0, abort_flag, a.status, a.wait_ns) && ok;
  tc_fence_after();

  // ---------------- C out: warp q < 4 reads TMEM lanes (rows of C) 32 q..
  if (mma && ok && warp < 4) {
    const int i = warp * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    float4* cd = reinterpret_cast<float4*>(a.C + off);
#pragma unroll 1
    for (int j0 = 0; j0 < D; j0 += 16) {
      uint32_t v[16];
      tmem_ld16(tl + j0, v);
      tmem_ld_wait();
#pragma unroll
      for (int t = 0; t < 4; ++t)
        cd[(j0 / 4 + t) * D + i] = make_float4(__uint_as_float(v[4 * t]), __uint_as_float(v[4 * t + 1]),
                                               __uint_as_float(v[4 * t + 2]), __uint_as_float(v[4 * t + 3]));
    }
  }

  // ---------------- teardown: the MMAs must be complete before TMEM is freed
  tc_fence_before();
  __syncthreads();
  if (mma && tid == 0 && *abort_flag) {
    mbar_wait(&bar[0], 0, nullptr, a.status, a.wait_ns);
    mbar_wait(&bar[1], 0, nullptr, a.status, a.wait_ns);
  }
  // Every thread's C_t and M_t stores precede the barrier above: publish the slot.
  if (tid == 0 && ok && !*abort_flag && a.ready != nullptr) {
    __threadfence();
    flag_release_gpu(a.ready + (long long)bh * (a.T - 1) + slot, 1u);
  }
  __syncthreads();
  if (warp == 0 && mma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

__global__ void recip_selftest_kernel(const float* x, float* y, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = recip(x[i]);
}

}  // namespace

bool solve_tc_supported(const Problem& p) { return p.bf16 && p.D == 128; }

cudaError_t launch_recip_selftest(const float* x, float* y, int n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  recip_selftest_kernel<<<(n + 255) / 256, 256, 0, s>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_solve_tc(const Problem& p, cudaStream_t s, int part) {
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(solve_tc_kernel), kSmemBytes);
  if (e != cudaSuccess) return e;
  const long long BH = (long long)p.B * p.H;
  // In the P form the solve runs as two grids: the text slots (S_T = B P on
  // tcgen05, operand images in shared memory), then the frame slots in compact
  // CTAs (about 2 KB of shared memory, no TMEM) that fit beside the statistics
  // kernel's CTAs on the same SM and start as soon as their slot's statistics
  // are stored. Otherwise one grid takes every slot.
  const bool split = p.pform != 0;
  const int key0 = (split && part == 1) ? (int)BH : 0;
  const int compact = (split && part == 1) ? 1 : 0;
  const long long n = split ? (part == 0 ? BH : BH * (p.T - 2)) : BH * (p.T - 1);
  if (n == 0) return cudaSuccess;
  SolveArgs a{p.B, p.H, p.T, p.ready, p.gready, p.A, p.Bm, p.alpha, p.M, p.C, static_cast<uint8_t*>(p.Msplit),
              p.status, p.spin_limit, p.pform, key0, compact};
  // After the tensor-core statistics kernel (or the text grid), launch as its
  // programmatic dependent: CTAs start on the SMs its CTAs leave room on.
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)n);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = compact ? kCompactSmemBytes : kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.gready != nullptr ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, solve_tc_kernel, a);
}

}  // namespace vda
