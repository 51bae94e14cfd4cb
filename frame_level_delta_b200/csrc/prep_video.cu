// Feature prep of the video keys and values (Video DeltaNet summary,
// onedev.kr/papers/80, section "how it differs": a depthwise 5x5 spatial and a
// 5-tap temporal convolution, then SiLU, on K and V; keys are L2-normalised).
//
// Per channel c of head h, with zero padding outside the latent grid and the clip:
//   y_t(i, j) = SiLU( sum_s wt[s] sum_{a,q} ws[a][q] x_{t+s-2}(i+a-2, j+q-2) )
// (cross-correlations; the spatial and temporal sums commute), then for K
// y <- y / sqrt(|y|^2 + eps) over the token's d channels.
//
// One CTA per (grid row i, block of kCW consecutive grid columns, b, h, K|V)
// walks the frames t = 0..T. A producer warp brings each frame's 5-row x
// (kCW + 4)-column neighbourhood of the block (all d channels of head h) into
// shared memory with one 4-D TMA load (zero fill outside the grid), two frames
// in flight, three CTAs per SM at d = 128. Each compute thread owns four
// consecutive tokens and four channels: it forms the four 5x5 spatial sums of
// the frame (each staged value it loads serves up to four taps, each weight
// load four tokens) and keeps the last five frames' sums in registers; the
// centred temporal sum of frame t - 2 follows, then SiLU, the key norm (a
// shuffle reduction over the token's d / 4 lanes) and the store of frames
// 1..T-2 in the prepared layout [B, H, T, U, d]. The kernel is bound by
// instruction issue and shared-memory bandwidth: four tokens per thread halve
// the shared-memory wavefronts per output and cut the instructions per output
// by about a third against two tokens per thread.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace vda {

namespace {

constexpr int kCW = 16;      // grid columns (tokens) per CTA
constexpr int kTileCols = kCW + 4;

template <typename TIn, int D>
struct PrepCfg {
  // Tokens per compute thread: four; two at d = 16, so that the compute
  // threads still fill a whole warp (the shuffles and __syncwarp take all lanes).
  static constexpr int kTPT = D >= 32 ? 4 : 2;
  static constexpr int kCompute = (kCW / kTPT) * (D / 4);  // compute threads
  static constexpr int kThreads = kCompute + 32;           // + producer warp
  static constexpr int kLanesPerGroup = D / 4;              // threads sharing a token group
  static constexpr int kStages = 2;                          // frames in flight per CTA
  static constexpr int kStageBytes = (5 * kTileCols * D * (int)sizeof(TIn) + 1023) / 1024 * 1024;
  static constexpr int kWOff = kStages * kStageBytes;       // spatial weights [25][D] fp32
  static constexpr int kWtOff = kWOff + 25 * D * 4;         // temporal weights [5][D] fp32
  static constexpr int kBarOff = kWtOff + 5 * D * 4;
  static constexpr int kSmemBytes = kBarOff + 128 + 1024;
  static constexpr int kMinBlocks = 3;                       // CTAs per SM (d = 128, bf16: 3 x 66 KB)
  static_assert(kSmemBytes <= 232448, "shared memory");
  static_assert(kCompute % 32 == 0, "compute threads fill whole warps");
};

template <typename TIn>
struct PrepIO;
template <>
struct PrepIO<__nv_bfloat16> {
  static __device__ __forceinline__ float4 load4(const uint8_t* p) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u), __uint_as_float(v.y << 16),
                       __uint_as_float(v.y & 0xffff0000u));
  }
  static __device__ __forceinline__ void store4(__nv_bfloat16* dst, float4 v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = sm100::bf162_bits(a);
    u.y = sm100::bf162_bits(b);
    *reinterpret_cast<uint2*>(dst) = u;
  }
};
template <>
struct PrepIO<float> {
  static __device__ __forceinline__ float4 load4(const uint8_t* p) { return *reinterpret_cast<const float4*>(p); }
  static __device__ __forceinline__ void store4(float* dst, float4 v) { *reinterpret_cast<float4*>(dst) = v; }
};

// SiLU. fp32 storage: x / (1 + e^-x) with the fast division intrinsic (a few
// ulp). bf16 storage: x sigmoid(x) = h + h tanh(h) with h = x / 2 and the
// hardware's approximate tanh (about 2^-11 error), one special-function
// operation instead of two, under the bf16 rounding of the output.
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
template <typename TIn>
__device__ __forceinline__ float silu(float x) {
  if constexpr (sizeof(TIn) == 2) {
    const float h = 0.5f * x;
    return fmaf(h, tanh_approx(h), h);
  } else {
    return __fdividef(x, 1.f + __expf(-x));
  }
}

template <typename TIn, int D>
__global__ void __launch_bounds__(PrepCfg<TIn, D>::kThreads, PrepCfg<TIn, D>::kMinBlocks)
    prep_video_kernel(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
                      const Problem p, const float* __restrict__ w) {
  using C = PrepCfg<TIn, D>;
  constexpr int kStages = C::kStages;
  constexpr int kTPT = C::kTPT;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  float* sw = reinterpret_cast<float*>(smem + C::kWOff);
  float* swt = reinterpret_cast<float*>(smem + C::kWtOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kStages);

  const int H = p.H, T = p.T, U = p.U, gw = p.gw;
  const int y = blockIdx.y, x0 = blockIdx.x * kCW;
  const int z = blockIdx.z, which = z & 1, bh = z >> 1, b = bh / H, h = bh % H;
  const CUtensorMap* map = which == 0 ? &mK : &mV;
  const int tid = threadIdx.x, lane = tid % 32;
  constexpr int kComputeWarps = C::kCompute / 32 > 0 ? C::kCompute / 32 : 1;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kComputeWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // Spatial and temporal weights of this (head, K|V) into shared memory as [tap][channel].
  const long long hd = (long long)H * D;
  const float* wsp = w + (which == 0 ? 0 : hd * 30) + (long long)h * D * 25;
  const float* wtp = w + (which == 0 ? hd * 25 : hd * 55) + (long long)h * D * 5;
  for (int e = tid; e < 25 * D; e += C::kThreads) {
    const int c = e / 25, tap = e % 25;
    sw[tap * D + c] = wsp[e];
  }
  for (int e = tid; e < 5 * D; e += C::kThreads) {
    const int c = e / 5, tap = e % 5;
    swt[tap * D + c] = wtp[e];
  }
  __syncthreads();

  if (tid >= C::kCompute) {
    // ---------------- producer warp: frame t into stage t % kStages
    if (tid == C::kCompute) {
      prefetch_tmap(map);
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int s = t % kStages;
        if (t >= kStages && !mbar_wait(&empty[s], ((t / kStages) - 1) & 1, abort_flag, p.status, p.spin_limit)) break;
        mbar_arrive_expect_tx(&full[s], 5 * kTileCols * D * (int)sizeof(TIn));
        tma_load_4d(smem + s * C::kStageBytes, map, &full[s], h * D, x0 - 2, y - 2, b * T + t);
        issued = t + 1;
      }
      // On abort, let the loads still in flight land before the CTA retires.
      if (*abort_flag)
        for (int t = (issued > kStages ? issued - kStages : 0); t < issued; ++t)
          mbar_wait(&full[t % kStages], (t / kStages) & 1, nullptr, p.status, p.spin_limit);
    }
    return;
  }

  // ---------------- compute threads: tokens x0 + kTPT xg .. + kTPT - 1, channels 4 g .. 4 g + 3
  const int xg = tid / C::kLanesPerGroup, g = tid % C::kLanesPerGroup;
  const int ch = 4 * g;
  float ring[5][kTPT][4];  // spatial sums of frames t-4 .. t (zero outside the clip)
#pragma unroll
  for (int s = 0; s < 5; ++s)
#pragma unroll
    for (int k = 0; k < kTPT; ++k)
#pragma unroll
      for (int c = 0; c < 4; ++c) ring[s][k][c] = 0.f;
  TIn* out = static_cast<TIn*>(which == 0 ? p.Kp : p.Vp);
  bool ok = true;

  for (int t = 0; t <= T; ++t) {
    float acc[kTPT][4];
#pragma unroll
    for (int k = 0; k < kTPT; ++k)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[k][c] = 0.f;
    if (t < T && ok) {
      const int s = t % kStages;
      ok = mbar_wait(&full[s], (t / kStages) & 1, abort_flag, p.status, p.spin_limit);
      if (ok) {
        const uint8_t* tile = smem + s * C::kStageBytes;
#pragma unroll
        for (int a = 0; a < 5; ++a) {
          float4 d[kTPT + 4];
#pragma unroll
          for (int c = 0; c < kTPT + 4; ++c)
            d[c] = PrepIO<TIn>::load4(tile + ((size_t)(a * kTileCols + kTPT * xg + c) * D + ch) * sizeof(TIn));
#pragma unroll
          for (int q = 0; q < 5; ++q) {
            const float4 wv = *reinterpret_cast<const float4*>(sw + (a * 5 + q) * D + ch);
#pragma unroll
            for (int k = 0; k < kTPT; ++k) {  // packed fp32x2 FMAs, each lane as fmaf
              const float2 lo = __ffma2_rn(make_float2(wv.x, wv.y), make_float2(d[k + q].x, d[k + q].y),
                                           make_float2(acc[k][0], acc[k][1]));
              const float2 hi = __ffma2_rn(make_float2(wv.z, wv.w), make_float2(d[k + q].z, d[k + q].w),
                                           make_float2(acc[k][2], acc[k][3]));
              acc[k][0] = lo.x; acc[k][1] = lo.y; acc[k][2] = hi.x; acc[k][3] = hi.y;
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);  // this warp is done with stage s
    }
#pragma unroll
    for (int s = 0; s < 4; ++s)
#pragma unroll
      for (int k = 0; k < kTPT; ++k)
#pragma unroll
        for (int c = 0; c < 4; ++c) ring[s][k][c] = ring[s + 1][k][c];
#pragma unroll
    for (int k = 0; k < kTPT; ++k)
#pragma unroll
      for (int c = 0; c < 4; ++c) ring[4][k][c] = acc[k][c];
    // Frame t - 2 now has all five temporal taps (frames t-4 .. t).
    const int to = t - 2;
    if (to >= 1 && to <= T - 2) {
      float ft[5][4];
#pragma unroll
      for (int s = 0; s < 5; ++s) {
        const float4 f = *reinterpret_cast<const float4*>(swt + s * D + ch);
        ft[s][0] = f.x; ft[s][1] = f.y; ft[s][2] = f.z; ft[s][3] = f.w;
      }
      float o[kTPT][4];
#pragma unroll
      for (int k = 0; k < kTPT; ++k) {
#pragma unroll
        for (int cp = 0; cp < 2; ++cp) {  // channel pairs: packed fp32x2 FMAs, each lane as fmaf
          float2 v = make_float2(0.f, 0.f);
#pragma unroll
          for (int s = 0; s < 5; ++s)
            v = __ffma2_rn(make_float2(ft[s][2 * cp], ft[s][2 * cp + 1]),
                           make_float2(ring[s][k][2 * cp], ring[s][k][2 * cp + 1]), v);
          o[k][2 * cp] = silu<TIn>(v.x);
          o[k][2 * cp + 1] = silu<TIn>(v.y);
        }
      }
      // Key norm: each token's sum of squares over the lanes of its channel group.
      float sc[kTPT];
#pragma unroll
      for (int k = 0; k < kTPT; ++k) sc[k] = 1.f;
      if (which == 0) {
        float ss[kTPT];
#pragma unroll
        for (int k = 0; k < kTPT; ++k)
          ss[k] = o[k][0] * o[k][0] + o[k][1] * o[k][1] + o[k][2] * o[k][2] + o[k][3] * o[k][3];
        if constexpr (C::kLanesPerGroup == 32 && kTPT == 4) {
          // The four tokens' sums at once over the whole warp (ten shuffles, not
          // twenty): after the halving steps lane l holds token (l >> 3) & 3's.
          const bool b4 = lane & 16, b3 = lane & 8;
          float a2[2];
#pragma unroll
          for (int i = 0; i < 2; ++i)
            a2[i] = (b4 ? ss[i + 2] : ss[i]) + __shfl_xor_sync(0xffffffffu, b4 ? ss[i] : ss[i + 2], 16);
          float e = (b3 ? a2[1] : a2[0]) + __shfl_xor_sync(0xffffffffu, b3 ? a2[0] : a2[1], 8);
#pragma unroll
          for (int off = 4; off; off >>= 1) e += __shfl_xor_sync(0xffffffffu, e, off);
          const float mine = rsqrtf(e + p.l2_eps);
#pragma unroll
          for (int k = 0; k < kTPT; ++k) sc[k] = __shfl_sync(0xffffffffu, mine, k << 3);
        } else {
#pragma unroll
          for (int k = 0; k < kTPT; ++k) {
            float v = ss[k];
#pragma unroll
            for (int off = C::kLanesPerGroup / 2; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
            sc[k] = rsqrtf(v + p.l2_eps);
          }
        }
      }
#pragma unroll
      for (int k = 0; k < kTPT; ++k) {
        const int x = x0 + kTPT * xg + k;
        if (x < gw) {
          const long long ot = (((long long)b * H + h) * T + to) * U + (long long)y * gw + x;
          PrepIO<TIn>::store4(out + ot * D + ch,
                              make_float4(o[k][0] * sc[k], o[k][1] * sc[k], o[k][2] * sc[k], o[k][3] * sc[k]));
        }
      }
    }
  }
}

template <typename TIn, int D>
cudaError_t launch_typed(const Problem& p, const void* K, const void* V, const float* w, cudaStream_t s) {
  using C = PrepCfg<TIn, D>;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(prep_video_kernel<TIn, D>), C::kSmemBytes);
  if (e != cudaSuccess) return e;
  // [B * T frames][gh rows][gw columns][H * D channels], channels innermost; a
  // grid column's row holds Ht * D channels, of which this problem's H * D
  // start at K and V.
  const uint64_t esz = sizeof(TIn);
  const uint64_t dims[4] = {(uint64_t)p.H * D, (uint64_t)p.gw, (uint64_t)p.gh, (uint64_t)p.B * p.T};
  const uint64_t row = (uint64_t)p.Ht * D * esz;
  const uint64_t strides[3] = {row, row * dims[1], row * dims[1] * dims[2]};
  const uint32_t box[4] = {(uint32_t)D, (uint32_t)kTileCols, 5u, 1u};
  const CUtensorMapDataType dt = sizeof(TIn) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  CUtensorMap mK, mV;
  e = make_tmap_typed(&mK, dt, K, 4, dims, strides, box);
  if (e != cudaSuccess) return e;
  e = make_tmap_typed(&mV, dt, V, 4, dims, strides, box);
  if (e != cudaSuccess) return e;
  dim3 grid((p.gw + kCW - 1) / kCW, p.gh, p.B * p.H * 2);
  prep_video_kernel<TIn, D><<<grid, C::kThreads, C::kSmemBytes, s>>>(mK, mV, p, w);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prep_video(const Problem& p, const void* K, const void* V, const float* conv_w, cudaStream_t s) {
  if ((long long)p.B * p.H * 2 > 65535 || p.gh > 65535) return cudaErrorInvalidConfiguration;
  if (p.bf16) {
    switch (p.D) {
      case 16: return launch_typed<__nv_bfloat16, 16>(p, K, V, conv_w, s);
      case 32: return launch_typed<__nv_bfloat16, 32>(p, K, V, conv_w, s);
      case 64: return launch_typed<__nv_bfloat16, 64>(p, K, V, conv_w, s);
      case 128: return launch_typed<__nv_bfloat16, 128>(p, K, V, conv_w, s);
    }
  } else {
    switch (p.D) {
      case 16: return launch_typed<float, 16>(p, K, V, conv_w, s);
      case 32: return launch_typed<float, 32>(p, K, V, conv_w, s);
      case 64: return launch_typed<float, 64>(p, K, V, conv_w, s);
      case 128: return launch_typed<float, 128>(p, K, V, conv_w, s);
    }
  }
  return cudaErrorNotSupported;
}

}  // namespace vda
