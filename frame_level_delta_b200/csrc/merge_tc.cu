// Hybrid merge of the two branches of the attention layer on tcgen05 tensor
// cores (Video DeltaNet summary, onedev.kr/papers/80, section "how it differs":
// the softmax and the linear readout each pass their own gate and output
// projection and are summed; VDN-H3 post, section "hybrid attention
// structure"):
//   Y = O~S W_S^T + O~L W_L^T      Y [M, N], O~ [M, K], W [N, K]  (bf16, fp32 accumulation)
// with the projections in the [out, in] layout of a linear layer. One GEMM whose
// contraction runs over both branches: the K loop takes the softmax operands,
// then the linear ones, into the same accumulator.
//
// Persistent CTAs walk 128 x 256 output tiles (N fastest, so the CTAs working at
// any moment share one 128-row block of the branch outputs through L2). TMA
// brings 64-wide K slices of A (128 rows) and B (256 rows) with 128-byte
// swizzle into a four-stage ring; one thread issues M128 N256 K16 MMAs into one
// of two 256-column TMEM accumulators, so the epilogue of a tile overlaps the
// MMAs of the next. Warp roles: 0 = TMA producer, 1 = TMEM owner + MMA issuer,
// 2..5 = epilogue (warp w reads TMEM lanes 32 (w % 4) ..).
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace vda {

namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kABytes = kBM * kBK * 2;   // 16 KB
constexpr int kBBytes = kBN * kBK * 2;   // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kBarOff = kStages * kStageBytes;
constexpr int kSmemBytes = kBarOff + 256 + 1024;
constexpr uint32_t kIdesc = sm100::idesc_bf16_f32(kBM, kBN, false, false);
static_assert(kSmemBytes <= 232448, "more shared memory than a CTA may use");

struct MergeArgs {
  int M, N, K1, K2;
  int mb, nb;   // tile counts along M and N
  __nv_bfloat16* Y;
  uint32_t* status;
  unsigned long long wait_ns;
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  return sm100::bf162_bits(__floats2bfloat162_rn(a, b));
}

__global__ void __launch_bounds__(kThreads, 1)
    merge_tc_kernel(const __grid_constant__ CUtensorMap mA1, const __grid_constant__ CUtensorMap mB1,
                    const __grid_constant__ CUtensorMap mA2, const __grid_constant__ CUtensorMap mB2,
                    const MergeArgs a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int ntiles = a.mb * a.nb;
  const int nk1 = (a.K1 + kBK - 1) / kBK, nk2 = (a.K2 + kBK - 1) / kBK, nk = nk1 + nk2;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&mA1);
    prefetch_tmap(&mB1);
    prefetch_tmap(&mA2);
    prefetch_tmap(&mB2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  int issued = 0;  // producer only

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const int m0 = (t / a.nb) * kBM, n0 = (t % a.nb) * kBN;
        for (int ks = 0; ks < nk; ++ks, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, abort_flag, a.status, a.wait_ns)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], kStageBytes);
          uint8_t* st = smem + s * kStageBytes;
          if (ks < nk1) {
            tma_load_2d(st, &mA1, &full[s], ks * kBK, m0);
            tma_load_2d(st + kABytes, &mB1, &full[s], ks * kBK, n0);
          } else {
            tma_load_2d(st, &mA2, &full[s], (ks - nk1) * kBK, m0);
            tma_load_2d(st + kABytes, &mB2, &full[s], (ks - nk1) * kBK, n0);
          }
          issued = it + 1;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int it = 0, tl = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++tl) {
        const int tb = tl & 1;
        if (!mbar_wait(&tempty[tb], ((tl >> 1) & 1) ^ 1, abort_flag, a.status, a.wait_ns)) break;
        tc_fence_after();
        const uint32_t acc = tmem + tb * kBN;
        for (int ks = 0; ks < nk; ++ks, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&full[s], (it / kStages) & 1, abort_flag, a.status, a.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t ab = smem_u32(smem + s * kStageBytes), bb = ab + kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t da = smem_desc_sw128(ab + kk * 32, 16, 1024);
            const uint64_t db = smem_desc_sw128(bb + kk * 32, 16, 1024);
            mma_f16(acc, da, db, kIdesc, (ks > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(&tfull[tb]);
      }
      mma_commit(drain);
    }
  } else {
    const int quad = warp % 4;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    int tl = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++tl) {
      const int tb = tl & 1;
      const bool got = mbar_wait(&tfull[tb], (tl >> 1) & 1, abort_flag, a.status, a.wait_ns);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int m = (t / a.nb) * kBM + r, n0 = (t % a.nb) * kBN;
      const bool live = m < a.M;
      __nv_bfloat16* yrow = a.Y + (long long)(live ? m : 0) * a.N;
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t v[32];
        const uint32_t ta = tmem + lane_off + tb * kBN + c * 32;
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
            "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
            "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
              "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
              "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
              "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
            : "r"(ta));
        tmem_ld_wait();
        const int n = n0 + c * 32;
        if (!live || n >= a.N) continue;
        const int groups = min(4, (a.N - n) / 8);  // N is a multiple of 8
        uint4* dst = reinterpret_cast<uint4*>(yrow + n);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 w;
          w.x = pack_bf16(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
          w.y = pack_bf16(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
          w.z = pack_bf16(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
          w.w = pack_bf16(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
          if (q < groups) dst[q] = w;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[tb]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      int last = -1;
      for (int i = s; i < issued; i += kStages) last = i;
      if (last >= 0) mbar_wait(&full[s], (last / kStages) & 1, nullptr, a.status, a.wait_ns);
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

cudaError_t launch_merge_tc(const void* A1, const void* B1, const void* A2, const void* B2, void* Y, int M, int N,
                            int K1, int K2, uint32_t* status, unsigned long long wait_ns, cudaStream_t s) {
  MergeArgs a{};
  a.M = M; a.N = N; a.K1 = K1; a.K2 = K2;
  a.mb = (M + kBM - 1) / kBM;
  a.nb = (N + kBN - 1) / kBN;
  a.Y = static_cast<__nv_bfloat16*>(Y);
  a.status = status;
  a.wait_ns = wait_ns;
  const long long tiles = (long long)a.mb * a.nb;
  if (tiles == 0) return cudaSuccess;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(merge_tc_kernel), kSmemBytes);
  if (e != cudaSuccess) return e;
  CUtensorMap mA1, mB1, mA2, mB2;
  const uint32_t boxA[2] = {kBK, kBM}, boxB[2] = {kBK, kBN};
  {
    const uint64_t dA[2] = {(uint64_t)K1, (uint64_t)M}, sA[1] = {(uint64_t)K1 * 2};
    const uint64_t dB[2] = {(uint64_t)K1, (uint64_t)N}, sB[1] = {(uint64_t)K1 * 2};
    if ((e = make_tmap_bf16(&mA1, A1, 2, dA, sA, boxA)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16(&mB1, B1, 2, dB, sB, boxB)) != cudaSuccess) return e;
  }
  {
    const uint64_t dA[2] = {(uint64_t)K2, (uint64_t)M}, sA[1] = {(uint64_t)K2 * 2};
    const uint64_t dB[2] = {(uint64_t)K2, (uint64_t)N}, sB[1] = {(uint64_t)K2 * 2};
    if ((e = make_tmap_bf16(&mA2, A2, 2, dA, sA, boxA)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16(&mB2, B2, 2, dB, sB, boxB)) != cudaSuccess) return e;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = (int)std::min<long long>(tiles, sms);
  merge_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(mA1, mB1, mA2, mB2, a);
  return cudaGetLastError();
}

}  // namespace vda
