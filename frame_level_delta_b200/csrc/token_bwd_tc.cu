// Per-token part of the frame-step backward on tcgen05 tensor cores. After the
// per-frame adjoints Gx = dS P and Gsym = GA + GA^T (GA = -S_t^T Gx) are in the
// workspace (row-major fp32, written by solve_bwd_simt_kernel), every token u of
// frame t gets
//   dk_u = beta_u (Gsym k_u + Gx^T v_u),  dv_u = beta_u Gx k_u,
//   dbeta_u = (k_u . (Gsym k_u + Gx^T v_u) + v_u . Gx k_u) / 2
// (the chain rule of S_t = (S_{t-1} Diag(alpha_t) + B_t)(I + A_t)^-1 through
// A_t = K_t^T Diag(beta_t) K_t and B_t = V_t^T Diag(beta_t) K_t; Video DeltaNet
// summary, onedev.kr/papers/80, section "how to use"). As products over a tile
// of 128 tokens (M = 128, K = d):
//   acc1 = K Gsym + V Gx    (the B operands are Gsym's rows and Gx's columns)
//   acc2 = K Gx^T           (Gx's rows)
// dK = beta acc1, dV = beta acc2, dbeta = (k . acc1 + v . acc2) / 2.
// One CTA per (b, h, frame): the prologue writes the three d x d operand images
// (bf16, K-major, 128-byte swizzle) once; K and V tiles stream through two TMA
// stages with the tile's beta; TMEM holds acc1 and acc2, double-buffered.
// Warp roles: 0 = TMA producer, 1 = TMEM owner + MMA issuer, 2..9 = prologue and
// epilogue (two warps per TMEM lane quadrant, one per half of the columns).
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace vda {

namespace {

constexpr int D = 128;
constexpr int kTileM = 128;
constexpr int kThreads = 320;
constexpr int kEpi = 256;
constexpr int kStages = 2;
constexpr int kAtom = kTileM * 128;      // one 64-channel box of a 128-token tile (16 KB)
constexpr int kTileBytes = 2 * kAtom;    // one bf16 tile of 128 tokens (32 KB)
constexpr int kImg = D * D * 2;          // one bf16 d x d image (32 KB, two 64-column atoms)
constexpr int kImgAtom = D * 128;
constexpr int kGsOff = 0, kGxTOff = kImg, kGxOff = 2 * kImg;
constexpr int kStageOff = 3 * kImg;      // stage s: K tile, then V tile
constexpr int kBetaOff = kStageOff + kStages * 2 * kTileBytes;
constexpr int kXchgOff = kBetaOff + kStages * kTileM * 4;  // [128] the second half's partial dbeta
constexpr int kBarOff = kXchgOff + kTileM * 4;
constexpr int kSmemBytes = kBarOff + 256 + 1024;
constexpr uint32_t kIdesc = sm100::idesc_bf16_f32(128, D, false, false);
static_assert(kSmemBytes <= 232448, "more shared memory than a CTA may use");

struct TbArgs {
  int B, H, T, U, Ht;
  const float* beta;   // [B, H, T, U]
  const float* Gx;     // workspace slot layout [B, H, T-1, D, D] row-major
  const float* Gsym;
  __nv_bfloat16* dK;   // [B, T*U, Ht, D] from this problem's first head
  __nv_bfloat16* dV;
  float* dbeta;        // [B, H, T, U]
  uint32_t* status;
  unsigned long long wait_ns;
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  return sm100::bf162_bits(__floats2bfloat162_rn(a, b));
}

__global__ void __launch_bounds__(kThreads, 1)
    token_bwd_tc_kernel(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
                        const TbArgs a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint8_t* sGs = smem + kGsOff;
  uint8_t* sGxT = smem + kGxTOff;
  uint8_t* sGx = smem + kGxOff;
  float* sbeta = reinterpret_cast<float*>(smem + kBetaOff);  // [kStages][128]
  float* sxch = reinterpret_cast<float*>(smem + kXchgOff);   // [128]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* iready = tempty + 2;
  uint64_t* drain = iready + 1;
  uint64_t* epibar = drain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epibar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // Frame t = 1 .. T-2 of (b, h): blockIdx.x = (b * H + h) * (T - 2) + (t - 1).
  const int t = 1 + blockIdx.x % (a.T - 2), bh = blockIdx.x / (a.T - 2);
  const int b = bh / a.H, h = bh % a.H;
  const int ntiles = (a.U + kTileM - 1) / kTileM;
  const long long tok_frame = (long long)b * a.T * a.U + (long long)t * a.U;  // flat index of the frame's token 0

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1 + 32);  // TMA bytes + the 32 lanes' beta copies
      mbar_init(&empty[s], 1 + 8);  // MMA commit + the 8 epilogue warps (they read k, v rows)
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 8);
    }
    mbar_init(iready, 8);
    mbar_init(drain, 1);
    mbar_init(epibar, kEpi);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&mK);
    prefetch_tmap(&mV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  int issued = 0;

  if (warp == 0) {
    const float* beta = a.beta + (((long long)b * a.H + h) * a.T + t) * a.U;
    for (int n = 0; n < ntiles; ++n) {
      const int s = n % kStages;
      int good = 1;
      if (lane == 0) good = mbar_wait(&empty[s], ((n / kStages) & 1) ^ 1, abort_flag, a.status, a.wait_ns) ? 1 : 0;
      good = __shfl_sync(0xffffffffu, good, 0);
      if (!good) break;
      const int u0 = n * kTileM;
      uint8_t* st = smem + kStageOff + s * 2 * kTileBytes;
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], 2 * kTileBytes);
#pragma unroll
        for (int at = 0; at < 2; ++at) {
          tma_load_3d(st + at * kAtom, &mK, &full[s], at * 64, h, (int)(tok_frame + u0));
          tma_load_3d(st + kTileBytes + at * kAtom, &mV, &full[s], at * 64, h, (int)(tok_frame + u0));
        }
      }
#pragma unroll
      for (int j = 0; j < kTileM / 32; ++j) {
        const int row = j * 32 + lane;
        const bool in = u0 + row < a.U;
        cp_async_4(sbeta + s * kTileM + row, in ? beta + u0 + row : beta, in ? 4u : 0u);
      }
      cp_async_mbar_arrive_noinc(&full[s]);
      if (lane == 0) issued = n + 1;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(iready, 0, abort_flag, a.status, a.wait_ns);
      const uint32_t gs = smem_u32(sGs), gxt = smem_u32(sGxT), gx = smem_u32(sGx);
      for (int n = 0; n < ntiles && ok; ++n) {
        const int s = n % kStages, tb = n & 1;
        if (!mbar_wait(&full[s], (n / kStages) & 1, abort_flag, a.status, a.wait_ns)) break;
        if (!mbar_wait(&tempty[tb], ((n >> 1) & 1) ^ 1, abort_flag, a.status, a.wait_ns)) break;
        tc_fence_after();
        const uint32_t kb = smem_u32(smem + kStageOff + s * 2 * kTileBytes), vb = kb + kTileBytes;
        const uint32_t acc1 = tmem + tb * 2 * D, acc2 = acc1 + D;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t o = (kk / 4) * kAtom + (kk % 4) * 32;      // token tiles: 128-row atoms
          const uint32_t oi = (kk / 4) * kImgAtom + (kk % 4) * 32;  // images: 128-row atoms
          const uint64_t dk = smem_desc_sw128(kb + o, 16, 1024), dv = smem_desc_sw128(vb + o, 16, 1024);
          mma_f16(acc1, dk, smem_desc_sw128(gs + oi, 16, 1024), kIdesc, kk > 0 ? 1u : 0u);
          mma_f16(acc1, dv, smem_desc_sw128(gxt + oi, 16, 1024), kIdesc, 1u);
          mma_f16(acc2, dk, smem_desc_sw128(gx + oi, 16, 1024), kIdesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(&empty[s]);
        mma_commit(&tfull[tb]);
      }
      mma_commit(drain);
    }
  } else {
    const int et = threadIdx.x - 64;  // 0..255
    const int quad = warp % 4, hf = (warp - 2) / 4;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    uint32_t ephase = 0;
    auto epi_sync = [&]() -> bool {
      mbar_arrive(epibar);
      const bool ok = mbar_wait(epibar, ephase, abort_flag, a.status, a.wait_ns);
      ephase ^= 1;
      return ok;
    };
    // ---- prologue: the three operand images (bf16, K-major: row n, columns k)
    const long long off = (((long long)b * a.H + h) * (a.T - 1) + t) * (long long)D * D;
    const float* Gs = a.Gsym + off;
    const float* Gx = a.Gx + off;
    for (int e = et; e < D * (D / 8); e += kEpi) {
      const int c8 = e / D, n = e % D;  // row n, columns 8 c8 .. 8 c8 + 7
      const int boff = (c8 / 8) * kImgAtom + n * 128 + (((c8 % 8) ^ (n & 7)) << 4);
      const float4 g0 = *reinterpret_cast<const float4*>(Gs + n * D + 8 * c8);
      const float4 g1 = *reinterpret_cast<const float4*>(Gs + n * D + 8 * c8 + 4);
      *reinterpret_cast<uint4*>(sGs + boff) =
          make_uint4(pack_bf16(g0.x, g0.y), pack_bf16(g0.z, g0.w), pack_bf16(g1.x, g1.y), pack_bf16(g1.z, g1.w));
      const float4 x0 = *reinterpret_cast<const float4*>(Gx + n * D + 8 * c8);
      const float4 x1 = *reinterpret_cast<const float4*>(Gx + n * D + 8 * c8 + 4);
      *reinterpret_cast<uint4*>(sGx + boff) =
          make_uint4(pack_bf16(x0.x, x0.y), pack_bf16(x0.z, x0.w), pack_bf16(x1.x, x1.y), pack_bf16(x1.z, x1.w));
      float c[8];  // column n of Gx, rows 8 c8 .. 8 c8 + 7
#pragma unroll
      for (int q = 0; q < 8; ++q) c[q] = Gx[(8 * c8 + q) * D + n];
      *reinterpret_cast<uint4*>(sGxT + boff) =
          make_uint4(pack_bf16(c[0], c[1]), pack_bf16(c[2], c[3]), pack_bf16(c[4], c[5]), pack_bf16(c[6], c[7]));
    }
    fence_proxy_async_smem();
    bool ok = epi_sync();
    if (ok && lane == 0) mbar_arrive(iready);
    // ---- epilogue per tile
    for (int n = 0; n < ntiles && ok; ++n) {
      const int s = n % kStages, tb = n & 1;
      const bool got = mbar_wait(&tfull[tb], (n >> 1) & 1, abort_flag, a.status, a.wait_ns) &&
                       mbar_wait(&full[s], (n / kStages) & 1, abort_flag, a.status, a.wait_ns);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int u = n * kTileM + r;
      const bool live = u < a.U;
      const float bt = sbeta[s * kTileM + r];
      // This thread's half rows of k and v (64 channels: the tile's atom hf).
      const uint8_t* krow = smem + kStageOff + s * 2 * kTileBytes + hf * kAtom + r * 128;
      const uint8_t* vrow = krow + kTileBytes;
      const long long row = (tok_frame + (live ? u : 0)) * a.Ht + h;
      uint4* dkdst = reinterpret_cast<uint4*>(a.dK + row * D) + hf * 8;
      uint4* dvdst = reinterpret_cast<uint4*>(a.dV + row * D) + hf * 8;
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // 16 columns per step: chunks 2c, 2c + 1 of the half row
        uint32_t v1[16], v2[16];
        tmem_ld16(tmem + lane_off + tb * 2 * D + hf * 64 + c * 16, v1);
        tmem_ld16(tmem + lane_off + tb * 2 * D + D + hf * 64 + c * 16, v2);
        tmem_ld_wait();
        uint32_t wk[8], wv[8];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int ch = 2 * c + h2;
          const uint4 kq = *reinterpret_cast<const uint4*>(krow + ((ch ^ (r & 7)) << 4));
          const uint4 vq = *reinterpret_cast<const uint4*>(vrow + ((ch ^ (r & 7)) << 4));
          const uint32_t kw[4] = {kq.x, kq.y, kq.z, kq.w}, vw[4] = {vq.x, vq.y, vq.z, vq.w};
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const float2 kf = __bfloat1622float2(bits_bf162(kw[p]));
            const float2 vf = __bfloat1622float2(bits_bf162(vw[p]));
            const float a0 = __uint_as_float(v1[h2 * 8 + 2 * p]), a1 = __uint_as_float(v1[h2 * 8 + 2 * p + 1]);
            const float b0 = __uint_as_float(v2[h2 * 8 + 2 * p]), b1 = __uint_as_float(v2[h2 * 8 + 2 * p + 1]);
            dot = fmaf(kf.x, a0, fmaf(kf.y, a1, fmaf(vf.x, b0, fmaf(vf.y, b1, dot))));
            wk[h2 * 4 + p] = pack_bf16(bt * a0, bt * a1);
            wv[h2 * 4 + p] = pack_bf16(bt * b0, bt * b1);
          }
        }
        if (live) {
          dkdst[2 * c] = make_uint4(wk[0], wk[1], wk[2], wk[3]);
          dkdst[2 * c + 1] = make_uint4(wk[4], wk[5], wk[6], wk[7]);
          dvdst[2 * c] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          dvdst[2 * c + 1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&tempty[tb]);
        mbar_arrive(&empty[s]);
      }
      // dbeta: the two halves of the row add their dot products.
      if (hf == 1) sxch[r] = dot;
      if (!epi_sync()) break;
      if (hf == 0 && live) a.dbeta[(((long long)b * a.H + h) * a.T + t) * a.U + u] = 0.5f * (dot + sxch[r]);
      if (!epi_sync()) break;  // the exchange slots may be rewritten by the next tile
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      int last = -1;
      for (int n = s; n < issued; n += kStages) last = n;
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

bool token_bwd_tc_supported(const Problem& p) {
  return p.bf16 && p.D == D && (long long)p.B * p.T * p.U < (1LL << 31);
}

cudaError_t launch_token_bwd_tc(const Problem& p, const void* K, const void* V, float* dbeta, void* dK, void* dV,
                                cudaStream_t s) {
  if (p.T < 3) return cudaSuccess;
  TbArgs a{p.B, p.H, p.T, p.U, p.Ht, p.beta, p.M, p.C, static_cast<__nv_bfloat16*>(dK),
           static_cast<__nv_bfloat16*>(dV), dbeta, p.status, p.spin_limit};
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(token_bwd_tc_kernel), kSmemBytes);
  if (e != cudaSuccess) return e;
  const uint64_t dims[3] = {(uint64_t)D, (uint64_t)p.H, (uint64_t)p.B * p.T * p.U};
  const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)p.Ht * D * 2};
  const uint32_t box[3] = {64u, 1u, (uint32_t)kTileM};
  CUtensorMap mK, mV;
  if ((e = make_tmap_bf16(&mK, K, 3, dims, strides, box)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&mV, V, 3, dims, strides, box)) != cudaSuccess) return e;
  const long long grid = (long long)p.B * p.H * (p.T - 2);
  token_bwd_tc_kernel<<<(unsigned)grid, kThreads, kSmemBytes, s>>>(mK, mV, a);
  return cudaGetLastError();
}

}  // namespace vda
