// Frame statistics from FP8 keys and values on tcgen05 tensor cores
// (kind::f8f6f4): the statistics of gram_tc.cu,
//   A = K^T Diag(beta) K,   B = V^T Diag(beta) K
// (Video DeltaNet summary, onedev.kr/papers/80, section "how to use"), for keys
// and values stored as e4m3 with one float32 scale per (token, head) shared by
// the token's key and value: k = s k8, v = s v8. One byte per channel is
// streamed instead of two (the pages run their large products in FP8 / MXFP8:
// section "assumptions and limits"; VDN-H3 post, "compared with existing
// methods").
//
// With R_u = beta_u s_u^2 k8_u:  A = K8^T R,  B = V8^T R  (sums over tokens u).
// R leaves the CUDA cores as two e4m3 parts under a power-of-two scale per
// (b, h, slot), 2^E R = hi + lo (about 2^-8 relative), chosen by a pre-pass so
// that 2^E beta_u s_u^2 448 <= 240 for every token of the slot; the epilogue
// multiplies by 2^-E. Both operands are MN-major (channels contiguous), as in
// the bf16 kernel: a 64-token stage holds one 128-byte-wide box of K8 and one
// of V8; per 32 tokens four M128 N128 K32 MMAs (K8 hi, K8 lo into A; V8 hi,
// V8 lo into B). Warp roles as in gram_tc.cu: 0 = TMA producer (+ beta and
// scale copies), 1 = MMA issuer, 2..5 = write-operand warps, 6..9 = epilogue.
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <algorithm>

#include "internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace vda {

namespace {

constexpr int D = 128;
constexpr int kTileU = 64;                 // tokens per stage
constexpr int kBox = kTileU * D;           // one e4m3 box: 64 tokens x 128 channels (8 KB)
constexpr int kStages = 8;
constexpr int kStageBytes = 2 * kBox;      // K8 and V8
constexpr int kRSlots = 2;
constexpr int kRBytes = 2 * kBox;          // R hi and R lo
constexpr int kThreads = 320;
constexpr int kTmemCols = 256;             // A (128) and B (128) per unit
constexpr int kBetaOff = kStages * kStageBytes + kRSlots * kRBytes;
constexpr int kBarOff = kBetaOff + 2 * kStages * kTileU * 4;  // beta and scale per stage token
constexpr int kSmemBytes = kBarOff + 512 + 1024;
// kind::f8f6f4: D f32, A and B e4m3, both MN-major, M = 128, N = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 15) | (1u << 16) | ((uint32_t)(128 >> 3) << 17) |
                            ((uint32_t)(128 >> 4) << 24);
static_assert(kSmemBytes <= 232448, "more shared memory than a CTA may use");

struct Gram8Args {
  int B, H, T, U, L, Ht;
  const float* beta;
  const float* beta_txt;
  const float* kv_scale;   // [B, T*U, Ht] from this problem's first head
  const float* kvt_scale;  // [B, L, Ht]
  const int* unit_exp;     // [B, H, T-1] exponent E per slot (the pre-pass)
  float* A;
  float* Bm;
  uint32_t* status;
  uint32_t* gready;
  unsigned long long wait_ns;
};

struct Unit {
  int b, h, slot, n;
};
__device__ __forceinline__ Unit unit_of(const Gram8Args& a, int u) {
  Unit x;
  int bh;
  key_slot(u, a.B * a.H, a.T - 1, bh, x.slot);
  x.b = bh / a.H;
  x.h = bh % a.H;
  x.n = x.slot == 0 ? a.L : a.U;
  return x;
}

__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(kIdesc), "r"(accumulate)
      : "memory");
}


// Pre-pass: E per (b, h, slot) with 2^E max_u(beta_u s_u^2) 448 <= 240, so every
// entry of 2^E R fits e4m3 (|k8| <= 448). One warp per slot.
__global__ void fp8_unit_exp_kernel(Gram8Args a, int* exps) {
  const int w = (blockIdx.x * blockDim.x + threadIdx.x) / 32, lane = threadIdx.x % 32;
  const int nslots = a.B * a.H * (a.T - 1);
  if (w >= nslots) return;
  const int slot = w % (a.T - 1), bh = w / (a.T - 1), b = bh / a.H, h = bh % a.H;
  float m = 0.f;
  if (slot == 0) {
    for (int u = lane; u < a.L; u += 32) {
      const float s = a.kvt_scale[((long long)b * a.L + u) * a.Ht + h];
      m = fmaxf(m, a.beta_txt[(long long)bh * a.L + u] * s * s);
    }
  } else {
    for (int u = lane; u < a.U; u += 32) {
      const float s = a.kv_scale[(((long long)b * a.T + slot) * a.U + u) * a.Ht + h];
      m = fmaxf(m, a.beta[((long long)bh * a.T + slot) * a.U + u] * s * s);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) exps[w] = m > 0.f ? max(-100, min(100, (int)floorf(log2f(240.f / (m * 448.f))))) : 0;
}

__global__ void __launch_bounds__(kThreads, 1)
    gram_fp8_tc_kernel(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
                       const __grid_constant__ CUtensorMap mKt, const __grid_constant__ CUtensorMap mVt,
                       const Gram8Args a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint8_t* rring = smem + kStages * kStageBytes;
  float* sbeta = reinterpret_cast<float*>(smem + kBetaOff);    // [kStages][64]
  float* sscale = sbeta + kStages * kTileU;                     // [kStages][64]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* empty = full + kStages;
  uint64_t* rf = empty + kStages;
  uint64_t* re = rf + kRSlots;
  uint64_t* tfull = re + kRSlots;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* issued_slot = reinterpret_cast<int*>(tmem_slot + 2);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nunits = a.B * a.H * (a.T - 1);
  const int G = gridDim.x;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1 + 32);  // TMA bytes + the 32 lanes' beta and scale copies
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < kRSlots; ++i) {
      mbar_init(&rf[i], 4);
      mbar_init(&re[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *issued_slot = 0;
    fence_mbar_init();
    prefetch_tmap(&mK);
    prefetch_tmap(&mV);
    prefetch_tmap(&mKt);
    prefetch_tmap(&mVt);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < nunits && ok; u += G) {
      const Unit x = unit_of(a, u);
      const CUtensorMap* mk = x.slot == 0 ? &mKt : &mK;
      const CUtensorMap* mv = x.slot == 0 ? &mVt : &mV;
      const float* beta = x.slot == 0 ? a.beta_txt + ((long long)x.b * a.H + x.h) * a.L
                                      : a.beta + (((long long)x.b * a.H + x.h) * a.T + x.slot) * (long long)a.U;
      // scale of token uu of this slot: base[uu * Ht]
      const float* scl = x.slot == 0 ? a.kvt_scale + (long long)x.b * a.L * a.Ht + x.h
                                     : a.kv_scale + (((long long)x.b * a.T + x.slot) * a.U) * a.Ht + x.h;
      const int ntiles = (x.n + kTileU - 1) / kTileU;
      for (int tt = 0; tt < ntiles; ++tt, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        int good = 1;
        if (lane == 0) good = mbar_wait(&empty[s], ph ^ 1, abort_flag, a.status, a.wait_ns) ? 1 : 0;
        good = __shfl_sync(0xffffffffu, good, 0);
        if (!good) { ok = false; break; }
        const int u0 = tt * kTileU;
        if (lane == 0) {
          uint8_t* st = smem + s * kStageBytes;
          mbar_arrive_expect_tx(&full[s], 2 * kBox);
          tma_load_5d(st, mk, &full[s], 0, x.h, u0, x.slot, x.b);
          tma_load_5d(st + kBox, mv, &full[s], 0, x.h, u0, x.slot, x.b);
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int uu = u0 + half * 32 + lane;
          const bool in = uu < x.n;
          cp_async_4(sbeta + s * kTileU + half * 32 + lane, in ? beta + uu : beta, in ? 4u : 0u);
          cp_async_4(sscale + s * kTileU + half * 32 + lane, in ? scl + (long long)uu * a.Ht : scl, in ? 4u : 0u);
        }
        cp_async_mbar_arrive_noinc(&full[s]);
      }
    }
    if (lane == 0) *issued_slot = it;
  } else if (warp == 1) {
    if (lane == 0) {
      int it = 0, k = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < nunits && ok; u += G, ++k) {
        const Unit x = unit_of(a, u);
        const int ntiles = (x.n + kTileU - 1) / kTileU;
        const int ub = k & 1;
        const uint32_t tacc = tmem + ub * kTmemCols;
        if (!mbar_wait(&tempty[ub], ((k >> 1) & 1) ^ 1, abort_flag, a.status, a.wait_ns)) break;
        tc_fence_after();
        for (int tt = 0; tt < ntiles; ++tt, ++it) {
          const int s = it % kStages, rs = it % kRSlots;
          if (!mbar_wait(&full[s], (it / kStages) & 1, abort_flag, a.status, a.wait_ns) ||
              !mbar_wait(&rf[rs], (it / kRSlots) & 1, abort_flag, a.status, a.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kb = smem_u32(smem + s * kStageBytes), vb = kb + kBox;
          const uint32_t hb = smem_u32(rring + rs * kRBytes), lb = hb + kBox;
#pragma unroll
          for (int ks = 0; ks < kTileU / 32; ++ks) {
            const uint32_t o = ks * 32 * 128;  // 32 token rows of 128 bytes
            const uint32_t acc = (tt > 0 || ks > 0) ? 1u : 0u;
            const uint64_t dk = smem_desc_sw128(kb + o, kBox, 1024), dv = smem_desc_sw128(vb + o, kBox, 1024);
            const uint64_t dh = smem_desc_sw128(hb + o, kBox, 1024), dl = smem_desc_sw128(lb + o, kBox, 1024);
            mma_f8(tacc, dk, dh, acc);
            mma_f8(tacc, dk, dl, 1u);
            mma_f8(tacc + 128, dv, dh, acc);
            mma_f8(tacc + 128, dv, dl, 1u);
          }
          mma_commit(&empty[s]);
          mma_commit(&re[rs]);
        }
        if (ok) mma_commit(&tfull[ub]);
      }
      mma_commit(drain);
    }
  } else if (warp < 6) {
    // ---------------- write operand R = 2^E beta s^2 k8 as e4m3 hi + lo (warps 2..5)
    // Thread: token row `row` of the stage, channel chunks c0 .. c0 + 3 (16 bytes each).
    const int tid = threadIdx.x - 64;  // 0..127
    const int row = tid / 2, c0 = (tid % 2) * 4;
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < nunits && ok; u += G) {
      const Unit x = unit_of(a, u);
      const float pe = ldexpf(1.f, a.unit_exp[((long long)x.b * a.H + x.h) * (a.T - 1) + x.slot]);
      const int ntiles = (x.n + kTileU - 1) / kTileU;
      for (int tt = 0; tt < ntiles; ++tt, ++it) {
        const int s = it % kStages, rs = it % kRSlots;
        if (!mbar_wait(&re[rs], ((it / kRSlots) & 1) ^ 1, abort_flag, a.status, a.wait_ns) ||
            !mbar_wait(&full[s], (it / kStages) & 1, abort_flag, a.status, a.wait_ns)) {
          ok = false;
          break;
        }
        const float sc = sbeta[s * kTileU + row] * sscale[s * kTileU + row] * sscale[s * kTileU + row] * pe;
        // The product and the split run on f16 pairs: c k8 <= 240 fits f16, whose
        // 2^-11 rounding is well below the 2^-8 of the two-part e4m3 form.
        const __half2 c2 = __float2half2_rn(sc);
        const uint8_t* src = smem + s * kStageBytes + row * 128;
        uint8_t* dh = rring + rs * kRBytes + row * 128;
        uint8_t* dl = dh + kBox;
#pragma unroll
        for (int c = c0; c < c0 + 4; ++c) {
          const int pc = c ^ (row & 7);
          const uint4 v = *reinterpret_cast<const uint4*>(src + pc * 16);
          const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
          // Pairs unpacked and packed by shifts (no type-punned accesses).
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint16_t e = (uint16_t)(vw[q >> 1] >> ((q & 1) * 16));
            const __half2 r = __hmul2(__half2(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)e, __NV_E4M3)), c2);
            const uint16_t hh = (uint16_t)__nv_cvt_halfraw2_to_fp8x2(__half2_raw(r), __NV_SATFINITE, __NV_E4M3);
            const __half2 hb = __half2(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)hh, __NV_E4M3));
            const uint16_t ll =
                (uint16_t)__nv_cvt_halfraw2_to_fp8x2(__half2_raw(__hsub2(r, hb)), __NV_SATFINITE, __NV_E4M3);
            if (q & 1) {
              hw[q >> 1] |= (uint32_t)hh << 16;
              lw[q >> 1] |= (uint32_t)ll << 16;
            } else {
              hw[q >> 1] = hh;
              lw[q >> 1] = ll;
            }
          }
          *reinterpret_cast<uint4*>(dh + pc * 16) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(dl + pc * 16) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&rf[rs]);
      }
    }
  } else {
    // ---------------- epilogue (warps 6..9): 2^-E * TMEM -> A, B in column quads
    const int q = warp % 4;
    const int r = q * 32 + lane;
    int k = 0;
    for (int u = blockIdx.x; u < nunits; u += G, ++k) {
      const Unit x = unit_of(a, u);
      const int ub = k & 1;
      if (!mbar_wait(&tfull[ub], (k >> 1) & 1, abort_flag, a.status, a.wait_ns)) break;
      tc_fence_after();
      const float ie = ldexpf(1.f, -a.unit_exp[((long long)x.b * a.H + x.h) * (a.T - 1) + x.slot]);
      const uint32_t taddr = tmem + ub * kTmemCols + ((uint32_t)(q * 32) << 16);
      const long long off = (((long long)x.b * a.H + x.h) * (a.T - 1) + x.slot) * (long long)D * D;
#pragma unroll 2
      for (int c = 0; c < 16; ++c) {
        uint32_t v[16];
        tmem_ld16(taddr + c * 16, v);
        tmem_ld_wait();
        float4* dst = reinterpret_cast<float4*>((c < 8 ? a.A : a.Bm) + off);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          dst[((c % 8) * 4 + j) * D + r] =
              make_float4(__uint_as_float(v[4 * j]) * ie, __uint_as_float(v[4 * j + 1]) * ie,
                          __uint_as_float(v[4 * j + 2]) * ie, __uint_as_float(v[4 * j + 3]) * ie);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&tempty[ub]);
        if (a.gready != nullptr) {
          __threadfence();
          flag_add_release_gpu(a.gready + ((long long)x.b * a.H + x.h) * (a.T - 1) + x.slot, 1u);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    const int issued = *issued_slot;
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
    tmem_dealloc(tmem, 2 * kTmemCols);
  }
}

}  // namespace

cudaError_t launch_gram_fp8_tc(const Problem& p, const void* K8, const void* V8, const float* kv_scale,
                               const void* Kt8, const void* Vt8, const float* kvt_scale, int* unit_exp,
                               cudaStream_t s) {
  if (p.D != D) return cudaErrorNotSupported;
  Gram8Args a{p.B, p.H, p.T, p.U, p.L, p.Ht, p.beta, p.beta_txt, kv_scale, kvt_scale, unit_exp,
              p.A, p.Bm, p.status, p.gready, p.spin_limit};
  const int nunits = p.B * p.H * (p.T - 1);
  fp8_unit_exp_kernel<<<(nunits * 32 + 255) / 256, 256, 0, s>>>(a, unit_exp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = set_max_dynamic_smem(reinterpret_cast<const void*>(gram_fp8_tc_kernel), kSmemBytes);
  if (e != cudaSuccess) return e;
  const uint64_t H = p.H, T = p.T, U = p.U, L = p.L, B = p.B, Ht = p.Ht;
  // [B, T*U, Ht, 128] e4m3 from this problem's first head: dims (d, h, u, t, b);
  // heads are adjacent in a token row (stride d bytes), tokens Ht * d bytes apart.
  const uint64_t dv[5] = {D, H, U, T, B};
  const uint32_t box[5] = {(uint32_t)D, 1u, (uint32_t)kTileU, 1u, 1u};
  const uint64_t st5[4] = {D, Ht * D, U * Ht * D, T * U * Ht * D};
  CUtensorMap mK, mV, mKt, mVt;
  if ((e = make_tmap_typed(&mK, CU_TENSOR_MAP_DATA_TYPE_UINT8, K8, 5, dv, st5, box, CU_TENSOR_MAP_SWIZZLE_128B)))
    return e;
  if ((e = make_tmap_typed(&mV, CU_TENSOR_MAP_DATA_TYPE_UINT8, V8, 5, dv, st5, box, CU_TENSOR_MAP_SWIZZLE_128B)))
    return e;
  // [B, L, Ht, 128]: dims (d, h, u, 1, b)
  const uint64_t dt[5] = {D, H, L, 1, B};
  const uint64_t stt[4] = {D, Ht * D, L * Ht * D, L * Ht * D};
  if ((e = make_tmap_typed(&mKt, CU_TENSOR_MAP_DATA_TYPE_UINT8, Kt8, 5, dt, stt, box, CU_TENSOR_MAP_SWIZZLE_128B)))
    return e;
  if ((e = make_tmap_typed(&mVt, CU_TENSOR_MAP_DATA_TYPE_UINT8, Vt8, 5, dt, stt, box, CU_TENSOR_MAP_SWIZZLE_128B)))
    return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int rounds = (nunits + sms - 1) / sms;
  const int grid = (nunits + rounds - 1) / rounds;
  gram_fp8_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(mK, mV, mKt, mVt, a);
  return cudaGetLastError();
}

}  // namespace vda
