// Frame statistics on tcgen05 tensor cores: for every (b, h, slot)
//   A = K^T Diag(beta) K   (d_k x d_k),   B = V^T Diag(beta) K   (d_v x d_k),
// slot 0 over the text tokens, slot t over the U tokens of frame t (Video
// DeltaNet summary, onedev.kr/papers/80, section "how to use": the key
// correlation and value-key write statistics of a frame).
//
// Both products contract over tokens, the slow axis of a [tokens x d] tile, so
// both tcgen05 operands are MN-major: TMA brings K and V token tiles (64 tokens
// x 64 channels per box, 128-byte swizzle, zero fill past the frame's last token)
// into shared memory (six stages in flight), four warps write beta*K (bf16,
// round to nearest) into a two-slot ring that the MMAs release, and one thread
// issues tcgen05.mma with fp32 accumulation in TMEM: A = K^T (beta K),
// B = V^T (beta K). Warp roles: 0 = TMA producer, 1 = TMEM owner + MMA issuer,
// 2..5 = beta scaling, 6..9 = TMEM -> global epilogue.
//
// d = 128: two M=128 N=128 MMAs per 16-token step (K-part -> TMEM columns
// 0..127, V-part -> 128..255). d = 64: one M=128 N=64 MMA whose A operand is
// [K | V] stacked along M (rows 0..63 give A, rows 64..127 give B).
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace vda {

namespace {

constexpr int kTileU = 64;                    // tokens per pipeline stage
constexpr int kBoxBytes = kTileU * 128;       // one box: 64 tokens x 64 bf16
constexpr int kThreads = 320;  // 10 warps: producer, MMA, 4 scaling, 4 epilogue

template <int D>
struct GramCfg {
  static constexpr int kBoxes = D / 64;                     // boxes per operand tile
  static constexpr int kStageBytes = 2 * kBoxes * kBoxBytes;  // K and V token tiles
  // HBM reads in flight per SM. At d = 128 five 32 KB stages leave ~32 KB of the
  // SM's shared memory and ~42k registers free, room for two compact frame-solve
  // CTAs beside this one.
  static constexpr int kStages = D == 128 ? 5 : 12;
  static constexpr int kBkSlots = 2;                        // beta*K ring, released by the MMAs
  static constexpr int kBkBytes = kBoxes * kBoxBytes;
  static constexpr int kTmemCols = D == 128 ? 256 : 64;
  static constexpr uint32_t kIdesc =
      D == 128 ? sm100::idesc_bf16_f32(128, 128, true, true) : sm100::idesc_bf16_f32(128, 64, true, true);
  static constexpr int kBetaBytes = kStages * kTileU * 4;  // beta of each stage's tokens
  static constexpr int kBarrierBytes = (2 * kStages + 2 * kBkSlots + 5) * 8 + 16;  // mbarriers + TMEM slot, flags
  static constexpr int kSmemBytes = kStages * kStageBytes + kBkSlots * kBkBytes + kBetaBytes + 1024 /*align*/ + 512;
  static_assert(kBarrierBytes <= 512, "barrier block overflows its allowance");
  static_assert(kSmemBytes <= 232448, "more shared memory than a CTA may use");
};

struct GramArgs {
  int B, H, T, U, L;
  int layout;  // 0: token-major [B, tokens, H, d]; 1: frame-major [B, H, frames, tokens, d]
  const float* beta;
  const float* beta_txt;
  float* A;
  float* Bm;
  uint32_t* status;
  uint32_t* gready;  // [B,H,T-1] per-slot counts raised after the stores, or nullptr
  unsigned long long wait_ns;
};

// Unit u = (b, h, slot) in the key order the solve consumes slots in (slot 0,
// then slots k and T-1-k for k = 1, 2, ...), heads fastest within a slot, so
// the CTAs working at any moment cover all heads of the same frames (one 6 KB
// token row holds every head).
struct Unit {
  int b, h, slot, n;
};
__device__ __forceinline__ Unit unit_of(const GramArgs& a, int u) {
  Unit x;
  int bh;
  key_slot(u, a.B * a.H, a.T - 1, bh, x.slot);
  x.b = bh / a.H;
  x.h = bh % a.H;
  x.n = x.slot == 0 ? a.L : a.U;
  return x;
}

// Persistent: CTA p takes units p, p + G, p + 2G, ... and streams their token
// tiles through one continuous TMA pipeline; the accumulator alternates between
// two TMEM buffers so the epilogue of one unit overlaps the MMAs of the next.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    gram_tc_kernel(const __grid_constant__ CUtensorMap mK, const __grid_constant__ CUtensorMap mV,
                   const __grid_constant__ CUtensorMap mKt, const __grid_constant__ CUtensorMap mVt,
                   const GramArgs a) {
  using C = GramCfg<D>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = sm100::align_smem_1024(smem_raw);
  uint8_t* bkring = smem + C::kStages * C::kStageBytes;  // beta*K slots
  float* sbeta = reinterpret_cast<float*>(bkring + C::kBkSlots * C::kBkBytes);  // [kStages][kTileU]
  uint64_t* full = reinterpret_cast<uint64_t*>(sbeta + C::kStages * kTileU);
  uint64_t* empty = full + C::kStages;
  uint64_t* bkf = empty + C::kStages;     // [kBkSlots] beta*K written
  uint64_t* bke = bkf + C::kBkSlots;      // [kBkSlots] beta*K slot free again
  uint64_t* tfull = bke + C::kBkSlots;    // [2]
  uint64_t* tempty = tfull + 2;          // [2]
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* issued_slot = reinterpret_cast<int*>(tmem_slot + 2);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nunits = a.B * a.H * (a.T - 1);
  const int G = gridDim.x;
  // The solve may launch now: its CTAs take the SMs this grid leaves and wait
  // for their slot's count.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1 + 32);  // TMA bytes + the 32 lanes' beta copies
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < C::kBkSlots; ++i) {
      mbar_init(&bkf[i], 4);
      mbar_init(&bke[i], 1);
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
    tmem_alloc(tmem_slot, 2 * C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- producer warp: TMA loads of K, V (lane 0) and asynchronous
    // copies of the stage's beta values (all lanes), all completing on full[s],
    // so beta arrives as far ahead of its use as the token tiles do.
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < nunits && ok; u += G) {
      const Unit x = unit_of(a, u);
      const CUtensorMap* mk = x.slot == 0 ? &mKt : &mK;
      const CUtensorMap* mv = x.slot == 0 ? &mVt : &mV;
      const float* beta = x.slot == 0 ? a.beta_txt + ((long long)x.b * a.H + x.h) * a.L
                                      : a.beta + (((long long)x.b * a.H + x.h) * a.T + x.slot) * (long long)a.U;
      const int ntiles = (x.n + kTileU - 1) / kTileU;
      for (int tt = 0; tt < ntiles; ++tt, ++it) {
        const int s = it % C::kStages;
        const uint32_t ph = (it / C::kStages) & 1;
        int good = 1;
        if (lane == 0) good = mbar_wait(&empty[s], ph ^ 1, abort_flag, a.status, a.wait_ns) ? 1 : 0;
        good = __shfl_sync(0xffffffffu, good, 0);
        if (!good) { ok = false; break; }
        const int u0 = tt * kTileU;
        if (lane == 0) {
          uint8_t* st = smem + s * C::kStageBytes;
          mbar_arrive_expect_tx(&full[s], 2 * C::kBoxes * kBoxBytes);
#pragma unroll
          for (int box = 0; box < C::kBoxes; ++box) {
            const int d0 = box * 64;
            if (a.layout == 0) {
              tma_load_5d(st + box * kBoxBytes, mk, &full[s], d0, x.h, u0, x.slot, x.b);
              tma_load_5d(st + (C::kBoxes + box) * kBoxBytes, mv, &full[s], d0, x.h, u0, x.slot, x.b);
            } else {
              tma_load_5d(st + box * kBoxBytes, mk, &full[s], d0, u0, x.slot, x.h, x.b);
              tma_load_5d(st + (C::kBoxes + box) * kBoxBytes, mv, &full[s], d0, u0, x.slot, x.h, x.b);
            }
          }
        }
        // beta of tokens u0 + lane and u0 + 32 + lane (zero past the slot's last token)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int uu = u0 + half * 32 + lane;
          const bool in = uu < x.n;
          cp_async_4(sbeta + s * kTileU + half * 32 + lane, in ? beta + uu : beta, in ? 4u : 0u);
        }
        cp_async_mbar_arrive_noinc(&full[s]);
      }
    }
    if (lane == 0) *issued_slot = it;
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int it = 0, k = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < nunits && ok; u += G, ++k) {
        const Unit x = unit_of(a, u);
        const int ntiles = (x.n + kTileU - 1) / kTileU;
        const int ub = k & 1;
        const uint32_t tacc = tmem + ub * C::kTmemCols;
        if (!mbar_wait(&tempty[ub], ((k >> 1) & 1) ^ 1, abort_flag, a.status, a.wait_ns)) break;
        tc_fence_after();
        for (int tt = 0; tt < ntiles; ++tt, ++it) {
          const int s = it % C::kStages;
          const uint32_t ph = (it / C::kStages) & 1;
          const int bs = it % C::kBkSlots;
          const uint32_t bph = (it / C::kBkSlots) & 1;
          if (!mbar_wait(&full[s], ph, abort_flag, a.status, a.wait_ns) ||
              !mbar_wait(&bkf[bs], bph, abort_flag, a.status, a.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t base = smem_u32(smem + s * C::kStageBytes);
          const uint32_t bkb = smem_u32(bkring + bs * C::kBkBytes);
#pragma unroll
          for (int kk = 0; kk < kTileU / 16; ++kk) {
            const uint32_t koff = kk * 16 * 128;  // 16 token rows of 128 bytes
            const uint32_t acc = (tt > 0 || kk > 0) ? 1u : 0u;
            const uint64_t dB = smem_desc_sw128(bkb + koff, kBoxBytes, 1024);  // beta*K
            if constexpr (D == 128) {
              const uint64_t dK = smem_desc_sw128(base + koff, kBoxBytes, 1024);
              const uint64_t dV = smem_desc_sw128(base + 2 * kBoxBytes + koff, kBoxBytes, 1024);
              mma_f16(tacc, dK, dB, C::kIdesc, acc);
              mma_f16(tacc + 128, dV, dB, C::kIdesc, acc);
            } else {
              const uint64_t dKV = smem_desc_sw128(base + koff, kBoxBytes, 1024);  // K box then V box
              mma_f16(tacc, dKV, dB, C::kIdesc, acc);
            }
          }
          mma_commit(&empty[s]);
          mma_commit(&bke[bs]);
        }
        if (ok) mma_commit(&tfull[ub]);
      }
      mma_commit(drain);  // completes once every MMA issued above has finished
    }
  } else if (warp < 6) {
    // ---------------- beta*K into the ring (warps 2..5)
    const int tid = threadIdx.x - 64;  // 0..127
    int row, box, c0, c1;
    if constexpr (D == 128) {
      box = tid / 64;
      row = tid % 64;
      c0 = 0;
      c1 = 8;
    } else {
      box = 0;
      row = tid / 2;
      c0 = (tid % 2) * 4;
      c1 = c0 + 4;
    }
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < nunits && ok; u += G) {
      const Unit x = unit_of(a, u);
      const int ntiles = (x.n + kTileU - 1) / kTileU;
      for (int tt = 0; tt < ntiles; ++tt, ++it) {
        const int s = it % C::kStages;
        const uint32_t ph = (it / C::kStages) & 1;
        const int bs = it % C::kBkSlots;
        const uint32_t bph = (it / C::kBkSlots) & 1;
        if (!mbar_wait(&bke[bs], bph ^ 1, abort_flag, a.status, a.wait_ns) ||
            !mbar_wait(&full[s], ph, abort_flag, a.status, a.wait_ns)) {
          ok = false;
          break;
        }
        const float bb = sbeta[s * kTileU + row];  // zero past the slot's last token
        const uint8_t* src = smem + s * C::kStageBytes + box * kBoxBytes + row * 128;
        uint8_t* dst = bkring + bs * C::kBkBytes + box * kBoxBytes + row * 128;
        for (int c = c0; c < c1; ++c) {
          const int pc = c ^ (row & 7);  // any chunk order works; this one avoids bank conflicts
          const uint4 v = *reinterpret_cast<const uint4*>(src + pc * 16);
          uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(bits_bf162(w[q]));
            w[q] = bf162_bits(__floats2bfloat162_rn(f.x * bb, f.y * bb));
          }
          *reinterpret_cast<uint4*>(dst + pc * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bkf[bs]);
      }
    }
  } else {
    // ---------------- epilogue (warps 6..9): TMEM -> A, B in global memory
    const int q = warp % 4;  // this warp may read TMEM lanes 32q .. 32q+31
    const int r = q * 32 + lane;
    int k = 0;
    for (int u = blockIdx.x; u < nunits; u += G, ++k) {
      const Unit x = unit_of(a, u);
      const int ub = k & 1;
      if (!mbar_wait(&tfull[ub], (k >> 1) & 1, abort_flag, a.status, a.wait_ns)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + ub * C::kTmemCols + ((uint32_t)(q * 32) << 16);
      const long long off = (((long long)x.b * a.H + x.h) * (a.T - 1) + x.slot) * (long long)D * D;
      if constexpr (D == 128) {
#pragma unroll 2
        for (int c = 0; c < 16; ++c) {
          uint32_t v[16];
          tmem_ld16(taddr + c * 16, v);
          tmem_ld_wait();
          float4* dst = reinterpret_cast<float4*>((c < 8 ? a.A : a.Bm) + off);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[((c % 8) * 4 + j) * D + r] =
                make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                            __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
        }
      } else {
        // Rows 0..63 of the stacked accumulator are A_t, rows 64..127 are B_t.
        float4* dst = reinterpret_cast<float4*>((r < 64 ? a.A : a.Bm) + off);
        const int rr = r & 63;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t v[16];
          tmem_ld16(taddr + c * 16, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[(c * 4 + j) * 64 + rr] =
                make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                            __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&tempty[ub]);
        // This warp's rows of A_t and B_t are stored (the warp barrier orders the
        // other lanes' stores before this fence): count them for the solve.
        if (a.gready != nullptr) {
          __threadfence();
          flag_add_release_gpu(a.gready + ((long long)x.b * a.H + x.h) * (a.T - 1) + x.slot, 1u);
        }
      }
    }
  }

  // ---------------- teardown: nothing may be in flight when TMEM and smem go away
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    // Wait (bounded) for the last TMA load issued into each stage.
    const int issued = *issued_slot;
    for (int s = 0; s < C::kStages; ++s) {
      int last = -1;
      for (int it = s; it < issued; it += C::kStages) last = it;
      if (last >= 0) mbar_wait(&full[s], (last / C::kStages) & 1, nullptr, a.status, a.wait_ns);
    }
  }
  if (warp == 1) {
    if (lane == 0) mbar_wait(drain, 0, nullptr, a.status, a.wait_ns);  // all MMAs retired
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 2 * C::kTmemCols);
  }
}

cudaError_t encode_maps(const Problem& p, CUtensorMap* mK, CUtensorMap* mV, CUtensorMap* mKt, CUtensorMap* mVt,
                        int* layout) {
  const uint64_t D = p.D, H = p.H, T = p.T, U = p.U, L = p.L, B = p.B, Ht = p.Ht;
  const bool prep = (p.flags & VDA_PREP_CONV) != 0;
  *layout = prep ? 1 : 0;
  cudaError_t e;
  if (!prep) {
    // [B, T*U, Ht, D] from this problem's first head on: dims (d, h, u, t, b)
    uint64_t dv[5] = {D, H, U, T, B};
    uint64_t sv[4] = {D * 2, Ht * D * 2, U * Ht * D * 2, T * U * Ht * D * 2};
    uint32_t box[5] = {64, 1, (uint32_t)kTileU, 1, 1};
    if ((e = make_tmap_bf16(mK, p.Kv.p, 5, dv, sv, box)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16(mV, p.Vv.p, 5, dv, sv, box)) != cudaSuccess) return e;
    // [B, L, Ht, D]: dims (d, h, u, 1, b)
    uint64_t dt[5] = {D, H, L, 1, B};
    uint64_t st[4] = {D * 2, Ht * D * 2, L * Ht * D * 2, L * Ht * D * 2};
    if ((e = make_tmap_bf16(mKt, p.Kt.p, 5, dt, st, box)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16(mVt, p.Vt.p, 5, dt, st, box)) != cudaSuccess) return e;
  } else {
    // [B, H, T, U, D]: dims (d, u, t, h, b)
    uint64_t dv[5] = {D, U, T, H, B};
    uint64_t sv[4] = {D * 2, U * D * 2, T * U * D * 2, H * T * U * D * 2};
    uint32_t box[5] = {64, (uint32_t)kTileU, 1, 1, 1};
    if ((e = make_tmap_bf16(mK, p.Kv.p, 5, dv, sv, box)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16(mV, p.Vv.p, 5, dv, sv, box)) != cudaSuccess) return e;
    // [B, H, L, D]: dims (d, u, 1, h, b)
    uint64_t dt[5] = {D, L, 1, H, B};
    uint64_t st[4] = {D * 2, L * D * 2, L * D * 2, H * L * D * 2};
    if ((e = make_tmap_bf16(mKt, p.Kt.p, 5, dt, st, box)) != cudaSuccess) return e;
    if ((e = make_tmap_bf16(mVt, p.Vt.p, 5, dt, st, box)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <int D>
cudaError_t launch_d(const Problem& p, cudaStream_t s) {
  using C = GramCfg<D>;
  CUtensorMap mK, mV, mKt, mVt;
  GramArgs a{p.B, p.H, p.T, p.U, p.L, 0, p.beta, p.beta_txt, p.A, p.Bm, p.status, p.gready, p.spin_limit};
  cudaError_t e = encode_maps(p, &mK, &mV, &mKt, &mVt, &a.layout);
  if (e != cudaSuccess) return e;
  e = set_max_dynamic_smem(reinterpret_cast<const void*>(gram_tc_kernel<D>), C::kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // As few CTAs as keep the same number of units on the busiest one: the
  // kernel is bound by HBM, not by SMs, so a grid that divides the units evenly
  // ends without a partial last round, and the SMs left over start the solve early.
  // One round more than the SM count needs, on problems of two or more rounds:
  // the statistics still saturate HBM on ~80% of the SMs, and the SMs left over
  // run solve CTAs beside them (measured at the H3-like clip: 117 CTAs of 8
  // units, 0.431 ms per step, against 134 of 7, 0.435 ms).
  const int nunits = p.B * p.H * (p.T - 1);
  const int rounds = (nunits + sms - 1) / sms + (nunits >= 2 * sms ? 1 : 0);
  const int grid = (nunits + rounds - 1) / rounds;
  gram_tc_kernel<D><<<grid, kThreads, C::kSmemBytes, s>>>(mK, mV, mKt, mVt, a);
  return cudaGetLastError();
}

}  // namespace

bool gram_tc_supported(const Problem& p) { return p.bf16 && (p.D == 64 || p.D == 128); }

cudaError_t launch_gram_tc(const Problem& p, cudaStream_t s) {
  if (p.D == 128) return launch_d<128>(p, s);
  if (p.D == 64) return launch_d<64>(p, s);
  return cudaErrorNotSupported;
}

}  // namespace vda
