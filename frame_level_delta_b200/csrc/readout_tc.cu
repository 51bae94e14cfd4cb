// Readout on tcgen05 tensor cores with the gather prologue and the fused
// epilogue (Video DeltaNet summary, onedev.kr/papers/80: section "how it works"
// -- query frame t of chunk j reads o = S-> q + S<- q from the states outside its
// chunk window; section "how it differs" -- L2-normalised queries, RMS norm and
// a sigmoid output gate on the linear readout).
//
// Tiles of 128 consecutive tokens of one chunk's non-anchor frames form one
// linear list over (b, h, chunk); each persistent CTA takes a contiguous range of
// it. Per (b, h, chunk) the prologue forms S = S-> + S<- in fp32 and splits it
// into bf16 hi + lo parts stored as K-major swizzled B operands, so
//   O_tile = Q_tile S_hi^T + Q_tile S_lo^T   (M = 128 tokens, N = d_v, K = d_k)
// accumulates in fp32 in TMEM with the state carried to ~2^-17 relative. Q tiles
// arrive by TMA (K-major, 128-byte swizzle). TMEM is double-buffered so the
// epilogue of one tile overlaps the MMAs of the next. The epilogue (one thread
// per token row) applies 1/|q| (conv prep), RMSNorm and the gate, converts to
// bf16, stages the tile in shared memory and writes it with a TMA store (plain
// stores for the last, partial tile of a chunk).
// Warp roles: 0 = TMA producer, 1 = TMEM owner + MMA issuer, 2..5 = prologue
// and epilogue.
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace vda {

namespace {

constexpr int kTileM = 128;
constexpr int kThreads = 192;
constexpr int kStages = 2;

template <int D>
struct RoCfg {
  static constexpr int kBoxes = D / 64;                   // 64-channel boxes per token tile
  static constexpr int kTileBytes = kTileM * D * 2;       // one bf16 token tile
  static constexpr int kSAtomBytes = D * 128;             // one K-atom (64 k) of S: D rows x 128 B
  static constexpr int kSBytes = kBoxes * kSAtomBytes;    // one bf16 copy of S
  static constexpr int kTmemCols = 2 * D;                 // two accumulators
  static constexpr uint32_t kIdesc = sm100::idesc_bf16_f32(128, D, false, false);
  // layout: S_hi | S_lo | Q[kStages] | AUX[kStages] | barriers
  static constexpr int kSmemBytes = 2 * kSBytes + 2 * kStages * kTileBytes + 1024 + 256;
};

struct RoArgs {
  int B, H, T, U, c, J;
  unsigned flags;
  float l2_eps, rms_eps;
  const float* Sf;
  const float* Sr;
  __nv_bfloat16* O;
  uint32_t* status;
  unsigned long long wait_ns;
  long long total_tiles;
  long long tiles_per_cta;
};

// Non-anchor frame range [t_lo, t_hi) of chunk j.
__device__ __forceinline__ void chunk_frames(const RoArgs& a, int j, int& t_lo, int& t_hi) {
  t_lo = max(a.c * j, 1);
  t_hi = min(a.c * (j + 1), a.T - 1);
}
__device__ __forceinline__ int chunk_tiles(const RoArgs& a, int j) {
  int lo, hi;
  chunk_frames(a, j, lo, hi);
  return lo < hi ? (int)(((long long)(hi - lo) * a.U + kTileM - 1) / kTileM) : 0;
}

struct TileInfo {
  int bh;            // b * H + h
  int j;             // chunk
  long long tok0;    // first token of the tile (flat index over B*T*U)
  int nvalid;        // rows of the tile inside the chunk
};

__device__ __forceinline__ TileInfo tile_info(const RoArgs& a, long long id, int tiles_per_head) {
  TileInfo ti;
  ti.bh = (int)(id / tiles_per_head);
  int local = (int)(id % tiles_per_head);
  int j = 0;
  for (;; ++j) {
    const int n = chunk_tiles(a, j);
    if (local < n) break;
    local -= n;
  }
  ti.j = j;
  int lo, hi;
  chunk_frames(a, j, lo, hi);
  const long long first = (long long)lo * a.U + (long long)local * kTileM;
  const long long end = (long long)hi * a.U;
  ti.nvalid = (int)min((long long)kTileM, end - first);
  const int b = ti.bh / a.H;
  ti.tok0 = (long long)b * a.T * a.U + first;
  return ti;
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(sm100::smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ float sigmoid_f(float x) { return 1.0f / (1.0f + __expf(-x)); }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    readout_tc_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mG,
                      const __grid_constant__ CUtensorMap mO, const RoArgs a) {
  using C = RoCfg<D>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sShi = smem;
  uint8_t* sSlo = smem + C::kSBytes;
  uint8_t* sQ = smem + 2 * C::kSBytes;
  uint8_t* sAux = sQ + kStages * C::kTileBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sAux + kStages * C::kTileBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* sready = tempty + 2;
  uint64_t* drain = sready + 1;
  uint64_t* epibar = drain + 1;  // bounded barrier of the 128 epilogue threads
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epibar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const bool gate = (a.flags & VDA_READOUT_NORM_GATE) != 0;
  const bool qnorm = (a.flags & VDA_PREP_CONV) != 0;
  int tiles_per_head = 0;
  for (int j = 0; j < a.J; ++j) tiles_per_head += chunk_tiles(a, j);
  const long long t_begin = (long long)blockIdx.x * a.tiles_per_cta;
  const long long t_end = min(a.total_tiles, t_begin + a.tiles_per_cta);
  const int ntiles = t_begin < t_end ? (int)(t_end - t_begin) : 0;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 2);  // MMA commit + epilogue
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);
    }
    mbar_init(sready, 4);
    mbar_init(drain, 1);
    mbar_init(epibar, 128);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&mQ);
    prefetch_tmap(&mO);
    if (gate) prefetch_tmap(&mG);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  int issued = 0;  // producer only

  if (warp == 0) {
    // ---------------- TMA producer: Q tile (+ gate tile) per stage
    if (lane == 0) {
      const uint32_t bytes = C::kTileBytes * (gate ? 2 : 1);
      for (int it = 0; it < ntiles; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, a.status, a.wait_ns)) break;
        const TileInfo ti = tile_info(a, t_begin + it, tiles_per_head);
        const int h = ti.bh % a.H;
        mbar_arrive_expect_tx(&full[s], bytes);
#pragma unroll
        for (int box = 0; box < C::kBoxes; ++box) {
          tma_load_3d(sQ + s * C::kTileBytes + box * (kTileM * 128), &mQ, &full[s], box * 64, h, (int)ti.tok0);
          if (gate)
            tma_load_3d(sAux + s * C::kTileBytes + box * (kTileM * 128), &mG, &full[s], box * 64, h,
                        (int)ti.tok0);
        }
        issued = it + 1;
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int g_prev = -1, gi = 0;
      for (int it = 0; it < ntiles; ++it) {
        const TileInfo ti = tile_info(a, t_begin + it, tiles_per_head);
        const int g = ti.bh * a.J + ti.j;
        if (g != g_prev) {
          if (!mbar_wait(sready, gi & 1, abort_flag, a.status, a.wait_ns)) break;
          ++gi;
          g_prev = g;
        }
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        const int tb = it & 1;
        const uint32_t tph = (it >> 1) & 1;
        if (!mbar_wait(&full[s], ph, abort_flag, a.status, a.wait_ns)) break;
        if (!mbar_wait(&tempty[tb], tph ^ 1, abort_flag, a.status, a.wait_ns)) break;
        tc_fence_after();
        const uint32_t qb = smem_u32(sQ + s * C::kTileBytes);
        const uint32_t hb = smem_u32(sShi), lb = smem_u32(sSlo);
        const uint32_t dtm = tmem + tb * D;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int atom = kk / 4;
          const uint32_t koff = (kk % 4) * 32;
          const uint64_t dq = smem_desc_sw128(qb + atom * (kTileM * 128) + koff, 16, 1024);
          const uint64_t dh = smem_desc_sw128(hb + atom * C::kSAtomBytes + koff, 16, 1024);
          const uint64_t dl = smem_desc_sw128(lb + atom * C::kSAtomBytes + koff, 16, 1024);
          mma_f16(dtm, dq, dh, C::kIdesc, kk > 0 ? 1u : 0u);
          mma_f16(dtm, dq, dl, C::kIdesc, 1u);
        }
        mma_commit(&empty[s]);
        mma_commit(&tfull[tb]);
      }
      mma_commit(drain);  // completes once every MMA issued above has finished
    }
  } else {
    // ---------------- prologue (S = S-> + S<-, split hi/lo) and epilogue
    const int et = threadIdx.x - 64;  // 0..127 == tile row == TMEM lane
    const int q = warp % 4;
    const int r = q * 32 + lane;      // TMEM lane this warp may read
    int g_prev = -1;
    bool ok = true;
    uint32_t epi_phase = 0;
    // All 128 epilogue threads meet here; bounded, so a timed-out peer cannot
    // leave the others waiting.
    auto epi_sync = [&]() -> bool {
      mbar_arrive(epibar);
      const bool r = mbar_wait(epibar, epi_phase, abort_flag, a.status, a.wait_ns);
      epi_phase ^= 1;
      return r;
    };
    for (int it = 0; it < ntiles && ok; ++it) {
      const TileInfo ti = tile_info(a, t_begin + it, tiles_per_head);
      const int g = ti.bh * a.J + ti.j;
      if (g != g_prev) {
        // The MMAs of the previous tile are complete (its accumulator was read
        // below) and the next MMA waits for `sready`: S may be overwritten.
        const long long off = ((long long)ti.bh * a.J + ti.j) * (long long)D * D;
        for (int e = et; e < D * (D / 8); e += 128) {
          const int i = e / (D / 8), c8 = e % (D / 8);  // row i, 8 consecutive k
          const float4* pf = reinterpret_cast<const float4*>(a.Sf + off + (long long)i * D + c8 * 8);
          const float4* pr = reinterpret_cast<const float4*>(a.Sr + off + (long long)i * D + c8 * 8);
          float x[8];
          const float4 f0 = pf[0], f1 = pf[1], r0 = pr[0], r1 = pr[1];
          x[0] = f0.x + r0.x; x[1] = f0.y + r0.y; x[2] = f0.z + r0.z; x[3] = f0.w + r0.w;
          x[4] = f1.x + r1.x; x[5] = f1.y + r1.y; x[6] = f1.z + r1.z; x[7] = f1.w + r1.w;
          uint4 hv, lv;
          __nv_bfloat162* hp = reinterpret_cast<__nv_bfloat162*>(&hv);
          __nv_bfloat162* lp = reinterpret_cast<__nv_bfloat162*>(&lv);
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2) {
            const __nv_bfloat162 hh = __floats2bfloat162_rn(x[2 * k2], x[2 * k2 + 1]);
            const float2 hf = __bfloat1622float2(hh);
            hp[k2] = hh;
            lp[k2] = __floats2bfloat162_rn(x[2 * k2] - hf.x, x[2 * k2 + 1] - hf.y);
          }
          const int atom = c8 / 8, chunk = c8 % 8;
          const int boff = atom * C::kSAtomBytes + i * 128 + ((chunk ^ (i & 7)) * 16);
          *reinterpret_cast<uint4*>(sShi + boff) = hv;
          *reinterpret_cast<uint4*>(sSlo + boff) = lv;
        }
        fence_proxy_async_smem();
        if (!epi_sync()) { ok = false; break; }
        if (lane == 0) mbar_arrive(sready);
        g_prev = g;
      }
      const int s = it % kStages;
      const uint32_t ph = (it / kStages) & 1;
      const int tb = it & 1;
      const uint32_t tph = (it >> 1) & 1;
      if (!mbar_wait(&tfull[tb], tph, abort_flag, a.status, a.wait_ns)) { ok = false; break; }
      if (!mbar_wait(&full[s], ph, abort_flag, a.status, a.wait_ns)) { ok = false; break; }
      tc_fence_after();
      const uint8_t* qrow = sQ + s * C::kTileBytes + r * 128;
      uint8_t* arow = sAux + s * C::kTileBytes + r * 128;
      float scale = 1.f;
      if (qnorm) {
        float qq = 0.f;
#pragma unroll
        for (int box = 0; box < C::kBoxes; ++box)
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(qrow + box * (kTileM * 128) + c * 16);
            const __nv_bfloat162* e = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2) {
              const float2 f = __bfloat1622float2(e[k2]);
              qq = fmaf(f.x, f.x, fmaf(f.y, f.y, qq));
            }
          }
        scale = rsqrtf(qq + a.l2_eps);
      }
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + tb * D;
      float rn = 1.f;
      if (gate) {
        float ss = 0.f;
#pragma unroll 1
        for (int cc = 0; cc < D / 16; ++cc) {
          uint32_t v[16];
          tmem_ld16(taddr + cc * 16, v);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float x = __uint_as_float(v[k]) * scale;
            ss = fmaf(x, x, ss);
          }
        }
        rn = rsqrtf(ss / D + a.rms_eps);
      }
      const bool partial = ti.nvalid < kTileM;
      const int h = ti.bh % a.H;
      __nv_bfloat16* orow = a.O + ((ti.tok0 + r) * a.H + h) * (long long)D;
#pragma unroll 1
      for (int cc = 0; cc < D / 16; ++cc) {
        uint32_t v[16];
        tmem_ld16(taddr + cc * 16, v);
        tmem_ld_wait();
        const int box = cc / 4, c16 = (cc % 4) * 2;  // two 16-byte chunks per 16 columns
        uint4 outv[2];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int pc = (c16 + half) ^ (r & 7);
          float g8[8];
          if (gate) {
            const uint4 gv = *reinterpret_cast<const uint4*>(arow + box * (kTileM * 128) + pc * 16);
            const __nv_bfloat162* ge = reinterpret_cast<const __nv_bfloat162*>(&gv);
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2) {
              const float2 f = __bfloat1622float2(ge[k2]);
              g8[2 * k2] = sigmoid_f(f.x) * rn;
              g8[2 * k2 + 1] = sigmoid_f(f.y) * rn;
            }
          } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) g8[k] = 1.f;
          }
          __nv_bfloat162* op = reinterpret_cast<__nv_bfloat162*>(&outv[half]);
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2)
            op[k2] = __floats2bfloat162_rn(__uint_as_float(v[half * 8 + 2 * k2]) * scale * g8[2 * k2],
                                           __uint_as_float(v[half * 8 + 2 * k2 + 1]) * scale * g8[2 * k2 + 1]);
          if (!partial) {
            *reinterpret_cast<uint4*>(arow + box * (kTileM * 128) + pc * 16) = outv[half];
          }
        }
        if (partial && r < ti.nvalid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 16);
          dst[0] = outv[0];
          dst[1] = outv[1];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[tb]);
      fence_proxy_async_smem();
      if (!epi_sync()) { ok = false; break; }
      if (et == 0) {
        if (!partial) {
#pragma unroll
          for (int box = 0; box < C::kBoxes; ++box)
            tma_store_3d(&mO, sAux + s * C::kTileBytes + box * (kTileM * 128), box * 64, h, (int)ti.tok0);
          bulk_commit();
          bulk_wait_read0();
        }
        mbar_arrive(&empty[s]);
      }
    }
    if (et == 0) bulk_wait0();  // all output writes done before the CTA retires
  }

  // ---------------- teardown
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      int last = -1;
      for (int it = s; it < issued; it += kStages) last = it;
      if (last >= 0) mbar_wait(&full[s], (last / kStages) & 1, nullptr, a.status, a.wait_ns);
    }
  }
  if (warp == 1) {
    if (lane == 0) mbar_wait(drain, 0, nullptr, a.status, a.wait_ns);  // all MMAs retired
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D>
cudaError_t launch_d(const Problem& p, const void* gate, void* O, cudaStream_t s) {
  using C = RoCfg<D>;
  RoArgs a{};
  a.B = p.B; a.H = p.H; a.T = p.T; a.U = p.U; a.c = p.c; a.J = p.J;
  a.flags = p.flags; a.l2_eps = p.l2_eps; a.rms_eps = p.rms_eps;
  a.Sf = p.Sf; a.Sr = p.Sr; a.O = static_cast<__nv_bfloat16*>(O);
  a.status = p.status; a.wait_ns = p.spin_limit;
  long long tiles_per_head = 0;
  for (int j = 0; j < p.J; ++j) {
    const int lo = std::max(p.c * j, 1), hi = std::min(p.c * (j + 1), p.T - 1);
    if (lo < hi) tiles_per_head += ((long long)(hi - lo) * p.U + kTileM - 1) / kTileM;
  }
  a.total_tiles = tiles_per_head * p.B * p.H;
  if (a.total_tiles == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static bool attr_set = false;
  cudaError_t e;
  if (!attr_set) {
    e = cudaFuncSetAttribute(readout_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  int per_sm = 1;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, readout_tc_kernel<D>, kThreads, C::kSmemBytes);
  if (per_sm < 1) per_sm = 1;
  const long long grid = std::min<long long>(a.total_tiles, (long long)sms * per_sm);
  a.tiles_per_cta = (a.total_tiles + grid - 1) / grid;
  const long long ncta = (a.total_tiles + a.tiles_per_cta - 1) / a.tiles_per_cta;

  // [B*T*U tokens, H, D] views of Q, gate and O: dims (d, h, token)
  const uint64_t D64 = D, H = p.H, NT = (uint64_t)p.B * p.T * p.U;
  uint64_t dims[3] = {D64, H, NT};
  uint64_t strides[2] = {D64 * 2, H * D64 * 2};
  uint32_t box[3] = {64, 1, (uint32_t)kTileM};
  CUtensorMap mQ, mG, mO;
  if ((e = make_tmap_bf16(&mQ, p.Q, 3, dims, strides, box)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&mO, O, 3, dims, strides, box)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&mG, gate ? gate : p.Q, 3, dims, strides, box)) != cudaSuccess) return e;
  readout_tc_kernel<D><<<(unsigned)ncta, kThreads, C::kSmemBytes, s>>>(mQ, mG, mO, a);
  return cudaGetLastError();
}

}  // namespace

bool readout_tc_supported(const Problem& p) {
  return p.bf16 && (p.D == 64 || p.D == 128) && (long long)p.B * p.T * p.U < (1LL << 31);
}

cudaError_t launch_readout_tc(const Problem& p, const void* gate, void* O, cudaStream_t s) {
  if (p.D == 128) return launch_d<128>(p, gate, O, s);
  if (p.D == 64) return launch_d<64>(p, gate, O, s);
  return cudaErrorNotSupported;
}

}  // namespace vda
