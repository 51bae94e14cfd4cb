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
// epilogue of one tile overlaps the MMAs of the next. The epilogue (two threads
// per token row, one per half of the columns) applies 1/|q| (conv prep), RMSNorm and the gate, converts to
// bf16, stages the tile in shared memory and writes it with a TMA store (plain
// stores for the last, partial tile of a chunk).
// Warp roles: 0 = TMA producer, 1 = TMEM owner + MMA issuer, 2..9 = prologue
// and epilogue (two warps per TMEM lane quadrant, one per half of the output
// columns).
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace vda {

namespace {

constexpr int kTileM = 128;
constexpr int kThreads = 320;     // TMA warp, MMA warp, eight epilogue warps
constexpr int kEpiThreads = 256;

template <int D, bool GATE>
struct RoCfg {
  static constexpr int kBoxes = D / 64;                   // 64-channel boxes per token tile
  static constexpr int kTileBytes = kTileM * D * 2;       // one bf16 token tile
  static constexpr int kSAtomBytes = D * 128;             // one K-atom (64 k) of S: D rows x 128 B
  static constexpr int kSBytes = kBoxes * kSAtomBytes;    // one bf16 copy of S
  // TMEM: two accumulators of D columns, then 4 columns for the row halves' partial sums.
  static constexpr uint32_t kXchgCol = 2 * D;
  static constexpr int kTmemAlloc = D == 128 ? 512 : 256;
  static constexpr uint32_t kIdesc = sm100::idesc_bf16_f32(128, D, false, false);
  // Q tiles are the only stream without the gate: four stages deep. With the
  // gate, a stage holds a Q tile and a gate tile: two stages.
  static constexpr int kStages = GATE ? 2 : (D == 128 ? 4 : 6);
  static constexpr int kStageBytes = kTileBytes * (GATE ? 2 : 1);
  // layout: S_hi | S_lo | stages | output staging tile | barriers
  static constexpr int kSmemBytes = 2 * kSBytes + kStages * kStageBytes + kTileBytes + 1024 + 256;
  static_assert((232448 / kSmemBytes) * kTmemAlloc <= 512, "CTAs that fit on an SM must fit in its TMEM");
  static_assert((2 * kStages + 7) * 8 + 16 <= 256, "barrier block overflows its allowance");
  static_assert(kSmemBytes <= 232448, "more shared memory than a CTA may use");
};

struct RoArgs {
  int B, H, T, U, c, J;
  int Ht;  // heads per token row of Q, gate and O (O points at this problem's first head)
  unsigned flags;
  float l2_eps, rms_eps;
  const float* Sf;
  const float* Sr;
  __nv_bfloat16* O;
  uint32_t* status;
  unsigned long long wait_ns;
  int BH;           // B * H
  int nseg;         // token segments per (b, h); CTA p serves (b, h) = p % BH, segment p / BH
  int tiles_per_seg;
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


// The tiles of one (b, h) in order, one step at a time: chunk j and tile
// `local` within it (the direct lookup walks every earlier chunk).
struct TileIter {
  int j, local, n;  // chunk, tile within the chunk, tiles in the chunk
  __device__ __forceinline__ void start(const RoArgs& a, int t) {
    j = 0;
    for (;; ++j) {
      n = chunk_tiles(a, j);
      if (t < n) break;
      t -= n;
    }
    local = t;
  }
  // Valid only while tiles remain.
  __device__ __forceinline__ void next(const RoArgs& a) {
    if (++local < n) return;
    local = 0;
    do {
      n = chunk_tiles(a, ++j);
    } while (n == 0);
  }
  __device__ __forceinline__ TileInfo info(const RoArgs& a, int bh) const {
    TileInfo ti;
    ti.bh = bh;
    ti.j = j;
    int lo, hi;
    chunk_frames(a, j, lo, hi);
    const long long first = (long long)lo * a.U + (long long)local * kTileM;
    const long long end = (long long)hi * a.U;
    ti.nvalid = (int)min((long long)kTileM, end - first);
    ti.tok0 = (long long)(bh / a.H) * a.T * a.U + first;
    return ti;
  }
};

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(sm100::smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// The hardware's approximate tanh (about 2^-11 relative error, below the bf16
// rounding of the output): sigmoid(x) = (1 + tanh(x / 2)) / 2, one special-
// function operation instead of an exponential and a reciprocal.
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D, bool GATE>
__global__ void __launch_bounds__(kThreads, 1)
    readout_tc_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mG,
                      const __grid_constant__ CUtensorMap mO, const RoArgs a) {
  using C = RoCfg<D, GATE>;
  constexpr int kStages = C::kStages;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = sm100::align_smem_1024(smem_raw);
  uint8_t* sShi = smem;
  uint8_t* sSlo = smem + C::kSBytes;
  uint8_t* sQ = smem + 2 * C::kSBytes;  // stage s: Q tile at s * kStageBytes, gate tile after it
  uint8_t* sO = sQ + kStages * C::kStageBytes;  // output tile staged for the TMA store
  uint64_t* full = reinterpret_cast<uint64_t*>(sO + C::kTileBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* sready = tempty + 2;
  uint64_t* drain = sready + 1;
  uint64_t* epibar = drain + 1;  // bounded barrier of the 128 epilogue threads
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epibar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  constexpr bool gate = GATE;
  const bool qnorm = (a.flags & VDA_PREP_CONV) != 0;
  const bool stage_read = qnorm || GATE;  // the epilogue reads the stage's tiles
  int tiles_per_head = 0;
  for (int j = 0; j < a.J; ++j) tiles_per_head += chunk_tiles(a, j);
  // CTA p serves head pair bh = p % BH over its token segment p / BH: the CTAs of
  // one segment walk the same tokens of all heads in step, which keeps their
  // strided reads and writes within the same DRAM rows.
  const int my_bh = blockIdx.x % a.BH, seg = blockIdx.x / a.BH;
  const int t_begin = seg * a.tiles_per_seg;
  const int t_end = min(tiles_per_head, t_begin + a.tiles_per_seg);
  const int ntiles = t_begin < t_end ? t_end - t_begin : 0;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], stage_read ? 9 : 1);  // MMA commit (+ 8 epilogue warps)
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 8);
    }
    mbar_init(sready, 8);
    mbar_init(drain, 1);
    mbar_init(epibar, kEpiThreads);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&mQ);
    prefetch_tmap(&mO);
    if (gate) prefetch_tmap(&mG);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemAlloc);
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
      TileIter tit;
      if (ntiles > 0) tit.start(a, t_begin);
      for (int it = 0; it < ntiles; ++it) {
        if (it > 0) tit.next(a);
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, a.status, a.wait_ns)) break;
        const TileInfo ti = tit.info(a, my_bh);
        const int h = ti.bh % a.H;
        mbar_arrive_expect_tx(&full[s], bytes);
#pragma unroll
        for (int box = 0; box < C::kBoxes; ++box) {
          tma_load_3d(sQ + s * C::kStageBytes + box * (kTileM * 128), &mQ, &full[s], box * 64, h, (int)ti.tok0);
          if constexpr (GATE)
            tma_load_3d(sQ + s * C::kStageBytes + C::kTileBytes + box * (kTileM * 128), &mG, &full[s], box * 64,
                        h, (int)ti.tok0);
        }
        issued = it + 1;
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int g_prev = -1, gi = 0;
      TileIter tit;
      if (ntiles > 0) tit.start(a, t_begin);
      for (int it = 0; it < ntiles; ++it) {
        if (it > 0) tit.next(a);
        const TileInfo ti = tit.info(a, my_bh);
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
        const uint32_t qb = smem_u32(sQ + s * C::kStageBytes);
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
    // Eight warps: warp w reads TMEM lanes (tile rows) 32 (w % 4).. and owns
    // output columns hf * D / 2 .. of them.
    const int et = threadIdx.x - 64;  // 0..255
    const int q = warp % 4;
    const int hf = (warp - 2) / 4;
    const int r = q * 32 + lane;      // tile row == TMEM lane this warp may read
    // Anchor frames 0 and T-1 read no linear memory: while the first tile's
    // MMAs are in flight these threads zero this CTA's share of their rows (per
    // batch and anchor, U token rows of this problem's H * D values, at a row
    // stride of Ht * D; one contiguous slab when Ht == H).
    {
      const long long rw = (long long)a.H * D * 2 / 16;  // uint4 words per token row
      const long long per16 = (long long)a.U * rw;       // uint4 words per slab
      const long long G = gridDim.x;
      const long long lo = per16 * blockIdx.x / G, hi = per16 * (blockIdx.x + 1) / G;
      for (int slab = 0; slab < 2 * a.B; ++slab) {
        const long long b = slab >> 1, f = (slab & 1) ? a.T - 1 : 0;
        uint4* base = reinterpret_cast<uint4*>(a.O + (b * a.T + f) * (long long)a.U * a.Ht * D);
        const long long row16 = (long long)a.Ht * D * 2 / 16;
        for (long long w = lo + et; w < hi; w += kEpiThreads) base[(w / rw) * row16 + w % rw] = make_uint4(0, 0, 0, 0);
      }
    }
    int g_prev = -1;
    bool ok = true;
    uint32_t epi_phase = 0;
    // All 256 epilogue threads meet here; bounded, so a timed-out peer cannot
    // leave the others waiting.
    auto epi_sync = [&]() -> bool {
      mbar_arrive(epibar);
      const bool r = mbar_wait(epibar, epi_phase, abort_flag, a.status, a.wait_ns);
      epi_phase ^= 1;
      return r;
    };
    TileIter tit;
    if (ntiles > 0) tit.start(a, t_begin);
    for (int it = 0; it < ntiles && ok; ++it) {
      if (it > 0) tit.next(a);
      const TileInfo ti = tit.info(a, my_bh);
      const int g = ti.bh * a.J + ti.j;
      if (g != g_prev) {
        // The MMAs of the previous tile are complete (its accumulator was read
        // below) and the next MMA waits for `sready`: S may be overwritten.
        const long long off = ((long long)ti.bh * a.J + ti.j) * (long long)D * D;
        const float4* pf = reinterpret_cast<const float4*>(a.Sf + off);
        const float4* pr = reinterpret_cast<const float4*>(a.Sr + off);
        // Each thread takes kItems (row, 8-column) items; the loads of a batch of
        // them are issued before any is used, so a batch costs one L2 round trip.
        constexpr int kItems = D * (D / 8) / kEpiThreads;
        constexpr int kBatch = kItems < 4 ? kItems : 4;
        static_assert(kItems % kBatch == 0 && D * (D / 8) % kEpiThreads == 0, "prologue items");
#pragma unroll
        for (int b0 = 0; b0 < kItems; b0 += kBatch) {
          float4 f[kBatch][2], rv[kBatch][2];
#pragma unroll
          for (int bi = 0; bi < kBatch; ++bi) {
            const int e = et + (b0 + bi) * kEpiThreads;
            const int c8 = e / D, i = e % D;  // row i, 8 consecutive k (column quads 2 c8, 2 c8 + 1)
            f[bi][0] = pf[(2 * c8) * D + i];
            f[bi][1] = pf[(2 * c8 + 1) * D + i];
            rv[bi][0] = pr[(2 * c8) * D + i];
            rv[bi][1] = pr[(2 * c8 + 1) * D + i];
          }
#pragma unroll
          for (int bi = 0; bi < kBatch; ++bi) {
            const int e = et + (b0 + bi) * kEpiThreads;
            const int c8 = e / D, i = e % D;
            const float4 f0 = f[bi][0], f1 = f[bi][1], r0 = rv[bi][0], r1 = rv[bi][1];
            float x[8];
            x[0] = f0.x + r0.x; x[1] = f0.y + r0.y; x[2] = f0.z + r0.z; x[3] = f0.w + r0.w;
            x[4] = f1.x + r1.x; x[5] = f1.y + r1.y; x[6] = f1.z + r1.z; x[7] = f1.w + r1.w;
            uint32_t hp[4], lp[4];
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2) {
              const __nv_bfloat162 hh = __floats2bfloat162_rn(x[2 * k2], x[2 * k2 + 1]);
              const float2 hf = __bfloat1622float2(hh);
              hp[k2] = bf162_bits(hh);
              lp[k2] = bf162_bits(__floats2bfloat162_rn(x[2 * k2] - hf.x, x[2 * k2 + 1] - hf.y));
            }
            const uint4 hv = make_uint4(hp[0], hp[1], hp[2], hp[3]);
            const uint4 lv = make_uint4(lp[0], lp[1], lp[2], lp[3]);
            const int atom = c8 / 8, chunk = c8 % 8;
            const int boff = atom * C::kSAtomBytes + i * 128 + ((chunk ^ (i & 7)) * 16);
            *reinterpret_cast<uint4*>(sShi + boff) = hv;
            *reinterpret_cast<uint4*>(sSlo + boff) = lv;
          }
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
      tc_fence_after();
      // The Q tile (and gate tile) of this stage stay valid until this epilogue
      // releases the stage; without q-norm or gate the MMA commit alone releases it.
      if (stage_read && !mbar_wait(&full[s], ph, abort_flag, a.status, a.wait_ns)) { ok = false; break; }
      const uint8_t* qrow = sQ + s * C::kStageBytes + r * 128;
      const uint8_t* grow = qrow + C::kTileBytes;
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + tb * D;
      constexpr int kHalf = D / 2;  // output columns of this warp: col0 .. col0 + kHalf - 1
      const int col0 = hf * kHalf;
      // Sums over the whole row: each half adds its channels (|q|^2) and its
      // accumulator columns (|o|^2 before the 1/|q| scale, for the RMS norm); the
      // two halves of a row swap their partial sums through two spare TMEM columns.
      float av[GATE ? kHalf : 1];
      uint4 gr[GATE ? kHalf / 8 : 1];
      float scale = 1.f, rn = 1.f;
      if (qnorm || GATE) {
        float qq = 0.f, ss = 0.f;
        if (qnorm) {
          constexpr int kChunks = D / 16;  // 16-byte chunks of this half of the q row
#pragma unroll
          for (int c = 0; c < kChunks; ++c) {
            const int gc = hf * kChunks + c;  // chunk of the whole row (swizzled order: the sum needs none)
            const uint4 v = *reinterpret_cast<const uint4*>(qrow + (gc / 8) * (kTileM * 128) + (gc % 8) * 16);
            const __nv_bfloat162 e[4] = {bits_bf162(v.x), bits_bf162(v.y), bits_bf162(v.z), bits_bf162(v.w)};
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2) {
              const float2 f = __bfloat1622float2(e[k2]);
              qq = fmaf(f.x, f.x, fmaf(f.y, f.y, qq));
            }
          }
        }
        if constexpr (GATE) {
          // This half row of the gate into registers, so the stage can go back at once.
#pragma unroll
          for (int c = 0; c < kHalf / 8; ++c) {
            const int gcc = col0 / 8 + c;  // 8-column chunk of the whole row
            gr[c] = *reinterpret_cast<const uint4*>(grow + (gcc / 8) * (kTileM * 128) + (((gcc % 8) ^ (r & 7)) * 16));
          }
        }
        __syncwarp();
        if (lane == 0 && stage_read) mbar_arrive(&empty[s]);  // Q (and gate) tile read: release the stage
        if constexpr (GATE) {
#pragma unroll
          for (int cc = 0; cc < kHalf / 16; ++cc) {
            uint32_t v[16];
            tmem_ld16(taddr + col0 + cc * 16, v);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              av[cc * 16 + k] = __uint_as_float(v[k]);
              ss = fmaf(av[cc * 16 + k], av[cc * 16 + k], ss);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[tb]);  // accumulator read: the MMAs may reuse it
        }
        const uint32_t xaddr = tmem + ((uint32_t)(q * 32) << 16) + C::kXchgCol;
        tmem_st2(xaddr + 2 * hf, __float_as_uint(qq), __float_as_uint(ss));
        tmem_st_wait();
        tc_fence_before();
        if (!epi_sync()) { ok = false; break; }
        tc_fence_after();
        uint32_t pq, ps;
        tmem_ld2(xaddr + 2 * (1 - hf), pq, ps);
        tmem_ld_wait();
        if (qnorm) scale = rsqrtf(qq + __uint_as_float(pq) + a.l2_eps);
        if constexpr (GATE) rn = rsqrtf(scale * scale * (ss + __uint_as_float(ps)) / D + a.rms_eps);
      }
      const float hr = 0.5f * rn;
      // Output half row into registers: 16-byte chunk pair (2cc, 2cc+1) holds columns col0+16cc..+15.
      uint4 outs[kHalf / 8];
#pragma unroll
      for (int cc = 0; cc < kHalf / 16; ++cc) {
        float vf[16];
        if constexpr (GATE) {
#pragma unroll
          for (int k = 0; k < 16; ++k) vf[k] = av[cc * 16 + k];
        } else {
          uint32_t v[16];
          tmem_ld16(taddr + col0 + cc * 16, v);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 16; ++k) vf[k] = __uint_as_float(v[k]);
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float g8[8];
          if constexpr (GATE) {
            const uint4 gv = gr[2 * cc + half];
            const __nv_bfloat162 ge[4] = {bits_bf162(gv.x), bits_bf162(gv.y), bits_bf162(gv.z), bits_bf162(gv.w)};
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2) {  // rn * sigmoid(g) = hr + hr * tanh(g / 2), hr = rn / 2
              const float2 f = __bfloat1622float2(ge[k2]);
              g8[2 * k2] = fmaf(hr, tanh_approx(0.5f * f.x), hr);
              g8[2 * k2 + 1] = fmaf(hr, tanh_approx(0.5f * f.y), hr);
            }
          } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) g8[k] = 1.f;
          }
          uint32_t op[4];
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2)
            op[k2] = bf162_bits(__floats2bfloat162_rn(vf[half * 8 + 2 * k2] * scale * g8[2 * k2],
                                                      vf[half * 8 + 2 * k2 + 1] * scale * g8[2 * k2 + 1]));
          outs[2 * cc + half] = make_uint4(op[0], op[1], op[2], op[3]);
        }
      }
      if constexpr (!GATE) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[tb]);
      }
      // The staging buffer must have been read by the previous tile's TMA store.
      if (et == 0) bulk_wait_read0();
      if (!epi_sync()) { ok = false; break; }
      const bool partial = ti.nvalid < kTileM;
      const int h = ti.bh % a.H;
      if (!partial) {
        uint8_t* orow = sO + r * 128;
#pragma unroll
        for (int c = 0; c < kHalf / 8; ++c) {
          const int gcc = col0 / 8 + c;  // 8-column chunk of the whole row
          const int box = gcc / 8, pc = (gcc % 8) ^ (r & 7);
          *reinterpret_cast<uint4*>(orow + box * (kTileM * 128) + pc * 16) = outs[c];
        }
      } else if (r < ti.nvalid) {
        uint4* dst = reinterpret_cast<uint4*>(a.O + ((ti.tok0 + r) * a.Ht + h) * (long long)D) + col0 / 8;
#pragma unroll
        for (int c = 0; c < kHalf / 8; ++c) dst[c] = outs[c];
      }
      fence_proxy_async_smem();
      if (!epi_sync()) { ok = false; break; }
      if (et == 0 && !partial) {
#pragma unroll
        for (int box = 0; box < C::kBoxes; ++box)
          tma_store_3d(&mO, sO + box * (kTileM * 128), box * 64, h, (int)ti.tok0);
        bulk_commit();
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
    tmem_dealloc(tmem, C::kTmemAlloc);
  }
}

template <int D, bool GATE>
cudaError_t launch_dg(const Problem& p, const void* gate, void* O, cudaStream_t s) {
  using C = RoCfg<D, GATE>;
  RoArgs a{};
  a.B = p.B; a.H = p.H; a.T = p.T; a.U = p.U; a.c = p.c; a.J = p.J; a.Ht = p.Ht;
  a.flags = p.flags; a.l2_eps = p.l2_eps; a.rms_eps = p.rms_eps;
  a.Sf = p.Sf; a.Sr = p.Sr; a.O = static_cast<__nv_bfloat16*>(O);
  a.status = p.status; a.wait_ns = p.spin_limit;
  long long tiles_per_head = 0;
  for (int j = 0; j < p.J; ++j) {
    const int lo = std::max(p.c * j, 1), hi = std::min(p.c * (j + 1), p.T - 1);
    if (lo < hi) tiles_per_head += ((long long)(hi - lo) * p.U + kTileM - 1) / kTileM;
  }
  if (tiles_per_head == 0) return cudaSuccess;
  a.BH = p.B * p.H;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaError_t e;
  e = set_max_dynamic_smem(reinterpret_cast<const void*>(readout_tc_kernel<D, GATE>), C::kSmemBytes);
  if (e != cudaSuccess) return e;
  int per_sm = 1;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, readout_tc_kernel<D, GATE>, kThreads, C::kSmemBytes);
  if (per_sm < 1) per_sm = 1;
  const long long slots = (long long)sms * per_sm;
  a.nseg = (int)std::max<long long>(1, std::min<long long>(slots / a.BH, tiles_per_head));
  a.tiles_per_seg = (int)((tiles_per_head + a.nseg - 1) / a.nseg);
  const long long ncta = (long long)a.BH * a.nseg;

  // [B*T*U tokens, H, D] views of Q, gate and O from this problem's first head
  // (rows of Ht * D values): dims (d, h, token)
  const uint64_t D64 = D, H = p.H, NT = (uint64_t)p.B * p.T * p.U;
  uint64_t dims[3] = {D64, H, NT};
  uint64_t strides[2] = {D64 * 2, (uint64_t)p.Ht * D64 * 2};
  uint32_t box[3] = {64, 1, (uint32_t)kTileM};
  CUtensorMap mQ, mG, mO;
  if ((e = make_tmap_bf16(&mQ, p.Q, 3, dims, strides, box)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&mO, O, 3, dims, strides, box)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&mG, gate ? gate : p.Q, 3, dims, strides, box)) != cudaSuccess) return e;
  readout_tc_kernel<D, GATE><<<(unsigned)ncta, kThreads, C::kSmemBytes, s>>>(mQ, mG, mO, a);
  return cudaGetLastError();
}


template <int D>
cudaError_t launch_d(const Problem& p, const void* gate, void* O, cudaStream_t s) {
  return (p.flags & VDA_READOUT_NORM_GATE) ? launch_dg<D, true>(p, gate, O, s) : launch_dg<D, false>(p, gate, O, s);
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
