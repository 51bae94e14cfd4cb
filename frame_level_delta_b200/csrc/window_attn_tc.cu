// Softmax branch of the hybrid layer on tcgen05 tensor cores: attention over
// the +-1-chunk window and the two boundary anchor frames, with the branch's
// sigmoid output gate fused into the epilogue (Video DeltaNet summary,
// onedev.kr/papers/80, section "how it works": each query chunk attends
// densely to the chunks j-1..j+1 and to the first and last frame, and the
// anchor frames attend to every frame; section "how it differs": the softmax
// readout has its own content-dependent sigmoid gate; VDN-H3 post, section
// "hybrid attention structure": chunks of five latent frames and the four-way
// anchor links).
//
// Query groups: the non-anchor frames of chunk j (j = floor(t / c)) share one
// key set, frames max(0, c(j-1)) .. min(T-1, c(j+2)-1) plus frames 0 and T-1,
// i.e. at most three contiguous token ranges; the queries of frame 0 and of
// frame T-1 see every token. One CTA takes one tile of 128 queries of one group
// (tiles never straddle a group; the last tile of a group is ragged) and walks
// the group's keys in blocks of 128 tokens (a block never straddles a range;
// the last block of a range is masked per column).
//
// Per key block i:  S_i = Q K_i^T  (M = 128 queries, N = 128 keys, K = d) into
// one of two TMEM buffers; four softmax warps (one thread per query row) read
// S_i, keep the running row maximum m (log2 domain, logits scaled by
// log2(e)/sqrt(d)) and sum l, and write P_i = 2^(s - m) as bf16 into one of two
// TMEM operand buffers; then  O += P_i V_i  (A = P_i from TMEM, B = V_i from
// shared memory, N = d) accumulates in TMEM. The MMA of S_{i+1} runs while the
// softmax works on S_i. O is rescaled only when a row's maximum grows by more
// than 2^8 over the value its P entries were taken against, and then only after
// the previous P V product has completed; smaller growth leaves P entries up to
// 2^8, well inside bf16 and fp32. The epilogue divides by l, applies
// sigmoid(g^S) and writes bf16 rows.
//
// Warp roles: 0 = TMA producer (Q once; K and V blocks through separate
// three-stage rings), 1 = TMEM owner and MMA issuer, 2..5 = softmax and
// epilogue (warp w reads TMEM lanes 32 (w % 4) ..).
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace vda {

namespace {

constexpr int kTile = 128;     // queries per tile, keys per block
constexpr int kThreads = 192;  // TMA warp, MMA warp, four softmax warps
constexpr int kStages = 3;     // K blocks in flight; V blocks in flight

template <int D>
struct WaCfg {
  static constexpr int kAtoms = D / 64;               // 64-channel boxes per token tile
  static constexpr int kTileBytes = kTile * D * 2;    // one bf16 tile of 128 tokens
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kTileBytes;
  static constexpr int kVOff = kKOff + kStages * kTileBytes;
  static constexpr int kBarOff = kVOff + kStages * kTileBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;  // + room to align the base to 1024 bytes
  // TMEM columns: S0 | S1 (128 fp32 each) | P0 | P1 (64 packed bf16 pairs each) | O (D fp32)
  static constexpr uint32_t kS0 = 0, kS1 = 128, kP0 = 256, kP1 = 320, kO = 384;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kIdescS = sm100::idesc_bf16_f32(128, 128, false, false);  // Q, K both K-major
  static constexpr uint32_t kIdescO = sm100::idesc_bf16_f32(128, D, false, true);     // P (TMEM), V MN-major
  static_assert(kSmemBytes <= 232448, "more shared memory than a CTA may use");
  static_assert(kO + D <= kTmemCols, "TMEM overflow");
};

struct WaArgs {
  int B, H, T, U, c, J;
  int Ht;  // heads per token row of Q, K, V, gate, O (pointers advanced to this problem's first head)
  float sl;  // log2(e) / sqrt(d): logits in the log2 domain
  __nv_bfloat16* O;
  const __nv_bfloat16* gate;  // nullable: no gate
  uint32_t* status;
  unsigned long long wait_ns;
  int BH;
  int tiles_per_head;
};

// Query group g of one (b, h): g = 0: anchor frame 0; g = 1: anchor frame T-1;
// g = 2 + j: the non-anchor frames of chunk j. Token indices are within the
// batch item (t * U + u).
struct Group {
  int q_lo, q_hi;  // query tokens [q_lo, q_hi)
  int nr;          // key ranges
  int ra[3], rb[3];
};

__device__ __forceinline__ Group group_of(const WaArgs& a, int g) {
  Group G;
  const int TU = a.T * a.U;
  if (g < 2) {
    const int f = g == 0 ? 0 : a.T - 1;
    G.q_lo = f * a.U;
    G.q_hi = G.q_lo + a.U;
    G.nr = 1;
    G.ra[0] = 0;
    G.rb[0] = TU;
    return G;
  }
  const int j = g - 2;
  const int t_lo = max(a.c * j, 1), t_hi = min(a.c * (j + 1), a.T - 1);
  G.q_lo = t_lo * a.U;
  G.q_hi = max(t_lo, t_hi) * a.U;
  const int w_lo = max(0, a.c * (j - 1)), w_hi = min(a.T - 1, a.c * (j + 2) - 1);  // window frames, inclusive
  // Ranges in increasing token order, adjacent ones merged.
  int n = 0;
  if (w_lo > 0) {
    G.ra[n] = 0;
    G.rb[n] = a.U;
    ++n;
  }
  if (n > 0 && G.rb[n - 1] == w_lo * a.U) {
    G.rb[n - 1] = (w_hi + 1) * a.U;
  } else {
    G.ra[n] = w_lo * a.U;
    G.rb[n] = (w_hi + 1) * a.U;
    ++n;
  }
  if (w_hi < a.T - 1) {
    if (G.rb[n - 1] == (a.T - 1) * a.U) {
      G.rb[n - 1] = TU;
    } else {
      G.ra[n] = (a.T - 1) * a.U;
      G.rb[n] = TU;
      ++n;
    }
  }
  G.nr = n;
  return G;
}

__device__ __forceinline__ int group_tiles(const Group& G) { return (G.q_hi - G.q_lo + kTile - 1) / kTile; }

// Tile x of one head's list (anchor tiles first: they carry the most keys).
__device__ __forceinline__ void tile_of(const WaArgs& a, int x, Group& G, int& q0, int& nq) {
  for (int g = 0;; ++g) {
    G = group_of(a, g);
    const int n = group_tiles(G);
    if (x < n) {
      q0 = G.q_lo + x * kTile;
      nq = min(kTile, G.q_hi - q0);
      return;
    }
    x -= n;
  }
}

// Walk of a group's key blocks: range r, first key kb, valid keys in the block.
struct KeyIter {
  int r, kb;
  __device__ __forceinline__ void start(const Group& G) {
    r = 0;
    kb = G.ra[0];
  }
  __device__ __forceinline__ int valid(const Group& G) const { return min(kTile, G.rb[r] - kb); }
  __device__ __forceinline__ void next(const Group& G) {
    kb += kTile;
    if (kb >= G.rb[r] && r + 1 < G.nr) {
      ++r;
      kb = G.ra[r];
    }
  }
};

__device__ __forceinline__ int key_blocks(const Group& G) {
  int n = 0;
  for (int r = 0; r < G.nr; ++r) n += (G.rb[r] - G.ra[r] + kTile - 1) / kTile;
  return n;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// The hardware's approximate tanh: sigmoid(x) = (1 + tanh(x / 2)) / 2.
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  return sm100::bf162_bits(__floats2bfloat162_rn(a, b));
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    window_attn_tc_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mK,
                          const __grid_constant__ CUtensorMap mV, const WaArgs a) {
  using C = WaCfg<D>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint8_t* sQ = smem + C::kQOff;
  uint8_t* sK = smem + C::kKOff;
  uint8_t* sV = smem + C::kVOff;
  uint64_t* qfull = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* kfull = qfull + 1;
  uint64_t* kempty = kfull + kStages;
  uint64_t* vfull = kempty + kStages;
  uint64_t* vempty = vfull + kStages;
  uint64_t* sfull = vempty + kStages;  // [2] S_i in TMEM
  uint64_t* sempty = sfull + 2;        // [2] S_i read by the softmax warps
  uint64_t* pfull = sempty + 2;        // [2] P_i written (and O rescaled) by the softmax warps
  uint64_t* pvdone = pfull + 2;        // [2] O += P_i V_i complete
  uint64_t* drain = pvdone + 2;        // every MMA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  static_assert((1 + 4 * kStages + 9) * 8 + 8 <= 256, "barrier block overflows its allowance");

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int bh = blockIdx.x % a.BH, x = blockIdx.x / a.BH;
  const int b = bh / a.H, h = bh % a.H;
  Group G;
  int q0, nq;
  tile_of(a, x, G, q0, nq);
  const int nblk = key_blocks(G);
  const int tok_base = b * a.T * a.U;  // flat token index of this batch item's first token

  if (warp == 0 && lane == 0) {
    mbar_init(qfull, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kempty[s], 1);
      mbar_init(&vfull[s], 1);
      mbar_init(&vempty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&sempty[i], 4);
      mbar_init(&pfull[i], 4);
      mbar_init(&pvdone[i], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&mQ);
    prefetch_tmap(&mK);
    prefetch_tmap(&mV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  int kissued = 0, vissued = 0;  // producer only

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(qfull, C::kTileBytes);
#pragma unroll
      for (int at = 0; at < C::kAtoms; ++at)
        tma_load_3d(sQ + at * (kTile * 128), &mQ, qfull, at * 64, h, tok_base + q0);
      // K_i then V_i, each into its own ring. K_i waits for S_{i-3} and V_i for
      // P_{i-3} V_{i-3}; neither product waits on a later copy, so the order
      // cannot deadlock, and both blocks are in flight about three blocks ahead.
      KeyIter it;
      it.start(G);
      for (int i = 0; i < nblk; ++i) {
        const int s = i % kStages;
        const uint32_t par = ((i / kStages) & 1) ^ 1;
        if (!mbar_wait(&kempty[s], par, abort_flag, a.status, a.wait_ns)) break;
        mbar_arrive_expect_tx(&kfull[s], C::kTileBytes);
#pragma unroll
        for (int at = 0; at < C::kAtoms; ++at)
          tma_load_3d(sK + s * C::kTileBytes + at * (kTile * 128), &mK, &kfull[s], at * 64, h, tok_base + it.kb);
        kissued = i + 1;
        if (!mbar_wait(&vempty[s], par, abort_flag, a.status, a.wait_ns)) break;
        mbar_arrive_expect_tx(&vfull[s], C::kTileBytes);
#pragma unroll
        for (int at = 0; at < C::kAtoms; ++at)
          tma_load_3d(sV + s * C::kTileBytes + at * (kTile * 128), &mV, &vfull[s], at * 64, h, tok_base + it.kb);
        vissued = i + 1;
        it.next(G);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(qfull, 0, abort_flag, a.status, a.wait_ns);
      const uint32_t qb = smem_u32(sQ);
      // O += P_j V_j for block j.
      auto issue_pv = [&](int j) -> bool {
        const int vs = j % kStages;
        if (!mbar_wait(&pfull[j & 1], (j >> 1) & 1, abort_flag, a.status, a.wait_ns)) return false;
        if (!mbar_wait(&vfull[vs], (j / kStages) & 1, abort_flag, a.status, a.wait_ns)) return false;
        tc_fence_after();
        const uint32_t vb = smem_u32(sV + vs * C::kTileBytes);
        const uint32_t pa = tmem + ((j & 1) ? C::kP1 : C::kP0);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          const uint64_t dv = smem_desc_sw128(vb + kk * 2048, kTile * 128, 1024);
          mma_f16_ts(tmem + C::kO, pa + kk * 8, dv, C::kIdescO, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&vempty[vs]);
        mma_commit(&pvdone[j & 1]);
        return true;
      };
      for (int i = 0; i < nblk && ok; ++i) {
        const int s = i % kStages;
        if (!mbar_wait(&kfull[s], (i / kStages) & 1, abort_flag, a.status, a.wait_ns)) { ok = false; break; }
        if (!mbar_wait(&sempty[i & 1], ((i >> 1) & 1) ^ 1, abort_flag, a.status, a.wait_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kb = smem_u32(sK + s * C::kTileBytes);
        const uint32_t sd = tmem + ((i & 1) ? C::kS1 : C::kS0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int at = kk / 4;
          const uint32_t koff = (kk % 4) * 32;
          const uint64_t dq = smem_desc_sw128(qb + at * (kTile * 128) + koff, 16, 1024);
          const uint64_t dk = smem_desc_sw128(kb + at * (kTile * 128) + koff, 16, 1024);
          mma_f16(sd, dq, dk, C::kIdescS, kk > 0 ? 1u : 0u);
        }
        mma_commit(&kempty[s]);
        mma_commit(&sfull[i & 1]);
        if (i > 0 && !issue_pv(i - 1)) { ok = false; break; }
      }
      if (ok && nblk > 0) issue_pv(nblk - 1);
      mma_commit(drain);  // completes once every MMA issued above has finished
    }
  } else {
    // ---------------- softmax and epilogue: one query row per thread
    const int quad = warp % 4;
    const int r = quad * 32 + lane;  // tile row == TMEM lane
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    // Every lane waits; the warp goes on only if all of them saw the phase, so
    // the warp-wide TMEM accesses below never run with lanes missing.
    auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      const bool r = mbar_wait(bar, parity, abort_flag, a.status, a.wait_ns);
      return __all_sync(0xffffffffu, r);
    };
    KeyIter it;
    it.start(G);
    for (int i = 0; i < nblk; ++i) {
      const int valid = it.valid(G);
      it.next(G);
      if (!warp_wait(&sfull[i & 1], (i >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      float s[kTile];
      {
        const uint32_t sa = tmem + lane_off + ((i & 1) ? C::kS1 : C::kS0);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t v[32];
          tmem_ld32(sa + c4 * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) s[c4 * 32 + k] = __uint_as_float(v[k]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sempty[i & 1]);  // S_i is in registers: the buffer may take S_{i+2}
      // Columns past the block's keys are masked; the row maximum of the raw
      // logits over eight independent chains, then taken to the log2 domain
      // (sl > 0, and rounding is monotone: the same value as the maximum of the
      // scaled logits).
      if (valid < kTile) {
#pragma unroll
        for (int k = 0; k < kTile; ++k)
          if (k >= valid) s[k] = -INFINITY;
      }
      float mx[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) mx[q] = s[q];
#pragma unroll
      for (int k = 8; k < kTile; ++k) mx[k & 7] = fmaxf(mx[k & 7], s[k]);
#pragma unroll
      for (int q = 0; q < 4; ++q) mx[q] = fmaxf(mx[q], mx[q + 4]);
      const float mb = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * a.sl;
      // Rescale when the maximum grows by more than 2^8 over the reference the
      // earlier P entries used (the whole warp takes part in the TMEM access).
      const bool grow = i > 0 && mb > m_run + 8.f;
      if (i == 0) m_run = mb;
      if (__any_sync(0xffffffffu, grow)) {
        // O must hold every earlier product: P_{i-1} V_{i-1} complete.
        if (!warp_wait(&pvdone[(i - 1) & 1], ((i - 1) >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const float f = grow ? ex2_approx(m_run - mb) : 1.f;
        const uint32_t oa = tmem + lane_off + C::kO;
#pragma unroll
        for (int c4 = 0; c4 < D / 32; ++c4) {
          uint32_t v[32];
          tmem_ld32(oa + c4 * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * f);
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t w[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) w[k] = v[q * 16 + k];
            tmem_st16(oa + c4 * 32 + q * 16, w);
          }
        }
        if (grow) {
          l_run *= f;
          m_run = mb;
        }
      }
      // P_i goes where P_{i-2} was: that product must be complete.
      if (i >= 2 && !warp_wait(&pvdone[i & 1], ((i - 2) >> 1) & 1)) { ok = false; break; }
      tc_fence_after();
      // p = 2^(s sl - m): one packed FMA per pair of logits; the row sum over
      // four independent packed chains.
      const uint32_t pa = tmem + lane_off + ((i & 1) ? C::kP1 : C::kP0);
      const float2 sl2 = make_float2(a.sl, a.sl), nm2 = make_float2(-m_run, -m_run);
      float2 ls2[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) ls2[q] = make_float2(0.f, 0.f);
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t w[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float2 x = __ffma2_rn(make_float2(s[c4 * 32 + 2 * k], s[c4 * 32 + 2 * k + 1]), sl2, nm2);
          const float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);
          ls2[k & 3] = __fadd2_rn(ls2[k & 3], make_float2(p0, p1));
          w[k] = pack_bf16(p0, p1);
        }
        tmem_st16(pa + c4 * 16, w);
      }
      l_run += ((ls2[0].x + ls2[0].y) + (ls2[1].x + ls2[1].y)) + ((ls2[2].x + ls2[2].y) + (ls2[3].x + ls2[3].y));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pfull[i & 1]);
    }
    // ---------------- epilogue: O / l, gate, bf16 row to global memory
    if (ok && nblk > 0 && warp_wait(&pvdone[(nblk - 1) & 1], ((nblk - 1) >> 1) & 1)) {
      tc_fence_after();
      const float inv = 1.f / l_run;
      const bool live = r < nq;
      const long long row = ((long long)tok_base + q0 + (live ? r : 0)) * a.Ht + h;
      uint4* dst = reinterpret_cast<uint4*>(a.O + row * D);
      const uint4* gsrc = a.gate ? reinterpret_cast<const uint4*>(a.gate + row * D) : nullptr;
      const uint32_t oa = tmem + lane_off + C::kO;
#pragma unroll
      for (int c4 = 0; c4 < D / 32; ++c4) {
        uint32_t v[32];
        tmem_ld32(oa + c4 * 32, v);
        tmem_ld_wait();
        if (!live) continue;
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          float g8[8];
          if (gsrc) {
            const uint4 gv = gsrc[c4 * 4 + q8];
            const __nv_bfloat162 ge[4] = {sm100::bits_bf162(gv.x), sm100::bits_bf162(gv.y), sm100::bits_bf162(gv.z),
                                          sm100::bits_bf162(gv.w)};
#pragma unroll
            for (int k2 = 0; k2 < 4; ++k2) {
              const float2 f = __bfloat1622float2(ge[k2]);
              g8[2 * k2] = fmaf(0.5f, tanh_approx(0.5f * f.x), 0.5f);
              g8[2 * k2 + 1] = fmaf(0.5f, tanh_approx(0.5f * f.y), 0.5f);
            }
          } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) g8[k] = 1.f;
          }
          uint32_t op[4];
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2)
            op[k2] = pack_bf16(__uint_as_float(v[q8 * 8 + 2 * k2]) * inv * g8[2 * k2],
                               __uint_as_float(v[q8 * 8 + 2 * k2 + 1]) * inv * g8[2 * k2 + 1]);
          dst[c4 * 4 + q8] = make_uint4(op[0], op[1], op[2], op[3]);
        }
      }
    }
  }

  // ---------------- teardown
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) {
    // Let every issued copy land before the CTA's shared memory is released.
    mbar_wait(qfull, 0, nullptr, a.status, a.wait_ns);
    for (int s = 0; s < kStages; ++s) {
      int last = -1;
      for (int i = s; i < kissued; i += kStages) last = i;
      if (last >= 0) mbar_wait(&kfull[s], (last / kStages) & 1, nullptr, a.status, a.wait_ns);
      last = -1;
      for (int i = s; i < vissued; i += kStages) last = i;
      if (last >= 0) mbar_wait(&vfull[s], (last / kStages) & 1, nullptr, a.status, a.wait_ns);
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
cudaError_t launch_d(const Problem& p, const void* Q, const void* K, const void* V, const void* gate, void* O,
                     cudaStream_t s) {
  using C = WaCfg<D>;
  WaArgs a{};
  a.B = p.B; a.H = p.H; a.T = p.T; a.U = p.U; a.c = p.c; a.J = p.J; a.Ht = p.Ht;
  a.sl = 1.4426950408889634f / sqrtf((float)D);
  a.O = static_cast<__nv_bfloat16*>(O);
  a.gate = static_cast<const __nv_bfloat16*>(gate);
  a.status = p.status;
  a.wait_ns = p.spin_limit;
  a.BH = p.B * p.H;
  long long tiles = 2LL * ((p.U + kTile - 1) / kTile);  // the two anchor frames
  for (int j = 0; j < p.J; ++j) {
    const int lo = std::max(p.c * j, 1), hi = std::min(p.c * (j + 1), p.T - 1);
    if (lo < hi) tiles += ((long long)(hi - lo) * p.U + kTile - 1) / kTile;
  }
  a.tiles_per_head = (int)tiles;
  const long long grid = tiles * a.BH;
  if (grid == 0) return cudaSuccess;
  if (grid >= (1LL << 31)) return cudaErrorInvalidConfiguration;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(window_attn_tc_kernel<D>), C::kSmemBytes);
  if (e != cudaSuccess) return e;
  // [B*T*U tokens, H, D] views from this problem's first head (rows of Ht * D values): dims (d, h, token)
  const uint64_t NT = (uint64_t)p.B * p.T * p.U;
  uint64_t dims[3] = {(uint64_t)D, (uint64_t)p.H, NT};
  uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)p.Ht * D * 2};
  uint32_t box[3] = {64, 1, (uint32_t)kTile};
  CUtensorMap mQ, mK, mV;
  if ((e = make_tmap_bf16(&mQ, Q, 3, dims, strides, box)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&mK, K, 3, dims, strides, box)) != cudaSuccess) return e;
  if ((e = make_tmap_bf16(&mV, V, 3, dims, strides, box)) != cudaSuccess) return e;
  window_attn_tc_kernel<D><<<(unsigned)grid, kThreads, C::kSmemBytes, s>>>(mQ, mK, mV, a);
  return cudaGetLastError();
}

}  // namespace

bool window_attn_tc_supported(const Problem& p) {
  return p.bf16 && (p.D == 64 || p.D == 128) && (long long)p.B * p.T * p.U < (1LL << 31);
}

cudaError_t launch_window_attn_tc(const Problem& p, const void* Q, const void* K, const void* V, const void* gate,
                                  void* O, cudaStream_t s) {
  if (p.D == 128) return launch_d<128>(p, Q, K, V, gate, O, s);
  if (p.D == 64) return launch_d<64>(p, Q, K, V, gate, O, s);
  return cudaErrorNotSupported;
}

}  // namespace vda
