// Readout with FP8 queries on tcgen05 tensor cores (kind::f8f6f4): the query
// tensor arrives as e4m3 values with one float32 scale per (token, head),
// q = s_q * q8, so the kernel streams one byte per query channel instead of two
// (the pages run their large products in FP8 / MXFP8: Video DeltaNet summary,
// onedev.kr/papers/80, section "assumptions and limits"; VDN-H3 post, section
// "compared with existing methods"). The readout itself is that of the bf16
// kernel: query frame t of chunk j reads o = (S->_j + S<-_j) q (section "how it
// works"), anchor frames read zero.
//
// Per (b, h, chunk) the prologue forms S = S-> + S<- in fp32, takes a power of
// two 2^E that brings max |S| to at most 240 (inside e4m3's 448), and splits
// 2^E S into e4m3 hi + lo parts (S = 2^-E (hi + lo) to about 2^-8 relative)
// stored as K-major swizzled B operands. Per tile of 128 tokens
//   acc = Q8 hi^T + Q8 lo^T        (M = 128 tokens, N = d_v, K = d_k, fp32 in TMEM)
// and the epilogue writes o = s_q 2^-E acc as bf16. Persistent CTAs walk the
// same (head, token segment) tile lists as the bf16 readout.
// Warp roles: 0 = TMA producer, 1 = TMEM owner + MMA issuer, 2..9 = prologue
// and epilogue (two warps per TMEM lane quadrant, one per half of the output
// columns); full tiles leave through a staging tile and TMA stores.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <algorithm>

#include "internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace vda {

namespace {

constexpr int D = 128;
constexpr int kTileM = 128;
constexpr int kThreads = 320;  // TMA warp, MMA warp, eight epilogue warps
constexpr int kEpi = 256;
constexpr int kStages = 6;
constexpr int kTileBytes = kTileM * D;  // one e4m3 tile of 128 tokens (16 KB)
constexpr int kSBytes = D * D;          // one e4m3 image of S (16 KB)
constexpr int kSHiOff = 0, kSLoOff = kSBytes, kQOff = 2 * kSBytes;
constexpr int kOOff = kQOff + kStages * kTileBytes;  // bf16 output tile staged for the TMA store (32 KB)
constexpr int kOBox = kTileM * 128;                      // one 64-column box of it
constexpr int kScOff = kOOff + 2 * kOBox;               // per stage, the tile's 128 query scales
constexpr int kBarOff = kScOff + kStages * kTileM * 4;
constexpr int kSmemBytes = kBarOff + 256 + 1024;
// kind::f8f6f4: D f32, A and B e4m3, both K-major, M = 128, N = 128.
constexpr uint32_t kIdesc = (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(D >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
static_assert(kSmemBytes <= 232448, "more shared memory than a CTA may use");

struct Ro8Args {
  int B, H, T, U, c, J, Ht;
  const float* Sf;
  const float* Sr;
  const float* q_scale;  // [B, T*U, Ht] (advanced to this problem's first head)
  __nv_bfloat16* O;
  uint32_t* status;
  unsigned long long wait_ns;
  int BH, tiles_per_seg;
};

__device__ __forceinline__ void chunk_frames(const Ro8Args& a, int j, int& lo, int& hi) {
  lo = max(a.c * j, 1);
  hi = min(a.c * (j + 1), a.T - 1);
}
__device__ __forceinline__ int chunk_tiles(const Ro8Args& a, int j) {
  int lo, hi;
  chunk_frames(a, j, lo, hi);
  return lo < hi ? (int)(((long long)(hi - lo) * a.U + kTileM - 1) / kTileM) : 0;
}

struct Tile {
  int j;
  long long tok0;  // first token of the tile, flat over B*T*U
  int nvalid;
};

// The tiles of one (b, h) in order, one step at a time.
struct Iter {
  int j, local, n;
  __device__ __forceinline__ void start(const Ro8Args& a, int t) {
    j = 0;
    for (;; ++j) {
      n = chunk_tiles(a, j);
      if (t < n) break;
      t -= n;
    }
    local = t;
  }
  __device__ __forceinline__ void next(const Ro8Args& a) {
    if (++local < n) return;
    local = 0;
    do {
      n = chunk_tiles(a, ++j);
    } while (n == 0);
  }
  __device__ __forceinline__ Tile tile(const Ro8Args& a, int bh) const {
    Tile ti;
    ti.j = j;
    int lo, hi;
    chunk_frames(a, j, lo, hi);
    const long long first = (long long)lo * a.U + (long long)local * kTileM;
    ti.nvalid = (int)min((long long)kTileM, (long long)hi * a.U - first);
    ti.tok0 = (long long)(bh / a.H) * a.T * a.U + first;
    return ti;
  }
};

__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Two floats to two e4m3 values (round to nearest, saturating), low byte first.
__device__ __forceinline__ uint16_t to_e4m3x2(float lo, float hi) {
  return (uint16_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float2 from_e4m3x2(uint16_t v) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)v, __NV_E4M3);
  return __half22float2(__half2(h));
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

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  return sm100::bf162_bits(__floats2bfloat162_rn(a, b));
}

__global__ void __launch_bounds__(kThreads, 1)
    readout_fp8_tc_kernel(const __grid_constant__ CUtensorMap mQ, const __grid_constant__ CUtensorMap mO,
                          const Ro8Args a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint8_t* sHi = smem + kSHiOff;
  uint8_t* sLo = smem + kSLoOff;
  uint8_t* sQ = smem + kQOff;
  uint8_t* sO = smem + kOOff;
  float* sscale = reinterpret_cast<float*>(smem + kScOff);  // [kStages][kTileM]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* sready = tempty + 2;
  uint64_t* drain = sready + 1;
  uint64_t* epibar = drain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epibar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* sred = reinterpret_cast<float*>(tmem_slot + 4);  // [8] per-warp maxima
  static_assert((2 * kStages + 7) * 8 + 16 + 32 <= 256, "barrier block overflows its allowance");

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  int tiles_per_head = 0;
  for (int j = 0; j < a.J; ++j) tiles_per_head += chunk_tiles(a, j);
  const int my_bh = blockIdx.x % a.BH, seg = blockIdx.x / a.BH;
  const int t_begin = seg * a.tiles_per_seg;
  const int t_end = min(tiles_per_head, t_begin + a.tiles_per_seg);
  const int ntiles = t_begin < t_end ? t_end - t_begin : 0;
  const int h = my_bh % a.H;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1 + 32);  // TMA bytes + the 32 lanes' scale copies
      mbar_init(&empty[s], 1 + 8);  // MMA commit + the 8 epilogue warps (they read the scales)
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 8);
    }
    mbar_init(sready, 8);
    mbar_init(drain, 1);
    mbar_init(epibar, kEpi);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&mQ);
    prefetch_tmap(&mO);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  int issued = 0;

  if (warp == 0) {
    // Q tile by TMA (lane 0); the tile's query scales by 4-byte asynchronous
    // copies (all lanes, zero past the tile's last valid row), on the same barrier.
    Iter it;
    if (ntiles > 0) it.start(a, t_begin);
    for (int n = 0; n < ntiles; ++n) {
      if (n > 0) it.next(a);
      const int s = n % kStages;
      int good = 1;
      if (lane == 0) good = mbar_wait(&empty[s], ((n / kStages) & 1) ^ 1, abort_flag, a.status, a.wait_ns) ? 1 : 0;
      good = __shfl_sync(0xffffffffu, good, 0);
      if (!good) break;
      const Tile ti = it.tile(a, my_bh);
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], kTileBytes);
        tma_load_3d(sQ + s * kTileBytes, &mQ, &full[s], 0, h, (int)ti.tok0);
      }
#pragma unroll
      for (int j = 0; j < kTileM / 32; ++j) {
        const int row = j * 32 + lane;
        const bool in = row < ti.nvalid;
        const float* src = a.q_scale + (ti.tok0 + (in ? row : 0)) * a.Ht + h;
        cp_async_4(sscale + s * kTileM + row, src, in ? 4u : 0u);
      }
      cp_async_mbar_arrive_noinc(&full[s]);
      if (lane == 0) issued = n + 1;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int j_prev = -1, gi = 0;
      Iter it;
      if (ntiles > 0) it.start(a, t_begin);
      for (int n = 0; n < ntiles; ++n) {
        if (n > 0) it.next(a);
        if (it.j != j_prev) {
          if (!mbar_wait(sready, gi & 1, abort_flag, a.status, a.wait_ns)) break;
          ++gi;
          j_prev = it.j;
        }
        const int s = n % kStages, tb = n & 1;
        if (!mbar_wait(&full[s], (n / kStages) & 1, abort_flag, a.status, a.wait_ns)) break;
        if (!mbar_wait(&tempty[tb], ((n >> 1) & 1) ^ 1, abort_flag, a.status, a.wait_ns)) break;
        tc_fence_after();
        const uint32_t qb = smem_u32(sQ + s * kTileBytes), hb = smem_u32(sHi), lb = smem_u32(sLo);
        const uint32_t acc = tmem + tb * D;
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk) {  // 32 e4m3 values = 32 bytes per step
          const uint64_t dq = smem_desc_sw128(qb + kk * 32, 16, 1024);
          mma_f8(acc, dq, smem_desc_sw128(hb + kk * 32, 16, 1024), kIdesc, kk > 0 ? 1u : 0u);
          mma_f8(acc, dq, smem_desc_sw128(lb + kk * 32, 16, 1024), kIdesc, 1u);
        }
        mma_commit(&empty[s]);
        mma_commit(&tfull[tb]);
      }
      mma_commit(drain);
    }
  } else {
    const int et = threadIdx.x - 64;  // 0..255
    const int quad = warp % 4;
    const int hf = (warp - 2) / 4;    // output columns 64 hf .. 64 hf + 63
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    // Anchor frames 0 and T-1 read zero: this CTA's share of their rows (per batch
    // and anchor, U token rows of H * D values at a row stride of Ht * D).
    {
      const long long rw = (long long)a.H * D * 2 / 16, per16 = (long long)a.U * rw;
      const long long row16 = (long long)a.Ht * D * 2 / 16;
      const long long G = gridDim.x;
      const long long lo = per16 * blockIdx.x / G, hi = per16 * (blockIdx.x + 1) / G;
      for (int slab = 0; slab < 2 * a.B; ++slab) {
        const long long b = slab >> 1, f = (slab & 1) ? a.T - 1 : 0;
        uint4* base = reinterpret_cast<uint4*>(a.O + (b * a.T + f) * (long long)a.U * a.Ht * D);
        for (long long w = lo + et; w < hi; w += kEpi) base[(w / rw) * row16 + w % rw] = make_uint4(0, 0, 0, 0);
      }
    }
    uint32_t ephase = 0;
    auto epi_sync = [&]() -> bool {
      mbar_arrive(epibar);
      const bool ok = mbar_wait(epibar, ephase, abort_flag, a.status, a.wait_ns);
      ephase ^= 1;
      return ok;
    };
    int j_prev = -1;
    float inv_scale = 1.f;
    Iter it;
    if (ntiles > 0) it.start(a, t_begin);
    for (int n = 0; n < ntiles; ++n) {
      if (n > 0) it.next(a);
      const Tile ti = it.tile(a, my_bh);
      if (ti.j != j_prev) {
        // The previous chunk's MMAs are complete (its last accumulator was read
        // below) and the next MMA waits for `sready`: S may be rewritten.
        const long long off = ((long long)my_bh * a.J + ti.j) * (long long)D * D;
        const float4* pf = reinterpret_cast<const float4*>(a.Sf + off);
        const float4* pr = reinterpret_cast<const float4*>(a.Sr + off);
        // Loads issued in batches before they are used: one L2 round trip per
        // batch instead of per item.
        float mx = 0.f;
        constexpr int kMaxItems = D * D / 4 / kEpi, kMaxBatch = 4;
        static_assert(D * D / 4 % kEpi == 0 && kMaxItems % kMaxBatch == 0, "prologue items");
#pragma unroll
        for (int b0 = 0; b0 < kMaxItems; b0 += kMaxBatch) {
          float4 f[kMaxBatch], g[kMaxBatch];
#pragma unroll
          for (int bi = 0; bi < kMaxBatch; ++bi) {
            f[bi] = pf[et + (b0 + bi) * kEpi];
            g[bi] = pr[et + (b0 + bi) * kEpi];
          }
#pragma unroll
          for (int bi = 0; bi < kMaxBatch; ++bi)
            mx = fmaxf(mx, fmaxf(fmaxf(fabsf(f[bi].x + g[bi].x), fabsf(f[bi].y + g[bi].y)),
                                 fmaxf(fabsf(f[bi].z + g[bi].z), fabsf(f[bi].w + g[bi].w))));
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) sred[warp - 2] = mx;
        if (!epi_sync()) break;
#pragma unroll
        for (int w = 0; w < 8; ++w) mx = fmaxf(mx, sred[w]);
        // 2^E with max |S| 2^E <= 240 (an exact power of two; 0 when S is zero)
        const int E = mx > 0.f ? max(-100, min(100, (int)floorf(log2f(240.f / mx)))) : 0;
        const float sc = ldexpf(1.f, E);
        inv_scale = ldexpf(1.f, -E);
        // Row i, 16 consecutive k (column quads 4 c .. 4 c + 3) per work item,
        // the loads of two items issued before either is used.
        constexpr int kItems = D * (D / 16) / kEpi, kBatch = kItems < 2 ? kItems : 2;
        static_assert(D * (D / 16) % kEpi == 0 && kItems % kBatch == 0, "prologue items");
#pragma unroll
        for (int b0 = 0; b0 < kItems; b0 += kBatch) {
          float4 fb[kBatch][4], gb[kBatch][4];
#pragma unroll
          for (int bi = 0; bi < kBatch; ++bi) {
            const int e = et + (b0 + bi) * kEpi, c16 = e / D, i = e % D;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              fb[bi][q] = pf[(4 * c16 + q) * D + i];
              gb[bi][q] = pr[(4 * c16 + q) * D + i];
            }
          }
#pragma unroll
          for (int bi = 0; bi < kBatch; ++bi) {
            const int e = et + (b0 + bi) * kEpi, c16 = e / D, i = e % D;
            float x[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float4 f = fb[bi][q], g = gb[bi][q];
              x[4 * q] = (f.x + g.x) * sc;
              x[4 * q + 1] = (f.y + g.y) * sc;
              x[4 * q + 2] = (f.z + g.z) * sc;
              x[4 * q + 3] = (f.w + g.w) * sc;
            }
            // Pairs packed into 32-bit words by shifts (no type-punned stores).
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const uint16_t hh = to_e4m3x2(x[2 * q], x[2 * q + 1]);
              const float2 hf = from_e4m3x2(hh);
              const uint16_t ll = to_e4m3x2(x[2 * q] - hf.x, x[2 * q + 1] - hf.y);
              if (q & 1) {
                hw[q >> 1] |= (uint32_t)hh << 16;
                lw[q >> 1] |= (uint32_t)ll << 16;
              } else {
                hw[q >> 1] = hh;
                lw[q >> 1] = ll;
              }
            }
            const uint4 hv = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            const uint4 lv = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            const int boff = i * 128 + ((c16 ^ (i & 7)) << 4);
            *reinterpret_cast<uint4*>(sHi + boff) = hv;
            *reinterpret_cast<uint4*>(sLo + boff) = lv;
          }
        }
        fence_proxy_async_smem();
        if (!epi_sync()) break;
        if (lane == 0) mbar_arrive(sready);
        j_prev = ti.j;
      }
      const int tb = n & 1;
      const bool got = mbar_wait(&tfull[tb], (n >> 1) & 1, abort_flag, a.status, a.wait_ns);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const bool live = r < ti.nvalid;
      const long long tok = ti.tok0 + (live ? r : 0);
      // The stage's scales have landed once its barrier completes; read this row's
      // and give the stage back (with the MMA commit, the ninth arrival).
      const int s = n % kStages;
      const bool sgot = mbar_wait(&full[s], (n / kStages) & 1, abort_flag, a.status, a.wait_ns);
      if (!__all_sync(0xffffffffu, sgot)) break;
      const float scale = sscale[s * kTileM + r] * inv_scale;
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      // This warp's half row: 64 columns as eight 16-byte chunks of bf16.
      uint4 outs[8];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t v[16];
        tmem_ld16(tmem + lane_off + tb * D + hf * 64 + c * 16, v);
        tmem_ld_wait();
        uint32_t w[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) w[k] = pack_bf16(__uint_as_float(v[2 * k]) * scale, __uint_as_float(v[2 * k + 1]) * scale);
        outs[2 * c] = make_uint4(w[0], w[1], w[2], w[3]);
        outs[2 * c + 1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[tb]);  // accumulator read: the MMAs may reuse it
      const bool partial = ti.nvalid < kTileM;
      // The staging tile must have been read by the previous tile's TMA store.
      if (et == 0) bulk_wait_read0();
      if (!epi_sync()) break;
      if (!partial) {
        uint8_t* orow = sO + hf * kOBox + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(orow + ((c ^ (r & 7)) << 4)) = outs[c];
      } else if (live) {
        uint4* dst = reinterpret_cast<uint4*>(a.O + (tok * a.Ht + h) * (long long)D) + hf * 8;
#pragma unroll
        for (int c = 0; c < 8; ++c) dst[c] = outs[c];
      }
      fence_proxy_async_smem();
      if (!epi_sync()) break;
      if (et == 0 && !partial) {
        tma_store_3d(&mO, sO, 0, h, (int)ti.tok0);
        tma_store_3d(&mO, sO + kOBox, 64, h, (int)ti.tok0);
        bulk_commit();
      }
    }
    if (et == 0) bulk_wait0();  // every output write done before the CTA retires
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
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

bool readout_fp8_tc_supported(const Problem& p) {
  return p.D == D && (long long)p.B * p.T * p.U < (1LL << 31) && !(p.flags & (VDA_PREP_CONV | VDA_READOUT_NORM_GATE));
}

cudaError_t launch_readout_fp8_tc(const Problem& p, const void* Q8, const float* q_scale, void* O, cudaStream_t s) {
  Ro8Args a{};
  a.B = p.B; a.H = p.H; a.T = p.T; a.U = p.U; a.c = p.c; a.J = p.J; a.Ht = p.Ht;
  a.Sf = p.Sf; a.Sr = p.Sr; a.q_scale = q_scale;
  a.O = static_cast<__nv_bfloat16*>(O);
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
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(readout_fp8_tc_kernel), kSmemBytes);
  if (e != cudaSuccess) return e;
  const long long nseg = std::max<long long>(1, std::min<long long>(sms / a.BH, tiles_per_head));
  a.tiles_per_seg = (int)((tiles_per_head + nseg - 1) / nseg);
  const long long ncta = (long long)a.BH * nseg;
  // [B*T*U tokens, H, D] e4m3 view of Q from this problem's first head (rows of Ht * D bytes)
  const uint64_t dims[3] = {(uint64_t)D, (uint64_t)p.H, (uint64_t)p.B * p.T * p.U};
  const uint64_t strides[2] = {(uint64_t)D, (uint64_t)p.Ht * D};
  const uint32_t box[3] = {(uint32_t)D, 1u, (uint32_t)kTileM};
  CUtensorMap mQ, mO;
  if ((e = make_tmap_typed(&mQ, CU_TENSOR_MAP_DATA_TYPE_UINT8, Q8, 3, dims, strides, box,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != cudaSuccess)
    return e;
  // O: bf16 [B*T*U tokens, H, D] from this problem's first head, 64-column boxes.
  const uint64_t ostrides[2] = {(uint64_t)D * 2, (uint64_t)p.Ht * D * 2};
  const uint32_t obox[3] = {64u, 1u, (uint32_t)kTileM};
  if ((e = make_tmap_bf16(&mO, O, 3, dims, ostrides, obox)) != cudaSuccess) return e;
  readout_fp8_tc_kernel<<<(unsigned)ncta, kThreads, kSmemBytes, s>>>(mQ, mO, a);
  return cudaGetLastError();
}

}  // namespace vda
