// Chunk composition for the bidirectional scan (Video DeltaNet summary,
// onedev.kr/papers/80, section "how to use", kernel notes: the frame maps of a
// VAE chunk compose into S_out = S_in M_chunk + J_chunk, and the shorter chunk
// sequence is scanned in both directions).
//
// One CTA per (chunk m, direction, b*h). The forward direction composes the
// chunk's non-anchor frames in increasing order, the reverse direction in
// decreasing order (the reverse scan absorbs later frames first):
//   (MM, JJ) <- (M_f0, C_f0);  for each next frame f: (MM, JJ) <- (MM M_f, JJ M_f + C_f).
// Only the chunks the readout states need are composed: forward m = 0..J-3,
// reverse m = 2..J-1; an empty chunk gets the identity map (I, 0).
// Both products use the split operands of the tensor-core scan: MM and JJ as
// bf16 hi/lo K-major images, M_f as the hi/lo image the solve wrote, three
// products per pair, fp32 accumulation in TMEM (columns 0..127: MM M_f,
// 128..255: JJ M_f). The final MM is stored as a hi/lo operand image and JJ as
// fp32, exactly the operands of the chunk-level scan.
#include <cuda_bf16.h>

#include "internal.h"
#include "sm100.cuh"

namespace vda {

namespace {

constexpr int D = 128;
constexpr int kThreads = 128;
constexpr int kImg = D * D * 2;   // one bf16 operand image
constexpr int kPair = 2 * kImg;   // hi + lo
constexpr int kMMOff = 0, kJJOff = kPair, kMfOff = 2 * kPair, kBarOff = 3 * kPair;
constexpr int kSmemBytes = kBarOff + 64 + 1024;
constexpr uint32_t kIdesc = sm100::idesc_bf16_f32(128, 128, false, true);  // A K-major, B MN-major

struct ComposeArgs {
  int H, T, c, J;
  const uint8_t* Mi;  // per-frame M hi/lo images [B*H][T-1]
  const float* C;     // per-frame C [B*H][T-1][D][D]
  uint8_t* CMi;       // [B*H][2][J] hi/lo images
  float* CC;          // [B*H][2][J][D][D]
  uint32_t* status;
  unsigned long long wait_ns;
};

__device__ __forceinline__ uint32_t img_off(int row, int col) {
  const int atom = col >> 6, cc = col & 63;
  return (uint32_t)(atom * D * 128 + row * 128 + ((((cc >> 3) ^ (row & 7))) << 4) + (cc & 7) * 2);
}

__device__ __forceinline__ void split8(const float* x, uint4& hi, uint4& lo) {
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&hi);
  __nv_bfloat162* l = reinterpret_cast<__nv_bfloat162*>(&lo);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __nv_bfloat162 hh = __floats2bfloat162_rn(x[2 * q], x[2 * q + 1]);
    const float2 hf = __bfloat1622float2(hh);
    h[q] = hh;
    l[q] = __floats2bfloat162_rn(x[2 * q] - hf.x, x[2 * q + 1] - hf.y);
  }
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          sm100::smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(sm100::smem_u32(bar))
      : "memory");
}

// Store a split row chunk (8 values at columns col..col+7 of row `row`) into a hi/lo image pair.
__device__ __forceinline__ void put8(uint8_t* pair, int row, int col, const float* x) {
  uint4 hi, lo;
  split8(x, hi, lo);
  const uint32_t o = img_off(row, col);
  *reinterpret_cast<uint4*>(pair + o) = hi;
  *reinterpret_cast<uint4*>(pair + kImg + o) = lo;
}

__global__ void __launch_bounds__(kThreads, 1) compose_tc_kernel(const ComposeArgs a) {
  using namespace sm100;
  const int m = blockIdx.x, dir = blockIdx.y, bh = blockIdx.z;
  const int c = a.c, T = a.T, J = a.J;
  if (dir == 0 ? (m > J - 3) : (m < 2)) return;  // map not needed by any readout state
  const int lo = dir == 0 ? max(1, c * m) : c * m;
  const int hi = dir == 0 ? c * (m + 1) - 1 : min(c * (m + 1) - 1, T - 2);
  const int nf = hi >= lo ? hi - lo + 1 : 0;
  auto frame = [&](int k) { return dir == 0 ? lo + k : hi - k; };
  const long long slots = (long long)bh * (T - 1);
  const long long oc = ((long long)bh * 2 + dir) * J + m;  // output chunk index
  uint8_t* out_img = a.CMi + oc * kPair;
  float* out_c = a.CC + oc * (long long)D * D;
  const int i = threadIdx.x;  // matrix row == TMEM lane
  const int warp = threadIdx.x / 32;

  if (nf <= 1) {
    // Identity map for an empty chunk; a one-frame chunk is that frame's map.
    const float4* csrc = nf == 1 ? reinterpret_cast<const float4*>(a.C + (slots + frame(0)) * (long long)D * D) : nullptr;
    const uint8_t* msrc = nf == 1 ? a.Mi + (slots + frame(0)) * (long long)kPair : nullptr;
    for (int c8 = 0; c8 < D / 8; ++c8) {
      const uint32_t o = img_off(i, c8 * 8);
      if (nf == 1) {
        *reinterpret_cast<uint4*>(out_img + o) = *reinterpret_cast<const uint4*>(msrc + o);
        *reinterpret_cast<uint4*>(out_img + kImg + o) = *reinterpret_cast<const uint4*>(msrc + kImg + o);
      } else {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = (c8 * 8 + u == i) ? 1.f : 0.f;
        uint4 hv, lv;
        split8(x, hv, lv);
        *reinterpret_cast<uint4*>(out_img + o) = hv;
        *reinterpret_cast<uint4*>(out_img + kImg + o) = lv;
      }
    }
    float4* cd = reinterpret_cast<float4*>(out_c);
    for (int t = 0; t < D / 4; ++t) cd[t * D + i] = nf == 1 ? csrc[t * D + i] : make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = sm100::align_smem_1024(smem_raw);
  uint8_t* sMM = smem + kMMOff;
  uint8_t* sJJ = smem + kJJOff;
  uint8_t* sMf = smem + kMfOff;
  uint64_t* ldbar = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* mmabar = ldbar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ldbar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    mbar_init(ldbar, 1);
    mbar_init(mmabar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    // MM <- M_f0 (its image is already the K-major operand layout) and the next frame's M.
    mbar_arrive_expect_tx(ldbar, 2 * kPair);
    const uint8_t* m0 = a.Mi + (slots + frame(0)) * (long long)kPair;
    const uint8_t* m1 = a.Mi + (slots + frame(1)) * (long long)kPair;
    bulk_load(sMM, m0, kImg, ldbar);
    bulk_load(sMM + kImg, m0 + kImg, kImg, ldbar);
    bulk_load(sMf, m1, kImg, ldbar);
    bulk_load(sMf + kImg, m1 + kImg, kImg, ldbar);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  // JJ <- C_f0 as a split image (row i).
  {
    const float4* src = reinterpret_cast<const float4*>(a.C + (slots + frame(0)) * (long long)D * D);
    for (int c8 = 0; c8 < D / 8; ++c8) {
      const float4 v0 = src[(2 * c8) * D + i];
      const float4 v1 = src[(2 * c8 + 1) * D + i];
      const float x[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      put8(sJJ, i, c8 * 8, x);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
  // Thread 0 owns the operand loads and the MMAs and tracks what is in flight,
  // so that an abandoned step can be drained before TMEM and smem go away.
  uint32_t ldph = 0, mph = 0;
  bool ld_inflight = true, mma_inflight = false;

  for (int k = 1; k < nf; ++k) {
    const int f = frame(k);
    bool ok = true;
    if (threadIdx.x == 0) {
      ok = mbar_wait(ldbar, ldph, abort_flag, a.status, a.wait_ns);
      if (ok) {
        ldph ^= 1;
        ld_inflight = false;
        tc_fence_after();
        const uint32_t mmh = smem_u32(sMM), mml = mmh + kImg, jjh = smem_u32(sJJ), jjl = jjh + kImg;
        const uint32_t mfh = smem_u32(sMf), mfl = mfh + kImg;
        const uint32_t as[3] = {0, 0, 1}, bs[3] = {0, 1, 0};
#pragma unroll
        for (int t = 0; t < 3; ++t)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koffA = (kk / 4) * (D * 128) + (kk % 4) * 32;
            const uint64_t db = smem_desc_sw128((bs[t] ? mfl : mfh) + kk * 2048, D * 128, 1024);
            const uint32_t acc = (t == 0 && kk == 0) ? 0u : 1u;
            mma_f16(tmem, smem_desc_sw128((as[t] ? mml : mmh) + koffA, 16, 1024), db, kIdesc, acc);
            mma_f16(tmem + 128, smem_desc_sw128((as[t] ? jjl : jjh) + koffA, 16, 1024), db, kIdesc, acc);
          }
        mma_commit(mmabar);
        mma_inflight = true;
      }
    }
    // C_f row i, fetched while the MMAs run.
    const float4* csrc = reinterpret_cast<const float4*>(a.C + (slots + f) * (long long)D * D);
    float crow[D];
#pragma unroll
    for (int t = 0; t < D / 4; ++t) {
      const float4 v = csrc[t * D + i];
      crow[4 * t] = v.x; crow[4 * t + 1] = v.y; crow[4 * t + 2] = v.z; crow[4 * t + 3] = v.w;
    }
    // A failed load wait in thread 0 sets the abort flag, which ends the others' waits.
    if (ok) ok = mbar_wait(mmabar, mph, abort_flag, a.status, a.wait_ns);
    if (ok) {
      mph ^= 1;
      if (threadIdx.x == 0) mma_inflight = false;
    }
    // Every thread takes the same exit, so the block barriers below stay matched.
    if (__syncthreads_or(!ok)) break;
    tc_fence_after();
    // The MMAs are done with sMM, sJJ and sMf: prefetch the next frame's M.
    if (threadIdx.x == 0 && k + 1 < nf) {
      const uint8_t* mn = a.Mi + (slots + frame(k + 1)) * (long long)kPair;
      mbar_arrive_expect_tx(ldbar, kPair);
      bulk_load(sMf, mn, kImg, ldbar);
      bulk_load(sMf + kImg, mn + kImg, kImg, ldbar);
      ld_inflight = true;
    }
    const bool last = k + 1 == nf;
#pragma unroll
    for (int c16 = 0; c16 < D / 16; ++c16) {
      uint32_t v[16], w[16];
      tmem_ld16(tl + c16 * 16, v);
      tmem_ld16(tl + 128 + c16 * 16, w);
      tmem_ld_wait();
      float xm[16], xj[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        xm[t] = __uint_as_float(v[t]);
        xj[t] = __uint_as_float(w[t]) + crow[c16 * 16 + t];
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int col = c16 * 16 + 8 * hh;
        if (last) {
          put8(out_img, i, col, xm + 8 * hh);
          float4* cd = reinterpret_cast<float4*>(out_c);
          cd[(col / 4) * D + i] = make_float4(xj[8 * hh], xj[8 * hh + 1], xj[8 * hh + 2], xj[8 * hh + 3]);
          cd[(col / 4 + 1) * D + i] = make_float4(xj[8 * hh + 4], xj[8 * hh + 5], xj[8 * hh + 6], xj[8 * hh + 7]);
        } else {
          put8(sMM, i, col, xm + 8 * hh);
          put8(sJJ, i, col, xj + 8 * hh);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
  }

  // ---------------- teardown: nothing may be in flight when TMEM and smem go away
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    if (mma_inflight) mbar_wait(mmabar, mph, nullptr, a.status, a.wait_ns);
    if (ld_inflight) mbar_wait(ldbar, ldph, nullptr, a.status, a.wait_ns);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

cudaError_t launch_compose_tc(const Problem& p, cudaStream_t s) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(compose_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  if (p.J < 3) return cudaSuccess;  // no readout state sees a composed chunk
  if ((long long)p.B * p.H > 65535) return cudaErrorInvalidConfiguration;
  ComposeArgs a{p.H, p.T, p.c, p.J, static_cast<const uint8_t*>(p.Msplit), p.C, static_cast<uint8_t*>(p.CMi),
                p.CC, p.status, p.spin_limit};
  dim3 grid(p.J, 2, p.B * p.H);
  compose_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(a);
  return cudaGetLastError();
}

}  // namespace vda
