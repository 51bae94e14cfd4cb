// Generic CUDA-core kernels for every stage of the VDA linear branch.
//
// They serve the float32 storage path (where tensor-core rounding would not be
// float32-faithful), head sizes without a tensor-core kernel, and cross-checks
// of the tcgen05 kernels (VDA_FORCE_SIMT). All arithmetic is float32.
//
// Method: Video DeltaNet summary (onedev.kr/papers/80), section "how to use"
// (frame statistics, frame solve, transition M_t), section "how it works"
// (bidirectional readout from S_T/2), section "how it differs" (conv + SiLU
// + L2 prep, RMSNorm + sigmoid gate on the readout).
#include <cuda_bf16.h>

#include <type_traits>

#include "internal.h"

namespace vda {

__device__ __forceinline__ float ld_tok(const void* p, long long i, int bf16) {
  return bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i])
              : static_cast<const float*>(p)[i];
}
__device__ __forceinline__ void st_tok(void* p, long long i, float v, int bf16) {
  if (bf16)
    static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else
    static_cast<float*>(p)[i] = v;
}
__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + __expf(-x)); }
__device__ __forceinline__ float sigmoid_f(float x) { return 1.0f / (1.0f + __expf(-x)); }

// ---------------------------------------------------------------------------
// Frame statistics: A = K^T Diag(beta) K, B = V^T Diag(beta) K per (b, h, slot).
// Grid (T-1, H, B); slot 0 = text tokens, slot t = frame t. Each thread owns a
// (D/16) x (D/16) tile of both outputs; tokens stream through shared memory.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) gram_simt_kernel(Problem p) {
  constexpr int TI = D / 16;
  constexpr int TU = 32;
  __shared__ float sK[TU][D + 1];
  __shared__ float sV[TU][D + 1];
  __shared__ float sb[TU];
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const TokView kv = s == 0 ? p.Kt : p.Kv;
  const TokView vv = s == 0 ? p.Vt : p.Vv;
  const long long tsel = s == 0 ? 0 : s;
  const long long bk = b * kv.s_b + h * kv.s_h + tsel * kv.s_t;
  const long long bv = b * vv.s_b + h * vv.s_h + tsel * vv.s_t;
  const int n = s == 0 ? p.L : p.U;
  const float* beta = s == 0 ? p.beta_txt + ((long long)b * p.H + h) * p.L
                             : p.beta + (((long long)b * p.H + h) * p.T + s) * p.U;
  float accA[TI][TI], accB[TI][TI];
#pragma unroll
  for (int a = 0; a < TI; ++a)
#pragma unroll
    for (int c = 0; c < TI; ++c) accA[a][c] = accB[a][c] = 0.f;

  for (int u0 = 0; u0 < n; u0 += TU) {
    for (int e = threadIdx.x; e < TU * D; e += blockDim.x) {
      const int uu = e / D, k = e % D, u = u0 + uu;
      float x = 0.f, y = 0.f;
      if (u < n) {
        x = ld_tok(kv.p, bk + u * kv.s_u + k, p.bf16);
        y = ld_tok(vv.p, bv + u * vv.s_u + k, p.bf16);
      }
      sK[uu][k] = x;
      sV[uu][k] = y;
    }
    if (threadIdx.x < TU) sb[threadIdx.x] = (u0 + (int)threadIdx.x < n) ? beta[u0 + threadIdx.x] : 0.f;
    __syncthreads();
#pragma unroll 4
    for (int uu = 0; uu < TU; ++uu) {
      float ki[TI], vi[TI], kj[TI];
      const float bb = sb[uu];
#pragma unroll
      for (int a = 0; a < TI; ++a) {
        ki[a] = sK[uu][ty + 16 * a];
        vi[a] = sV[uu][ty + 16 * a];
        kj[a] = bb * sK[uu][tx + 16 * a];
      }
#pragma unroll
      for (int a = 0; a < TI; ++a)
#pragma unroll
        for (int c = 0; c < TI; ++c) {
          accA[a][c] = fmaf(ki[a], kj[c], accA[a][c]);
          accB[a][c] = fmaf(vi[a], kj[c], accB[a][c]);
        }
    }
    __syncthreads();
  }
  const long long off = slot_off(p, b, h, s);
#pragma unroll
  for (int a = 0; a < TI; ++a)
#pragma unroll
    for (int c = 0; c < TI; ++c) {
      const int i = ty + 16 * a, j = tx + 16 * c;
      p.A[off + quad_off(D, i, j)] = accA[a][c];
      p.Bm[off + quad_off(D, i, j)] = accB[a][c];
    }
}

// ---------------------------------------------------------------------------
// Frame solve: Cholesky I + A = L L^T, Y = L^-1, P = Y^T Y = (I + A)^-1,
// M = Diag(alpha) P, C = B P. Slot 0 (text) writes only C = S_T.
// Grid (T-1, H, B), 256 threads, 2 * D * (D+1) floats of shared memory.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) solve_simt_kernel(Problem p) {
  constexpr int LD = D + 1;
  extern __shared__ float smem[];
  float* X = smem;           // I + A, then L (lower), then P
  float* Y = smem + D * LD;  // L^-1 (lower)
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, nt = blockDim.x;
  const long long off = slot_off(p, b, h, s);
  const float* A = p.A + off;
  for (int e = tid; e < D * D; e += nt) {
    const int i = quad_row(D, e), j = quad_col(D, e);
    X[i * LD + j] = A[e] + (i == j ? 1.f : 0.f);
  }
  __syncthreads();
  // Right-looking Cholesky, column by column.
  for (int k = 0; k < D; ++k) {
    if (tid == 0) X[k * LD + k] = sqrtf(X[k * LD + k]);
    __syncthreads();
    const float dkk = X[k * LD + k];
    for (int i = k + 1 + tid; i < D; i += nt) X[i * LD + k] /= dkk;
    __syncthreads();
    const int n = D - k - 1;
    for (int e = tid; e < n * n; e += nt) {
      const int i = k + 1 + e / n, j = k + 1 + e % n;
      if (j <= i) X[i * LD + j] -= X[i * LD + k] * X[j * LD + k];
    }
    __syncthreads();
  }
  // Y = L^-1 by forward substitution, one row at a time, all columns in parallel.
  for (int i = 0; i < D; ++i) {
    const float lii = X[i * LD + i];
    for (int j = tid; j <= i; j += nt) {
      float acc = (i == j) ? 1.f : 0.f;
      for (int k = j; k < i; ++k) acc -= X[i * LD + k] * Y[k * LD + j];
      Y[i * LD + j] = acc / lii;
    }
    __syncthreads();
  }
  // P = Y^T Y (symmetric); P[i][j] = sum_{k >= max(i,j)} Y[k][i] Y[k][j].
  for (int e = tid; e < D * D; e += nt) {
    const int i = e / D, j = e % D, m = i > j ? i : j;
    float acc = 0.f;
    for (int k = m; k < D; ++k) acc = fmaf(Y[k * LD + i], Y[k * LD + j], acc);
    X[i * LD + j] = acc;
  }
  __syncthreads();
  if (s > 0) {
    const float* alpha = p.alpha + (((long long)b * p.H + h) * p.T + s) * D;
    for (int e = tid; e < D * D; e += nt) {
      const int i = quad_row(D, e), j = quad_col(D, e);
      p.M[off + e] = alpha[i] * X[i * LD + j];
    }
  }
  const float* Bm = p.Bm + off;
  for (int e = tid; e < D * D; e += nt) {
    const int i = quad_row(D, e), j = quad_col(D, e);
    float acc = 0.f;
    for (int k = 0; k < D; ++k) acc = fmaf(Bm[quad_off(D, i, k)], X[k * LD + j], acc);
    p.C[off + e] = acc;
  }
}

// ---------------------------------------------------------------------------
// Bidirectional scan. Grid (B*H, 2 directions, D/16 row slabs). The rows of the
// state evolve independently under S <- S M + C, so each CTA carries 16 rows.
// Forward: F(0) = S_T/2, F(f) = F(f-1) M_f + C_f for f = 1 .. c(J-2)-1.
// Reverse: R(T-1) = S_T/2, R(f) = R(f+1) M_f + C_f for f = T-2 .. 2c.
// Chunk j's forward readout state is F(max(0, c(j-1)-1)); its reverse one is
// R(min(T-1, c(j+2))).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) scan_simt_kernel(Problem p) {
  constexpr int R = 16, NC = D / 16;
  __shared__ float sS[R][D + 1];
  const int bh = blockIdx.x, dir = blockIdx.y, r0 = blockIdx.z * R;
  const int b = bh / p.H, h = bh % p.H;
  const int r = threadIdx.x / 16, l = threadIdx.x % 16;
  const float* S_T = p.C + slot_off(p, b, h, 0);
  float* out = dir == 0 ? p.Sf : p.Sr;
  const int c = p.c, T = p.T, J = p.J;
#pragma unroll
  for (int m = 0; m < NC; ++m) sS[r][l + 16 * m] = 0.5f * S_T[quad_off(D, r0 + r, l + 16 * m)];
  __syncthreads();
  auto store = [&](int j) {
    const long long o = chunk_off(p, b, h, j);
#pragma unroll
    for (int m = 0; m < NC; ++m) out[o + quad_off(D, r0 + r, l + 16 * m)] = sS[r][l + 16 * m];
  };
  for (int j = 0; j < J; ++j)
    if (dir == 0 ? (c * (j - 1) - 1 <= 0) : (c * (j + 2) >= T - 1)) store(j);
  const int f_first = dir == 0 ? 1 : T - 2;
  const int f_last = dir == 0 ? c * (J - 2) - 1 : 2 * c;
  const int nsteps = dir == 0 ? f_last - f_first + 1 : f_first - f_last + 1;
  for (int st = 0; st < nsteps; ++st) {
    const int f = dir == 0 ? f_first + st : f_first - st;
    const float* Mf = p.M + slot_off(p, b, h, f);
    const float* Cf = p.C + slot_off(p, b, h, f);
    float acc[NC];
#pragma unroll
    for (int m = 0; m < NC; ++m) acc[m] = Cf[quad_off(D, r0 + r, l + 16 * m)];
#pragma unroll 4
    for (int k = 0; k < D; ++k) {
      const float sv = sS[r][k];
#pragma unroll
      for (int m = 0; m < NC; ++m) acc[m] = fmaf(sv, Mf[quad_off(D, k, l + 16 * m)], acc[m]);
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < NC; ++m) sS[r][l + 16 * m] = acc[m];
    __syncthreads();
    if (dir == 0) {
      if ((f + 1) % c == 0 && (f + 1) / c + 1 < J) store((f + 1) / c + 1);
    } else {
      if (f % c == 0 && f / c - 2 >= 0) store(f / c - 2);
    }
  }
}

// ---------------------------------------------------------------------------
// Readout. Grid (J * tiles, H, B); a CTA owns 64 consecutive tokens of the
// non-anchor frames of chunk j and the chunk's summed state S-> + S<-.
// Thread (token u = tid/4, quarter q = tid%4) computes rows i = q + 4m of o_u.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) readout_simt_kernel(Problem p, const void* gate, void* O,
                                                           int tiles_per_chunk) {
  constexpr int LD = D + 1, TT = 64, NR = D / 4;
  extern __shared__ float smem[];
  float* sS = smem;            // [D][LD]  S-> + S<-
  float* sQ = smem + D * LD;   // [TT][LD]
  const int h = blockIdx.y, b = blockIdx.z;
  const int j = blockIdx.x / tiles_per_chunk, tile = blockIdx.x % tiles_per_chunk;
  const int t_lo = max(p.c * j, 1), t_hi = min(p.c * (j + 1), p.T - 1);
  if (t_lo >= t_hi) return;
  const long long tok_hi = (long long)t_hi * p.U;
  const long long tok0 = (long long)t_lo * p.U + (long long)tile * TT;
  if (tok0 >= tok_hi) return;
  const int ntok = (int)min((long long)TT, tok_hi - tok0);
  const long long co = chunk_off(p, b, h, j);
  for (int e = threadIdx.x; e < D * D; e += blockDim.x)
    sS[quad_row(D, e) * LD + quad_col(D, e)] = p.Sf[co + e] + p.Sr[co + e];
  const long long rowstride = (long long)p.H * D;
  const long long qbase = ((long long)b * p.T * p.U) * rowstride + (long long)h * D;
  for (int e = threadIdx.x; e < TT * D; e += blockDim.x) {
    const int uu = e / D, k = e % D;
    sQ[uu * LD + k] = uu < ntok ? ld_tok(p.Q, qbase + (tok0 + uu) * rowstride + k, p.bf16) : 0.f;
  }
  __syncthreads();
  const int uu = threadIdx.x / 4, q4 = threadIdx.x % 4;
  float acc[NR];
#pragma unroll
  for (int m = 0; m < NR; ++m) acc[m] = 0.f;
  float qq = 0.f;
#pragma unroll 4
  for (int k = 0; k < D; ++k) {
    const float qk = sQ[uu * LD + k];
    qq = fmaf(qk, qk, qq);
#pragma unroll
    for (int m = 0; m < NR; ++m) acc[m] = fmaf(sS[(q4 + 4 * m) * LD + k], qk, acc[m]);
  }
  const bool valid = uu < ntok;  // all lanes stay for the warp shuffles below
  const float scale = (p.flags & VDA_PREP_CONV) ? rsqrtf(qq + p.l2_eps) : 1.f;
  const long long obase = qbase + (tok0 + (valid ? uu : 0)) * rowstride;
  if (p.flags & VDA_READOUT_NORM_GATE) {
    float ss = 0.f;
#pragma unroll
    for (int m = 0; m < NR; ++m) {
      acc[m] *= scale;
      ss = fmaf(acc[m], acc[m], ss);
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    const float rn = rsqrtf(ss / D + p.rms_eps);
    if (!valid) return;
#pragma unroll
    for (int m = 0; m < NR; ++m) {
      const float g = ld_tok(gate, obase + q4 + 4 * m, p.bf16);
      st_tok(O, obase + q4 + 4 * m, acc[m] * rn * sigmoid_f(g), p.bf16);
    }
  } else {
    if (!valid) return;
#pragma unroll
    for (int m = 0; m < NR; ++m) st_tok(O, obase + q4 + 4 * m, acc[m] * scale, p.bf16);
  }
}

// Anchor frames 0 and T-1 read out exactly zero: for each batch element both
// frames are contiguous ranges of U*H*D elements of O.
// Grid (x, 2 * B): blockIdx.y names one contiguous slab (batch b, anchor frame
// 0 or T-1) of U * H * D values; the x blocks stride over its 16-byte words.
__global__ void zero_anchors_kernel(Problem p, void* O) {
  const long long per = (long long)p.U * p.H * p.D;
  const int esz = p.bf16 ? 2 : 4;
  const long long words = per * esz / 16;  // per is a multiple of 16 (D >= 16)
  const long long b = blockIdx.y >> 1, frame = (blockIdx.y & 1) ? p.T - 1 : 0;
  uint4* base = reinterpret_cast<uint4*>(static_cast<char*>(O) + (b * p.T + frame) * per * esz);
  for (long long w = blockIdx.x * (long long)blockDim.x + threadIdx.x; w < words;
       w += (long long)gridDim.x * blockDim.x)
    base[w] = make_uint4(0, 0, 0, 0);
}

// Text prep: SiLU on K_txt and V_txt, then L2 on K_txt; one warp per token.
// Output layout [B, H, L, D].
__global__ void prep_text_kernel(Problem p, const void* Kt, const void* Vt) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) / 32, lane = threadIdx.x % 32;
  const int D = p.D, H = p.H, L = p.L;
  if (warp >= p.B * L * H) return;
  const int h = warp % H, l = (warp / H) % L, b = warp / (H * L);
  const long long ib = (((long long)b * L + l) * H + h) * D;
  const long long ob = (((long long)b * H + h) * L + l) * D;
  float ss = 0.f;
  for (int k = lane; k < D; k += 32) {
    const float x = silu_f(ld_tok(Kt, ib + k, p.bf16));
    ss = fmaf(x, x, ss);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float sc = rsqrtf(ss + p.l2_eps);
  for (int k = lane; k < D; k += 32) {
    st_tok(p.Ktp, ob + k, silu_f(ld_tok(Kt, ib + k, p.bf16)) * sc, p.bf16);
    st_tok(p.Vtp, ob + k, silu_f(ld_tok(Vt, ib + k, p.bf16)), p.bf16);
  }
}

// Failure-detection self test: wait on a flag that nothing ever sets.
__device__ unsigned int g_never_set_flag = 0;
__global__ void selftest_wait_kernel(uint32_t* status, unsigned long long spins) {
  unsigned long long n = 0;
  while (*reinterpret_cast<volatile unsigned int*>(&g_never_set_flag) == 0) {
    if (++n >= spins) {
      atomicExch(status, (uint32_t)VDA_ERR_TIMEOUT);
      return;
    }
    __nanosleep(256);
  }
}

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
template <typename F>
static cudaError_t dispatch_d(int D, F&& f) {
  switch (D) {
    case 16: return f(std::integral_constant<int, 16>{});
    case 32: return f(std::integral_constant<int, 32>{});
    case 64: return f(std::integral_constant<int, 64>{});
    case 128: return f(std::integral_constant<int, 128>{});
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gram_simt(const Problem& p, cudaStream_t s) {
  dim3 grid(p.T - 1, p.H, p.B);
  return dispatch_d(p.D, [&](auto dc) {
    constexpr int D = decltype(dc)::value;
    gram_simt_kernel<D><<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
  });
}

cudaError_t launch_solve_simt(const Problem& p, cudaStream_t s) {
  dim3 grid(p.T - 1, p.H, p.B);
  return dispatch_d(p.D, [&](auto dc) {
    constexpr int D = decltype(dc)::value;
    const size_t smem = 2ull * D * (D + 1) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(solve_simt_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    solve_simt_kernel<D><<<grid, 256, smem, s>>>(p);
    return cudaGetLastError();
  });
}

cudaError_t launch_scan_simt(const Problem& p, cudaStream_t s) {
  dim3 grid(p.B * p.H, 2, p.D / 16);
  return dispatch_d(p.D, [&](auto dc) {
    constexpr int D = decltype(dc)::value;
    scan_simt_kernel<D><<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
  });
}

cudaError_t launch_readout_simt(const Problem& p, const void* gate, void* O, cudaStream_t s) {
  const int tiles = (int)((p.c * (long long)p.U + 63) / 64);
  dim3 grid(p.J * tiles, p.H, p.B);
  return dispatch_d(p.D, [&](auto dc) {
    constexpr int D = decltype(dc)::value;
    const size_t smem = (size_t)(D + 64) * (D + 1) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(readout_simt_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    readout_simt_kernel<D><<<grid, 256, smem, s>>>(p, gate, O, tiles);
    return cudaGetLastError();
  });
}

cudaError_t launch_zero_anchors(const Problem& p, void* O, cudaStream_t s) {
  zero_anchors_kernel<<<dim3(148, 2 * p.B), 256, 0, s>>>(p, O);
  return cudaGetLastError();
}

cudaError_t launch_prep_text(const Problem& p, const void* Kt, const void* Vt, cudaStream_t s) {
  const long long warps = (long long)p.B * p.L * p.H;
  const int blocks = (int)((warps * 32 + 255) / 256);
  prep_text_kernel<<<blocks, 256, 0, s>>>(p, Kt, Vt);
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait(uint32_t* status, unsigned long long spins, cudaStream_t s) {
  selftest_wait_kernel<<<1, 1, 0, s>>>(status, spins);
  return cudaGetLastError();
}

}  // namespace vda
