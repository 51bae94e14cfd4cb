// Internal definitions shared by the host orchestration (vda_api.cu) and the
// kernel translation units. Not part of the C ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/vda.h"

namespace vda {

// A strided view of token vectors: element (b, h, t, u, k) of a token tensor
// lives at p + b*s_b + h*s_h + t*s_t + u*s_u + k (in elements).
struct TokView {
  const void* p;
  long long s_b, s_h, s_t, s_u;
};

// Everything a kernel needs, passed by value.
struct Problem {
  int B, H, T, U, L, D, c, J, gh, gw;
  // Heads per token row of the token tensors (Q, K, V, K_txt, V_txt, gate, O):
  // H_total of the config. Their pointers here are already advanced to the
  // context's first head, so head h of this problem sits at channel offset h*D
  // of a row of Ht*D values.
  int Ht;
  int bf16;            // 1: token tensors are bf16, 0: fp32
  unsigned flags;
  float l2_eps, rms_eps;
  // Video and text keys/values as read by the statistics kernel (raw inputs, or
  // the prepared copies in the workspace under VDA_PREP_CONV).
  TokView Kv, Vv, Kt, Vt;
  const float* alpha;     // [B,H,T,D]
  const float* beta;      // [B,H,T,U]
  const float* beta_txt;  // [B,H,L]
  const void* Q;          // [B,T*U,H,D]
  // Workspace regions (fp32 unless noted).
  uint32_t* status;
  float* A;     // [B,H,T-1,D,D]
  float* Bm;    // [B,H,T-1,D,D]
  float* M;     // [B,H,T-1,D,D]
  float* C;     // [B,H,T-1,D,D]; slot 0 = S_T
  float* Sf;    // [B,H,J,D,D]
  float* Sr;    // [B,H,J,D,D]
  void* Kp;     // [B,H,T,U,D] storage dtype (prep)
  void* Vp;
  void* Ktp;    // [B,H,L,D]
  void* Vtp;
  void* Msplit;  // [B,H,T-1] x 2 bf16 d*d images of M_t (hi, lo) for the tensor-core scan
  void* CMi;     // [B,H,2,J] x 2 bf16 d*d images: composed chunk transitions per direction
  float* CC;     // [B,H,2,J,D,D]: composed chunk injections per direction
  // [B,H,T-1] slot-ready words (zeroed at the start of every prepare): the
  // tensor-core sweep solve sets word (b,h,s) to 1 once slot s's C_t and M_t
  // images are written, and the frame scan, launched to overlap the solve's
  // last CTAs, acquires each word before it reads that slot. nullptr when the
  // solve that ran does not publish them (the scan then waits for nothing).
  uint32_t* ready;
  // [B,H,T-1] words the tensor-core statistics kernel raises (one count per
  // epilogue warp, kGramReadyCount in all) once slot s's A_t and B_t are written,
  // for the sweep solve, launched to overlap that kernel's last units. nullptr
  // when the statistics kernel that ran does not raise them.
  uint32_t* gready;
  // 1 when the sweep solve writes P_t's images (not M_t's, and no C_t for
  // frames) because the frame scan forms S Diag(alpha_t) + B_t itself.
  int pform;
  unsigned long long spin_limit;  // wall-time bound (ns) of every device-side wait
};

constexpr uint32_t kGramReadyCount = 4;

// The order in which the statistics kernel, the solve and the frame scan treat
// the n = T-1 slots of the BH heads: every head's slot 0 (S_T, read by both
// scan directions first), then for key k = 1, 2, ...: slot k of every head
// (forward step k-1), slot n-k of every head (reverse step k-1), and for even n
// the middle slot n/2 last. Position idx in 0 .. BH*n-1 maps to (bh, slot).
inline __host__ __device__ void key_slot(int idx, int BH, int n, int& bh, int& slot) {
  if (idx < BH) {
    bh = idx;
    slot = 0;
    return;
  }
  const int l = idx - BH, npairs = (n - 1) / 2;
  if (l < npairs * 2 * BH) {
    const int k = 1 + l / (2 * BH), w = l % (2 * BH);
    bh = w % BH;
    slot = w >= BH ? n - k : k;
  } else {
    bh = l - npairs * 2 * BH;
    slot = n / 2;
  }
}

// Slot s of the statistics / solve arrays: 0 = text, t = frame t (1..T-2).
inline __host__ __device__ long long slot_off(const Problem& p, int b, int h, int s) {
  return (((long long)b * p.H + h) * (p.T - 1) + s) * (long long)p.D * p.D;
}
inline __host__ __device__ long long chunk_off(const Problem& p, int b, int h, int j) {
  return (((long long)b * p.H + h) * p.J + j) * (long long)p.D * p.D;
}

// Every d x d fp32 matrix of the workspace (A_t, B_t, M_t, C_t, the readout
// states, the composed chunk injections) is stored in column quads: element
// (i, j) at float index ((j / 4) * d + i) * 4 + j % 4, i.e. float4 number
// (j / 4) * d + i. Threads that own consecutive rows (the tensor-core epilogues
// map matrix row i to TMEM lane i) then move 512 contiguous bytes per warp and
// float4 access instead of touching 32 separate lines.
inline __host__ __device__ long long quad_off(int D, int i, int j) {
  return ((long long)(j >> 2) * D + i) * 4 + (j & 3);
}
// Row and column of storage index e (0 <= e < d*d) in that layout.
inline __host__ __device__ int quad_row(int D, int e) { return (e >> 2) % D; }
inline __host__ __device__ int quad_col(int D, int e) { return ((e >> 2) / D) * 4 + (e & 3); }

// Kernel ids for launch accounting and profiling.
enum KernelId {
  K_PREP_VIDEO = 0,
  K_PREP_TEXT,
  K_GRAM_SIMT,
  K_GRAM_TC,
  K_SOLVE_SIMT,
  K_SCAN_SIMT,
  K_READOUT_SIMT,
  K_READOUT_TC,
  K_ZERO_ANCHORS,
  K_SOLVE_TC,
  K_SCAN_TC,
  K_COMPOSE_TC,
  K_SOLVE_CHOL_TC,
  K_WINDOW_ATTN_TC,
  K_MERGE_TC,
  K_FRAME_BWD_SIMT,
  K_SOLVE_TC_FRAMES,
  K_READOUT_FP8_TC,
  K_GRAM_FP8_TC,
  K_TOKEN_BWD_TC,
  K_SCAN_SPLIT_TC,
  K_NUM_KERNELS
};
const char* kernel_name(int id);

// Launchers (return cudaGetLastError() after the launch).
cudaError_t launch_prep_video(const Problem& p, const void* K, const void* V, const float* conv_w,
                              cudaStream_t s);
cudaError_t launch_prep_text(const Problem& p, const void* Kt, const void* Vt, cudaStream_t s);
cudaError_t launch_gram_simt(const Problem& p, cudaStream_t s);
cudaError_t launch_solve_simt(const Problem& p, cudaStream_t s);
cudaError_t launch_scan_simt(const Problem& p, cudaStream_t s);
cudaError_t launch_readout_simt(const Problem& p, const void* gate, void* O, cudaStream_t s);
cudaError_t launch_zero_anchors(const Problem& p, void* O, cudaStream_t s);
cudaError_t launch_selftest_wait(uint32_t* status, unsigned long long spins, cudaStream_t s);
// Backward of the frame step for frames 1..T-2 (after the statistics kernel has
// written A_t, B_t): writes dS_prev, dalpha, dbeta, dK, dV (and Gx, Gsym into the
// workspace's M and C slots). Two launches.
cudaError_t launch_frame_bwd_simt(const Problem& p, const float* S_prev, const float* dS, float* dS_prev,
                                  float* dalpha, float* dbeta, void* dK, void* dV, cudaStream_t s,
                                  bool tokens = true);
// The per-token part of that backward on tcgen05 (bf16, D = 128), after the
// per-frame adjoints are in the workspace's M (Gx) and C (Gsym) slots.
bool token_bwd_tc_supported(const Problem& p);
cudaError_t launch_token_bwd_tc(const Problem& p, const void* K, const void* V, float* dbeta, void* dK, void* dV,
                                cudaStream_t s);
// The sweep solve's pivot reciprocal applied to x[0..n) (for an error bound test).
cudaError_t launch_recip_selftest(const float* x, float* y, int n, cudaStream_t s);

// Tensor-core (tcgen05) kernels, bf16 with D in {64, 128}.
bool gram_tc_supported(const Problem& p);
cudaError_t launch_gram_tc(const Problem& p, cudaStream_t s);
bool readout_tc_supported(const Problem& p);
bool solve_tc_supported(const Problem& p);
// Raise `func`'s dynamic shared-memory limit to `bytes` on the current device,
// once per (function, device): the attribute belongs to the device's context.
cudaError_t set_max_dynamic_smem(const void* func, int bytes);
// part 0: the text slots (or, unless the P form is used, every slot); part 1:
// the frame slots of the P form (compact CTAs). Nothing for part 1 otherwise.
cudaError_t launch_solve_tc(const Problem& p, cudaStream_t s, int part);
cudaError_t launch_solve_chol_tc(const Problem& p, cudaStream_t s);
bool scan_tc_supported(const Problem& p);
cudaError_t launch_scan_tc(const Problem& p, cudaStream_t s, bool chunked);
// Frame scan with each state's 64-column halves on the two CTAs of a cluster
// (after the sweep solve, injections formed in the scan).
bool scan_split_tc_supported(const Problem& p);
cudaError_t launch_scan_split_tc(const Problem& p, cudaStream_t s);
cudaError_t launch_compose_tc(const Problem& p, cudaStream_t s);
cudaError_t launch_readout_tc(const Problem& p, const void* gate, void* O, cudaStream_t s);

// Softmax branch: window + anchor attention with the sigmoid gate (bf16, D in {64, 128}).
// Q, K, V, gate and O are advanced to the problem's first head (rows of Ht * D values).
bool window_attn_tc_supported(const Problem& p);
cudaError_t launch_window_attn_tc(const Problem& p, const void* Q, const void* K, const void* V, const void* gate,
                                  void* O, cudaStream_t s);
// Readout from e4m3 queries with per-(token, head) scales (D = 128, no conv
// prep or gate); Q8 and q_scale advanced to the problem's first head.
bool readout_fp8_tc_supported(const Problem& p);
cudaError_t launch_readout_fp8_tc(const Problem& p, const void* Q8, const float* q_scale, void* O, cudaStream_t s);
// Statistics from e4m3 keys and values with per-(token, head) scales shared by
// the token's key and value (D = 128): a pre-pass writes each slot's exponent to
// unit_exp, then the tensor-core kernel writes A, B. Two launches.
cudaError_t launch_gram_fp8_tc(const Problem& p, const void* K8, const void* V8, const float* kv_scale,
                               const void* Kt8, const void* Vt8, const float* kvt_scale, int* unit_exp,
                               cudaStream_t s);
// Hybrid merge Y = A1 B1^T + A2 B2^T (bf16, K-major rows; Y [M, N] bf16).
cudaError_t launch_merge_tc(const void* A1, const void* B1, const void* A2, const void* B2, void* Y, int M, int N,
                            int K1, int K2, uint32_t* status, unsigned long long wait_ns, cudaStream_t s);

}  // namespace vda
