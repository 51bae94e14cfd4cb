/*
 * vda.h -- C ABI of libvda.so: Video Delta Attention (VDA), the linear branch
 * of Video DeltaNet, as a bidirectional frame-level delta scan with a windowed
 * readout, for NVIDIA B200 (sm_100a).
 *
 * Method (Video DeltaNet summary, onedev.kr/papers/80):
 *  - section "how to use": per frame t, with keys K_t [U x d_k], values V_t
 *    [U x d_v], write strengths beta_t [U] and decay alpha_t [d_k],
 *      A_t = K_t^T Diag(beta_t) K_t,   B_t = V_t^T Diag(beta_t) K_t,
 *      S_t = (S_{t-1} Diag(alpha_t) + B_t)(I + A_t)^-1
 *    i.e. the minimiser of 1/2|S - Sbar|_F^2 + 1/2 sum_u beta_u |S k_u - v_u|^2,
 *    with M_t = Diag(alpha_t)(I + A_t)^-1 (non-expansive) and the injection
 *    C_t = B_t (I + A_t)^-1, so S_t = S_{t-1} M_t + C_t;
 *  - section "how it works": a forward state summarises the frames before a
 *    query chunk's softmax window (chunks j-1..j+1), a reverse state the frames
 *    after it; both start at S_T/2 where S_T summarises the text tokens; the
 *    query reads o = S-> q + S<- q;
 *  - section "assumptions and limits": the boundary anchors (frames 0 and T-1)
 *    are excluded from the linear state;
 *  - section "how it differs": separable short conv (depthwise 5x5 spatial and
 *    5-tap temporal) then SiLU on K and V, L2 norm on Q and K; RMS norm and a
 *    sigmoid output gate on the linear readout.
 *
 * Readings fixed by this library where the pages are silent: S is d_v x d_k and
 * o = S q; S_T = B_txt (I + A_txt)^-1 (the frame solve from S = 0 over the text
 * tokens); the reverse scan uses the same M_t, C_t; chunk j = floor(t / c); the
 * forward readout state of chunk j is the state after frame c(j-1)-1 (S_T/2 when
 * that is < 1) and the reverse one the state after frame c(j+2) (S_T/2 when that
 * is > T-2); anchor frames read out exactly zero.
 *
 * Conventions shared by every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller, in memory of
 *    the device that is current when the call is made. The library does not
 *    check what kind of memory a pointer addresses (a host pointer reaches the
 *    kernels as it is); the Python binding checks its tensors first. The library
 *    never allocates or frees device memory; its only device memory is the
 *    caller's workspace.
 *  - Every call only enqueues work on the caller's CUDA stream (passed as
 *    void*, a cudaStream_t; NULL is the legacy default stream) and never
 *    synchronises, except vda_poll_device_status.
 *  - Every call returns a vda_status and never aborts or prints. Argument errors
 *    are detected before any launch and leave device memory untouched.
 *  - Input pointers given to vda_prepare must stay valid until the matching
 *    vda_readout has completed on the stream.
 *  - A context is not thread-safe; use one per host thread.
 */
#ifndef VDA_H_
#define VDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum vda_status {
  VDA_OK = 0,
  VDA_ERR_INVALID_ARG = 1,          /* null pointer, bad shape, inconsistent sizes */
  VDA_ERR_UNSUPPORTED = 2,          /* valid but not implemented (e.g. d not in {16,32,64,128}) */
  VDA_ERR_ALIGNMENT = 3,            /* a pointer is not 16-byte aligned (256 for the workspace) */
  VDA_ERR_WORKSPACE_TOO_SMALL = 4,  /* workspace_bytes < vda_workspace_size() */
  VDA_ERR_CUDA = 5,                 /* a CUDA runtime/driver call or a launch failed */
  VDA_ERR_TIMEOUT = 6,              /* a bounded device-side wait gave up (see vda_poll_device_status) */
  VDA_ERR_STATE = 7                 /* calls out of order (scan before prepare, ...) */
} vda_status;

typedef enum vda_dtype {
  VDA_F32 = 0,  /* Q, K, V, K_txt, V_txt, gate and O stored as float32 */
  VDA_BF16 = 1  /* ... stored as bfloat16; state, statistics and solves are always float32 */
} vda_dtype;

/* vda_config.flags */
#define VDA_PREP_CONV 0x1u         /* video K, V: depthwise 5x5 spatial + centred 5-tap temporal
                                      cross-correlation (zero padding, no bias) then SiLU; text K, V:
                                      SiLU; then K, K_txt and Q divided by sqrt(|x|^2 + l2_eps).
                                      Needs grid_h <= 65535 and 2 * B * H <= 65535, else
                                      VDA_ERR_UNSUPPORTED from vda_create */
#define VDA_READOUT_NORM_GATE 0x2u /* o <- o / sqrt(mean(o^2) + rms_eps) * sigmoid(gate) */
#define VDA_SOLVE_CHOLESKY 0x4u    /* tensor-core frame solve by blocked Cholesky of I + A_t and
                                      the triangular inverse, instead of the default symmetric
                                      sweep (Gauss-Jordan) in registers; the same M_t and C_t */
#define VDA_SCAN_CHUNKED 0x8u      /* tensor-core scan over composed chunk maps (each chunk's frame
                                      maps composed in parallel first) instead of the default scan
                                      frame by frame; the same readout states. Needs
                                      B * H <= 65535, else VDA_ERR_UNSUPPORTED from vda_create */
#define VDA_SCAN_SPLIT 0x10u       /* tensor-core frame scan on a two-CTA cluster per (b, h,
                                      direction), each CTA computing half of every state's columns
                                      and sending its half of the next left factor to the other,
                                      instead of the default one CTA per (b, h, direction) (the same
                                      readout states; no effect with VDA_SCAN_CHUNKED) */
#define VDA_FORCE_SIMT 0x100u      /* run the generic CUDA-core kernels even where a tensor-core
                                      kernel exists (diagnostics and cross-checks) */

typedef struct vda_config {
  int B;        /* batch */
  int H;        /* heads */
  int T;        /* latent frames, >= 3 */
  int U;        /* tokens per frame, == grid_h * grid_w */
  int grid_h;   /* latent grid rows (row-major token order u = y * grid_w + x) */
  int grid_w;   /* latent grid columns */
  int L;        /* text tokens, >= 1 */
  int d_k;      /* key channels; must equal d_v; one of 16, 32, 64, 128 */
  int d_v;      /* value channels */
  int chunk;    /* c: latent frames per chunk; chunk j holds frames c*j .. c*j+c-1 */
  int dtype;    /* vda_dtype of the token tensors */
  unsigned flags;
  float l2_eps;  /* default 1e-6 */
  float rms_eps; /* default 1e-6 */
  /* Head slice, for running a subset of the heads of a larger token tensor (one
   * rank's share when the heads are split across GPUs). The token tensors Q, K,
   * V, K_txt, V_txt, gate and O hold H_total heads per token row ([B, tokens,
   * H_total, d]); this context reads and writes heads h0 .. h0 + H - 1 of them
   * and never touches the others. 0 for H_total means H_total = H (then h0 must
   * be 0). The per-head parameters alpha, beta, beta_txt and conv_w are given
   * for this context's H heads only. */
  int H_total;
  int h0;
} vda_config;

typedef struct vda_ctx vda_ctx; /* opaque host object; owns no device memory */

/* Validate cfg and create a context. Host-only; touches no GPU. */
vda_status vda_create(const vda_config* cfg, vda_ctx** out);
vda_status vda_destroy(vda_ctx* ctx);

/* Bytes of device workspace the caller must provide to vda_prepare. Host-only. */
vda_status vda_workspace_size(const vda_config* cfg, size_t* bytes);

/*
 * Stage 1: feature prep (VDA_PREP_CONV only), frame statistics A_t, B_t for the
 * text slot and frames 1..T-2, and the frame solve giving S_T and each frame's
 * transition and injection (the inverse of I + A_t by the symmetric sweep, or by
 * Cholesky under VDA_SOLVE_CHOLESKY; see VDA_REGION_C and VDA_REGION_M_SPLIT for
 * what is stored). Layouts (row-major, innermost last):
 *   Q, K, V       [B, T*U, H, d]   token-major with heads interleaved; token
 *                                  index t*U + u for frame t, grid position u
 *   K_txt, V_txt  [B, L, H, d]
 *   alpha         [B, H, T, d_k]   float32 in [0, 1] (entries of anchor frames unused)
 *   beta          [B, H, T, U]     float32 >= 0
 *   beta_txt      [B, H, L]        float32 >= 0
 *   conv_w        float32, 60*H*d values: K-spatial [H*d,5,5], K-temporal [H*d,5],
 *                 V-spatial [H*d,5,5], V-temporal [H*d,5] concatenated (channel
 *                 h*d + k filters channel k of head h); required with
 *                 VDA_PREP_CONV, ignored (may be NULL) otherwise.
 *   workspace     >= vda_workspace_size(cfg) bytes, 256-byte aligned.
 * All token tensors use the storage type cfg.dtype; all pointers 16-byte aligned.
 */
vda_status vda_prepare(vda_ctx* ctx, const void* Q, const void* K, const void* V,
                       const void* K_txt, const void* V_txt, const float* alpha,
                       const float* beta, const float* beta_txt, const float* conv_w,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * Stage 2: the bidirectional scan. Forward F(0) = S_T/2, F(t) = F(t-1) M_t + C_t
 * for t = 1 ..; reverse R(T-1) = S_T/2, R(t) = R(t+1) M_t + C_t for t = T-2 ..
 * down. Writes, for every chunk j, its forward and reverse readout states into
 * the workspace. VDA_ERR_STATE unless vda_prepare succeeded on this context.
 * Queued on the stream of the vda_prepare call, the tensor-core frame scan is
 * launched as a programmatic dependent of the solve and starts while the
 * solve's last CTAs still run, reading each slot once its ready word is set
 * (see VDA_REGION_STATUS); results do not depend on the overlap.
 */
vda_status vda_scan_bidir(vda_ctx* ctx, void* stream);

/*
 * Stage 3: the readout. For every token of non-anchor frame t in chunk j:
 * o = (S->_j + S<-_j) q (q divided by sqrt(|q|^2 + l2_eps) under
 * VDA_PREP_CONV), then RMSNorm and the sigmoid gate under VDA_READOUT_NORM_GATE.
 * Tokens of anchor frames 0 and T-1 are written as zeros.
 *   gate  [B, T*U, H, d_v] storage dtype; required with VDA_READOUT_NORM_GATE.
 *   O     [B, T*U, H, d_v] storage dtype; fully overwritten.
 * VDA_ERR_STATE unless vda_scan_bidir succeeded after the last vda_prepare.
 */
vda_status vda_readout(vda_ctx* ctx, const void* gate, void* O, void* stream);

/*
 * Stage 1 with FP8 keys and values (NEXT to vda_readout_fp8 in the FP8 form of
 * the path): the frame statistics and the frame solve of vda_prepare, from keys
 * and values stored as e4m3 with one float32 scale per (token, head) shared by
 * the token's key and value, k = s K8, v = s V8, read at one byte per channel
 * (Video DeltaNet summary, section "assumptions and limits": FP8 / MXFP8 for the
 * large products). The write operand beta s^2 K8 enters the tensor cores as two
 * e4m3 parts under a power-of-two scale per (b, h, slot) (about 2^-8 relative).
 *   K8, V8          [B, T*U, H_total, d] e4m3      kv_scale   [B, T*U, H_total] float32
 *   Kt8, Vt8        [B, L, H_total, d] e4m3        kvt_scale  [B, L, H_total] float32
 *   alpha, beta, beta_txt, workspace: as for vda_prepare.
 * Needs d = 128, bf16 storage of the other tensors, no VDA_PREP_CONV or
 * VDA_FORCE_SIMT (else VDA_ERR_UNSUPPORTED). Then vda_scan_bidir and vda_readout
 * or vda_readout_fp8 as after vda_prepare (vda_readout needs the bf16 Q; this
 * call has none, so use vda_readout_fp8).
 */
vda_status vda_prepare_fp8(vda_ctx* ctx, const void* K8, const void* V8, const float* kv_scale, const void* Kt8,
                           const void* Vt8, const float* kvt_scale, const float* alpha, const float* beta,
                           const float* beta_txt, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Stage 3 with FP8 queries (the pages run their large products in FP8 / MXFP8:
 * Video DeltaNet summary, section "assumptions and limits"; VDN-H3 post, section
 * "compared with existing methods"): the readout of vda_readout for queries
 * given as e4m3 values with one float32 scale per (token, head),
 * q = q_scale * Q8, read at one byte per channel.
 *   Q8       [B, T*U, H_total, d] e4m3 (OCP FP8, 4 exponent and 3 mantissa bits)
 *   q_scale  [B, T*U, H_total] float32
 *   O        [B, T*U, H_total, d_v] bf16; anchor frames written as zeros
 * The gathered state S->_j + S<-_j enters the tensor cores as two e4m3 parts
 * under a power-of-two scale per (b, h, chunk) (about 2^-8 relative), products
 * accumulate in fp32. Needs d = 128, bf16 storage, and neither VDA_PREP_CONV nor
 * VDA_READOUT_NORM_GATE (else VDA_ERR_UNSUPPORTED); VDA_ERR_STATE unless
 * vda_scan_bidir succeeded after the last vda_prepare. The Q given to
 * vda_prepare is not read by this call.
 */
vda_status vda_readout_fp8(vda_ctx* ctx, const void* Q8, const float* q_scale, void* O, void* stream);

/*
 * Synchronise `stream`, read the device status words of the last vda_prepare
 * workspace and of the last vda_window_attention workspace, clear them and return
 * VDA_ERR_TIMEOUT if a bounded device-side wait gave up since the last poll,
 * VDA_OK otherwise (VDA_ERR_STATE before any vda_prepare or vda_window_attention).
 */
vda_status vda_poll_device_status(vda_ctx* ctx, void* stream);

/*
 * The softmax half of the hybrid attention layer, on the same Q, K, V as the
 * linear branch (Video DeltaNet summary, onedev.kr/papers/80, section "how it
 * works": each query chunk attends densely to chunks j-1 .. j+1 and to the
 * boundary anchors; section "how it differs": its own sigmoid output gate; VDN-H3
 * post, section "hybrid attention structure": the four-way anchor links).
 * For every token of frame t (chunk j = floor(t / c)), every head:
 *   o = softmax(q K_vis^T / sqrt(d)) V_vis,  then  o <- o * sigmoid(g)  (gate given)
 * where the visible keys are every token of frames max(0, c(j-1)) .. min(T-1,
 * c(j+2)-1) and of frames 0 and T-1 when t is not an anchor, and every video
 * token when t is 0 or T-1 (text tokens are not part of this branch).
 *   Q, K, V, gate, O  [B, T*U, H_total, d] storage dtype (this context's heads
 *                     h0 .. h0 + H - 1 are read and written); gate may be NULL.
 *   workspace         >= 256 bytes of device memory, 256-byte aligned; its first
 *                     word is this call's device status word (cleared here, read
 *                     by vda_poll_device_status). Separate calls that may run at
 *                     the same time need separate workspaces.
 * Needs bf16 storage and d in {64, 128} (tensor-core kernel), else
 * VDA_ERR_UNSUPPORTED. Independent of vda_prepare; only enqueues work.
 */
vda_status vda_window_attention(vda_ctx* ctx, const void* Q, const void* K, const void* V, const void* gate,
                                void* O, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward of one frame step of the scan, for training: for every head and every
 * non-anchor frame t = 1 .. T-2, the vector-Jacobian product of
 *   S_t = (S_{t-1} Diag(alpha_t) + B_t)(I + A_t)^-1,  A_t = K_t^T Diag(beta_t) K_t,
 *   B_t = V_t^T Diag(beta_t) K_t
 * (Video DeltaNet summary, onedev.kr/papers/80, section "how to use": the frame
 * solve; section "assumptions and limits": the update is trained end to end; the
 * pages print no backward, so this is the chain rule of the forward step). Given
 * dS = dL/dS_t it returns dL/dS_{t-1}, dL/dK_t, dL/dV_t, dL/dbeta_t, dL/dalpha_t.
 *   K, V           [B, T*U, H_total, d] storage dtype (prepared keys and values)
 *   alpha, beta    [B, H, T, d_k], [B, H, T, U] float32, as for vda_prepare
 *   S_prev, dS     [B, H, T, d_v, d_k] float32 row-major: entry t is S_{t-1} and
 *                  dL/dS_t (entries of anchor frames 0 and T-1 are not read)
 *   dK, dV         [B, T*U, H_total, d] storage dtype; dS_prev [B, H, T, d_v, d_k],
 *   dalpha, dbeta  [B, H, T, d_k], [B, H, T, U] float32: written for frames
 *                  1 .. T-2 only, every other entry is left as it was
 *   workspace      >= vda_workspace_size(cfg) bytes, 256-byte aligned (its A, B,
 *                  M and C regions are overwritten; a later vda_scan_bidir needs a
 *                  new vda_prepare)
 * Not with VDA_PREP_CONV (VDA_ERR_UNSUPPORTED). Only enqueues work; device-side
 * timeouts are read with vda_poll_device_status.
 */
vda_status vda_frame_solve_backward(vda_ctx* ctx, const void* K, const void* V, const float* alpha,
                                    const float* beta, const float* S_prev, const float* dS, void* dK, void* dV,
                                    float* dalpha, float* dbeta, float* dS_prev, void* workspace,
                                    size_t workspace_bytes, void* stream);

/*
 * The hybrid merge of the two gated branch outputs (Video DeltaNet summary,
 * section "how it differs": each branch has its own output projection and the
 * two are summed; VDN-H3 post, section "hybrid attention structure"):
 *   Y = O_soft W_soft^T + O_lin W_lin^T
 *   O_soft, O_lin  [M, K] bf16: the gated branch outputs with the heads
 *                  concatenated (a [B, T*U, H, d] output is [M = B*T*U, K = H*d])
 *   W_soft, W_lin  [N, K] bf16: the output projections, [out, in] as a linear
 *                  layer stores them
 *   Y              [M, N] bf16 (fp32 accumulation on the tensor cores)
 *   workspace      >= 256 bytes of device memory, 256-byte aligned: the call's
 *                  device status word (cleared here; non-zero after a bounded
 *                  device-side wait gave up)
 * N and K must be multiples of 8 and every pointer 16-byte aligned, else
 * VDA_ERR_INVALID_ARG / VDA_ERR_ALIGNMENT before any launch. Only enqueues work.
 */
vda_status vda_hybrid_merge(const void* O_soft, const void* W_soft, const void* O_lin, const void* W_lin, void* Y,
                            int M, int N, int K, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Regions of the workspace, for staged parity checks and debugging. Every
 * float32 d x d matrix below (one per slot, chunk or direction) is stored in
 * column quads: element (i, j) at float index ((j / 4) * d + i) * 4 + j % 4 of
 * its matrix, so that threads owning consecutive rows access contiguous
 * memory. The shapes name the logical indices, outermost first.
 */
typedef enum vda_region {
  VDA_REGION_STATUS = 0, /* uint32 device status word (+ padding to byte 256), then uint32 [B, H, T-1]
                            slot-ready words of the solve, then uint32 [B, H, T-1] slot counts of the
                            statistics kernel: vda_prepare clears the region; the tensor-core sweep
                            solve sets word (b, h, s) to 1 once everything the scan reads from slot s
                            is written (the hi/lo images of M_t, or of P_t under "inject=scan", and
                            C_t where it is formed; S_T for the text slot), and the tensor-core frame
                            scan (which may start while the solve's last CTAs run) reads a slot only
                            after its word is 1 */
  VDA_REGION_A = 1,      /* float32 [B, H, T-1, d_k, d_k]; slot 0 = text, slot t = frame t */
  VDA_REGION_B = 2,      /* float32 [B, H, T-1, d_v, d_k]; same slots */
  VDA_REGION_M = 3,      /* float32 [B, H, T-1, d_k, d_k]; slot t = M_t (slot 0 unused); written by the
                            CUDA-core solve only: the tensor-core solves write M_t as the hi/lo images of
                            VDA_REGION_M_SPLIT, the form their scan reads */
  VDA_REGION_C = 4,      /* float32 [B, H, T-1, d_v, d_k]; slot 0 = S_T, slot t = C_t. When vda_describe
                            reports "inject=scan", only slot 0 is written: the tensor-core frame scan
                            forms each step as (S Diag(alpha_t) + B_t) P_t and C_t never exists */
  VDA_REGION_S_FWD = 5,  /* float32 [B, H, J, d_v, d_k]; forward readout state of chunk j */
  VDA_REGION_S_REV = 6,  /* float32 [B, H, J, d_v, d_k]; reverse readout state of chunk j */
  VDA_REGION_K_PREP = 7, /* storage dtype [B, H, T, U, d]; prepared K (VDA_PREP_CONV only) */
  VDA_REGION_V_PREP = 8, /* storage dtype [B, H, T, U, d]; prepared V (VDA_PREP_CONV only) */
  VDA_REGION_KT_PREP = 9,  /* storage dtype [B, H, L, d]; prepared K_txt (VDA_PREP_CONV only) */
  VDA_REGION_VT_PREP = 10, /* storage dtype [B, H, L, d]; prepared V_txt (VDA_PREP_CONV only) */
  VDA_REGION_M_SPLIT = 11, /* bf16 [B, H, T-1, 2, d*d]: M_t as hi + lo parts (M = hi + lo to ~2^-16),
                              each in the swizzled shared-memory operand layout of the tensor-core
                              scan: element (i, j) at byte (j / 64) * d * 128 + i * 128 +
                              (((j % 64) / 8) XOR (i % 8)) * 16 + (j % 8) * 2 of its image
                              (written by the tensor-core solves, unused otherwise). Under
                              "inject=scan" the images hold P_t = (I + A_t)^-1 itself, and
                              M_t = Diag(alpha_t) P_t */
  VDA_REGION_CHUNK_M = 12, /* bf16 [B, H, 2, J, 2, d*d]: per direction and chunk, the composed transition
                              of the chunk's frames (hi, lo operand images; identity for empty chunks) */
  VDA_REGION_CHUNK_C = 13, /* float32 [B, H, 2, J, d_v, d_k]: the composed injection of those frames */
  VDA_NUM_REGIONS = 14
} vda_region;

/* Byte offset and size of a region inside the workspace (size 0 if unused). Host-only. */
vda_status vda_workspace_region(const vda_config* cfg, int region, size_t* offset, size_t* bytes);

/* Static text for a status code. */
const char* vda_status_string(vda_status s);

/* Text of the last error recorded on this context ("" if none). */
const char* vda_last_error(const vda_ctx* ctx);

/*
 * Per-kernel timing with CUDA events recorded on the launching stream around
 * every kernel this context launches. Enabling resets the accumulators.
 * vda_profile_read synchronises the recorded events, returns the number of
 * launches and their summed duration (ms) for kernel id `kernel`, and the
 * kernel's name through *name (static storage). Ids run 0 .. vda_num_kernels()-1.
 */
vda_status vda_profile_enable(vda_ctx* ctx, int enable);
int vda_num_kernels(void);
vda_status vda_profile_read(vda_ctx* ctx, int kernel, const char** name, int* launches,
                            double* total_ms);

/* Number of kernels this context has launched since it was created. */
vda_status vda_launch_count(const vda_ctx* ctx, uint64_t* launches);

/* Which implementation each stage uses for cfg: writes a static string such as
 * "gram=tcgen05 solve=simt scan=simt readout=tcgen05". Host-only. */
vda_status vda_describe(const vda_config* cfg, const char** text);

/*
 * Failure-detection self test: launch one kernel that waits, with an iteration
 * limit `spins`, on a device flag that nothing sets, then writes
 * VDA_ERR_TIMEOUT into the uint32 at `status_dev` (device pointer) and returns.
 * Lets a test check that a bounded wait gives up and reports without faulting.
 */
vda_status vda_selftest_bounded_wait(uint32_t* status_dev, uint64_t spins, void* stream);

/*
 * Numerical self test of the sweep solve's pivot reciprocal: y[i] = r(x[i]) for
 * i < n, where r is the device function every pivot step of the tensor-core
 * sweep uses (the hardware's approximate reciprocal refined by one Newton-Raphson
 * step). x and y are device float32 arrays of n values. Lets a test bound r's
 * error against the correctly rounded 1/x over the pivot range (x >= 1).
 */
vda_status vda_selftest_recip(const float* x, float* y, int n, void* stream);

/*
 * The whole path (vda_prepare, vda_scan_bidir, vda_readout) in one call whose
 * scratch lives in a static device array owned by the library, for callers that
 * cannot allocate device memory: code that has no allocator at hand (a plugin
 * given only its input and output buffers by a host application), a process that
 * must not grow its device footprint after start-up, or a caller that must avoid
 * the allocator's implicit synchronisation. The method pages have no counterpart
 * of this call; it is a deployment convenience.
 *  - Capacity: vda_static_workspace_capacity() bytes (64 MiB) on every device that
 *    loads the library, held until the process exits. A cfg whose
 *    vda_workspace_size() exceeds it returns VDA_ERR_WORKSPACE_TOO_SMALL before any
 *    launch (the small workloads fit; the full-size clips need the caller-workspace
 *    calls above).
 *  - The first call on a device looks up that device's address of the array
 *    (cudaGetSymbolAddress); make that first call before any stream capture.
 *  - Every call shares the one array and leaves its contents behind: calls that
 *    overlap on the GPU (other streams, other host threads) race and corrupt each
 *    other's results, so serialise them.
 *  - No cudaMalloc, cudaFree or allocating library routine is called.
 *  - A bounded device-side wait that gives up does not change the return code
 *    (the call only enqueues work): read it with vda_static_workspace_poll.
 * Arguments are those of vda_prepare and vda_readout; the call only enqueues
 * work on `stream`.
 */
size_t vda_static_workspace_capacity(void);
vda_status vda_run_static_workspace(const vda_config* cfg, const void* Q, const void* K, const void* V,
                                    const void* K_txt, const void* V_txt, const float* alpha,
                                    const float* beta, const float* beta_txt, const float* conv_w,
                                    const void* gate, void* O, void* stream);

/*
 * The device status word of the static array, for vda_run_static_workspace
 * what vda_poll_device_status is for the caller-workspace calls: synchronise
 * `stream`, read the word, clear it, and return VDA_ERR_TIMEOUT if a bounded
 * device-side wait of the last call on this device gave up, VDA_OK otherwise.
 * Each vda_run_static_workspace call clears the word when it starts, so poll
 * after a call and before the next one. Allocates nothing; the first use on a
 * device looks up the array's address as vda_run_static_workspace does.
 */
vda_status vda_static_workspace_poll(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* VDA_H_ */
