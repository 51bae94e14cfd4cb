// Host side of the C ABI declared in include/vda.h: argument validation,
// workspace carving, stage orchestration, launch accounting and per-kernel
// event timing. Every call only enqueues work on the caller's stream.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <mutex>
#include <set>
#include <string>
#include <type_traits>
#include <utility>
#include <vector>

#include "internal.h"

namespace vda {

const char* kernel_name(int id) {
  static const char* names[K_NUM_KERNELS] = {
      "prep_video", "prep_text", "gram_simt", "gram_tc", "solve_simt",
      "scan_simt", "readout_simt", "readout_tc", "zero_anchors", "solve_tc", "scan_tc", "compose_tc",
      "solve_chol_tc", "window_attn_tc", "merge_tc", "frame_bwd_simt", "solve_tc_frames", "readout_fp8_tc",
      "gram_fp8_tc", "token_bwd_tc", "scan_split_tc"};
  return (id >= 0 && id < K_NUM_KERNELS) ? names[id] : "?";
}

cudaError_t set_max_dynamic_smem(const void* func, int bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({func, dev})) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  // Every tensor-core kernel asks for the largest shared-memory carveout, so that
  // CTAs of kernels that overlap (the statistics kernel and the compact solve
  // CTAs beside it, the solve's last wave and the scan) find the SM in the same
  // configuration and can be resident together.
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) done.insert({func, dev});
  return e;
}

}  // namespace vda

using namespace vda;

struct EventPair {
  cudaEvent_t a, b;
};

struct vda_ctx {
  vda_config cfg;
  Problem p;
  bool prepared = false, scanned = false;
  std::string err;
  uint64_t launches = 0;
  bool prof = false;
  std::vector<EventPair> pending[K_NUM_KERNELS];
  std::vector<EventPair> pool;
  int prof_launches[K_NUM_KERNELS] = {};
  double prof_ms[K_NUM_KERNELS] = {};
  uint32_t* attn_status = nullptr;  // status word of the last vda_window_attention call
};

namespace {

constexpr size_t kRegionAlign = 1024;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int d_of(const vda_config& c) { return c.d_k; }
int J_of(const vda_config& c) { return (c.T + c.chunk - 1) / c.chunk; }

vda_status check_config(const vda_config* c, std::string* why) {
  auto bad = [&](const char* m) {
    if (why) *why = m;
    return VDA_ERR_INVALID_ARG;
  };
  if (!c) return bad("config is NULL");
  if (c->B < 1 || c->H < 1) return bad("B and H must be >= 1");
  if (c->T < 3) return bad("T must be >= 3 (two anchors and one scanned frame)");
  if (c->grid_h < 1 || c->grid_w < 1) return bad("grid_h and grid_w must be >= 1");
  if ((long long)c->grid_h * c->grid_w != c->U) return bad("U must equal grid_h * grid_w");
  if (c->L < 1) return bad("L (text tokens) must be >= 1");
  if (c->chunk < 1) return bad("chunk must be >= 1");
  if (c->dtype != VDA_F32 && c->dtype != VDA_BF16) return bad("dtype must be VDA_F32 or VDA_BF16");
  if (!(c->l2_eps >= 0.f) || !(c->rms_eps >= 0.f)) return bad("eps must be >= 0");
  if (c->flags &
      ~(VDA_PREP_CONV | VDA_READOUT_NORM_GATE | VDA_SOLVE_CHOLESKY | VDA_SCAN_CHUNKED | VDA_SCAN_SPLIT | VDA_FORCE_SIMT))
    return bad("unknown flag bits");
  if (c->d_k != c->d_v) {
    if (why) *why = "d_k != d_v is not supported";
    return VDA_ERR_UNSUPPORTED;
  }
  const int d = c->d_k;
  if (d != 16 && d != 32 && d != 64 && d != 128) {
    if (why) *why = "d must be one of 16, 32, 64, 128";
    return VDA_ERR_UNSUPPORTED;
  }
  // Launch-grid limits, checked here so that no call fails after it has begun
  // to enqueue work: the conv prep runs grid rows on grid.y and (b, h, K|V) on
  // grid.z; the chunk composition runs (b, h) on grid.z.
  if ((c->flags & VDA_PREP_CONV) && (c->grid_h > 65535 || (long long)c->B * c->H * 2 > 65535)) {
    if (why) *why = "conv prep needs grid_h <= 65535 and 2 * B * H <= 65535";
    return VDA_ERR_UNSUPPORTED;
  }
  if ((c->flags & VDA_SCAN_CHUNKED) && (long long)c->B * c->H > 65535) {
    if (why) *why = "the chunked scan needs B * H <= 65535";
    return VDA_ERR_UNSUPPORTED;
  }
  if (c->H_total < 0 || c->h0 < 0) return bad("H_total and h0 must be >= 0");
  if (c->H_total == 0 && c->h0 != 0) return bad("h0 must be 0 when H_total is 0 (all heads)");
  if (c->H_total > 0 && (long long)c->h0 + c->H > c->H_total) return bad("h0 + H must be <= H_total");
  const long long tokens = (long long)c->B * c->T * c->U * (c->H_total > 0 ? c->H_total : c->H) * d;
  if (tokens >= (1LL << 40)) return bad("tensor too large");
  return VDA_OK;
}

struct Layout {
  size_t off[VDA_NUM_REGIONS];
  size_t bytes[VDA_NUM_REGIONS];
  size_t total;
};

Layout make_layout(const vda_config& c) {
  Layout L{};
  const size_t d = (size_t)d_of(c), BH = (size_t)c.B * c.H;
  const size_t esz = c.dtype == VDA_BF16 ? 2 : 4;
  const bool prep = (c.flags & VDA_PREP_CONV) != 0;
  // Status word (+ padding), then at byte 256 the [B,H,T-1] uint32 slot-ready
  // words of the solve, then those of the statistics kernel.
  L.bytes[VDA_REGION_STATUS] = 256 + 2 * align_up(BH * (c.T - 1) * 4, 256);
  L.bytes[VDA_REGION_A] = BH * (c.T - 1) * d * d * 4;
  L.bytes[VDA_REGION_B] = BH * (c.T - 1) * d * d * 4;
  L.bytes[VDA_REGION_M] = BH * (c.T - 1) * d * d * 4;
  L.bytes[VDA_REGION_C] = BH * (c.T - 1) * d * d * 4;
  L.bytes[VDA_REGION_S_FWD] = BH * J_of(c) * d * d * 4;
  L.bytes[VDA_REGION_S_REV] = BH * J_of(c) * d * d * 4;
  L.bytes[VDA_REGION_K_PREP] = prep ? BH * c.T * (size_t)c.U * d * esz : 0;
  L.bytes[VDA_REGION_V_PREP] = prep ? BH * c.T * (size_t)c.U * d * esz : 0;
  L.bytes[VDA_REGION_KT_PREP] = prep ? BH * c.L * d * esz : 0;
  L.bytes[VDA_REGION_VT_PREP] = prep ? BH * c.L * d * esz : 0;
  L.bytes[VDA_REGION_M_SPLIT] = BH * (c.T - 1) * 2 * d * d * 2;
  L.bytes[VDA_REGION_CHUNK_M] = BH * 2 * J_of(c) * 2 * d * d * 2;
  L.bytes[VDA_REGION_CHUNK_C] = BH * 2 * J_of(c) * d * d * 4;
  size_t o = 0;
  for (int r = 0; r < VDA_NUM_REGIONS; ++r) {
    L.off[r] = o;
    o = align_up(o + L.bytes[r], kRegionAlign);
  }
  L.total = o;
  return L;
}

bool aligned16(const void* ptr) { return ((uintptr_t)ptr & 15) == 0; }

vda_status fail(vda_ctx* ctx, vda_status s, const std::string& msg) {
  if (ctx) ctx->err = msg;
  return s;
}

vda_status cuda_fail(vda_ctx* ctx, cudaError_t e, const char* what) {
  std::string m = std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
  return fail(ctx, VDA_ERR_CUDA, m);
}

EventPair take_pair(vda_ctx* ctx) {
  if (!ctx->pool.empty()) {
    EventPair e = ctx->pool.back();
    ctx->pool.pop_back();
    return e;
  }
  EventPair e{};
  cudaEventCreate(&e.a);
  cudaEventCreate(&e.b);
  return e;
}

// Fold finished timing pairs into the accumulators (synchronising on them).
void drain_events(vda_ctx* ctx) {
  for (int k = 0; k < K_NUM_KERNELS; ++k) {
    for (EventPair& e : ctx->pending[k]) {
      float ms = 0.f;
      if (cudaEventSynchronize(e.b) == cudaSuccess && cudaEventElapsedTime(&ms, e.a, e.b) == cudaSuccess) {
        ctx->prof_launches[k] += 1;
        ctx->prof_ms[k] += ms;
      }
      ctx->pool.push_back(e);
    }
    ctx->pending[k].clear();
  }
}

template <typename F>
vda_status run_kernel(vda_ctx* ctx, int id, cudaStream_t s, F&& launch) {
  EventPair ev{};
  const bool prof = ctx->prof;
  if (prof) {
    if (ctx->pending[id].size() > 4096) drain_events(ctx);
    ev = take_pair(ctx);
    cudaEventRecord(ev.a, s);
  }
  cudaError_t e = launch();
  if (e != cudaSuccess) return cuda_fail(ctx, e, kernel_name(id));
  ctx->launches += 1;
  if (prof) {
    cudaEventRecord(ev.b, s);
    ctx->pending[id].push_back(ev);
  }
  return VDA_OK;
}

bool use_simt_only(const vda_config& c) { return (c.flags & VDA_FORCE_SIMT) != 0; }

int heads_total(const vda_config& c) { return c.H_total > 0 ? c.H_total : c.H; }

// A token-tensor pointer advanced to head h0 of its rows.
template <typename P>
P head_slice(const vda_config& c, P ptr) {
  if (ptr == nullptr) return ptr;
  const size_t esz = c.dtype == VDA_BF16 ? 2 : 4;
  using Byte = typename std::conditional<std::is_const<typename std::remove_pointer<P>::type>::value, const char,
                                         char>::type;
  return reinterpret_cast<P>(reinterpret_cast<Byte*>(ptr) + (size_t)c.h0 * c.d_k * esz);
}

}  // namespace

extern "C" {

const char* vda_status_string(vda_status s) {
  switch (s) {
    case VDA_OK: return "VDA_OK";
    case VDA_ERR_INVALID_ARG: return "VDA_ERR_INVALID_ARG";
    case VDA_ERR_UNSUPPORTED: return "VDA_ERR_UNSUPPORTED";
    case VDA_ERR_ALIGNMENT: return "VDA_ERR_ALIGNMENT";
    case VDA_ERR_WORKSPACE_TOO_SMALL: return "VDA_ERR_WORKSPACE_TOO_SMALL";
    case VDA_ERR_CUDA: return "VDA_ERR_CUDA";
    case VDA_ERR_TIMEOUT: return "VDA_ERR_TIMEOUT";
    case VDA_ERR_STATE: return "VDA_ERR_STATE";
  }
  return "VDA_ERR_UNKNOWN";
}

vda_status vda_create(const vda_config* cfg, vda_ctx** out) {
  if (!out) return VDA_ERR_INVALID_ARG;
  *out = nullptr;
  vda_status st = check_config(cfg, nullptr);
  if (st != VDA_OK) return st;
  vda_ctx* ctx = new (std::nothrow) vda_ctx();
  if (!ctx) return VDA_ERR_UNSUPPORTED;  // host allocation failed
  ctx->cfg = *cfg;
  *out = ctx;
  return VDA_OK;
}

vda_status vda_destroy(vda_ctx* ctx) {
  if (!ctx) return VDA_ERR_INVALID_ARG;
  for (int k = 0; k < K_NUM_KERNELS; ++k)
    for (EventPair& e : ctx->pending[k]) ctx->pool.push_back(e);
  for (EventPair& e : ctx->pool) {
    cudaEventDestroy(e.a);
    cudaEventDestroy(e.b);
  }
  delete ctx;
  return VDA_OK;
}

vda_status vda_workspace_size(const vda_config* cfg, size_t* bytes) {
  if (!bytes) return VDA_ERR_INVALID_ARG;
  vda_status st = check_config(cfg, nullptr);
  if (st != VDA_OK) return st;
  *bytes = make_layout(*cfg).total;
  return VDA_OK;
}

vda_status vda_workspace_region(const vda_config* cfg, int region, size_t* offset, size_t* bytes) {
  if (!offset || !bytes || region < 0 || region >= VDA_NUM_REGIONS) return VDA_ERR_INVALID_ARG;
  vda_status st = check_config(cfg, nullptr);
  if (st != VDA_OK) return st;
  Layout L = make_layout(*cfg);
  *offset = L.off[region];
  *bytes = L.bytes[region];
  return VDA_OK;
}

const char* vda_last_error(const vda_ctx* ctx) { return ctx ? ctx->err.c_str() : ""; }

// Whether the sweep solve leaves the frames' injections to the tensor-core
// frame scan (S M_t + C_t = (S Diag(alpha_t) + B_t) P_t): writes P_t's images
// and no C_t. Not with the chunked scan, which composes M_t and C_t.
static bool pform_of(const vda_config& c, const Problem& p) {
  if (use_simt_only(c) || !solve_tc_supported(p) || !scan_tc_supported(p)) return false;
  if (c.flags & VDA_SOLVE_CHOLESKY) return false;
  const bool chunked = (c.flags & VDA_SCAN_CHUNKED) && c.chunk > 1 && J_of(c) >= 3;
  return !chunked;
}

vda_status vda_describe(const vda_config* cfg, const char** text) {
  if (!text) return VDA_ERR_INVALID_ARG;
  vda_status st = check_config(cfg, nullptr);
  if (st != VDA_OK) return st;
  Problem p{};
  p.D = cfg->d_k;
  p.bf16 = cfg->dtype == VDA_BF16;
  p.flags = cfg->flags;
  const bool simt = use_simt_only(*cfg);
  const bool g = !simt && gram_tc_supported(p), r = !simt && readout_tc_supported(p);
  const bool v = !simt && solve_tc_supported(p), n = !simt && scan_tc_supported(p);
  const bool chol = v && (cfg->flags & VDA_SOLVE_CHOLESKY);
  const bool pf = pform_of(*cfg, p);
  p.pform = pf ? 1 : 0;
  const bool split = n && (cfg->flags & VDA_SCAN_SPLIT) && scan_split_tc_supported(p);
  static char table[2][2][2][2][2][2][2][120];
  char* t = table[g][v][chol][n][split][r][pf];
  std::snprintf(t, 120, "gram=%s solve=%s scan=%s readout=%s%s", g ? "tcgen05" : "simt",
                v ? (chol ? "tcgen05-cholesky" : "tcgen05") : "simt",
                n ? (split ? "tcgen05-split" : "tcgen05") : "simt", r ? "tcgen05" : "simt", pf ? " inject=scan" : "");
  *text = t;
  return VDA_OK;
}

vda_status vda_prepare(vda_ctx* ctx, const void* Q, const void* K, const void* V, const void* K_txt,
                       const void* V_txt, const float* alpha, const float* beta, const float* beta_txt,
                       const float* conv_w, void* workspace, size_t workspace_bytes, void* stream) {
  if (!ctx) return VDA_ERR_INVALID_ARG;
  ctx->prepared = ctx->scanned = false;
  const vda_config& c = ctx->cfg;
  const bool prep = (c.flags & VDA_PREP_CONV) != 0;
  if (!Q || !K || !V || !K_txt || !V_txt || !alpha || !beta || !beta_txt || !workspace)
    return fail(ctx, VDA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (prep && !conv_w) return fail(ctx, VDA_ERR_INVALID_ARG, "conv_w is required with VDA_PREP_CONV");
  const void* ptrs[] = {Q, K, V, K_txt, V_txt, alpha, beta, beta_txt};
  for (const void* q : ptrs)
    if (!aligned16(q)) return fail(ctx, VDA_ERR_ALIGNMENT, "token tensors, alpha and beta must be 16-byte aligned");
  if (prep && !aligned16(conv_w)) return fail(ctx, VDA_ERR_ALIGNMENT, "conv_w must be 16-byte aligned");
  if (((uintptr_t)workspace & 255) != 0) return fail(ctx, VDA_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  const Layout L = make_layout(c);
  if (workspace_bytes < L.total) return fail(ctx, VDA_ERR_WORKSPACE_TOO_SMALL, "workspace smaller than vda_workspace_size()");

  char* ws = static_cast<char*>(workspace);
  Problem& p = ctx->p;
  p = Problem{};
  p.B = c.B; p.H = c.H; p.T = c.T; p.U = c.U; p.L = c.L; p.D = c.d_k; p.c = c.chunk; p.J = J_of(c);
  p.Ht = heads_total(c);
  // Token tensors: advance to this context's first head (h0 * d elements; a
  // multiple of 32 bytes, so 16-byte alignment is kept).
  Q = head_slice(c, Q);
  K = head_slice(c, K);
  V = head_slice(c, V);
  K_txt = head_slice(c, K_txt);
  V_txt = head_slice(c, V_txt);
  p.gh = c.grid_h; p.gw = c.grid_w;
  p.bf16 = c.dtype == VDA_BF16;
  p.flags = c.flags;
  p.l2_eps = c.l2_eps;
  p.rms_eps = c.rms_eps;
  p.alpha = alpha; p.beta = beta; p.beta_txt = beta_txt; p.Q = Q;
  p.status = reinterpret_cast<uint32_t*>(ws + L.off[VDA_REGION_STATUS]);
  p.A = reinterpret_cast<float*>(ws + L.off[VDA_REGION_A]);
  p.Bm = reinterpret_cast<float*>(ws + L.off[VDA_REGION_B]);
  p.M = reinterpret_cast<float*>(ws + L.off[VDA_REGION_M]);
  p.C = reinterpret_cast<float*>(ws + L.off[VDA_REGION_C]);
  p.Sf = reinterpret_cast<float*>(ws + L.off[VDA_REGION_S_FWD]);
  p.Sr = reinterpret_cast<float*>(ws + L.off[VDA_REGION_S_REV]);
  p.Msplit = ws + L.off[VDA_REGION_M_SPLIT];
  p.CMi = ws + L.off[VDA_REGION_CHUNK_M];
  p.CC = reinterpret_cast<float*>(ws + L.off[VDA_REGION_CHUNK_C]);
  p.spin_limit = 2000000000ull;  // 2 s of wall time per device-side wait
  const long long D = p.D, H = p.H, T = p.T, U = p.U, Lt = p.L, Ht = p.Ht;
  if (prep) {
    p.Kp = ws + L.off[VDA_REGION_K_PREP];
    p.Vp = ws + L.off[VDA_REGION_V_PREP];
    p.Ktp = ws + L.off[VDA_REGION_KT_PREP];
    p.Vtp = ws + L.off[VDA_REGION_VT_PREP];
    p.Kv = TokView{p.Kp, H * T * U * D, T * U * D, U * D, D};
    p.Vv = TokView{p.Vp, H * T * U * D, T * U * D, U * D, D};
    p.Kt = TokView{p.Ktp, H * Lt * D, Lt * D, 0, D};
    p.Vt = TokView{p.Vtp, H * Lt * D, Lt * D, 0, D};
  } else {
    p.Kv = TokView{K, T * U * Ht * D, D, U * Ht * D, Ht * D};
    p.Vv = TokView{V, T * U * Ht * D, D, U * Ht * D, Ht * D};
    p.Kt = TokView{K_txt, Lt * Ht * D, D, 0, Ht * D};
    p.Vt = TokView{V_txt, Lt * Ht * D, D, 0, Ht * D};
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Clears the status word and the slot-ready words the solve raises.
  cudaError_t e = cudaMemsetAsync(p.status, 0, L.bytes[VDA_REGION_STATUS], s);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "status reset");
  vda_status st;
  if (prep) {
    st = run_kernel(ctx, K_PREP_VIDEO, s, [&] { return launch_prep_video(p, K, V, conv_w, s); });
    if (st != VDA_OK) return st;
    st = run_kernel(ctx, K_PREP_TEXT, s, [&] { return launch_prep_text(p, K_txt, V_txt, s); });
    if (st != VDA_OK) return st;
  }
  const bool gram_tc = !use_simt_only(c) && gram_tc_supported(p);
  const bool sweep_tc = !use_simt_only(c) && solve_tc_supported(p) && !(c.flags & VDA_SOLVE_CHOLESKY);
  // Per-slot ready words let the sweep solve overlap the statistics kernel's
  // last units, and the frame scan the solve's last CTAs.
  const size_t words = align_up((size_t)p.B * p.H * (p.T - 1) * 4, 256) / 4;
  if (gram_tc && sweep_tc) p.gready = p.status + 64 + words;
  if (gram_tc)
    st = run_kernel(ctx, K_GRAM_TC, s, [&] { return launch_gram_tc(p, s); });
  else
    st = run_kernel(ctx, K_GRAM_SIMT, s, [&] { return launch_gram_simt(p, s); });
  if (st != VDA_OK) return st;
  if (!use_simt_only(c) && solve_tc_supported(p) && (c.flags & VDA_SOLVE_CHOLESKY))
    st = run_kernel(ctx, K_SOLVE_CHOL_TC, s, [&] { return launch_solve_chol_tc(p, s); });
  else if (sweep_tc) {
    p.ready = p.status + 64;
    p.pform = pform_of(c, p) ? 1 : 0;
    st = run_kernel(ctx, K_SOLVE_TC, s, [&] { return launch_solve_tc(p, s, 0); });
    if (st == VDA_OK && p.pform && p.T > 2)
      st = run_kernel(ctx, K_SOLVE_TC_FRAMES, s, [&] { return launch_solve_tc(p, s, 1); });
  }
  else
    st = run_kernel(ctx, K_SOLVE_SIMT, s, [&] { return launch_solve_simt(p, s); });
  if (st != VDA_OK) return st;
  ctx->prepared = true;
  return VDA_OK;
}

vda_status vda_prepare_fp8(vda_ctx* ctx, const void* K8, const void* V8, const float* kv_scale, const void* Kt8,
                           const void* Vt8, const float* kvt_scale, const float* alpha, const float* beta,
                           const float* beta_txt, void* workspace, size_t workspace_bytes, void* stream) {
  if (!ctx) return VDA_ERR_INVALID_ARG;
  ctx->prepared = ctx->scanned = false;
  const vda_config& c = ctx->cfg;
  if (!K8 || !V8 || !kv_scale || !Kt8 || !Vt8 || !kvt_scale || !alpha || !beta || !beta_txt || !workspace)
    return fail(ctx, VDA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (c.d_k != 128 || c.dtype != VDA_BF16 || (c.flags & (VDA_PREP_CONV | VDA_FORCE_SIMT)))
    return fail(ctx, VDA_ERR_UNSUPPORTED, "the FP8 statistics need d = 128, bf16 outputs and no conv prep");
  const void* a16[] = {K8, V8, Kt8, Vt8, alpha, beta, beta_txt};
  for (const void* q : a16)
    if (!aligned16(q)) return fail(ctx, VDA_ERR_ALIGNMENT, "token tensors, alpha and beta must be 16-byte aligned");
  if (((uintptr_t)kv_scale & 3) || ((uintptr_t)kvt_scale & 3))
    return fail(ctx, VDA_ERR_ALIGNMENT, "the scales must be 4-byte aligned");
  if (((uintptr_t)workspace & 255) != 0) return fail(ctx, VDA_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  const Layout L = make_layout(c);
  if (workspace_bytes < L.total) return fail(ctx, VDA_ERR_WORKSPACE_TOO_SMALL, "workspace smaller than vda_workspace_size()");
  char* ws = static_cast<char*>(workspace);
  Problem& p = ctx->p;
  p = Problem{};
  p.B = c.B; p.H = c.H; p.T = c.T; p.U = c.U; p.L = c.L; p.D = c.d_k; p.c = c.chunk; p.J = J_of(c);
  p.gh = c.grid_h; p.gw = c.grid_w; p.Ht = heads_total(c);
  p.bf16 = 1;
  p.flags = c.flags;
  p.l2_eps = c.l2_eps;
  p.rms_eps = c.rms_eps;
  p.alpha = alpha; p.beta = beta; p.beta_txt = beta_txt; p.Q = nullptr;
  p.status = reinterpret_cast<uint32_t*>(ws + L.off[VDA_REGION_STATUS]);
  p.A = reinterpret_cast<float*>(ws + L.off[VDA_REGION_A]);
  p.Bm = reinterpret_cast<float*>(ws + L.off[VDA_REGION_B]);
  p.M = reinterpret_cast<float*>(ws + L.off[VDA_REGION_M]);
  p.C = reinterpret_cast<float*>(ws + L.off[VDA_REGION_C]);
  p.Sf = reinterpret_cast<float*>(ws + L.off[VDA_REGION_S_FWD]);
  p.Sr = reinterpret_cast<float*>(ws + L.off[VDA_REGION_S_REV]);
  p.Msplit = ws + L.off[VDA_REGION_M_SPLIT];
  p.CMi = ws + L.off[VDA_REGION_CHUNK_M];
  p.CC = reinterpret_cast<float*>(ws + L.off[VDA_REGION_CHUNK_C]);
  p.spin_limit = 2000000000ull;
  // One byte per channel: advance the e4m3 tensors to head h0 by h0 * d bytes,
  // the scales by h0 floats.
  const size_t hb = (size_t)c.h0 * c.d_k;
  K8 = static_cast<const char*>(K8) + hb;
  V8 = static_cast<const char*>(V8) + hb;
  Kt8 = static_cast<const char*>(Kt8) + hb;
  Vt8 = static_cast<const char*>(Vt8) + hb;
  kv_scale += c.h0;
  kvt_scale += c.h0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(p.status, 0, L.bytes[VDA_REGION_STATUS], s);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "status reset");
  const bool sweep_tc = solve_tc_supported(p) && !(c.flags & VDA_SOLVE_CHOLESKY);
  const size_t words = align_up((size_t)p.B * p.H * (p.T - 1) * 4, 256) / 4;
  if (sweep_tc) p.gready = p.status + 64 + words;
  // The slot exponents live in the M region (the tensor-core solves do not use it).
  int* exps = reinterpret_cast<int*>(p.M);
  vda_status st = run_kernel(ctx, K_GRAM_FP8_TC, s, [&] {
    return launch_gram_fp8_tc(p, K8, V8, kv_scale, Kt8, Vt8, kvt_scale, exps, s);
  });
  if (st != VDA_OK) return st;
  ctx->launches += 1;  // the exponent pre-pass
  if (c.flags & VDA_SOLVE_CHOLESKY)
    st = run_kernel(ctx, K_SOLVE_CHOL_TC, s, [&] { return launch_solve_chol_tc(p, s); });
  else {
    p.ready = p.status + 64;
    p.pform = pform_of(c, p) ? 1 : 0;
    st = run_kernel(ctx, K_SOLVE_TC, s, [&] { return launch_solve_tc(p, s, 0); });
    if (st == VDA_OK && p.pform && p.T > 2)
      st = run_kernel(ctx, K_SOLVE_TC_FRAMES, s, [&] { return launch_solve_tc(p, s, 1); });
  }
  if (st != VDA_OK) return st;
  ctx->prepared = true;
  return VDA_OK;
}

vda_status vda_scan_bidir(vda_ctx* ctx, void* stream) {
  if (!ctx) return VDA_ERR_INVALID_ARG;
  if (!ctx->prepared) return fail(ctx, VDA_ERR_STATE, "vda_scan_bidir before a successful vda_prepare");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  vda_status st;
  if (!use_simt_only(ctx->cfg) && scan_tc_supported(ctx->p)) {
    // Frame by frame by default (measured faster at the H3-like and long clips);
    // on request, compose each chunk's frame maps in parallel and scan the
    // chunks (with single-frame chunks composition is a copy: scan frames).
    const bool chunked = (ctx->cfg.flags & VDA_SCAN_CHUNKED) && ctx->p.c > 1 && ctx->p.J >= 3;
    if (chunked) {
      st = run_kernel(ctx, K_COMPOSE_TC, s, [&] { return launch_compose_tc(ctx->p, s); });
      if (st != VDA_OK) return st;
    }
    // On request, frame by frame on two-CTA clusters (each CTA half of every
    // state's columns). One CTA per (b, h, direction) is the default: each step
    // is bound by the MMA -> epilogue -> operand hand-offs, not by the MMAs or
    // the epilogue's arithmetic that the split halves, and the split adds the
    // exchange of the left factor's halves (measured at the H3-like clip:
    // 93 us against 71 us).
    if (!chunked && (ctx->cfg.flags & VDA_SCAN_SPLIT) && scan_split_tc_supported(ctx->p))
      st = run_kernel(ctx, K_SCAN_SPLIT_TC, s, [&] { return launch_scan_split_tc(ctx->p, s); });
    else
      st = run_kernel(ctx, K_SCAN_TC, s, [&] { return launch_scan_tc(ctx->p, s, chunked); });
  } else
    st = run_kernel(ctx, K_SCAN_SIMT, s, [&] { return launch_scan_simt(ctx->p, s); });
  if (st != VDA_OK) return st;
  ctx->scanned = true;
  return VDA_OK;
}

vda_status vda_readout(vda_ctx* ctx, const void* gate, void* O, void* stream) {
  if (!ctx) return VDA_ERR_INVALID_ARG;
  if (!ctx->scanned) return fail(ctx, VDA_ERR_STATE, "vda_readout before a successful vda_scan_bidir");
  if (!O) return fail(ctx, VDA_ERR_INVALID_ARG, "O is NULL");
  if ((ctx->cfg.flags & VDA_READOUT_NORM_GATE) && !gate)
    return fail(ctx, VDA_ERR_INVALID_ARG, "gate is required with VDA_READOUT_NORM_GATE");
  if (!aligned16(O) || (gate && !aligned16(gate))) return fail(ctx, VDA_ERR_ALIGNMENT, "O and gate must be 16-byte aligned");
  O = head_slice(ctx->cfg, O);
  gate = head_slice(ctx->cfg, gate);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Problem& p = ctx->p;
  // The tensor-core readout zeroes the anchor frames itself.
  if (!use_simt_only(ctx->cfg) && readout_tc_supported(p))
    return run_kernel(ctx, K_READOUT_TC, s, [&] { return launch_readout_tc(p, gate, O, s); });
  vda_status st = run_kernel(ctx, K_ZERO_ANCHORS, s, [&] { return launch_zero_anchors(p, O, s); });
  if (st != VDA_OK) return st;
  return run_kernel(ctx, K_READOUT_SIMT, s, [&] { return launch_readout_simt(p, gate, O, s); });
}

vda_status vda_readout_fp8(vda_ctx* ctx, const void* Q8, const float* q_scale, void* O, void* stream) {
  if (!ctx) return VDA_ERR_INVALID_ARG;
  if (!ctx->scanned) return fail(ctx, VDA_ERR_STATE, "vda_readout_fp8 before a successful vda_scan_bidir");
  if (!Q8 || !q_scale || !O) return fail(ctx, VDA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned16(Q8) || !aligned16(O) || ((uintptr_t)q_scale & 3) != 0)
    return fail(ctx, VDA_ERR_ALIGNMENT, "Q8 and O must be 16-byte aligned, q_scale 4-byte aligned");
  const vda_config& c = ctx->cfg;
  if (use_simt_only(c) || !readout_fp8_tc_supported(ctx->p) || c.dtype != VDA_BF16)
    return fail(ctx, VDA_ERR_UNSUPPORTED, "the FP8 readout needs d = 128, bf16 output and no conv prep or gate");
  const char* q8 = static_cast<const char*>(Q8) + (size_t)c.h0 * c.d_k;  // one byte per channel
  const float* qs = q_scale + c.h0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return run_kernel(ctx, K_READOUT_FP8_TC, s,
                    [&] { return launch_readout_fp8_tc(ctx->p, q8, qs, head_slice(c, O), s); });
}

vda_status vda_poll_device_status(vda_ctx* ctx, void* stream) {
  if (!ctx) return VDA_ERR_INVALID_ARG;
  if (!ctx->p.status && !ctx->attn_status) return fail(ctx, VDA_ERR_STATE, "no workspace bound yet");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  bool timeout = false;
  for (uint32_t* w : {ctx->p.status, ctx->attn_status}) {
    if (!w) continue;
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, w, sizeof(word), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "status read");
    if (word != 0) {
      e = cudaMemsetAsync(w, 0, sizeof(word), s);
      if (e != cudaSuccess) return cuda_fail(ctx, e, "status clear");
      timeout = true;
    }
  }
  if (timeout) return fail(ctx, VDA_ERR_TIMEOUT, "a bounded device-side wait gave up");
  return VDA_OK;
}

vda_status vda_window_attention(vda_ctx* ctx, const void* Q, const void* K, const void* V, const void* gate,
                                void* O, void* workspace, size_t workspace_bytes, void* stream) {
  if (!ctx) return VDA_ERR_INVALID_ARG;
  const vda_config& c = ctx->cfg;
  if (!Q || !K || !V || !O || !workspace) return fail(ctx, VDA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || (gate && !aligned16(gate)))
    return fail(ctx, VDA_ERR_ALIGNMENT, "Q, K, V, gate and O must be 16-byte aligned");
  if (((uintptr_t)workspace & 255) != 0) return fail(ctx, VDA_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  if (workspace_bytes < 256) return fail(ctx, VDA_ERR_WORKSPACE_TOO_SMALL, "the attention needs 256 bytes of workspace");
  Problem p{};
  p.B = c.B; p.H = c.H; p.T = c.T; p.U = c.U; p.L = c.L; p.D = c.d_k; p.c = c.chunk; p.J = J_of(c);
  p.gh = c.grid_h; p.gw = c.grid_w; p.Ht = heads_total(c);
  p.bf16 = c.dtype == VDA_BF16;
  p.flags = c.flags;
  p.status = static_cast<uint32_t*>(workspace);
  p.spin_limit = 2000000000ull;
  if (use_simt_only(c) || !window_attn_tc_supported(p))
    return fail(ctx, VDA_ERR_UNSUPPORTED, "the window attention needs bf16 storage and d in {64, 128}");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(p.status, 0, sizeof(uint32_t), s);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "status reset");
  ctx->attn_status = p.status;
  return run_kernel(ctx, K_WINDOW_ATTN_TC, s, [&] {
    return launch_window_attn_tc(p, head_slice(c, Q), head_slice(c, K), head_slice(c, V), head_slice(c, gate),
                                 head_slice(c, O), s);
  });
}

vda_status vda_profile_enable(vda_ctx* ctx, int enable) {
  if (!ctx) return VDA_ERR_INVALID_ARG;
  drain_events(ctx);
  for (int k = 0; k < K_NUM_KERNELS; ++k) {
    ctx->prof_launches[k] = 0;
    ctx->prof_ms[k] = 0.0;
  }
  ctx->prof = enable != 0;
  return VDA_OK;
}

int vda_num_kernels(void) { return K_NUM_KERNELS; }

vda_status vda_profile_read(vda_ctx* ctx, int kernel, const char** name, int* launches, double* total_ms) {
  if (!ctx || kernel < 0 || kernel >= K_NUM_KERNELS) return VDA_ERR_INVALID_ARG;
  drain_events(ctx);
  if (name) *name = kernel_name(kernel);
  if (launches) *launches = ctx->prof_launches[kernel];
  if (total_ms) *total_ms = ctx->prof_ms[kernel];
  return VDA_OK;
}

vda_status vda_launch_count(const vda_ctx* ctx, uint64_t* launches) {
  if (!ctx || !launches) return VDA_ERR_INVALID_ARG;
  *launches = ctx->launches;
  return VDA_OK;
}

vda_status vda_selftest_bounded_wait(uint32_t* status_dev, uint64_t spins, void* stream) {
  if (!status_dev || !aligned16(status_dev)) return VDA_ERR_INVALID_ARG;
  cudaError_t e = launch_selftest_wait(status_dev, spins, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VDA_OK : VDA_ERR_CUDA;
}

vda_status vda_frame_solve_backward(vda_ctx* ctx, const void* K, const void* V, const float* alpha,
                                    const float* beta, const float* S_prev, const float* dS, void* dK, void* dV,
                                    float* dalpha, float* dbeta, float* dS_prev, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  if (!ctx) return VDA_ERR_INVALID_ARG;
  const vda_config& c = ctx->cfg;
  if (c.flags & VDA_PREP_CONV)
    return fail(ctx, VDA_ERR_UNSUPPORTED, "the frame-step backward takes prepared keys and values (no conv prep)");
  const void* ptrs[] = {K, V, alpha, beta, S_prev, dS, dK, dV, dalpha, dbeta, dS_prev};
  for (const void* q : ptrs)
    if (!q) return fail(ctx, VDA_ERR_INVALID_ARG, "a required pointer is NULL");
  for (const void* q : ptrs)
    if (!aligned16(q)) return fail(ctx, VDA_ERR_ALIGNMENT, "every tensor must be 16-byte aligned");
  if (!workspace) return fail(ctx, VDA_ERR_INVALID_ARG, "workspace is NULL");
  if (((uintptr_t)workspace & 255) != 0) return fail(ctx, VDA_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  const Layout L = make_layout(c);
  if (workspace_bytes < L.total) return fail(ctx, VDA_ERR_WORKSPACE_TOO_SMALL, "workspace smaller than vda_workspace_size()");
  char* ws = static_cast<char*>(workspace);
  Problem p{};
  p.B = c.B; p.H = c.H; p.T = c.T; p.U = c.U; p.D = c.d_k; p.c = c.chunk; p.J = J_of(c);
  p.gh = c.grid_h; p.gw = c.grid_w; p.Ht = heads_total(c);
  p.bf16 = c.dtype == VDA_BF16;
  p.flags = c.flags;
  p.alpha = alpha;
  p.beta = beta;
  p.status = reinterpret_cast<uint32_t*>(ws + L.off[VDA_REGION_STATUS]);
  p.A = reinterpret_cast<float*>(ws + L.off[VDA_REGION_A]);
  p.Bm = reinterpret_cast<float*>(ws + L.off[VDA_REGION_B]);
  p.M = reinterpret_cast<float*>(ws + L.off[VDA_REGION_M]);
  p.C = reinterpret_cast<float*>(ws + L.off[VDA_REGION_C]);
  p.spin_limit = 2000000000ull;
  const long long D = p.D, T = p.T, U = p.U, Ht = p.Ht;
  K = head_slice(c, K);
  V = head_slice(c, V);
  dK = head_slice(c, dK);
  dV = head_slice(c, dV);
  p.Kv = TokView{K, T * U * Ht * D, D, U * Ht * D, Ht * D};
  p.Vv = TokView{V, T * U * Ht * D, D, U * Ht * D, Ht * D};
  // The statistics kernels also form a text slot (slot 0), which the backward
  // does not use: point it at one token of the video keys.
  p.L = 1;
  p.Kt = TokView{K, Ht * D, D, 0, Ht * D};
  p.Vt = TokView{V, Ht * D, D, 0, Ht * D};
  p.beta_txt = beta;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(p.status, 0, L.bytes[VDA_REGION_STATUS], s);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "status reset");
  ctx->p.status = p.status;  // for vda_poll_device_status
  vda_status st;
  if (!use_simt_only(c) && gram_tc_supported(p))
    st = run_kernel(ctx, K_GRAM_TC, s, [&] { return launch_gram_tc(p, s); });
  else
    st = run_kernel(ctx, K_GRAM_SIMT, s, [&] { return launch_gram_simt(p, s); });
  if (st != VDA_OK) return st;
  ctx->prepared = ctx->scanned = false;  // the workspace no longer holds a forward pass
  const bool tc = !use_simt_only(c) && token_bwd_tc_supported(p);
  st = run_kernel(ctx, K_FRAME_BWD_SIMT, s, [&] {
    return launch_frame_bwd_simt(p, S_prev, dS, dS_prev, dalpha, dbeta, dK, dV, s, !tc);
  });
  if (st != VDA_OK || !tc) return st;
  return run_kernel(ctx, K_TOKEN_BWD_TC, s, [&] { return launch_token_bwd_tc(p, K, V, dbeta, dK, dV, s); });
}

vda_status vda_hybrid_merge(const void* O_soft, const void* W_soft, const void* O_lin, const void* W_lin, void* Y,
                            int M, int N, int K, void* workspace, size_t workspace_bytes, void* stream) {
  if (!O_soft || !W_soft || !O_lin || !W_lin || !Y || !workspace) return VDA_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 1 || N % 8 != 0 || K % 8 != 0) return VDA_ERR_INVALID_ARG;
  if ((long long)M * N >= (1LL << 40) || (long long)M * K >= (1LL << 40)) return VDA_ERR_INVALID_ARG;
  const void* ptrs[] = {O_soft, W_soft, O_lin, W_lin, Y};
  for (const void* q : ptrs)
    if (!aligned16(q)) return VDA_ERR_ALIGNMENT;
  if (((uintptr_t)workspace & 255) != 0) return VDA_ERR_ALIGNMENT;
  if (workspace_bytes < 256) return VDA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), s) != cudaSuccess) return VDA_ERR_CUDA;
  cudaError_t e = launch_merge_tc(O_soft, W_soft, O_lin, W_lin, Y, M, N, K, K, status, 2000000000ull, s);
  return e == cudaSuccess ? VDA_OK : VDA_ERR_CUDA;
}

vda_status vda_selftest_recip(const float* x, float* y, int n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return VDA_ERR_INVALID_ARG;
  cudaError_t e = launch_recip_selftest(x, y, n, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VDA_OK : VDA_ERR_CUDA;
}

}  // extern "C"
