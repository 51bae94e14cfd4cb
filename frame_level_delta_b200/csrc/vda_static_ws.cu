// One-call entry point whose scratch memory is a static device array, for
// callers that cannot allocate device memory: code running where no allocator
// is available (a plugin handed only input and output buffers by its host
// application, a process that must not grow its device footprint after start
// up, or a caller that must not trigger the allocator's synchronisation). The
// caller still owns Q, K, V, ..., gate and O; everything in between lives in
// `g_static_workspace`, which every GPU that loads this library holds (64 MiB)
// until the process exits.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kStaticWorkspaceBytes = 64ull << 20;  // 64 MiB
__device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

constexpr int kMaxDevices = 64;
// Device address of the array, per device: set once under the mutex, then read
// without it.
std::atomic<void*> g_workspace_addr[kMaxDevices];
std::mutex g_lookup_mu;

// The current device's address of the array. In host code `g_static_workspace`
// names a host-side stand-in, not a device address: the runtime is asked once
// per device, with that device current.
vda_status workspace_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return VDA_ERR_CUDA;
  void* p = g_workspace_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lock(g_lookup_mu);
    p = g_workspace_addr[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
      if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr) return VDA_ERR_CUDA;
      g_workspace_addr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return VDA_OK;
}

}  // namespace

extern "C" {

size_t vda_static_workspace_capacity(void) { return kStaticWorkspaceBytes; }

vda_status vda_run_static_workspace(const vda_config* cfg, const void* Q, const void* K, const void* V,
                                    const void* K_txt, const void* V_txt, const float* alpha, const float* beta,
                                    const float* beta_txt, const float* conv_w, const void* gate, void* O,
                                    void* stream) {
  size_t need = 0;
  vda_status st = vda_workspace_size(cfg, &need);
  if (st != VDA_OK) return st;
  if (need > kStaticWorkspaceBytes) return VDA_ERR_WORKSPACE_TOO_SMALL;
  void* ws = nullptr;
  if ((st = workspace_address(&ws)) != VDA_OK) return st;
  vda_ctx* ctx = nullptr;
  st = vda_create(cfg, &ctx);
  if (st != VDA_OK) return st;
  // vda_prepare clears the status word and the slot-ready words at the start of
  // the workspace; every other region is fully written before it is read, so
  // stale contents of an earlier call do not matter.
  st = vda_prepare(ctx, Q, K, V, K_txt, V_txt, alpha, beta, beta_txt, conv_w, ws, kStaticWorkspaceBytes, stream);
  if (st == VDA_OK) st = vda_scan_bidir(ctx, stream);
  if (st == VDA_OK) st = vda_readout(ctx, gate, O, stream);
  vda_destroy(ctx);
  return st;
}

vda_status vda_static_workspace_poll(void* stream) {
  void* ws = nullptr;
  vda_status st = workspace_address(&ws);
  if (st != VDA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return VDA_ERR_CUDA;
  if (word == 0) return VDA_OK;
  if (cudaMemsetAsync(ws, 0, sizeof(word), s) != cudaSuccess) return VDA_ERR_CUDA;
  return VDA_ERR_TIMEOUT;
}

}  // extern "C"
