// ar_tune_step_noalloc: the tuning step with its scratch in a fixed device array.
//
// Some callers cannot hand the library a workspace from cudaMalloc: a host
// process whose device memory is owned end to end by another allocator (a
// framework's caching allocator that has reserved the GPU's memory, where an
// extra cudaMalloc fails or forces the cache to be flushed), or a
// latency-critical loop that cannot afford the implicit device
// synchronisation of cudaMalloc/cudaFree.  For them this entry point runs the
// same kernels as ar_tune_step, but takes its scratch from the array below,
// which the CUDA runtime allocates once per device when the library's device
// code is loaded and which stays allocated until the process exits.
#include <stdio.h>

#include <mutex>

#include "../../include/autoround.h"
#include "ar_internal.h"

namespace ar {
namespace {

// Scratch shared by every ar_tune_step_noalloc call on a device.  In host code
// this name is only a host-side stand-in for the device array: its device
// address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[AR_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array for the current device.  The first call
// on a device looks it up (cudaGetSymbolAddress, with that device current) and
// caches it; the lock makes concurrent first calls from several host threads
// safe.  A cudaDeviceReset() unloads the library's device code, so the cached
// address of that device is stale afterwards (documented in autoround.h).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace ar

extern "C" ar_status ar_tune_step_noalloc(int block_kind, const ar_layer* layers, int n_layers, const uint16_t* X,
                                          int64_t M, const float* Y, const ar_qconfig* cfg, int n_steps,
                                          float* loss_per_step, const ar_grads* grads, ar_stream_t stream) {
  const size_t need = ar_tune_step_workspace(block_kind, layers, n_layers, M, cfg, n_steps);
  if (need == 0) {
    // ar_tune_step reports the precise validation error.
    return ar_tune_step(block_kind, layers, n_layers, X, M, Y, cfg, n_steps, loss_per_step, grads, nullptr, 0,
                        stream);
  }
  if (need > static_cast<size_t>(AR_NOALLOC_SCRATCH_BYTES)) {
    static thread_local char msg[256];
    snprintf(msg, sizeof(msg),
             "ar_tune_step_noalloc: this problem needs %zu bytes of scratch, above the fixed %d-byte limit; "
             "use ar_tune_step with a caller workspace",
             need, AR_NOALLOC_SCRATCH_BYTES);
    ar::set_last_error(msg);
    return AR_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  const cudaError_t e = ar::scratch_address(&scratch);
  if (e != cudaSuccess) {
    static thread_local char msg[256];
    snprintf(msg, sizeof(msg), "ar_tune_step_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
    ar::set_last_error(msg);
    return AR_ERR_CUDA;
  }
  return ar_tune_step(block_kind, layers, n_layers, X, M, Y, cfg, n_steps, loss_per_step, grads, scratch,
                      static_cast<size_t>(AR_NOALLOC_SCRATCH_BYTES), stream);
}
