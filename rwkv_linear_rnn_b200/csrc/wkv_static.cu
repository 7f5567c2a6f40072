// wkv_static.cu -- a backward entry point that needs no caller workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// backward: code inside a custom allocator or memory-pool callback, plugin
// hosts that hand out only fixed buffers, or runtimes that forbid
// cudaMalloc on their execution thread.  wkv_backward_static gives them the
// ordinary backward with its scratch in a statically sized device array
// instead of a caller workspace.  It is a thin wrapper: the kernels and the
// numerics are exactly those of wkv_backward.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/wkv.h"

namespace {

// File-scope scratch.  Every GPU that loads the library holds it until the
// process exits.  In host code `g_wkv_scratch` is only a host-side stand-in
// for the symbol: its device address must be fetched per device.
constexpr size_t kStaticScratch = WKV_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_wkv_scratch[kStaticScratch];

constexpr int kMaxDevices = 64;
std::atomic<void *> g_scratch_ptr[kMaxDevices];

// Device address of the scratch on the current device.  The first call on a
// device looks the address up and zero-fills the array (the workspace
// protocol needs a zeroed header once); later calls only read the cached
// pointer.  Returns nullptr on failure.
void *scratch_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  void *p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p) return p;
  void *q = nullptr;
  if (cudaGetSymbolAddress(&q, g_wkv_scratch) != cudaSuccess || !q) return nullptr;
  if (cudaMemset(q, 0, kStaticScratch) != cudaSuccess) return nullptr;
  if (cudaDeviceSynchronize() != cudaSuccess) return nullptr;
  void *expected = nullptr;
  if (!g_scratch_ptr[dev].compare_exchange_strong(expected, q, std::memory_order_acq_rel))
    return expected;  // another thread finished the set-up first
  return q;
}

}  // namespace

extern "C" int wkv_backward_static(int64_t B, int64_t T, int64_t C, int dtype, const float *w,
                                   const float *u, const void *k, const void *v,
                                   const void *grad_y, const float *state_in, const float *ckpt,
                                   float *grad_w, float *grad_u, void *grad_k, void *grad_v,
                                   void *stream) {
  const size_t need = wkv_workspace_size(WKV_OP_BACKWARD, B, T, C, dtype);
  if (need == 0) return WKV_ERR_INVALID_ARG;
  if (need > kStaticScratch) return WKV_ERR_WORKSPACE;
  void *ws = scratch_for_current_device();
  if (!ws) return WKV_ERR_CUDA;
  // The per-launch counters of the scratch header (block ticket and
  // finished-block count, bytes 4..11; grid-barrier arrivals, bytes 20..23)
  // must read zero when a launch starts.  Launches leave them at zero;
  // clearing them here makes that explicit.  The launch epoch (bytes 0..3)
  // must persist across calls and is kept, and so is the status word.
  unsigned char *h = static_cast<unsigned char *>(ws);
  if (cudaMemsetAsync(h + 4, 0, 8, (cudaStream_t)stream) != cudaSuccess ||
      cudaMemsetAsync(h + 20, 0, 4, (cudaStream_t)stream) != cudaSuccess)
    return WKV_ERR_CUDA;
  return wkv_backward(B, T, C, dtype, w, u, k, v, grad_y, state_in, ckpt, grad_w, grad_u, grad_k,
                      grad_v, ws, kStaticScratch, stream);
}
