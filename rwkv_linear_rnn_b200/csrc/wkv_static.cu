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
#include <mutex>

#include "../../include/wkv.h"

namespace {

// File-scope scratch.  Every GPU that loads the library holds it until the
// process exits.  In host code `g_wkv_scratch` is only a host-side stand-in
// for the symbol: its device address must be looked up in the context that
// runs the kernels.
constexpr size_t kStaticScratch = WKV_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_wkv_scratch[kStaticScratch];

// Device addresses of the array that have been zero-filled.  Every context
// that loads the library gets its own instance of the array, at its own
// address in the process's unified address space; an address not in this
// set belongs to a context not set up yet (the first call on a device, or the
// first after the device was reset and the library's module loaded again).
constexpr int kSlots = 64;
std::atomic<void *> g_ready[kSlots];
std::atomic<int> g_next{0};
std::mutex g_setup;

bool ready(void *q) {
  for (int i = 0; i < kSlots; ++i)
    if (g_ready[i].load(std::memory_order_acquire) == q) return true;
  return false;
}

// Device address of the scratch in the current context.  The address is
// looked up on every call (cudaGetSymbolAddress allocates nothing), so it is
// never stale; the first call that meets a new address zero-fills the array
// synchronously (the workspace protocol needs a zeroed header once).
// Returns nullptr on failure.
void *scratch_for_current_context() {
  void *q = nullptr;
  if (cudaGetSymbolAddress(&q, g_wkv_scratch) != cudaSuccess || !q) return nullptr;
  if (ready(q)) return q;
  std::lock_guard<std::mutex> lock(g_setup);
  if (ready(q)) return q;
  if (cudaMemset(q, 0, kStaticScratch) != cudaSuccess) return nullptr;
  if (cudaDeviceSynchronize() != cudaSuccess) return nullptr;
  g_ready[g_next.fetch_add(1) % kSlots].store(q, std::memory_order_release);
  return q;
}

}  // namespace

// The launch protocol keeps the array consistent from call to call: the
// per-launch counters of its header (ticket, finished blocks, grid-barrier
// arrivals) are back at zero when every launch ends, and the launch epoch in
// the header makes the flags of earlier calls read as stale.  So nothing is
// cleared between calls, and a call that fails its argument checks has
// launched nothing.
extern "C" int wkv_backward_static(int64_t B, int64_t T, int64_t C, int dtype, const float *w,
                                   const float *u, const void *k, const void *v,
                                   const void *grad_y, const float *state_in, const float *ckpt,
                                   float *grad_w, float *grad_u, void *grad_k, void *grad_v,
                                   void *stream) {
  const size_t need = wkv_workspace_size(WKV_OP_BACKWARD, B, T, C, dtype);
  if (need == 0) return WKV_ERR_INVALID_ARG;
  if (need > kStaticScratch) return WKV_ERR_WORKSPACE;
  void *ws = scratch_for_current_context();
  if (!ws) return WKV_ERR_CUDA;
  return wkv_backward(B, T, C, dtype, w, u, k, v, grad_y, state_in, ckpt, grad_w, grad_u, grad_k,
                      grad_v, ws, kStaticScratch, stream);
}

extern "C" int wkv_backward_static_status(void *stream) {
  void *ws = scratch_for_current_context();
  if (!ws) return WKV_ERR_CUDA;
  return wkv_get_status(ws, stream);
}
