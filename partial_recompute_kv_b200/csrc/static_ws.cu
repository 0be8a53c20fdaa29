// A layer-step entry point that allocates nothing: its scratch memory is a
// file-scope device array instead of a caller-supplied workspace.
//
// Some callers cannot call cudaMalloc.  Examples: code that runs while a stream
// is being captured into a CUDA graph under the global capture mode (an
// allocation there invalidates the capture), real-time paths whose latency
// budget cannot absorb a driver allocation, and embedding runtimes or plugins
// that hand out device memory only through their own pool and give the
// library no pool handle.  plk_layer_step_partial_static serves them with the
// same kernels as plk_layer_step_partial, using the array below as workspace.
#include "plk_common.cuh"
#include "plk_internal.h"

namespace plk {

// Shared by every call on a device and held until the process exits.
static __device__ __align__(256) uint8_t g_static_ws[PLK_STATIC_WS_BYTES];

// Device address of g_static_ws, resolved once per device (index = device ordinal).
static void* g_static_ws_ptr[64] = {nullptr};

static int static_ws_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return PLK_ERR_CUDA;
  if (!g_static_ws_ptr[dev]) {
    void* p = nullptr;
    // In host code g_static_ws names a host-side shadow; only this call yields
    // the device address a kernel may use.
    if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || p == nullptr) return PLK_ERR_CUDA;
    g_static_ws_ptr[dev] = p;
  }
  *out = g_static_ws_ptr[dev];
  return PLK_OK;
}

}  // namespace plk

extern "C" int plk_layer_step_partial_static(const plk_dims* dims, const plk_weights* w, const void* X,
                                             const int32_t* idx, const int32_t* seg_ptr, void* K_cache,
                                             void* V_cache, void* Y, void* stream) {
  const size_t need = plk_workspace_bytes(dims);
  if (need == 0)  // invalid dims (or no device): the regular entry point reports which
    return plk_layer_step_partial(dims, w, X, idx, seg_ptr, K_cache, V_cache, Y, nullptr, 0, stream);
  if (need > (size_t)PLK_STATIC_WS_BYTES) return PLK_ERR_WORKSPACE;
  void* ws = nullptr;
  const int e = plk::static_ws_address(&ws);
  if (e != PLK_OK) return e;
  return plk_layer_step_partial(dims, w, X, idx, seg_ptr, K_cache, V_cache, Y, ws, (size_t)PLK_STATIC_WS_BYTES,
                                stream);
}
