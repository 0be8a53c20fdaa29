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
#include <atomic>
#include <mutex>

#include "plk_common.cuh"
#include "plk_internal.h"

namespace plk {

// Shared by every call on a device and held until the process exits.
static __device__ __align__(256) uint8_t g_static_ws[PLK_STATIC_WS_BYTES];

// Device address of g_static_ws per device ordinal, with the id of the CUDA
// context it was resolved in.  A device reset (cudaDeviceReset, or the primary
// context being destroyed and created again) loads the module anew, possibly at
// another address, under a new context id: the address is then resolved again.
struct StaticWsSlot {
  std::atomic<void*> ptr{nullptr};
  std::atomic<unsigned long long> ctx_id{0};
};
static StaticWsSlot g_static_ws_slot[64];
static std::mutex g_static_ws_mutex;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Id of the context current on this thread; 0 when there is none (or the query fails).
static unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// The set-up: once per device (and again after a reset), with the device current.
static int static_ws_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return PLK_ERR_CUDA;
  StaticWsSlot& slot = g_static_ws_slot[dev];
  const unsigned long long id = current_ctx_id();
  void* p = slot.ptr.load(std::memory_order_acquire);
  if (p && id != 0 && slot.ctx_id.load(std::memory_order_acquire) == id) {
    *out = p;
    return PLK_OK;
  }
  std::lock_guard<std::mutex> lock(g_static_ws_mutex);
  // In host code g_static_ws names a host-side shadow; only this call yields
  // the device address a kernel may use.  It also makes the device's primary
  // context current when no context was yet.
  p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || p == nullptr) return PLK_ERR_CUDA;
  slot.ctx_id.store(current_ctx_id(), std::memory_order_release);
  slot.ptr.store(p, std::memory_order_release);
  *out = p;
  return PLK_OK;
}

}  // namespace plk

extern "C" int plk_layer_step_partial_static(const plk_dims* dims, const plk_weights* w, const void* X,
                                             const int32_t* idx, const int32_t* seg_ptr, void* K_cache,
                                             void* V_cache, void* Y, void* stream) {
  // the checks of plk_layer_step_partial first, then the size limit, then the set-up
  const int e = plk::check_layer_args(dims, w, X, idx, seg_ptr, K_cache, V_cache, Y);
  if (e != PLK_OK) return e;
  const size_t need = plk_workspace_bytes(dims);
  if (need == 0) return PLK_ERR_CUDA;  // valid dims: only a failed device query gives 0
  if (need > (size_t)PLK_STATIC_WS_BYTES) return PLK_ERR_WORKSPACE;
  void* ws = nullptr;
  const int r = plk::static_ws_address(&ws);
  if (r != PLK_OK) return r;
  return plk_layer_step_partial(dims, w, X, idx, seg_ptr, K_cache, V_cache, Y, ws, (size_t)PLK_STATIC_WS_BYTES,
                                stream);
}
