// extern "C" boundary of the partial-recompute library: argument validation on
// the host, then asynchronous launches on the caller's stream.  Declarations and
// the contract of every call are in include/plk.h.
#include "plk_common.cuh"
#include "plk_internal.h"

namespace plk {

static int check_dims(const plk_dims* d) {
  if (!d) return PLK_ERR_ARG;
  if (d->dtype != PLK_F32 && d->dtype != PLK_BF16) return PLK_ERR_DTYPE;
  if (d->B < 1 || d->N < 1 || d->d < 1 || d->H < 1 || d->hd < 1 || d->F < 1) return PLK_ERR_SHAPE;
  if ((long long)d->H * d->hd != d->d) return PLK_ERR_SHAPE;
  if (d->Hkv < 0 || d->Hkv > d->H || (d->Hkv > 0 && d->H % d->Hkv != 0)) return PLK_ERR_SHAPE;
  if ((long long)d->B * d->N >= (1LL << 31)) return PLK_ERR_SHAPE;
  if (!(d->eps >= 0.f)) return PLK_ERR_ARG;
  if (!(d->rope_theta >= 0.f) || d->rope_theta > 3.0e38f) return PLK_ERR_ARG;
  if (d->dtype == PLK_BF16) {
    if (d->hd != 128 || d->d % 256 != 0 || d->F % 128 != 0) return PLK_ERR_SHAPE;
  } else {
    if (d->hd != 16 && d->hd != 32 && d->hd != 64 && d->hd != 128) return PLK_ERR_SHAPE;
  }
  return PLK_OK;
}

// The kernels move these tensors with 16-byte vectors or TMA: their base addresses must be
// 16-byte aligned (rows stay aligned: d, F and bf16 proxy ranks are multiples of 16 elements).
static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool weights_ok(const plk_weights* w) {
  if (!w || !w->g1 || !w->w_qkv || !w->w_o || !w->g2 || !w->w_gu || !w->w_down) return false;
  return aligned16(w->g1) && aligned16(w->w_qkv) && aligned16(w->w_o) && aligned16(w->g2) && aligned16(w->w_gu) &&
         aligned16(w->w_down);
}
static bool caches_ok(const void* K_cache, const void* V_cache, const void* Y) {
  return K_cache && V_cache && Y && aligned16(K_cache) && aligned16(V_cache) && aligned16(Y);
}

// The argument checks of plk_layer_step_partial (dims, weights, inputs and caches;
// the workspace is checked where it is laid out).
int check_layer_args(const plk_dims* dims, const plk_weights* w, const void* X, const int32_t* idx,
                     const int32_t* seg_ptr, const void* K_cache, const void* V_cache, const void* Y) {
  const int e = check_dims(dims);
  if (e != PLK_OK) return e;
  if (!weights_ok(w)) return PLK_ERR_ARG;
  if (!X || !aligned16(X) || !idx || !seg_ptr || !caches_ok(K_cache, V_cache, Y)) return PLK_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(idx) | reinterpret_cast<uintptr_t>(seg_ptr)) & 3u) return PLK_ERR_ARG;
  return PLK_OK;
}

}  // namespace plk

using namespace plk;

extern "C" {

int plk_version(void) { return 100; }

const char* plk_error_string(int code) {
  switch (code) {
    case PLK_OK: return "ok";
    case PLK_ERR_ARG: return "invalid argument";
    case PLK_ERR_SHAPE: return "unsupported shape";
    case PLK_ERR_DTYPE: return "unknown dtype";
    case PLK_ERR_CUDA: return "CUDA call failed";
    case PLK_ERR_TIMEOUT: return "device wait exceeded its limit";
    case PLK_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    default: return "unknown error code";
  }
}

size_t plk_workspace_bytes(const plk_dims* dims) {
  if (check_dims(dims) != PLK_OK) return 0;
  const int nsm = device_sm_count();
  if (nsm <= 0) return 0;
  return workspace_layout(dims, nsm).total;
}

int plk_score_drift(const plk_dims* dims, const void* X, const void* Ut, int r, const float* proxy_cache,
                    int metric, float* proxy_out, float* score_out, void* stream) {
  const int e = check_dims(dims);
  if (e != PLK_OK) return e;
  if (!X || !Ut || !proxy_cache || !score_out) return PLK_ERR_ARG;
  if (!aligned16(X) || !aligned16(Ut) || !aligned16(proxy_cache) || !aligned16(proxy_out)) return PLK_ERR_ARG;
  if (metric != PLK_METRIC_COS && metric != PLK_METRIC_L2) return PLK_ERR_ARG;
  if (proxy_out && proxy_out == proxy_cache) return PLK_ERR_ARG;
  if (dims->dtype == PLK_BF16) {
    if (r < 16 || r > 256 || r % 16 != 0 || dims->d % 64 != 0) return PLK_ERR_ARG;
  } else {
    if (r < 1 || r > 256) return PLK_ERR_ARG;
  }
  return launch_score(dims, X, Ut, r, proxy_cache, metric, proxy_out, score_out, (cudaStream_t)stream);
}

int plk_select_active(const plk_dims* dims, const float* score, const uint8_t* lock_in, uint8_t* lock_out,
                      int mode, float tau, int k, int32_t* idx_out, int32_t* seg_ptr, void* stream) {
  if (!dims) return PLK_ERR_ARG;
  if (dims->B < 1 || dims->N < 1 || (long long)dims->B * dims->N >= (1LL << 31)) return PLK_ERR_SHAPE;
  if (!score || !lock_in || !lock_out || !idx_out || !seg_ptr) return PLK_ERR_ARG;
  if (mode < PLK_SEL_THRESH_GT || mode > PLK_SEL_TOPK_SMALLEST) return PLK_ERR_ARG;
  if ((mode == PLK_SEL_TOPK_LARGEST || mode == PLK_SEL_TOPK_SMALLEST) && k < 0) return PLK_ERR_ARG;
  return launch_select(dims, score, lock_in, lock_out, mode, tau, k, idx_out, seg_ptr, (cudaStream_t)stream);
}

int plk_kl_lock(const plk_dims* dims, int V, const void* logits_t, const void* logits_prev, const uint8_t* lock_in,
                uint8_t* lock_out, float eps, float h_max, float* kl_out, float* h_out, void* stream) {
  if (!dims) return PLK_ERR_ARG;
  if (dims->dtype != PLK_F32 && dims->dtype != PLK_BF16) return PLK_ERR_DTYPE;
  if (dims->B < 1 || dims->N < 1 || (long long)dims->B * dims->N >= (1LL << 31)) return PLK_ERR_SHAPE;
  if (V < 1 || !logits_t || !logits_prev || !lock_in || !lock_out) return PLK_ERR_ARG;
  if (eps != eps || h_max != h_max) return PLK_ERR_ARG;
  return launch_kl_lock(dims, V, logits_t, logits_prev, lock_in, lock_out, eps, h_max, kl_out, h_out,
                        (cudaStream_t)stream);
}

int plk_slowfast_step(const plk_dims* dims, const plk_sf_params* params, const float* conf, uint8_t* masked,
                      plk_sf_state* state, uint8_t* unmask_out, uint8_t* lock_out, void* stream) {
  if (!dims || !params) return PLK_ERR_ARG;
  if (dims->B < 1 || dims->N < 1 || dims->N > (1 << 20) || (long long)dims->B * dims->N >= (1LL << 31))
    return PLK_ERR_SHAPE;
  if (!conf || !masked || !state) return PLK_ERR_ARG;
  if (params->k < 1 || params->w_hist < 1 || params->w_hist > PLK_SF_HIST_MAX || params->k_max < 1)
    return PLK_ERR_ARG;
  if (params->tau_conv != params->tau_conv || params->tau_high != params->tau_high ||
      params->var_stable != params->var_stable)
    return PLK_ERR_ARG;
  if (unmask_out == masked || lock_out == masked || (unmask_out && unmask_out == lock_out)) return PLK_ERR_ARG;
  return launch_slowfast(dims, params, conf, masked, state, unmask_out, lock_out, (cudaStream_t)stream);
}

int plk_layer_step_partial(const plk_dims* dims, const plk_weights* w, const void* X, const int32_t* idx,
                           const int32_t* seg_ptr, void* K_cache, void* V_cache, void* Y, void* workspace,
                           size_t ws_bytes, void* stream) {
  const int e = check_layer_args(dims, w, X, idx, seg_ptr, K_cache, V_cache, Y);
  if (e != PLK_OK) return e;
  return run_layer(dims, w, X, idx, seg_ptr, false, K_cache, V_cache, Y, workspace, ws_bytes,
                   (cudaStream_t)stream);
}

int plk_full_layer_step(const plk_dims* dims, const plk_weights* w, const void* X, void* K_cache, void* V_cache,
                        void* Y, void* workspace, size_t ws_bytes, void* stream) {
  const int e = check_dims(dims);
  if (e != PLK_OK) return e;
  if (!weights_ok(w)) return PLK_ERR_ARG;
  if (!X || !aligned16(X) || !caches_ok(K_cache, V_cache, Y)) return PLK_ERR_ARG;
  return run_layer(dims, w, X, nullptr, nullptr, true, K_cache, V_cache, Y, workspace, ws_bytes,
                   (cudaStream_t)stream);
}

int plk_proxy_commit(const plk_dims* dims, int r, const int32_t* idx, const int32_t* seg_ptr,
                     const float* proxy_new, float* proxy_cache, void* stream) {
  if (!dims) return PLK_ERR_ARG;
  if (dims->B < 1 || dims->N < 1) return PLK_ERR_SHAPE;
  if (r < 1 || r > 256 || !idx || !seg_ptr || !proxy_new || !proxy_cache) return PLK_ERR_ARG;
  return launch_proxy_commit(dims, r, idx, seg_ptr, proxy_new, proxy_cache, (cudaStream_t)stream);
}

}  // extern "C"

namespace plk {
// Layout of the workspace of plk_denoise_step_host behind the layer step's own:
// score [B*N] fp32, fresh proxies [B*N*r] fp32, idx [B*N], seg_ptr [B+1], X [B*N*d].
struct StepWs {
  size_t layer = 0, score = 0, pnew = 0, idx = 0, seg = 0, x = 0, total = 0;
};
static size_t up256(size_t v) { return (v + 255) / 256 * 256; }
static StepWs step_ws_layout(const plk_dims* d, int r) {
  StepWs s;
  const size_t BN = (size_t)d->B * d->N, es = d->dtype == PLK_BF16 ? 2 : 4;
  s.layer = 0;
  size_t off = up256(plk_workspace_bytes(d));
  s.score = off;
  off = up256(off + 4 * BN);
  s.pnew = off;
  off = up256(off + 4 * BN * (size_t)r);
  s.idx = off;
  off = up256(off + 4 * BN);
  s.seg = off;
  off = up256(off + 4 * ((size_t)d->B + 1));
  s.x = off;
  off = up256(off + es * BN * (size_t)d->d);
  s.total = off;
  return s;
}
static int check_score_args(const plk_dims* dims, int r, int metric) {
  if (metric != PLK_METRIC_COS && metric != PLK_METRIC_L2) return PLK_ERR_ARG;
  if (dims->dtype == PLK_BF16) {
    if (r < 16 || r > 256 || r % 16 != 0 || dims->d % 64 != 0) return PLK_ERR_ARG;
  } else {
    if (r < 1 || r > 256) return PLK_ERR_ARG;
  }
  return PLK_OK;
}
}  // namespace plk

extern "C" {

size_t plk_step_workspace_bytes(const plk_dims* dims, int r) {
  if (check_dims(dims) != PLK_OK || check_score_args(dims, r, PLK_METRIC_L2) != PLK_OK) return 0;
  if (plk_workspace_bytes(dims) == 0) return 0;
  return step_ws_layout(dims, r).total;
}

}  // extern "C"

namespace plk {
// The checks of the whole-step entry points (PLK_OK or the error code); X may be a host or a
// device pointer (only checked for null here).
static int check_step_args(const plk_dims* dims, const plk_weights* w, const void* Ut, int r, int metric, int mode,
                           int k, const float* proxy_cache, const uint8_t* lock, const void* K_cache,
                           const void* V_cache, const void* Y, const void* X) {
  int e = check_dims(dims);
  if (e != PLK_OK) return e;
  if ((e = check_score_args(dims, r, metric)) != PLK_OK) return e;
  if (!Ut || !proxy_cache || !lock || !X) return PLK_ERR_ARG;
  if (!aligned16(Ut) || !aligned16(proxy_cache)) return PLK_ERR_ARG;
  if (mode < PLK_SEL_THRESH_GT || mode > PLK_SEL_TOPK_SMALLEST) return PLK_ERR_ARG;
  if ((mode == PLK_SEL_TOPK_LARGEST || mode == PLK_SEL_TOPK_SMALLEST) && k < 0) return PLK_ERR_ARG;
  if (!weights_ok(w) || !caches_ok(K_cache, V_cache, Y)) return PLK_ERR_ARG;
  if (plk_workspace_bytes(dims) == 0) return PLK_ERR_CUDA;
  return PLK_OK;
}

// score -> select (in place) -> layer step with the proxy refresh folded into its last kernel
static int run_step(const plk_dims* dims, const plk_weights* w, const void* Ut, int r, int metric, int mode,
                    float tau, int k, float* proxy_cache, uint8_t* lock, void* K_cache, void* V_cache, void* Y,
                    const void* X, uint8_t* ws, const StepWs& L, cudaStream_t st) {
  float* score = (float*)(ws + L.score);
  float* pnew = (float*)(ws + L.pnew);
  int32_t* idx = (int32_t*)(ws + L.idx);
  int32_t* seg = (int32_t*)(ws + L.seg);
  int e;
  if ((e = launch_score(dims, X, Ut, r, proxy_cache, metric, pnew, score, st)) != PLK_OK) return e;
  if ((e = launch_select(dims, score, lock, lock, mode, tau, k, idx, seg, st)) != PLK_OK) return e;
  ProxyRefresh pr;
  pr.r = r;
  pr.proxy_new = pnew;
  pr.proxy_cache = proxy_cache;
  return run_layer(dims, w, X, idx, seg, false, K_cache, V_cache, Y, ws, L.score, st, &pr);
}
}  // namespace plk

extern "C" {

int plk_denoise_step(const plk_dims* dims, const plk_weights* w, const void* Ut, int r, int metric, int mode,
                     float tau, int k, float* proxy_cache, uint8_t* lock, void* K_cache, void* V_cache, void* Y,
                     const void* X, void* workspace, size_t ws_bytes, void* stream) {
  int e = check_step_args(dims, w, Ut, r, metric, mode, k, proxy_cache, lock, K_cache, V_cache, Y, X);
  if (e != PLK_OK) return e;
  if (!aligned16(X)) return PLK_ERR_ARG;
  const StepWs L = step_ws_layout(dims, r);
  if (!workspace || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return PLK_ERR_WORKSPACE;
  return run_step(dims, w, Ut, r, metric, mode, tau, k, proxy_cache, lock, K_cache, V_cache, Y, X,
                  (uint8_t*)workspace, L, (cudaStream_t)stream);
}

int plk_denoise_step_host(const plk_dims* dims, const plk_weights* w, const void* Ut, int r, int metric,
                          int mode, float tau, int k, float* proxy_cache, uint8_t* lock, void* K_cache,
                          void* V_cache, void* Y, const void* X_host, void* Y_host, void* workspace,
                          size_t ws_bytes, void* stream) {
  int e = check_step_args(dims, w, Ut, r, metric, mode, k, proxy_cache, lock, K_cache, V_cache, Y, X_host);
  if (e != PLK_OK) return e;
  if (!Y_host) return PLK_ERR_ARG;
  const StepWs L = step_ws_layout(dims, r);
  if (!workspace || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return PLK_ERR_WORKSPACE;
  uint8_t* ws = (uint8_t*)workspace;
  void* X = ws + L.x;
  const size_t BN = (size_t)dims->B * dims->N, es = dims->dtype == PLK_BF16 ? 2 : 4;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemcpyAsync(X, X_host, es * BN * dims->d, cudaMemcpyHostToDevice, st) != cudaSuccess) return PLK_ERR_CUDA;
  if ((e = run_step(dims, w, Ut, r, metric, mode, tau, k, proxy_cache, lock, K_cache, V_cache, Y, X, ws, L, st)) !=
      PLK_OK)
    return e;
  if (cudaMemcpyAsync(Y_host, Y, es * BN * dims->d, cudaMemcpyDeviceToHost, st) != cudaSuccess) return PLK_ERR_CUDA;
  return PLK_OK;
}

}  // extern "C"

namespace plk {
// Workspace of plk_denoise_steps_host: the one-step layout, then a second X buffer and two
// snapshots of Y (the inputs and outputs of consecutive steps in flight).
struct StepsWs {
  StepWs one;
  size_t x2 = 0, y0 = 0, y1 = 0, total = 0;
};
static StepsWs steps_ws_layout(const plk_dims* d, int r) {
  StepsWs s;
  s.one = step_ws_layout(d, r);
  const size_t bytes = (size_t)d->B * d->N * d->d * (d->dtype == PLK_BF16 ? 2 : 4);
  s.x2 = up256(s.one.total);
  s.y0 = up256(s.x2 + bytes);
  s.y1 = up256(s.y0 + bytes);
  s.total = up256(s.y1 + bytes);
  return s;
}

// dst = src in 16-byte vectors (the snapshot of Y after a step): a grid-stride copy on the SMs,
// chained to the step's last kernel by programmatic dependent launch
__global__ void snapshot_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, size_t n16) {
  pdl_wait();
  pdl_trigger();
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += (size_t)gridDim.x * blockDim.x)
    dst[i] = __ldcs(src + i);
}

// One step of plk_denoise_steps_host on `st`: the step, then Y copied into the snapshot buffer
// that the download of this step reads.
static int run_step_snapshot(const plk_dims* dims, const plk_weights* w, const void* Ut, int r, int metric, int mode,
                             float tau, int k, float* proxy_cache, uint8_t* lock, void* K_cache, void* V_cache,
                             void* Y, const void* X, uint8_t* ws, const StepWs& L, void* Ysnap, cudaStream_t st) {
  const int e = run_step(dims, w, Ut, r, metric, mode, tau, k, proxy_cache, lock, K_cache, V_cache, Y, X, ws, L, st);
  if (e != PLK_OK) return e;
  const size_t bytes = (size_t)dims->B * dims->N * dims->d * (dims->dtype == PLK_BF16 ? 2 : 4);
  return launch_pdl(snapshot_kernel, dim3(4 * (unsigned)device_sm_count()), dim3(256), 0, st, (const uint4*)Y,
                    (uint4*)Ysnap, bytes / 16);
}

// The step captured as a CUDA graph, one per X buffer, for the duration of one
// plk_denoise_steps_host call: one launch per step instead of the step's dozen
// kernel launches and their descriptor set-up, whose host time comes close to the
// step's device time and would let host jitter idle the GPU.
struct StepGraphs {
  cudaGraphExec_t exec[2] = {nullptr, nullptr};
  bool ok = false;
  ~StepGraphs() {
    for (cudaGraphExec_t e : exec)
      if (e) cudaGraphExecDestroy(e);  // an instance still in flight is freed when it completes
  }
  // Captures the step and its snapshot copy for both X buffers on a private stream (nothing runs
  // during capture).
  // Any failure leaves ok false and the caller launches the steps directly.
  void build(const plk_dims* dims, const plk_weights* w, const void* Ut, int r, int metric, int mode, float tau,
             int k, float* proxy_cache, uint8_t* lock, void* K_cache, void* V_cache, void* Y, void* const Xb[2],
             void* const Ys[2], uint8_t* ws, const StepWs& L) {
    cudaStream_t cs = nullptr;
    if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return;
    bool good = true;
    for (int b = 0; b < 2 && good; ++b) {
      cudaGraph_t graph = nullptr;
      good = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) == cudaSuccess;
      if (!good) break;
      const int e = run_step_snapshot(dims, w, Ut, r, metric, mode, tau, k, proxy_cache, lock, K_cache, V_cache, Y,
                                      Xb[b], ws, L, Ys[b], cs);
      const bool ended = cudaStreamEndCapture(cs, &graph) == cudaSuccess;
      good = e == PLK_OK && ended && graph != nullptr &&
             cudaGraphInstantiate(&exec[b], graph, 0) == cudaSuccess;
      if (graph) cudaGraphDestroy(graph);
    }
    cudaStreamDestroy(cs);
    (void)cudaGetLastError();  // a failed capture is not the caller's error: the direct path follows
    ok = good;
  }
};

// The events of one plk_denoise_steps_host call, destroyed with it (a recorded event that has
// not completed is released by the driver once it does).
struct StepEvents {
  cudaEvent_t up[2] = {}, comp[2] = {}, down[2] = {}, start = nullptr;
  bool ok = true;
  StepEvents() {
    for (cudaEvent_t* e : {&up[0], &up[1], &comp[0], &comp[1], &down[0], &down[1], &start})
      ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
  }
  ~StepEvents() {
    for (cudaEvent_t e : {up[0], up[1], comp[0], comp[1], down[0], down[1], start})
      if (e) cudaEventDestroy(e);
  }
};
}  // namespace plk

extern "C" {

size_t plk_steps_workspace_bytes(const plk_dims* dims, int r) {
  if (plk_step_workspace_bytes(dims, r) == 0) return 0;
  return steps_ws_layout(dims, r).total;
}

int plk_denoise_steps_host(const plk_dims* dims, const plk_weights* w, const void* Ut, int r, int metric,
                           int mode, float tau, int k, float* proxy_cache, uint8_t* lock, void* K_cache,
                           void* V_cache, void* Y, int T, const void* const* X_hosts, void* const* Y_hosts,
                           void* workspace, size_t ws_bytes, void* stream, void* upload_stream,
                           void* download_stream) {
  if (T < 1 || !X_hosts || !Y_hosts) return PLK_ERR_ARG;
  for (int t = 0; t < T; ++t)
    if (!X_hosts[t] || !Y_hosts[t]) return PLK_ERR_ARG;
  int e = check_step_args(dims, w, Ut, r, metric, mode, k, proxy_cache, lock, K_cache, V_cache, Y, X_hosts[0]);
  if (e != PLK_OK) return e;
  const StepsWs L = steps_ws_layout(dims, r);
  if (!workspace || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return PLK_ERR_WORKSPACE;
  uint8_t* ws = (uint8_t*)workspace;
  void* Xb[2] = {ws + L.one.x, ws + L.x2};
  void* Ys[2] = {ws + L.y0, ws + L.y1};
  const size_t bytes = (size_t)dims->B * dims->N * dims->d * (dims->dtype == PLK_BF16 ? 2 : 4);
  cudaStream_t S = (cudaStream_t)stream, U = (cudaStream_t)upload_stream, D = (cudaStream_t)download_stream;
  StepEvents ev;
  if (!ev.ok) return PLK_ERR_CUDA;
  // from three steps on, capture the step once per X buffer and launch it as a graph (not while
  // plk_trace_events records events between the kernels)
  StepGraphs graphs;
  if (T >= 3 && g_ntrace == 0)
    graphs.build(dims, w, Ut, r, metric, mode, tau, k, proxy_cache, lock, K_cache, V_cache, Y, Xb, Ys, ws, L.one);
#define PLK_CU(x)                                 \
  do {                                            \
    if ((x) != cudaSuccess) return PLK_ERR_CUDA;  \
  } while (0)
  // the copy streams start after the work already on `stream` (an earlier call's use of the
  // workspace included)
  PLK_CU(cudaEventRecord(ev.start, S));
  PLK_CU(cudaStreamWaitEvent(U, ev.start, 0));
  PLK_CU(cudaStreamWaitEvent(D, ev.start, 0));
  PLK_CU(cudaMemcpyAsync(Xb[0], X_hosts[0], bytes, cudaMemcpyHostToDevice, U));
  PLK_CU(cudaEventRecord(ev.up[0], U));
  for (int t = 0; t < T; ++t) {
    const int b = t & 1, nb = b ^ 1;
    if (t + 1 < T) {  // the next input, into the buffer step t - 1 read
      if (t >= 1) PLK_CU(cudaStreamWaitEvent(U, ev.comp[nb], 0));
      PLK_CU(cudaMemcpyAsync(Xb[nb], X_hosts[t + 1], bytes, cudaMemcpyHostToDevice, U));
      PLK_CU(cudaEventRecord(ev.up[nb], U));
    }
    // step t reads X buffer b, and ends by snapshotting Y (step t + 1 updates Y in place) into
    // snapshot buffer b, which the download of step t - 2 must have read by then
    PLK_CU(cudaStreamWaitEvent(S, ev.up[b], 0));
    if (t >= 2) PLK_CU(cudaStreamWaitEvent(S, ev.down[b], 0));
    if (graphs.ok) {
      PLK_CU(cudaGraphLaunch(graphs.exec[b], S));
    } else if ((e = run_step_snapshot(dims, w, Ut, r, metric, mode, tau, k, proxy_cache, lock, K_cache, V_cache, Y,
                                      Xb[b], ws, L.one, Ys[b], S)) != PLK_OK) {
      return e;
    }
    PLK_CU(cudaEventRecord(ev.comp[b], S));
    PLK_CU(cudaStreamWaitEvent(D, ev.comp[b], 0));
    PLK_CU(cudaMemcpyAsync(Y_hosts[t], Ys[b], bytes, cudaMemcpyDeviceToHost, D));
    PLK_CU(cudaEventRecord(ev.down[b], D));
  }
  // `stream` ends after the last download (the downloads run in step order on one stream)
  PLK_CU(cudaStreamWaitEvent(S, ev.down[(T - 1) & 1], 0));
#undef PLK_CU
  return PLK_OK;
}

int plk_get_status(void* stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return PLK_ERR_CUDA;
  int v = PLK_OK;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return PLK_ERR_CUDA;
  const int zero = PLK_OK;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return PLK_ERR_CUDA;
  return v;
}

int plk_trace_events(void* const* events, int n) {
  if (n < 0 || n > 16 || (n > 0 && !events)) return PLK_ERR_ARG;
  for (int i = 0; i < 16; ++i) g_trace[i] = (i < n) ? (cudaEvent_t)events[i] : nullptr;
  g_ntrace = n;
  return PLK_OK;
}

int plk_set_deterministic(int on) {
  if (on != 0 && on != 1) return PLK_ERR_ARG;
  g_deterministic = on;
  return PLK_OK;
}

int plk_set_wait_limit(long long cycles) {
  if (cycles < 1) return PLK_ERR_ARG;
  return cudaMemcpyToSymbol(g_wait_limit, &cycles, sizeof(cycles)) == cudaSuccess ? PLK_OK : PLK_ERR_CUDA;
}

}  // extern "C"

namespace plk {
__device__ uint32_t g_never_set = 0u;

// One thread spins on a flag nothing writes; the bounded spin records
// PLK_ERR_TIMEOUT and returns.
__global__ void selftest_wait_kernel() {
  if (threadIdx.x == 0) (void)spin_until_geq(&g_never_set, 1u);
}
}  // namespace plk

extern "C" int plk_selftest_exp2(const float* t, float* out, int n, void* stream) {
  if (n < 0 || (n > 0 && (!t || !out))) return PLK_ERR_ARG;
  if (n == 0) return PLK_OK;
  return plk::launch_exp2_selftest(t, out, n, (cudaStream_t)stream);
}

extern "C" int plk_selftest_wait_timeout(void* stream) {
  plk::selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>();
  return cudaPeekAtLastError() == cudaSuccess ? PLK_OK : PLK_ERR_CUDA;
}
