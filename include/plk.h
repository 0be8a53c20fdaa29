/*
 * plk.h -- C ABI of the partial-recompute K/V library (B200, sm_100a).
 *
 * The library runs the partial-recompute denoising step of one bidirectional
 * masked diffusion-LM layer on one GPU:
 *
 *   score_drift      S1   per-token drift on a low-rank singular proxy
 *   select_active    S2-3 lock converged rows, compact the M active rows
 *   layer_step_partial S4-10 RMSNorm -> QKV -> attention of the M active
 *                    queries over all N keys -> O -> SwiGLU FFN on the M rows,
 *                    fresh K/V and outputs scattered into the caches
 *   full_layer_step  the same block for all N rows (the baseline sampler)
 *   proxy_commit     S10  refresh the proxy cache of the recomputed rows
 *
 * Sources (web pages, cited by title and section):
 *   [SL]  "Stopping Computation for Converged Tokens in Masked Diffusion-LM
 *         Decoding" (SureLock), Sec. 2 Methodology: Locking Condition,
 *         Permanent Deactivation, Continued Attention, Algorithmic Complexity.
 *   [SPA] "SPA-Cache: Singular Proxies for Adaptive Caching in Diffusion
 *         Language Models", part 1 (singular proxies), part 2 (adaptive budget).
 *   [PS]  "Polestar: Drift-Aware Cache Calibration and Token Commitment for
 *         Efficient Inference of Diffusion LLMs" (refresh the most-drifted rows).
 *
 * Conventions for every call:
 *   - All pointers are DEVICE pointers unless stated otherwise; the caller owns
 *     all memory.  No call allocates device memory.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream) and returns PLK_OK after enqueueing.
 *     Argument and shape errors are detected on the host before any launch and
 *     return a negative code with nothing enqueued.  PLK_ERR_CUDA reports a
 *     failed launch.  A device-side wait that exceeded its limit is reported
 *     later by plk_get_status().
 *   - Tensors are dense row-major.  Token row (b, i) of a [B, N, ...] tensor is
 *     flattened row b*N + i.
 *   - The tensors the kernels move with 16-byte vectors or TMA start on a
 *     16-byte boundary: X, Ut, proxy_cache and proxy_out of the score, the
 *     weights and the K_cache, V_cache and Y of the layer steps (cudaMalloc and
 *     PyTorch allocations are 256-byte aligned); idx and seg_ptr on a 4-byte
 *     one.  A misaligned pointer returns PLK_ERR_ARG with nothing enqueued.
 *   - dtype PLK_BF16: hidden states, weights, Ut, K/V/Y caches are bf16;
 *     proxies and scores are fp32; accumulation is fp32.  dtype PLK_F32: all
 *     of those are fp32 (fp32 arithmetic, no tensor cores).
 *   - The active set is never copied to the host: M = seg_ptr[B] lives on the
 *     device and every kernel reads it there.
 */
#ifndef PLK_H
#define PLK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* return codes */
#define PLK_OK             0
#define PLK_ERR_ARG       -1  /* null pointer, bad enum, k/r out of range      */
#define PLK_ERR_SHAPE     -2  /* shape this build does not support             */
#define PLK_ERR_DTYPE     -3  /* unknown dtype                                 */
#define PLK_ERR_CUDA      -4  /* a CUDA runtime/driver call failed             */
#define PLK_ERR_TIMEOUT   -5  /* a device wait gave up (from plk_get_status)   */
#define PLK_ERR_WORKSPACE -6  /* workspace missing, not 256-byte aligned, or smaller than required */

/* dtypes */
#define PLK_F32  0
#define PLK_BF16 1

/* drift metrics of plk_score_drift */
#define PLK_METRIC_COS 0  /* cosine similarity: high = converged            */
#define PLK_METRIC_L2  1  /* Euclidean distance: high = drifted             */

/* selection modes of plk_select_active */
#define PLK_SEL_THRESH_GT     0  /* lock when score >  tau (permanent)         */
#define PLK_SEL_THRESH_LT     1  /* lock when score <  tau (permanent)         */
#define PLK_SEL_TOPK_LARGEST  2  /* keep the k largest scores active           */
#define PLK_SEL_TOPK_SMALLEST 3  /* keep the k smallest scores active          */

/* Shape of one layer: B sequences of N tokens, model dim d = H*hd, FFN dim F.
 * PLK_BF16 requires hd == 128, d % 256 == 0, F % 128 == 0 (the projection GEMM
 * computes 256-feature tiles on pairs of SMs).
 * PLK_F32 requires hd in {16, 32, 64, 128}.  B*N < 2^31.  0 <= Hkv <= H and,
 * when Hkv > 0, H % Hkv == 0. */
typedef struct {
  int B, N, d, H, hd, F;
  float eps;    /* RMSNorm epsilon                                      */
  int dtype;    /* PLK_F32 or PLK_BF16                                   */
  float rope_theta; /* rotary position embedding base for q and k; 0 = none.
                     * With theta > 0 the pair (x_i, x_{i+hd/2}) of every
                     * head of q and k of the token at position n of its
                     * sequence turns by n * theta^(-2i/hd) before it is
                     * stored (K is cached after the rotation).            */
  int Hkv;      /* K/V heads (grouped-query attention): 0 or H = one per
                 * query head; otherwise 0 < Hkv < H with H % Hkv == 0 and
                 * query head h attends with K/V head h / (H / Hkv).  The
                 * K/V rows are dkv = Hkv*hd wide (dkv = d when Hkv is 0). */
} plk_dims;

/* Layer weights, nn.Linear layout [out_features, in_features], row-major:
 *   g1, g2   [d]       RMSNorm gains
 *   w_qkv    [d + 2 dkv, d]  rows 0..d-1 -> Q, the next dkv rows -> K, the
 *                      last dkv rows -> V (dkv = d without grouping: [3d, d]);
 *                      head h of Q (K/V head g of K, V) is columns
 *                      h*hd .. h*hd+hd-1 (g*hd .. g*hd+hd-1)
 *   w_o      [d, d]
 *   w_gu     [2F, d]   rows 0..F-1 gate, F..2F-1 up
 *   w_down   [d, F]
 * Gains and weights have the layer dtype. */
typedef struct {
  const void *g1, *w_qkv, *w_o, *g2, *w_gu, *w_down;
} plk_weights;

/*
 * S1  Drift score on the singular proxy ([SPA] part 1; [PS] drift signal).
 *   p_i = Ut x_i  for every row i of X [B, N, d]   (Ut [r, d]: r proxy
 *   directions as rows, layer dtype), then
 *   PLK_METRIC_COS: score_i = p_i . c_i / max(|p_i| |c_i|, 1e-30)
 *   PLK_METRIC_L2:  score_i = |p_i - c_i|
 *   with c_i = proxy_cache[i] ([B, N, r] fp32).
 * Outputs: score_out [B, N] fp32; proxy_out [B, N] x r fp32 (may be NULL;
 * receives p).  proxy_out must not alias proxy_cache.
 * PLK_BF16 requires r % 16 == 0 and 16 <= r <= 256; PLK_F32 1 <= r <= 256.
 */
int plk_score_drift(const plk_dims* dims, const void* X, const void* Ut, int r,
                    const float* proxy_cache, int metric, float* proxy_out,
                    float* score_out, void* stream);

/*
 * S2 + S3  Lock update and compaction of the active set.
 *   lock_in, lock_out [B, N] uint8 (1 = locked, 0 = active); may be the same
 *   buffer.  score [B, N] fp32 (unused by no mode may be NULL).
 *   PLK_SEL_THRESH_GT/LT ([SL] Sec. 2 "Locking Condition" and "Permanent
 *     Deactivation"):  lock_out = lock_in | (score > tau)  [or < tau].  A NaN
 *     score never locks; a locked row never unlocks.
 *   PLK_SEL_TOPK_LARGEST/SMALLEST ([SPA] part 2 budget; [PS] most-drifted
 *     refresh):  per sequence, among the rows with lock_in == 0, the k rows
 *     with the largest (smallest) score stay active and every other row gets
 *     lock_out = 1.  Equal scores go to the lower index; +0 == -0; NaN is never
 *     preferred; with fewer than k candidates all of them stay active.
 *   Compaction: idx_out [B*N] int32 receives the flattened indices b*N + i of
 *   the active rows, ascending; seg_ptr [B+1] int32 receives the prefix counts
 *   (seg_ptr[0] = 0, M = seg_ptr[B]).  Entries of idx_out past M are not
 *   written.  Results are bit-exact and deterministic.
 */
int plk_select_active(const plk_dims* dims, const float* score, const uint8_t* lock_in,
                      uint8_t* lock_out, int mode, float tau, int k,
                      int32_t* idx_out, int32_t* seg_ptr, void* stream);

/*
 * S4..S10  One partial-recompute layer step ([SL] Sec. 2 "Permanent
 * Deactivation", "Continued Attention", "Algorithmic Complexity").
 *   X [B, N, d]: layer input hidden states.  idx / seg_ptr: the active rows
 *   as written by plk_select_active (M = seg_ptr[B], read on the device); idx
 *   is a [B*N] buffer: entries past M are read (so that their loads overlap
 *   the read of M) but never used.
 *   For every active row j (token row t = idx[j] of sequence b):
 *     xn = RMSNorm(x_t) * g1;   [q|k|v] = xn W_qkv^T
 *     K_cache[t] = k, V_cache[t] = v          (before attention)
 *     a  = per head softmax(q K_cache[b]^T / sqrt(hd)) V_cache[b], over all N
 *          keys of sequence b (non-causal)
 *     h  = x_t + a W_o^T;  hn = RMSNorm(h) * g2
 *     Y[t] = h + (silu(hn W_g^T) * (hn W_u^T)) W_down^T
 *   Rows not in idx are not read as queries and their K_cache, V_cache and Y
 *   rows are never written.  K_cache, V_cache: [B, N, dkv]; Y: [B, N, d]; in/out.
 *   With grouped-query attention (dims->Hkv > 0) the projection makes Hkv
 *   K/V heads and query head h uses K/V head h / (H / Hkv).
 *   PLK_BF16 rounds to bf16 only the values it stores in the caller's tensors
 *   (the K/V cache rows and Y).  The activations that feed tensor-core products
 *   (xn, q, a, hn and the SwiGLU product) are held as bf16 pairs hi + lo with
 *   lo = bf16(v - hi), ~16 significant bits; the residual stream h and every
 *   sum are fp32.  M = 0 is a no-op.
 *   workspace: device buffer of at least plk_workspace_bytes(dims) bytes, any
 *   content, 256-byte aligned; it must not be used by another call that runs
 *   concurrently.
 */
int plk_layer_step_partial(const plk_dims* dims, const plk_weights* w, const void* X,
                           const int32_t* idx, const int32_t* seg_ptr,
                           void* K_cache, void* V_cache, void* Y,
                           void* workspace, size_t ws_bytes, void* stream);

/*
 * The baseline sampler ([SL] Sec. 1): the same block for all N rows of every
 * sequence; writes every row of K_cache, V_cache and Y.  Same workspace rule.
 */
int plk_full_layer_step(const plk_dims* dims, const plk_weights* w, const void* X,
                        void* K_cache, void* V_cache, void* Y,
                        void* workspace, size_t ws_bytes, void* stream);

/*
 * S2' SureLock's locking condition on logits ([SL] Sec. 2 "Locking
 * Condition"): for every row i with lock_in[i] == 0,
 *   KL_i = KL(p_t || p_{t-1}),  p = softmax over the V vocabulary logits,
 *   H_i  = entropy of p_t in nats (the optional "confidence gate"),
 *   lock_out[i] = (KL_i <= eps && H_i <= h_max)   (h_max = +INFINITY: gate off).
 * Rows with lock_in[i] == 1 are not read and get lock_out[i] = 1.
 * logits_t, logits_prev: [B, N, V] in the layer dtype (dims->dtype), row-major,
 * the logits of the current and the previous step.  kl_out, h_out: [B, N] fp32
 * or NULL; written only at examined rows.  lock_in and lock_out may alias.
 * Only dims->B, dims->N and dims->dtype are used.  Errors: PLK_ERR_ARG for a
 * NULL input, V < 1 or a NaN eps / h_max; PLK_ERR_SHAPE for B*N >= 2^31.
 */
int plk_kl_lock(const plk_dims* dims, int V, const void* logits_t, const void* logits_prev,
                const uint8_t* lock_in, uint8_t* lock_out, float eps, float h_max,
                float* kl_out, float* h_out, void* stream);

/*
 * SlowFast span policy ("Accelerating Diffusion Large Language Models with
 * SlowFast Sampling: The Three Golden Principles", part 2 "Methodology": the
 * two-stage pipeline of an exploratory (slow) and an accelerated (fast) stage;
 * part 4 "Ablation Studies": K_max = 8, W_hist = 2, variance threshold 1.0).
 * One decoding step per call, per sequence b, on conf [B, N] fp32 (the
 * confidence of each position's prediction at this step) and masked [B, N]
 * uint8 (1 = still masked; in/out):
 *   slow phase: a cycle starts at s = the first masked position.  The k most
 *     confident masked positions >= s are unmasked (larger first, NaN last,
 *     equal values to the lower index).  The end point e_t = the largest masked
 *     position >= s with conf > tau_conv (s when none), taken before this
 *     step's unmasking, is recorded.  When the cycle has W_hist end points and
 *     the population variance of the last W_hist is < var_stable, or after
 *     K_max slow steps, the phase turns fast with the span [s, e_t].
 *   fast phase: every masked position of [s, e] with conf > tau_high is
 *     unmasked; when there is none, the k most confident masked positions of
 *     the span are (the fallback).  A span without masked positions unmasks
 *     nothing.
 *   When the span holds no masked position after the step, the cycle ends and
 *     the state returns to all zeros.  A sequence with nothing masked is left
 *     unchanged.
 * Outputs (may be NULL; must not alias masked):
 *   unmask_out [B, N] uint8: 1 at the positions unmasked by this step.
 *   lock_out   [B, N] uint8: the rows the next forward pass may skip (the
 *     out-of-span caching): in the fast phase those outside [s, e], in the slow
 *     phase none, once nothing is masked all of them.  It is a lock_in for
 *     plk_select_active(PLK_SEL_THRESH_GT, tau = +INFINITY), which compacts
 *     the remaining rows.
 * state [B] plk_sf_state (device, in/out): all zeros before the first step of
 *   a sequence.  Other contents give unspecified decisions (never an
 *   out-of-bounds access); a phase other than 0/1 or nslow < 0 reads as zeros.
 * params (host): k >= 1, 1 <= w_hist <= PLK_SF_HIST_MAX, k_max >= 1,
 *   thresholds not NaN.  Only dims->B and dims->N are used; N <= 2^20 keeps the
 *   variance test exact.  Decisions are bit-exact and deterministic.
 * Errors: PLK_ERR_ARG (NULL input, bad params, aliasing), PLK_ERR_SHAPE.
 */
#define PLK_SF_HIST_MAX 16
typedef struct {
  int32_t phase;                  /* 0 slow, 1 fast                           */
  int32_t s, e;                   /* cycle start; span end (fast phase)       */
  int32_t nslow;                  /* slow steps taken in this cycle           */
  int32_t hist[PLK_SF_HIST_MAX];  /* end point of slow step n at n % w_hist   */
} plk_sf_state;
typedef struct {
  int k;             /* positions per slow step and per fallback         */
  int w_hist;        /* W_hist: end points in the variance window        */
  int k_max;         /* K_max: slow steps after which the span is taken  */
  float tau_conv;    /* confidence of a converged position (end point)   */
  float tau_high;    /* tau_high_conf: in-span parallel unmasking        */
  float var_stable;  /* sigma^2_stable                                   */
} plk_sf_params;
int plk_slowfast_step(const plk_dims* dims, const plk_sf_params* params, const float* conf,
                      uint8_t* masked, plk_sf_state* state, uint8_t* unmask_out,
                      uint8_t* lock_out, void* stream);

/*
 * S10 (proxy half)  proxy_cache[idx[j]] = proxy_new[idx[j]] for j < M = seg_ptr[B].
 * idx is a [B*N] buffer (entries past M are read, never used).
 * Both [B, N, r] fp32; rows not in idx are untouched.
 */
int plk_proxy_commit(const plk_dims* dims, int r, const int32_t* idx, const int32_t* seg_ptr,
                     const float* proxy_new, float* proxy_cache, void* stream);

/*
 * plk_layer_step_partial without a caller workspace.  (The pages have no
 * counterpart: this is a deployment variant of the layer step above.)
 * Some callers cannot call cudaMalloc -- code running inside a global-mode
 * stream capture (an allocation there breaks the capture), real-time paths that
 * cannot absorb an allocation's latency, and plugins whose host runtime owns
 * every device allocation.  This entry point runs the same kernels as
 * plk_layer_step_partial with its scratch in a file-scope device array of
 * PLK_STATIC_WS_BYTES, which every GPU that loads the library holds until the
 * process exits.  Arguments and results are those of plk_layer_step_partial.
 *   - It calls no cudaMalloc, cudaFree or allocating library routine.
 *   - Errors: first every error plk_layer_step_partial reports for the same
 *     arguments (dims, weights, inputs, caches); then PLK_ERR_WORKSPACE,
 *     enqueueing nothing, when plk_workspace_bytes(dims) exceeds
 *     PLK_STATIC_WS_BYTES.
 *   - The first call on a device resolves the array's device address
 *     (cudaGetSymbolAddress); make that first call outside any stream capture.
 *     The address is kept per device together with the id of the CUDA context
 *     it belongs to; after a device reset the next call resolves it again (so
 *     that call, too, belongs outside a capture).  Host threads may call
 *     concurrently; the set-up is serialised internally.
 *   - All calls on a device share the array, which keeps the last call's
 *     contents (every kernel initialises what it reads): calls that overlap on
 *     the GPU, e.g. on two streams, race and must be serialised by the caller.
 */
#define PLK_STATIC_WS_BYTES (32u << 20)
int plk_layer_step_partial_static(const plk_dims* dims, const plk_weights* w, const void* X,
                                  const int32_t* idx, const int32_t* seg_ptr,
                                  void* K_cache, void* V_cache, void* Y, void* stream);

/* Bytes of workspace plk_layer_step_partial / plk_full_layer_step need for these
 * dims on the current device (0 for invalid dims). */
size_t plk_workspace_bytes(const plk_dims* dims);

/*
 * The whole denoising step of one layer on device buffers: in stream order
 *   plk_score_drift(X, Ut, r, proxy_cache, metric) -> score and fresh proxies;
 *   plk_select_active(score, lock, mode, tau, k) -> lock (in place), idx, seg_ptr;
 *   plk_layer_step_partial -> K_cache, V_cache, Y (device, in/out), with
 *   plk_proxy_commit -> proxy_cache folded into the layer step's last kernel
 *   (bf16; fp32 runs it as a separate launch).
 * X [B, N, d] device (layer dtype).  Same arguments, rules, workspace
 * (plk_step_workspace_bytes) and errors as plk_denoise_step_host below, without
 * the host copies.
 */
int plk_denoise_step(const plk_dims* dims, const plk_weights* w, const void* Ut, int r, int metric, int mode,
                     float tau, int k, float* proxy_cache, uint8_t* lock, void* K_cache, void* V_cache, void* Y,
                     const void* X, void* workspace, size_t ws_bytes, void* stream);

/*
 * The whole denoising step of one layer from host memory: the step S1..S10 as the
 * calls above chain it, with the layer input coming from and the output going to
 * host buffers ([SL] Sec. 2; [SPA] part 1 for the proxy refresh).  In stream order:
 *   X_host [B, N, d] (host memory, layer dtype) is copied into the workspace;
 *   plk_score_drift(X, Ut, r, proxy_cache, metric) -> score and fresh proxies;
 *   plk_select_active(score, lock, mode, tau, k) -> lock (in place), idx, seg_ptr;
 *   plk_layer_step_partial -> K_cache, V_cache, Y (device, in/out);
 *   plk_proxy_commit -> proxy_cache (device [B, N, r] fp32, in/out);
 *   Y [B, N, d] is copied to Y_host (host memory).
 * One cudaMemcpyAsync each way on `stream`; the call returns after enqueueing
 * (synchronise the stream before reading Y_host).  Host buffers should be pinned
 * (cudaHostAlloc / cudaHostRegister) for the copies to be asynchronous.
 * lock [B, N] uint8 is device memory (in/out).  The argument rules of the calls it
 * chains apply (r, metric, mode, k).  workspace: device buffer of at least
 * plk_step_workspace_bytes(dims, r) bytes, 256-byte aligned, not shared with a
 * concurrent call.  Errors: those of the chained calls, checked before anything
 * is enqueued, and PLK_ERR_WORKSPACE.
 */
int plk_denoise_step_host(const plk_dims* dims, const plk_weights* w, const void* Ut, int r, int metric,
                          int mode, float tau, int k, float* proxy_cache, uint8_t* lock,
                          void* K_cache, void* V_cache, void* Y, const void* X_host, void* Y_host,
                          void* workspace, size_t ws_bytes, void* stream);
/* Workspace of plk_denoise_step_host (0 for invalid dims or r). */
size_t plk_step_workspace_bytes(const plk_dims* dims, int r);

/*
 * T consecutive denoising steps of one layer from host memory, with the host
 * copies overlapped with the compute of neighbouring steps.  Step t (t < T) is
 * plk_denoise_step_host with X_hosts[t] in and Y_hosts[t] out: it reads the
 * layer input X_hosts[t] ([B, N, d], host, layer dtype) and leaves in
 * Y_hosts[t] ([B, N, d], host) the output cache Y as it stands after step t.
 * lock, proxy_cache, K_cache, V_cache and Y carry over from step to step as in
 * T separate calls, and the results are those of T separate calls.
 *   - upload_stream copies X_hosts[t + 1] into a second device buffer while
 *     step t computes on `stream`;
 *   - after step t, Y is copied on the device into one of two snapshot buffers
 *     (step t + 1 updates Y in place), and download_stream copies the snapshot
 *     to Y_hosts[t] while step t + 1 computes.
 * Each step still moves its whole X in and its whole Y out; the copies of
 * consecutive steps run concurrently with the compute (on separate copy
 * engines when the host buffers are pinned).  For T >= 3 the call captures the
 * step as CUDA graphs (one per X buffer) and launches one graph per step; with
 * tracing on (plk_trace_events) or if the capture fails it launches the
 * kernels directly.  The results are the same either way.  The three streams are the
 * caller's (upload_stream and download_stream should be two further streams;
 * passing `stream` for them runs everything in order).  The copies start after
 * the work already enqueued on `stream`, and `stream` waits for the last
 * download: synchronise `stream` before reading any Y_hosts[t].  Y_hosts[t]
 * may repeat (the downloads run in step order).  workspace: at least
 * plk_steps_workspace_bytes(dims, r) bytes, 256-byte aligned, not shared with
 * a concurrent call.  Errors: PLK_ERR_ARG for T < 1 or a null X_hosts[t] or
 * Y_hosts[t], then those of plk_denoise_step_host, all checked before anything
 * is enqueued; PLK_ERR_CUDA when a copy or launch fails part way (synchronise
 * all three streams before reusing the buffers).
 */
int plk_denoise_steps_host(const plk_dims* dims, const plk_weights* w, const void* Ut, int r, int metric,
                           int mode, float tau, int k, float* proxy_cache, uint8_t* lock,
                           void* K_cache, void* V_cache, void* Y, int T, const void* const* X_hosts,
                           void* const* Y_hosts, void* workspace, size_t ws_bytes, void* stream,
                           void* upload_stream, void* download_stream);
/* Workspace of plk_denoise_steps_host (0 for invalid dims or r). */
size_t plk_steps_workspace_bytes(const plk_dims* dims, int r);

/* Synchronises `stream`, returns the device status word of the current device
 * (PLK_OK or PLK_ERR_TIMEOUT) and clears it. */
int plk_get_status(void* stream);

/* Upper bound, in SM clock cycles, of every device-side wait (default 4e9,
 * about two seconds).  Values < 1 are rejected. */
int plk_set_wait_limit(long long cycles);

/* Reproducible mode for the bf16 layer step (host-side setting, process-wide;
 * default off).  Off: the O and down projections add the pieces of a split tile
 * into the residual stream in the order they arrive, so h and Y may differ in
 * the last bits between runs (q, K, V and the SwiGLU input never do).  On: those
 * pieces land in a fixed order too, and every output of plk_layer_step_partial,
 * plk_full_layer_step and plk_denoise_step_host is bit-reproducible for the same
 * inputs on the same GPU model, at ~35 us more per step at the 8B shape with 256
 * rows (the pieces of a tile wait for one another).  on is 0 or 1. */
int plk_set_deterministic(int on);

/* Launches one block that waits on a device flag nothing ever sets, bounded by
 * the current wait limit; the wait then records PLK_ERR_TIMEOUT in the status
 * word.  Exists to test the timeout path without faulting or hanging a GPU. */
int plk_selftest_wait_timeout(void* stream);

/* out[i] = 2^t[i] (n values, device pointers) by the FMA-pipe exponential the
 * attention softmax can compute for a share of its weights (range reduction to
 * [-1/2, 1/2] and a degree-4 minimax polynomial; relative error <= 3e-6; t < -126
 * gives 0; the build gives it no share: the MUFU ex2 alone measured faster).
 * Exists so that the polynomial can be tested against exp2 on a GPU. */
int plk_selftest_exp2(const float* t, float* out, int n, void* stream);

/* Tracing.  Registers up to 16 cudaEvent_t handles (passed as void*).  While
 * registered, plk_layer_step_partial and plk_full_layer_step record events[0]
 * on their stream before their first kernel and events[i] after their i-th
 * kernel of the chain (the bf16 step has 10: RMSNorm1, QKV GEMM, QKV finish,
 * attention, O GEMM, RMSNorm2, gate/up GEMM, SwiGLU finish, down GEMM, output
 * finish), so a caller can time every kernel with
 * cudaEventElapsedTime on the launching stream.  n = 0 unregisters.  The events
 * must outlive their registration.  Host-side state, not thread-safe. */
int plk_trace_events(void* const* events, int n);

/* Static description of a return code. */
const char* plk_error_string(int code);

/* Library version, 100*major + minor. */
int plk_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PLK_H */
