// Host-side internals of the partial-recompute library: launch functions of
// each kernel family, the workspace layout and TMA descriptor helpers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "../../include/plk.h"

namespace plk {

// ---- tile constants of the tcgen05 GEMM ------------------------------------
constexpr int kGemmBM = 128;      // feature rows per CTA (a CTA pair computes 256)
constexpr int kGemmBNMax = 256;   // tokens per tile (UMMA N, runtime 128 or 256; each CTA loads half)
constexpr int kGemmBK = 64;       // K per stage: one 128-byte swizzle row of bf16
constexpr int kGemmStages = 4;  // 48 KB each: weight tile + the hi and lo activation tiles
constexpr int kGemmThreads = 192; // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue

// ---- attention key split over several CTA pairs --------------------------------
// Per-unit arrival counters of the attention kernel (zeroed by the QKV
// finishing kernel, which runs just before it, in the RMSNorm1 output buffer
// that the QKV GEMM has consumed by then).
constexpr int kAttPartCounters = 128;

// ---- grouped-query attention --------------------------------------------------
inline int kv_heads(const plk_dims* d) { return d->Hkv > 0 ? d->Hkv : d->H; }
inline int kv_width(const plk_dims* d) { return kv_heads(d) * d->hd; }  // dkv: K and V row width

// ---- launch with programmatic stream serialization ---------------------------
// The kernel may start while its predecessor in the stream finishes; it orders
// itself with pdl_wait() (plk_common.cuh).
template <typename... KArgs, typename... Args>
inline int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                      Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess ? PLK_OK : PLK_ERR_CUDA;
}

// ---- workspace layout -------------------------------------------------------
struct Workspace {
  size_t total = 0;
  // offsets (bytes)
  size_t iota = 0, seg = 0;              // identity active set for the full step
  size_t xn = 0, q = 0, a = 0, h32 = 0, hn = 0, act = 0;
  size_t xn_lo = 0, q_lo = 0, a_lo = 0, hn_lo = 0, act_lo = 0;  // bf16: low halves (v - bf16(v))
  size_t c32 = 0;                        // fp32 GEMM sums [Mcap, max(d + 2 dkv, 2F)] (QKV, then gate/up;
                                         // in between, the attention's partial outputs)
  size_t c32_bytes = 0;
  // bf16 path: the pieces-done counts ([8 x tiles]) of the QKV, O, gate/up and down GEMMs in
  // turn (O and down used in reproducible mode only), cleared by RMSNorm1 at every step
  size_t gsync = 0;
  int gsync_ints = 0;
  int gsync_tiles[4] = {0, 0, 0, 0};
  int num_sms = 0;
};
Workspace workspace_layout(const plk_dims* d, int num_sms);
// plk_set_deterministic: the O and down projections land split-tile pieces in a fixed order too
extern int g_deterministic;
int device_sm_count();

// ---- TMA descriptors ---------------------------------------------------------
// 2D bf16 tensor [rows, cols] row-major (cols contiguous), 128-byte swizzle,
// box {64 cols, box_rows rows}.
int make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);
// 2D fp32 tensor [rows, cols] row-major, no swizzle, box {32 cols, 32 rows}:
// the target of the GEMM's bulk reduce-adds.
int make_tmap_f32(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols);

// ---- launches (all asynchronous on `st`; return PLK_OK / PLK_ERR_CUDA) -------
int launch_select(const plk_dims* dims, const float* score, const uint8_t* lock_in, uint8_t* lock_out,
                  int mode, float tau, int k, int32_t* idx_out, int32_t* seg_ptr, cudaStream_t st);

int launch_score(const plk_dims* dims, const void* X, const void* Ut, int r, const float* proxy_cache,
                 int metric, float* proxy_out, float* score_out, cudaStream_t st);

int launch_proxy_commit(const plk_dims* dims, int r, const int32_t* idx, const int32_t* seg_ptr,
                        const float* proxy_new, float* proxy_cache, cudaStream_t st);

int launch_kl_lock(const plk_dims* dims, int V, const void* logits_t, const void* logits_prev, const uint8_t* lock_in,
                   uint8_t* lock_out, float eps, float h_max, float* kl_out, float* h_out, cudaStream_t st);

int launch_slowfast(const plk_dims* dims, const plk_sf_params* prm, const float* conf, uint8_t* masked,
                    plk_sf_state* state, uint8_t* unmask_out, uint8_t* lock_out, cudaStream_t st);

// The argument checks shared by the layer-step entry points (PLK_OK or the error code).
int check_layer_args(const plk_dims* dims, const plk_weights* w, const void* X, const int32_t* idx,
                     const int32_t* seg_ptr, const void* K_cache, const void* V_cache, const void* Y);

// Optional proxy refresh folded into the layer step's last kernel (bf16 path):
// proxy_cache[idx[j]] = proxy_new[idx[j]] (r fp32 values per row) for j < M.
struct ProxyRefresh {
  int r = 0;
  const float* proxy_new = nullptr;
  float* proxy_cache = nullptr;
};
int run_layer(const plk_dims* dims, const plk_weights* w, const void* X, const int32_t* idx,
              const int32_t* seg_ptr, bool full, void* K_cache, void* V_cache, void* Y, void* ws,
              size_t ws_bytes, cudaStream_t st, const ProxyRefresh* pr = nullptr);

// Arguments of the tcgen05 GEMM out[t, f] += sum_k (Xhi[t, k] + Xlo[t, k]) W[f, k]
// over the M = seg_ptr[B] compact tokens (fp32 out, added with bulk reduce-adds;
// the activation enters as its bf16 hi/lo pair).
struct GemmArgs {
  int K;                   // reduction length, multiple of 64
  int ftiles;              // 128-row feature tiles (even: a CTA pair takes two)
  int gu_F;                // gate/up GEMM: F (tile f = gate rows f*64.. and up rows F + f*64..), else 0
  const int32_t* seg_ptr;  // M = seg_ptr[B]
  int B;
  int num_sms;             // SM count: at most one persistent CTA per SM, in pairs
  // Per (pair tile, CTA, epilogue warp): the count of the tile's pieces that have landed in the
  // output, [tiles * 8], zero on entry (nullptr: one piece per tile only, e.g. no split).
  uint32_t* done = nullptr;
  int store_first = 0;     // 1: the output starts undefined, the tail piece stores; 0: every piece adds
};
int launch_gemm_tc(const CUtensorMap& tmW, const CUtensorMap& tmXhi, const CUtensorMap& tmXlo,
                   const CUtensorMap& tmOut, const GemmArgs& a, cudaStream_t st);

// part_scratch / part_bytes: free device memory for the partial outputs of a key
// split over several CTA pairs (used when the units leave pairs idle); part_cnt:
// kAttPartCounters ints, zero on entry, zero again on exit.
// q, q_lo: the queries as a bf16 hi/lo pair; a_out, a_lo: the output as one.
int launch_attention_bf16(const plk_dims* dims, const void* q, const void* q_lo, const void* K_cache,
                          const void* V_cache, void* a_out, void* a_lo, const int32_t* seg_ptr, int num_sms,
                          float* part_scratch, size_t part_bytes, int* part_cnt, cudaStream_t st);
// out[i] = 2^t[i] by the attention softmax's FMA-pipe exponential (test hook)
int launch_exp2_selftest(const float* t, float* out, int n, cudaStream_t st);
int launch_attention_f32(const plk_dims* dims, const float* q, const float* K_cache, const float* V_cache,
                         float* a_out, const int32_t* seg_ptr, int Mcap, cudaStream_t st);

}  // namespace plk
