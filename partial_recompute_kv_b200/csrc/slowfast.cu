// SlowFast span policy: the two-stage decoding schedule of the SlowFast
// Sampling page ("Accelerating Diffusion Large Language Models with SlowFast
// Sampling: The Three Golden Principles", part 2 "Methodology", the two-stage
// pipeline; part 4 "Ablation Studies" for K_max, W_hist and the variance
// threshold), one decoding step per call, as the unmasking and caching rule
// on top of the lock and compaction step.
//
// Per sequence, on the caller's fp32 confidences of this step:
//   slow step  s = first masked position when a cycle starts; unmask the k most
//              confident masked positions >= s (ties to the lower index, NaN
//              last); end point e_t = the largest masked position >= s with
//              c > tau_conv, else s (taken before the unmasking).  Switch to the
//              fast phase with the span [s, e_t] when the last W_hist end points
//              of this cycle have population variance < var_stable, or after
//              K_max slow steps.
//   fast step  unmask every masked position of the span with c > tau_high, or,
//              when there is none, the k most confident masked positions of the
//              span (the fallback).
//   The cycle ends (state back to zero) when the span holds no masked position.
//   lock_out marks the rows the next forward pass may skip: outside the span in
//   the fast phase, none in the slow phase, all once nothing is masked.
//
// One CTA of 1024 threads per sequence, a handful of block-wide passes over the
// sequence's N positions (counts, the end point, a radix select for the top-k,
// the ordered write pass): latency-bound by design (a few microseconds for
// N <= 8192), so no attempt is made to spread one sequence over several CTAs.
// The variance test is exact: with end points below 2^20 and W_hist <= 16 the
// integer W*S2 - S1^2 and var_stable*W^2 are exact doubles.
#include <limits.h>

#include "plk_common.cuh"
#include "plk_internal.h"

namespace plk {

constexpr int kSfThreads = 1024;

struct SfArgs {
  int k, w_hist, k_max;
  float tau_conv, tau_high, var_stable;
};

__device__ __forceinline__ int block_max_int(int v, int* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  int t = (threadIdx.x < nw) ? sh[threadIdx.x] : INT_MIN;
  if (warp == 0) {
#pragma unroll
    for (int o = 16; o; o >>= 1) t = max(t, __shfl_xor_sync(0xffffffffu, t, o));
    if (lane == 0) sh[32] = t;
  }
  __syncthreads();
  return sh[32];
}

__global__ void __launch_bounds__(kSfThreads) slowfast_kernel(const float* __restrict__ conf_all, uint8_t* masked_all,
                                                              plk_sf_state* states, int N, SfArgs p,
                                                              uint8_t* unmask_out, uint8_t* lock_out) {
  __shared__ int hist[256];
  __shared__ int sh[33];
  __shared__ uint32_t s_prefix;
  __shared__ int s_remaining;
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x;
  const long long base = (long long)b * N;
  const float* conf = conf_all + base;
  uint8_t* masked = masked_all + base;
  plk_sf_state* stp = states + b;

  // every thread reads the state; thread 0 writes it back at the end (after the
  // last block-wide barrier, so no thread reads a half-written state)
  int phase = stp->phase, s = stp->s, e = stp->e, nslow = stp->nslow;
  if ((phase != 0 && phase != 1) || nslow < 0) phase = 0, s = 0, e = 0, nslow = 0;

  // pass 1: masked count and the first masked position
  int cnt = 0, first = INT_MAX;
  for (int i = threadIdx.x; i < N; i += blockDim.x)
    if (masked[i]) ++cnt, first = min(first, i);
  const int npend = block_sum(cnt, sh);
  if (npend == 0) {  // nothing to decode: state unchanged, nothing to recompute
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
      if (unmask_out) unmask_out[base + i] = 0;
      if (lock_out) lock_out[base + i] = 1;
    }
    return;
  }
  first = -block_max_int(-first, sh);

  const bool slow = phase == 0;
  if (slow && nslow == 0) s = first;
  const int lo = s, hi = slow ? N - 1 : e;
  auto cand = [masked, lo, hi](int i) { return masked[i] != 0 && lo <= i && i <= hi; };

  // pass 2: candidates, the converged end point (slow) or the hot count (fast)
  int ccnt = 0, hcnt = 0, emax = -1;
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    if (!cand(i)) continue;
    ++ccnt;
    const float c = conf[i];
    if (slow && c > p.tau_conv) emax = max(emax, i);  // NaN compares false
    if (!slow && c > p.tau_high) ++hcnt;
  }
  const int ncand = block_sum(ccnt, sh);
  const int nhot = slow ? 0 : block_sum(hcnt, sh);
  const int end_t = slow ? block_max_int(emax, sh) : -1;

  // which rule unmasks: 0 nothing (empty span), 1 the hot positions, 2 top-k
  int rule = 2;
  bool reset = false;
  if (!slow && ncand == 0) rule = 0, reset = true;
  else if (!slow && nhot > 0) rule = 1;

  int slot = -1, end = 0;
  if (slow) {
    end = end_t >= 0 ? end_t : s;
    slot = nslow % p.w_hist;
    ++nslow;
    bool stable = false;
    if (nslow >= p.w_hist) {
      // population variance of the ring (the last w_hist end points) < var_stable,
      // as w*S2 - S1^2 < var_stable * w^2 (end points taken relative to s)
      double s1 = 0.0, s2 = 0.0;
      for (int j = 0; j < p.w_hist; ++j) {
        const double v = (double)((j == slot ? end : stp->hist[j]) - (long long)s);
        s1 += v;
        s2 += v * v;
      }
      const double w = (double)p.w_hist;
      stable = w * s2 - s1 * s1 < (double)p.var_stable * w * w;
    }
    if (stable || nslow >= p.k_max) phase = 1, e = end;
  }
  if (reset) phase = 0, s = 0, e = 0, nslow = 0;

  // top-k threshold among the candidates
  const int keep_n = rule == 2 ? min(p.k, ncand) : 0;
  const bool keep_all = keep_n == ncand;
  uint32_t kth = 0u;
  int remaining = 0;
  if (rule == 2 && keep_n > 0 && !keep_all)
    block_radix_kth(conf, N, keep_n, true, cand, hist, &s_prefix, &s_remaining, &kth, &remaining);

  // pass 3 (ordered): unmask, and count what is left in the span and overall
  int taken_eq = 0, left_span = 0, left_all = 0;
  for (int c0 = 0; c0 < N; c0 += blockDim.x) {
    const int i = c0 + threadIdx.x;
    const bool in = i < N;
    const bool m = in && masked[i] != 0;
    const bool cd = in && cand(i);
    const float c = in ? conf[i] : 0.f;
    bool gt = false, eq = false;
    if (rule == 2 && cd && keep_n > 0 && !keep_all) {
      const uint32_t key = pref_key(c, true);
      gt = key > kth;
      eq = key == kth;
    }
    int total;
    const int r = block_rank(eq ? 1 : 0, sh, &total);
    bool take = false;
    if (rule == 1) take = cd && c > p.tau_high;
    if (rule == 2) take = cd && keep_n > 0 && (keep_all || gt || (eq && taken_eq + r < remaining));
    taken_eq += total;
    if (take) masked[i] = 0;
    if (in && unmask_out) unmask_out[base + i] = take ? 1 : 0;
    const bool left = m && !take;
    left_all += left ? 1 : 0;
    left_span += (left && s <= i && i <= e) ? 1 : 0;
  }
  left_all = block_sum(left_all, sh);
  left_span = block_sum(left_span, sh);
  if (phase == 1 && left_span == 0) phase = 0, s = 0, e = 0, nslow = 0;  // the span is decoded

  if (lock_out) {
    for (int i = threadIdx.x; i < N; i += blockDim.x)
      lock_out[base + i] = left_all == 0 ? 1 : (phase == 1 ? ((s <= i && i <= e) ? 0 : 1) : 0);
  }
  if (threadIdx.x == 0) {
    if (slot >= 0) stp->hist[slot] = end;
    stp->phase = phase;
    stp->s = s;
    stp->e = e;
    stp->nslow = nslow;
  }
}

int launch_slowfast(const plk_dims* dims, const plk_sf_params* prm, const float* conf, uint8_t* masked,
                    plk_sf_state* state, uint8_t* unmask_out, uint8_t* lock_out, cudaStream_t st) {
  SfArgs a;
  a.k = prm->k;
  a.w_hist = prm->w_hist;
  a.k_max = prm->k_max;
  a.tau_conv = prm->tau_conv;
  a.tau_high = prm->tau_high;
  a.var_stable = prm->var_stable;
  return launch_pdl(slowfast_kernel, dim3(dims->B), dim3(kSfThreads), 0, st, conf, masked, state, dims->N, a,
                    unmask_out, lock_out);
}

}  // namespace plk
