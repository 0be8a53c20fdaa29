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
// One CTA of 512 threads per sequence (latency-bound: a few microseconds).
// Up to 16384 positions the sequence's confidences and mask flags are staged
// in shared memory in one pass whose loads are all independent, so the later
// passes cost shared-memory latency only; reductions combine four values per
// block barrier pair; k <= 16 positions are picked by k rounds of a block-wide
// arg-max over (preference key, lower index) instead of the four-pass radix
// select, which serves larger k and sequences too long to stage.
// The variance test is exact: with end points below 2^20 and W_hist <= 16 the
// integer W*S2 - S1^2 and var_stable*W^2 are exact doubles.
#include <limits.h>

#include "plk_common.cuh"
#include "plk_internal.h"

namespace plk {

constexpr int kSfThreads = 512;
constexpr int kSfStageMaxN = 16384;  // positions staged in shared memory (5 bytes each): <= 32 per thread
constexpr int kSfRoundsMaxK = 16;    // top-k by repeated block arg-max up to this k

struct SfArgs {
  int k, w_hist, k_max;
  float tau_conv, tau_high, var_stable;
};

__device__ __forceinline__ int4 warp_reduce_ssmm(int4 v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    v.x += __shfl_xor_sync(0xffffffffu, v.x, o);
    v.y += __shfl_xor_sync(0xffffffffu, v.y, o);
    v.z = max(v.z, __shfl_xor_sync(0xffffffffu, v.z, o));
    v.w = max(v.w, __shfl_xor_sync(0xffffffffu, v.w, o));
  }
  return v;
}

// Block reduction of (sum, sum, max, max) with one barrier pair; every thread
// gets the result (each warp re-reduces the per-warp partials, one per lane).
__device__ __forceinline__ int4 block_reduce_ssmm(int4 v, int4* sh4) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_reduce_ssmm(v);
  __syncthreads();  // earlier readers of sh4 are done
  if (lane == 0) sh4[warp] = v;
  __syncthreads();
  return warp_reduce_ssmm(lane < nw ? sh4[lane] : make_int4(0, 0, INT_MIN, INT_MIN));
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const unsigned long long t = __shfl_xor_sync(0xffffffffu, v, o);
    v = t > v ? t : v;
  }
  return v;
}

__device__ __forceinline__ unsigned long long block_max_u64(unsigned long long v, unsigned long long* sh8) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_max_u64(v);
  __syncthreads();
  if (lane == 0) sh8[warp] = v;
  __syncthreads();
  return warp_max_u64(lane < nw ? sh8[lane] : 0ull);
}

template <bool kStaged>
__global__ void __launch_bounds__(kSfThreads) slowfast_kernel(const float* __restrict__ conf_all, uint8_t* masked_all,
                                                              plk_sf_state* states, int N, SfArgs p,
                                                              uint8_t* unmask_out, uint8_t* lock_out) {
  extern __shared__ __align__(16) uint8_t sf_dyn[];
  __shared__ int hist[256];
  __shared__ int sh[33];
  __shared__ int4 sh4[32];
  __shared__ unsigned long long sh8[32];
  __shared__ uint32_t s_prefix;
  __shared__ int s_remaining;
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x;
  const long long base = (long long)b * N;
  const float* conf_g = conf_all + base;
  uint8_t* masked_g = masked_all + base;
  plk_sf_state* stp = states + b;

  // every thread reads the state (and the end-point ring, in flight with the
  // staging loads); thread 0 writes it back at the end, after the last
  // block-wide barrier, so no thread reads a half-written state
  int phase = stp->phase, s = stp->s, e = stp->e, nslow = stp->nslow;
  int ring[PLK_SF_HIST_MAX];
#pragma unroll
  for (int j = 0; j < PLK_SF_HIST_MAX; ++j) ring[j] = j < p.w_hist ? stp->hist[j] : 0;

  // pass 1 (staging): masked count and the first masked position
  float* s_conf = reinterpret_cast<float*>(sf_dyn);
  uint8_t* s_mask = sf_dyn + 4 * ((N + 15) & ~15);
  int cnt = 0, first = INT_MAX;
#pragma unroll 8
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    const uint8_t mv = masked_g[i];
    if (kStaged) {
      s_conf[i] = conf_g[i];
      s_mask[i] = mv;
    }
    if (mv) ++cnt, first = min(first, i);
  }
  const int4 r1 = block_reduce_ssmm(make_int4(cnt, 0, -first, INT_MIN), sh4);  // also publishes the staging
  const int npend = r1.x;
  if (npend == 0) {  // nothing to decode: state unchanged, nothing to recompute
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
      if (unmask_out) unmask_out[base + i] = 0;
      if (lock_out) lock_out[base + i] = 1;
    }
    return;
  }
  first = -r1.z;
  if ((phase != 0 && phase != 1) || nslow < 0) phase = 0, s = 0, e = 0, nslow = 0;
  const float* cf = kStaged ? s_conf : conf_g;
  const uint8_t* mk = kStaged ? s_mask : masked_g;

  const bool slow = phase == 0;
  if (slow && nslow == 0) s = first;
  const int lo = s, hi = slow ? N - 1 : e;
  auto cand = [mk, lo, hi](int i) { return mk[i] != 0 && lo <= i && i <= hi; };

  // pass 2: candidates, the converged end point (slow) or the hot count (fast)
  int ccnt = 0, hcnt = 0, emax = -1;
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    if (!cand(i)) continue;
    ++ccnt;
    const float c = cf[i];
    if (slow && c > p.tau_conv) emax = max(emax, i);  // NaN compares false
    if (!slow && c > p.tau_high) ++hcnt;
  }
  const int4 r2 = block_reduce_ssmm(make_int4(ccnt, hcnt, emax, INT_MIN), sh4);
  const int ncand = r2.x;
  const int nhot = slow ? 0 : r2.y;
  const int end_t = slow ? r2.z : -1;

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
#pragma unroll
      for (int j = 0; j < PLK_SF_HIST_MAX; ++j) {
        if (j >= p.w_hist) break;
        const double v = (double)((j == slot ? end : ring[j]) - (long long)s);
        s1 += v;
        s2 += v * v;
      }
      const double w = (double)p.w_hist;
      stable = w * s2 - s1 * s1 < (double)p.var_stable * w * w;
    }
    if (stable || nslow >= p.k_max) phase = 1, e = end;
  }
  if (reset) phase = 0, s = 0, e = 0, nslow = 0;

  // the k most confident candidates (rule 2)
  const int keep_n = rule == 2 ? min(p.k, ncand) : 0;
  const bool select = rule == 2 && keep_n > 0 && keep_n < ncand;  // else all candidates or none
  const bool rounds = kStaged && select && keep_n <= kSfRoundsMaxK;
  uint32_t mine = 0u;  // rounds: bit j = this thread's j-th position was picked
  uint32_t kth = 0u;
  int remaining = 0;
  if (rounds) {
    // each round takes the most preferred candidate not yet taken: the largest
    // (key << 32 | ~index), i.e. the largest key and among equal keys the lowest index
    for (int r = 0; r < keep_n; ++r) {
      unsigned long long best = 0ull;
      int j = 0;
      for (int i = threadIdx.x; i < N; i += blockDim.x, ++j) {
        if (((mine >> j) & 1u) || !cand(i)) continue;
        const unsigned long long v = ((unsigned long long)pref_key(cf[i], true) << 32) | (uint32_t)~i;
        best = v > best ? v : best;
      }
      best = block_max_u64(best, sh8);  // > 0: keep_n < ncand leaves a candidate every round
      const int w = (int)~(uint32_t)best;
      if (w % (int)blockDim.x == (int)threadIdx.x) mine |= 1u << (w / (int)blockDim.x);
    }
  } else if (select) {
    block_radix_kth(cf, N, keep_n, true, cand, hist, &s_prefix, &s_remaining, &kth, &remaining);
  }

  // pass 3 (ordered): unmask, and count what is left in the span and overall
  int taken_eq = 0, left_span = 0, left_all = 0, j = 0;
  for (int c0 = 0; c0 < N; c0 += blockDim.x, ++j) {
    const int i = c0 + threadIdx.x;
    const bool in = i < N;
    const bool m = in && mk[i] != 0;
    const bool cd = in && cand(i);
    const float c = in ? cf[i] : 0.f;
    bool take = false;
    if (rule == 1) {
      take = cd && c > p.tau_high;
    } else if (rule == 2) {
      if (!select) {
        take = cd && keep_n > 0;
      } else if (rounds) {
        take = (mine >> j) & 1u;
      } else {  // radix: keys above the k-th, then the first `remaining` equal ones in index order
        bool gt = false, eq = false;
        if (cd) {
          const uint32_t key = pref_key(c, true);
          gt = key > kth;
          eq = key == kth;
        }
        int total;
        const int r = block_rank(eq ? 1 : 0, sh, &total);
        take = cd && (gt || (eq && taken_eq + r < remaining));
        taken_eq += total;
      }
    }
    if (take) masked_g[i] = 0;
    if (in && unmask_out) unmask_out[base + i] = take ? 1 : 0;
    const bool left = m && !take;
    left_all += left ? 1 : 0;
    left_span += (left && s <= i && i <= e) ? 1 : 0;
  }
  const int4 r3 = block_reduce_ssmm(make_int4(left_all, left_span, INT_MIN, INT_MIN), sh4);
  if (phase == 1 && r3.y == 0) phase = 0, s = 0, e = 0, nslow = 0;  // the span is decoded

  if (lock_out) {
    for (int i = threadIdx.x; i < N; i += blockDim.x)
      lock_out[base + i] = r3.x == 0 ? 1 : (phase == 1 ? ((s <= i && i <= e) ? 0 : 1) : 0);
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
  const int N = dims->N;
  if (N <= kSfStageMaxN) {
    const size_t dyn = (size_t)5 * ((N + 15) & ~15);
    if (dyn > (40u << 10) &&
        cudaFuncSetAttribute(slowfast_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn) !=
            cudaSuccess)
      return PLK_ERR_CUDA;
    return launch_pdl(slowfast_kernel<true>, dim3(dims->B), dim3(kSfThreads), dyn, st, conf, masked, state, N, a,
                      unmask_out, lock_out);
  }
  return launch_pdl(slowfast_kernel<false>, dim3(dims->B), dim3(kSfThreads), 0, st, conf, masked, state, N, a,
                    unmask_out, lock_out);
}

}  // namespace plk
