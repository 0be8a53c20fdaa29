// S2 + S3: lock rules and active-set compaction.
//
// Lock rules: the threshold lock of the SureLock page ("Stopping Computation
// for Converged Tokens in Masked Diffusion-LM Decoding", Sec. 2 "Locking
// Condition", "Permanent Deactivation") and the top-k budget of the SPA-Cache
// page ("SPA-Cache: Singular Proxies for Adaptive Caching in Diffusion Language
// Models", part 2) / Polestar-Cache's most-drifted refresh.
//
// One CTA per sequence decides every row's lock (threshold: compare; top-k:
// radix select of the k-th key, then an ordered tie-break) and compacts its active rows chunk by chunk with warp
// ballots, popcounts and a block scan of the 32 warp counts.  A single
// sequence is done in that one launch.  With B > 1 sequences the decide launch
// leaves each sequence's active count in seg_ptr[b + 1] (encoded as -(count+1))
// and a second launch compacts: CTA b finds its output offset by walking
// seg_ptr down from b, adding encoded counts until it meets an entry another
// CTA has already turned into its final prefix sum (no inter-CTA waiting, no
// scratch memory, O(B) reads per CTA).  Indices come out ascending and
// deterministic.
#include "plk_common.cuh"
#include "plk_internal.h"

namespace plk {

constexpr int kSelThreads = 1024;

__device__ __forceinline__ uint8_t derive_lock(int mode, const float* score, const uint8_t* lock_src,
                                               float tau, long long i) {
  uint8_t l = lock_src[i];
  if (!l && mode == PLK_SEL_THRESH_GT) l = (score[i] > tau) ? 1 : 0;  // NaN compares false
  if (!l && mode == PLK_SEL_THRESH_LT) l = (score[i] < tau) ? 1 : 0;
  return l;
}

__device__ __forceinline__ int block_sum(int v, int* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  int t = (threadIdx.x < nw) ? sh[threadIdx.x] : 0;
  if (warp == 0) {
#pragma unroll
    for (int o = 16; o; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) sh[32] = t;
  }
  __syncthreads();
  return sh[32];
}

// Exclusive block scan of a 0/1 flag; returns this thread's rank and the chunk total.
__device__ __forceinline__ int block_rank(int flag, int* sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  const int wpre = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) sh[warp] = __popc(bal);
  __syncthreads();
  if (warp == 0) {
    const int v = (lane < nw) ? sh[lane] : 0;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += n;
    }
    sh[lane] = inc - v;
    if (lane == 31) sh[32] = inc;
  }
  __syncthreads();
  const int r = sh[warp] + wpre;
  *total = sh[32];
  __syncthreads();
  return r;
}

// The threshold rules, one CTA per sequence: lock_out = lock_in | (score > tau)
// [or < tau].  direct (a single sequence): the active rows are compacted here and
// seg_ptr is final; otherwise seg_ptr[b + 1] = -(active count + 1) for the
// compaction launch.
__global__ void __launch_bounds__(kSelThreads) thresh_decide_kernel(int mode, const float* __restrict__ score,
                                                                    const uint8_t* lock_src, uint8_t* lock_out,
                                                                    int N, float tau, int direct,
                                                                    int32_t* __restrict__ idx_out,
                                                                    int32_t* __restrict__ seg_ptr) {
  __shared__ int sh[33];
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x;
  const long long base = (long long)b * N;
  int running = 0;
  for (int c0 = 0; c0 < N; c0 += blockDim.x) {
    const int i = c0 + threadIdx.x;
    int act = 0;
    if (i < N) {
      const uint8_t l = derive_lock(mode, score, lock_src, tau, base + i);
      lock_out[base + i] = l;
      act = l ? 0 : 1;
    }
    int total;
    const int r = block_rank(act, sh, &total);
    if (direct && act) idx_out[running + r] = (int32_t)(base + i);
    running += total;
  }
  if (threadIdx.x == 0) {
    if (direct) {
      seg_ptr[0] = 0;
      seg_ptr[1] = running;
    } else {
      seg_ptr[b + 1] = -(running + 1);
    }
  }
}

// Output offset of sequence b: the active rows of sequences 0 .. b-1.  seg_ptr[j]
// (j >= 1) holds either -(count of sequence j-1) - 1, left by the decide launch,
// or the final prefix count of sequences 0 .. j-1, written by CTA j-1 of this
// launch; both are single 32-bit writes, so any value read is one of the two.
__device__ __forceinline__ int sel_offset(const int32_t* seg_ptr, int b) {
  int total = 0;
  for (int j = b; j >= 1; --j) {
    const int v = *reinterpret_cast<const volatile int32_t*>(seg_ptr + j);
    if (v >= 0) return total + v;
    total += -v - 1;
  }
  return total;
}

// Compaction of sequence b's rows with lock[b, i] == 0 into idx_out at its
// offset; seg_ptr[b + 1] becomes the final prefix count.
__global__ void __launch_bounds__(kSelThreads) compact_lock_kernel(const uint8_t* __restrict__ lock, int N,
                                                                   int32_t* __restrict__ idx_out,
                                                                   int32_t* __restrict__ seg_ptr) {
  __shared__ int sh[33];
  __shared__ int s_off;
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x;
  const long long base = (long long)b * N;
  if (threadIdx.x == 0) s_off = sel_offset(seg_ptr, b);
  __syncthreads();
  const int offset = s_off;
  int running = 0;
  for (int c0 = 0; c0 < N; c0 += blockDim.x) {
    const int i = c0 + threadIdx.x;
    const int act = (i < N && lock[base + i] == 0) ? 1 : 0;
    int total;
    const int r = block_rank(act, sh, &total);
    if (act) idx_out[offset + running + r] = (int32_t)(base + i);
    running += total;
  }
  if (threadIdx.x == 0) {
    seg_ptr[b + 1] = offset + running;
    if (b == 0) seg_ptr[0] = 0;
  }
}

// Order-preserving key: larger key = more preferred.  NaN maps to 0, below
// every other key; -0 maps like +0.
__device__ __forceinline__ uint32_t pref_key(float s, bool largest) {
  uint32_t u = __float_as_uint(s);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return 0u;  // NaN
  if ((u & 0x7FFFFFFFu) == 0u) u = 0u;               // -0 -> +0
  uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return largest ? k : ~k;
}

// Block-wide radix select on 8-bit digits of pref_key: the key *kth of the
// keep_n-th most preferred candidate (cand(i) true, i < N) and the number
// *remaining of candidates with exactly that key that are kept (the lowest
// indices first).  Requires 0 < keep_n < candidates; every thread of the block
// calls it.  hist[256], s_prefix and s_remaining are shared scratch.
template <typename Cand>
__device__ void block_radix_kth(const float* __restrict__ score, int N, int keep_n, bool largest, Cand cand,
                                int* hist, uint32_t* s_prefix, int* s_remaining, uint32_t* kth, int* remaining) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t prefix = 0, pmask = 0;
  int rem = keep_n;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int t = threadIdx.x; t < 256; t += blockDim.x) hist[t] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < N; i += blockDim.x) {
      if (!cand(i)) continue;
      const uint32_t key = pref_key(score[i], largest);
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns bins 255-8l .. 248-8l (descending); find the bin holding the
      // rem-th most preferred key
      int cnt[8], tot = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        cnt[j] = hist[255 - 8 * lane - j];
        tot += cnt[j];
      }
      int inc = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
      }
      int above = inc - tot;
      if (above < rem && rem <= inc) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (above + cnt[j] >= rem) {
            *s_prefix = prefix | ((uint32_t)(255 - 8 * lane - j) << shift);
            *s_remaining = rem - above;
            break;
          }
          above += cnt[j];
        }
      }
    }
    __syncthreads();
    prefix = *s_prefix;
    rem = *s_remaining;
    pmask |= 0xFFu << shift;
    __syncthreads();
  }
  *kth = prefix;
  *remaining = rem;
}

// One CTA per sequence: among rows with lock_in == 0 keep the k most preferred
// (ties to the lower index) and lock every other row.  Radix select on 8-bit
// digits finds the k-th key (warp-parallel bin search); an ordered block scan
// breaks ties.  direct (a single sequence): the
// kept rows are compacted here; otherwise seg_ptr[b + 1] = -(kept + 1) for the
// compaction launch.  lock_in and lock_out may alias: a CTA reads only its own
// sequence, and each row's lock_in before its lock_out.
__global__ void __launch_bounds__(kSelThreads) topk_decide_kernel(const float* __restrict__ score,
                                                                  const uint8_t* lock_in, uint8_t* lock_out,
                                                                  int N, int k, int largest, int direct,
                                                                  int32_t* __restrict__ idx_out,
                                                                  int32_t* __restrict__ seg_ptr) {
  __shared__ int hist[256];
  __shared__ int sh[33];
  __shared__ uint32_t s_prefix;
  __shared__ int s_remaining;
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x;
  const long long base = (long long)b * N;
  const bool lg = largest != 0;
  int c = 0;
  for (int i = threadIdx.x; i < N; i += blockDim.x) c += lock_in[base + i] ? 0 : 1;
  const int ncand = block_sum(c, sh);
  const int keep_n = k <= 0 ? 0 : min(k, ncand);
  uint32_t kth = 0u;
  int remaining = 0;
  const bool keep_none = keep_n == 0;
  const bool keep_all = !keep_none && keep_n == ncand;
  if (!keep_none && !keep_all) {
    const uint8_t* lk = lock_in + base;
    block_radix_kth(score + base, N, keep_n, lg, [lk](int i) { return lk[i] == 0; }, hist, &s_prefix,
                    &s_remaining, &kth, &remaining);
  }
  // keep: candidates with key > kth, plus the first `remaining` with key == kth
  int taken_eq = 0, running = 0;
  for (int c0 = 0; c0 < N; c0 += blockDim.x) {
    const int i = c0 + threadIdx.x;
    bool cand = false, eq = false, gt = false;
    if (i < N) {
      cand = lock_in[base + i] == 0;
      if (cand && !keep_all && !keep_none) {
        const uint32_t key = pref_key(score[base + i], lg);
        gt = key > kth;
        eq = key == kth;
      }
    }
    int total;
    const int r = block_rank(eq ? 1 : 0, sh, &total);
    const bool keep = cand && !keep_none && (keep_all || gt || (eq && taken_eq + r < remaining));
    taken_eq += total;
    if (i < N) lock_out[base + i] = keep ? 0 : 1;
    int kt;
    const int kr = block_rank(keep ? 1 : 0, sh, &kt);
    if (direct && keep) idx_out[running + kr] = (int32_t)(base + i);
    running += kt;
  }
  if (threadIdx.x == 0) {
    if (direct) {
      seg_ptr[0] = 0;
      seg_ptr[1] = running;
    } else {
      seg_ptr[b + 1] = -(running + 1);
    }
  }
}

int launch_select(const plk_dims* dims, const float* score, const uint8_t* lock_in, uint8_t* lock_out,
                  int mode, float tau, int k, int32_t* idx_out, int32_t* seg_ptr, cudaStream_t st) {
  const int B = dims->B, N = dims->N;
  const int direct = B == 1 ? 1 : 0;
  int e;
  if (mode == PLK_SEL_TOPK_LARGEST || mode == PLK_SEL_TOPK_SMALLEST) {
    e = launch_pdl(topk_decide_kernel, dim3(B), dim3(kSelThreads), 0, st, score, lock_in, lock_out, N, k,
                   (int)(mode == PLK_SEL_TOPK_LARGEST), direct, idx_out, seg_ptr);
  } else
    e = launch_pdl(thresh_decide_kernel, dim3(B), dim3(kSelThreads), 0, st, mode, score, lock_in, lock_out, N, tau,
                   direct, idx_out, seg_ptr);
  if (e != PLK_OK || direct) return e;
  return launch_pdl(compact_lock_kernel, dim3(B), dim3(kSelThreads), 0, st, (const uint8_t*)lock_out, N, idx_out,
                    seg_ptr);
}

}  // namespace plk
