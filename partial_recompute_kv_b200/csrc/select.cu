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
// ballots, popcounts and a block scan of the 32 warp counts; top-k on sequences
// of 2049 .. 32768 rows runs on a cluster of up to 8 CTAs per sequence instead
// (keys in registers, histograms merged through distributed shared memory).  A
// single sequence is done in that one launch.  With B > 1 sequences the decide launch
// leaves each sequence's active count in seg_ptr[b + 1] (encoded as -(count+1))
// and a second launch compacts: CTA b finds its output offset by walking
// seg_ptr down from b, adding encoded counts until it meets an entry another
// CTA has already turned into its final prefix sum (no inter-CTA waiting, no
// scratch memory, O(B) reads per CTA).  Indices come out ascending and
// deterministic.
#include <algorithm>

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

// ---------------------------------------------------------------------------
// The top-k rule with the keys in registers, on a cluster of 2 <= S <= 8 CTAs of
// NT threads per sequence (sequences of more than 2048 rows).  CTA s owns rows
// [s L, min((s + 1) L, N)), L = ceil(N / S); thread t keeps the keys of rows
// s L + t + NT j (j < KPT), so the scores are read once.  Every radix pass
// builds a 256-bin histogram per CTA (two buffers, alternating, so one cluster
// barrier per pass suffices) and every CTA sums the S histograms through
// distributed shared memory and finds the same digit; the first pass's bins
// also count the candidates.  Then each CTA publishes its count of rows kept
// for sure and of ties at the k-th key: the ties kept are the lowest indices,
// so a CTA's ties and kept rows come after those of the CTAs of lower rank and
// the result equals the one-CTA kernel's.  direct (one sequence): the CTAs
// compact their kept rows at their offsets; otherwise rank 0 leaves
// seg_ptr[b + 1] = -(kept + 1) for the compaction launch.
__device__ __forceinline__ int ld_dsmem_s32(const int* p, uint32_t rank) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(dsmem_addr(smem_u32(p), rank)));
  return v;
}
// p's value summed over the S CTAs of the cluster (the loads are all issued before the adds)
__device__ __forceinline__ int cluster_sum(const int* p, int S, int upto) {
  int v[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) v[r] = ld_dsmem_s32(p, (uint32_t)(r < S ? r : 0));
  int tot = 0;
#pragma unroll
  for (int r = 0; r < 8; ++r) tot += r < upto ? v[r] : 0;
  return tot;
}

constexpr int kSelClusterThreads = 256;

template <int KPT, int NT, bool CL>
__global__ void __launch_bounds__(NT) topk_cluster_kernel(const float* __restrict__ score,
                                                                          const uint8_t* lock_in, uint8_t* lock_out,
                                                                          int N, int k, int largest, int direct,
                                                                          int S, int32_t* __restrict__ idx_out,
                                                                          int32_t* __restrict__ seg_ptr) {
  __shared__ int hist[2][256];
  __shared__ int gh[256];    // the cluster's histogram of the current pass
  __shared__ int pub[2];     // published to the cluster: rows kept for sure, ties at the k-th key
  __shared__ int sh[33];
  __shared__ uint32_t s_prefix;
  __shared__ int s_rem, s_ncand;
  pdl_wait();
  pdl_trigger();
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int s = CL ? (int)cluster_ctarank() : 0;
  const int b = blockIdx.y;
  const long long base = (long long)b * N;
  const int L = (N + S - 1) / S;
  const int lo = s * L, hi = min(N, lo + L);
  const bool lg = largest != 0;
  uint32_t key[KPT];
  bool cand[KPT];
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    const int i = lo + t + NT * j;
    cand[j] = i < hi && lock_in[base + i] == 0;
    key[j] = cand[j] ? pref_key(score[base + i], lg) : 0u;
  }
  uint32_t prefix = 0u, pmask = 0u;
  int rem = 0, ncand = 0, keep_n = 0;
  bool keep_none = true, keep_all = false;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    int* hb = hist[pass & 1];  // the other buffer may still be read by the cluster
    if (t < 256) hb[t] = 0;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < KPT; ++j)
      if (cand[j] && (key[j] & pmask) == prefix) atomicAdd(&hb[(key[j] >> shift) & 255u], 1);
    if (CL) {
      cluster_sync_all();  // every CTA's histogram of this pass is complete
      if (t < 256) gh[t] = cluster_sum(&hb[t], S, S);
    } else {
      __syncthreads();
      if (t < 256) gh[t] = hb[t];
    }
    __syncthreads();
    if (pass == 0) {  // every candidate is in the first pass's histogram
      if (warp == 0) {
        int c = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) c += gh[lane * 8 + q];
#pragma unroll
        for (int o = 16; o; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        if (lane == 0) s_ncand = c;
      }
      __syncthreads();
      ncand = s_ncand;
      keep_n = k <= 0 ? 0 : min(k, ncand);
      keep_none = keep_n == 0;
      keep_all = !keep_none && keep_n == ncand;
      rem = keep_n;
      if (keep_none || keep_all) break;  // the same in every CTA
    }
    if (warp == 0) {
      // lane l owns bins 255-8l .. 248-8l (descending); find the bin holding the
      // rem-th most preferred key
      int cnt[8], tt = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        cnt[q] = gh[255 - 8 * lane - q];
        tt += cnt[q];
      }
      int inc = tt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += n;
      }
      int above = inc - tt;
      if (above < rem && rem <= inc) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (above + cnt[q] >= rem) {
            s_prefix = prefix | ((uint32_t)(255 - 8 * lane - q) << shift);
            s_rem = rem - above;
            break;
          }
          above += cnt[q];
        }
      }
    }
    __syncthreads();
    prefix = s_prefix;
    rem = s_rem;
    pmask |= 0xFFu << shift;
  }
  const bool sel = !keep_none && !keep_all;
  const uint32_t kth = prefix;
  const int remaining = sel ? rem : 0;  // ties at kth that are kept, lowest indices first
  // this CTA's rows kept for sure (every candidate, or the keys above the k-th) and its ties
  int gtc = 0, eqc = 0;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {
    gtc += (cand[j] && (keep_all || (sel && key[j] > kth))) ? 1 : 0;
    eqc += (sel && cand[j] && key[j] == kth) ? 1 : 0;
  }
  gtc = block_sum(gtc, sh);
  eqc = block_sum(eqc, sh);
  if (t == 0) {
    pub[0] = gtc;
    pub[1] = eqc;
  }
  if (CL)
    cluster_sync_all();
  else
    __syncthreads();
  // kept rows of CTA r: its sure rows plus its share of the ties, taken in rank order
  int before = 0, all = 0, eq_before = 0;
  {
    int gv[8], ev[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      gv[r] = CL ? ld_dsmem_s32(&pub[0], (uint32_t)(r < S ? r : 0)) : pub[0];
      ev[r] = CL ? ld_dsmem_s32(&pub[1], (uint32_t)(r < S ? r : 0)) : pub[1];
    }
    int taken = 0;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      if (r < S) {
        const int kr = gv[r] + max(0, min(ev[r], remaining - taken));
        if (r < s) {
          before += kr;
          eq_before += ev[r];
        }
        all += kr;
        taken += ev[r];
      }
    }
  }
  int taken_eq = eq_before, running = before;
#pragma unroll
  for (int j = 0; j < KPT; ++j) {  // row order: j, then t
    const bool eq = sel && cand[j] && key[j] == kth;
    const bool gt = sel && cand[j] && key[j] > kth;
    int total;
    const int r = block_rank(eq ? 1 : 0, sh, &total);
    const bool keep = cand[j] && !keep_none && (keep_all || gt || (eq && taken_eq + r < remaining));
    taken_eq += total;
    const int i = lo + t + NT * j;
    if (i < hi) lock_out[base + i] = keep ? 0 : 1;
    if (direct) {
      int kt;
      const int kr = block_rank(keep ? 1 : 0, sh, &kt);
      if (keep) idx_out[running + kr] = (int32_t)(base + i);
      running += kt;
    }
  }
  if (s == 0 && t == 0) {
    if (direct) {
      seg_ptr[0] = 0;
      seg_ptr[1] = all;
    } else {
      seg_ptr[b + 1] = -(all + 1);
    }
  }
  if (CL) cluster_sync_all();  // no CTA leaves while another can still read its shared memory
}

int launch_select(const plk_dims* dims, const float* score, const uint8_t* lock_in, uint8_t* lock_out,
                  int mode, float tau, int k, int32_t* idx_out, int32_t* seg_ptr, cudaStream_t st) {
  const int B = dims->B, N = dims->N;
  const int direct = B == 1 ? 1 : 0;
  int e;
  const int largest = (int)(mode == PLK_SEL_TOPK_LARGEST);
  const bool topk = mode == PLK_SEL_TOPK_LARGEST || mode == PLK_SEL_TOPK_SMALLEST;
  // keys in registers: sequences of up to 2048 rows on one CTA of 1024 threads, longer
  // ones on a cluster of S CTAs of 256 threads (512 rows each and more, at most 4096
  // each); longer than 8 x 4096 rows: the one-CTA kernel that reads the scores per pass
  const int S = std::min(8, ceil_div(N, 512));
  const int NT = kSelClusterThreads;
  const int kpt = ceil_div(ceil_div(N, S), NT);
  if (topk && N <= kSelThreads) {
    e = launch_pdl(topk_cluster_kernel<1, kSelThreads, false>, dim3(1, B), dim3(kSelThreads), 0, st, score,
                   lock_in, lock_out, N, k, largest, direct, 1, idx_out, seg_ptr);
  } else if (topk && N <= 2 * kSelThreads) {
    e = launch_pdl(topk_cluster_kernel<2, kSelThreads, false>, dim3(1, B), dim3(kSelThreads), 0, st, score,
                   lock_in, lock_out, N, k, largest, direct, 1, idx_out, seg_ptr);
  } else if (topk && kpt <= 16) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)S, (unsigned)B, 1);
    cfg.blockDim = dim3((unsigned)NT, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    at[1].id = cudaLaunchAttributeClusterDimension;
    at[1].val.clusterDim.x = (unsigned)S;
    at[1].val.clusterDim.y = 1;
    at[1].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    cudaError_t ce;
#define PLK_TOPK_LAUNCH(KPT_, NT_)                                                                        \
  ce = cudaLaunchKernelEx(&cfg, topk_cluster_kernel<KPT_, NT_, true>, score, lock_in, lock_out, N, k, largest, \
                          direct, S, idx_out, seg_ptr)
    if (kpt <= 2)
      PLK_TOPK_LAUNCH(2, kSelClusterThreads);
    else if (kpt <= 4)
      PLK_TOPK_LAUNCH(4, kSelClusterThreads);
    else if (kpt <= 8)
      PLK_TOPK_LAUNCH(8, kSelClusterThreads);
    else
      PLK_TOPK_LAUNCH(16, kSelClusterThreads);
#undef PLK_TOPK_LAUNCH
    e = ce == cudaSuccess ? PLK_OK : PLK_ERR_CUDA;
  } else if (topk) {  // longer sequences: the one-CTA kernel that reads the scores per pass
    e = launch_pdl(topk_decide_kernel, dim3(B), dim3(kSelThreads), 0, st, score, lock_in, lock_out, N, k, largest,
                   direct, idx_out, seg_ptr);
  } else
    e = launch_pdl(thresh_decide_kernel, dim3(B), dim3(kSelThreads), 0, st, mode, score, lock_in, lock_out, N, tau,
                   direct, idx_out, seg_ptr);
  if (e != PLK_OK || direct) return e;
  return launch_pdl(compact_lock_kernel, dim3(B), dim3(kSelThreads), 0, st, (const uint8_t*)lock_out, N, idx_out,
                    seg_ptr);
}

}  // namespace plk
