// S7: non-causal attention of the M active queries over all N cached keys of
// their sequence ("Continued Attention" of the SureLock page, "Stopping
// Computation for Converged Tokens in Masked Diffusion-LM Decoding", Sec. 2:
// active tokens keep attending to locked tokens through their cached K/V; cost
// O(M N d) instead of O(N^2 d), Sec. 2 "Algorithmic Complexity").
//
// bf16, hd = 128, on the tcgen05 tensor cores: a CTA takes 128 active queries
// of one sequence and one head and a contiguous range of 64-key chunks.  Warp
// 0 stages Q once and K, V chunk by chunk with TMA (128-byte swizzle, 3-stage
// rings); one thread of warp 1 issues S = Q K^T into TMEM (double-buffered,
// 64 columns each) and O += P V into TMEM (128 columns); warps 2-5 own one
// query row per thread: they read the row's scores from TMEM, keep the running
// row max and sum (online softmax), and write P to shared memory as a bf16 high
// part and a bf16 residual, both multiplied with V, so the softmax weights
// enter P V with ~16 significant bits (a bf16-rounded P would perturb the
// attention output by ~1e-3 relative, which later bf16 roundings amplify).  A
// row keeps a stale max until the new one exceeds it by 2^8 (the weights stay
// below 256, exact in fp32); only then is its O row rescaled in TMEM.  Keys are
// split over CTAs when the query tiles alone leave SMs idle; a combine kernel
// merges the splits.  Keys past N are masked.
// fp32: one thread per (query row, head), online softmax, SIMT.
#include <math.h>

#include <algorithm>

#include "plk_common.cuh"
#include "plk_internal.h"

namespace plk {

namespace {
constexpr int kAttHD = 128;
constexpr int kAttBQ = 128;                    // queries per CTA (UMMA M, one TMEM lane each)
constexpr int kAttBK = 64;                     // keys per chunk (UMMA N of S, K of P V)
constexpr int kAttStages = 3;                  // K and V ring depth
constexpr int kAttThreads = 192;               // warp 0 TMA, warp 1 MMA, warps 2-5 softmax
constexpr int kAttQBytes = kAttBQ * kAttHD * 2;   // 32 KB
constexpr int kAttKVBytes = kAttBK * kAttHD * 2;  // 16 KB
constexpr int kAttPBytes = kAttBQ * kAttBK * 2;   // 16 KB (high or low part)
constexpr size_t kAttOffK = kAttQBytes;
constexpr size_t kAttOffV = kAttOffK + (size_t)kAttStages * kAttKVBytes;
constexpr size_t kAttOffP = kAttOffV + (size_t)kAttStages * kAttKVBytes;  // [2 buffers][high, low]
constexpr size_t kAttOffBar = kAttOffP + 4 * (size_t)kAttPBytes;
constexpr int kAttSmem = (int)kAttOffBar + 256 + 1024;
constexpr uint32_t kAttTmemCols = 256;         // O: 0..127, S buffers: 128..191, 192..255
constexpr float kAttStaleMax = 8.f;            // log2 headroom before a row's O is rescaled

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// hi = bf16(x) packed, lo = bf16(x - hi) packed
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
  __nv_bfloat162 hv;
  hv.x = h0;
  hv.y = h1;
  hi = *reinterpret_cast<uint32_t*>(&hv);
  lo = pack_bf16(x0 - __bfloat162float(h0), x1 - __bfloat162float(h1));
}

// Shared-memory descriptor of an MN-major operand tile with 128-byte swizzle:
// rows of 64 MN-elements (128 B), 8-row groups 1024 B apart along K, 64-wide MN
// blocks `mn_block_bytes` apart.  The V chunk [64 keys][128 dims], stored as two
// 64-dim TMA boxes, is the B operand of P V in this form (K = keys, N = dims).
__device__ __forceinline__ uint64_t sdesc_sw128_mn(uint32_t saddr, uint32_t mn_block_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((mn_block_bytes >> 4) & 0x3FFFu) << 16;  // leading byte offset: next MN block
  d |= (uint64_t)(1024 >> 4) << 32;                          // stride byte offset: next 8 K-rows
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
}  // namespace

// Key splits for the current active set (device-side M, no host sync): the
// split count s <= smax minimising whole waves of CTAs x chunks per CTA, one
// CTA per SM, plus one chunk's worth for the combine when s > 1.  Splits are
// considered only while the query tiles x heads leave SMs idle.  Computed
// identically by the attention and combine kernels.
__device__ __forceinline__ int attn_qtiles(const int32_t* seg_ptr, int B) {
  int qt = 0;
  for (int b = 0; b < B; ++b) qt += ceil_div(seg_ptr[b + 1] - seg_ptr[b], kAttBQ);
  return qt;
}
__device__ __forceinline__ int attn_splits(const int32_t* seg_ptr, int B, int H, int N, int smax, int nsm) {
  const int items = attn_qtiles(seg_ptr, B) * H;
  if (items == 0 || items >= nsm) return 1;
  const int nch = ceil_div(N, kAttBK);
  int best = 1, best_cost = 1 << 30;
  for (int s = 1; s <= smax && s <= nch; ++s) {
    const int cost = ceil_div(items * s, nsm) * ceil_div(nch, s) * 2 + (s > 1 ? 1 : 0);
    if (cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

// Split partials: o_part[s][row][d] (unnormalised, fp32) and ml[s][row][h] = (max, sum)
// in the log2 domain; rows are compact active-row indices below part_rows.
struct AttnSplit {
  float* o_part;
  float2* ml;
  int smax, part_rows, nsm;
};

// One work item: 128 queries [r0, r0 + nrows) of sequence b, head h, chunks [c0, c1).
struct AttnItem {
  int b, h, split, r0, nrows, c0, c1;
};
__device__ __forceinline__ AttnItem attn_item(int i, const int32_t* seg_ptr, int B, int H, int N, int S) {
  AttnItem it;
  it.split = i % S;
  const int rest = i / S;
  it.h = rest % H;
  int qi = rest / H, b = 0;
  for (; b < B; ++b) {
    const int qt = ceil_div(seg_ptr[b + 1] - seg_ptr[b], kAttBQ);
    if (qi < qt) break;
    qi -= qt;
  }
  it.b = b;
  it.r0 = seg_ptr[b] + qi * kAttBQ;
  it.nrows = min(kAttBQ, seg_ptr[b + 1] - it.r0);
  const int nch = ceil_div(N, kAttBK);
  it.c0 = it.split * nch / S;
  it.c1 = (it.split + 1) * nch / S;
  return it;
}

__global__ void __launch_bounds__(kAttThreads, 1) attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                               const __grid_constant__ CUtensorMap tmK,
                                                               const __grid_constant__ CUtensorMap tmV,
                                                               __nv_bfloat16* __restrict__ Aout,
                                                               const int32_t* __restrict__ seg_ptr, int B, int N,
                                                               int H, int d, float scale_log2, AttnSplit sp) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kAttOffK;
  uint8_t* sV = smem + kAttOffV;
  uint8_t* sP = smem + kAttOffP;  // buffer x: high part at 2x, low part at 2x + 1 (16 KB each)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kAttOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_free = bars + 1;
  uint64_t* k_full = bars + 2;    // [3]
  uint64_t* k_empty = bars + 5;   // [3]
  uint64_t* v_full = bars + 8;    // [3]
  uint64_t* v_empty = bars + 11;  // [3]
  uint64_t* s_full = bars + 14;   // [2] scores of a chunk in TMEM
  uint64_t* s_free = bars + 16;   // [2] scores read by the 4 softmax warps
  uint64_t* p_full = bars + 18;   // [2] P of a chunk in shared memory (4 softmax warps)
  uint64_t* p_free = bars + 20;   // [2] the P V that read P buffer x has completed
  uint64_t* o_free = bars + 22;   // O read out by the 4 softmax warps
  uint64_t* drain = bars + 23;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 24);
  volatile int* s_abort = reinterpret_cast<volatile int*>(bars + 25);

  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = attn_splits(seg_ptr, B, H, N, sp.smax, sp.nsm);
  const int nitems = attn_qtiles(seg_ptr, B) * H * S;
  if ((int)blockIdx.x >= nitems) return;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_free, 1);
    for (int i = 0; i < kAttStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&p_free[i], 1);
    }
    mbar_init(o_free, 4);
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kAttTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      long long g = 0;  // chunk counter over this CTA's items
      int t = 0;        // item counter
      for (int i = blockIdx.x; i < nitems && !*s_abort; i += gridDim.x, ++t) {
        const AttnItem it = attn_item(i, seg_ptr, B, H, N, S);
        const int hc = it.h * kAttHD;
        if (!mbar_wait(q_free, (uint32_t)((t & 1) ^ 1))) {
          *s_abort = 1;
          break;
        }
        mbar_expect_tx(q_full, kAttQBytes);
        tma_load_2d(sQ, &tmQ, hc, it.r0, q_full);
        tma_load_2d(sQ + kAttQBytes / 2, &tmQ, hc + 64, it.r0, q_full);
        for (int c = it.c0; c < it.c1; ++c, ++g) {
          const int st = (int)(g % kAttStages);
          const uint32_t ph = (uint32_t)((g / kAttStages) & 1);
          const int y = it.b * N + c * kAttBK;
          if (!mbar_wait(&k_empty[st], ph ^ 1)) {
            *s_abort = 1;
            break;
          }
          mbar_expect_tx(&k_full[st], kAttKVBytes);
          tma_load_2d(sK + st * kAttKVBytes, &tmK, hc, y, &k_full[st]);
          tma_load_2d(sK + st * kAttKVBytes + kAttKVBytes / 2, &tmK, hc + 64, y, &k_full[st]);
          if (!mbar_wait(&v_empty[st], ph ^ 1)) {
            *s_abort = 1;
            break;
          }
          mbar_expect_tx(&v_full[st], kAttKVBytes);
          tma_load_2d(sV + st * kAttKVBytes, &tmV, hc, y, &v_full[st]);
          tma_load_2d(sV + st * kAttKVBytes + kAttKVBytes / 2, &tmV, hc + 64, y, &v_full[st]);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      const uint32_t idesc_s = idesc_bf16(kAttBQ, kAttBK);
      const uint32_t idesc_pv = idesc_bf16(kAttBQ, kAttHD) | (1u << 16);  // B = V chunk, MN-major
      const uint32_t q0 = smem_u32(sQ);
      long long g = 0;
      int t = 0;
      bool any = false;
      // O += P_hi V + P_lo V for global chunk gj (first: the item's first chunk overwrites O)
      auto issue_pv = [&](long long gj, bool first) -> bool {
        const int pb = (int)(gj & 1), st = (int)(gj % kAttStages);
        if (first && !mbar_wait(o_free, (uint32_t)((t & 1) ^ 1))) return false;  // last item's O read
        if (!mbar_wait(&p_full[pb], (uint32_t)((gj >> 1) & 1))) return false;
        if (!mbar_wait(&v_full[st], (uint32_t)((gj / kAttStages) & 1))) return false;
        tc_fence_after();
        const uint32_t vb = smem_u32(sV + st * kAttKVBytes);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint64_t pdesc = sdesc_sw128(smem_u32(sP + (2 * pb + part) * kAttPBytes));
#pragma unroll
          for (int k = 0; k < kAttBK / 16; ++k)  // 16 keys per step: +32 B of P rows, +2 KB of V rows
            umma_bf16(tmem_base, pdesc + 2 * k, sdesc_sw128_mn(vb + k * 2048, kAttKVBytes / 2), idesc_pv,
                      (!first || part > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(&v_empty[st]);
        umma_commit(&p_free[pb]);  // also: every earlier MMA, so O holds chunks <= gj
        return true;
      };
      for (int i = blockIdx.x; i < nitems && !*s_abort; i += gridDim.x, ++t) {
        const AttnItem it = attn_item(i, seg_ptr, B, H, N, S);
        const int n = it.c1 - it.c0;
        bool ok = mbar_wait(q_full, (uint32_t)(t & 1));
        tc_fence_after();
        for (int j = 0; j < n && ok; ++j) {
          const long long gj = g + j;
          const int sb = (int)(gj & 1), st = (int)(gj % kAttStages);
          ok = mbar_wait(&s_free[sb], (uint32_t)(((gj >> 1) & 1) ^ 1)) &&
               mbar_wait(&k_full[st], (uint32_t)((gj / kAttStages) & 1));
          if (!ok) break;
          tc_fence_after();
          const uint32_t kb = smem_u32(sK + st * kAttKVBytes);
#pragma unroll
          for (int k = 0; k < kAttHD / 16; ++k) {  // 16 dims per step: box k / 4, +32 B within it
            const uint32_t qa = q0 + (k >> 2) * (kAttQBytes / 2), ka = kb + (k >> 2) * (kAttKVBytes / 2);
            umma_bf16(tmem_base + 128 + sb * 64, sdesc_sw128(qa) + 2 * (k & 3), sdesc_sw128(ka) + 2 * (k & 3),
                      idesc_s, k > 0 ? 1u : 0u);
          }
          any = true;
          umma_commit(&s_full[sb]);
          umma_commit(&k_empty[st]);
          if (j >= 1) ok = issue_pv(gj - 1, j == 1);  // P V of the previous chunk overlaps this softmax
        }
        if (ok) ok = issue_pv(g + n - 1, n == 1);
        if (!ok) {
          *s_abort = 1;
          break;
        }
        umma_commit(q_free);  // every MMA reading this Q has completed
        g += n;
      }
      if (*s_abort && any) {
        umma_commit(drain);
        (void)mbar_wait(drain, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax: one query row per thread
    const int q = warp & 3;  // a warp reads TMEM lanes 32 * (warp % 4) ..
    const int row = q * 32 + lane;
    const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);
    const int nch = ceil_div(N, kAttBK);
    long long g = 0;
    int t = 0;
    bool ok = true;
    // waits until the P V of global chunk k (and every MMA before it) has completed; k's
    // buffer cannot have moved on, its next P V needs P of chunk k + 2 from these warps
    auto wait_pv = [&](long long k) -> bool {
      return k < 0 || mbar_wait(&p_free[k & 1], (uint32_t)((k >> 1) & 1));
    };
    for (int i = blockIdx.x; i < nitems && ok; i += gridDim.x, ++t) {
      const AttnItem it = attn_item(i, seg_ptr, B, H, N, S);
      const int n = it.c1 - it.c0;
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j < n; ++j) {
        const long long gj = g + j;
        const int sb = (int)(gj & 1);
        ok = mbar_wait(&s_full[sb], (uint32_t)((gj >> 1) & 1)) && !*s_abort;
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t ra[32], rb[32];
        tmem_ld32(lane_base + 128 + sb * 64, ra);
        tmem_ld32(lane_base + 128 + sb * 64 + 32, rb);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[sb]);
        float sc[kAttBK];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          sc[e] = __uint_as_float(ra[e]);
          sc[32 + e] = __uint_as_float(rb[e]);
        }
        const int key0 = (it.c0 + j) * kAttBK;
        if (key0 + kAttBK > N) {
#pragma unroll
          for (int e = 0; e < kAttBK; ++e)
            if (key0 + e >= N) sc[e] = -INFINITY;
        }
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < kAttBK; ++e) mx = fmaxf(mx, sc[e]);
        const float mc = mx * scale_log2;  // every chunk holds at least one key < N
        const bool need = mc > m_used + kAttStaleMax;
        float factor = 1.f;
        if (need) {
          factor = exp2f(m_used - mc);  // 0 for the first chunk
          m_used = mc;
        }
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          // the previous chunks' P V must be complete before O rows are rescaled
          ok = wait_pv(gj - 1);
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int cb = 0; cb < kAttHD / 32; ++cb) {
            uint32_t o[32];
            tmem_ld32(lane_base + cb * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
            tmem_st32(lane_base + cb * 32, o);
          }
          tmem_st_wait();
        }
        l *= factor;
        ok = wait_pv(gj - 2);  // the P V that read P buffer sb has completed
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        // P = 2^(s * scale - m_used) <= 2^8, as bf16 high + low parts, K-major with 128-byte swizzle
        uint8_t* ph = sP + (2 * sb) * kAttPBytes;
        uint8_t* pl = ph + kAttPBytes;
        const uint32_t rowoff = (uint32_t)((row >> 3) * 1024 + (row & 7) * 128);
#pragma unroll
        for (int c = 0; c < kAttBK / 8; ++c) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float p0 = exp2f(fmaf(sc[c * 8 + 2 * e], scale_log2, -m_used));
            const float p1 = exp2f(fmaf(sc[c * 8 + 2 * e + 1], scale_log2, -m_used));
            l += p0 + p1;
            split_pair(p0, p1, hi[e], lo[e]);
          }
          const uint32_t off = rowoff + ((uint32_t)(c ^ (row & 7)) << 4);
          *reinterpret_cast<uint4*>(ph + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(pl + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
        fence_proxy_async_smem();  // P visible to the tensor cores
        tc_fence_before();         // and any O rescale ordered before the next P V
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[sb]);
      }
      if (!ok) break;
      ok = wait_pv(g + n - 1);  // O is final
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool whole = (n == nch);  // no key split: normalise and store bf16
      const int grow = it.r0 + row;
      const float inv = 1.0f / l;
#pragma unroll
      for (int cb = 0; cb < kAttHD / 32; ++cb) {
        uint32_t o[32];
        tmem_ld32(lane_base + cb * 32, o);
        tmem_ld_wait();
        if (row < it.nrows) {
          if (whole) {
            uint4* dst = reinterpret_cast<uint4*>(Aout + (size_t)grow * d + it.h * kAttHD + cb * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(pack_bf16(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv),
                                  pack_bf16(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv),
                                  pack_bf16(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv),
                                  pack_bf16(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv));
          } else {
            float4* dst = reinterpret_cast<float4*>(sp.o_part + ((size_t)it.split * sp.part_rows + grow) * d +
                                                    it.h * kAttHD + cb * 32);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[v] = make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                   __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
          }
        }
      }
      if (!whole && row < it.nrows) sp.ml[((size_t)it.split * sp.part_rows + grow) * H + it.h] = make_float2(m_used, l);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);
      g += n;
    }
    if (!ok && lane == 0) *s_abort = 1;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kAttTmemCols);
  }
}

// out[row, h] = sum_s 2^(m_s - m) o_s / sum_s 2^(m_s - m) l_s, one CTA per active row.
__global__ void __launch_bounds__(256) attn_combine_kernel(const int32_t* __restrict__ seg_ptr, int B, int H,
                                                           int N, int d, AttnSplit sp,
                                                           __nv_bfloat16* __restrict__ Aout) {
  pdl_wait();
  pdl_trigger();
  const int j = blockIdx.x;
  if (j >= seg_ptr[B]) return;
  const int S = attn_splits(seg_ptr, B, H, N, sp.smax, sp.nsm);
  if (S == 1) return;
  for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4) {
    const int h = c / kAttHD;
    float m = -INFINITY;
    for (int s = 0; s < S; ++s) m = fmaxf(m, sp.ml[((size_t)s * sp.part_rows + j) * H + h].x);
    float l = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < S; ++s) {
      const float2 ml = sp.ml[((size_t)s * sp.part_rows + j) * H + h];
      const float w = exp2f(ml.x - m);
      l = fmaf(w, ml.y, l);
      const float4 o = *reinterpret_cast<const float4*>(sp.o_part + ((size_t)s * sp.part_rows + j) * d + c);
      acc[0] = fmaf(w, o.x, acc[0]);
      acc[1] = fmaf(w, o.y, acc[1]);
      acc[2] = fmaf(w, o.z, acc[2]);
      acc[3] = fmaf(w, o.w, acc[3]);
    }
    const float inv = 1.0f / l;
    uint2 u;
    u.x = pack_bf16(acc[0] * inv, acc[1] * inv);
    u.y = pack_bf16(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(Aout + (size_t)j * d + c) = u;
  }
}

template <int HD>
__global__ void attn_f32_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                                const float* __restrict__ V, float* __restrict__ A,
                                const int32_t* __restrict__ seg_ptr, int B, int N, int d, int H, float scale) {
  const int gid = blockIdx.x * blockDim.x + threadIdx.x;
  const int j = gid / H, h = gid - j * H;
  const int M = seg_ptr[B];
  if (j >= M) return;
  int b = 0;
  while (b + 1 < B && seg_ptr[b + 1] <= j) ++b;
  float q[HD], o[HD];
#pragma unroll
  for (int c = 0; c < HD; ++c) {
    q[c] = Q[(size_t)j * d + h * HD + c];
    o[c] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int n = 0; n < N; ++n) {
    const float* kr = K + ((size_t)b * N + n) * d + h * HD;
    const float* vr = V + ((size_t)b * N + n) * d + h * HD;
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < HD; ++c) s = fmaf(q[c], kr[c], s);
    s *= scale;
    const float m_new = fmaxf(m, s);
    const float alpha = expf(m - m_new), p = expf(s - m_new);
    l = l * alpha + p;
#pragma unroll
    for (int c = 0; c < HD; ++c) o[c] = fmaf(p, vr[c], o[c] * alpha);
    m = m_new;
  }
  const float inv = 1.0f / l;
#pragma unroll
  for (int c = 0; c < HD; ++c) A[(size_t)j * d + h * HD + c] = o[c] * inv;
}

int attn_split_rows(const plk_dims* dims, int num_sms) {
  // keys are split only while query tiles x heads < SMs, so fewer active rows than this
  const int rows = ceil_div(num_sms, dims->H) * kAttBQ;
  return std::min(dims->B * dims->N, rows);
}

int launch_attention_bf16(const plk_dims* dims, const void* q, const void* K_cache, const void* V_cache,
                          void* a_out, const int32_t* seg_ptr, float* o_part, void* ml, int smax, int part_rows,
                          int num_sms, cudaStream_t st) {
  const int B = dims->B, N = dims->N, d = dims->d, H = dims->H;
  CUtensorMap tmQ, tmK, tmV;
  if (make_tmap_bf16(&tmQ, q, (uint64_t)B * N, (uint64_t)d, kAttBQ) != PLK_OK) return PLK_ERR_CUDA;
  if (make_tmap_bf16(&tmK, K_cache, (uint64_t)B * N, (uint64_t)d, kAttBK) != PLK_OK) return PLK_ERR_CUDA;
  if (make_tmap_bf16(&tmV, V_cache, (uint64_t)B * N, (uint64_t)d, kAttBK) != PLK_OK) return PLK_ERR_CUDA;
  static int attr_done[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PLK_ERR_CUDA;
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttSmem) != cudaSuccess)
      return PLK_ERR_CUDA;
    attr_done[dev] = 1;
  }
  const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)dims->hd));
  AttnSplit sp{o_part, (float2*)ml, std::max(1, std::min(smax, ceil_div(N, kAttBK))), part_rows, num_sms};
  // persistent: one CTA per SM walks the (query tile, head, key split) items
  const int rc = launch_pdl(attn_tc_kernel, dim3(num_sms), dim3(kAttThreads), kAttSmem, st, tmQ, tmK, tmV,
                            (__nv_bfloat16*)a_out, seg_ptr, B, N, H, d, scale_log2, sp);
  if (rc != PLK_OK || sp.smax == 1) return rc;
  return launch_pdl(attn_combine_kernel, dim3(part_rows), dim3(256), 0, st, seg_ptr, B, H, N, d, sp,
                    (__nv_bfloat16*)a_out);
}

int launch_attention_f32(const plk_dims* dims, const float* q, const float* K_cache, const float* V_cache,
                         float* a_out, const int32_t* seg_ptr, int Mcap, cudaStream_t st) {
  const int B = dims->B, N = dims->N, d = dims->d, H = dims->H, hd = dims->hd;
  const float scale = (float)(1.0 / sqrt((double)hd));
  const int threads = 128, blocks = ceil_div(Mcap * H, threads);
  switch (hd) {
    case 16: attn_f32_kernel<16><<<blocks, threads, 0, st>>>(q, K_cache, V_cache, a_out, seg_ptr, B, N, d, H, scale); break;
    case 32: attn_f32_kernel<32><<<blocks, threads, 0, st>>>(q, K_cache, V_cache, a_out, seg_ptr, B, N, d, H, scale); break;
    case 64: attn_f32_kernel<64><<<blocks, threads, 0, st>>>(q, K_cache, V_cache, a_out, seg_ptr, B, N, d, H, scale); break;
    case 128: attn_f32_kernel<128><<<blocks, threads, 0, st>>>(q, K_cache, V_cache, a_out, seg_ptr, B, N, d, H, scale); break;
    default: return PLK_ERR_SHAPE;
  }
  return cudaPeekAtLastError() == cudaSuccess ? PLK_OK : PLK_ERR_CUDA;
}

}  // namespace plk
