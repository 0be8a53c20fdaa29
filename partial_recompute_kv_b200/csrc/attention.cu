// S7: non-causal attention of the M active queries over all N cached keys of
// their sequence ("Continued Attention" of the SureLock page, "Stopping
// Computation for Converged Tokens in Masked Diffusion-LM Decoding", Sec. 2:
// active tokens keep attending to locked tokens through their cached K/V; cost
// O(M N d) instead of O(N^2 d), Sec. 2 "Algorithmic Complexity").
//
// bf16, hd = 128, on the tcgen05 tensor cores: a CTA takes 128 active queries
// of one sequence and one head and a contiguous range of 64-key chunks.  The
// queries come as a bf16 pair q = q_hi + q_lo (q_lo = bf16(q - q_hi)), so the
// scores see ~16 significant bits of q.  Warp 0 stages both Q tiles once and K
// chunk by chunk, warp 10 stages V chunk by chunk, with TMA (128-byte swizzle;
// a 3-stage K ring and a 2-stage V ring, each with its own producer so a K load
// never waits behind a V stage); one thread of warp 1 issues
// S = Q_hi K^T + Q_lo K^T into TMEM (double-buffered, 64 columns each) and
// O += P V into TMEM (128 columns); warps 2-5 own one
// query row per thread: they read the row's scores from TMEM, keep the running
// row max and sum (online softmax), and write P to shared memory as a bf16 high
// part and a bf16 residual, both multiplied with V, so the softmax weights
// enter P V with ~16 significant bits (a bf16-rounded P would perturb the
// attention output by ~1e-3 relative, which later bf16 roundings amplify).  A
// row keeps a stale max until the new one exceeds it by 2^8 (the weights stay
// below 256, exact in fp32); only then is its O row rescaled in TMEM.  When the
// query tiles alone leave SMs idle, the two CTAs of a cluster pair split a
// tile's keys: the odd CTA hands its partial O, row max and row sum to the even
// CTA through distributed shared memory, which merges and writes the tile.  When
// even that leaves pairs idle, a unit's keys are cut into up to 4 parts, one
// pair each; the pairs store their partials in global scratch and the pair
// that completes the unit last (a per-unit counter) merges them.
// The output a goes out as a bf16 hi/lo pair as well.
// Keys past N are masked.  Under grouped-query attention the K/V tiles of query
// head h come from K/V head h / (H / Hkv) of the Hkv-head caches; the query
// heads of a group are separate units whose K/V reads meet in L2.
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
constexpr int kAttKStages = 3;                 // K ring depth
constexpr int kAttVStages = 2;                 // V ring depth
constexpr int kAttSoftWarps = 8;               // two warps per TMEM lane quarter, one per half row
constexpr int kAttVWarp = 2 + kAttSoftWarps;   // warp 10: the V producer
constexpr int kAttThreads = 32 * (3 + kAttSoftWarps);  // warp 0 Q/K TMA, warp 1 MMA, warps 2-9 softmax, warp 10 V TMA
constexpr int kAttQBytes = kAttBQ * kAttHD * 2;   // 32 KB (hi or lo part)
constexpr int kAttKVBytes = kAttBK * kAttHD * 2;  // 16 KB
constexpr int kAttPBytes = kAttBQ * kAttBK * 2;   // 16 KB (high or low part)
constexpr size_t kAttOffK = 2 * (size_t)kAttQBytes;
constexpr size_t kAttOffV = kAttOffK + (size_t)kAttKStages * kAttKVBytes;
constexpr size_t kAttOffP = kAttOffV + (size_t)kAttVStages * kAttKVBytes;  // [2 buffers][high, low]
constexpr size_t kAttOffML = kAttOffP + 4 * (size_t)kAttPBytes;            // [128] (max, sum) of the odd CTA
constexpr size_t kAttOffXM = kAttOffML + kAttBQ * 8;                       // [2][2 halves][128] row max
constexpr size_t kAttOffXL = kAttOffXM + 2 * 2 * kAttBQ * 4;               // [2 halves][128] row sum
constexpr size_t kAttOffBar = kAttOffXL + 2 * kAttBQ * 4;
constexpr int kAttSmem = (int)kAttOffBar + 512 + 1024;
static_assert(kAttSmem <= 232448, "shared memory budget");
constexpr uint32_t kAttTmemCols = 256;         // O: 0..127, S buffers: 128..191, 192..255
constexpr float kAttStaleMax = 8.f;            // log2 headroom before a row's O is rescaled
static_assert(4 * kAttPBytes == kAttBQ * kAttHD * 4, "the P region holds one fp32 O tile");

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// The softmax weights as a bf16 pair without conversion instructions: hi keeps
// the upper 16 bits of each fp32 weight (bf16 by truncation), the remainder
// x - hi is exact in fp32, and lo keeps its upper 16 bits.  For 0 <= x the pair
// hi + lo is within 2^-15 x below x (16 significant bits), computed on the
// integer and FMA pipes only; the packed element order matches bf16x2 (x0 low).
__device__ __forceinline__ void split_pair_trunc(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const uint32_t u0 = __float_as_uint(x0), u1 = __float_as_uint(x1);
  hi = __byte_perm(u0, u1, 0x7632);
  const float r0 = x0 - __uint_as_float(u0 & 0xFFFF0000u);
  const float r1 = x1 - __uint_as_float(u1 & 0xFFFF0000u);
  lo = __byte_perm(__float_as_uint(r0), __float_as_uint(r1), 0x7632);
}

// 2^t on the FMA and integer pipes, for a share of the softmax's exponentials
// (the rest go to the MUFU unit's ex2): Cody-Waite style reduction t = n + f with
// n = round(t) (1.5 * 2^23 added and subtracted in fp32) and f in [-1/2, 1/2];
// 2^f by the degree-4 polynomial minimising the relative error on that interval
// (Remez exchange fit; 2.7e-6 maximum in fp32 Horner form, against 2^-15 of the
// bf16 pair the weights are stored in); 2^n added to the exponent field.
// t < -126 gives 0 (below any weight that matters: weights are <= 2^8 here).
__device__ __forceinline__ float exp2_fma(float t) {
  const float tc = fmaxf(t, -126.0f);
  const float j = tc + 12582912.0f;  // the low mantissa bits of j hold n
  const float f = tc - (j - 12582912.0f);
  float p = 9.5701022e-3f;
  p = fmaf(p, f, 5.5917859e-2f);
  p = fmaf(p, f, 2.4024744e-1f);
  p = fmaf(p, f, 6.9312179e-1f);
  p = fmaf(p, f, 9.9999928e-1f);
  const float r = __int_as_float(__float_as_int(p) + (__float_as_int(j) << 23));
  return t >= -126.0f ? r : 0.0f;
}
// every kAttPolyEvery-th exponential of a thread's chunk row goes to exp2_fma (0: none).  With
// the MUFU path a bare ex2 instruction (exp2_mufu) the FMA share no longer pays: at 1024 keys
// the kernel took 21.4 us with every 4th exponential on the FMA pipe, 20.8 with every 8th and
// 20.5 with none (52.3 against 54.8 us at 8192 keys).
constexpr int kAttPolyEvery = 0;
// 2^t by the MUFU unit's approximate ex2 alone (PTX ex2.approx.ftz.f32: relative error about
// 2^-22, subnormal results flushed to 0), for the softmax weights: they are stored with ~16
// significant bits and weights below 2^-126 do not matter.
__device__ __forceinline__ float exp2_mufu(float t) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(t));
  return r;
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
// Bulk copy of `bytes` (multiple of 16) from this CTA's shared memory to another CTA's of
// the cluster, completing the bytes on an mbarrier of that CTA (shared::cluster addresses).
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t mbar) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "r"(src), "r"(bytes), "r"(mbar)
               : "memory");
}
__device__ __forceinline__ void st_dsmem_v4(uint32_t addr, float4 v) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_dsmem_v2(uint32_t addr, float2 v) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(v.x), "f"(v.y) : "memory");
}
}  // namespace

// Work units: (128-query tile of one sequence, head).  Computed on the device
// from seg_ptr (no host synchronisation).
__device__ __forceinline__ int attn_units(const int32_t* seg_ptr, int B, int H) {
  int qt = 0;
  for (int b = 0; b < B; ++b) qt += ceil_div(seg_ptr[b + 1] - seg_ptr[b], kAttBQ);
  return qt * H;
}
struct AttnUnit {
  int b, h, r0, nrows;
};
__device__ __forceinline__ AttnUnit attn_unit(int u, const int32_t* seg_ptr, int B, int H) {
  AttnUnit it;
  it.h = u % H;
  int qi = u / H, b = 0;
  for (; b < B; ++b) {
    const int qt = ceil_div(seg_ptr[b + 1] - seg_ptr[b], kAttBQ);
    if (qi < qt) break;
    qi -= qt;
  }
  it.b = b;
  it.r0 = seg_ptr[b] + qi * kAttBQ;
  it.nrows = min(kAttBQ, seg_ptr[b + 1] - it.r0);
  return it;
}

// The grid is clusters of two CTAs.  When every unit fits on a CTA pair at once
// (2 x units <= CTAs) the two CTAs of a cluster split the unit's keys in halves
// and the odd CTA hands its partial (O, max, sum) to the even one through
// distributed shared memory; otherwise every CTA takes whole units on its own.
// When the units leave more than half of the pairs idle, each unit's keys are
// further cut into `parts` ranges, one pair each: the even CTA of every pair
// stores its merged partial in global scratch, and the pair that finishes a
// unit last (a device-scope counter per unit) merges the parts and writes the
// output.  The work items are then (unit, part) pairs, part fastest.
constexpr int kAttMaxParts = 4;
struct AttnPlan {
  int split;   // 1 or 2
  int parts;   // key ranges per unit, one CTA pair each (1 unless split == 2)
  int first;   // first work item of this CTA
  int stride;  // work-item stride
  int units;   // (tile, head) units
  int items;   // units * parts
};
__device__ __forceinline__ AttnPlan attn_plan(const int32_t* seg_ptr, int B, int H, int N, int part_cap) {
  AttnPlan p;
  p.units = attn_units(seg_ptr, B, H);
  const int nch = ceil_div(N, kAttBK);
  p.split = (2 * p.units <= (int)gridDim.x && nch >= 2) ? 2 : 1;
  p.parts = 1;
  if (p.split == 2) {
    const int pairs = (int)gridDim.x >> 1;
    int parts = min(min(pairs / p.units, nch / 2), kAttMaxParts);
    if (p.units > 0) parts = min(parts, part_cap / p.units);  // scratch tiles for the partials
    if (parts >= 2 && p.units <= kAttPartCounters) p.parts = parts;  // units <= CTAs / 4 here
    p.first = blockIdx.x >> 1;
    p.stride = pairs;
  } else {
    p.first = blockIdx.x;
    p.stride = gridDim.x;
  }
  p.items = p.units * p.parts;
  return p;
}
// Key chunks [c0, c1) of work item w for this CTA (rank in its cluster): the
// item's part of the nch chunks, halved between the two CTAs of a split pair.
// Every CTA gets at least one chunk (parts <= nch / 2).
__device__ __forceinline__ void attn_chunks(const AttnPlan& p, int w, int rank, int nch, int& c0, int& c1) {
  const int part = w % p.parts;
  const int p0 = part * nch / p.parts, p1 = (part + 1) * nch / p.parts;
  if (p.split == 2) {
    c0 = p0 + rank * (p1 - p0) / 2;
    c1 = p0 + (rank + 1) * (p1 - p0) / 2;
  } else {
    c0 = p0;
    c1 = p1;
  }
}

__global__ void __launch_bounds__(kAttThreads, 1) attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                               const __grid_constant__ CUtensorMap tmQlo,
                                                               const __grid_constant__ CUtensorMap tmK,
                                                               const __grid_constant__ CUtensorMap tmV,
                                                               __nv_bfloat16* __restrict__ Aout,
                                                               __nv_bfloat16* __restrict__ Aout_lo,
                                                               const int32_t* __restrict__ seg_ptr, int B, int N,
                                                               int H, int d, int kv_group, float scale_log2,
                                                               float* __restrict__ opart, int* __restrict__ part_cnt,
                                                               int part_cap) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);  // same offset in both CTAs
  uint8_t* sQ = smem;                  // q_hi tile; the q_lo tile follows at + kAttQBytes
  uint8_t* sK = smem + kAttOffK;
  uint8_t* sV = smem + kAttOffV;
  uint8_t* sP = smem + kAttOffP;  // buffer x: high part at 2x, low part at 2x + 1 (16 KB each)
  float* xmax = reinterpret_cast<float*>(smem + kAttOffXM);  // [chunk parity][half][row]
  float* xl = reinterpret_cast<float*>(smem + kAttOffXL);    // [half][row]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kAttOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_free = bars + 1;
  uint64_t* k_full = bars + 2;    // [kAttKStages <= 3]
  uint64_t* k_empty = bars + 5;   // [kAttKStages <= 3]
  uint64_t* v_full = bars + 8;    // [kAttVStages <= 3]
  uint64_t* v_empty = bars + 11;  // [kAttVStages <= 3]
  uint64_t* s_full = bars + 14;   // [2] scores of a chunk in TMEM
  uint64_t* s_free = bars + 16;   // [2] scores read by the 8 softmax warps
  uint64_t* p_full = bars + 18;   // [2] P of a chunk in shared memory (8 softmax warps)
  uint64_t* p_free = bars + 20;   // [2] the P V that read P buffer x has completed
  uint64_t* o_free = bars + 22;   // O read out by the 8 softmax warps
  uint64_t* drain = bars + 23;
  uint64_t* xo_full = bars + 24;  // even CTA: the odd CTA's partial is in my P region (bulk copy bytes)
  uint64_t* xo_free = bars + 25;  // odd CTA: the even CTA's P region is free and armed for my partial
  uint64_t* xmb = bars + 26;      // [4 quarters][2] row-max exchange of the two warps of a quarter
  uint64_t* xlb = bars + 34;      // [4 quarters] row-sum exchange
  uint64_t* xo_done = bars + 38;  // odd CTA: my bulk copies to the even CTA have landed (source free)
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 39);
  volatile int* s_abort = reinterpret_cast<volatile int*>(bars + 40);
  uint64_t* part_written = bars + 41;  // parts > 1: the 8 softmax warps stored this CTA's partial
  uint64_t* part_decided = bars + 42;  // parts > 1: warp 2 took the unit's counter (s_last is set)
  volatile int* s_last = reinterpret_cast<volatile int*>(bars + 43);
  uint64_t* sm_bar = bars + 44;        // the 8 softmax warps meet (one arrival per warp)

  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = (int)cluster_ctarank();
  const AttnPlan plan = attn_plan(seg_ptr, B, H, N, part_cap);
  const int nch = ceil_div(N, kAttBK);
  // the two CTAs of a cluster see the same plan; with a split they also see the same items
  if (plan.first >= plan.items) return;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_free, 1);
    for (int i = 0; i < kAttKStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < kAttVStages; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], kAttSoftWarps);
      mbar_init(&p_full[i], kAttSoftWarps);
      mbar_init(&p_free[i], 1);
    }
    mbar_init(o_free, kAttSoftWarps);
    mbar_init(drain, 1);
    mbar_init(xo_full, 1);
    mbar_init(xo_free, 1);
    for (int i = 0; i < 8; ++i) mbar_init(&xmb[i], 2);
    for (int i = 0; i < 4; ++i) mbar_init(&xlb[i], 2);
    mbar_init(xo_done, 1);
    mbar_init(sm_bar, kAttSoftWarps);
    mbar_init(part_written, kAttSoftWarps);
    mbar_init(part_decided, 1);
    *s_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmQlo);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kAttTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  if (plan.split == 2)
    cluster_sync_all();  // the partner's exchange barriers are initialised
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      long long g = 0;  // chunk counter over this CTA's units
      int t = 0;        // unit counter
      for (int w = plan.first; w < plan.items && !*s_abort; w += plan.stride, ++t) {
        const AttnUnit it = attn_unit(w / plan.parts, seg_ptr, B, H);
        int c0, c1;
        attn_chunks(plan, w, rank, nch, c0, c1);
        const int hc = it.h * kAttHD;                  // query head columns
        const int kc = (it.h / kv_group) * kAttHD;     // its K/V head (grouped-query attention)
        if (!mbar_wait(q_free, (uint32_t)((t & 1) ^ 1))) {
          *s_abort = 1;
          break;
        }
        mbar_expect_tx(q_full, 2 * kAttQBytes);
        tma_load_2d(sQ, &tmQ, hc, it.r0, q_full);
        tma_load_2d(sQ + kAttQBytes / 2, &tmQ, hc + 64, it.r0, q_full);
        tma_load_2d(sQ + kAttQBytes, &tmQlo, hc, it.r0, q_full);
        tma_load_2d(sQ + kAttQBytes + kAttQBytes / 2, &tmQlo, hc + 64, it.r0, q_full);
        for (int c = c0; c < c1; ++c, ++g) {
          const int st = (int)(g % kAttKStages);
          const uint32_t ph = (uint32_t)((g / kAttKStages) & 1);
          const int y = it.b * N + c * kAttBK;
          if (!mbar_wait(&k_empty[st], ph ^ 1)) {
            *s_abort = 1;
            break;
          }
          mbar_expect_tx(&k_full[st], kAttKVBytes);
          tma_load_2d(sK + st * kAttKVBytes, &tmK, kc, y, &k_full[st]);
          tma_load_2d(sK + st * kAttKVBytes + kAttKVBytes / 2, &tmK, kc + 64, y, &k_full[st]);
        }
      }
    }
    __syncwarp();
  } else if (warp == kAttVWarp) {
    // ------------------------------------------------------------ V producer
    if (elect_one()) {
      long long g = 0;
      for (int w = plan.first; w < plan.items && !*s_abort; w += plan.stride) {
        const AttnUnit it = attn_unit(w / plan.parts, seg_ptr, B, H);
        int c0, c1;
        attn_chunks(plan, w, rank, nch, c0, c1);
        const int kc = (it.h / kv_group) * kAttHD;
        for (int c = c0; c < c1; ++c, ++g) {
          const int st = (int)(g % kAttVStages);
          const uint32_t ph = (uint32_t)((g / kAttVStages) & 1);
          const int y = it.b * N + c * kAttBK;
          if (!mbar_wait(&v_empty[st], ph ^ 1)) {
            *s_abort = 1;
            break;
          }
          mbar_expect_tx(&v_full[st], kAttKVBytes);
          tma_load_2d(sV + st * kAttKVBytes, &tmV, kc, y, &v_full[st]);
          tma_load_2d(sV + st * kAttKVBytes + kAttKVBytes / 2, &tmV, kc + 64, y, &v_full[st]);
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
      // O += P_hi V + P_lo V for global chunk gj (first: the unit's first chunk overwrites O)
      auto issue_pv = [&](long long gj, bool first) -> bool {
        const int pb = (int)(gj & 1), st = (int)(gj % kAttVStages);
        if (first && !mbar_wait(o_free, (uint32_t)((t & 1) ^ 1))) return false;  // last unit's O read
        if (!mbar_wait(&p_full[pb], (uint32_t)((gj >> 1) & 1))) return false;
        if (!mbar_wait(&v_full[st], (uint32_t)((gj / kAttVStages) & 1))) return false;
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
      for (int w = plan.first; w < plan.items && !*s_abort; w += plan.stride, ++t) {
        int c0, c1;
        attn_chunks(plan, w, rank, nch, c0, c1);
        const int n = c1 - c0;
        bool ok = mbar_wait(q_full, (uint32_t)(t & 1));
        tc_fence_after();
        for (int j = 0; j < n && ok; ++j) {
          const long long gj = g + j;
          const int sb = (int)(gj & 1), st = (int)(gj % kAttKStages);
          ok = mbar_wait(&s_free[sb], (uint32_t)(((gj >> 1) & 1) ^ 1)) &&
               mbar_wait(&k_full[st], (uint32_t)((gj / kAttKStages) & 1));
          if (!ok) break;
          tc_fence_after();
          const uint32_t kb = smem_u32(sK + st * kAttKVBytes);
#pragma unroll
          for (int k = 0; k < kAttHD / 16; ++k) {  // 16 dims per step: box k / 4, +32 B within it
            const uint32_t qa = q0 + (k >> 2) * (kAttQBytes / 2), ka = kb + (k >> 2) * (kAttKVBytes / 2);
            const uint64_t kdesc = sdesc_sw128(ka) + 2 * (k & 3);
            umma_bf16(tmem_base + 128 + sb * 64, sdesc_sw128(qa) + 2 * (k & 3), kdesc, idesc_s, k > 0 ? 1u : 0u);
            umma_bf16(tmem_base + 128 + sb * 64, sdesc_sw128(qa + kAttQBytes) + 2 * (k & 3), kdesc, idesc_s, 1u);
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
    // ------------------------------------------------------------ softmax: half a query row per thread
    const int q = warp & 3;              // a warp reads TMEM lanes 32 * (warp % 4) ..
    const int hf = (warp - 2) >> 2;      // warps 2-5 take keys 0-31 of a chunk (O dims 0-63), 6-9 the rest
    const int row = q * 32 + lane;
    const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);
    // the two warps sharing these rows exchange through shared memory; lane 0 of each arrives
    // on an mbarrier (count 2) after the warp's writes, and both warps wait on it (bounded)
    auto pair_exchange = [&](uint64_t* bar, uint32_t parity) -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
      return mbar_wait(bar, parity);
    };
    float* ml = reinterpret_cast<float*>(smem + kAttOffML);
    long long g = 0;
    int t = 0;
    bool ok = true;
    // the 8 softmax warps meet: lane 0 of each arrives, every lane waits (bounded)
    uint32_t sm_phase = 0;
    auto soft_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(sm_bar);
      const bool r = mbar_wait(sm_bar, sm_phase);
      sm_phase ^= 1u;
      return r;
    };
    // waits until the P V of global chunk k (and every MMA before it) has completed; k's
    // buffer cannot have moved on, its next P V needs P of chunk k + 2 from these warps
    auto wait_pv = [&](long long k) -> bool {
      return k < 0 || mbar_wait(&p_free[k & 1], (uint32_t)((k >> 1) & 1));
    };
    for (int w = plan.first; w < plan.items && ok; w += plan.stride, ++t) {
      const int u = w / plan.parts;
      const AttnUnit it = attn_unit(u, seg_ptr, B, H);
      int c0, c1;
      attn_chunks(plan, w, rank, nch, c0, c1);
      const int n = c1 - c0;
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
        uint32_t ra[32];
        tmem_ld32(lane_base + 128 + sb * 64 + hf * 32, ra);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[sb]);
        float sc[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) sc[e] = __uint_as_float(ra[e]);
        const int key0 = (c0 + j) * kAttBK + hf * 32;
        if (key0 + 32 > N) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (key0 + e >= N) sc[e] = -INFINITY;
        }
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < 32; ++e) mx = fmaxf(mx, sc[e]);
        // the row max over both halves (double-buffered by chunk parity)
        float* xm = xmax + (size_t)(gj & 1) * 2 * kAttBQ;
        xm[hf * kAttBQ + row] = mx;
        ok = pair_exchange(&xmb[q * 2 + (int)(gj & 1)], (uint32_t)((gj >> 1) & 1));
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        mx = fmaxf(mx, xm[(1 - hf) * kAttBQ + row]);
        const float mc = mx * scale_log2;  // every chunk holds at least one key < N
        const bool need = mc > m_used + kAttStaleMax;  // identical in both halves of the row
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
          for (int cb = 0; cb < 2; ++cb) {
            uint32_t o[32];
            tmem_ld32(lane_base + hf * 64 + cb * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
            tmem_st32(lane_base + hf * 64 + cb * 32, o);
          }
          tmem_st_wait();
        }
        l *= factor;
        ok = wait_pv(gj - 2);  // the P V that read P buffer sb has completed
        // odd CTA with a split: the last unit's partial, staged in the P region, has been copied out
        if (plan.split == 2 && rank == 1 && j == 0 && t > 0) ok = ok && mbar_wait_cluster(xo_done, (uint32_t)((t - 1) & 1));
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        // P = 2^(s * scale - m_used) <= 2^8, as bf16 high + low parts, K-major with 128-byte swizzle
        uint8_t* ph = sP + (2 * sb) * kAttPBytes;
        uint8_t* pl = ph + kAttPBytes;
        const uint32_t rowoff = (uint32_t)((row >> 3) * 1024 + (row & 7) * 128);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i0 = cc * 8 + 2 * e, i1 = i0 + 1;
            const float t0 = fmaf(sc[i0], scale_log2, -m_used), t1 = fmaf(sc[i1], scale_log2, -m_used);
            const bool f0 = kAttPolyEvery > 0 && i0 % (kAttPolyEvery > 0 ? kAttPolyEvery : 1) == kAttPolyEvery - 1;
            const bool f1 = kAttPolyEvery > 0 && i1 % (kAttPolyEvery > 0 ? kAttPolyEvery : 1) == kAttPolyEvery - 1;
            const float p0 = f0 ? exp2_fma(t0) : exp2_mufu(t0);
            const float p1 = f1 ? exp2_fma(t1) : exp2_mufu(t1);
            l += p0 + p1;
            split_pair_trunc(p0, p1, hi[e], lo[e]);
          }
          const uint32_t off = rowoff + ((uint32_t)((hf * 4 + cc) ^ (row & 7)) << 4);
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
      xl[hf * kAttBQ + row] = l;
      ok = pair_exchange(&xlb[q], (uint32_t)(t & 1));
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      const float l_row = xl[row] + xl[kAttBQ + row];
      float o[64];
#pragma unroll
      for (int cb = 0; cb < 2; ++cb) {
        uint32_t r[32];
        tmem_ld32(lane_base + hf * 64 + cb * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) o[cb * 32 + e] = __uint_as_float(r[e]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);
      if (plan.split == 2 && rank == 1) {
        // hand (O, max, sum) of my key half to the even CTA: stage it in my own P region (free:
        // every P V of this unit has completed), row r's 32 16-byte slots at r * 32 + (c ^ (r & 7))
        // so that a warp's 32 rows cover every bank, then one thread moves the 64 KB (and the
        // 1 KB of (max, sum)) into the even CTA's P region with bulk copies that complete on its
        // xo_full barrier
        float4* xs = reinterpret_cast<float4*>(sP);
#pragma unroll
        for (int v = 0; v < 16; ++v)
          xs[row * 32 + ((hf * 16 + v) ^ (row & 7))] = make_float4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
        if (hf == 0) reinterpret_cast<float2*>(ml)[row] = make_float2(m_used, l_row);
        fence_proxy_async_smem();  // the bulk copy reads these through the async proxy
        ok = soft_sync();
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        if (warp == 2 && lane == 0) {
          if (mbar_wait_cluster(xo_free, (uint32_t)(t & 1))) {  // its P region is free, the bytes expected
            const uint32_t full_r = dsmem_addr(smem_u32(xo_full), 0);
            bulk_copy_to_peer(dsmem_addr(smem_u32(sP), 0), smem_u32(sP), kAttBQ * kAttHD * 4, full_r);
            bulk_copy_to_peer(dsmem_addr(smem_u32(ml), 0), smem_u32(ml), kAttBQ * 8, full_r);
          } else {
            *s_abort = 1;
          }
        }
      } else {
        float m_row = m_used, l_tot = l_row;
        if (plan.split == 2) {
          // my P region is free once every softmax warp is here (every P V of this unit has
          // completed): one thread arms xo_full for the odd CTA's 64 KB + 1 KB and lets it send
          ok = soft_sync();
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
          if (warp == 2 && lane == 0) {
            mbar_expect_tx(xo_full, kAttBQ * kAttHD * 4 + kAttBQ * 8);
            mbar_arrive_remote(dsmem_addr(smem_u32(xo_free), 1));
          }
          ok = mbar_wait(xo_full, (uint32_t)(t & 1));
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
          // the copies have landed, so they have read their source: the odd CTA may reuse its P region
          if (warp == 2 && lane == 0) mbar_arrive_remote(dsmem_addr(smem_u32(xo_done), 1));
          const float2 pm = reinterpret_cast<const float2*>(ml)[row];  // odd CTA's (max, sum)
          const float m = fmaxf(m_used, pm.x);
          const float w_own = exp2f(m_used - m);
          const float w_odd = exp2f(pm.x - m);
          m_row = m;
          l_tot = w_own * l_row + w_odd * pm.y;
          const float4* xo = reinterpret_cast<const float4*>(sP);
#pragma unroll
          for (int v = 0; v < 16; ++v) {
            const float4 x = xo[row * 32 + ((hf * 16 + v) ^ (row & 7))];
            o[4 * v] = fmaf(w_own, o[4 * v], w_odd * x.x);
            o[4 * v + 1] = fmaf(w_own, o[4 * v + 1], w_odd * x.y);
            o[4 * v + 2] = fmaf(w_own, o[4 * v + 2], w_odd * x.z);
            o[4 * v + 3] = fmaf(w_own, o[4 * v + 3], w_odd * x.w);
          }
        }
        float inv = 1.0f / l_tot;
        bool write_out = true;
        if (plan.parts > 1) {
          // this pair's key range is one part of the unit: store (O, max, sum), unnormalised,
          // and let the pair that completes the unit last merge the parts
          // column-major partial tiles ([item][column][row]): a warp's store of one column is
          // 32 consecutive rows, 128 contiguous bytes
          float2* mlp = reinterpret_cast<float2*>(opart + (size_t)part_cap * kAttBQ * kAttHD);
          float* op = opart + ((size_t)w * kAttHD + hf * 64) * kAttBQ + row;
#pragma unroll
          for (int e = 0; e < 64; ++e) op[(size_t)e * kAttBQ] = o[e];
          if (hf == 0) mlp[(size_t)w * kAttBQ + row] = make_float2(m_row, l_tot);
          __threadfence();
          __syncwarp();
          if (lane == 0) mbar_arrive(part_written);
          if (warp == 2) {
            int okd = 1;
            if (lane == 0) {
              okd = mbar_wait(part_written, (uint32_t)(t & 1)) ? 1 : 0;
              int last = 0;
              if (okd) {
                __threadfence();
                last = atomicAdd(part_cnt + u, 1) == plan.parts - 1 ? 1 : 0;
              }
              *s_last = last;
              mbar_arrive(part_decided);
            }
            ok = ok && __shfl_sync(0xffffffffu, okd, 0) != 0;
          }
          ok = ok && mbar_wait(part_decided, (uint32_t)(t & 1));
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
          write_out = *s_last != 0;
          if (write_out) {
            __threadfence();
            const size_t w0 = (size_t)u * plan.parts;
            float mm = -INFINITY;
            for (int q2 = 0; q2 < plan.parts; ++q2) mm = fmaxf(mm, __ldcg(&mlp[(w0 + q2) * kAttBQ + row]).x);
            float lt = 0.f;
#pragma unroll
            for (int e = 0; e < 64; ++e) o[e] = 0.f;
            for (int q2 = 0; q2 < plan.parts; ++q2) {
              const float2 pq = __ldcg(&mlp[(w0 + q2) * kAttBQ + row]);
              const float wq = exp2f(pq.x - mm);
              lt = fmaf(wq, pq.y, lt);
              const float* src = opart + ((w0 + q2) * kAttHD + hf * 64) * kAttBQ + row;
#pragma unroll
              for (int e = 0; e < 64; ++e) o[e] = fmaf(wq, __ldcg(src + (size_t)e * kAttBQ), o[e]);
            }
            inv = 1.0f / lt;
            if (warp == 2 && lane == 0) part_cnt[u] = 0;  // every part has counted: reset for the next launch
          }
        }
        if (write_out) {
          // the normalised tile as hi/lo bf16 pairs, staged in the P region (rows of 16 16-byte
          // chunks, chunk c of row r at r * 16 + (c ^ (r & 7)): conflict-free both ways) and
          // stored two rows per warp instruction, each row 256 contiguous bytes of hi and of lo
          ok = soft_sync();  // every warp is done with the P region (and the odd CTA's partial in it)
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
          uint4* sh = reinterpret_cast<uint4*>(sP);
          uint4* sl = reinterpret_cast<uint4*>(sP + kAttBQ * kAttHD * 2);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) split_pair(o[8 * v + 2 * e] * inv, o[8 * v + 2 * e + 1] * inv, hi[e], lo[e]);
            const int slot = row * 16 + ((hf * 8 + v) ^ (row & 7));
            sh[slot] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            sl[slot] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
          }
          ok = soft_sync();
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
          const int sw = warp - 2, ch = lane & 15;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = sw * 16 + 2 * i + (lane >> 4);
            if (r < it.nrows) {
              const size_t off = (size_t)(it.r0 + r) * d + it.h * kAttHD + ch * 8;
              const int slot = r * 16 + (ch ^ (r & 7));
              *reinterpret_cast<uint4*>(Aout + off) = sh[slot];
              *reinterpret_cast<uint4*>(Aout_lo + off) = sl[slot];
            }
          }
          ok = soft_sync();  // the P region may take the next unit's weights
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
        }
      }
      g += n;
    }
    if (!ok && lane == 0) *s_abort = 1;
  }

  tc_fence_before();
  if (plan.split == 2)
    cluster_sync_all();  // no CTA leaves while its partner may still touch its shared memory
  else
    __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kAttTmemCols);
  }
}

template <int HD>
__global__ void attn_f32_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                                const float* __restrict__ V, float* __restrict__ A,
                                const int32_t* __restrict__ seg_ptr, int B, int N, int d, int H, int dkv,
                                int kv_group, float scale) {
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
    const float* kr = K + ((size_t)b * N + n) * dkv + (h / kv_group) * HD;
    const float* vr = V + ((size_t)b * N + n) * dkv + (h / kv_group) * HD;
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

int launch_attention_bf16(const plk_dims* dims, const void* q, const void* q_lo, const void* K_cache,
                          const void* V_cache, void* a_out, void* a_lo, const int32_t* seg_ptr, int num_sms,
                          float* part_scratch, size_t part_bytes, int* part_cnt, cudaStream_t st) {
  const int B = dims->B, N = dims->N, d = dims->d, H = dims->H, dkv = kv_width(dims);
  CUtensorMap tmQ, tmQlo, tmK, tmV;
  if (make_tmap_bf16(&tmQ, q, (uint64_t)B * N, (uint64_t)d, kAttBQ) != PLK_OK) return PLK_ERR_CUDA;
  if (make_tmap_bf16(&tmQlo, q_lo, (uint64_t)B * N, (uint64_t)d, kAttBQ) != PLK_OK) return PLK_ERR_CUDA;
  if (make_tmap_bf16(&tmK, K_cache, (uint64_t)B * N, (uint64_t)dkv, kAttBK) != PLK_OK) return PLK_ERR_CUDA;
  if (make_tmap_bf16(&tmV, V_cache, (uint64_t)B * N, (uint64_t)dkv, kAttBK) != PLK_OK) return PLK_ERR_CUDA;
  static int attr_done[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PLK_ERR_CUDA;
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttSmem) != cudaSuccess)
      return PLK_ERR_CUDA;
    attr_done[dev] = 1;
  }
  const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)dims->hd));
  // persistent clusters of two CTAs, one CTA per SM, over the (query tile, head) units
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(num_sms & ~1));
  cfg.blockDim = dim3(kAttThreads);
  cfg.dynamicSmemBytes = kAttSmem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  // partial tiles (128 x 128 fp32) and their (max, sum) rows that fit in the scratch
  const size_t tile_bytes = (size_t)kAttBQ * kAttHD * 4 + (size_t)kAttBQ * 8;
  const int part_cap = part_scratch ? (int)std::min(part_bytes / tile_bytes, (size_t)1 << 20) : 0;
  if (cudaLaunchKernelEx(&cfg, attn_tc_kernel, tmQ, tmQlo, tmK, tmV, (__nv_bfloat16*)a_out, (__nv_bfloat16*)a_lo,
                         seg_ptr, B, N, H, d,
                         H / kv_heads(dims), scale_log2, part_scratch, part_cnt, part_cap) != cudaSuccess)
    return PLK_ERR_CUDA;
  return PLK_OK;
}

__global__ void exp2_selftest_kernel(const float* __restrict__ t, float* __restrict__ out, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) out[i] = exp2_fma(t[i]);
}

int launch_exp2_selftest(const float* t, float* out, int n, cudaStream_t st) {
  exp2_selftest_kernel<<<std::min(ceil_div(std::max(n, 1), 256), 1024), 256, 0, st>>>(t, out, n);
  return cudaPeekAtLastError() == cudaSuccess ? PLK_OK : PLK_ERR_CUDA;
}

int launch_attention_f32(const plk_dims* dims, const float* q, const float* K_cache, const float* V_cache,
                         float* a_out, const int32_t* seg_ptr, int Mcap, cudaStream_t st) {
  const int B = dims->B, N = dims->N, d = dims->d, H = dims->H, hd = dims->hd;
  const int dkv = kv_width(dims), g = H / kv_heads(dims);
  const float scale = (float)(1.0 / sqrt((double)hd));
  const int threads = 128, blocks = ceil_div(Mcap * H, threads);
  switch (hd) {
    case 16:
      attn_f32_kernel<16><<<blocks, threads, 0, st>>>(q, K_cache, V_cache, a_out, seg_ptr, B, N, d, H, dkv, g, scale);
      break;
    case 32:
      attn_f32_kernel<32><<<blocks, threads, 0, st>>>(q, K_cache, V_cache, a_out, seg_ptr, B, N, d, H, dkv, g, scale);
      break;
    case 64:
      attn_f32_kernel<64><<<blocks, threads, 0, st>>>(q, K_cache, V_cache, a_out, seg_ptr, B, N, d, H, dkv, g, scale);
      break;
    case 128:
      attn_f32_kernel<128><<<blocks, threads, 0, st>>>(q, K_cache, V_cache, a_out, seg_ptr, B, N, d, H, dkv, g, scale);
      break;
    default: return PLK_ERR_SHAPE;
  }
  return cudaPeekAtLastError() == cudaSuccess ? PLK_OK : PLK_ERR_CUDA;
}

}  // namespace plk
