// tcgen05 GEMM for the projections of the partial-recompute layer step:
// out[token, f] += sum_k X[token, k] * W[f, k] on the M active rows only (the
// SureLock page, "Stopping Computation for Converged Tokens in Masked
// Diffusion-LM Decoding", Sec. 2: Q/K/V, output projection and FFN run for the
// active subset, cost O(M d^2)).
//
// Design (sm_100a):
//  * CTA pairs (cta_group::2): the even CTA issues one tcgen05.mma of
//    M = 256 feature rows x N = 128 or 256 tokens that runs on the tensor cores
//    of both SMs.  Each CTA stages its own 128 weight rows and HALF of the
//    token tile, so an SM ingests 16 KB of weights and 32 KB of activations
//    (hi and lo, below) per 64-deep k-block instead of 16 + 64 KB for a one-CTA
//    128 x 256 tile.  Accumulation is fp32 in TMEM; each CTA's TMEM holds its
//    128 rows x N columns.
//  * Weights are the A operand and the compacted activations the B operand;
//    at M <= 256 every weight byte is read from HBM once.  The activation comes
//    as a bf16 pair, X = Xhi + Xlo (Xlo = bf16(X - Xhi)), so that it enters the
//    product with ~16 significant bits: every k-block stages one weight tile and
//    both activation tiles, and the pair MMA runs W Xhi^T and W Xlo^T into the
//    same fp32 accumulator.  All tiles are K-major bf16, loaded by TMA with a
//    128-byte swizzle into a 4-stage ring of 48 KB stages.
//  * Warp roles: warp 0 issues TMA in both CTAs, every load counting its bytes
//    on the even CTA's stage barrier; one thread of warp 1 of the even CTA
//    issues the pair MMAs; warps 2-5 of both CTAs drain their TMEM.
//  * Persistent stream-K: each pair owns an equal, contiguous share of the
//    (256-feature tile) x (k-block) iteration space.  A tile piece
//    accumulates its whole k range in TMEM, then goes into the fp32 output by
//    TMA bulk store or bulk reduce-add (cp.reduce.async.bulk.tensor .add.f32,
//    applied in the L2).  The output is the residual stream h (O and down
//    projections: every piece adds, in the order the pieces arrive, so h may
//    differ in the last fp32 bit between runs) or an fp32 sums buffer that a
//    finishing kernel turns into bf16 (QKV -> Q and the K/V cache rows;
//    gate/up -> silu(g) u), which is not zeroed: the piece of the last k range
//    stores.  Into a sums buffer the pieces of a split tile land in a fixed
//    order, last k range first (it is its pair's first piece, done early):
//    each later piece waits (bounded) until the pieces of higher k have
//    landed, a count per (tile, CTA, warp) that every piece but the first-k
//    one raises once its bulk operation is complete.  A waiting pair waits
//    only on pairs of higher index whose piece is their first, so no wait
//    closes a cycle, and the sums are the same in every run.  (For the O and
//    down projections, 16 tiles split 5-6 ways at 256 rows, such a chain
//    costs ~18 us per launch.)
//  * Two 256-column TMEM accumulators per CTA: the epilogue drains one tile
//    piece while the MMA fills the next; the producers run ahead across
//    pieces.
//  * Each epilogue warp stages its 32 tokens x 32 features token-major in a
//    double-buffered shared-memory block (rows past M zeroed) and issues one
//    bulk reduce per block; the CTA's last piece stages all its blocks in the
//    then idle operand ring so that every reduce is in flight at once.  A
//    gate/up tile of a CTA (64 gate + 64 up rows of the same features) lands
//    in the gate and up halves of its [M, 2F] buffer.
#include "plk_common.cuh"
#include "plk_internal.h"

namespace plk {

namespace {

constexpr int kHalfTok = kGemmBNMax / 2;            // token rows of B staged per CTA
constexpr int kStageA = kGemmBM * kGemmBK * 2;      // 16 KB
constexpr int kStageB = kHalfTok * kGemmBK * 2;     // 16 KB (hi part; the lo part the same)
constexpr size_t kOffB = (size_t)kGemmStages * kStageA;
constexpr size_t kOffBlo = kOffB + (size_t)kGemmStages * kStageB;
constexpr size_t kOffBar = kOffBlo + (size_t)kGemmStages * kStageB;
constexpr size_t kOffStg = kOffBar + 256;
constexpr int kBlk = 32 * 32;                       // a warp's block: 32 tokens x 32 features (fp32)
constexpr size_t kSmemUsed = kOffStg + 4 * 2 * kBlk * 4;
constexpr size_t kSmemBytes = kSmemUsed + 1024;     // slack for 1024-byte alignment
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert((size_t)4 * 8 * kBlk * 4 <= kOffBar, "the last piece's blocks fit the operand ring");
// Longest run of k-blocks accumulated in one TMEM chain before its partial is
// added into the fp32 output.  Every chain is one more fp32 read-modify-write
// of its tile (measured over the four projections: chains of 16 k-blocks cost
// 5% at 256 tokens and 15% at 2048 tokens against no limit).  With the
// activations split into hi/lo pairs no bf16 rounding follows a sum before the
// layer's stored outputs, so the small per-step drift of the tensor core's fp32
// accumulation stays small against the bf16 step of K, V and Y: no limit.
constexpr int kGemmChainKB = 1 << 20;

// bulk reduce-add of a [32 rows][32 fp32] smem block into the tensor at (x, y)
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* tm, int x, int y, const void* smem_src,
                                                  uint64_t policy) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group.L2::cache_hint [%0, {%1, %2}], [%3], %4;" ::"l"(
          reinterpret_cast<uint64_t>(tm)),
      "r"(x), "r"(y), "r"(smem_u32(smem_src)), "l"(policy)
      : "memory");
}
// bulk store of a [32 rows][32 fp32] smem block into the tensor at (x, y)
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* tm, int x, int y, const void* smem_src,
                                             uint64_t policy) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%1, %2}], [%3], %4;" ::"l"(
                   reinterpret_cast<uint64_t>(tm)),
               "r"(x), "r"(y), "r"(smem_u32(smem_src)), "l"(policy)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// waits until at most n committed bulk groups still read their shared-memory source
template <int n>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(n) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

}  // namespace

// The flattened iteration space of one GEMM: tiles x KB k-blocks, pair tile
// u = pt * ttiles + tt (token tiles fastest, so pairs that run at the same
// time share a weight tile in L2).  Pair c owns iterations [c*T/G, (c+1)*T/G);
// a segment is the part of that range inside one tile and one aligned run of
// kGemmChainKB k-blocks.
struct SegWalk {
  long long i, iend;
  int KB;
  __device__ SegWalk(int pair, int npairs, int tiles, int KB_) : KB(KB_) {
    const long long T = (long long)tiles * KB_;
    i = T * pair / npairs;
    iend = T * (pair + 1) / npairs;
  }
  __device__ bool next(int& u, int& kb0, int& kb1) {
    if (i >= iend) return false;
    u = (int)(i / KB);
    kb0 = (int)(i - (long long)u * KB);
    kb1 = (int)min((long long)min(KB, (kb0 / kGemmChainKB + 1) * kGemmChainKB), kb0 + (iend - i));
    i += kb1 - kb0;
    return true;
  }
  __device__ bool done() const { return i >= iend; }
};

// Order of the pieces of a split tile.  Pair c owns iterations [start(c), start(c + 1)),
// start(c) = floor(c T / G); iteration x lies in the range of pair floor(((x + 1) G - 1) / T).
// With T > G every range is nonempty and a tile's pieces belong to consecutive pairs; with
// T <= G every nonempty range is one iteration, so every k-block of a tile is a piece.
struct SplitPlan {
  long long T;
  int G, KB;
  __device__ int pair_of(long long x) const { return (int)(((x + 1) * G - 1) / T); }
  // pieces of tile u with a higher k range than the piece of `pair` starting at k-block kb0
  __device__ int rank_from_tail(int u, int pair, int kb0) const {
    if (T <= G) return KB - 1 - kb0;
    return pair_of((long long)u * KB + KB - 1) - pair;
  }
};

// Geometry of pair tile u as seen by CTA `rank` of the pair.
struct TileGeom {
  int ft;     // this CTA's 128-row feature tile (pair tile pt covers 2 pt and 2 pt + 1)
  int tok0;   // first token of the tile
  int ntok;   // valid tokens
  int ncols;  // UMMA N: 128 or 256 (each CTA stages ncols / 2 token rows)
  __device__ TileGeom(int u, int ttiles, int M, int rank) {
    const int pt = u / ttiles;
    ft = 2 * pt + rank;
    tok0 = (u - pt * ttiles) * kGemmBNMax;
    ntok = min(kGemmBNMax, M - tok0);
    ncols = (ntok + 127) & ~127;
  }
};

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                   const __grid_constant__ CUtensorMap tmXlo, const __grid_constant__ CUtensorMap tmOut,
                   const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);  // same offset in both CTAs of a pair
  uint8_t* sA = smem;
  uint8_t* sB = smem + kOffB;
  uint8_t* sBlo = smem + kOffBlo;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* full = bars;                        // [stages] stage landed, both halves (even CTA's used)
  uint64_t* empty = bars + kGemmStages;         // [stages] stage consumed by the pair MMA
  uint64_t* tfull = bars + 2 * kGemmStages;     // [2] accumulator ready for the epilogue
  uint64_t* tempty = bars + 2 * kGemmStages + 2;  // [2] accumulator drained (even CTA: 8 warps)
  uint64_t* drain = bars + 2 * kGemmStages + 4;   // MMA completion on the abort path
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2 * kGemmStages + 5);
  volatile int* s_abort = reinterpret_cast<volatile int*>(bars + 2 * kGemmStages + 6);
  float* stg_all = reinterpret_cast<float*>(smem + kOffStg);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = (int)cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  // seg_ptr comes from a kernel before the predecessor: already complete (see pdl_wait)
  const int M = args.seg_ptr[args.B];
  const int ttiles = ceil_div(max(M, 0), kGemmBNMax);
  const int tiles = (args.ftiles >> 1) * ttiles;
  const int KB = args.K / kGemmBK;
  if (M <= 0 || SegWalk(pair, npairs, tiles, KB).done()) {  // the same for both CTAs of the pair
    pdl_wait();
    return;
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGemmStages; ++i) {
      mbar_init(&full[i], 1);  // the even CTA's expect-arrive; both CTAs' loads complete on it
      mbar_init(&empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);  // one arrival per epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmXlo);
    tma_prefetch_desc(&tmOut);
  }
  if (warp == 1) {
    tmem_alloc_pair(s_tmem, 512);  // two 256-column fp32 accumulators in each CTA
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  if (warp != 0) {
    pdl_wait();
    pdl_trigger();
  }

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (elect_one()) {
      // L2 policies: with a single token tile every weight tile is read by one pair only
      // (streamed: evict first) and every pair reads the activations (evict last)
      const uint64_t pol_w = ttiles == 1 ? l2_policy_evict_first() : l2_policy_evict_normal();
      const uint64_t pol_x = ttiles == 1 ? l2_policy_evict_last() : l2_policy_evict_normal();
      // this CTA's 128 weight rows of tile t (gate/up tile: 64 gate rows, then the 64 up rows)
      const uint32_t lead_full0 = dsmem_addr(smem_u32(&full[0]), 0);
      auto load_a = [&](int stage, const TileGeom& t, int kb) {
        const int yA0 = args.gu_F ? t.ft * 64 : t.ft * kGemmBM;
        const int yA1 = args.gu_F ? args.gu_F + t.ft * 64 : t.ft * kGemmBM + 64;
        uint8_t* a = sA + stage * kStageA;
        const uint32_t fb = lead_full0 + (uint32_t)(stage * 8);
        tma_load_2d_pair_hint(a, &tmW, kb * kGemmBK, yA0, fb, pol_w);
        tma_load_2d_pair_hint(a + 8192, &tmW, kb * kGemmBK, yA1, fb, pol_w);
      };
      // bytes of one stage, both CTAs: 2 x (A rows + hi and lo of half of the token rows)
      auto stage_bytes = [](const TileGeom& t) {
        return (uint32_t)(2 * (kStageA + 2 * (t.ncols >> 7) * (64 * kGemmBK * 2)));
      };
      SegWalk w(pair, npairs, tiles, KB);
      int u, kb0, kb1, stage = 0;
      // The weights are no kernel's output: the first stages' weight loads start
      // before the wait for the predecessor, overlapping its tail.
      int pre = 0;
      {
        SegWalk w2 = w;
        while (pre < kGemmStages && w2.next(u, kb0, kb1)) {
          const TileGeom t(u, ttiles, M, rank);
          for (int kb = kb0; kb < kb1 && pre < kGemmStages; ++kb, ++pre) {
            if (rank == 0) mbar_expect_tx(&full[pre], stage_bytes(t));
            load_a(pre, t, kb);
          }
        }
      }
      pdl_wait();
      pdl_trigger();
      uint32_t phase = 0;
      long long issued = 0;
      while (!*s_abort && w.next(u, kb0, kb1)) {
        const TileGeom t(u, ttiles, M, rank);
        const int half = t.ncols >> 1, nbox = half >> 6;
        const int trow = t.tok0 + rank * half;  // this CTA's token rows: MMA columns rank*half ..
        for (int kb = kb0; kb < kb1; ++kb) {
          if (issued >= pre) {  // stages past the prefetched ones: wait for a free slot
            if (!mbar_wait(&empty[stage], phase ^ 1)) {
              *s_abort = 1;
              break;
            }
            if (rank == 0) mbar_expect_tx(&full[stage], stage_bytes(t));
            load_a(stage, t, kb);
          }
          uint8_t* b = sB + stage * kStageB;
          uint8_t* blo = sBlo + stage * kStageB;
          for (int j = 0; j < nbox; ++j) {
            tma_load_2d_pair_hint(b + j * 8192, &tmX, kb * kGemmBK, trow + j * 64,
                                  lead_full0 + (uint32_t)(stage * 8), pol_x);
            tma_load_2d_pair_hint(blo + j * 8192, &tmXlo, kb * kGemmBK, trow + j * 64,
                                  lead_full0 + (uint32_t)(stage * 8), pol_x);
          }
          ++issued;
          if (++stage == kGemmStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*s_abort && rank == 0) {
        // let the pair's copies land before the CTAs move on (bounded; the odd
        // CTA's copies complete on these barriers too)
        for (long long i = issued > kGemmStages ? issued - kGemmStages : 0; i < issued; ++i)
          (void)mbar_wait(&full[i % kGemmStages], (uint32_t)((i / kGemmStages) & 1));
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (rank == 0) {
      // ---------------------------------------------------------- pair MMA issuer (even CTA)
      if (elect_one()) {
        const uint32_t peer_empty0 = dsmem_addr(smem_u32(&empty[0]), 1);
        const uint32_t peer_tfull0 = dsmem_addr(smem_u32(&tfull[0]), 1);
        SegWalk w(pair, npairs, tiles, KB);
        int u, kb0, kb1, stage = 0, j = 0;
        uint32_t phase = 0;
        bool any = false;
        while (!*s_abort && w.next(u, kb0, kb1)) {
          const TileGeom t(u, ttiles, M, rank);
          const int b = j & 1;
          if (!mbar_wait_cluster(&tempty[b], ((j >> 1) & 1) ^ 1)) {  // both epilogues have drained it
            *s_abort = 1;
            break;
          }
          tc_fence_after();
          const uint32_t acc = tmem_base + (uint32_t)(b * 256);
          const uint32_t idesc = idesc_bf16(2 * kGemmBM, t.ncols);
          for (int kb = kb0; kb < kb1; ++kb) {
            if (!mbar_wait(&full[stage], phase)) {  // both CTAs' halves of the stage landed
              *s_abort = 1;
              break;
            }
            tc_fence_after();
            const uint64_t adesc = sdesc_sw128(smem_u32(sA + stage * kStageA));
            const uint64_t bdesc = sdesc_sw128(smem_u32(sB + stage * kStageB));
            const uint64_t bdesc_lo = sdesc_sw128(smem_u32(sBlo + stage * kStageB));
#pragma unroll
            for (int k = 0; k < kGemmBK / 16; ++k) {  // +32 bytes of K per step = 2 descriptor units
              umma_bf16_pair(acc, adesc + 2 * k, bdesc + 2 * k, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
              umma_bf16_pair(acc, adesc + 2 * k, bdesc_lo + 2 * k, idesc, 1u);
            }
            any = true;
            umma_commit_pair(smem_u32(&empty[stage]));  // the stage is free in both CTAs
            umma_commit_pair(peer_empty0 + (uint32_t)(stage * 8));
            if (++stage == kGemmStages) {
              stage = 0;
              phase ^= 1;
            }
          }
          if (*s_abort) break;
          umma_commit_pair(smem_u32(&tfull[b]));  // the accumulators are complete in both CTAs
          umma_commit_pair(peer_tfull0 + (uint32_t)(b * 8));
          ++j;
        }
        if (*s_abort && any) {
          umma_commit_pair(smem_u32(drain));  // wait for the MMAs in flight before TMEM is freed
          (void)mbar_wait(drain, 0);
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;  // a warp reads TMEM lanes 32 * (warp % 4) ..
    const uint32_t lead_tempty0 = rank == 0 ? 0u : dsmem_addr(smem_u32(&tempty[0]), 0);
    // the sums are read again soon (the finishing kernel, the next piece's adds): keep them in L2
    // when the weights stream past them (a single token tile)
    const uint64_t pol_out = ttiles == 1 ? l2_policy_evict_last() : l2_policy_evict_normal();
    const SplitPlan plan{(long long)tiles * KB, npairs, KB};
    SegWalk w(pair, npairs, tiles, KB);
    int u, kb0, kb1, j = 0, n = 0;
    while (w.next(u, kb0, kb1)) {
      const bool last = w.done();  // no MMA or TMA follows: the stage buffers are free for staging
      const TileGeom t(u, ttiles, M, rank);
      const int b = j & 1;
      const bool ok = mbar_wait(&tfull[b], (j >> 1) & 1) && !*s_abort;
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) *s_abort = 1;
        break;
      }
      tc_fence_after();
      // output column of this warp's 32 features (gate/up tile: lanes 0-63 gate, 64-127 up)
      const int col = args.gu_F ? (q < 2 ? t.ft * 64 + q * 32 : args.gu_F + t.ft * 64 + (q - 2) * 32)
                                : t.ft * kGemmBM + q * 32;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * 256);
      const int nchunks = t.ncols >> 5;
      // The pieces of a split tile go into the output one after another in a fixed order, from
      // the last k range (the tail, which is its pair's first piece and is done early) down to
      // the first: the tail stores (an output that starts undefined) or adds, every other piece
      // waits until the rho pieces of higher k have landed (a per-(tile, CTA, warp) count of the
      // pieces done), then adds.  The fp32 sums therefore come out the same in every run.  A
      // whole tile is one piece.
      const int rho = plan.rank_from_tail(u, pair, kb0);
      const bool store = args.store_first && kb1 == KB;
      uint32_t* done = (args.done && kb0 > 0) ? args.done + ((2 * u + rank) * 4 + q) : nullptr;  // not the head
      if (args.done && rho > 0) {
        bool got = true;
        if (lane == 0) {
          got = spin_until_geq(args.done + ((2 * u + rank) * 4 + q), (uint32_t)rho);  // bounded; see above
          fence_proxy_async_global();  // the landed pieces before this warp's bulk adds
        }
        if (__shfl_sync(0xffffffffu, got ? 1 : 0, 0) == 0 && lane == 0) *s_abort = 1;
      }
      for (int c = 0; c < nchunks; ++c) {
        float* blk;
        if (last) {
          blk = reinterpret_cast<float*>(smem) + (q * 8 + c) * kBlk;  // 4 warps x 8 chunks x 4 KB
        } else {
          blk = stg_all + (q * 2 + (n & 1)) * kBlk;
          if (n >= 2) {
            if (lane == 0) bulk_wait_read<1>();  // the reduce that used this buffer has read it
            __syncwarp();
          }
          ++n;
        }
        uint32_t r[32];
        tmem_ld32(taddr + (uint32_t)(c * 32), r);
        tmem_ld_wait();
        if (c == nchunks - 1) {  // accumulator b drained: the pair MMA may reuse it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (rank == 0)
              mbar_arrive(&tempty[b]);
            else
              mbar_arrive_remote(lead_tempty0 + (uint32_t)(b * 8));
          }
        }
        const int nval = t.ntok - c * 32;  // tokens past M contribute zeros
#pragma unroll
        for (int i = 0; i < 32; ++i) blk[i * 32 + lane] = i < nval ? __uint_as_float(r[i]) : 0.f;
        fence_proxy_async_smem();  // make the block visible to the bulk-copy unit
        __syncwarp();
        if (lane == 0) {
          if (store)
            tma_store_2d(&tmOut, col, t.tok0 + c * 32, blk, pol_out);
          else
            tma_reduce_add_2d(&tmOut, col, t.tok0 + c * 32, blk, pol_out);
          bulk_commit();
        }
      }
      if (done) {  // every piece but the head: landed, the next lower k range may add
        if (lane == 0) {
          bulk_wait_all();
          fence_proxy_async_global();
          red_release_add_u32(done, 1u);
        }
        __syncwarp();
      }
      ++j;
    }
    if (lane == 0) bulk_wait_all();  // sources read and adds complete before the CTA ends
    __syncwarp();
  }

  // Neither CTA may leave while the pair MMA can still read its shared memory
  // or the other CTA can still arrive on its barriers.
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

// Pairs that can be resident at once (cluster of 2, one CTA per SM), per device.
static int resident_pairs(int num_sms) {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms & ~1);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel, &cfg) != cudaSuccess || n <= 0) return 0;
  n = std::min(n, num_sms / 2);
  if (dev < 64) cached[dev] = n;
  return n;
}

int launch_gemm_tc(const CUtensorMap& tmW, const CUtensorMap& tmX, const CUtensorMap& tmXlo,
                   const CUtensorMap& tmOut, const GemmArgs& a, cudaStream_t st) {
  if (a.ftiles <= 0 || (a.ftiles & 1) || a.K % kGemmBK != 0) return PLK_ERR_SHAPE;
  static int attr_done[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PLK_ERR_CUDA;
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) !=
        cudaSuccess)
      return PLK_ERR_CUDA;
    attr_done[dev] = 1;
  }
  // persistent: every resident CTA pair owns an equal share of the k-block iterations
  const int pairs = resident_pairs(a.num_sms);
  if (pairs <= 0) return PLK_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
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
  if (cudaLaunchKernelEx(&cfg, gemm_tc_kernel, tmW, tmX, tmXlo, tmOut, a) != cudaSuccess) return PLK_ERR_CUDA;
  return PLK_OK;
}

}  // namespace plk
