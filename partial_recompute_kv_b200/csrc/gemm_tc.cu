// tcgen05 GEMM for the projections of the partial-recompute layer step:
// out[token, f] += sum_k X[token, k] * W[f, k] on the M active rows only (the
// SureLock page, "Stopping Computation for Converged Tokens in Masked
// Diffusion-LM Decoding", Sec. 2: Q/K/V, output projection and FFN run for the
// active subset, cost O(M d^2)).
//
// Design (sm_100a):
//  * Weights are the UMMA A operand (M = 128 feature rows per tile) and the
//    compacted activations the B operand (N = 64..256 tokens, chosen on the
//    device from M = seg_ptr[B]); at M <= 256 every weight byte is read from HBM
//    once.  Both operands are K-major bf16 tiles loaded by TMA with a 128-byte
//    swizzle into a 4-stage ring; accumulation is fp32 in TMEM.
//  * Warp roles: warp 0 issues TMA, one thread of warp 1 issues tcgen05.mma,
//    warps 2-5 drain TMEM (tcgen05.ld).
//  * Persistent stream-K without inter-CTA waiting: one CTA per SM owns an
//    equal, contiguous share of the tiles x k-blocks iteration space and adds
//    the fp32 partial of each tile piece it covers into the fp32 output with
//    TMA bulk reduce-add (cp.reduce.async.bulk.tensor ... .add.f32), which the
//    L2 applies atomically.  The output is either the residual stream h (the O
//    and down projections: h += a W_o^T, then h += act W_down^T) or a zeroed
//    fp32 buffer whose finishing kernel applies the nonlinear or scattering
//    epilogue (QKV -> Q and the K/V cache rows; gate/up -> silu(g) * u).  At
//    M <= 256 the O and down projections have only 32 tiles of 128 features;
//    stream-K keeps all SMs busy regardless.  The order of the reduce-adds is
//    not fixed, so results may differ in the last fp32 bit between runs.
//  * Two 256-column TMEM accumulators: the epilogue drains one tile piece while
//    the MMA fills the next, and the TMA producer runs ahead across pieces.
//  * Each epilogue warp stages its 32 tokens x 32 features token-major in a
//    double-buffered shared-memory block (rows past M zeroed) and issues one
//    bulk reduce per block; the CTA's last piece stages all its blocks in the
//    then idle operand ring so that every reduce is in flight at once.  A
//    gate/up tile (64 gate + 64 up rows of the same features) lands in the
//    gate and up halves of its [M, 2F] buffer.
#include "plk_common.cuh"
#include "plk_internal.h"

namespace plk {

namespace {

constexpr int kStageA = kGemmBM * kGemmBK * 2;     // 16 KB
constexpr int kStageB = kGemmBNMax * kGemmBK * 2;  // 32 KB
constexpr size_t kOffB = (size_t)kGemmStages * kStageA;
constexpr size_t kOffBar = kOffB + (size_t)kGemmStages * kStageB;
constexpr size_t kOffStg = kOffBar + 128;
constexpr int kBlk = 32 * 32;                      // a warp's block: 32 tokens x 32 features (fp32)
constexpr size_t kSmemUsed = kOffStg + 4 * 2 * kBlk * 4;
constexpr size_t kSmemBytes = kSmemUsed + 1024;    // slack for 1024-byte alignment
static_assert(kSmemBytes <= 232448, "shared memory budget");

// bulk reduce-add of a [32 rows][32 fp32] smem block into the tensor at (x, y)
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* tm, int x, int y, const void* smem_src) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
          reinterpret_cast<uint64_t>(tm)),
      "r"(x), "r"(y), "r"(smem_u32(smem_src))
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// waits until at most n committed bulk groups still read their shared-memory source
template <int n>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(n) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

}  // namespace

// The flattened iteration space of one GEMM: tiles x KB k-blocks, tile u =
// ft * ttiles + tt (token tiles fastest, so CTAs that run at the same time share
// a weight tile in L2).  CTA c owns iterations [c*T/G, (c+1)*T/G); a segment is
// the part of that range inside one tile.
struct SegWalk {
  long long i, iend;
  int KB;
  __device__ SegWalk(int cta, int nctas, int tiles, int KB_) : KB(KB_) {
    const long long T = (long long)tiles * KB_;
    i = T * cta / nctas;
    iend = T * (cta + 1) / nctas;
  }
  __device__ bool next(int& u, int& kb0, int& kb1) {
    if (i >= iend) return false;
    u = (int)(i / KB);
    kb0 = (int)(i - (long long)u * KB);
    kb1 = (int)min((long long)KB, kb0 + (iend - i));
    i += kb1 - kb0;
    return true;
  }
  __device__ bool done() const { return i >= iend; }
};

struct TileGeom {
  int ft, tok0, ntok, ncols;
  __device__ TileGeom(int u, int ttiles, int M) {
    ft = u / ttiles;
    tok0 = (u - ft * ttiles) * kGemmBNMax;
    ntok = min(kGemmBNMax, M - tok0);
    ncols = (ntok + 63) & ~63;  // UMMA N: whole 64-token boxes
  }
};

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                   const __grid_constant__ CUtensorMap tmOut, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kOffB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* full = bars;            // [4] TMA -> MMA
  uint64_t* empty = bars + 4;       // [4] MMA -> TMA
  uint64_t* tfull = bars + 8;       // [2] MMA -> epilogue, per TMEM accumulator
  uint64_t* tempty = bars + 10;     // [2] epilogue -> MMA
  uint64_t* drain = bars + 12;      // MMA completion on the abort path
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* s_abort = reinterpret_cast<volatile int*>(bars + 14);
  float* stg_all = reinterpret_cast<float*>(smem + kOffStg);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // seg_ptr comes from a kernel before the predecessor: already complete (see pdl_wait)
  const int M = args.seg_ptr[args.B];
  const int ttiles = ceil_div(max(M, 0), kGemmBNMax);
  const int tiles = args.ftiles * ttiles;
  const int KB = args.K / kGemmBK;
  if (M <= 0 || SegWalk(blockIdx.x, gridDim.x, tiles, KB).done()) {  // no iterations for this CTA
    pdl_wait();
    return;
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGemmStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmOut);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, 512);  // two 256-column fp32 accumulators
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  if (warp != 0) {
    pdl_wait();
    pdl_trigger();
  }

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      // weight rows of tile t (gate/up tile: 64 gate rows, then the 64 up rows)
      auto load_a = [&](int stage, const TileGeom& t, int kb) {
        const int yA0 = args.gu_F ? t.ft * 64 : t.ft * kGemmBM;
        const int yA1 = args.gu_F ? args.gu_F + t.ft * 64 : t.ft * kGemmBM + 64;
        uint8_t* a = sA + stage * kStageA;
        tma_load_2d(a, &tmW, kb * kGemmBK, yA0, &full[stage]);
        tma_load_2d(a + 8192, &tmW, kb * kGemmBK, yA1, &full[stage]);
      };
      auto stage_bytes = [](const TileGeom& t) { return (uint32_t)(kStageA + (t.ncols >> 6) * (64 * kGemmBK * 2)); };
      SegWalk w(blockIdx.x, gridDim.x, tiles, KB);
      int u, kb0, kb1, stage = 0;
      // The weights are no kernel's output: the first stages' weight loads start
      // before the wait for the predecessor, overlapping its tail.
      int pre = 0;
      {
        SegWalk w2 = w;
        while (pre < kGemmStages && w2.next(u, kb0, kb1)) {
          const TileGeom t(u, ttiles, M);
          for (int kb = kb0; kb < kb1 && pre < kGemmStages; ++kb, ++pre) {
            mbar_expect_tx(&full[pre], stage_bytes(t));
            load_a(pre, t, kb);
          }
        }
      }
      pdl_wait();
      pdl_trigger();
      uint32_t phase = 0;
      long long issued = 0;
      while (!*s_abort && w.next(u, kb0, kb1)) {
        const TileGeom t(u, ttiles, M);
        const int nbox = t.ncols >> 6;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (issued >= pre) {  // stages past the prefetched ones: wait for a free slot
            if (!mbar_wait(&empty[stage], phase ^ 1)) {
              *s_abort = 1;
              break;
            }
            mbar_expect_tx(&full[stage], stage_bytes(t));
            load_a(stage, t, kb);
          }
          uint8_t* b = sB + stage * kStageB;
          for (int j = 0; j < nbox; ++j)
            tma_load_2d(b + j * 8192, &tmX, kb * kGemmBK, t.tok0 + j * 64, &full[stage]);
          ++issued;
          if (++stage == kGemmStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*s_abort) {
        // let the copies this thread started land before the CTA moves on
        for (long long i = issued > kGemmStages ? issued - kGemmStages : 0; i < issued; ++i)
          (void)mbar_wait(&full[i % kGemmStages], (uint32_t)((i / kGemmStages) & 1));
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      SegWalk w(blockIdx.x, gridDim.x, tiles, KB);
      int u, kb0, kb1, stage = 0, j = 0;
      uint32_t phase = 0;
      bool any = false;
      while (!*s_abort && w.next(u, kb0, kb1)) {
        const TileGeom t(u, ttiles, M);
        const int b = j & 1;
        if (!mbar_wait(&tempty[b], ((j >> 1) & 1) ^ 1)) {  // the epilogue has drained this accumulator
          *s_abort = 1;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem_base + (uint32_t)(b * 256);
        const uint32_t idesc = idesc_bf16(kGemmBM, t.ncols);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase)) {
            *s_abort = 1;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = sdesc_sw128(smem_u32(sA + stage * kStageA));
          const uint64_t bdesc = sdesc_sw128(smem_u32(sB + stage * kStageB));
#pragma unroll
          for (int k = 0; k < kGemmBK / 16; ++k)  // +32 bytes of K per step = 2 descriptor units
            umma_bf16(acc, adesc + 2 * k, bdesc + 2 * k, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          any = true;
          umma_commit(&empty[stage]);
          if (++stage == kGemmStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (*s_abort) break;
        umma_commit(&tfull[b]);  // arrives once every MMA of this segment is complete
        ++j;
      }
      if (*s_abort && any) {
        umma_commit(drain);  // wait for the MMAs in flight before TMEM is freed
        (void)mbar_wait(drain, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // a warp reads TMEM lanes 32 * (warp % 4) ..
    SegWalk w(blockIdx.x, gridDim.x, tiles, KB);
    int u, kb0, kb1, j = 0, n = 0;
    while (w.next(u, kb0, kb1)) {
      const bool last = w.done();  // no MMA or TMA follows: the stage buffers are free for staging
      const TileGeom t(u, ttiles, M);
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
        if (c == nchunks - 1) {  // accumulator b drained: the MMA may reuse it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[b]);
        }
        const int nval = t.ntok - c * 32;  // tokens past M contribute zeros
#pragma unroll
        for (int i = 0; i < 32; ++i) blk[i * 32 + lane] = i < nval ? __uint_as_float(r[i]) : 0.f;
        fence_proxy_async_smem();  // make the block visible to the bulk-copy unit
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_2d(&tmOut, col, t.tok0 + c * 32, blk);
          bulk_commit();
        }
      }
      ++j;
    }
    if (lane == 0) bulk_wait_all();  // sources read and adds complete before the CTA ends
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

int launch_gemm_tc(const CUtensorMap& tmW, const CUtensorMap& tmX, const CUtensorMap& tmOut, const GemmArgs& a,
                   cudaStream_t st) {
  static int attr_done[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PLK_ERR_CUDA;
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) !=
        cudaSuccess)
      return PLK_ERR_CUDA;
    attr_done[dev] = 1;
  }
  // persistent: one CTA per SM, each owning an equal share of the k-block iterations
  return launch_pdl(gemm_tc_kernel, dim3(a.num_sms), dim3(kGemmThreads), kSmemBytes, st, tmW, tmX, tmOut, a);
}

}  // namespace plk
