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
//  * Split-K without inter-CTA waiting: CTA (s, tile) accumulates the s-th of
//    S contiguous K ranges and adds its fp32 partial into the fp32 output with
//    TMA bulk reduce-add (cp.reduce.async.bulk.tensor ... .add.f32), which the
//    L2 applies atomically.  The output is either the residual stream h (the O
//    and down projections: h += a W_o^T, then h += act W_down^T) or a zeroed
//    fp32 buffer whose finishing kernel applies the nonlinear or scattering
//    epilogue (QKV -> Q and the K/V cache rows; gate/up -> silu(g) * u).  S is
//    chosen per GEMM on the host so that tiles x S fills the SMs (at M <= 256
//    the O and down projections have only 32 tiles of 128 features).  The
//    order of the reduce-adds is not fixed, so results may differ in the last
//    fp32 bit between runs.
//  * Each epilogue warp stages its 32 tokens x 32 features token-major in a
//    double-buffered shared-memory block (rows past M zeroed) and issues one
//    bulk reduce per block; a gate/up tile (64 gate + 64 up rows of the same
//    features) lands in the gate and up halves of its [M, 2F] buffer.
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

// K slices for `tiles` output tiles of `kblocks` k-blocks on `nsm` SMs: the
// split that minimises the makespan, counted in k-block times as whole waves
// of tiles x S CTAs times (k-blocks per slice + a fixed per-CTA cost for the
// pipeline fill and the epilogue).  Host and device evaluate the same function.
__host__ __device__ inline int gemm_split(int tiles, int kblocks, int nsm) {
  int best = 1;
  float best_t = 3.0e38f;
  for (int s = 1; s <= kGemmSplitMax; ++s) {
    if (kblocks / s < 2) break;
    const int waves = (tiles * s + nsm - 1) / nsm;
    const float t = (float)waves * (float)((kblocks + s - 1) / s + 5);
    if (t < best_t * 0.999f) {
      best_t = t;
      best = s;
    }
  }
  return best;
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                   const __grid_constant__ CUtensorMap tmOut, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kOffB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* full = bars;        // [4] TMA -> MMA
  uint64_t* empty = bars + 4;   // [4] MMA -> TMA
  uint64_t* tfull = bars + 8;   // MMA -> epilogue
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 9);
  volatile int* s_abort = reinterpret_cast<volatile int*>(bars + 10);
  float* stg_all = reinterpret_cast<float*>(smem + kOffStg);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int M = args.seg_ptr[args.B];
  const int ft = blockIdx.y / args.ttiles_max, tt = blockIdx.y - ft * args.ttiles_max;
  const int tok0 = tt * kGemmBNMax;
  if (tok0 >= M) return;
  const int ntok = min(kGemmBNMax, M - tok0);
  const int ncols = (ntok + 63) & ~63, nchunks = ncols >> 5;
  const int KB = args.K / kGemmBK;
  // K slices for the live tile count; the grid holds the most any M can use
  const int S = min((int)gridDim.x, gemm_split(args.ftiles * ceil_div(M, kGemmBNMax), KB, args.num_sms));
  const int ks = blockIdx.x;
  if (ks >= S) return;
  const int kb0 = ks * KB / S, kb1 = (ks + 1) * KB / S;
  if (kb1 <= kb0) return;  // an empty K slice adds nothing

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGemmStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(tfull, 1);
    *s_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmOut);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      const int nbox = ncols >> 6;
      const uint32_t bytes = kStageA + nbox * (64 * kGemmBK * 2);
      const int yA0 = args.gu_F ? ft * 64 : ft * kGemmBM;
      const int yA1 = args.gu_F ? args.gu_F + ft * 64 : ft * kGemmBM + 64;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1)) {
          *s_abort = 1;
          break;
        }
        mbar_expect_tx(&full[stage], bytes);
        uint8_t* a = sA + stage * kStageA;
        uint8_t* b = sB + stage * kStageB;
        const int x = kb * kGemmBK;
        tma_load_2d(a, &tmW, x, yA0, &full[stage]);
        tma_load_2d(a + 8192, &tmW, x, yA1, &full[stage]);
        for (int j = 0; j < nbox; ++j) tma_load_2d(b + j * 8192, &tmX, x, tok0 + j * 64, &full[stage]);
        ++issued;
        if (++stage == kGemmStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (*s_abort) {
        // let the copies this thread started land before the CTA moves on
        for (int i = issued - kGemmStages < 0 ? 0 : issued - kGemmStages; i < issued; ++i)
          (void)mbar_wait(&full[i % kGemmStages], (uint32_t)((i / kGemmStages) & 1));
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t idesc = idesc_bf16(kGemmBM, ncols);
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
          umma_bf16(tmem_base, adesc + 2 * k, bdesc + 2 * k, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
        umma_commit(&empty[stage]);
        if (++stage == kGemmStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      umma_commit(tfull);  // also the drain: arrives once every MMA above is complete
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter of this warp
    // output column of this warp's 32 features (gate/up tile: lanes 0-63 gate, 64-127 up)
    const int col = args.gu_F ? (q < 2 ? ft * 64 + q * 32 : args.gu_F + ft * 64 + (q - 2) * 32)
                              : ft * kGemmBM + q * 32;
    const bool ok = mbar_wait(tfull, 0) && !*s_abort;
    tc_fence_after();
    if (__all_sync(0xffffffffu, ok)) {
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16);
      for (int c = 0; c < nchunks; ++c) {
        float* blk = stg_all + (q * 2 + (c & 1)) * kBlk;
        if (c >= 2) {
          if (lane == 0) bulk_wait_read<1>();  // the reduce that used this buffer has read it
          __syncwarp();
        }
        uint32_t r[32];
        tmem_ld32(taddr + (uint32_t)(c * 32), r);
        tmem_ld_wait();
        const int nval = ntok - c * 32;  // tokens past M contribute zeros
#pragma unroll
        for (int i = 0; i < 32; ++i) blk[i * 32 + lane] = i < nval ? __uint_as_float(r[i]) : 0.f;
        fence_proxy_async_smem();  // make the block visible to the bulk-copy unit
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_2d(&tmOut, col, tok0 + c * 32, blk);
          bulk_commit();
        }
      }
      if (lane == 0) bulk_wait_all();  // sources read and adds issued before the CTA ends
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
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
  // the grid is sized for one token tile (M <= 256), the regime where the
  // projections have too few tiles to fill the GPU; CTAs beyond the split the
  // live M calls for exit at once
  const int S = gemm_split(a.ftiles, a.K / kGemmBK, a.num_sms);
  const dim3 grid(S, a.ftiles * a.ttiles_max);
  gemm_tc_kernel<<<grid, kGemmThreads, kSmemBytes, st>>>(tmW, tmX, tmOut, a);
  return cudaPeekAtLastError() == cudaSuccess ? PLK_OK : PLK_ERR_CUDA;
}

}  // namespace plk
