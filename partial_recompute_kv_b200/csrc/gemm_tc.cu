// tcgen05 GEMM for the projections of the partial-recompute layer step:
// out[token, f] = sum_k X[token, k] * W[f, k] on the M active rows only (the
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
//    warps 2-5 drain TMEM (tcgen05.ld) and run the fused epilogue.
//  * Split-K over a thread-block cluster: the CS CTAs of a cluster share one
//    output tile, each accumulating a contiguous 1/CS of K.  After the main loop
//    each CTA parks its fp32 partial in its own (now idle) stage buffers; then
//    CTA r finishes the token chunks c with c % CS == r, summing the CS partials
//    through distributed shared memory, so the reduction stays on chip and the
//    epilogue is spread over the cluster.  CS is chosen per GEMM on the host so
//    that tiles x CS fills the SMs (at M <= 256 the O and down projections have
//    only 32 tiles of 128 features).  CS = 1 drains TMEM straight into the
//    epilogue.
//  * Epilogues: QKV (Q compact; K and V scattered straight into the cache rows,
//    the K/V refresh of SureLock Sec. 2), O (h += a W_o^T, fp32), GU (tile =
//    64 gate rows + 64 up rows of the same features; silu(g) * u), DOWN
//    (h + act W_down^T, scattered into the output cache rows).  Each warp's
//    32 features x 32 tokens leave through a small staging buffer as 16-byte
//    token-major stores.
#include "plk_common.cuh"
#include "plk_internal.h"

namespace plk {

namespace {

constexpr int kStageA = kGemmBM * kGemmBK * 2;     // 16 KB
constexpr int kStageB = kGemmBNMax * kGemmBK * 2;  // 32 KB
constexpr size_t kOffB = (size_t)kGemmStages * kStageA;
constexpr size_t kOffBar = kOffB + (size_t)kGemmStages * kStageB;
constexpr size_t kOffIdx = kOffBar + 128;
constexpr size_t kOffStg = kOffIdx + kGemmBNMax * 4;
constexpr int kStgFloats = 32 * 32;                // per epilogue warp: 32 tokens x 32 features
constexpr size_t kSmemUsed = kOffStg + 4 * kStgFloats * 4;
constexpr size_t kSmemBytes = kSmemUsed + 1024;    // slack for 1024-byte alignment
// Partial parked for the cluster reduction, in the stage area once the main loop
// is over: [chunk][lane quarter][lane][36] fp32 (36 = 32 + padding: 16-byte
// accesses of 8 consecutive lanes hit distinct banks).
constexpr int kRbLane = 36;
constexpr int kRbQuarter = 32 * kRbLane;
constexpr int kRbChunk = 4 * kRbQuarter;
static_assert((size_t)8 * kRbChunk * 4 <= kOffBar, "partial must fit the stage buffers");

// silu(g) = g / (1 + e^-g) with the fast exp and divide intrinsics: their ~1e-6
// relative error is far below the bf16 rounding the product gets next.
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

__device__ __forceinline__ float4 ld_dsmem_v4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

}  // namespace

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                   const GemmArgs args) {
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
  volatile int* s_epi_abort = reinterpret_cast<volatile int*>(bars + 11);
  int* s_idx = reinterpret_cast<int*>(smem + kOffIdx);
  float* stg_all = reinterpret_cast<float*>(smem + kOffStg);
  float* rb = reinterpret_cast<float*>(smem);  // partial for the cluster reduction

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int CS = gridDim.x, kr = blockIdx.x;  // cluster = the CS CTAs along x
  const int M = args.seg_ptr[args.B];
  const int ft = blockIdx.y / args.ttiles_max, tt = blockIdx.y - ft * args.ttiles_max;
  const int tok0 = tt * kGemmBNMax;
  if (tok0 >= M) return;  // same decision in every CTA of the cluster: it exits as a whole
  const int ntok = min(kGemmBNMax, M - tok0);
  const int ncols = (ntok + 63) & ~63, nchunks = ncols >> 5;
  const int KB = args.K / kGemmBK;
  const int kb0 = kr * KB / CS, kb1 = (kr + 1) * KB / CS;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGemmStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(tfull, 1);
    *s_abort = 0;
    *s_epi_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  // epilogue state shared by the direct (CS = 1) and reduced (CS > 1) paths
  const int q = warp & 3;           // TMEM lane quarter this warp may access
  const int lr = q * 32 + lane;     // tile row = TMEM lane = feature row in tile
  const int et = threadIdx.x - 64;  // 0..127 in the epilogue warps
  const int d = args.d;
  const bool resid = args.epi == EPI_O || args.epi == EPI_DOWN;
  const int f128 = ft * kGemmBM + lr;
  float* stg = stg_all + q * kStgFloats;
  __nv_bfloat16* stg_h = reinterpret_cast<__nv_bfloat16*>(stg);
  const int fbase = ft * kGemmBM + q * 32;  // first feature of this warp

  // residual operand (fp32 h, contiguous rows); rows past ntok are clamped to a
  // valid row and never stored, so every load is issued unconditionally
  auto load_res = [&](int c, float (&dst)[32]) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int jj = min(c * 32 + i, ntok - 1);
      dst[i] = __ldcg(&args.h32[(size_t)(tok0 + jj) * d + f128]);
    }
  };
  // fused epilogue of token chunk c (tokens tok0 + 32c ..) from this thread's
  // accumulator row v and residuals res
  auto apply = [&](int c, const float (&v)[32], const float (&res)[32]) {
    const int jb = c * 32;
    const int nval = ntok - jb;
    if (args.epi == EPI_QKV || args.epi == EPI_DOWN) {
#pragma unroll
      for (int i = 0; i < 32; ++i) stg_h[i * 32 + lane] = f2bf(args.epi == EPI_DOWN ? res[i] + v[i] : v[i]);
      __syncwarp();
      const int part = fbase / d, col = fbase - part * d;
      __nv_bfloat16* dst =
          args.epi == EPI_DOWN
              ? (__nv_bfloat16*)args.y_cache
              : (part == 0 ? (__nv_bfloat16*)args.q_out
                           : (part == 1 ? (__nv_bfloat16*)args.k_cache : (__nv_bfloat16*)args.v_cache));
      const bool compact = args.epi == EPI_QKV && part == 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int tk = k * 8 + (lane >> 2);
        if (tk < nval) {
          const size_t row = compact ? (size_t)(tok0 + jb + tk) : (size_t)s_idx[jb + tk];
          *reinterpret_cast<uint4*>(dst + row * d + col + (lane & 3) * 8) =
              reinterpret_cast<const uint4*>(stg_h)[tk * 4 + (lane & 3)];
        }
      }
      __syncwarp();
    } else if (args.epi == EPI_O) {
#pragma unroll
      for (int i = 0; i < 32; ++i) stg[i * 32 + lane] = v[i] + res[i];
      __syncwarp();
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int tk = k * 4 + (lane >> 3);
        if (tk < nval)
          *reinterpret_cast<float4*>(args.h32 + (size_t)(tok0 + jb + tk) * d + fbase + (lane & 7) * 4) =
              reinterpret_cast<const float4*>(stg)[tk * 8 + (lane & 7)];
      }
      __syncwarp();
    } else {  // EPI_GU
      // gate rows are TMEM lanes 0-63 (warps q = 0, 1), up rows lanes 64-127
      // (q = 2, 3): warp q+2 parks its values in its staging buffer, warp q reads
      // them, forms silu(g) * u and stores it; two 64-thread barriers per chunk
      if (q >= 2) {
#pragma unroll
        for (int i = 0; i < 32; ++i) stg[i * 32 + lane] = v[i];
      }
      named_bar_sync(2 + (q & 1), 64);
      if (q < 2) {
        const float* up = stg_all + (q + 2) * kStgFloats;
#pragma unroll
        for (int i = 0; i < 32; ++i) stg_h[i * 32 + lane] = f2bf(silu_f(v[i]) * up[i * 32 + lane]);
        __syncwarp();
        const int F = args.gu_F;
        __nv_bfloat16* out = (__nv_bfloat16*)args.act_out + ft * 64 + q * 32;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int tk = k * 8 + (lane >> 2);
          if (tk < nval)
            *reinterpret_cast<uint4*>(out + (size_t)(tok0 + jb + tk) * F + (lane & 3) * 8) =
                reinterpret_cast<const uint4*>(stg_h)[tk * 4 + (lane & 3)];
        }
        __syncwarp();
      }
      named_bar_sync(2 + (q & 1), 64);  // warp q+2 may refill its buffer
    }
  };

  float res[32];  // epilogue warps: residuals of the chunk being finished

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      const int nbox = ncols >> 6;
      const uint32_t bytes = kStageA + nbox * (64 * kGemmBK * 2);
      const int yA0 = (args.epi == EPI_GU) ? ft * 64 : ft * kGemmBM;
      const int yA1 = (args.epi == EPI_GU) ? args.gu_F + ft * 64 : ft * kGemmBM + 64;
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
    // ------------------------------------------------------------ epilogue, part 1
    for (int j = et; j < ntok; j += 128) s_idx[j] = args.idx[tok0 + j];
    if (!mbar_wait(tfull, 0)) *s_epi_abort = 1;
    named_bar_sync(1, 128);
    tc_fence_after();
    // a K range of zero length (more slices than k-blocks) leaves TMEM unwritten
    const bool have_acc = !*s_epi_abort && !*s_abort && kb1 > kb0;
    const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16);
    if (CS == 1) {
      float res_nx[32];
      if (resid) load_res(0, res_nx);
      for (int c = 0; c < nchunks && have_acc; ++c) {
        if (resid) {
#pragma unroll
          for (int i = 0; i < 32; ++i) res[i] = res_nx[i];
          if (c + 1 < nchunks) load_res(c + 1, res_nx);
        }
        uint32_t r[32];
        tmem_ld32(taddr + (uint32_t)(c * 32), r);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
        apply(c, v, res);
      }
    } else {
      // residuals of the first chunk this CTA will finish, in flight across the barrier
      if (resid && kr < nchunks) load_res(kr, res);
      // park this CTA's partial for the cluster reduction
      for (int c = 0; c < nchunks; ++c) {
        uint32_t r[32];
        if (have_acc) {
          tmem_ld32(taddr + (uint32_t)(c * 32), r);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = 0u;
        }
        float4* dst = reinterpret_cast<float4*>(rb + c * kRbChunk + q * kRbQuarter + lane * kRbLane);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          dst[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                               __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
      }
    }
  }

  tc_fence_before();
  if (CS > 1)
    cluster_sync_all();  // every CTA's partial is parked
  else
    __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
  }
  if (CS > 1) {
    if (warp >= 2) {
      // ---------------------------------------------------------- epilogue, part 2
      // this CTA finishes chunks c = kr, kr + CS, ... summing the CS partials
      const uint32_t mine = smem_u32(rb + q * kRbQuarter + lane * kRbLane);
      for (int c = kr; c < nchunks; c += CS) {
        if (resid && c != kr) load_res(c, res);  // the first chunk's were loaded before the barrier
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
        for (int p = 0; p < CS; ++p) {
          const uint32_t src = dsmem_addr(mine + (uint32_t)(c * kRbChunk * 4), (uint32_t)p);
          float4 t[8];  // all of a peer's loads in flight before the first add
#pragma unroll
          for (int i = 0; i < 8; ++i) t[i] = ld_dsmem_v4(src + 16u * i);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            v[4 * i] += t[i].x;
            v[4 * i + 1] += t[i].y;
            v[4 * i + 2] += t[i].z;
            v[4 * i + 3] += t[i].w;
          }
        }
        apply(c, v, res);
      }
    }
    cluster_sync_all();  // peers are done reading this CTA's partial
  }
}

// Cluster size for a GEMM: the K split that minimises the makespan in k-block
// times, counting whole waves of tiles x CS CTAs over the SMs plus a small
// reduction cost per wave.  Chosen from the tile count at M <= 256 tokens, the
// regime where the projections have too few tiles to fill the GPU.
static int choose_cluster(int ftiles, int kblocks, int nsm) {
  int best = 1;
  double best_t = 1e30;
  for (int cs = 1; cs <= 8; ++cs) {
    if (kblocks / cs < 2) break;
    const int waves = ceil_div(ftiles * cs, nsm);
    const double t = (double)waves * ceil_div(kblocks, cs) + (cs > 1 ? 3.0 * waves : 1.0);
    if (t < best_t - 1e-9) {
      best_t = t;
      best = cs;
    }
  }
  return best;
}

int launch_gemm_tc(const CUtensorMap& tmW, const CUtensorMap& tmX, const GemmArgs& a, cudaStream_t st) {
  static int attr_done[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PLK_ERR_CUDA;
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) !=
        cudaSuccess)
      return PLK_ERR_CUDA;
    attr_done[dev] = 1;
  }
  const int cs = choose_cluster(a.ftiles, a.K / kGemmBK, a.num_sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, a.ftiles * a.ttiles_max, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = cs;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = cs > 1 ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, gemm_tc_kernel, tmW, tmX, a) != cudaSuccess) return PLK_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? PLK_OK : PLK_ERR_CUDA;
}

}  // namespace plk
