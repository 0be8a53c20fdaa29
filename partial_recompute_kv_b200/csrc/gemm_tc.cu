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
//  * Epilogues (one kernel instantiation each): QKV (Q compact; K and V
//    scattered straight into the cache rows, the K/V refresh of SureLock
//    Sec. 2), O (h += a W_o^T, fp32), GU (tile = 64 gate rows + 64 up rows of
//    the same features; silu(g) * u), DOWN (h + act W_down^T, scattered into
//    the output cache rows).  Each warp's 32 tokens x 32 features are staged
//    token-major in shared memory and leave as 16-byte stores; the parked
//    partial uses the same token-major layout, so every remote read of the
//    reduction is 512 contiguous bytes per warp instruction.
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
constexpr int kBlk = 32 * 32;                      // a warp's block: 32 tokens x 32 features (fp32)
constexpr size_t kSmemUsed = kOffStg + 4 * kBlk * 4;
constexpr size_t kSmemBytes = kSmemUsed + 1024;    // slack for 1024-byte alignment
// Partial parked for the cluster reduction, in the stage area once the main loop
// is over: [chunk][lane quarter][token][feature] fp32.
constexpr int kRbChunk = 4 * kBlk;
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

__device__ __forceinline__ float4 add4(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

__device__ __forceinline__ uint4 pack8_bf16(float4 a, float4 b) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
  h[0] = __floats2bfloat162_rn(a.x, a.y);
  h[1] = __floats2bfloat162_rn(a.z, a.w);
  h[2] = __floats2bfloat162_rn(b.x, b.y);
  h[3] = __floats2bfloat162_rn(b.z, b.w);
  return u;
}

// Epilogue of one warp block.  The block (32 tokens x 32 features, fp32,
// token-major) sits in shared memory at `blk`; token t of the block is token
// tok0 + jb + t of the tile, feature j is feature fbase + j.
//   Items for bf16 outputs: lane l handles 8 features (group l & 3) of tokens
//   k*8 + (l >> 2), k = 0..3.  Items for the fp32 output: 4 features (group
//   l & 7) of tokens k*4 + (l >> 3), k = 0..7.  Residuals for those items are
//   loaded by load_res into r[8] (float4).
struct EpiCtx {
  int tok0, jb, nval, fbase, d, lane;
  const int* s_idx;
};

template <int EPI>
__device__ __forceinline__ void load_res(const GemmArgs& a, const EpiCtx& e, int ntok, float4 (&r)[8]) {
  if (EPI == EPI_O) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int tk = min(e.jb + k * 4 + (e.lane >> 3), ntok - 1);  // clamped: always a valid row
      r[k] = __ldcg(reinterpret_cast<const float4*>(a.h32 + (size_t)(e.tok0 + tk) * e.d + e.fbase +
                                                    (e.lane & 7) * 4));
    }
  } else if (EPI == EPI_DOWN) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int tk = min(e.jb + k * 8 + (e.lane >> 2), ntok - 1);
      const float4* src =
          reinterpret_cast<const float4*>(a.h32 + (size_t)(e.tok0 + tk) * e.d + e.fbase + (e.lane & 3) * 8);
      r[2 * k] = __ldcg(src);
      r[2 * k + 1] = __ldcg(src + 1);
    }
  }
}

}  // namespace

namespace {

template <int EPI>
__device__ __forceinline__ void finish_block(const GemmArgs& a, const EpiCtx& e, const float* blk,
                                             const float* up_blk, const float4 (&r)[8]) {
  const int l = e.lane;
  if (EPI == EPI_O) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int t = k * 4 + (l >> 3);
      if (t < e.nval) {
        const float4 x = add4(reinterpret_cast<const float4*>(blk)[t * 8 + (l & 7)], r[k]);
        *reinterpret_cast<float4*>(a.h32 + (size_t)(e.tok0 + e.jb + t) * e.d + e.fbase + (l & 7) * 4) = x;
      }
    }
    return;
  }
  __nv_bfloat16* dst;
  int col = 0;
  size_t ld = (size_t)e.d;
  bool compact = false;
  if (EPI == EPI_QKV) {
    const int part = e.fbase / e.d;
    col = e.fbase - part * e.d;
    dst = (__nv_bfloat16*)(part == 0 ? a.q_out : (part == 1 ? a.k_cache : a.v_cache));
    compact = part == 0;
  } else if (EPI == EPI_DOWN) {
    dst = (__nv_bfloat16*)a.y_cache;
    col = e.fbase;
  } else {  // EPI_GU: features fbase index the [gate | up] tile rows; output column ft*64 + j
    dst = (__nv_bfloat16*)a.act_out;
    col = e.fbase;  // caller passes the output column of this warp's gate features
    ld = (size_t)a.gu_F;
    compact = true;
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int t = k * 8 + (l >> 2);
    if (t < e.nval) {
      const float4* src = reinterpret_cast<const float4*>(blk) + t * 8 + (l & 3) * 2;
      float4 x0 = src[0], x1 = src[1];
      if (EPI == EPI_DOWN) {
        x0 = add4(x0, r[2 * k]);
        x1 = add4(x1, r[2 * k + 1]);
      } else if (EPI == EPI_GU) {
        const float4* u = reinterpret_cast<const float4*>(up_blk) + t * 8 + (l & 3) * 2;
        const float4 u0 = u[0], u1 = u[1];
        x0 = make_float4(silu_f(x0.x) * u0.x, silu_f(x0.y) * u0.y, silu_f(x0.z) * u0.z, silu_f(x0.w) * u0.w);
        x1 = make_float4(silu_f(x1.x) * u1.x, silu_f(x1.y) * u1.y, silu_f(x1.z) * u1.z, silu_f(x1.w) * u1.w);
      }
      const size_t row = compact ? (size_t)(e.tok0 + e.jb + t) : (size_t)e.s_idx[e.jb + t];
      *reinterpret_cast<uint4*>(dst + row * ld + col + (l & 3) * 8) = pack8_bf16(x0, x1);
    }
  }
}

}  // namespace

template <int EPI>
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

  // epilogue state
  const int q = warp & 3;  // TMEM lane quarter this warp may access (warps 2-5)
  float* stg = stg_all + q * kBlk;
  EpiCtx e;
  e.tok0 = tok0;
  e.jb = 0;
  e.nval = 0;
  e.fbase = EPI == EPI_GU ? ft * 64 + (q & 1) * 32 : ft * kGemmBM + q * 32;
  e.d = args.d;
  e.lane = lane;
  e.s_idx = s_idx;
  const bool gate_warp = EPI != EPI_GU || q < 2;  // GU: warps q >= 2 hold the up rows
  float4 res[8];
  auto at_chunk = [&](int c) {
    e.jb = c * 32;
    e.nval = ntok - e.jb;
  };
  // the warp's block of chunk c is in stg; finish it (GU: pair with warp q^2)
  auto finish = [&]() {
    if (EPI == EPI_GU) {
      named_bar_sync(2 + (q & 1), 64);  // both halves of the pair are staged
      if (gate_warp) finish_block<EPI>(args, e, stg, stg_all + (q + 2) * kBlk, res);
      named_bar_sync(2 + (q & 1), 64);  // warp q+2 may overwrite its block
    } else {
      finish_block<EPI>(args, e, stg, nullptr, res);
      __syncwarp();
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      const int nbox = ncols >> 6;
      const uint32_t bytes = kStageA + nbox * (64 * kGemmBK * 2);
      const int yA0 = (EPI == EPI_GU) ? ft * 64 : ft * kGemmBM;
      const int yA1 = (EPI == EPI_GU) ? args.gu_F + ft * 64 : ft * kGemmBM + 64;
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
    const int et = threadIdx.x - 64;
    for (int j = et; j < ntok; j += 128) s_idx[j] = args.idx[tok0 + j];
    if (!mbar_wait(tfull, 0)) *s_epi_abort = 1;
    named_bar_sync(1, 128);
    tc_fence_after();
    // a K range of zero length (more slices than k-blocks) leaves TMEM unwritten
    const bool have_acc = !*s_epi_abort && !*s_abort && kb1 > kb0;
    const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16);
    // TMEM chunk c -> token-major block at dst (this lane = feature, 32 tokens)
    auto drain_chunk = [&](int c, float* dst) {
      uint32_t r[32];
      if (have_acc) {
        tmem_ld32(taddr + (uint32_t)(c * 32), r);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = 0u;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) dst[i * 32 + lane] = __uint_as_float(r[i]);
    };
    if (CS == 1) {
      for (int c = 0; c < nchunks; ++c) {
        at_chunk(c);
        if (gate_warp) load_res<EPI>(args, e, ntok, res);
        drain_chunk(c, stg);
        __syncwarp();
        finish();
      }
    } else {
      // residuals of the first chunk this CTA finishes, in flight across the barrier
      if (kr < nchunks) {
        at_chunk(kr);
        load_res<EPI>(args, e, ntok, res);
      }
      for (int c = 0; c < nchunks; ++c) drain_chunk(c, rb + c * kRbChunk + q * kBlk);
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
      // this CTA finishes chunks c = kr, kr + CS, ...: lane l sums float4 l + 32j
      // (j = 0..7) of the warp's block over the CS partials, into its own block
      for (int c = kr; c < nchunks; c += CS) {
        at_chunk(c);
        if (c != kr) load_res<EPI>(args, e, ntok, res);
        const uint32_t base = smem_u32(rb + c * kRbChunk + q * kBlk) + 16u * lane;
        float4 acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int p = 0; p < CS; ++p) {
          const uint32_t src = dsmem_addr(base, (uint32_t)p);
          float4 t[8];  // a peer's eight loads in flight before the first add
#pragma unroll
          for (int j = 0; j < 8; ++j) t[j] = ld_dsmem_v4(src + 512u * j);
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[j] = add4(acc[j], t[j]);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) reinterpret_cast<float4*>(stg)[lane + 32 * j] = acc[j];
        __syncwarp();
        finish();
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

template <int EPI>
static int launch_epi(const CUtensorMap& tmW, const CUtensorMap& tmX, const GemmArgs& a, int cs,
                      cudaStream_t st) {
  static int attr_done[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PLK_ERR_CUDA;
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(gemm_tc_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes) != cudaSuccess)
      return PLK_ERR_CUDA;
    attr_done[dev] = 1;
  }
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
  if (cudaLaunchKernelEx(&cfg, gemm_tc_kernel<EPI>, tmW, tmX, a) != cudaSuccess) return PLK_ERR_CUDA;
  return cudaPeekAtLastError() == cudaSuccess ? PLK_OK : PLK_ERR_CUDA;
}

int launch_gemm_tc(const CUtensorMap& tmW, const CUtensorMap& tmX, const GemmArgs& a, cudaStream_t st) {
  const int cs = choose_cluster(a.ftiles, a.K / kGemmBK, a.num_sms);
  switch (a.epi) {
    case EPI_QKV: return launch_epi<EPI_QKV>(tmW, tmX, a, cs, st);
    case EPI_O: return launch_epi<EPI_O>(tmW, tmX, a, cs, st);
    case EPI_GU: return launch_epi<EPI_GU>(tmW, tmX, a, cs, st);
    case EPI_DOWN: return launch_epi<EPI_DOWN>(tmW, tmX, a, cs, st);
    default: return PLK_ERR_ARG;
  }
}

}  // namespace plk
