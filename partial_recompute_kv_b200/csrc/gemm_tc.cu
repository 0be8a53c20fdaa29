// Persistent tcgen05 GEMM for the projections of the partial-recompute layer
// step: out[token, f] = sum_k X[token, k] * W[f, k] on the M active rows only
// (the SureLock page, "Stopping Computation for Converged Tokens in Masked
// Diffusion-LM Decoding", Sec. 2: Q/K/V, output projection and FFN run for the
// active subset, cost O(M d^2)).
//
// Design (sm_100a):
//  * Weights are the UMMA A operand (M = 128 feature rows per tile) and the
//    compacted activations the B operand (N = 64..256 tokens, chosen on the
//    device from M = seg_ptr[B]); at M <= 256 every weight byte is read from HBM
//    exactly once.  Both operands are K-major bf16 tiles loaded by TMA with a
//    128-byte swizzle; accumulation is fp32 in TMEM (two 256-column buffers so
//    the epilogue of one tile overlaps the main loop of the next).
//  * Warp roles: warp 0 issues TMA, one thread of warp 1 issues tcgen05.mma,
//    warps 2-5 drain TMEM (tcgen05.ld) and run the fused epilogue.
//  * Stream-K: the (tile, k-block) iteration space is cut into gridDim.x equal
//    contiguous ranges, one per CTA (one CTA per SM).  A tile whose k-range is
//    split is finished by the CTA owning its k = 0 segment: the other CTAs
//    (whose range starts inside the tile, so they reach it first) store fp32
//    partials and release a flag; the owner waits for them (bounded), adds them
//    to its accumulator and runs the epilogue.  Every output element is written
//    once by a fused epilogue, no output buffer needs zeroing.
//  * Epilogues: QKV (Q compact; K and V scattered straight into the cache rows,
//    the K/V refresh of SureLock Sec. 2), O (h += a W_o^T, fp32), GU (tile =
//    64 gate rows + 64 up rows of the same features; silu(g) * u), DOWN
//    (+ fp32 residual, scattered into the output cache rows).
#include "plk_common.cuh"
#include "plk_internal.h"

namespace plk {

namespace {

constexpr int kStageA = kGemmBM * kGemmBK * 2;     // 16 KB
constexpr int kStageB = kGemmBNMax * kGemmBK * 2;  // 32 KB
constexpr int kTileCols = 256;                     // TMEM columns per accumulator buffer
constexpr int kSlotFloats = kGemmBNMax * kGemmBM;  // partial tile, [lane quarter][col][32 lanes]
constexpr size_t kOffB = (size_t)kGemmStages * kStageA;
constexpr size_t kOffBar = kOffB + (size_t)kGemmStages * kStageB;
constexpr size_t kOffIdx = kOffBar + 512;
constexpr int kRing = 8;                           // fix-up ring per epilogue warp: 8 pieces of 4 KB
constexpr int kPieceFloats = 32 * 32;              // one warp's chunk (32 columns x 32 lanes) of a partial
constexpr int kQuarterFloats = kGemmBNMax * 32;    // one lane quarter of a partial slot
constexpr size_t kOffStg = kOffIdx + kGemmBNMax * 4;
constexpr int kStgFloats = 32 * 32;                // per epilogue warp: 32 tokens x 32 features
constexpr size_t kSmemUsed = kOffStg + 4 * kStgFloats * 4;
constexpr size_t kSmemBytes = kSmemUsed + 1024;  // slack for 1024-byte alignment

struct Sched {
  int M, ttiles, kblocks, total, L, begin, end;
};

__device__ __forceinline__ void sched_init(Sched& s, const GemmArgs& a) {
  s.M = a.seg_ptr[a.B];
  s.ttiles = ceil_div(s.M, kGemmBNMax);
  s.kblocks = a.K / kGemmBK;
  s.total = a.ftiles * s.ttiles * s.kblocks;
  s.L = ceil_div(s.total, (int)gridDim.x);
  s.begin = min((int)blockIdx.x * s.L, s.total);
  s.end = min(s.begin + s.L, s.total);
}

struct Seg {
  int t, k0, k1, ft, tok0, ntok, ncols;
};

__device__ __forceinline__ void seg_decode(Seg& g, const Sched& s, int it) {
  g.t = it / s.kblocks;
  g.k0 = it - g.t * s.kblocks;
  g.k1 = min(s.kblocks, g.k0 + (s.end - it));
  g.ft = g.t / s.ttiles;
  const int tt = g.t - g.ft * s.ttiles;
  g.tok0 = tt * kGemmBNMax;
  g.ntok = min(kGemmBNMax, s.M - g.tok0);
  g.ncols = (g.ntok + 63) & ~63;
}

// bounded mbarrier wait that also gives up as soon as another role aborted
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* s_abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  const long long lim = g_wait_limit;
  while (!mbar_try_wait(bar, parity)) {
    if (*s_abort) return false;
    if (clock64() - t0 > lim) {
      report_timeout();
      *s_abort = 1;
      return false;
    }
  }
  return true;
}

// silu(g) = g / (1 + e^-g) with the fast exp and divide intrinsics: their ~1e-6
// relative error is far below the bf16 rounding the product gets next.
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

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
  uint64_t* full = bars;                  // [4] TMA -> MMA
  uint64_t* empty = bars + 4;             // [4] MMA -> TMA
  uint64_t* tfull = bars + 8;             // [2] MMA -> epilogue
  uint64_t* tempty = bars + 10;           // [2] epilogue -> MMA
  uint64_t* drain = bars + 12;            // MMA drain before TMEM release
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* s_abort = reinterpret_cast<volatile int*>(bars + 14);
  volatile int* s_epi_abort = reinterpret_cast<volatile int*>(bars + 15);
  uint64_t* fixbar = bars + 16;           // [4 warps][8] fix-up rings
  uint64_t* epi_done = bars + 48;         // epilogue warps finished with TMEM
  float* ring = reinterpret_cast<float*>(smem);
  int* s_idx = reinterpret_cast<int*>(smem + kOffIdx);
  float* stg_all = reinterpret_cast<float*>(smem + kOffStg);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Sched s;
  sched_init(s, args);
  if (s.M <= 0 || s.begin >= s.end) return;  // uniform over the CTA; nobody waits on an empty range

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGemmStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 128);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < 4 * kRing; ++i) mbar_init(&fixbar[i], 1);
    mbar_init(epi_done, 128);
    *s_abort = 0;
    *s_epi_abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, 512);
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
      uint32_t issued_parity[kGemmStages];
      bool issued[kGemmStages];
      for (int i = 0; i < kGemmStages; ++i) issued[i] = false;
      Seg g;
      for (int it = s.begin; it < s.end && !*s_abort; it += g.k1 - g.k0) {
        seg_decode(g, s, it);
        const int nbox = g.ncols >> 6;
        const uint32_t bytes = kStageA + nbox * (64 * kGemmBK * 2);
        const int yA0 = (args.epi == EPI_GU) ? g.ft * 64 : g.ft * kGemmBM;
        const int yA1 = (args.epi == EPI_GU) ? args.gu_F + g.ft * 64 : g.ft * kGemmBM + 64;
        for (int kb = g.k0; kb < g.k1; ++kb) {
          if (!wait_or_abort(&empty[stage], phase ^ 1, s_abort)) break;
          mbar_expect_tx(&full[stage], bytes);
          uint8_t* a = sA + stage * kStageA;
          uint8_t* b = sB + stage * kStageB;
          const int x = kb * kGemmBK;
          tma_load_2d(a, &tmW, x, yA0, &full[stage]);
          tma_load_2d(a + 8192, &tmW, x, yA1, &full[stage]);
          for (int j = 0; j < nbox; ++j) tma_load_2d(b + j * 8192, &tmX, x, g.tok0 + j * 64, &full[stage]);
          issued[stage] = true;
          issued_parity[stage] = phase;
          if (++stage == kGemmStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*s_abort) {
        // let every copy this thread started land before the CTA exits
        for (int i = 0; i < kGemmStages; ++i)
          if (issued[i]) (void)mbar_wait(&full[i], issued_parity[i]);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, accph = 0;
      Seg g;
      for (int it = s.begin; it < s.end && !*s_abort; it += g.k1 - g.k0) {
        seg_decode(g, s, it);
        if (!wait_or_abort(&tempty[acc], accph ^ 1, s_abort)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kTileCols);
        const uint32_t idesc = idesc_bf16(kGemmBM, g.ncols);
        bool ok = true;
        for (int kb = g.k0; kb < g.k1; ++kb) {
          if (!wait_or_abort(&full[stage], phase, s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = sdesc_sw128(smem_u32(sA + stage * kStageA));
          const uint64_t bdesc = sdesc_sw128(smem_u32(sB + stage * kStageB));
#pragma unroll
          for (int k = 0; k < kGemmBK / 16; ++k) {
            // +32 bytes of K per step, in 16-byte units of the descriptor address field
            umma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb > g.k0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == kGemmStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) accph ^= 1;
      }
      // no MMA may still be running when TMEM is released
      umma_commit(drain);
      (void)mbar_wait(drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;           // TMEM lane quarter this warp may access
    const int lr = q * 32 + lane;     // tile row = TMEM lane = feature row in tile
    const int et = threadIdx.x - 64;  // 0..127
    const int d = args.d;
    int acc = 0;
    uint32_t accph = 0;
    Seg g;
    for (int it = s.begin; it < s.end; it += g.k1 - g.k0) {
      seg_decode(g, s, it);
      const bool is_head = g.k0 == 0;
      const bool is_full = is_head && g.k1 == s.kblocks;
      named_bar_sync(1, 128);
      for (int j = et; j < g.ntok; j += 128) s_idx[j] = args.idx[g.tok0 + j];
      // The break decision must be the same in all four epilogue warps, so it is
      // taken from a flag that is only written before this barrier.
      bool bad = !wait_or_abort(&tfull[acc], accph, s_abort);
      int c_last = (int)blockIdx.x;
      if (is_head && !is_full) {
        c_last = ((g.t + 1) * s.kblocks - 1) / s.L;
        if (!bad) bad = !spin_until_geq(&args.flags[g.t], (uint32_t)(c_last - (int)blockIdx.x));
      }
      if (bad) {
        *s_epi_abort = 1;
        *s_abort = 1;
      }
      named_bar_sync(1, 128);
      if (*s_epi_abort) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t)(acc * kTileCols) + ((uint32_t)(q * 32) << 16);
      const int nchunks = g.ncols >> 5;
      // Split tile owned here: each warp streams its lane quarter of the other
      // CTAs' partials (4 KB per chunk and slot, contiguous) through its own ring
      // in the idle stage buffers; no cross-warp synchronisation is needed.
      const int nother = (is_head && !is_full) ? c_last - (int)blockIdx.x : 0;
      const int npieces = nchunks * nother;
      float* wring = ring + q * (kRing * kPieceFloats);
      uint64_t* wbar = fixbar + q * kRing;
      auto issue_piece = [&](int p) {
        const int c = p / nother, sl = (int)blockIdx.x + 1 + p % nother, b = p % kRing;
        mbar_expect_tx(&wbar[b], kPieceFloats * 4);
        bulk_load(wring + b * kPieceFloats,
                  args.partials + (size_t)sl * kSlotFloats + (size_t)q * kQuarterFloats + (size_t)c * kPieceFloats,
                  kPieceFloats * 4, &wbar[b]);
      };
      int issued_hi = 0, consumed = 0;
      if (npieces > 0 && lane == 0) {
        fence_proxy_async_global();
        issued_hi = npieces < kRing ? npieces : kRing;
        for (int p = 0; p < issued_hi; ++p) issue_piece(p);
      }
      const bool resid = is_head && (args.epi == EPI_O || args.epi == EPI_DOWN);
      const int f128 = g.ft * kGemmBM + lr;
      // residual operand (fp32 h, contiguous rows), loaded one chunk ahead so its
      // latency hides behind the previous chunk; rows past ntok are clamped to a
      // valid row and never stored
      float res[32], res_nx[32];
      auto load_res = [&](int c, float (&dst)[32]) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int jj = min(c * 32 + i, g.ntok - 1);
          dst[i] = __ldcg(&args.h32[(size_t)(g.tok0 + jj) * d + f128]);
        }
      };
      if (resid) load_res(0, res_nx);
      for (int c = 0; c < nchunks; ++c) {
        const int jb = c * 32;
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
        if (!is_head) {
          float* slot = args.partials + (size_t)blockIdx.x * kSlotFloats + (size_t)q * kQuarterFloats + jb * 32;
#pragma unroll
          for (int i = 0; i < 32; ++i) slot[i * 32 + lane] = v[i];
          continue;
        }
        for (int so = 0; so < nother; ++so) {
          const int p = c * nother + so, b = p % kRing;
          if (!*s_abort && !mbar_wait(&wbar[b], (uint32_t)((p / kRing) & 1))) *s_abort = 1;
          if (!*s_abort) {
            consumed = p + 1;
            const float* buf = wring + b * kPieceFloats;
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] += buf[i * 32 + lane];
          }
          __syncwarp();  // the whole warp is done with buffer b
          if (lane == 0 && p + kRing < npieces && !*s_abort) {
            issue_piece(p + kRing);
            issued_hi = p + kRing + 1;
          }
        }
        // Output: the warp's 32 features x 32 tokens go through its staging buffer
        // and leave token-major as 16-byte stores (64 B of each token row).
        const int nval = g.ntok - jb;  // valid tokens in this chunk (may exceed 32)
        float* stg = stg_all + q * kStgFloats;
        __nv_bfloat16* stg_h = reinterpret_cast<__nv_bfloat16*>(stg);
        const int fbase = g.ft * kGemmBM + q * 32;  // first feature of this warp
        if (args.epi == EPI_QKV || args.epi == EPI_DOWN) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            stg_h[i * 32 + lane] = f2bf(args.epi == EPI_DOWN ? res[i] + v[i] : v[i]);
          __syncwarp();
          const int part = fbase / d, col = fbase - part * d;
          __nv_bfloat16* dst = args.epi == EPI_DOWN
                                   ? (__nv_bfloat16*)args.y_cache
                                   : (part == 0 ? (__nv_bfloat16*)args.q_out
                                                : (part == 1 ? (__nv_bfloat16*)args.k_cache
                                                             : (__nv_bfloat16*)args.v_cache));
          const bool compact = args.epi == EPI_QKV && part == 0;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int tk = k * 8 + (lane >> 2);
            if (tk < nval) {
              const size_t row = compact ? (size_t)(g.tok0 + jb + tk) : (size_t)s_idx[jb + tk];
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
              *reinterpret_cast<float4*>(args.h32 + (size_t)(g.tok0 + jb + tk) * d + fbase + (lane & 7) * 4) =
                  reinterpret_cast<const float4*>(stg)[tk * 8 + (lane & 7)];
          }
          __syncwarp();
        } else {  // EPI_GU
          // gate rows are TMEM lanes 0-63 (warps q = 0, 1), up rows lanes 64-127
          // (q = 2, 3): warp q+2 parks its values in its staging buffer, warp q
          // reads them, forms silu(g) * u and stores it; two 64-thread barriers
          // per chunk and pair
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
            __nv_bfloat16* out = (__nv_bfloat16*)args.act_out + g.ft * 64 + q * 32;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int tk = k * 8 + (lane >> 2);
              if (tk < nval)
                *reinterpret_cast<uint4*>(out + (size_t)(g.tok0 + jb + tk) * F + (lane & 3) * 8) =
                    reinterpret_cast<const uint4*>(stg_h)[tk * 4 + (lane & 3)];
            }
            __syncwarp();
          }
          named_bar_sync(2 + (q & 1), 64);  // warp q+2 may refill its buffer
        }
      }
      if (lane == 0 && *s_abort) {
        // bounded wait for this warp's fix-up copies still in flight before exit
        for (int p = consumed; p < issued_hi; ++p) (void)mbar_wait(&wbar[p % kRing], (uint32_t)((p / kRing) & 1));
      }
      __syncwarp();
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      if (!is_head) {
        __threadfence();
        fence_proxy_async_global();  // the owner reads this partial with bulk copies
        named_bar_sync(1, 128);
        if (et == 0) red_release_add_u32(&args.flags[g.t], 1u);
      } else if (!is_full) {
        named_bar_sync(1, 128);
        if (et == 0) args.flags[g.t] = 0u;  // ready for the next GEMM of the step
      }
      acc ^= 1;
      if (acc == 0) accph ^= 1;
    }
    tc_fence_before();
    mbar_arrive(epi_done);  // every epilogue thread is done with TMEM
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // the epilogue warps signal their last TMEM read on their own barrier, so
    // the columns are released only after it
    (void)mbar_wait(epi_done, 0);
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
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
  gemm_tc_kernel<<<a.nslots, kGemmThreads, kSmemBytes, st>>>(tmW, tmX, a);
  return cudaPeekAtLastError() == cudaSuccess ? PLK_OK : PLK_ERR_CUDA;
}

}  // namespace plk
