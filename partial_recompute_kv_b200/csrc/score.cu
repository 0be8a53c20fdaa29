// S1: drift score on the singular proxy (the SPA-Cache page, "SPA-Cache:
// Singular Proxies for Adaptive Caching in Diffusion Language Models", part 1:
// compare a low-dimensional snapshot instead of the full hidden state; the
// Polestar page uses the same drift signal to pick rows to refresh).
//
//   p_i = Ut x_i (rank r),  score_i = cos(p_i, c_i)  or  |p_i - c_i|
//
// bf16: one CTA per 128 rows, X tile (128 x 64) and Ut tile (r x 64) staged by
// TMA, tcgen05.mma into an fp32 TMEM accumulator of r columns, and the row-wise
// distance computed straight from TMEM (thread = row) against the cached proxy.
// The kernel streams X once from HBM; Ut stays in L2.  When there are too few
// 128-row tiles to fill the GPU, the K dimension is split over a thread-block
// cluster of S CTAs: once every CTA's loads and MMAs are done (a cluster
// barrier), each CTA stages its partial projection in its own shared memory and
// moves each 128/S-row slice with one bulk copy into the idle stage buffers of
// the CTA that finishes those rows (the copies complete on that CTA's
// mbarrier); every CTA then sums its S slices locally (no global scratch, no
// remote loads, no thread-issued remote stores).  When there are more 128-row tiles
// than SMs, two CTAs share each SM with half the stage ring each, so that every tile
// runs in the first wave.
// fp32: a SIMT kernel, one warp per row.
#include "plk_common.cuh"
#include "plk_internal.h"

namespace plk {

namespace {
constexpr int kScStagesMax = 6;
constexpr int kScA = 128 * 64 * 2;  // 16 KB of X per stage
constexpr int kScRingBudget = 200 * 1024;

// Ring depth for proxy rank r: as many (X, U) stages as fit 200 KB, 2..6.  The
// X loads are HBM-latency bound, so the more stages in flight the better.
inline int sc_stages(int r) {
  const int stage_bytes = kScA + ((r * 128 + 1023) & ~1023);
  const int n = kScRingBudget / stage_bytes;
  return n < 2 ? 2 : (n > kScStagesMax ? kScStagesMax : n);
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
}  // namespace

__global__ void __launch_bounds__(128) score_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                                                       const __grid_constant__ CUtensorMap tmU, int rows, int d,
                                                       int r, int tmem_cols, const float* __restrict__ cache,
                                                       float* __restrict__ pout, float* __restrict__ score,
                                                       int metric, int stages, int x_stream) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const int stageB = r * 128;
  const int stage_bytes = kScA + ((stageB + 1023) & ~1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + stages * stage_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kScStagesMax;
  uint64_t* done = bars + 2 * kScStagesMax;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2 * kScStagesMax + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(bars + 2 * kScStagesMax + 2);
  uint64_t* slices = bars + 2 * kScStagesMax + 3;  // split-K: the S row slices of my rows have landed

  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * 128;
  const int S = gridDim.y, ks = blockIdx.y;  // K slices = cluster size (1 = no cluster)
  const int nkb_all = d / 64;
  const int kb0 = ks * nkb_all / S;
  const int nkb = (ks + 1) * nkb_all / S - kb0;
  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(done, 1);
    mbar_init(slices, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(s_tmem, (uint32_t)tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (S == 1 && warp == 3 && lane == 0) {
    // the cached proxies of this tile's rows, read by the epilogue: into L2 while X streams
    const int nrows = min(128, rows - row0);
    const char* src = reinterpret_cast<const char*>(cache + (size_t)row0 * r);
    for (uint32_t off = 0, bytes = (uint32_t)(nrows * r * 4); off < bytes; off += 16384u)
      bulk_prefetch_l2(src + off, min(16384u, bytes - off));
  }
  if (warp == 0) {
    if (elect_one()) {
      // X larger than the L2 is read once: evict first, so that the proxies and Ut stay
      const uint64_t pol_x = x_stream ? l2_policy_evict_first() : l2_policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1)) {
          *s_abort = 1;
          break;
        }
        uint8_t* a = smem + stage * stage_bytes;
        mbar_expect_tx(&full[stage], (uint32_t)(kScA + stageB));
        tma_load_2d_hint(a, &tmX, (kb0 + kb) * 64, row0, &full[stage], pol_x);
        tma_load_2d(a + kScA, &tmU, (kb0 + kb) * 64, 0, &full[stage]);
        ++issued;
        if (++stage == stages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (*s_abort) {  // let started copies land before exit
        for (int i = 0; i < stages && i < issued; ++i) {
          const int kb = issued - 1 - i;
          (void)mbar_wait(&full[kb % stages], (uint32_t)((kb / stages) & 1));
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t idesc = idesc_bf16(128, r);
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait(&full[stage], phase)) {
          *s_abort = 1;
          break;
        }
        tc_fence_after();
        uint8_t* a = smem + stage * stage_bytes;
        const uint64_t adesc = sdesc_sw128(smem_u32(a));
        const uint64_t bdesc = sdesc_sw128(smem_u32(a + kScA));
#pragma unroll
        for (int k = 0; k < 4; ++k) umma_bf16(tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) ? 1u : 0u);
        umma_commit(&empty[stage]);
        if (++stage == stages) {
          stage = 0;
          phase ^= 1;
        }
      }
      umma_commit(done);  // also the drain: arrives when every MMA above is complete
    }
    __syncwarp();
  }

  const bool ok = mbar_wait(done, 0);
  tc_fence_after();
  if (S > 1) {
    // split-K over the cluster.  Layout of a row block of r fp32 values: 16-byte chunk c of row
    // k sits at chunk c ^ (k & 7) of the row (c ^ (k & 3) when r / 4 is not a multiple of 8), so
    // a warp's 32 rows spread over the banks.  Each CTA
    // stages its whole partial [128 rows][r] in its own stage buffers, then one thread sends
    // slice q (rows q * rows_per ..) with one bulk copy to slot [ks] of CTA q; CTA q's slice
    // barrier counts the S copies' bytes.
    const int rows_per = 128 / S, tpr = 128 / rows_per;
    const int nch = r / 4;                                   // 16-byte chunks per row
    const int swz = (nch % 8 == 0) ? 7 : 3;                  // XOR key mask: stays inside the row
    float4* stage = reinterpret_cast<float4*>(smem);         // [128][nch] my partial (sender side)
    float* slots = reinterpret_cast<float*>(smem + (size_t)128 * r * 4);  // [S][rows_per][r] (receiver)
    const int rl = warp * 32 + lane;
    const bool good = __all_sync(0xffffffffu, ok && !*s_abort);
    if (good) {
      for (int c0 = 0; c0 < r; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 4; ++u)
          stage[rl * nch + ((c0 / 4 + u) ^ (rl & swz))] =
              make_float4(__uint_as_float(v[4 * u]), __uint_as_float(v[4 * u + 1]), __uint_as_float(v[4 * u + 2]),
                          __uint_as_float(v[4 * u + 3]));
      }
    } else {
      for (int c = 0; c < nch; ++c) stage[rl * nch + c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    fence_proxy_async_smem();  // the bulk copies read the staged partial through the async proxy
    if (threadIdx.x == 0) mbar_expect_tx(slices, (uint32_t)(S * rows_per * r * 4));
    // the receivers' slot buffers (behind their staged partials) are idle and armed: every
    // CTA's loads and MMAs are done and every CTA has staged its partial
    cluster_sync_all();
    if (threadIdx.x == 0) {
      for (int q = 0; q < S; ++q)
        asm volatile(
            "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                dsmem_addr(smem_u32(slots + (size_t)ks * rows_per * r), (uint32_t)q)),
            "r"(smem_u32(stage + (size_t)q * rows_per * nch)), "r"((uint32_t)(rows_per * r * 4)),
            "r"(dsmem_addr(smem_u32(slices), (uint32_t)q))
            : "memory");
    }
    const int lrow = (int)threadIdx.x / tpr, sub = (int)threadIdx.x % tpr;
    const int row = row0 + ks * rows_per + lrow;
    const int krow = ks * rows_per + lrow;  // the row's index in its sender's block (swizzle key)
    // the cached proxies of this thread's first 4 column groups, loaded while the slices travel
    float4 cpre[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = sub * 4 + i * 4 * tpr;
      cpre[i] = (c < r && row < rows) ? __ldg(reinterpret_cast<const float4*>(cache + (size_t)row * r + c))
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const bool landed = mbar_wait(slices, 0);
    float dot = 0.f, pp = 0.f, cc = 0.f, dd = 0.f;
    int ci = 0;
    for (int c = sub * 4; c < r && landed; c += 4 * tpr, ++ci) {
      float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int sr = 0; sr < S; ++sr) {
        const float4 x = reinterpret_cast<const float4*>(slots + ((size_t)sr * rows_per + lrow) * r)[(c / 4) ^ (krow & swz)];
        p.x += x.x;
        p.y += x.y;
        p.z += x.z;
        p.w += x.w;
      }
      if (row < rows) {
        const float4 cv = ci == 0   ? cpre[0]
                          : ci == 1 ? cpre[1]
                          : ci == 2 ? cpre[2]
                          : ci == 3 ? cpre[3]
                                    : __ldg(reinterpret_cast<const float4*>(cache + (size_t)row * r + c));
        const float pv[4] = {p.x, p.y, p.z, p.w};
        const float cvv[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          dot = fmaf(pv[e], cvv[e], dot);
          pp = fmaf(pv[e], pv[e], pp);
          cc = fmaf(cvv[e], cvv[e], cc);
          dd = fmaf(pv[e] - cvv[e], pv[e] - cvv[e], dd);
        }
        if (pout) *reinterpret_cast<float4*>(pout + (size_t)row * r + c) = p;
      }
    }
    for (int o = 1; o < tpr; o <<= 1) {
      dot += __shfl_xor_sync(0xffffffffu, dot, o);
      pp += __shfl_xor_sync(0xffffffffu, pp, o);
      cc += __shfl_xor_sync(0xffffffffu, cc, o);
      dd += __shfl_xor_sync(0xffffffffu, dd, o);
    }
    if (sub == 0 && row < rows && landed)
      score[row] = metric == PLK_METRIC_COS ? dot / fmaxf(sqrtf(pp) * sqrtf(cc), 1e-30f) : sqrtf(dd);
    tc_fence_before();
    cluster_sync_all();  // every copy has landed, so every source was read: CTAs may leave
    if (warp == 2) {
      tc_fence_after();
      tmem_dealloc(tmem, (uint32_t)tmem_cols);
    }
    return;
  }
  // epilogue: thread = row (TMEM lane)
  const int row = row0 + warp * 32 + lane;
  float dot = 0.f, pp = 0.f, cc = 0.f, dd = 0.f;
  // tcgen05.ld is warp-collective: take the decision once per warp
  if (__all_sync(0xffffffffu, ok && !*s_abort)) {
    for (int c0 = 0; c0 < r; c0 += 16) {
      uint32_t v[16];
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
      tmem_ld_wait();
      if (row < rows) {
        const float4* cp = reinterpret_cast<const float4*>(cache + (size_t)row * r + c0);
        float cv[16];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float4 t = __ldg(cp + u);
          cv[4 * u] = t.x;
          cv[4 * u + 1] = t.y;
          cv[4 * u + 2] = t.z;
          cv[4 * u + 3] = t.w;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p = __uint_as_float(v[i]);
          dot = fmaf(p, cv[i], dot);
          pp = fmaf(p, p, pp);
          cc = fmaf(cv[i], cv[i], cc);
          const float df = p - cv[i];
          dd = fmaf(df, df, dd);
        }
        if (pout) {
          float4* op = reinterpret_cast<float4*>(pout + (size_t)row * r + c0);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            op[u] = make_float4(__uint_as_float(v[4 * u]), __uint_as_float(v[4 * u + 1]),
                                __uint_as_float(v[4 * u + 2]), __uint_as_float(v[4 * u + 3]));
        }
      }
    }
    if (row < rows) {
      score[row] = metric == PLK_METRIC_COS ? dot / fmaxf(sqrtf(pp) * sqrtf(cc), 1e-30f) : sqrtf(dd);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, (uint32_t)tmem_cols);
  }
}

__global__ void __launch_bounds__(256) score_f32_kernel(const float* __restrict__ X, const float* __restrict__ Ut,
                                                        int rows, int d, int r, const float* __restrict__ cache,
                                                        float* __restrict__ pout, float* __restrict__ score,
                                                        int metric) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float* x = X + (size_t)row * d;
  float dot = 0.f, pp = 0.f, cc = 0.f, dd = 0.f;
  for (int c = 0; c < r; ++c) {
    float s = 0.f;
    for (int k = lane; k < d; k += 32) s = fmaf(x[k], Ut[(size_t)c * d + k], s);
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float cv = cache[(size_t)row * r + c];
    dot = fmaf(s, cv, dot);
    pp = fmaf(s, s, pp);
    cc = fmaf(cv, cv, cc);
    dd = fmaf(s - cv, s - cv, dd);
    if (pout && lane == 0) pout[(size_t)row * r + c] = s;
  }
  if (lane == 0) score[row] = metric == PLK_METRIC_COS ? dot / fmaxf(sqrtf(pp) * sqrtf(cc), 1e-30f) : sqrtf(dd);
}

// One warp per compact row j: idx has B*N entries, so idx[j] is loaded beside
// M = seg_ptr[B]; the row's r <= 256 values are all loaded before any store.
__global__ void proxy_commit_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ seg_ptr, int B,
                                    int rows, int r, const float* __restrict__ pnew, float* __restrict__ pc) {
  pdl_wait();
  pdl_trigger();
  const int j = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (j >= rows) return;
  const int M = seg_ptr[B];
  const size_t row = (size_t)idx[j];
  if (j >= M) return;
  const int lane = threadIdx.x & 31;
  float v[8];
#pragma unroll
  for (int u = 0; u < 8; ++u)
    if (lane + u * 32 < r) v[u] = pnew[row * r + lane + u * 32];
#pragma unroll
  for (int u = 0; u < 8; ++u)
    if (lane + u * 32 < r) pc[row * r + lane + u * 32] = v[u];
}

static int score_tc_smem(int r, int stages) {
  const int stage_bytes = kScA + ((r * 128 + 1023) & ~1023);
  return stages * stage_bytes + 128 + 1024;
}

// Dynamic shared memory one CTA may take so that two CTAs share an SM (per device, cached).
static int score_tc_half_sm_smem() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  int per_sm = 0, reserved = 0;
  if (cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
    return 0;
  const int v = per_sm / 2 - reserved;
  if (dev < 64) cached[dev] = v;
  return v;
}

int launch_score(const plk_dims* dims, const void* X, const void* Ut, int r, const float* proxy_cache,
                 int metric, float* proxy_out, float* score_out, cudaStream_t st) {
  const int rows = dims->B * dims->N, d = dims->d;
  if (dims->dtype == PLK_F32) {
    score_f32_kernel<<<ceil_div(rows, 8), 256, 0, st>>>((const float*)X, (const float*)Ut, rows, d, r,
                                                         proxy_cache, proxy_out, score_out, metric);
    return cudaPeekAtLastError() == cudaSuccess ? PLK_OK : PLK_ERR_CUDA;
  }
  CUtensorMap tmX, tmU;
  if (make_tmap_bf16(&tmX, X, (uint64_t)rows, (uint64_t)d, 128) != PLK_OK) return PLK_ERR_CUDA;
  if (make_tmap_bf16(&tmU, Ut, (uint64_t)r, (uint64_t)d, (uint32_t)r) != PLK_OK) return PLK_ERR_CUDA;
  int tcols = 32;
  while (tcols < r) tcols <<= 1;
  const int smem_max = score_tc_smem(r, sc_stages(r));
  static int attr_smem[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PLK_ERR_CUDA;
  if (dev < 64 && attr_smem[dev] < smem_max) {
    if (cudaFuncSetAttribute(score_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_max) != cudaSuccess)
      return PLK_ERR_CUDA;
    attr_smem[dev] = smem_max;
  }
  // K slices: grow the cluster while it still fits the GPU and leaves >= 2 k-blocks per slice.
  // The split needs the staged partial and the received slices ([128][r] fp32 each) inside the
  // stage ring: at r = 256 the ring is too small, and the kernel runs unsplit.
  const int tiles = ceil_div(rows, 128), nkb = d / 64, sms = device_sm_count();
  const int stage_bytes = kScA + ((r * 128 + 1023) & ~1023);
  int stages = sc_stages(r);
  const int ring = stages * stage_bytes;
  int S = 1;
  while (S < 8 && tiles * S * 2 <= sms && nkb % (S * 2) == 0 && nkb / (S * 2) >= 2 && 2 * 128 * r * 4 <= ring)
    S *= 2;
  // More row tiles than SMs: with one CTA per SM the tiles past the first wave run in a second,
  // partly idle one.  Two CTAs per SM with half the ring each keep as many X loads in flight
  // per SM and take every tile (up to two per SM) in one wave.
  if (S == 1 && tiles > sms) {
    const int fit = (score_tc_half_sm_smem() - 128 - 1024) / stage_bytes;
    if (fit >= 2 && fit < stages) stages = fit;
  }
  const int smem = score_tc_smem(r, stages);
  const int x_stream = (size_t)rows * d * 2 > ((size_t)64 << 20);  // more than half of the 126 MB L2
  if (S == 1) {
    return launch_pdl(score_tc_kernel, dim3(tiles), dim3(128), smem, st, tmX, tmU, rows, d, r, tcols, proxy_cache,
                      proxy_out, score_out, metric, stages, x_stream);
  } else {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(tiles, S, 1);
    cfg.blockDim = dim3(128, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 1;
    at[0].val.clusterDim.y = S;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, score_tc_kernel, tmX, tmU, rows, d, r, tcols, proxy_cache, proxy_out, score_out,
                           metric, stages, x_stream) != cudaSuccess)
      return PLK_ERR_CUDA;
  }
  return cudaPeekAtLastError() == cudaSuccess ? PLK_OK : PLK_ERR_CUDA;
}

int launch_proxy_commit(const plk_dims* dims, int r, const int32_t* idx, const int32_t* seg_ptr,
                        const float* proxy_new, float* proxy_cache, cudaStream_t st) {
  const int rows = dims->B * dims->N;
  return launch_pdl(proxy_commit_kernel, dim3(ceil_div(rows, 8)), dim3(256), 0, st, idx, seg_ptr, dims->B, rows, r,
                    proxy_new, proxy_cache);
}

}  // namespace plk
