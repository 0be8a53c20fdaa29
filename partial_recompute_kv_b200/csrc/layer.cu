// S4..S10: one partial-recompute layer step on the M active rows (the SureLock
// page, "Stopping Computation for Converged Tokens in Masked Diffusion-LM
// Decoding", Sec. 2 "Permanent Deactivation", "Continued Attention",
// "Algorithmic Complexity"), and the full-recompute baseline (Sec. 1).
//
// bf16 chain (10 launches, M read on the device, no host synchronisation):
//   1 gather rows idx[j] of X, RMSNorm1 -> xn, x -> h (fp32); clear the GEMMs'
//     split-tile counts
//   2 tcgen05 GEMM  xn W_qkv^T -> QKV sums (fp32; split tiles land in a fixed order)
//   3 QKV sums -> q (compact), K and V scattered into the cache rows idx[j] (bf16)
//   4 attention of the M queries over all N cached keys -> a
//   5 tcgen05 GEMM  h += a W_o^T (fp32)
//   6 RMSNorm2(h) -> hn
//   7 tcgen05 GEMM  hn [W_g; W_u]^T -> gate/up sums (fp32, fixed order as in 2)
//   8 act = silu(g) * u
//   9 tcgen05 GEMM  h += act W_down^T (fp32)
//  10 h -> Y rows idx[j] (bf16); in the whole-step call also the proxy refresh
// The layer stores bf16 only where its results land in the caller's tensors (the
// K/V cache rows and Y).  Every activation that feeds a tensor-core product (xn,
// q, a, hn, act) is held as a pair of bf16 tensors, hi = bf16(v) and
// lo = bf16(v - hi), and enters the product as hi + lo: ~16 significant bits,
// so the fp32 values between the stored tensors are not cut to bf16's 8.
// fp32 chain: the same steps with SIMT GEMMs into an fp32 scratch and
// elementwise epilogue kernels.
#include <math.h>

#include <algorithm>
#include <type_traits>

#include "plk_common.cuh"
#include "plk_internal.h"

namespace plk {

// ---------------------------------------------------------------------------
// host helpers
// ---------------------------------------------------------------------------
// events registered by plk_trace_events, recorded between the step's kernels
cudaEvent_t g_trace[16];
int g_ntrace = 0;
int g_deterministic = 0;
static inline void trace_mark(int i, cudaStream_t st) {
  if (i < g_ntrace && g_trace[i]) cudaEventRecord(g_trace[i], st);
}

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

Workspace workspace_layout(const plk_dims* dm, int num_sms) {
  Workspace w;
  const size_t Mcap = (size_t)dm->B * dm->N, d = dm->d, F = dm->F;
  const size_t es = dm->dtype == PLK_BF16 ? 2 : 4;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 1024);
    return o;
  };
  w.iota = take(4 * Mcap);
  w.seg = take(4 * ((size_t)dm->B + 1));
  const size_t lo = dm->dtype == PLK_BF16 ? 1 : 0;  // bf16: low halves of the split activations
  w.xn = take(es * Mcap * d);
  w.xn_lo = take(lo * es * Mcap * d);
  w.q = take(es * Mcap * d);
  w.q_lo = take(lo * es * Mcap * d);
  w.a = take(es * Mcap * d);
  w.a_lo = take(lo * es * Mcap * d);
  w.h32 = take(4 * Mcap * d);
  w.hn = take(es * Mcap * d);
  w.hn_lo = take(lo * es * Mcap * d);
  w.act = take(es * Mcap * F);
  w.act_lo = take(lo * es * Mcap * F);
  w.num_sms = num_sms;
  w.c32_bytes = 4 * Mcap * std::max(d + 2 * (size_t)kv_width(dm), 2 * F);
  w.c32 = take(w.c32_bytes);
  if (dm->dtype == PLK_BF16) {
    // pieces-done counts of the QKV, O, gate/up and down GEMMs: 8 per pair tile
    const size_t tt = (Mcap + kGemmBNMax - 1) / kGemmBNMax;
    w.gsync_tiles[0] = (int)(((d + 2 * (size_t)kv_width(dm)) / 256) * tt);
    w.gsync_tiles[1] = (int)((d / 256) * tt);
    w.gsync_tiles[2] = (int)((F / 128) * tt);
    w.gsync_tiles[3] = (int)((d / 256) * tt);
    w.gsync_ints = 8 * (w.gsync_tiles[0] + w.gsync_tiles[1] + w.gsync_tiles[2] + w.gsync_tiles[3]);
    w.gsync = take(4 * (size_t)w.gsync_ints);
  }
  w.total = off;
  return w;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

int make_tmap_f32(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return PLK_ERR_CUDA;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 4};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PLK_OK : PLK_ERR_CUDA;
}

int make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return PLK_ERR_CUDA;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PLK_OK : PLK_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// elementwise kernels
// ---------------------------------------------------------------------------
__device__ __forceinline__ float block_sum_f(float v, float* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  float t = (threadIdx.x < nw) ? sh[threadIdx.x] : 0.f;
  if (warp == 0) {
#pragma unroll
    for (int o = 16; o; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) sh[32] = t;
  }
  __syncthreads();
  return sh[32];
}


// out[j] = RMSNorm(src_row(j)) * g for j < M.  src_row(j) = X[idx[j]] (gather)
// or H[j] (idx == nullptr); res_out (optional) receives the fp32 source row;
// zero_ints (optional): nzero ints that the grid clears (counters and flags of
// later kernels of the step).  With a bf16 output, out receives
// hi = bf16(v) and out_lo (when given) lo = bf16(v - hi).
template <typename Tin, typename Tg, typename Tout>
__global__ void __launch_bounds__(256) rmsnorm_rows_kernel(const Tin* __restrict__ X, const int32_t* __restrict__ idx,
                                                           const int32_t* __restrict__ seg_ptr, int B,
                                                           const Tg* __restrict__ g, float eps, int d,
                                                           Tout* __restrict__ out, Tout* __restrict__ out_lo,
                                                           float* __restrict__ res_out, int* __restrict__ zero_ints,
                                                           int nzero) {
  __shared__ float sh[33];
  pdl_wait();
  pdl_trigger();
  if (zero_ints)
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nzero; i += gridDim.x * blockDim.x) zero_ints[i] = 0;
  const int M = seg_ptr[B];
  for (int j = blockIdx.x; j < M; j += gridDim.x) {  // grid-stride over the live rows (uniform per block)
  const size_t row = idx ? (size_t)idx[j] : (size_t)j;
  const Tin* x = X + row * d;
  float ss = 0.f;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    const float v = to_f(x[c]);
    ss = fmaf(v, v, ss);
    if (res_out) res_out[(size_t)j * d + c] = v;
  }
  ss = block_sum_f(ss, sh);
  const float inv = 1.0f / sqrtf(ss / (float)d + eps);
  Tout* o = out + (size_t)j * d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    const float v = to_f(x[c]) * inv * to_f(g[c]);
    const Tout hi = from_f<Tout>(v);
    o[c] = hi;
    if (out_lo) out_lo[(size_t)j * d + c] = from_f<Tout>(v - to_f(hi));
  }
  }
}

// Same as rmsnorm_rows_kernel with the row held in registers: each thread loads
// up to NV 16-byte vectors in one batch (so the loads overlap), squares and sums
// them, and writes its outputs from registers.  Requires d % (16/sizeof(Tin)) == 0
// and d <= NV * 256 * (16/sizeof(Tin)).
template <typename T>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int E = 8;
  __device__ static void unpack(const uint4& u, float* f) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = __bfloat1622float2(h[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
};
template <>
struct Vec16<float> {
  static constexpr int E = 4;
  __device__ static void unpack(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
};

// Stores E consecutive outputs with one (or two) vector stores.
template <typename T, int E>
__device__ __forceinline__ void store_vec(T* dst, const float* y);
template <>
__device__ __forceinline__ void store_vec<__nv_bfloat16, 8>(__nv_bfloat16* dst, const float* y) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(y[2 * i], y[2 * i + 1]);
  *reinterpret_cast<uint4*>(dst) = u;
}
template <>
__device__ __forceinline__ void store_vec<__nv_bfloat16, 4>(__nv_bfloat16* dst, const float* y) {
  uint2 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
  h[0] = __floats2bfloat162_rn(y[0], y[1]);
  h[1] = __floats2bfloat162_rn(y[2], y[3]);
  *reinterpret_cast<uint2*>(dst) = u;
}
template <>
__device__ __forceinline__ void store_vec<float, 4>(float* dst, const float* y) {
  *reinterpret_cast<float4*>(dst) = make_float4(y[0], y[1], y[2], y[3]);
}
template <>
__device__ __forceinline__ void store_vec<float, 8>(float* dst, const float* y) {
  reinterpret_cast<float4*>(dst)[0] = make_float4(y[0], y[1], y[2], y[3]);
  reinterpret_cast<float4*>(dst)[1] = make_float4(y[4], y[5], y[6], y[7]);
}

// The split of an activation that feeds a tensor-core product: hi = bf16(v) and
// lo = bf16(v - hi), E consecutive values each.
template <int E>
__device__ __forceinline__ void store_hilo(__nv_bfloat16* hi, __nv_bfloat16* lo, const float* y) {
  float h[E], l[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    h[e] = __bfloat162float(__float2bfloat16_rn(y[e]));
    l[e] = y[e] - h[e];  // exact in fp32
  }
  store_vec<__nv_bfloat16, E>(hi, h);  // h is already a bf16 value
  store_vec<__nv_bfloat16, E>(lo, l);
}

template <typename Tin, typename Tg, typename Tout, int NV>
__global__ void __launch_bounds__(256) rmsnorm_vec_kernel(const Tin* __restrict__ X, const int32_t* __restrict__ idx,
                                                          const int32_t* __restrict__ seg_ptr, int B, int Mcap,
                                                          const Tg* __restrict__ g, float eps, int d,
                                                          Tout* __restrict__ out, Tout* __restrict__ out_lo,
                                                          float* __restrict__ res_out, int* __restrict__ zero_ints,
                                                          int nzero) {
  constexpr int E = Vec16<Tin>::E;
  __shared__ float sh[33];
  pdl_wait();
  pdl_trigger();
  if (zero_ints)
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nzero; i += gridDim.x * blockDim.x) zero_ints[i] = 0;
  // M, the gains and the first row are loaded without waiting for one another
  const int M = seg_ptr[B];
  const int nvec = d / E;
  float gf[NV][E];
#pragma unroll
  for (int u = 0; u < NV; ++u) {
    const int vi = threadIdx.x + u * 256;
#pragma unroll
    for (int e = 0; e < E; ++e) gf[u][e] = vi < nvec ? to_f(g[vi * E + e]) : 0.f;
  }
  // Rows j < Mcap exist in idx (B*N entries) and in an un-gathered source
  // ([Mcap, d]), so their loads are issued before M is known; nothing of a row
  // j >= M is used.
  for (int j = blockIdx.x; j < Mcap; j += gridDim.x) {  // grid-stride over the rows (uniform per block)
    uint4 buf[NV];
    if (idx) {
      const size_t row = (size_t)idx[j];
      if (j >= M) return;
      const uint4* xv = reinterpret_cast<const uint4*>(X + row * d);
#pragma unroll
      for (int u = 0; u < NV; ++u) {
        const int vi = threadIdx.x + u * 256;
        if (vi < nvec) buf[u] = __ldg(xv + vi);
      }
    } else {
      const uint4* xv = reinterpret_cast<const uint4*>(X + (size_t)j * d);
#pragma unroll
      for (int u = 0; u < NV; ++u) {
        const int vi = threadIdx.x + u * 256;
        if (vi < nvec) buf[u] = __ldg(xv + vi);
      }
      if (j >= M) return;
    }
      float ss = 0.f;
#pragma unroll
    for (int u = 0; u < NV; ++u) {
      if (threadIdx.x + u * 256 < nvec) {
        float f[E];
        Vec16<Tin>::unpack(buf[u], f);
#pragma unroll
        for (int e = 0; e < E; ++e) ss = fmaf(f[e], f[e], ss);
      }
    }
    ss = block_sum_f(ss, sh);
    const float inv = 1.0f / sqrtf(ss / (float)d + eps);
    Tout* o = out + (size_t)j * d;
#pragma unroll
    for (int u = 0; u < NV; ++u) {
      const int vi = threadIdx.x + u * 256;
      if (vi < nvec) {
        float f[E];
        Vec16<Tin>::unpack(buf[u], f);
        if (res_out) store_vec<float, E>(res_out + (size_t)j * d + vi * E, f);
#pragma unroll
        for (int e = 0; e < E; ++e) f[e] = f[e] * inv * gf[u][e];
        if constexpr (std::is_same<Tout, __nv_bfloat16>::value) {
          if (out_lo) {
            store_hilo<E>(o + vi * E, out_lo + (size_t)j * d + vi * E, f);
            continue;
          }
        }
        store_vec<Tout, E>(o + vi * E, f);
      }
    }
  }
}

// Picks the register-resident kernel when the row fits, else the looping one.
template <typename Tin, typename Tg, typename Tout>
static int launch_rmsnorm(const Tin* X, const int32_t* idx, const int32_t* seg, int B, int Mcap, const Tg* g,
                          float eps, int d, Tout* out, Tout* out_lo, int grid, cudaStream_t st,
                          float* res_out = nullptr, int* zero_ints = nullptr, int nzero = 0) {
  constexpr int E = Vec16<Tin>::E;
  if (d % E == 0 && d <= 4 * 256 * E)
    return launch_pdl(rmsnorm_vec_kernel<Tin, Tg, Tout, 4>, dim3(grid), dim3(256), 0, st, X, idx, seg, B, Mcap, g,
                      eps, d, out, out_lo, res_out, zero_ints, nzero);
  return launch_pdl(rmsnorm_rows_kernel<Tin, Tg, Tout>, dim3(grid), dim3(256), 0, st, X, idx, seg, B, g, eps, d, out,
                    out_lo, res_out, zero_ints, nzero);
}

// ---------------------------------------------------------------------------
// finishing kernels of the bf16 path: the tcgen05 GEMM leaves fp32 sums; these
// apply the nonlinearity or scatter and store bf16.  One block per compact row
// (grid-stride over the M live rows), 8 features per thread and step.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

__device__ __forceinline__ void load8(const float* p, float* f) {
  const float4 a = __ldcs(reinterpret_cast<const float4*>(p));
  const float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
  f[0] = a.x, f[1] = a.y, f[2] = a.z, f[3] = a.w, f[4] = b.x, f[5] = b.y, f[6] = b.z, f[7] = b.w;
}

// Rotary position embedding: cos and sin of pos * theta^(-2i/hd) for the pair
// (x_i, x_{i+hd/2}) of a head.  The angle is formed and reduced modulo 2 pi in
// double, so that large positions keep full fp32 accuracy in sincosf.
__device__ __forceinline__ void rope_cs(int pos, int i, int hd, float log2_theta, float& c, float& s) {
  const double inv = exp2(-(2.0 * i / hd) * (double)log2_theta);
  double a = (double)pos * inv;
  const double two_pi = 6.283185307179586;
  a -= floor(a / two_pi) * two_pi;
  sincosf((float)a, &s, &c);
}

// [q | k | v] sums of compact row j (d + 2 dkv wide) -> q[j] (compact, d wide, as
// the hi/lo pair q, q_lo) and the K/V cache rows idx[j] (bf16, dkv wide: Hkv heads
// under grouped-query attention);
// with RoPE (log2_theta > 0) the heads of q and k are rotated by the row's
// position idx[j] % N
__global__ void __launch_bounds__(256) finish_qkv_kernel(const float* __restrict__ qkv32,
                                                         const int32_t* __restrict__ idx,
                                                         const int32_t* __restrict__ seg_ptr, int B, int N, int d,
                                                         int dkv, int hd, float log2_theta,
                                                         __nv_bfloat16* __restrict__ q,
                                                         __nv_bfloat16* __restrict__ q_lo,
                                                         __nv_bfloat16* __restrict__ Kc,
                                                         __nv_bfloat16* __restrict__ Vc, int* part_cnt) {
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0)  // the attention's per-unit counters (their buffer's reader, the QKV GEMM, is done)
    for (int i = threadIdx.x; i < kAttPartCounters; i += blockDim.x) part_cnt[i] = 0;
  const int M = seg_ptr[B];
  const bool rope = log2_theta > 0.f;
  const int W = d + 2 * dkv;
  const int qunits = d / 16;                        // 8 pairs (x_i, x_{i+hd/2}) per unit
  const int npair = rope ? qunits + dkv / 16 : 0;  // the q heads, then the k heads
  const int nv = W / 8;
  for (int j = blockIdx.x; j < M; j += gridDim.x) {
    const size_t row = (size_t)idx[j];
    const float* src = qkv32 + (size_t)j * W;
    if (!rope) {
      // every thread loads its (up to) 6 vectors of the row before it stores any: one round of
      // memory latency per row instead of one per vector
      constexpr int KV = 6;
      for (int base = 0; base < nv; base += KV * 256) {
        float f[KV][8];
#pragma unroll
        for (int k = 0; k < KV; ++k) {
          const int v = base + threadIdx.x + k * 256;
          if (v < nv) load8(src + v * 8, f[k]);
        }
#pragma unroll
        for (int k = 0; k < KV; ++k) {
          const int c = (base + threadIdx.x + k * 256) * 8;
          if (c >= W) continue;
          if (c < d)
            store_hilo<8>(q + (size_t)j * d + c, q_lo + (size_t)j * d + c, f[k]);
          else
            store_vec<__nv_bfloat16, 8>(c < d + dkv ? Kc + row * dkv + (c - d) : Vc + row * dkv + (c - d - dkv),
                                        f[k]);
        }
      }
      continue;
    }
    const int pos = (int)(row % (size_t)N);
    for (int u = threadIdx.x; u < npair; u += blockDim.x) {
      const bool isq = u < qunits;
      const int rem = isq ? u : u - qunits;
      const int h = rem / (hd / 16), i0 = (rem - h * (hd / 16)) * 8;
      const int c1 = h * hd + i0, c2 = c1 + hd / 2;
      const float* part = src + (isq ? 0 : d);
      float x1[8], x2[8];
      load8(part + c1, x1);
      load8(part + c2, x2);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float cs, sn;
        rope_cs(pos, i0 + e, hd, log2_theta, cs, sn);
        const float a = x1[e], b = x2[e];
        x1[e] = a * cs - b * sn;
        x2[e] = a * sn + b * cs;
      }
      if (isq) {
        store_hilo<8>(q + (size_t)j * d + c1, q_lo + (size_t)j * d + c1, x1);
        store_hilo<8>(q + (size_t)j * d + c2, q_lo + (size_t)j * d + c2, x2);
      } else {
        store_vec<__nv_bfloat16, 8>(Kc + row * dkv + c1, x1);
        store_vec<__nv_bfloat16, 8>(Kc + row * dkv + c2, x2);
      }
    }
    for (int v = threadIdx.x + (rope ? (d + dkv) / 8 : 0); v < nv; v += blockDim.x) {  // with RoPE: v only
      const int c = v * 8;
      float f[8];
      load8(src + c, f);
      if (c < d)
        store_hilo<8>(q + (size_t)j * d + c, q_lo + (size_t)j * d + c, f);
      else
        store_vec<__nv_bfloat16, 8>(c < d + dkv ? Kc + row * dkv + (c - d) : Vc + row * dkv + (c - d - dkv), f);
    }
  }
}

// [g | u] sums of compact row j -> act[j] = silu(g) * u, as the hi/lo pair act, act_lo
__global__ void __launch_bounds__(256) finish_gu_kernel(const float* __restrict__ gu32,
                                                        const int32_t* __restrict__ seg_ptr, int B, int F,
                                                        __nv_bfloat16* __restrict__ act,
                                                        __nv_bfloat16* __restrict__ act_lo) {
  pdl_wait();
  pdl_trigger();
  const int M = seg_ptr[B];
  const int nv = F / 8;
  constexpr int KV = 6;  // vectors a thread loads before it stores any (one memory latency per row)
  for (int j = blockIdx.x; j < M; j += gridDim.x) {
    const float* src = gu32 + (size_t)j * 2 * F;
    for (int base = 0; base < nv; base += KV * 256) {
      float g[KV][8], u[KV][8];
#pragma unroll
      for (int k = 0; k < KV; ++k) {
        const int v = base + threadIdx.x + k * 256;
        if (v < nv) {
          load8(src + v * 8, g[k]);
          load8(src + F + v * 8, u[k]);
        }
      }
#pragma unroll
      for (int k = 0; k < KV; ++k) {
        const int v = base + threadIdx.x + k * 256;
        if (v >= nv) continue;
#pragma unroll
        for (int e = 0; e < 8; ++e) g[k][e] = silu_f(g[k][e]) * u[k][e];
        store_hilo<8>(act + (size_t)j * F + v * 8, act_lo + (size_t)j * F + v * 8, g[k]);
      }
    }
  }
}

// residual-stream sums of compact row j -> Y cache row idx[j]; with pnew (the whole
// step's proxy refresh folded in) also pc[idx[j]] = pnew[idx[j]] (r fp32 values)
__global__ void __launch_bounds__(256) finish_y_kernel(const float* __restrict__ h32, const int32_t* __restrict__ idx,
                                                       const int32_t* __restrict__ seg_ptr, int B, int d,
                                                       __nv_bfloat16* __restrict__ Y, int r,
                                                       const float* __restrict__ pnew, float* __restrict__ pc) {
  pdl_wait();
  pdl_trigger();
  const int M = seg_ptr[B];
  const int nv = d / 8;
  constexpr int KV = 2;  // vectors a thread loads before it stores any
  for (int j = blockIdx.x; j < M; j += gridDim.x) {
    const size_t row = (size_t)idx[j];
    for (int base = 0; base < nv; base += KV * 256) {
      float f[KV][8];
#pragma unroll
      for (int k = 0; k < KV; ++k) {
        const int v = base + threadIdx.x + k * 256;
        if (v < nv) load8(h32 + (size_t)j * d + v * 8, f[k]);
      }
#pragma unroll
      for (int k = 0; k < KV; ++k) {
        const int v = base + threadIdx.x + k * 256;
        if (v < nv) store_vec<__nv_bfloat16, 8>(Y + row * d + v * 8, f[k]);
      }
    }
    if (pnew)
      for (int c = threadIdx.x; c < r; c += blockDim.x) pc[row * r + c] = pnew[row * r + c];
  }
}

__global__ void fill_identity_kernel(int32_t* iota, int32_t* seg, int B, int N) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < B * N) iota[i] = i;
  if (i <= B) seg[i] = i * N;
}

// ---- fp32 path --------------------------------------------------------------
// C[j, n] = sum_k A[j, k] W[n, k] for j < M (SIMT, 64x64 tiles)
__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* __restrict__ A, const float* __restrict__ W,
                                                       float* __restrict__ C, int Nout, int K,
                                                       const int32_t* __restrict__ seg_ptr, int B) {
  __shared__ float As[16][65], Ws[16][65];
  const int M = seg_ptr[B];
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  if (m0 >= M) return;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int e = threadIdx.x; e < 64 * 16; e += 256) {
      const int r = e >> 4, kk = e & 15;
      As[kk][r] = (m0 + r < M && k0 + kk < K) ? A[(size_t)(m0 + r) * K + k0 + kk] : 0.f;
      Ws[kk][r] = (n0 + r < Nout && k0 + kk < K) ? W[(size_t)(n0 + r) * K + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk)
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) acc[i][jj] = fmaf(As[kk][ty * 4 + i], Ws[kk][tx * 4 + jj], acc[i][jj]);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int m = m0 + ty * 4 + i, n = n0 + tx * 4 + jj;
      if (m < M && n < Nout) C[(size_t)m * Nout + n] = acc[i][jj];
    }
}

enum F32Epi { F32_QKV = 0, F32_O = 1, F32_GU = 2, F32_DOWN = 3 };

// Epilogues of the fp32 chain, one CTA per active row j.
__global__ void __launch_bounds__(256) epilogue_f32_kernel(int mode, const float* __restrict__ C,
                                                           const int32_t* __restrict__ idx,
                                                           const int32_t* __restrict__ seg_ptr, int B, int d, int F,
                                                           float* q, float* kc, float* vc, const float* x, float* h32,
                                                           float* act, float* y, int N, int hd, float log2_theta,
                                                           int dkv) {
  const int M = seg_ptr[B];
  const int j = blockIdx.x;
  if (j >= M) return;
  const size_t row = (size_t)idx[j];
  if (mode == F32_QKV) {  // [q | k | v] row of width d + 2 dkv; K/V cache rows dkv wide
    const float* c = C + (size_t)j * (d + 2 * dkv);
    if (log2_theta > 0.f) {  // RoPE on the q heads, then the k heads: pair (t, t + hd/2) of a head
      const int pos = (int)(row % (size_t)N), half = hd / 2;
      for (int u = threadIdx.x; u < (d + dkv) / 2; u += blockDim.x) {
        const bool isq = u < d / 2;
        const int uu = isq ? u : u - d / 2;
        const int h = uu / half, i = uu - h * half, t1 = h * hd + i, t2 = t1 + half;
        float cs, sn;
        rope_cs(pos, i, hd, log2_theta, cs, sn);
        const float* src = c + (isq ? 0 : d);
        float* dst = isq ? q + (size_t)j * d : kc + row * dkv;
        dst[t1] = src[t1] * cs - src[t2] * sn;
        dst[t2] = src[t1] * sn + src[t2] * cs;
      }
      for (int t = threadIdx.x; t < dkv; t += blockDim.x) vc[row * dkv + t] = c[d + dkv + t];
      return;
    }
    for (int t = threadIdx.x; t < d; t += blockDim.x) q[(size_t)j * d + t] = c[t];
    for (int t = threadIdx.x; t < dkv; t += blockDim.x) {
      kc[row * dkv + t] = c[d + t];
      vc[row * dkv + t] = c[d + dkv + t];
    }
  } else if (mode == F32_O) {
    for (int t = threadIdx.x; t < d; t += blockDim.x)
      h32[(size_t)j * d + t] = x[row * d + t] + C[(size_t)j * d + t];
  } else if (mode == F32_GU) {
    const float* c = C + (size_t)j * 2 * F;
    for (int t = threadIdx.x; t < F; t += blockDim.x) {
      const float gg = c[t];
      act[(size_t)j * F + t] = gg / (1.0f + expf(-gg)) * c[F + t];
    }
  } else {
    for (int t = threadIdx.x; t < d; t += blockDim.x)
      y[row * d + t] = h32[(size_t)j * d + t] + C[(size_t)j * d + t];
  }
}

// ---------------------------------------------------------------------------
// orchestration
// ---------------------------------------------------------------------------
#define PLK_TRY(...)                \
  do {                              \
    const int _r = (__VA_ARGS__);   \
    if (_r != PLK_OK) return _r;    \
  } while (0)
#define PLK_LAUNCHED() \
  do { if (cudaPeekAtLastError() != cudaSuccess) return PLK_ERR_CUDA; } while (0)

static int run_layer_f32(const plk_dims* dm, const plk_weights* w, const float* X, const int32_t* idx,
                         const int32_t* seg, float* Kc, float* Vc, float* Y, uint8_t* ws, const Workspace& L,
                         cudaStream_t st) {
  const int B = dm->B, d = dm->d, F = dm->F, Mcap = dm->B * dm->N, dkv = kv_width(dm);
  float* xn = (float*)(ws + L.xn);
  float* q = (float*)(ws + L.q);
  float* a = (float*)(ws + L.a);
  float* h32 = (float*)(ws + L.h32);
  float* hn = (float*)(ws + L.hn);
  float* act = (float*)(ws + L.act);
  float* c32 = (float*)(ws + L.c32);
  const dim3 rows(Mcap);
  auto gemm = [&](const float* A, const void* Wt, int Nout, int K) {
    dim3 grid(ceil_div(Nout, 64), ceil_div(Mcap, 64));
    gemm_f32_kernel<<<grid, 256, 0, st>>>(A, (const float*)Wt, c32, Nout, K, seg, B);
  };
  const int ngrid = std::min(Mcap, 2 * L.num_sms);  // row kernels: grid-stride over the M live rows
  PLK_TRY(launch_rmsnorm<float, float, float>(X, idx, seg, B, Mcap, (const float*)w->g1, dm->eps, d, xn, nullptr, ngrid,
                                              st));
  gemm(xn, w->w_qkv, d + 2 * dkv, d);
  epilogue_f32_kernel<<<rows, 256, 0, st>>>(F32_QKV, c32, idx, seg, B, d, F, q, Kc, Vc, X, h32, act, Y, dm->N,
                                            dm->hd, dm->rope_theta > 0.f ? log2f(dm->rope_theta) : 0.f, dkv);
  PLK_LAUNCHED();
  PLK_TRY(launch_attention_f32(dm, q, Kc, Vc, a, seg, Mcap, st));
  gemm(a, w->w_o, d, d);
  epilogue_f32_kernel<<<rows, 256, 0, st>>>(F32_O, c32, idx, seg, B, d, F, q, Kc, Vc, X, h32, act, Y, 0, 0, 0.f, 0);
  PLK_TRY(launch_rmsnorm<float, float, float>(h32, nullptr, seg, B, Mcap, (const float*)w->g2, dm->eps, d, hn, nullptr,
                                              ngrid, st));
  gemm(hn, w->w_gu, 2 * F, d);
  epilogue_f32_kernel<<<rows, 256, 0, st>>>(F32_GU, c32, idx, seg, B, d, F, q, Kc, Vc, X, h32, act, Y, 0, 0, 0.f, 0);
  gemm(act, w->w_down, d, F);
  epilogue_f32_kernel<<<rows, 256, 0, st>>>(F32_DOWN, c32, idx, seg, B, d, F, q, Kc, Vc, X, h32, act, Y, 0, 0, 0.f,
                                            0);
  PLK_LAUNCHED();
  return PLK_OK;
}

static int run_layer_bf16(const plk_dims* dm, const plk_weights* w, const __nv_bfloat16* X, const int32_t* idx,
                          const int32_t* seg, void* Kc, void* Vc, void* Y, uint8_t* ws, const Workspace& L,
                          cudaStream_t st, const ProxyRefresh* pr) {
  const int B = dm->B, d = dm->d, F = dm->F, Mcap = dm->B * dm->N, dkv = kv_width(dm);
  // activations that feed tensor-core products: hi/lo bf16 pairs
  __nv_bfloat16* xn = (__nv_bfloat16*)(ws + L.xn);
  __nv_bfloat16* xn_lo = (__nv_bfloat16*)(ws + L.xn_lo);
  __nv_bfloat16* q = (__nv_bfloat16*)(ws + L.q);
  __nv_bfloat16* q_lo = (__nv_bfloat16*)(ws + L.q_lo);
  __nv_bfloat16* a = (__nv_bfloat16*)(ws + L.a);
  __nv_bfloat16* a_lo = (__nv_bfloat16*)(ws + L.a_lo);
  float* h32 = (float*)(ws + L.h32);
  __nv_bfloat16* hn = (__nv_bfloat16*)(ws + L.hn);
  __nv_bfloat16* hn_lo = (__nv_bfloat16*)(ws + L.hn_lo);
  __nv_bfloat16* act = (__nv_bfloat16*)(ws + L.act);
  __nv_bfloat16* act_lo = (__nv_bfloat16*)(ws + L.act_lo);

  float* c32 = (float*)(ws + L.c32);  // [Mcap, d + 2 dkv] QKV sums, later [Mcap, 2F] gate/up sums

  CUtensorMap tW_qkv, tW_o, tW_gu, tW_down, tO_qkv, tO_h, tO_gu;
  CUtensorMap tX_xn[2], tX_a[2], tX_hn[2], tX_act[2];  // {hi, lo}
  PLK_TRY(make_tmap_bf16(&tW_qkv, w->w_qkv, (uint64_t)d + 2ull * dkv, d, 64));
  PLK_TRY(make_tmap_bf16(&tW_o, w->w_o, (uint64_t)d, d, 64));
  PLK_TRY(make_tmap_bf16(&tW_gu, w->w_gu, 2ull * F, d, 64));
  PLK_TRY(make_tmap_bf16(&tW_down, w->w_down, (uint64_t)d, F, 64));
  PLK_TRY(make_tmap_bf16(&tX_xn[0], xn, (uint64_t)Mcap, d, 64));
  PLK_TRY(make_tmap_bf16(&tX_xn[1], xn_lo, (uint64_t)Mcap, d, 64));
  PLK_TRY(make_tmap_bf16(&tX_a[0], a, (uint64_t)Mcap, d, 64));
  PLK_TRY(make_tmap_bf16(&tX_a[1], a_lo, (uint64_t)Mcap, d, 64));
  PLK_TRY(make_tmap_bf16(&tX_hn[0], hn, (uint64_t)Mcap, d, 64));
  PLK_TRY(make_tmap_bf16(&tX_hn[1], hn_lo, (uint64_t)Mcap, d, 64));
  PLK_TRY(make_tmap_bf16(&tX_act[0], act, (uint64_t)Mcap, F, 64));
  PLK_TRY(make_tmap_bf16(&tX_act[1], act_lo, (uint64_t)Mcap, F, 64));
  PLK_TRY(make_tmap_f32(&tO_qkv, c32, (uint64_t)Mcap, (uint64_t)d + 2ull * dkv));
  PLK_TRY(make_tmap_f32(&tO_h, h32, (uint64_t)Mcap, d));
  PLK_TRY(make_tmap_f32(&tO_gu, c32, (uint64_t)Mcap, 2ull * F));

  GemmArgs g{};
  g.seg_ptr = seg;
  g.B = B;
  g.num_sms = L.num_sms;
  const int rgrid = std::min(Mcap, 2 * L.num_sms);  // finishing kernels: grid-stride over M rows

  // in the QKV and gate/up GEMMs the pieces of a split tile land in a fixed order, counted per
  // (tile, CTA, warp), and their sums need no zeroing: the last k range's piece stores, the
  // others add
  int* gsync = (int*)(ws + L.gsync);
  uint32_t* done_qkv = (uint32_t*)gsync;
  uint32_t* done_o = done_qkv + 8 * L.gsync_tiles[0];
  uint32_t* done_gu = done_o + 8 * L.gsync_tiles[1];
  uint32_t* done_down = done_gu + 8 * L.gsync_tiles[2];

  trace_mark(0, st);
  // x (fp32) staged in h32 takes the O projection's adds; the GEMMs' pieces-done counts start at 0
  PLK_TRY(launch_rmsnorm<__nv_bfloat16, __nv_bfloat16, __nv_bfloat16>(X, idx, seg, B, Mcap, (const __nv_bfloat16*)w->g1,
                                                                      dm->eps, d, xn, xn_lo, rgrid, st, h32,
                                                                      gsync, L.gsync_ints));
  trace_mark(1, st);

  g.K = d;
  g.ftiles = (d + 2 * dkv) / kGemmBM;
  g.gu_F = 0;
  g.done = done_qkv;
  g.store_first = 1;
  PLK_TRY(launch_gemm_tc(tW_qkv, tX_xn[0], tX_xn[1], tO_qkv, g, st));
  trace_mark(2, st);

  const float log2_theta = dm->rope_theta > 0.f ? log2f(dm->rope_theta) : 0.f;
  int* part_cnt = (int*)(ws + L.xn);  // RMSNorm1's output, consumed by the QKV GEMM
  PLK_TRY(launch_pdl(finish_qkv_kernel, dim3(rgrid), dim3(256), 0, st, (const float*)c32, idx, seg, B, dm->N, d,
                     dkv, dm->hd, log2_theta, q, q_lo, (__nv_bfloat16*)Kc, (__nv_bfloat16*)Vc, part_cnt));
  trace_mark(3, st);

  // the QKV sums are consumed: c32 holds the attention's partial outputs until the gate/up GEMM
  PLK_TRY(launch_attention_bf16(dm, q, q_lo, Kc, Vc, a, a_lo, seg, L.num_sms, c32, L.c32_bytes, part_cnt, st));
  trace_mark(4, st);

  g.K = d;
  g.ftiles = d / kGemmBM;
  // h = x + a W_o^T: 16 tiles split 5-6 ways at 256 rows, where an ordered chain of their
  // pieces costs ~18 us; the pieces add in the order they arrive unless reproducible mode is on
  g.done = g_deterministic ? done_o : nullptr;
  g.store_first = 0;
  PLK_TRY(launch_gemm_tc(tW_o, tX_a[0], tX_a[1], tO_h, g, st));
  trace_mark(5, st);

  PLK_TRY(launch_rmsnorm<float, __nv_bfloat16, __nv_bfloat16>(h32, nullptr, seg, B, Mcap, (const __nv_bfloat16*)w->g2,
                                                              dm->eps, d, hn, hn_lo, rgrid, st));
  trace_mark(6, st);

  g.K = d;
  g.ftiles = F / 64;
  g.gu_F = F;
  g.done = done_gu;
  g.store_first = 1;
  PLK_TRY(launch_gemm_tc(tW_gu, tX_hn[0], tX_hn[1], tO_gu, g, st));
  trace_mark(7, st);

  PLK_TRY(launch_pdl(finish_gu_kernel, dim3(rgrid), dim3(256), 0, st, (const float*)c32, seg, B, F, act, act_lo));
  trace_mark(8, st);

  g.K = F;
  g.ftiles = d / kGemmBM;
  g.gu_F = 0;
  g.done = g_deterministic ? done_down : nullptr;  // y = h + act W_down^T, as for O
  g.store_first = 0;
  PLK_TRY(launch_gemm_tc(tW_down, tX_act[0], tX_act[1], tO_h, g, st));
  trace_mark(9, st);

  PLK_TRY(launch_pdl(finish_y_kernel, dim3(rgrid), dim3(256), 0, st, (const float*)h32, idx, seg, B, d,
                     (__nv_bfloat16*)Y, pr ? pr->r : 0, pr ? pr->proxy_new : nullptr,
                     pr ? pr->proxy_cache : nullptr));
  trace_mark(10, st);
  return PLK_OK;
}

int run_layer(const plk_dims* dm, const plk_weights* w, const void* X, const int32_t* idx, const int32_t* seg_ptr,
              bool full, void* Kc, void* Vc, void* Y, void* ws, size_t ws_bytes, cudaStream_t st,
              const ProxyRefresh* pr) {
  const int nsm = device_sm_count();
  if (nsm <= 0) return PLK_ERR_CUDA;
  const Workspace L = workspace_layout(dm, nsm);
  if (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return PLK_ERR_WORKSPACE;
  uint8_t* wsb = (uint8_t*)ws;
  if (full) {
    int32_t* iota = (int32_t*)(wsb + L.iota);
    int32_t* seg = (int32_t*)(wsb + L.seg);
    const int n = dm->B * dm->N + 1;
    fill_identity_kernel<<<ceil_div(n, 256), 256, 0, st>>>(iota, seg, dm->B, dm->N);
    PLK_LAUNCHED();
    idx = iota;
    seg_ptr = seg;
  }
  if (dm->dtype == PLK_F32) {
    PLK_TRY(run_layer_f32(dm, w, (const float*)X, idx, seg_ptr, (float*)Kc, (float*)Vc, (float*)Y, wsb, L, st));
    if (pr) return launch_proxy_commit(dm, pr->r, idx, seg_ptr, pr->proxy_new, pr->proxy_cache, st);
    return PLK_OK;
  }
  return run_layer_bf16(dm, w, (const __nv_bfloat16*)X, idx, seg_ptr, Kc, Vc, Y, wsb, L, st, pr);
}

}  // namespace plk
