// SureLock's locking condition on caller-supplied logits (the SureLock page,
// "Stopping Computation for Converged Tokens in Masked Diffusion-LM Decoding",
// Sec. 2 "Locking Condition"): a still-active position locks at step t when
// KL(p_t || p_{t-1}) <= eps, p = softmax of the position's vocabulary logits,
// and, with the optional confidence gate, when its entropy H(p_t) <= h_max.
//
// One CTA per row that is still active (locked rows exit at once); the row's V
// logits of both steps stream through 16-byte loads, four chunks in flight per
// thread.  Each thread keeps base-2 online sums with running maxima m_t, m_p:
//   s_t = sum 2^(y_t - m_t),  a = sum 2^(y_t - m_t) (z_t - z_p),
//   e   = sum 2^(y_t - m_t) z_t,  s_p = sum 2^(y_p - m_p),
//   u   = sum (2^(y_t - m_p) - 2^(y_p - m_p))          (y = z log2 e)
// and a block reduction merges them.  Then
//   KL = a / s_t - ln(1 + u / s_p),   H = (m_t ln 2 + ln s_t) - e / s_t.
// ln(1 + u / s_p) is ln E_q[e^(z_t - z_p)] = lse_t - lse_p without the
// cancellation of two large log-sum-exps, which keeps the small KL values near a
// locking threshold accurate in fp32; when some z_t is so far above max z_p that
// the u form would overflow, the plain difference of log-sum-exps is used.
// Two exp2 per element (ex2.approx; the third factor 2^(m_t - m_p) is one per
// chunk) keep the MUFU pipe near the time of the HBM stream of the two rows.
// Measured alternatives: a 4-CTA cluster per row and a shared-memory ring of
// bulk copies were both slower (the row's dependent instruction stream, not the
// memory system, sets the pace).
#include <math.h>

#include "plk_common.cuh"
#include "plk_internal.h"

namespace plk {

namespace {
constexpr int kKlThreads = 512;
constexpr int kKlUnroll = 4;  // 16-byte chunks of each tensor in flight per thread
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kKlFar = 64.f;  // log2 range of 2^(y_t - m_p) kept by the u form

struct KlAcc {
  float mt, st, a, e;  // current step: max y_t, sums
  float mp, sp, u;     // previous step: max y_p, sums
  int far;             // some y_t - m_p > kKlFar
};

// 2^x on the MUFU pipe (PTX ex2.approx: ~2 ulp, flushes results below 2^-126 to 0)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void kl_init(KlAcc& c) {
  c.mt = -INFINITY, c.st = 0.f, c.a = 0.f, c.e = 0.f;
  c.mp = -INFINITY, c.sp = 0.f, c.u = 0.f;
  c.far = 0;
}

// adds n logit pairs (n <= 8) to the sums, rescaling once per chunk
template <int n>
__device__ __forceinline__ void kl_add(KlAcc& c, const float (&zt)[8], const float (&zp)[8]) {
  float cmt = -INFINITY, cmp = -INFINITY;
#pragma unroll
  for (int k = 0; k < n; ++k) {
    cmt = fmaxf(cmt, zt[k]);
    cmp = fmaxf(cmp, zp[k]);
  }
  cmt *= kLog2e;
  cmp *= kLog2e;
  if (cmt > c.mt) {
    const float f = exp2f(c.mt - cmt);
    c.st *= f, c.a *= f, c.e *= f;
    c.mt = cmt;
  }
  if (cmp > c.mp) {
    const float f = exp2f(c.mp - cmp);
    c.sp *= f, c.u *= f;
    c.mp = cmp;
  }
  // 2^(y_t - m_p) = 2^(y_t - m_t) 2^(m_t - m_p): one exp2 per chunk instead of per element
  const float cexp = c.mt - c.mp;
  c.far |= cexp > kKlFar;
  const float scale = ex2(fminf(cexp, kKlFar));
#pragma unroll
  for (int k = 0; k < n; ++k) {
    const float wt = ex2(fmaf(zt[k], kLog2e, -c.mt)), wp = ex2(fmaf(zp[k], kLog2e, -c.mp));
    c.st += wt;
    c.sp += wp;
    c.a = fmaf(wt, zt[k] - zp[k], c.a);
    c.e = fmaf(wt, zt[k], c.e);
    c.u += fmaf(wt, scale, -wp);
  }
}

__device__ __forceinline__ void kl_merge(KlAcc& c, const KlAcc& o) {
  if (o.mt > -INFINITY) {
    const float m = fmaxf(c.mt, o.mt);
    const float f = exp2f(c.mt - m), g = exp2f(o.mt - m);
    c.st = c.st * f + o.st * g;
    c.a = c.a * f + o.a * g;
    c.e = c.e * f + o.e * g;
    c.mt = m;
  }
  if (o.mp > -INFINITY) {
    const float m = fmaxf(c.mp, o.mp);
    const float f = exp2f(c.mp - m), g = exp2f(o.mp - m);
    c.sp = c.sp * f + o.sp * g;
    c.u = c.u * f + o.u * g;
    c.mp = m;
  }
  c.far |= o.far;
}

__device__ __forceinline__ KlAcc kl_shfl(const KlAcc& c, int o) {
  KlAcc r;
  r.mt = __shfl_xor_sync(0xffffffffu, c.mt, o);
  r.st = __shfl_xor_sync(0xffffffffu, c.st, o);
  r.a = __shfl_xor_sync(0xffffffffu, c.a, o);
  r.e = __shfl_xor_sync(0xffffffffu, c.e, o);
  r.mp = __shfl_xor_sync(0xffffffffu, c.mp, o);
  r.sp = __shfl_xor_sync(0xffffffffu, c.sp, o);
  r.u = __shfl_xor_sync(0xffffffffu, c.u, o);
  r.far = __shfl_xor_sync(0xffffffffu, c.far, o);
  return r;
}

template <typename T>
struct KlLoad;
template <>
struct KlLoad<__nv_bfloat16> {
  static constexpr int E = 8;  // elements per 16 bytes
  __device__ static void unpack(const uint4& v, float (&f)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = __bfloat1622float2(h[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
};
template <>
struct KlLoad<float> {
  static constexpr int E = 4;
  __device__ static void unpack(const uint4& v, float (&f)[8]) {
    f[0] = __uint_as_float(v.x), f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z), f[3] = __uint_as_float(v.w);
  }
};
}  // namespace

template <typename T>
__global__ void __launch_bounds__(kKlThreads) kl_lock_kernel(const T* __restrict__ zt_all, const T* __restrict__ zp_all,
                                                            long long rows, int V, const uint8_t* lock_in,
                                                            uint8_t* lock_out, float eps, float h_max,
                                                            float* __restrict__ kl_out, float* __restrict__ h_out) {
  constexpr int E = KlLoad<T>::E;
  __shared__ KlAcc sh[kKlThreads / 32];
  pdl_wait();
  pdl_trigger();
  const long long row = blockIdx.x;
  if (row >= rows) return;
  if (lock_in[row]) {  // not examined, stays locked (lock_in and lock_out may alias)
    if (threadIdx.x == 0) lock_out[row] = 1;
    return;
  }
  const T* zt = zt_all + row * V;
  const T* zp = zp_all + row * V;
  KlAcc c;
  kl_init(c);
  float ft[8], fp[8];
  const bool vec = (V % E == 0) && ((reinterpret_cast<uintptr_t>(zt) | reinterpret_cast<uintptr_t>(zp)) % 16 == 0);
  int done = 0;
  if (vec) {
    const uint4* vt = reinterpret_cast<const uint4*>(zt);
    const uint4* vp = reinterpret_cast<const uint4*>(zp);
    const int nv = V / E;
    int i = threadIdx.x;
    // kKlUnroll chunks of each tensor in flight before the arithmetic
    for (; i + (kKlUnroll - 1) * kKlThreads < nv; i += kKlUnroll * kKlThreads) {
      uint4 bt[kKlUnroll], bp[kKlUnroll];
#pragma unroll
      for (int k = 0; k < kKlUnroll; ++k) {
        bt[k] = __ldcs(vt + i + k * kKlThreads);
        bp[k] = __ldcs(vp + i + k * kKlThreads);
      }
#pragma unroll
      for (int k = 0; k < kKlUnroll; ++k) {
        KlLoad<T>::unpack(bt[k], ft);
        KlLoad<T>::unpack(bp[k], fp);
        kl_add<E>(c, ft, fp);
      }
    }
    for (; i < nv; i += kKlThreads) {
      KlLoad<T>::unpack(__ldcs(vt + i), ft);
      KlLoad<T>::unpack(__ldcs(vp + i), fp);
      kl_add<E>(c, ft, fp);
    }
    done = V;
  }
  for (int v = done + threadIdx.x; v < V; v += kKlThreads) {  // unaligned rows: one element at a time
    ft[0] = to_f(zt[v]);
    fp[0] = to_f(zp[v]);
    kl_add<1>(c, ft, fp);
  }
  // block reduction of the sums
#pragma unroll
  for (int o = 16; o; o >>= 1) kl_merge(c, kl_shfl(c, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) sh[warp] = c;
  __syncthreads();
  if (warp == 0) {
    if (lane < kKlThreads / 32)
      c = sh[lane];
    else
      kl_init(c);
#pragma unroll
    for (int o = 16; o; o >>= 1) kl_merge(c, kl_shfl(c, o));
    if (lane == 0) {
      // ln E_q[e^(z_t - z_p)] = lse_t - lse_p
      const float dl = c.far ? (c.mt - c.mp) * kLn2 + logf(c.st) - logf(c.sp) : log1pf(c.u / c.sp);
      const float kl = c.a / c.st - dl;
      const float h = (c.mt * kLn2 + logf(c.st)) - c.e / c.st;
      lock_out[row] = (kl <= eps && h <= h_max) ? 1 : 0;
      if (kl_out) kl_out[row] = kl;
      if (h_out) h_out[row] = h;
    }
  }
}

int launch_kl_lock(const plk_dims* dims, int V, const void* logits_t, const void* logits_prev, const uint8_t* lock_in,
                   uint8_t* lock_out, float eps, float h_max, float* kl_out, float* h_out, cudaStream_t st) {
  const long long rows = (long long)dims->B * dims->N;
  if (dims->dtype == PLK_BF16)
    return launch_pdl(kl_lock_kernel<__nv_bfloat16>, dim3((unsigned)rows), dim3(kKlThreads), 0, st,
                      (const __nv_bfloat16*)logits_t, (const __nv_bfloat16*)logits_prev, rows, V, lock_in, lock_out,
                      eps, h_max, kl_out, h_out);
  return launch_pdl(kl_lock_kernel<float>, dim3((unsigned)rows), dim3(kKlThreads), 0, st, (const float*)logits_t,
                    (const float*)logits_prev, rows, V, lock_in, lock_out, eps, h_max, kl_out, h_out);
}

}  // namespace plk
