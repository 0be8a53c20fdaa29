// S7: non-causal attention of the M active queries over all N cached keys of
// their sequence ("Continued Attention" of the SureLock page, "Stopping
// Computation for Converged Tokens in Masked Diffusion-LM Decoding", Sec. 2:
// active tokens keep attending to locked tokens through their cached K/V; cost
// O(M N d) instead of O(N^2 d), Sec. 2 "Algorithmic Complexity").
//
// bf16, hd = 128: one CTA per (64-query tile, head, sequence), 4 warps of 16
// query rows.  K/V tiles of 64 keys x 128 dims are staged by TMA (128-byte
// swizzle, two boxes of 64 dims each) into a double-buffered shared-memory
// ring; Q fragments stay in registers; S = Q K^T and O += P V run on the tensor
// cores (mma.sync m16n8k16, fp32 accumulate) with an online softmax in
// registers (quad shuffles for the row max and sum).  P is split into a bf16
// high part and a bf16 residual and both are multiplied with V, so the softmax
// weights enter P V with ~16 significant bits: a bf16-rounded P would perturb
// the attention output by ~1e-3 relative, which later bf16 roundings amplify.
// Rows past the sequence's last active row and keys past N are masked.
// fp32: one thread per (query row, head), online softmax, SIMT.
#include <math.h>

#include <algorithm>

#include "plk_common.cuh"
#include "plk_internal.h"

namespace plk {

namespace {
constexpr int kAttBQ = 64, kAttBK = 64, kAttHD = 128, kAttThreads = 128;
constexpr int kAttTile = kAttBK * kAttHD * 2;  // 16 KB
constexpr int kAttSmem = 5 * kAttTile + 128 + 1024;

__device__ __forceinline__ uint32_t sw_addr(uint32_t base, int row, int col) {
  // [64 rows][128 cols] bf16 stored as two 64-column boxes with 128-byte swizzle
  return base + (uint32_t)((col >> 6) * 8192 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4));
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
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
}  // namespace

// Number of key splits for the current active set: enough CTAs to cover the
// GPU twice, at most smax.  Computed identically by the attention and combine
// kernels from seg_ptr (device-side M, no host synchronisation).
__device__ __forceinline__ int attn_splits(const int32_t* seg_ptr, int B, int H, int smax, int nsm) {
  int qtiles = 0;
  for (int b = 0; b < B; ++b) qtiles += ceil_div(seg_ptr[b + 1] - seg_ptr[b], kAttBQ);
  if (qtiles == 0) return 1;
  const int want = ceil_div(2 * nsm, qtiles * H);
  return max(1, min(smax, want));
}

// Split partials: o_part[s][row][d] (unnormalised, fp32) and ml[s][row][h] = (max, sum)
// in the log2 domain; rows are compact active-row indices below part_rows.
struct AttnSplit {
  float* o_part;
  float2* ml;
  int smax, part_rows, nsm;
};

__global__ void __launch_bounds__(kAttThreads) attn_bf16_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                const __grid_constant__ CUtensorMap tmV,
                                                                const __nv_bfloat16* __restrict__ Q,
                                                                __nv_bfloat16* __restrict__ Aout,
                                                                const int32_t* __restrict__ seg_ptr, int B, int N,
                                                                int d, float scale_log2, AttnSplit sp) {
  pdl_wait();
  pdl_trigger();
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z / sp.smax, split = blockIdx.z % sp.smax;
  const int seg0 = seg_ptr[b], seg1 = seg_ptr[b + 1];
  const int r0 = seg0 + qt * kAttBQ;
  if (r0 >= seg1) return;
  const int S = attn_splits(seg_ptr, B, gridDim.y, sp.smax, sp.nsm);
  if (split >= S) return;
  const int nrows = min(kAttBQ, seg1 - r0);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kAttTile;          // [2] stages
  uint8_t* sV = smem + 3 * kAttTile;      // [2] stages
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + 5 * kAttTile);
  volatile int* s_bad = reinterpret_cast<volatile int*>(full + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntiles_all = ceil_div(N, kAttBK);
  const int t0 = split * ntiles_all / S;                 // this split's key tiles [t0, t0 + ntiles)
  const int ntiles = (split + 1) * ntiles_all / S - t0;
  const int hcol = h * kAttHD;

  if (tid == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    *s_bad = 0;
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int j, int s) {
    const int y = b * N + (t0 + j) * kAttBK;
    mbar_expect_tx(&full[s], 2 * kAttTile);
    tma_load_2d(sK + s * kAttTile, &tmK, hcol, y, &full[s]);
    tma_load_2d(sK + s * kAttTile + 8192, &tmK, hcol + 64, y, &full[s]);
    tma_load_2d(sV + s * kAttTile, &tmV, hcol, y, &full[s]);
    tma_load_2d(sV + s * kAttTile + 8192, &tmV, hcol + 64, y, &full[s]);
  };
  int last_issued = -1;  // meaningful in thread 0, which issues every copy
  if (tid == 0) {
    issue(0, 0);
    last_issued = 0;
    if (ntiles > 1) {
      issue(1, 1);
      last_issued = 1;
    }
  }
  // Q tile -> shared memory in the same swizzled layout (zeros past the last row)
  for (int e = tid; e < kAttBQ * 16; e += kAttThreads) {
    const int row = e >> 4, ch = e & 15;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (row < nrows) v = *reinterpret_cast<const uint4*>(Q + (size_t)(r0 + row) * d + hcol + ch * 8);
    *reinterpret_cast<uint4*>(sQ + ((ch >> 3) * 8192 + row * 128 + (((ch & 7) ^ (row & 7)) << 4))) = v;
  }
  __syncthreads();

  const uint32_t qbase = smem_u32(sQ), kbase0 = smem_u32(sK), vbase0 = smem_u32(sV);
  const int mi = lane >> 3, ri = lane & 7;
  uint32_t qa[8][4];
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
    ldsm_x4(qa[ks], sw_addr(qbase, warp * 16 + (mi & 1) * 8 + ri, ks * 16 + (mi >> 1) * 8));

  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  const int cq = lane & 3;

  int jfail = ntiles;
  for (int j = 0; j < ntiles; ++j) {
    const int s = j & 1;
    if (!mbar_wait(&full[s], (uint32_t)((j >> 1) & 1))) *s_bad = 1;
    __syncthreads();
    if (*s_bad) {
      jfail = j;
      break;
    }
    const uint32_t kb = kbase0 + s * kAttTile, vb = vbase0 + s * kAttTile;
    float sc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t kr[4];
        ldsm_x4(kr, sw_addr(kb, (2 * np + (mi >> 1)) * 8 + ri, ks * 16 + (mi & 1) * 8));
        mma16816(sc[2 * np], qa[ks], kr[0], kr[1]);
        mma16816(sc[2 * np + 1], qa[ks], kr[2], kr[3]);
      }
    }
    const int key0 = (t0 + j) * kAttBK;
    if (key0 + kAttBK > N) {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (key0 + nt * 8 + 2 * cq + (e & 1) >= N) sc[nt][e] = -INFINITY;
    }
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) mx = fmaxf(mx, fmaxf(sc[nt][2 * hf], sc[nt][2 * hf + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_r[hf], mx * scale_log2);
      const float alpha = exp2f(m_r[hf] - m_new);
      m_r[hf] = m_new;
      float rs = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float p0 = exp2f(fmaf(sc[nt][2 * hf], scale_log2, -m_new));
        const float p1 = exp2f(fmaf(sc[nt][2 * hf + 1], scale_log2, -m_new));
        sc[nt][2 * hf] = p0;
        sc[nt][2 * hf + 1] = p1;
        rs += p0 + p1;
      }
      l_r[hf] = l_r[hf] * alpha + rs;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        o[nt][2 * hf] *= alpha;
        o[nt][2 * hf + 1] *= alpha;
      }
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t ah[4], al[4];
      split_pair(sc[2 * kk][0], sc[2 * kk][1], ah[0], al[0]);
      split_pair(sc[2 * kk][2], sc[2 * kk][3], ah[1], al[1]);
      split_pair(sc[2 * kk + 1][0], sc[2 * kk + 1][1], ah[2], al[2]);
      split_pair(sc[2 * kk + 1][2], sc[2 * kk + 1][3], ah[3], al[3]);
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        uint32_t vr[4];
        ldsm_x4_t(vr, sw_addr(vb, kk * 16 + (mi & 1) * 8 + ri, (2 * np + (mi >> 1)) * 8));
        mma16816(o[2 * np], ah, vr[0], vr[1]);
        mma16816(o[2 * np], al, vr[0], vr[1]);
        mma16816(o[2 * np + 1], ah, vr[2], vr[3]);
        mma16816(o[2 * np + 1], al, vr[2], vr[3]);
      }
    }
    __syncthreads();  // every warp is done with stage s
    if (tid == 0 && j + 2 < ntiles) {
      issue(j + 2, s);
      last_issued = j + 2;
    }
  }
  if (*s_bad) {
    // bounded wait for the copies this CTA started, then leave without writing
    if (tid == 0)
      for (int t = jfail; t <= last_issued; ++t) (void)mbar_wait(&full[t & 1], (uint32_t)((t >> 1) & 1));
    return;
  }
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    float l = l_r[hf];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    const int row = warp * 16 + (lane >> 2) + 8 * hf;
    if (row >= nrows) continue;
    if (S == 1) {
      const float inv = 1.0f / l;
      __nv_bfloat16* dst = Aout + (size_t)(r0 + row) * d + hcol + 2 * cq;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt)
        *reinterpret_cast<uint32_t*>(dst + nt * 8) = pack_bf16(o[nt][2 * hf] * inv, o[nt][2 * hf + 1] * inv);
    } else {
      float* dst = sp.o_part + ((size_t)split * sp.part_rows + (r0 + row)) * d + hcol + 2 * cq;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt)
        *reinterpret_cast<float2*>(dst + nt * 8) = make_float2(o[nt][2 * hf], o[nt][2 * hf + 1]);
      if (cq == 0) sp.ml[((size_t)split * sp.part_rows + (r0 + row)) * gridDim.y + h] = make_float2(m_r[hf], l);
    }
  }
}

// out[row, h] = sum_s 2^(m_s - m) o_s / sum_s 2^(m_s - m) l_s, one CTA per active row.
__global__ void __launch_bounds__(256) attn_combine_kernel(const int32_t* __restrict__ seg_ptr, int B, int H,
                                                           int d, AttnSplit sp, __nv_bfloat16* __restrict__ Aout) {
  pdl_wait();
  pdl_trigger();
  const int j = blockIdx.x;
  if (j >= seg_ptr[B]) return;
  const int S = attn_splits(seg_ptr, B, H, sp.smax, sp.nsm);
  if (S == 1) return;
  for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4) {
    const int h = c / kAttHD;
    float m = -INFINITY;
    for (int s = 0; s < S; ++s) m = fmaxf(m, sp.ml[((size_t)s * sp.part_rows + j) * H + h].x);
    float l = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < S; ++s) {
      const float2 ml = sp.ml[((size_t)s * sp.part_rows + j) * H + h];
      const float w = exp2f(ml.x - m);
      l = fmaf(w, ml.y, l);
      const float4 o = *reinterpret_cast<const float4*>(sp.o_part + ((size_t)s * sp.part_rows + j) * d + c);
      acc[0] = fmaf(w, o.x, acc[0]);
      acc[1] = fmaf(w, o.y, acc[1]);
      acc[2] = fmaf(w, o.z, acc[2]);
      acc[3] = fmaf(w, o.w, acc[3]);
    }
    const float inv = 1.0f / l;
    uint2 u;
    u.x = pack_bf16(acc[0] * inv, acc[1] * inv);
    u.y = pack_bf16(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(Aout + (size_t)j * d + c) = u;
  }
}

template <int HD>
__global__ void attn_f32_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                                const float* __restrict__ V, float* __restrict__ A,
                                const int32_t* __restrict__ seg_ptr, int B, int N, int d, int H, float scale) {
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
    const float* kr = K + ((size_t)b * N + n) * d + h * HD;
    const float* vr = V + ((size_t)b * N + n) * d + h * HD;
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

int attn_split_rows(const plk_dims* dims, int num_sms) {
  // splits are used only while q-tiles x heads < 2 x SMs, so fewer active rows
  const int rows = ceil_div(2 * num_sms, dims->H) * kAttBQ;
  return std::min(dims->B * dims->N, rows);
}

int launch_attention_bf16(const plk_dims* dims, const void* q, const void* K_cache, const void* V_cache,
                          void* a_out, const int32_t* seg_ptr, float* o_part, void* ml, int smax, int part_rows,
                          int num_sms, cudaStream_t st) {
  const int B = dims->B, N = dims->N, d = dims->d, H = dims->H;
  CUtensorMap tmK, tmV;
  if (make_tmap_bf16(&tmK, K_cache, (uint64_t)B * N, (uint64_t)d, 64) != PLK_OK) return PLK_ERR_CUDA;
  if (make_tmap_bf16(&tmV, V_cache, (uint64_t)B * N, (uint64_t)d, 64) != PLK_OK) return PLK_ERR_CUDA;
  static int attr_done[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PLK_ERR_CUDA;
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(attn_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAttSmem) !=
        cudaSuccess)
      return PLK_ERR_CUDA;
    attr_done[dev] = 1;
  }
  const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)dims->hd));
  AttnSplit sp{o_part, (float2*)ml, std::max(1, std::min(smax, ceil_div(N, kAttBK))), part_rows, num_sms};
  dim3 grid(ceil_div(N, kAttBQ), H, B * sp.smax);
  const int rc = launch_pdl(attn_bf16_kernel, grid, dim3(kAttThreads), kAttSmem, st, tmK, tmV,
                            (const __nv_bfloat16*)q, (__nv_bfloat16*)a_out, seg_ptr, B, N, d, scale_log2, sp);
  if (rc != PLK_OK || sp.smax == 1) return rc;
  return launch_pdl(attn_combine_kernel, dim3(part_rows), dim3(256), 0, st, seg_ptr, B, H, d, sp,
                    (__nv_bfloat16*)a_out);
}

int launch_attention_f32(const plk_dims* dims, const float* q, const float* K_cache, const float* V_cache,
                         float* a_out, const int32_t* seg_ptr, int Mcap, cudaStream_t st) {
  const int B = dims->B, N = dims->N, d = dims->d, H = dims->H, hd = dims->hd;
  const float scale = (float)(1.0 / sqrt((double)hd));
  const int threads = 128, blocks = ceil_div(Mcap * H, threads);
  switch (hd) {
    case 16: attn_f32_kernel<16><<<blocks, threads, 0, st>>>(q, K_cache, V_cache, a_out, seg_ptr, B, N, d, H, scale); break;
    case 32: attn_f32_kernel<32><<<blocks, threads, 0, st>>>(q, K_cache, V_cache, a_out, seg_ptr, B, N, d, H, scale); break;
    case 64: attn_f32_kernel<64><<<blocks, threads, 0, st>>>(q, K_cache, V_cache, a_out, seg_ptr, B, N, d, H, scale); break;
    case 128: attn_f32_kernel<128><<<blocks, threads, 0, st>>>(q, K_cache, V_cache, a_out, seg_ptr, B, N, d, H, scale); break;
    default: return PLK_ERR_SHAPE;
  }
  return cudaPeekAtLastError() == cudaSuccess ? PLK_OK : PLK_ERR_CUDA;
}

}  // namespace plk
