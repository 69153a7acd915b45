// Full attention layer with fused importance scores: SIMT fp32-accumulate kernels.
//
// This is the fp32-input path (tensor cores cannot hold 1e-4 accuracy on fp32 data)
// and the path for shapes the tcgen05 kernel does not take.  One CTA owns one
// (batch, query head, 64-query tile); 4 lanes share a row and split the head dim.
//
//   o_t      = sum_{i<=t} softmax_i(tau q_t.k_i) v_i            HySparse 3.4.1, o_t
//   S_{t,j}  = exp(m~_{t,j} - m_t) / l_t                         HySparse 3.4.1, S_t^i and
//              m~_{t,j} = max logit of block j clipped at t      the rescale pass (with exp)
//   part     = R over the tile's rows of S_{t,j}                 summed (or max) aggregation
//
// The block max logit m~ is recomputed in a second sweep over K (this path is not the
// performance path; the tcgen05 kernel keeps m~ from the first sweep instead).
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace hys {

namespace {

constexpr int kRows = 64;      // query rows per CTA (one 64-query tile)
constexpr int kThreads = 256;  // 4 lanes per row
constexpr int kKC = 32;        // keys per shared-memory chunk

template <typename T, int D>
__device__ __forceinline__ void load_chunk(float (*dst)[D], const T* src, int key0, int nkeys_total) {
  for (int e = threadIdx.x; e < kKC * D; e += kThreads) {
    const int kk = e / D, dd = e % D;
    const int key = key0 + kk;
    dst[kk][dd] = key < nkeys_total ? Elem<T>::load(src + (size_t)key * D + dd) : 0.0f;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) full_attn_simt_kernel(PrefillDims d, const T* __restrict__ q,
                                                                   const T* __restrict__ k,
                                                                   const T* __restrict__ v, T* __restrict__ o,
                                                                   float* __restrict__ lse,
                                                                   float* __restrict__ part, int want_scores,
                                                                   int red_max) {
  constexpr int DL = D / 4;
  __shared__ float sk[kKC][D];
  __shared__ float sv[kKC][D];
  __shared__ float sred[kThreads / 32];

  const int I = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / d.G();
  const int tid = threadIdx.x, r = tid >> 2, lg = tid & 3;
  const int t = I * kRows + r;
  const bool valid = t < d.N;
  const T* qh = q + ((size_t)b * d.Hq + h) * d.N * D;
  const T* kh = k + ((size_t)b * d.Hkv + g) * d.N * D;
  const T* vh = v + ((size_t)b * d.Hkv + g) * d.N * D;
  // logits in log2 units: fold tau * log2(e) into q
  const float qscale = kLog2e / sqrtf((float)D);

  float qr[DL], acc[DL];
#pragma unroll
  for (int c = 0; c < DL; ++c) {
    qr[c] = valid ? Elem<T>::load(qh + (size_t)t * D + c * 4 + lg) * qscale : 0.0f;
    acc[c] = 0.0f;
  }
  float m = -INFINITY, l = 0.0f;
  const int last = min(d.N - 1, I * kRows + kRows - 1);

  for (int c0 = 0; c0 <= last; c0 += kKC) {
    __syncthreads();
    load_chunk<T, D>(sk, kh, c0, d.N);
    load_chunk<T, D>(sv, vh, c0, d.N);
    __syncthreads();
    for (int ii = 0; ii < kKC; ++ii) {
      const int i = c0 + ii;
      float s = 0.0f;
#pragma unroll
      for (int c = 0; c < DL; ++c) s = fmaf(qr[c], sk[ii][c * 4 + lg], s);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (valid && i <= t) {
        if (s > m) {
          const float corr = exp2f(m - s);
          l = l * corr + 1.0f;
#pragma unroll
          for (int c = 0; c < DL; ++c) acc[c] = fmaf(acc[c], corr, sv[ii][c * 4 + lg]);
          m = s;
        } else {
          const float p = exp2f(s - m);
          l += p;
#pragma unroll
          for (int c = 0; c < DL; ++c) acc[c] = fmaf(p, sv[ii][c * 4 + lg], acc[c]);
        }
      }
    }
  }

  if (valid) {
    const float inv = 1.0f / l;
    T* oh = o + ((size_t)b * d.Hq + h) * d.N * D + (size_t)t * D;
#pragma unroll
    for (int c = 0; c < DL; ++c) Elem<T>::store(oh + c * 4 + lg, acc[c] * inv);
    if (lg == 0 && lse != nullptr)
      lse[((size_t)b * d.Hq + h) * d.N + t] = (m + log2f(l)) * 0.69314718055994531f;
  }
  if (!want_scores) return;

  // second sweep over K: block max logit clipped at t, rescaled by the final m, l
  const float inv_l = valid ? 1.0f / l : 0.0f;
  for (int j = 0; j <= I; ++j) {
    float mt = -INFINITY;
    for (int c0 = j * 64; c0 < j * 64 + 64 && c0 <= last; c0 += kKC) {
      __syncthreads();
      load_chunk<T, D>(sk, kh, c0, d.N);
      __syncthreads();
      for (int ii = 0; ii < kKC; ++ii) {
        const int i = c0 + ii;
        float s = 0.0f;
#pragma unroll
        for (int c = 0; c < DL; ++c) s = fmaf(qr[c], sk[ii][c * 4 + lg], s);
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        if (valid && i <= t) mt = fmaxf(mt, s);
      }
    }
    float val = (valid && lg == 0 && mt > -INFINITY) ? exp2f(mt - m) * inv_l : 0.0f;
    for (int off = 4; off < 32; off <<= 1) {
      const float o2 = __shfl_xor_sync(0xffffffffu, val, off);
      val = red_max ? fmaxf(val, o2) : val + o2;
    }
    if ((tid & 31) == 0) sred[tid >> 5] = val;
    __syncthreads();
    if (tid == 0) {
      float a = sred[0];
      for (int w = 1; w < kThreads / 32; ++w) a = red_max ? fmaxf(a, sred[w]) : a + sred[w];
      part[(((size_t)b * d.Hq + h) * d.T + I) * d.NB + j] = a;
    }
  }
}

// scores[b,g,I,j] = R_{h in g} part[b,h,I,j] for j <= I (heads in ascending order), else 0
__global__ void head_reduce_kernel(PrefillDims d, const float* __restrict__ part, float* __restrict__ scores,
                                   int red_max) {
  const int row = blockIdx.x;  // (b*Hkv + g)*T + I
  const int I = row % d.T;
  const int bg = row / d.T;
  const int b = bg / d.Hkv, g = bg % d.Hkv;
  const int G = d.G();
  for (int j = threadIdx.x; j < d.NB; j += blockDim.x) {
    float a = 0.0f;
    if (j <= I) {
      for (int hh = 0; hh < G; ++hh) {
        const float x = part[(((size_t)b * d.Hq + g * G + hh) * d.T + I) * d.NB + j];
        a = (hh == 0) ? x : (red_max ? fmaxf(a, x) : a + x);
      }
    }
    scores[(size_t)row * d.NB + j] = a;
  }
}

// Token scores: scores[b,g,I,i] = sum_{h in g} sum_{t in tile I, t >= i} exp(tau q_t.k_i - LSE_t)
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) token_scores_simt_kernel(PrefillDims d, const T* __restrict__ q,
                                                                     const T* __restrict__ k,
                                                                     const float* __restrict__ lse,
                                                                     float* __restrict__ scores) {
  constexpr int DL = D / 4;
  __shared__ float sk[kKC][D];
  __shared__ float spart[kThreads / 32][kKC];
  const int I = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int G = d.G();
  const int tid = threadIdx.x, r = tid >> 2, lg = tid & 3, warp = tid >> 5;
  const int t = I * kRows + r;
  const bool valid = t < d.N;
  const int last = min(d.N - 1, I * kRows + kRows - 1);
  const T* kh = k + ((size_t)b * d.Hkv + g) * d.N * D;
  float* srow = scores + (((size_t)b * d.Hkv + g) * d.T + I) * d.N;
  const float qscale = kLog2e / sqrtf((float)D);

  for (int hh = 0; hh < G; ++hh) {
    const int h = g * G + hh;
    const T* qh = q + ((size_t)b * d.Hq + h) * d.N * D;
    float qr[DL];
#pragma unroll
    for (int c = 0; c < DL; ++c) qr[c] = valid ? Elem<T>::load(qh + (size_t)t * D + c * 4 + lg) * qscale : 0.0f;
    const float lse2 = valid ? lse[((size_t)b * d.Hq + h) * d.N + t] * kLog2e : 0.0f;
    for (int c0 = 0; c0 <= last; c0 += kKC) {
      __syncthreads();
      load_chunk<T, D>(sk, kh, c0, d.N);
      __syncthreads();
      for (int ii = 0; ii < kKC; ++ii) {
        const int i = c0 + ii;
        float s = 0.0f;
#pragma unroll
        for (int c = 0; c < DL; ++c) s = fmaf(qr[c], sk[ii][c * 4 + lg], s);
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        float p = (valid && lg == 0 && i <= t) ? exp2f(s - lse2) : 0.0f;
        for (int off = 4; off < 32; off <<= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
        if ((tid & 31) == 0) spart[warp][ii] = p;
      }
      __syncthreads();
      if (tid < kKC) {
        const int i = c0 + tid;
        float a = 0.0f;
        for (int w = 0; w < kThreads / 32; ++w) a += spart[w][tid];
        if (i < d.N) srow[i] = (hh == 0) ? a : srow[i] + a;
      }
    }
  }
  // keys past the tile's last row receive no probability
  for (int i = last + 1 + tid; i < d.N; i += kThreads) srow[i] = 0.0f;
}

template <typename T, int D>
cudaError_t launch_full_typed(const PrefillDims& d, const void* q, const void* k, const void* v, void* o,
                              float* lse, float* part, bool want_scores, hys_reduce red, cudaStream_t s) {
  dim3 grid(d.T, d.Hq, d.B);
  full_attn_simt_kernel<T, D><<<grid, kThreads, 0, s>>>(d, (const T*)q, (const T*)k, (const T*)v, (T*)o, lse,
                                                        part, want_scores ? 1 : 0, red == HYS_REDUCE_MAX);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_tok_typed(const PrefillDims& d, const void* q, const void* k, const float* lse, float* sc,
                             cudaStream_t s) {
  dim3 grid(d.T, d.Hkv, d.B);
  token_scores_simt_kernel<T, D><<<grid, kThreads, 0, s>>>(d, (const T*)q, (const T*)k, lse, sc);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_full_attn_simt(const PrefillDims& d, hys_dtype dt, const void* q, const void* k, const void* v,
                                  void* o, float* lse, float* part, bool want_scores, hys_reduce red,
                                  cudaStream_t s) {
  if (dt == HYS_F32)
    return d.D == 64 ? launch_full_typed<float, 64>(d, q, k, v, o, lse, part, want_scores, red, s)
                     : launch_full_typed<float, 128>(d, q, k, v, o, lse, part, want_scores, red, s);
  return d.D == 64 ? launch_full_typed<__nv_bfloat16, 64>(d, q, k, v, o, lse, part, want_scores, red, s)
                   : launch_full_typed<__nv_bfloat16, 128>(d, q, k, v, o, lse, part, want_scores, red, s);
}

cudaError_t launch_head_reduce(const PrefillDims& d, const float* part, float* scores, hys_reduce red,
                               cudaStream_t s) {
  head_reduce_kernel<<<d.B * d.Hkv * d.T, 256, 0, s>>>(d, part, scores, red == HYS_REDUCE_MAX);
  return cudaGetLastError();
}

cudaError_t launch_token_scores_simt(const PrefillDims& d, hys_dtype dt, const void* q, const void* k,
                                     const float* lse, float* scores, cudaStream_t s) {
  if (dt == HYS_F32)
    return d.D == 64 ? launch_tok_typed<float, 64>(d, q, k, lse, scores, s)
                     : launch_tok_typed<float, 128>(d, q, k, lse, scores, s);
  return d.D == 64 ? launch_tok_typed<__nv_bfloat16, 64>(d, q, k, lse, scores, s)
                   : launch_tok_typed<__nv_bfloat16, 128>(d, q, k, lse, scores, s);
}

}  // namespace hys
