// Sparse layer, SIMT fp32-accumulate kernels (fp32 inputs and shapes the tcgen05 kernel
// does not take).
//
// Block variant (HySparse 3.4.3): row t of tile I runs two online softmaxes,
//   sparse branch  keys {i <= t : floor(i/64) in Sel_I} of the shared K, V (the gather
//                  K~, V~ = concat of the selected 64-token blocks is never materialised:
//                  each selected block is staged straight from the cache);
//   SWA branch     keys [max(0, t-w+1), t] of the layer's own K', V';
// and merges them with the sigmoid gates: o = s(g0) o~ + s(g1) o'.
// Token variant (HySparse2 explainer): one softmax over Sel_I united with the row's
// newest `forced` tokens, each token once; no gate.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace hys {

namespace {

constexpr int kThreads = 256;
constexpr int kKC = 32;

struct OnlineState {
  float m, l;
};

template <int DL>
__device__ __forceinline__ void online_update(float s, bool take, OnlineState& st, float (&acc)[DL],
                                              const float* vrow, int lg) {
  if (!take) return;
  if (s > st.m) {
    const float corr = exp2f(st.m - s);
    st.l = st.l * corr + 1.0f;
#pragma unroll
    for (int c = 0; c < DL; ++c) acc[c] = fmaf(acc[c], corr, vrow[c * 4 + lg]);
    st.m = s;
  } else {
    const float p = exp2f(s - st.m);
    st.l += p;
#pragma unroll
    for (int c = 0; c < DL; ++c) acc[c] = fmaf(p, vrow[c * 4 + lg], acc[c]);
  }
}

template <int DL>
__device__ __forceinline__ float row_dot(const float (&qr)[DL], const float* krow, int lg) {
  float s = 0.0f;
#pragma unroll
  for (int c = 0; c < DL; ++c) s = fmaf(qr[c], krow[c * 4 + lg], s);
  s += __shfl_xor_sync(0xffffffffu, s, 1);
  s += __shfl_xor_sync(0xffffffffu, s, 2);
  return s;
}

// stage kKC rows given by a position list (pos < 0 or >= N -> zeros)
template <typename T, int D>
__device__ __forceinline__ void stage_rows(float (*dk)[D], float (*dv)[D], const T* k, const T* v,
                                           const int* pos, int N) {
  for (int e = threadIdx.x; e < kKC * D; e += kThreads) {
    const int kk = e / D, dd = e % D;
    const int p = pos[kk];
    const bool ok = p >= 0 && p < N;
    dk[kk][dd] = ok ? Elem<T>::load(k + (size_t)p * D + dd) : 0.0f;
    dv[kk][dd] = ok ? Elem<T>::load(v + (size_t)p * D + dd) : 0.0f;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) sparse_attn_simt_kernel(
    PrefillDims d, const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
    const int* __restrict__ idx, int kb, const T* __restrict__ ks, const T* __restrict__ vs, int window,
    const float* __restrict__ gate, const float* __restrict__ sinks, T* __restrict__ o, float* __restrict__ blse,
    T* __restrict__ osp) {
  constexpr int DL = D / 4;
  __shared__ float sk[kKC][D];
  __shared__ float sv[kKC][D];
  __shared__ int spos[kKC];
  const int I = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / d.G();
  const int tid = threadIdx.x, r = tid >> 2, lg = tid & 3;
  const int t = I * 64 + r;
  const bool valid = t < d.N;
  const size_t kvoff = ((size_t)b * d.Hkv + g) * d.N * D;
  const T* qh = q + ((size_t)b * d.Hq + h) * d.N * D;
  const float qscale = kLog2e / sqrtf((float)D);
  float qr[DL], a_sp[DL], a_sw[DL];
#pragma unroll
  for (int c = 0; c < DL; ++c) {
    qr[c] = valid ? Elem<T>::load(qh + (size_t)t * D + c * 4 + lg) * qscale : 0.0f;
    a_sp[c] = 0.0f;
    a_sw[c] = 0.0f;
  }
  OnlineState st_sp{-INFINITY, 0.0f}, st_sw{-INFINITY, 0.0f};
  const int* sel = idx + (((size_t)b * d.Hkv + g) * d.T + I) * kb;

  // sparse branch over the selected blocks (entries outside [0, I] are ignored)
  for (int sIdx = 0; sIdx < kb; ++sIdx) {
    const int j = sel[sIdx];
    if (j < 0 || j > I) continue;
    for (int c0 = j * 64; c0 < j * 64 + 64; c0 += kKC) {
      __syncthreads();
      if (tid < kKC) spos[tid] = c0 + tid;
      __syncthreads();
      stage_rows<T, D>(sk, sv, k + kvoff, v + kvoff, spos, d.N);
      __syncthreads();
      for (int ii = 0; ii < kKC; ++ii) {
        const int i = c0 + ii;
        const float s = row_dot<DL>(qr, sk[ii], lg);
        online_update<DL>(s, valid && i <= t && i < d.N, st_sp, a_sp, sv[ii], lg);
      }
    }
  }
  // SWA branch over the tile's union window
  const int w0 = max(0, I * 64 - window + 1);
  const int w1 = min(d.N - 1, I * 64 + 63);
  for (int c0 = w0; c0 <= w1; c0 += kKC) {
    __syncthreads();
    if (tid < kKC) spos[tid] = (c0 + tid <= w1) ? c0 + tid : -1;
    __syncthreads();
    stage_rows<T, D>(sk, sv, ks + kvoff, vs + kvoff, spos, d.N);
    __syncthreads();
    for (int ii = 0; ii < kKC; ++ii) {
      const int i = c0 + ii;
      const float s = row_dot<DL>(qr, sk[ii], lg);
      online_update<DL>(s, valid && i <= t && i >= t - window + 1, st_sw, a_sw, sv[ii], lg);
    }
  }
  if (!valid) return;
  const float* gl = gate + (((size_t)b * d.Hq + h) * d.N + t) * 2;
  const float g0 = sigmoidf_(gl[0]), g1 = sigmoidf_(gl[1]);
  // each branch's sink logit joins its softmax as an entry with a zero value (log2 units here)
  const float l_sp = st_sp.l + (sinks ? exp2f(sinks[2 * h] * kLog2e - st_sp.m) : 0.0f);
  const float l_sw = st_sw.l + (sinks ? exp2f(sinks[2 * h + 1] * kLog2e - st_sw.m) : 0.0f);
  const float i_sp = l_sp > 0.0f ? g0 / l_sp : 0.0f;
  const float i_sw = l_sw > 0.0f ? g1 / l_sw : 0.0f;
  T* oh = o + ((size_t)b * d.Hq + h) * d.N * D + (size_t)t * D;
#pragma unroll
  for (int c = 0; c < DL; ++c) Elem<T>::store(oh + c * 4 + lg, a_sp[c] * i_sp + a_sw[c] * i_sw);
  if (blse != nullptr) {
    // training forward: each branch's LSE (natural-log units of the scaled logits, sink included;
    // a branch without keys: the sink alone, or -inf) and the gated sparse part sigmoid(g0) o~
    if (lg == 0) {
      const float sk0 = sinks ? sinks[2 * h] * kLog2e : -INFINITY, sk1 = sinks ? sinks[2 * h + 1] * kLog2e : -INFINITY;
      const float a = st_sp.m == -INFINITY ? sk0 : st_sp.m + log2f(l_sp);
      const float c = st_sw.m == -INFINITY ? sk1 : st_sw.m + log2f(l_sw);
      float* lrow = blse + (((size_t)b * d.Hq + h) * d.N + t) * 2;
      lrow[0] = a * 0.6931471805599453f;
      lrow[1] = c * 0.6931471805599453f;
    }
    T* sph = osp + ((size_t)b * d.Hq + h) * d.N * D + (size_t)t * D;
#pragma unroll
    for (int c = 0; c < DL; ++c) Elem<T>::store(sph + c * 4 + lg, a_sp[c] * i_sp);
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) sparse_tokens_simt_kernel(PrefillDims d, const T* __restrict__ q,
                                                                      const T* __restrict__ k,
                                                                      const T* __restrict__ v,
                                                                      const int* __restrict__ idx, int kt,
                                                                      int forced, T* __restrict__ o) {
  constexpr int DL = D / 4;
  __shared__ float sk[kKC][D];
  __shared__ float sv[kKC][D];
  __shared__ int spos[kKC];
  const int I = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / d.G();
  const int tid = threadIdx.x, r = tid >> 2, lg = tid & 3;
  const int t = I * 64 + r;
  const bool valid = t < d.N;
  const size_t kvoff = ((size_t)b * d.Hkv + g) * d.N * D;
  const T* qh = q + ((size_t)b * d.Hq + h) * d.N * D;
  const float qscale = kLog2e / sqrtf((float)D);
  float qr[DL], acc[DL];
#pragma unroll
  for (int c = 0; c < DL; ++c) {
    qr[c] = valid ? Elem<T>::load(qh + (size_t)t * D + c * 4 + lg) * qscale : 0.0f;
    acc[c] = 0.0f;
  }
  OnlineState st{-INFINITY, 0.0f};
  const int* sel = idx + (((size_t)b * d.Hkv + g) * d.T + I) * kt;
  // selected tokens that lie outside the row's own forced window (the window comes next)
  for (int c0 = 0; c0 < kt; c0 += kKC) {
    __syncthreads();
    if (tid < kKC) spos[tid] = (c0 + tid < kt) ? sel[c0 + tid] : -1;
    __syncthreads();
    stage_rows<T, D>(sk, sv, k + kvoff, v + kvoff, spos, d.N);
    __syncthreads();
    for (int ii = 0; ii < kKC; ++ii) {
      const int i = spos[ii];
      const float s = row_dot<DL>(qr, sk[ii], lg);
      online_update<DL>(s, valid && i >= 0 && i < d.N && i <= t && i < t - forced + 1, st, acc, sv[ii], lg);
    }
  }
  const int w0 = max(0, I * 64 - forced + 1);
  const int w1 = min(d.N - 1, I * 64 + 63);
  for (int c0 = w0; c0 <= w1; c0 += kKC) {
    __syncthreads();
    if (tid < kKC) spos[tid] = (c0 + tid <= w1) ? c0 + tid : -1;
    __syncthreads();
    stage_rows<T, D>(sk, sv, k + kvoff, v + kvoff, spos, d.N);
    __syncthreads();
    for (int ii = 0; ii < kKC; ++ii) {
      const int i = c0 + ii;
      const float s = row_dot<DL>(qr, sk[ii], lg);
      online_update<DL>(s, valid && i <= t && i >= t - forced + 1, st, acc, sv[ii], lg);
    }
  }
  if (!valid) return;
  const float inv = st.l > 0.0f ? 1.0f / st.l : 0.0f;
  T* oh = o + ((size_t)b * d.Hq + h) * d.N * D + (size_t)t * D;
#pragma unroll
  for (int c = 0; c < DL; ++c) Elem<T>::store(oh + c * 4 + lg, acc[c] * inv);
}

template <typename T, int D>
cudaError_t launch_sparse_typed(const PrefillDims& d, const void* q, const void* k, const void* v, const int* idx,
                                int kb, const void* ks, const void* vs, int window, const float* gate,
                                const float* sinks, void* o, cudaStream_t s, float* blse, void* osp) {
  dim3 grid(d.T, d.Hq, d.B);
  sparse_attn_simt_kernel<T, D><<<grid, kThreads, 0, s>>>(d, (const T*)q, (const T*)k, (const T*)v, idx, kb,
                                                          (const T*)ks, (const T*)vs, window, gate, sinks, (T*)o,
                                                          blse, (T*)osp);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_tokens_typed(const PrefillDims& d, const void* q, const void* k, const void* v, const int* idx,
                                int kt, int forced, void* o, cudaStream_t s) {
  dim3 grid(d.T, d.Hq, d.B);
  sparse_tokens_simt_kernel<T, D><<<grid, kThreads, 0, s>>>(d, (const T*)q, (const T*)k, (const T*)v, idx, kt,
                                                            forced, (T*)o);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_attn_simt(const PrefillDims& d, hys_dtype dt, const void* q, const void* k, const void* v,
                                    const int* idx, int kb, const void* ks, const void* vs, int window,
                                    const float* gate, const float* sinks, void* o, cudaStream_t s, float* blse,
                                    void* osp) {
  if (dt == HYS_F32)
    return d.D == 64
               ? launch_sparse_typed<float, 64>(d, q, k, v, idx, kb, ks, vs, window, gate, sinks, o, s, blse, osp)
               : launch_sparse_typed<float, 128>(d, q, k, v, idx, kb, ks, vs, window, gate, sinks, o, s, blse, osp);
  return d.D == 64 ? launch_sparse_typed<__nv_bfloat16, 64>(d, q, k, v, idx, kb, ks, vs, window, gate, sinks, o, s,
                                                            blse, osp)
                   : launch_sparse_typed<__nv_bfloat16, 128>(d, q, k, v, idx, kb, ks, vs, window, gate, sinks, o, s,
                                                             blse, osp);
}

cudaError_t launch_sparse_tokens_simt(const PrefillDims& d, hys_dtype dt, const void* q, const void* k,
                                      const void* v, const int* idx, int kt, int forced, void* o, cudaStream_t s) {
  if (dt == HYS_F32)
    return d.D == 64 ? launch_tokens_typed<float, 64>(d, q, k, v, idx, kt, forced, o, s)
                     : launch_tokens_typed<float, 128>(d, q, k, v, idx, kt, forced, o, s);
  return d.D == 64 ? launch_tokens_typed<__nv_bfloat16, 64>(d, q, k, v, idx, kt, forced, o, s)
                   : launch_tokens_typed<__nv_bfloat16, 128>(d, q, k, v, idx, kt, forced, o, s);
}

}  // namespace hys
