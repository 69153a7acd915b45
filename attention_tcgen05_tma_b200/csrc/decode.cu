// Single-token decode against the shared KV cache (HySparse2 explainer, "Twenty lines of
// algorithmic intuition"; HySparse 3.4.1 for the block scores, 3.4.3 for the sparse layer).
//
// Full layer: split-KV.  CTA (split, g, b) streams keys [split*1024, ...) of KV head g for
// all G query heads of the group and leaves per-head partial (m, l, acc[D]) plus the max
// logit of every 64-key block.  A combine kernel merges the splits, writes o and turns
// the block maxima into S_j = exp(m~_j - m)/l, aggregated over the group's heads.
// Sparse layer: CTA (g, b) attends the selected blocks of the shared cache and the
// layer's own SWA ring with two online softmaxes, then applies the sigmoid gate.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace hys {

namespace {

constexpr int kThreads = 256;
constexpr int kKC = 32;          // keys per staged chunk
constexpr int kSplit = 1024;     // keys per split (16 blocks)
constexpr int kMaxG = 16;

// Per-CTA decode state for G heads: running max/sum in shared memory, accumulators in
// registers (thread owns pairs e = tid + 256*r of the (head, dim) grid).
template <int D>
struct DecodeSmem {
  float q[kMaxG][D];
  float k[kKC][D];
  float v[kKC][D];
  float s[kMaxG][kKC];
  float m[kMaxG], l[kMaxG], corr[kMaxG];
  float bmax[kMaxG];
};

template <typename T, int D>
__device__ __forceinline__ void stage(DecodeSmem<D>& sm, const T* k, const T* v, const int* pos) {
  for (int e = threadIdx.x; e < kKC * D; e += kThreads) {
    const int kk = e / D, dd = e % D;
    const int p = pos[kk];
    sm.k[kk][dd] = p >= 0 ? Elem<T>::load(k + (size_t)p * D + dd) : 0.0f;
    sm.v[kk][dd] = p >= 0 ? Elem<T>::load(v + (size_t)p * D + dd) : 0.0f;
  }
}

// One chunk of keys for G heads: logits, online update of (m, l) and acc.
template <int D, int R>
__device__ __forceinline__ void chunk_update(DecodeSmem<D>& sm, int G, const int* pos, float (&acc)[R],
                                             bool track_bmax) {
  for (int p = threadIdx.x; p < G * kKC; p += kThreads) {
    const int hh = p / kKC, kk = p % kKC;
    float s = -INFINITY;
    if (pos[kk] >= 0) {
      s = 0.0f;
#pragma unroll 8
      for (int dd = 0; dd < D; ++dd) s = fmaf(sm.q[hh][dd], sm.k[kk][dd], s);
    }
    sm.s[hh][kk] = s;
  }
  __syncthreads();
  if (threadIdx.x < G) {
    const int hh = threadIdx.x;
    float mx = -INFINITY;
    for (int kk = 0; kk < kKC; ++kk) mx = fmaxf(mx, sm.s[hh][kk]);
    if (track_bmax) sm.bmax[hh] = fmaxf(sm.bmax[hh], mx);
    const float mnew = fmaxf(sm.m[hh], mx);
    const float corr = mnew == -INFINITY ? 1.0f : exp2f(sm.m[hh] - mnew);
    float sum = 0.0f;
    for (int kk = 0; kk < kKC; ++kk) {
      const float e = sm.s[hh][kk] == -INFINITY ? 0.0f : exp2f(sm.s[hh][kk] - mnew);
      sm.s[hh][kk] = e;
      sum += e;
    }
    sm.l[hh] = sm.l[hh] * corr + sum;
    sm.m[hh] = mnew;
    sm.corr[hh] = corr;
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int e = threadIdx.x + kThreads * r;
    if (e < G * D) {
      const int hh = e / D, dd = e % D;
      float a = acc[r] * sm.corr[hh];
      for (int kk = 0; kk < kKC; ++kk) a = fmaf(sm.s[hh][kk], sm.v[kk][dd], a);
      acc[r] = a;
    }
  }
  __syncthreads();
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) decode_full_split_kernel(DecodeDims d, const T* __restrict__ q,
                                                                     const T* __restrict__ kc,
                                                                     const T* __restrict__ vc,
                                                                     const int* __restrict__ seqlens,
                                                                     float* __restrict__ pm, float* __restrict__ pl,
                                                                     float* __restrict__ pacc,
                                                                     float* __restrict__ bmax_out, int nsplit) {
  constexpr int R = kMaxG * D / kThreads;
  __shared__ DecodeSmem<D> sm;
  __shared__ int spos[kKC];
  const int sp = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int G = d.G();
  const int Lb = seqlens ? max(1, min(seqlens[b], d.L)) : d.L;
  const float qscale = kLog2e / sqrtf((float)D);
  for (int e = threadIdx.x; e < G * D; e += kThreads)
    sm.q[e / D][e % D] = Elem<T>::load(q + ((size_t)b * d.Hq + g * G) * D + e) * qscale;
  if (threadIdx.x < G) {
    sm.m[threadIdx.x] = -INFINITY;
    sm.l[threadIdx.x] = 0.0f;
  }
  float acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.0f;
  const size_t kvoff = ((size_t)b * d.Hkv + g) * d.L * D;
  const int k0 = sp * kSplit, k1 = min(Lb, k0 + kSplit);
  for (int blk0 = k0; blk0 < k1; blk0 += 64) {
    if (threadIdx.x < G) sm.bmax[threadIdx.x] = -INFINITY;
    for (int c0 = blk0; c0 < blk0 + 64; c0 += kKC) {
      __syncthreads();
      if (threadIdx.x < kKC) spos[threadIdx.x] = (c0 + (int)threadIdx.x < k1) ? c0 + (int)threadIdx.x : -1;
      __syncthreads();
      stage<T, D>(sm, kc + kvoff, vc + kvoff, spos);
      __syncthreads();
      chunk_update<D, R>(sm, G, spos, acc, true);
    }
    if (threadIdx.x < G) bmax_out[((size_t)b * d.Hq + g * G + threadIdx.x) * d.NB + blk0 / 64] = sm.bmax[threadIdx.x];
  }
  __syncthreads();
  const size_t pbase = ((size_t)b * d.Hq + g * G) * nsplit;
  if (threadIdx.x < G) {
    pm[pbase + (size_t)threadIdx.x * nsplit + sp] = sm.m[threadIdx.x];
    pl[pbase + (size_t)threadIdx.x * nsplit + sp] = sm.l[threadIdx.x];
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int e = threadIdx.x + kThreads * r;
    if (e < G * D) {
      const int hh = e / D, dd = e % D;
      pacc[((pbase + (size_t)hh * nsplit + sp) * D) + dd] = acc[r];
    }
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) decode_combine_kernel(DecodeDims d, const int* __restrict__ seqlens,
                                                                  const float* __restrict__ pm,
                                                                  const float* __restrict__ pl,
                                                                  const float* __restrict__ pacc,
                                                                  const float* __restrict__ bmax, T* __restrict__ o,
                                                                  float* __restrict__ scores, int nsplit,
                                                                  int red_max) {
  __shared__ float sM[kMaxG], sInvL[kMaxG];
  const int g = blockIdx.x, b = blockIdx.y;
  const int G = d.G();
  const int Lb = seqlens ? max(1, min(seqlens[b], d.L)) : d.L;
  const int ns_b = (Lb + kSplit - 1) / kSplit;
  const int nb_b = (Lb + 63) / 64;
  const size_t pbase = ((size_t)b * d.Hq + g * G) * nsplit;
  if (threadIdx.x < G) {
    const int hh = threadIdx.x;
    float M = -INFINITY;
    for (int s = 0; s < ns_b; ++s) M = fmaxf(M, pm[pbase + (size_t)hh * nsplit + s]);
    float L = 0.0f;
    for (int s = 0; s < ns_b; ++s) L += pl[pbase + (size_t)hh * nsplit + s] * exp2f(pm[pbase + (size_t)hh * nsplit + s] - M);
    sM[hh] = M;
    sInvL[hh] = 1.0f / L;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < G * D; e += kThreads) {
    const int hh = e / D, dd = e % D;
    float a = 0.0f;
    for (int s = 0; s < ns_b; ++s)
      a = fmaf(pacc[(pbase + (size_t)hh * nsplit + s) * D + dd], exp2f(pm[pbase + (size_t)hh * nsplit + s] - sM[hh]), a);
    Elem<T>::store(o + ((size_t)b * d.Hq + g * G + hh) * D + dd, a * sInvL[hh]);
  }
  for (int j = threadIdx.x; j < d.NB; j += kThreads) {
    float a = 0.0f;
    if (j < nb_b) {
      for (int hh = 0; hh < G; ++hh) {
        const float x = exp2f(bmax[((size_t)b * d.Hq + g * G + hh) * d.NB + j] - sM[hh]) * sInvL[hh];
        a = hh == 0 ? x : (red_max ? fmaxf(a, x) : a + x);
      }
    }
    scores[((size_t)b * d.Hkv + g) * d.NB + j] = a;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) decode_sparse_kernel(DecodeDims d, const T* __restrict__ q,
                                                                 const T* __restrict__ kc, const T* __restrict__ vc,
                                                                 const int* __restrict__ seqlens,
                                                                 const int* __restrict__ idx, int kb,
                                                                 const T* __restrict__ kr, const T* __restrict__ vr,
                                                                 int W, const int* __restrict__ swa_len,
                                                                 const float* __restrict__ gate,
                                                                 const float* __restrict__ sinks, T* __restrict__ o) {
  constexpr int R = kMaxG * D / kThreads;
  __shared__ DecodeSmem<D> sm;
  __shared__ int spos[kKC];
  __shared__ float sM1[kMaxG], sL1[kMaxG];
  const int g = blockIdx.x, b = blockIdx.y;
  const int G = d.G();
  const int Lb = seqlens ? max(1, min(seqlens[b], d.L)) : d.L;
  const int nring = swa_len ? max(0, min(swa_len[b], W)) : W;
  const float qscale = kLog2e / sqrtf((float)D);
  for (int e = threadIdx.x; e < G * D; e += kThreads)
    sm.q[e / D][e % D] = Elem<T>::load(q + ((size_t)b * d.Hq + g * G) * D + e) * qscale;
  if (threadIdx.x < G) {
    sm.m[threadIdx.x] = -INFINITY;
    sm.l[threadIdx.x] = 0.0f;
  }
  float acc[R], acc1[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.0f;
  const size_t kvoff = ((size_t)b * d.Hkv + g) * d.L * D;
  const int* sel = idx + ((size_t)b * d.Hkv + g) * kb;
  const int nbl = (Lb + 63) / 64;
  // sparse branch: all cached tokens of the selected blocks
  for (int s = 0; s < kb; ++s) {
    const int j = sel[s];
    if (j < 0 || j >= nbl) continue;
    for (int c0 = j * 64; c0 < j * 64 + 64; c0 += kKC) {
      __syncthreads();
      if (threadIdx.x < kKC) spos[threadIdx.x] = (c0 + (int)threadIdx.x < Lb) ? c0 + (int)threadIdx.x : -1;
      __syncthreads();
      stage<T, D>(sm, kc + kvoff, vc + kvoff, spos);
      __syncthreads();
      chunk_update<D, R>(sm, G, spos, acc, false);
    }
  }
  __syncthreads();
  if (threadIdx.x < G) {
    sM1[threadIdx.x] = sm.m[threadIdx.x];
    sL1[threadIdx.x] = sm.l[threadIdx.x];
    sm.m[threadIdx.x] = -INFINITY;
    sm.l[threadIdx.x] = 0.0f;
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    acc1[r] = acc[r];
    acc[r] = 0.0f;
  }
  // SWA branch: the layer's own ring (order irrelevant)
  const size_t roff = ((size_t)b * d.Hkv + g) * W * D;
  for (int c0 = 0; c0 < nring; c0 += kKC) {
    __syncthreads();
    if (threadIdx.x < kKC) spos[threadIdx.x] = (c0 + (int)threadIdx.x < nring) ? c0 + (int)threadIdx.x : -1;
    __syncthreads();
    stage<T, D>(sm, kr + roff, vr + roff, spos);
    __syncthreads();
    chunk_update<D, R>(sm, G, spos, acc, false);
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int e = threadIdx.x + kThreads * r;
    if (e < G * D) {
      const int hh = e / D, dd = e % D;
      const int h = g * G + hh;
      const float g0 = sigmoidf_(gate[((size_t)b * d.Hq + h) * 2 + 0]);
      const float g1 = sigmoidf_(gate[((size_t)b * d.Hq + h) * 2 + 1]);
      // each branch's sink logit joins its softmax as an entry with a zero value (log2 units)
      const float l1 = sL1[hh] + (sinks ? exp2f(sinks[2 * h] * kLog2e - sM1[hh]) : 0.0f);
      const float l2 = sm.l[hh] + (sinks ? exp2f(sinks[2 * h + 1] * kLog2e - sm.m[hh]) : 0.0f);
      const float a = l1 > 0.0f ? acc1[r] * (g0 / l1) : 0.0f;
      const float c = l2 > 0.0f ? acc[r] * (g1 / l2) : 0.0f;
      Elem<T>::store(o + ((size_t)b * d.Hq + h) * D + dd, a + c);
    }
  }
}

inline int num_splits(const DecodeDims& d) { return (d.L + kSplit - 1) / kSplit; }

template <typename T, int D>
cudaError_t decode_full_typed(const DecodeDims& d, const void* q, const void* kc, const void* vc,
                              const int* seqlens, void* o, float* scores, hys_reduce red, void* ws, cudaStream_t s) {
  const int ns = num_splits(d);
  float* pm = (float*)ws;
  float* pl = pm + (size_t)d.B * d.Hq * ns;
  float* pacc = pl + (size_t)d.B * d.Hq * ns;
  float* bmax = pacc + (size_t)d.B * d.Hq * ns * D;
  dim3 g1(ns, d.Hkv, d.B);
  decode_full_split_kernel<T, D><<<g1, kThreads, 0, s>>>(d, (const T*)q, (const T*)kc, (const T*)vc, seqlens, pm,
                                                         pl, pacc, bmax, ns);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2(d.Hkv, d.B);
  decode_combine_kernel<T, D><<<g2, kThreads, 0, s>>>(d, seqlens, pm, pl, pacc, bmax, (T*)o, scores, ns,
                                                      red == HYS_REDUCE_MAX);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t decode_sparse_typed(const DecodeDims& d, const void* q, const void* kc, const void* vc,
                                const int* seqlens, const int* idx, int kb, const void* kr, const void* vr, int W,
                                const int* swa_len, const float* gate, const float* sinks, void* o, cudaStream_t s) {
  dim3 grid(d.Hkv, d.B);
  decode_sparse_kernel<T, D><<<grid, kThreads, 0, s>>>(d, (const T*)q, (const T*)kc, (const T*)vc, seqlens, idx, kb,
                                                       (const T*)kr, (const T*)vr, W, swa_len, gate, sinks, (T*)o);
  return cudaGetLastError();
}

}  // namespace

size_t decode_full_workspace(const DecodeDims& d) {
  const size_t ns = num_splits(d);
  return sizeof(float) * ((size_t)d.B * d.Hq * ns * (2 + d.D) + (size_t)d.B * d.Hq * d.NB);
}

cudaError_t launch_decode_full(const DecodeDims& d, hys_dtype dt, const void* q, const void* kc, const void* vc,
                               const int* seqlens, void* o, float* scores, hys_reduce red, void* ws,
                               cudaStream_t s) {
  if (dt == HYS_F32)
    return d.D == 64 ? decode_full_typed<float, 64>(d, q, kc, vc, seqlens, o, scores, red, ws, s)
                     : decode_full_typed<float, 128>(d, q, kc, vc, seqlens, o, scores, red, ws, s);
  return d.D == 64 ? decode_full_typed<__nv_bfloat16, 64>(d, q, kc, vc, seqlens, o, scores, red, ws, s)
                   : decode_full_typed<__nv_bfloat16, 128>(d, q, kc, vc, seqlens, o, scores, red, ws, s);
}

cudaError_t launch_decode_sparse(const DecodeDims& d, hys_dtype dt, const void* q, const void* kc, const void* vc,
                                 const int* seqlens, const int* idx, int kb, const void* kr, const void* vr, int W,
                                 const int* swa_len, const float* gate, const float* sinks, void* o, cudaStream_t s) {
  if (dt == HYS_F32)
    return d.D == 64
               ? decode_sparse_typed<float, 64>(d, q, kc, vc, seqlens, idx, kb, kr, vr, W, swa_len, gate, sinks, o, s)
               : decode_sparse_typed<float, 128>(d, q, kc, vc, seqlens, idx, kb, kr, vr, W, swa_len, gate, sinks, o, s);
  return d.D == 64 ? decode_sparse_typed<__nv_bfloat16, 64>(d, q, kc, vc, seqlens, idx, kb, kr, vr, W, swa_len, gate,
                                                            sinks, o, s)
                   : decode_sparse_typed<__nv_bfloat16, 128>(d, q, kc, vc, seqlens, idx, kb, kr, vr, W, swa_len, gate,
                                                             sinks, o, s);
}

}  // namespace hys
