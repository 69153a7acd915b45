// Backward of the hybrid block's layers: the row statistics, the inverse selection lists, the SIMT
// fp32-accumulate kernels (fp32 inputs and shapes the tcgen05 backward does not take) and the
// host sequences of the full-layer and sparse-layer backward.
//
// Gradients ([HS] 3.4.6, training: the selected blocks are constants of the step; the sparse
// layers' gradients reach the full layer's K, V through the shared cache).  For attention over a
// key set with p = softmax(tau q.k) (sink logits join as entries with a zero value) and a per-row
// factor sigma_t on the output (the branch's sigmoid gate, 1 for the full layer):
//   D_t  = sigma_t dO_t . o_t                    (o_t the branch output)
//   dS   = p (sigma_t dO_t . v_i - D_t)
//   dV_i = sum_t sigma_t p_ti dO_t,  dK_i = tau sum_t dS_ti q_t,  dQ_t = tau sum_i dS_ti k_i
//   d(sink) = -sum_t p_sink,t D_t
// and for the gated sparse layer o = sigmoid(g0) o~ + sigmoid(g1) o' ([HS] 3.4.3):
//   d g_b = sigmoid(g_b) (1 - sigmoid(g_b)) dO . o_b = (1 - sigmoid(g_b)) D^b_t.
// The training forward of the sparse layer saves each branch's LSE and the gated sparse part
// sigmoid(g0) o~; then D^sp = dO . (sigmoid(g0) o~) and D^sw = dO . o - D^sp need no recomputation.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace hys {
namespace {

constexpr int kModeFull = 0, kModeWindow = 1, kModeSparse = 2;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// dot product of two rows of D elements, one warp, D / 32 elements per lane
template <typename T, int D>
__device__ __forceinline__ float row_dot(const T* a, const T* b, int lane) {
  float acc = 0.0f;
#pragma unroll
  for (int c = 0; c < D / 32; ++c) acc = fmaf(Elem<T>::load(a + lane + 32 * c), Elem<T>::load(b + lane + 32 * c), acc);
  return warp_sum(acc);
}

// ------------------------------------------------------------------------------ row statistics
// Full layer: lse2 = LSE * log2(e) and D_t = dO_t . o_t, one warp per row.
template <typename T, int D>
__global__ void rows_full_kernel(const float* __restrict__ lse, const T* __restrict__ o, const T* __restrict__ d_o,
                                 float* __restrict__ lse2, float* __restrict__ dsum, long long rows) {
  const long long r = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const float a = row_dot<T, D>(o + r * D, d_o + r * D, lane);
  if (lane == 0) {
    dsum[r] = a;
    lse2[r] = lse[r] * kLog2e;
  }
}

// Sparse layer: per row and branch b in {sparse, window}: lse2_b, D^b, sigma_b; the gate gradient
// (1 - sigma_b) D^b; the sink gradients -exp(sink_b - LSE_b) D^b summed per head (atomics).
template <typename T, int D>
__global__ void rows_sparse_kernel(PrefillDims d, const float* __restrict__ blse, const T* __restrict__ o,
                                   const T* __restrict__ osp, const T* __restrict__ d_o,
                                   const float* __restrict__ gate, const float* __restrict__ sinks,
                                   float* __restrict__ rows6, float* __restrict__ dgate, float* __restrict__ dsinks,
                                   long long rows, long long stride) {
  const long long r = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const float dsp = row_dot<T, D>(osp + r * D, d_o + r * D, lane);
  const float dall = row_dot<T, D>(o + r * D, d_o + r * D, lane);
  if (lane != 0) return;
  const float dsw = dall - dsp;
  const float2 gl = reinterpret_cast<const float2*>(gate)[r];
  const float s0 = sigmoidf_(gl.x), s1 = sigmoidf_(gl.y);
  const float2 l = reinterpret_cast<const float2*>(blse)[r];
  rows6[0 * stride + r] = l.x * kLog2e;
  rows6[1 * stride + r] = dsp;
  rows6[2 * stride + r] = s0;
  rows6[3 * stride + r] = l.y * kLog2e;
  rows6[4 * stride + r] = dsw;
  rows6[5 * stride + r] = s1;
  reinterpret_cast<float2*>(dgate)[r] = make_float2((1.0f - s0) * dsp, (1.0f - s1) * dsw);
  if (sinks != nullptr) {
    const int h = (int)((r / d.N) % d.Hq);
    const float k0 = sinks[2 * h], k1 = sinks[2 * h + 1];
    if (l.x > -INFINITY) atomicAdd(dsinks + 2 * h, -__expf(k0 - l.x) * dsp);
    if (l.y > -INFINITY) atomicAdd(dsinks + 2 * h + 1, -__expf(k1 - l.y) * dsw);
  }
}

// ------------------------------------------------------------------------------ inverse selection
// mask[(bg * NK + j / 2) * T + I] |= 1 << (j & 1) for every selected block j <= I of tile I
__global__ void sel_scatter_kernel(const int* __restrict__ idx, int kb, int T, int NK, long long n,
                                   unsigned* __restrict__ mask) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n) return;
  const int j = idx[e];
  const long long row = e / kb;            // (bg, I)
  const int I = (int)(row % T);
  const long long bg = row / T;
  if (j < 0 || j > I) return;
  atomicOr(mask + ((size_t)bg * NK + j / 2) * T + I, 1u << (j & 1));
}

// per (bg, key tile kt): the query tiles I >= 2 kt whose mask is set, ascending, as I << 2 | mask
__global__ void sel_compact_kernel(const unsigned* __restrict__ mask, int T, int NK, int units, int* __restrict__ list,
                                   int* __restrict__ cnt) {
  const int u = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (u >= units) return;
  const int kt = u % NK;
  const unsigned* m = mask + (size_t)u * T;
  int* out = list + (size_t)u * T;
  int n = 0;
  for (int I0 = 2 * kt; I0 < T; I0 += 32) {
    const int I = I0 + lane;
    const unsigned mk = I < T ? m[I] : 0u;
    const unsigned bal = __ballot_sync(0xffffffffu, mk != 0u);
    if (mk != 0u) out[n + __popc(bal & ((1u << lane) - 1u))] = (I << 2) | (int)mk;
    n += __popc(bal);
  }
  if (lane == 0) cnt[u] = n;
}

// ------------------------------------------------------------------------------ SIMT backward
// dq_acc[row] += sum over the row's visible keys of dS_ti k_i (unscaled), one warp per row.
template <typename T, int D, int MODE>
__global__ void simt_dq_kernel(PrefillDims d, const T* __restrict__ q, const T* __restrict__ d_o,
                               const T* __restrict__ k, const T* __restrict__ v, const float* __restrict__ lse2,
                               const float* __restrict__ dsum, const float* __restrict__ sig,
                               const int* __restrict__ idx, int kb, int window, float* __restrict__ dq_acc) {
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)d.B * d.Hq * d.N;
  if (row >= rows) return;
  const int t = (int)(row % d.N);
  const int h = (int)((row / d.N) % d.Hq);
  const int b = (int)(row / ((long long)d.N * d.Hq));
  const int g = h / d.G();
  const T* kk = k + ((size_t)b * d.Hkv + g) * d.N * D;
  const T* vv = v + ((size_t)b * d.Hkv + g) * d.N * D;
  const T* qr = q + row * D;
  const T* dr = d_o + row * D;
  const float sc = kLog2e / sqrtf((float)D);
  const float l2 = lse2[row], dd = dsum[row], sg = sig ? sig[row] : 1.0f;
  float acc[D / 32];
#pragma unroll
  for (int c = 0; c < D / 32; ++c) acc[c] = 0.0f;
  auto visit = [&](int i) {
    const float s = row_dot<T, D>(qr, kk + (size_t)i * D, lane);
    const float dp = row_dot<T, D>(dr, vv + (size_t)i * D, lane);
    const float p = exp2f(s * sc - l2);
    const float ds = p * (sg * dp - dd);
#pragma unroll
    for (int c = 0; c < D / 32; ++c) acc[c] = fmaf(ds, Elem<T>::load(kk + (size_t)i * D + lane + 32 * c), acc[c]);
  };
  if (MODE == kModeFull) {
    for (int i = 0; i <= t; ++i) visit(i);
  } else if (MODE == kModeWindow) {
    for (int i = max(0, t - window + 1); i <= t; ++i) visit(i);
  } else {
    const int I = t / 64;
    const int* sel = idx + (((size_t)b * d.Hkv + g) * d.T + I) * kb;
    for (int e = 0; e < kb; ++e) {
      const int j = sel[e];
      if (j < 0 || j > I) continue;
      for (int i = 64 * j; i <= min(64 * j + 63, t); ++i) visit(i);
    }
  }
  float* out = dq_acc + row * D;
#pragma unroll
  for (int c = 0; c < D / 32; ++c) out[lane + 32 * c] += acc[c];
}

// dK, dV of one key i (one warp): the rows of every head of the group that attend it.
template <typename T, int D, int MODE>
__global__ void simt_dkv_kernel(PrefillDims d, const T* __restrict__ q, const T* __restrict__ d_o,
                                const T* __restrict__ k, const T* __restrict__ v, const float* __restrict__ lse2,
                                const float* __restrict__ dsum, const float* __restrict__ sig,
                                const int* __restrict__ list, const int* __restrict__ list_cnt, int window,
                                float* __restrict__ dk, float* __restrict__ dv, int accumulate) {
  const long long key = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long keys = (long long)d.B * d.Hkv * d.N;
  if (key >= keys) return;
  const int i = (int)(key % d.N);
  const long long bg = key / d.N;
  const int g = (int)(bg % d.Hkv), b = (int)(bg / d.Hkv);
  const int G = d.G();
  const T* krow = k + key * D;
  const T* vrow = v + key * D;
  const float sc = kLog2e / sqrtf((float)D);
  float ak[D / 32], av[D / 32];
#pragma unroll
  for (int c = 0; c < D / 32; ++c) ak[c] = av[c] = 0.0f;
  auto visit = [&](int t) {
    for (int h = g * G; h < (g + 1) * G; ++h) {
      const long long row = ((long long)b * d.Hq + h) * d.N + t;
      const T* qr = q + row * D;
      const T* dr = d_o + row * D;
      const float s = row_dot<T, D>(qr, krow, lane);
      const float dp = row_dot<T, D>(dr, vrow, lane);
      const float sg = sig ? sig[row] : 1.0f;
      const float p = exp2f(s * sc - lse2[row]);
      const float ds = p * (sg * dp - dsum[row]);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        av[c] = fmaf(sg * p, Elem<T>::load(dr + lane + 32 * c), av[c]);
        ak[c] = fmaf(ds, Elem<T>::load(qr + lane + 32 * c), ak[c]);
      }
    }
  };
  if (MODE == kModeFull) {
    for (int t = i; t < d.N; ++t) visit(t);
  } else if (MODE == kModeWindow) {
    for (int t = i; t < min(d.N, i + window); ++t) visit(t);
  } else {
    const int NK = (d.N + 127) / 128;
    const size_t lu = (size_t)bg * NK + i / 128;
    const int n = list_cnt[lu];
    const int half = (i / 64) & 1;
    for (int e = 0; e < n; ++e) {
      const int ent = list[lu * d.T + e];
      if (!((ent >> half) & 1)) continue;
      const int I = ent >> 2;
      for (int t = max(i, 64 * I); t < min(d.N, 64 * I + 64); ++t) visit(t);
    }
  }
  const float tau = 1.0f / sqrtf((float)D);
  float* kout = dk + key * D;
  float* vout = dv + key * D;
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    const float a = ak[c] * tau, bv = av[c];
    kout[lane + 32 * c] = accumulate ? kout[lane + 32 * c] + a : a;
    vout[lane + 32 * c] = accumulate ? vout[lane + 32 * c] + bv : bv;
  }
}

template <typename T>
__global__ void dq_out_kernel(const float* __restrict__ acc, T* __restrict__ dq, float tau, long long n) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) Elem<T>::store(dq + i, acc[i] * tau);
}

unsigned blocks_for(long long n, int per_block) { return (unsigned)((n + per_block - 1) / per_block); }

template <typename T, int D, int MODE>
cudaError_t simt_pass(const PrefillDims& d, const void* q, const void* d_o, const void* k, const void* v,
                      const float* lse2, const float* dsum, const float* sig, const int* idx, int kb,
                      const int* list, const int* list_cnt, int window, float* dq_acc, float* dk, float* dv,
                      int accumulate, cudaStream_t s) {
  const long long rows = (long long)d.B * d.Hq * d.N, keys = (long long)d.B * d.Hkv * d.N;
  simt_dq_kernel<T, D, MODE><<<blocks_for(rows, 8), 256, 0, s>>>(d, (const T*)q, (const T*)d_o, (const T*)k,
                                                                 (const T*)v, lse2, dsum, sig, idx, kb, window,
                                                                 dq_acc);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  simt_dkv_kernel<T, D, MODE><<<blocks_for(keys, 8), 256, 0, s>>>(d, (const T*)q, (const T*)d_o, (const T*)k,
                                                                  (const T*)v, lse2, dsum, sig, list, list_cnt,
                                                                  window, dk, dv, accumulate);
  return cudaGetLastError();
}

template <int MODE>
cudaError_t simt_pass_any(const PrefillDims& d, hys_dtype dt, const void* q, const void* d_o, const void* k,
                          const void* v, const float* lse2, const float* dsum, const float* sig, const int* idx,
                          int kb, const int* list, const int* list_cnt, int window, float* dq_acc, float* dk,
                          float* dv, int accumulate, cudaStream_t s) {
#define HYS_SIMT_PASS(T, DD)                                                                                   \
  simt_pass<T, DD, MODE>(d, q, d_o, k, v, lse2, dsum, sig, idx, kb, list, list_cnt, window, dq_acc, dk, dv, \
                         accumulate, s)
  if (dt == HYS_F32) return d.D == 64 ? HYS_SIMT_PASS(float, 64) : HYS_SIMT_PASS(float, 128);
  return d.D == 64 ? HYS_SIMT_PASS(__nv_bfloat16, 64) : HYS_SIMT_PASS(__nv_bfloat16, 128);
#undef HYS_SIMT_PASS
}

cudaError_t dq_out(hys_dtype dt, const float* acc, void* dq, long long n, float tau, cudaStream_t s) {
  if (dt == HYS_F32)
    dq_out_kernel<float><<<blocks_for(n, 256), 256, 0, s>>>(acc, (float*)dq, tau, n);
  else
    dq_out_kernel<__nv_bfloat16><<<blocks_for(n, 256), 256, 0, s>>>(acc, (__nv_bfloat16*)dq, tau, n);
  return cudaGetLastError();
}

// workspace of the sparse-layer backward
struct SparseWs {
  int* counter;
  float* rows6;     // 6 x rows: lse2_sp, D_sp, sigma0, lse2_sw, D_sw, sigma1
  float* dq_acc;    // rows x D
  unsigned* mask;   // units x T
  int* list;        // units x T
  int* cnt;         // units
  size_t bytes;
};

SparseWs carve_sparse(const PrefillDims& d, void* base) {
  const size_t rows = (size_t)d.B * d.Hq * d.N;
  const size_t units = (size_t)d.B * d.Hkv * ((d.N + 127) / 128);
  uint8_t* w = reinterpret_cast<uint8_t*>(base);
  SparseWs x;
  size_t off = 0;
  x.counter = reinterpret_cast<int*>(w + off);
  off += 256;
  x.rows6 = reinterpret_cast<float*>(w + off);
  off += align256(6 * rows * 4);
  x.dq_acc = reinterpret_cast<float*>(w + off);
  off += align256(rows * d.D * 4);
  x.mask = reinterpret_cast<unsigned*>(w + off);
  off += align256(units * d.T * 4);
  x.list = reinterpret_cast<int*>(w + off);
  off += align256(units * d.T * 4);
  x.cnt = reinterpret_cast<int*>(w + off);
  off += align256(units * 4);
  x.bytes = off;
  return x;
}

}  // namespace

// ------------------------------------------------------------------------------ full layer
size_t full_bwd_workspace(const PrefillDims& d, hys_dtype dt) {
  if (attn_bwd_tc_supported(d, dt)) return full_bwd_tc_workspace(d);
  const size_t rows = (size_t)d.B * d.Hq * d.N;
  return 2 * align256(rows * 4) + rows * d.D * 4;
}

cudaError_t launch_full_bwd(const PrefillDims& d, hys_dtype dt, const void* q, const void* k, const void* v,
                            const void* o, const void* d_o, const float* lse, void* dq, float* dk, float* dv,
                            int accumulate, void* ws, cudaStream_t s) {
  if (attn_bwd_tc_supported(d, dt)) return launch_full_bwd_tc(d, q, k, v, o, d_o, lse, dq, dk, dv, accumulate, ws, s);
  const size_t rows = (size_t)d.B * d.Hq * d.N;
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  float* lse2 = reinterpret_cast<float*>(w);
  float* dsum = reinterpret_cast<float*>(w + align256(rows * 4));
  float* acc = reinterpret_cast<float*>(w + 2 * align256(rows * 4));
  cudaError_t e = cudaMemsetAsync(acc, 0, rows * d.D * 4, s);
  if (e != cudaSuccess) return e;
#define HYS_ROWS_FULL(T, DD)                                                                                    \
  rows_full_kernel<T, DD><<<blocks_for((long long)rows, 8), 256, 0, s>>>(lse, (const T*)o, (const T*)d_o, lse2, \
                                                                          dsum, (long long)rows)
  if (dt == HYS_F32) {
    if (d.D == 64) HYS_ROWS_FULL(float, 64); else HYS_ROWS_FULL(float, 128);
  } else {
    if (d.D == 64) HYS_ROWS_FULL(__nv_bfloat16, 64); else HYS_ROWS_FULL(__nv_bfloat16, 128);
  }
#undef HYS_ROWS_FULL
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = simt_pass_any<kModeFull>(d, dt, q, d_o, k, v, lse2, dsum, nullptr, nullptr, 0, nullptr, nullptr, 0, acc, dk,
                               dv, accumulate, s);
  if (e != cudaSuccess) return e;
  return dq_out(dt, acc, dq, (long long)rows * d.D, 1.0f / sqrtf((float)d.D), s);
}

// ------------------------------------------------------------------------------ sparse layer
size_t sparse_bwd_workspace(const PrefillDims& d) { return carve_sparse(d, nullptr).bytes; }

cudaError_t launch_sparse_bwd(const PrefillDims& d, hys_dtype dt, const void* q, const void* k, const void* v,
                              const int* idx, int kb, const void* ks, const void* vs, int window, const float* gate,
                              const float* sinks, const void* o, const void* osp, const float* blse, const void* d_o,
                              void* dq, float* dk, float* dv, float* dks, float* dvs, float* dgate, float* dsinks,
                              void* ws, cudaStream_t s) {
  const SparseWs x = carve_sparse(d, ws);
  const long long rows = (long long)d.B * d.Hq * d.N;
  const int NK = (d.N + 127) / 128;
  const int units = d.B * d.Hkv * NK;
  cudaError_t e;
  if (sinks != nullptr && dsinks != nullptr) {
    e = cudaMemsetAsync(dsinks, 0, (size_t)d.Hq * 2 * 4, s);
    if (e != cudaSuccess) return e;
  }
  e = cudaMemsetAsync(x.dq_acc, 0, (size_t)rows * d.D * 4, s);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(x.mask, 0, (size_t)units * d.T * 4, s);
  if (e != cudaSuccess) return e;
#define HYS_ROWS_SPARSE(T, DD)                                                                                      \
  rows_sparse_kernel<T, DD><<<blocks_for(rows, 8), 256, 0, s>>>(d, blse, (const T*)o, (const T*)osp, (const T*)d_o, \
                                                                 gate, sinks, x.rows6, dgate,                       \
                                                                 sinks != nullptr ? dsinks : nullptr, rows, rows)
  if (dt == HYS_F32) {
    if (d.D == 64) HYS_ROWS_SPARSE(float, 64); else HYS_ROWS_SPARSE(float, 128);
  } else {
    if (d.D == 64) HYS_ROWS_SPARSE(__nv_bfloat16, 64); else HYS_ROWS_SPARSE(__nv_bfloat16, 128);
  }
#undef HYS_ROWS_SPARSE
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long nidx = (long long)d.B * d.Hkv * d.T * kb;
  sel_scatter_kernel<<<blocks_for(nidx, 256), 256, 0, s>>>(idx, kb, d.T, NK, nidx, x.mask);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  sel_compact_kernel<<<blocks_for(units, 8), 256, 0, s>>>(x.mask, d.T, NK, units, x.list, x.cnt);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const float* r6 = x.rows6;
  if (attn_bwd_tc_supported(d, dt)) {
    e = launch_attn_bwd_tc_window(d, q, d_o, ks, vs, r6 + 3 * rows, r6 + 4 * rows, r6 + 5 * rows, x.dq_acc, dks, dvs,
                                  window, x.counter, s);
    if (e != cudaSuccess) return e;
    e = launch_attn_bwd_tc_sparse(d, q, d_o, k, v, r6, r6 + rows, r6 + 2 * rows, x.dq_acc, dk, dv, x.list, x.cnt,
                                  x.counter, s);
    if (e != cudaSuccess) return e;
    return launch_bwd_dq_out(x.dq_acc, dq, (size_t)rows * d.D, s);
  }
  e = simt_pass_any<kModeWindow>(d, dt, q, d_o, ks, vs, r6 + 3 * rows, r6 + 4 * rows, r6 + 5 * rows, nullptr, 0,
                                 nullptr, nullptr, window, x.dq_acc, dks, dvs, 0, s);
  if (e != cudaSuccess) return e;
  e = simt_pass_any<kModeSparse>(d, dt, q, d_o, k, v, r6, r6 + rows, r6 + 2 * rows, idx, kb, x.list, x.cnt, 0,
                                 x.dq_acc, dk, dv, 1, s);
  if (e != cudaSuccess) return e;
  return dq_out(dt, x.dq_acc, dq, rows * d.D, 1.0f / sqrtf((float)d.D), s);
}

}  // namespace hys
