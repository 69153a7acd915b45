// TopK selection over block scores (HySparse 3.4.2) and over token scores with a forced
// recent window (HySparse2 explainer, "Precise retrieval without a separate indexer").
//
// Order: score descending, index ascending (ties go to the lower index).  The comparison
// runs on an order-preserving uint32 image of the fp32 score, so the selection is a
// deterministic function of the emitted scores.  Output indices are ascending and padded
// with -1.
#include "common.cuh"
#include "kernels.h"

namespace hys {

namespace {

constexpr int kTopkThreads = 256;

// Block-wide exclusive scan of one int per thread (blockDim.x == 256 or 1024).
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int x, int* total, int* sbuf /* >= NT/32 + 1 */) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) sbuf[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < NT / 32 ? sbuf[lane] : 0;
    int wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += y;
    }
    if (lane < NT / 32) sbuf[lane] = wi - w;
    if (lane == NT / 32 - 1) sbuf[NT / 32] = wi;
  }
  __syncthreads();
  const int res = sbuf[warp] + incl - x;
  *total = sbuf[NT / 32];
  __syncthreads();
  return res;
}

// One CTA per (b, g, I) row of candidates.  Candidates live in shared memory as keys;
// the rank of candidate c is the number of candidates that beat it.
__global__ void __launch_bounds__(kTopkThreads) topk_blocks_kernel(const float* __restrict__ scores,
                                                                   int* __restrict__ idx, int Hkv, int T, int NB,
                                                                   int k, const int* __restrict__ seqlens, int L,
                                                                   int decode) {
  extern __shared__ uint32_t skey[];  // NB keys
  __shared__ int sbuf[kTopkThreads / 32 + 1];
  const int row = blockIdx.x;
  int n;
  if (decode) {
    const int b = row / Hkv;
    const int Lb = seqlens ? max(1, min(seqlens[b], L)) : L;
    n = min(NB, (Lb + 63) / 64);
  } else {
    n = min(NB, row % T + 1);
  }
  const float* srow = scores + (size_t)row * NB;
  for (int c = threadIdx.x; c < n; c += kTopkThreads) skey[c] = order_key(srow[c]);
  __syncthreads();
  // contiguous segment per thread so that a scan gives ascending output positions
  const int seg = (n + kTopkThreads - 1) / kTopkThreads;
  const int c0 = min(n, threadIdx.x * seg), c1 = min(n, c0 + seg);
  uint32_t selmask = 0;  // seg <= 32 (n <= 8192)
  int cnt = 0;
  for (int c = c0; c < c1; ++c) {
    const uint32_t kc = skey[c];
    int rank = 0;
    for (int j = 0; j < n && rank < k; ++j) {
      const uint32_t kj = skey[j];
      rank += (kj > kc) || (kj == kc && j < c);
    }
    if (rank < k) {
      selmask |= 1u << (c - c0);
      ++cnt;
    }
  }
  int total;
  int pos = block_exclusive_scan<kTopkThreads>(cnt, &total, sbuf);
  int* out = idx + (size_t)row * k;
  for (int c = c0; c < c1; ++c)
    if (selmask & (1u << (c - c0))) out[pos++] = c;
  for (int p = total + threadIdx.x; p < k; p += kTopkThreads) out[p] = -1;
}

// ------------------------------------------------------------------ token top-k
constexpr int kTokThreads = 1024;

// One CTA per (b, g, I).  Radix select (4 passes of 8 bits) finds the k-th largest key;
// then one ordered sweep takes every key above it plus the lowest-index ties.
__global__ void __launch_bounds__(kTokThreads) topk_tokens_kernel(const float* __restrict__ scores,
                                                                  int* __restrict__ idx, int T, int N, int k,
                                                                  int forced) {
  __shared__ int hist[256];
  __shared__ int sbuf[kTokThreads / 32 + 1];
  __shared__ uint32_t s_prefix, s_need;
  const int row = blockIdx.x;
  const int I = row % T;
  const int e = min(N, (I + 1) * 64) - 1;
  const int n = max(0, e - forced + 1);
  const float* srow = scores + (size_t)row * N;
  int* out = idx + (size_t)row * k;
  const int tid = threadIdx.x;

  if (n <= k) {
    for (int c = tid; c < k; c += kTokThreads) out[c] = c < n ? c : -1;
    return;
  }
  // radix select of the k-th largest key
  uint32_t prefix = 0, pmask = 0;
  int need = k;  // how many to take among keys matching the prefix
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int c = tid; c < 256; c += kTokThreads) hist[c] = 0;
    __syncthreads();
    for (int c = tid; c < n; c += kTokThreads) {
      const uint32_t key = order_key(srow[c]);
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    if (tid == 0) {
      int acc = 0, bin = 255;
      for (; bin > 0; --bin) {
        if (acc + hist[bin] >= need) break;
        acc += hist[bin];
      }
      s_prefix = prefix | ((uint32_t)bin << shift);
      s_need = (uint32_t)(need - acc);
    }
    __syncthreads();
    prefix = s_prefix;
    need = (int)s_need;
    pmask |= 255u << shift;
    __syncthreads();
  }
  // prefix is now the k-th largest key; take all greater keys and the `need` lowest-index ties
  const uint32_t kth = prefix;
  int ties_before = 0, written = 0;
  for (int base = 0; base < n; base += kTokThreads) {
    const int c = base + tid;
    uint32_t key = 0;
    if (c < n) key = order_key(srow[c]);
    const int is_tie = (c < n && key == kth) ? 1 : 0;
    int tie_total;
    const int tie_rank = ties_before + block_exclusive_scan<kTokThreads>(is_tie, &tie_total, sbuf);
    ties_before += tie_total;
    const int sel = (c < n) && (key > kth || (is_tie && tie_rank < need));
    int sel_total;
    const int pos = written + block_exclusive_scan<kTokThreads>(sel, &sel_total, sbuf);
    if (sel) out[pos] = c;
    written += sel_total;
  }
  for (int p = written + tid; p < k; p += kTokThreads) out[p] = -1;
}

}  // namespace

cudaError_t launch_topk_blocks(const float* scores, int* idx, int B, int Hkv, int T, int NB, int k,
                               const int* seqlens, int L, bool decode, cudaStream_t s) {
  const int rows = decode ? B * Hkv : B * Hkv * T;
  const size_t smem = (size_t)NB * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(topk_blocks_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  topk_blocks_kernel<<<rows, kTopkThreads, smem, s>>>(scores, idx, Hkv, T, NB, k, seqlens, L, decode ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_topk_tokens(const PrefillDims& d, const float* scores, int k_tokens, int forced, int* idx,
                               cudaStream_t s) {
  topk_tokens_kernel<<<d.B * d.Hkv * d.T, kTokThreads, 0, s>>>(scores, idx, d.T, d.N, k_tokens, forced);
  return cudaGetLastError();
}

}  // namespace hys
