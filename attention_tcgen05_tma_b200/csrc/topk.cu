// TopK selection over block scores (HySparse 3.4.2) and over token scores with a forced
// recent window (HySparse2 explainer, "Precise retrieval without a separate indexer").
//
// Order: score descending, index ascending (ties go to the lower index).  The comparison
// runs on an order-preserving uint32 image of the fp32 score, so the selection is a
// deterministic function of the emitted scores.  Output indices are ascending and padded
// with -1.
//
// One CTA per candidate row.  Radix select finds the k-th largest key in four 8-bit passes
// (per-warp histograms in shared memory, then a suffix scan over the 256 bins); one
// index-ordered sweep then takes every key above it plus the lowest-index ties, and a
// block-wide scan places them in ascending order.  On long rows (token candidates) each thread
// loads eight keys before it touches the histogram (their latencies overlap), and the sweep
// gives each thread eight consecutive keys per step, so a step costs two block scans for
// 8 * NT keys; short rows keep one key per thread and step.
#include "common.cuh"
#include "kernels.h"

namespace hys {

namespace {

// Block-wide exclusive scan of one int per thread (NT threads, NT % 32 == 0, NT <= 1024).
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

template <int NW>
struct RadixSmem {
  int hist[NW][256];  // per-warp histograms
  int sbuf[33];
  uint32_t prefix;
  int need;
};

// Select the k largest of n keys (key(c) for c in [0, n)), ties to the lower index, and write
// their indices ascending to out[0..k) (n > k is required).  NT threads, NT >= 256.
template <int NT, typename KeyFn>
__device__ void radix_topk(KeyFn key, int n, int k, int* out, RadixSmem<NT / 32>& sm) {
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0, pmask = 0;
  int need = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < NW * 256; i += NT) (&sm.hist[0][0])[i] = 0;
    __syncthreads();
    if (NT < 1024 || n <= 2 * NT) {   // short rows (block candidates): one key per thread and step
      for (int c = tid; c < n; c += NT) {
        const uint32_t kc = key(c);
        if ((kc & pmask) == prefix) atomicAdd(&sm.hist[warp][(kc >> shift) & 255u], 1);
      }
    } else for (int c0 = tid; c0 < n; c0 += 8 * NT) {
      uint32_t kv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = c0 + u * NT;
        kv[u] = c < n ? key(c) : 0u;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (c0 + u * NT < n && (kv[u] & pmask) == prefix) atomicAdd(&sm.hist[warp][(kv[u] >> shift) & 255u], 1);
    }
    __syncthreads();
    // bin counts in descending bin order: thread t < 256 owns bin 255 - t
    int cnt = 0;
    if (tid < 256) {
      const int bin = 255 - tid;
      for (int w = 0; w < NW; ++w) cnt += sm.hist[w][bin];
    }
    int total;
    const int above = block_exclusive_scan<NT>(tid < 256 ? cnt : 0, &total, sm.sbuf);  // keys in higher bins
    if (tid < 256 && above < need && above + cnt >= need) {
      sm.prefix = prefix | ((uint32_t)(255 - tid) << shift);
      sm.need = need - above;
    }
    __syncthreads();
    prefix = sm.prefix;
    need = sm.need;
    pmask |= 255u << shift;
    __syncthreads();
  }
  (void)lane;
  // prefix is the k-th largest key: take the greater keys and the `need` lowest-index ties
  const uint32_t kth = prefix;
  int ties_before = 0, written = 0;
  if (NT < 1024 || n <= 2 * NT) {
    for (int base = 0; base < n; base += NT) {
      const int c = base + tid;
      const uint32_t kc = c < n ? key(c) : 0u;
      const int is_tie = (c < n && kc == kth) ? 1 : 0;
      int tie_total;
      const int tie_rank = ties_before + block_exclusive_scan<NT>(is_tie, &tie_total, sm.sbuf);
      ties_before += tie_total;
      const int sel = (c < n) && (kc > kth || (is_tie && tie_rank < need));
      int sel_total;
      const int pos = written + block_exclusive_scan<NT>(sel, &sel_total, sm.sbuf);
      if (sel) out[pos] = c;
      written += sel_total;
    }
    return;
  }
  for (int base = 0; base < n; base += 8 * NT) {
    const int c0 = base + 8 * tid;   // this thread's eight consecutive candidates
    uint32_t kv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) kv[u] = c0 + u < n ? key(c0 + u) : 0u;
    int nt = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) nt += (c0 + u < n && kv[u] == kth) ? 1 : 0;
    int tie_total;
    int tie_rank = ties_before + block_exclusive_scan<NT>(nt, &tie_total, sm.sbuf);
    ties_before += tie_total;
    uint32_t selm = 0u;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (c0 + u >= n) continue;
      if (kv[u] > kth) {
        selm |= 1u << u;
      } else if (kv[u] == kth) {
        if (tie_rank < need) selm |= 1u << u;
        ++tie_rank;
      }
    }
    int sel_total;
    int pos = written + block_exclusive_scan<NT>(__popc(selm), &sel_total, sm.sbuf);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if ((selm >> u) & 1u) out[pos++] = c0 + u;
    written += sel_total;
  }
}

constexpr int kBlkThreads = 256;

__global__ void __launch_bounds__(kBlkThreads) topk_blocks_kernel(const float* __restrict__ scores,
                                                                  int* __restrict__ idx, int Hkv, int T, int NB, int k,
                                                                  const int* __restrict__ seqlens, int L, int decode) {
  extern __shared__ uint32_t skey[];  // NB keys
  __shared__ RadixSmem<kBlkThreads / 32> sm;
  const int row = blockIdx.x;
  int n;
  if (decode == 2) {   // per-position rows (L = N): row t has blocks 0 .. floor(t/64)
    n = min(NB, (row % L) / 64 + 1);
  } else if (decode) {
    const int b = row / Hkv;
    const int Lb = seqlens ? max(1, min(seqlens[b], L)) : L;
    n = min(NB, (Lb + 63) / 64);
  } else {
    n = min(NB, row % T + 1);
  }
  int* out = idx + (size_t)row * k;
  if (n <= k) {
    for (int c = threadIdx.x; c < k; c += kBlkThreads) out[c] = c < n ? c : -1;
    return;
  }
  const float* srow = scores + (size_t)row * NB;
  for (int c = threadIdx.x; c < n; c += kBlkThreads) skey[c] = order_key(srow[c]);
  __syncthreads();
  radix_topk<kBlkThreads>([&](int c) { return skey[c]; }, n, k, out, sm);
}

constexpr int kTokThreads = 1024;

// Token candidates of tile I are positions [0, e_I - forced], e_I = min(64I+63, N-1).  In decode
// (one row per sequence and KV group, N = L) the new token is e = L_b - 1.
__global__ void __launch_bounds__(kTokThreads) topk_tokens_kernel(const float* __restrict__ scores,
                                                                  int* __restrict__ idx, int T, int N, int k,
                                                                  int forced, const int* __restrict__ seqlens,
                                                                  int Hkv, int decode) {
  __shared__ RadixSmem<kTokThreads / 32> sm;
  const int row = blockIdx.x;
  int e;
  if (decode) {
    const int b = row / Hkv;
    e = (seqlens ? max(1, min(seqlens[b], N)) : N) - 1;
  } else {
    const int I = row % T;
    e = min(N, (I + 1) * 64) - 1;
  }
  const int n = max(0, e - forced + 1);
  const float* srow = scores + (size_t)row * N;
  int* out = idx + (size_t)row * k;
  if (n <= k) {
    for (int c = threadIdx.x; c < k; c += kTokThreads) out[c] = c < n ? c : -1;
    return;
  }
  radix_topk<kTokThreads>([&](int c) { return order_key(srow[c]); }, n, k, out, sm);
}

}  // namespace

cudaError_t launch_topk_blocks(const float* scores, int* idx, int B, int Hkv, int T, int NB, int k,
                               const int* seqlens, int L, bool decode, cudaStream_t s) {
  const int rows = decode ? B * Hkv : B * Hkv * T;
  const size_t smem = (size_t)NB * sizeof(uint32_t);
  const size_t static_smem = sizeof(RadixSmem<kBlkThreads / 32>);
  if (smem + static_smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(topk_blocks_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  topk_blocks_kernel<<<rows, kBlkThreads, smem, s>>>(scores, idx, Hkv, T, NB, k, seqlens, L, decode ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_topk_blocks_rows(const float* scores, int* idx, int B, int Hkv, int N, int NB, int k,
                                    cudaStream_t s) {
  const size_t smem = (size_t)NB * sizeof(uint32_t);
  const size_t static_smem = sizeof(RadixSmem<kBlkThreads / 32>);
  if (smem + static_smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(topk_blocks_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  topk_blocks_kernel<<<(unsigned)((size_t)B * Hkv * N), kBlkThreads, smem, s>>>(scores, idx, Hkv, 1, NB, k, nullptr,
                                                                                N, 2);
  return cudaGetLastError();
}

cudaError_t launch_topk_tokens(const PrefillDims& d, const float* scores, int k_tokens, int forced, int* idx,
                               cudaStream_t s) {
  topk_tokens_kernel<<<d.B * d.Hkv * d.T, kTokThreads, 0, s>>>(scores, idx, d.T, d.N, k_tokens, forced, nullptr,
                                                                d.Hkv, 0);
  return cudaGetLastError();
}

cudaError_t launch_topk_decode_tokens(const float* scores, int* idx, int B, int Hkv, int L, int k_tokens, int forced,
                                      const int* seqlens, cudaStream_t s) {
  topk_tokens_kernel<<<B * Hkv, kTokThreads, 0, s>>>(scores, idx, 1, L, k_tokens, forced, seqlens, Hkv, 1);
  return cudaGetLastError();
}

}  // namespace hys
