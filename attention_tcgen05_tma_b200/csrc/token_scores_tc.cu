// Token-granularity importance scores on the tensor cores (HySparse2 explainer, "Precise
// retrieval without a separate indexer"): the second pass of the token variant.
//
//   score[b,g,I,i] = sum_{h in g} sum_{t in tile I, t >= i} exp(tau q_t.k_i - LSE_t)
//
// LSE_t comes from the first pass (the full-attention kernel), so every probability is
// exact without an online softmax.  Per 128-key tile and 128-row M-tile (two heads x the
// 64 positions of tile I, as in the full layer): S = Q K^T (tcgen05, TMEM); the softmax
// warpgroup writes P * 2^12 as fp16 into shared memory (the scale keeps probabilities down
// to 1.5e-8 in the normal fp16 range; the sum is scaled back at the end); the column sums
// over the 128 rows are one more MMA, D = ONES(128 x 128) * P, accumulated over both
// M-tiles of a round in TMEM.  Warps 2-3 drain D (double-buffered) into the score row;
// later rounds of a unit add to what the first wrote, in a fixed order (deterministic).
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tma_host.h"
#include "tc_ptx.cuh"

namespace hys {

namespace {

constexpr int kThreads = 384;
constexpr int kStages = 2;        // K ring
constexpr int kMaxGrid = 148;
constexpr float kPScaleLog2 = 12.0f;

struct Params {
  int B, N, Hq, Hkv, G, T;
  int num_units;
  const float* lse;   // [B,Hq,N] natural log
  float* scores;      // [B,Hkv,T,N]
  int* counter;
  int* status;
  float scale_log2;
};

struct Bars {
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t q_full[2], q_empty[2], s_full[2], p_full[2], p_empty[2], d_full[2], d_empty[2];
  uint64_t mma_drain, spare;
  tc::UnitQueue queue;
};

template <int D>
struct Cfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kKBytes = 128 * D * 2;
  static constexpr int kPBytes = 128 * 128 * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = 2 * kQBytes;
  static constexpr int kOffP = kOffK + kStages * kKBytes;
  static constexpr int kOffOnes = kOffP + 2 * kPBytes;
  static constexpr int kOffBar = kOffOnes + 16384;
  static constexpr int kOffMisc = kOffBar + (int)((sizeof(Bars) + 15) / 16 * 16);
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;
};

__device__ __forceinline__ void unit_coords(const Params& p, int u, int& b, int& g, int& I) {
  const int bg = u / p.T;
  I = p.T - 1 - u % p.T;
  b = bg / p.Hkv;
  g = bg % p.Hkv;
}

__device__ __forceinline__ void fail(volatile int* abort, int* status) {
  *abort = 1;
  report_status(status, HYS_ERR_TIMEOUT);
}

// instruction descriptor: fp16 A and B (kind::f16 format 0), fp32 accumulate
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, bool b_mn_major) {
  return (1u << 4) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    token_scores_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int MT = p.G / 2;
  const int rounds = (MT + 1) / 2;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(&bars->k_full[i], 1);
      tc::mbar_init(&bars->k_empty[i], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->q_full[s], 1);
      tc::mbar_init(&bars->q_empty[s], 1);
      tc::mbar_init(&bars->s_full[s], 1);
      tc::mbar_init(&bars->p_full[s], 128);
      tc::mbar_init(&bars->p_empty[s], 1);
      tc::mbar_init(&bars->d_full[s], 1);
      tc::mbar_init(&bars->d_empty[s], 64);
    }
    tc::mbar_init(&bars->mma_drain, 1);
    tc::queue_init(&bars->queue, 1 + 256 + 64);  // MMA thread, softmax warpgroups, drain warps
    *abort = 0;
    tc::fence_barrier_init();
  }
  // the all-ones A operand: 128 rows x 64 fp16 (one 128-byte swizzled chunk, reused for both k halves)
  {
    uint4* ones = reinterpret_cast<uint4*>(smem + C::kOffOnes);
    const uint32_t one2 = 0x3C003C00u;
    for (int i = threadIdx.x; i < 16384 / 16; i += kThreads) ones[i] = make_uint4(one2, one2, one2, one2);
    tc::fence_proxy_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tensormap(&tmQ);
    tc::prefetch_tensormap(&tmK);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ============================================================== TMA producer
    if (lane == 0) {
      uint32_t k_it = 0, q_cnt[2] = {0, 0};
      bool ok = true;
      for (uint32_t n = 0; ok; ++n) {
        const int c = atomicAdd(p.counter, 1);
        const int u = c < p.num_units ? c : -1;
        if (!(ok = tc::queue_push(&bars->queue, n, u, abort))) break;
        if (u < 0) break;
        int b, g, I;
        unit_coords(p, u, b, g, I);
        const int nkt = I / 2 + 1;
        for (int r = 0; r < rounds && ok; ++r) {
          for (int s = 0; s < 2 && ok; ++s) {
            const int mt = 2 * r + s;
            if (mt >= MT) continue;
            if (!(ok = tc::mbar_wait(&bars->q_empty[s], (q_cnt[s] & 1u) ^ 1u, abort))) break;
            ++q_cnt[s];
            tc::mbar_arrive_expect_tx(&bars->q_full[s], C::kQBytes);
            uint8_t* qdst = smem + C::kOffQ + s * C::kQBytes;
            const int h0 = g * p.G + 2 * mt;
            for (int hh = 0; hh < 2; ++hh)
              for (int ch = 0; ch < C::kChunks; ++ch)
                tc::tma_load_3d(&tmQ, &bars->q_full[s], qdst + ch * 16384 + hh * 8192, ch * 64, 64 * I,
                                b * p.Hq + h0 + hh);
          }
          for (int tau = 0; tau < nkt && ok; ++tau) {
            const uint32_t st = k_it % kStages;
            if (!(ok = tc::mbar_wait(&bars->k_empty[st], ((k_it / kStages) & 1u) ^ 1u, abort))) break;
            tc::mbar_arrive_expect_tx(&bars->k_full[st], C::kKBytes);
            uint8_t* dst = smem + C::kOffK + st * C::kKBytes;
            for (int ch = 0; ch < C::kChunks; ++ch)
              tc::tma_load_3d(&tmK, &bars->k_full[st], dst + ch * 16384, ch * 64, 128 * tau, b * p.Hkv + g);
            ++k_it;
          }
        }
      }
      if (!ok) fail(abort, p.status);
      for (uint32_t i = (k_it > kStages ? k_it - kStages : 0); i < k_it; ++i)
        tc::mbar_wait(&bars->k_full[i % kStages], (i / kStages) & 1u, abort, 100000000ull);
      for (int s = 0; s < 2; ++s)
        if (q_cnt[s] > 0) tc::mbar_wait(&bars->q_full[s], (q_cnt[s] - 1) & 1u, abort, 100000000ull);
    }
  } else if (warp == 1) {
    // ============================================================== MMA issuer
    if (lane == 0) {
      const uint32_t idS = tc::idesc_bf16_f32(128, 128, false);
      const uint32_t idC = idesc_f16_f32(128, 128, true);
      const uint32_t tS[2] = {tmem_base, tmem_base + 128};
      const uint32_t tD[2] = {tmem_base + 256, tmem_base + 384};
      const uint32_t qaddr = tc::smem_u32(smem + C::kOffQ);
      const uint32_t kaddr = tc::smem_u32(smem + C::kOffK);
      const uint32_t paddr = tc::smem_u32(smem + C::kOffP);
      const uint32_t oaddr = tc::smem_u32(smem + C::kOffOnes);
      uint32_t k_it = 0, q_cnt[2] = {0, 0}, p_cnt[2] = {0, 0}, d_cnt = 0;
      bool ok = true;
      auto issue_S = [&](int s, uint32_t st) {
        const uint32_t qb = qaddr + s * C::kQBytes, kb = kaddr + st * C::kKBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc::mma_ss(tS[s], tc::sdesc_sw128(qb + off, 16, 1024), tc::sdesc_sw128(kb + off, 16, 1024), idS,
                     kk > 0 ? 1u : 0u);
        }
      };
      // D[buf] (+)= ONES * P_s : K = the 128 query rows of the M-tile, N = the 128 keys
      auto issue_C = [&](int s, uint32_t buf, bool acc) {
        const uint32_t pb = paddr + s * C::kPBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_ss(tD[buf], tc::sdesc_sw128(oaddr + (kk & 3) * 32, 16, 1024),
                     tc::sdesc_sw128(pb + kk * 2048, 16384, 1024), idC, (acc || kk > 0) ? 1u : 0u);
      };
      for (uint32_t n = 0; ok; ++n) {
        const int u = tc::queue_pop(&bars->queue, n, abort, ok);
        if (u < 0) break;
        int b, g, I;
        unit_coords(p, u, b, g, I);
        const int nkt = I / 2 + 1;
        for (int r = 0; r < rounds && ok; ++r) {
          bool act[2];
          for (int s = 0; s < 2; ++s) {
            act[s] = (2 * r + s) < MT;
            if (act[s] && ok) {
              ok = tc::mbar_wait(&bars->q_full[s], q_cnt[s] & 1u, abort);
              ++q_cnt[s];
            }
          }
          if (!ok) break;
          uint32_t kst = k_it % kStages;
          if (!(ok = tc::mbar_wait(&bars->k_full[kst], (k_it / kStages) & 1u, abort))) break;
          ++k_it;
          tc::fence_after_sync();
          for (int s = 0; s < 2; ++s)
            if (act[s]) {
              issue_S(s, kst);
              tc::mma_commit(&bars->s_full[s]);
            }
          tc::mma_commit(&bars->k_empty[kst]);
          for (int tau = 1; tau <= nkt && ok; ++tau) {
            // column sums of tile tau-1 into D[d_cnt & 1], then S of tile tau
            const uint32_t buf = d_cnt & 1u;
            if (!(ok = tc::mbar_wait(&bars->d_empty[buf], ((d_cnt >> 1) & 1u) ^ 1u, abort))) break;
            bool have_k = false, first = true;
            for (int s = 0; s < 2 && ok; ++s) {
              if (!act[s]) continue;
              if (!(ok = tc::mbar_wait(&bars->p_full[s], p_cnt[s] & 1u, abort))) break;
              ++p_cnt[s];
              tc::fence_after_sync();
              issue_C(s, buf, !first);
              first = false;
              tc::mma_commit(&bars->p_empty[s]);
              if (tau < nkt) {
                if (!have_k) {
                  kst = k_it % kStages;
                  if (!(ok = tc::mbar_wait(&bars->k_full[kst], (k_it / kStages) & 1u, abort))) break;
                  ++k_it;
                  have_k = true;
                  tc::fence_after_sync();
                }
                issue_S(s, kst);
                tc::mma_commit(&bars->s_full[s]);
              }
            }
            tc::mma_commit(&bars->d_full[buf]);
            ++d_cnt;
            if (have_k) tc::mma_commit(&bars->k_empty[kst]);
          }
          for (int s = 0; s < 2; ++s)
            if (act[s]) tc::mma_commit(&bars->q_empty[s]);
        }
      }
      if (!ok) fail(abort, p.status);
      tc::mma_commit(&bars->mma_drain);
      tc::mbar_wait(&bars->mma_drain, 0, abort, 100000000ull);
    }
  } else if (warp == 2 || warp == 3) {
    // ============================================================== column-sum drain
    // All rows of D are equal; warp w reads its own TMEM lane quarter and lane l keeps column l.
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const int half = warp - 2;  // columns [64*half, 64*half + 64)
    const float inv = exp2f(-kPScaleLog2);
    uint32_t d_cnt = 0;
    bool ok = true;
    for (uint32_t n = 0; ok; ++n) {
      const int u = tc::queue_pop(&bars->queue, n, abort, ok);
      ok = __all_sync(0xffffffffu, ok);   // warp-uniform: TMEM accesses are warp-collective
      if (__any_sync(0xffffffffu, u < 0)) break;
      int b, g, I;
      unit_coords(p, u, b, g, I);
      const int nkt = I / 2 + 1;
      float* srow = p.scores + (((size_t)b * p.Hkv + g) * p.T + I) * (size_t)p.N;
      // keys past the last key tile receive no probability
      for (int i = 128 * nkt + 64 * half + lane; i < p.N; i += 64) srow[i] = 0.0f;
      for (int r = 0; r < rounds && ok; ++r) {
        for (int tau = 0; tau < nkt; ++tau) {
          const uint32_t buf = d_cnt & 1u;
          if (!(ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->d_full[buf], (d_cnt >> 1) & 1u, abort)))) break;
          ++d_cnt;
          tc::fence_after_sync();
          uint32_t v0[32], v1[32];
          tc::tmem_ld32(tmem_base + 256 + 128 * buf + 64 * half + lane_off, v0);
          tc::tmem_ld32(tmem_base + 256 + 128 * buf + 64 * half + 32 + lane_off, v1);
          tc::tmem_wait_ld();
          float a = 0.0f, c = 0.0f;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            a = (i == lane) ? __uint_as_float(v0[i]) : a;
            c = (i == lane) ? __uint_as_float(v1[i]) : c;
          }
          tc::fence_before_sync();
          tc::mbar_arrive(&bars->d_empty[buf]);
          const int i0 = 128 * tau + 64 * half + lane, i1 = i0 + 32;
          if (i0 < p.N) srow[i0] = (r == 0 ? 0.0f : srow[i0]) + a * inv;
          if (i1 < p.N) srow[i1] = (r == 0 ? 0.0f : srow[i1]) + c * inv;
        }
      }
    }
    if (!ok) fail(abort, p.status);
  } else if (warp >= 4) {
    // ============================================================== probabilities -> fp16 P in smem
    const int s = (warp - 4) >> 2;
    const int row = 32 * (warp & 3) + lane;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tSrow = tmem_base + 128 * s + lane_off;
    uint8_t* pbuf = smem + C::kOffP + s * C::kPBytes;
    const float sc = p.scale_log2;
    uint32_t s_cnt = 0, pe_cnt = 0;
    bool ok = true;
    for (uint32_t n = 0; ok; ++n) {
      const int u = tc::queue_pop(&bars->queue, n, abort, ok);
      ok = __all_sync(0xffffffffu, ok);   // warp-uniform: TMEM accesses are warp-collective
      if (__any_sync(0xffffffffu, u < 0)) break;
      int b, g, I;
      unit_coords(p, u, b, g, I);
      const int nkt = I / 2 + 1;
      for (int r = 0; r < rounds && ok; ++r) {
        const int mt = 2 * r + s;
        if (mt >= MT) continue;
        const int h = g * p.G + 2 * mt + (row >> 6);
        const int t = 64 * I + (row & 63);
        const bool valid = t < p.N;
        // p * 2^12 = exp2(s * sc - LSE_t * log2(e) + 12); invalid rows contribute nothing
        const float bias = valid ? kPScaleLog2 - p.lse[((size_t)b * p.Hq + h) * p.N + t] * kLog2e : -INFINITY;
        for (int tau = 0; tau < nkt; ++tau) {
          if (!(ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->s_full[s], s_cnt & 1u, abort)))) break;
          ++s_cnt;
          tc::fence_after_sync();
          uint32_t r0[32], r1[32], r2[32], r3[32];
          tc::tmem_ld32(tSrow + 0, r0);
          tc::tmem_ld32(tSrow + 32, r1);
          tc::tmem_ld32(tSrow + 64, r2);
          tc::tmem_ld32(tSrow + 96, r3);
          tc::tmem_wait_ld();
          // P buffer of this slot is free once the previous column-sum MMA has read it
          if (!(ok = tc::mbar_wait(&bars->p_empty[s], (pe_cnt & 1u) ^ 1u, abort))) break;
          ++pe_cnt;
          const int cmax = (tau == nkt - 1) ? t - 128 * tau : 127;  // causal: keys <= t
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {        // 64-key chunk
#pragma unroll
            for (int un = 0; un < 8; ++un) {      // 16-byte unit = 8 keys
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int col = 64 * ch + 8 * un + 2 * e;
                const uint32_t* src = ch == 0 ? (col < 32 ? r0 : r1) : (col < 96 ? r2 : r3);
                const int ci = col & 31;
                const float x0 = col <= cmax ? exp2f(fmaf(__uint_as_float(src[ci]), sc, bias)) : 0.0f;
                const float x1 = col + 1 <= cmax ? exp2f(fmaf(__uint_as_float(src[ci + 1]), sc, bias)) : 0.0f;
                w[e] = pack_f16x2(x0, x1);
              }
              // MN-major 128-byte swizzle: row `row`, 16-byte unit `un` of chunk `ch`
              *reinterpret_cast<uint4*>(pbuf + ch * 16384 + row * 128 + ((un ^ (row & 7)) << 4)) =
                  make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
          tc::fence_proxy_async_shared();  // generic-proxy writes -> visible to the tensor core
          tc::fence_before_sync();
          tc::mbar_arrive(&bars->p_full[s]);
        }
      }
    }
    if (!ok) fail(abort, p.status);
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem_base, 512);
  }
}

bool make_map(CUtensorMap* m, const void* base, int D, int rows, int heads, int box_rows) {
  EncodeTiledFn fn = tma_encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_units(const PrefillDims& d) { return d.B * d.Hkv * d.T; }
int grid_size(const PrefillDims& d) { return num_units(d) < kMaxGrid ? num_units(d) : kMaxGrid; }

template <int D>
cudaError_t launch_typed(const PrefillDims& d, const void* q, const void* k, const float* lse, float* scores,
                         void* ws, cudaStream_t s) {
  CUtensorMap mq, mk;
  if (!make_map(&mq, q, D, d.N, d.B * d.Hq, 64) || !make_map(&mk, k, D, d.N, d.B * d.Hkv, 128))
    return cudaErrorInvalidValue;
  Params p;
  p.B = d.B;
  p.N = d.N;
  p.Hq = d.Hq;
  p.Hkv = d.Hkv;
  p.G = d.G();
  p.T = d.T;
  p.num_units = num_units(d);
  p.lse = lse;
  p.scores = scores;
  p.counter = reinterpret_cast<int*>(ws);
  p.status = device_status_ptr();
  p.scale_log2 = kLog2e / sqrtf((float)D);
  const int smem = Cfg<D>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(token_scores_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(p.counter, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  token_scores_tc_kernel<D><<<grid_size(d), kThreads, smem, s>>>(mq, mk, p);
  return cudaGetLastError();
}

}  // namespace

bool token_scores_tc_supported(const PrefillDims& d, hys_dtype dt) {
  return dt == HYS_BF16 && (d.D == 64 || d.D == 128) && d.G() % 2 == 0;
}

cudaError_t launch_token_scores_tc(const PrefillDims& d, const void* q, const void* k, const float* lse,
                                   float* scores, void* ws, cudaStream_t s) {
  if (ws == nullptr) return cudaErrorInvalidValue;
  return d.D == 64 ? launch_typed<64>(d, q, k, lse, scores, ws, s) : launch_typed<128>(d, q, k, lse, scores, ws, s);
}

}  // namespace hys
