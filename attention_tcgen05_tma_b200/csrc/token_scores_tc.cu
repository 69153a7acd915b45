// Token-granularity importance scores on the tensor cores (HySparse2 explainer, "Precise
// retrieval without a separate indexer"): the second pass of the token variant.
//
//   score[b,g,I,i] = sum_{h in g} sum_{t in tile I, t >= i} exp(tau q_t.k_i - LSE_t)
//
// LSE_t comes from the first pass (the full-attention kernel), so every probability is exact
// without an online softmax.  The scores are column sums of P, so the kernel computes the
// transposed logits S^T = K Q^T (tcgen05, TMEM): a TMEM lane is then a key and its 128 columns
// are the query rows of an M-tile (two heads x the 64 positions of tile I), and each key's sum
// over the rows is a sum inside one thread -- no cross-thread reduction, no P in shared memory.
//
// A work unit is (b, g, I); up to four M-tiles (head pairs) stay in shared memory while the
// key tiles 0..I/2 stream through a two-stage ring.  Every (key tile, M-tile) item is one MMA
// into one of four 128-column TMEM buffers (a ring over the items).  Two softmax warpgroups
// take the items of even and odd M-tiles; per key tile the odd group's per-key partial goes to
// the even group through shared memory, which adds its own and writes score[b,g,I,key] once
// (fixed order: deterministic).  Part of the exponentials run as a polynomial on the FMA pipe.
#include <cuda.h>
#include <stdlib.h>

#include "common.cuh"
#include "kernels.h"
#include "tma_host.h"
#include "tc_ptx.cuh"

namespace hys {

namespace {

constexpr int kThreads = 384;     // warp 0 TMA, warp 1 MMA, warps 4-7 / 8-11 softmax groups 0 / 1
constexpr int kStages = 2;        // K ring
constexpr int kMaxMT = 4;         // M-tiles resident per round
constexpr int kBufs = 4;          // TMEM buffers of 128 columns
constexpr int kMaxGrid = 148;
#ifndef HYS_TSCORE_POLY_PAIRS
#define HYS_TSCORE_POLY_PAIRS 24
#endif
// column pairs (of the 64 in a 128-row item) whose exp2 runs on the FMA pipe instead of MUFU
constexpr int kPolyPairs = HYS_TSCORE_POLY_PAIRS;

struct Params {
  int B, N, Hq, Hkv, G, T;
  int num_units;
  const float* lse;   // [B,Hq,N] natural log
  float* scores;      // [B,Hkv,T,N]
  int* counter;
  int* status;
  float scale_log2;
  uint64_t wait_ns;   // limit of every bounded wait
  int probe;          // watchdog probe: the producer never issues the first unit's Q copies
};

struct Bars {
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t q_full, q_empty, s_full[kBufs], s_free[kBufs];
  uint64_t rows_ready[2], comb_full[2], comb_empty[2];
  uint64_t mma_drain, spare;
};

template <int D>
struct Cfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kQBytes = 128 * D * 2;   // one M-tile
  static constexpr int kKBytes = 128 * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kMaxMT * kQBytes;
  static constexpr int kOffLse = kOffK + kStages * kKBytes;      // [2 rounds][kMaxMT][128] lse2
  static constexpr int kOffRed = kOffLse + 2 * kMaxMT * 128 * 4; // [2][128] odd-group partials
  static constexpr int kOffBar = kOffRed + 2 * 128 * 4;
  static constexpr int kOffMisc = kOffBar + (int)((sizeof(Bars) + 15) / 16 * 16);
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;
};
static_assert(Cfg<128>::kSmemBytes <= 232448, "shared memory of one CTA");

// unit u -> (b, g, I), the longest (largest I) first over all (b, g)
__device__ __forceinline__ void unit_coords(const Params& p, int u, int& b, int& g, int& I) {
  const int bg = u % (p.B * p.Hkv);
  I = p.T - 1 - u / (p.B * p.Hkv);
  b = bg / p.Hkv;
  g = bg % p.Hkv;
}

__device__ __forceinline__ void fail(volatile int* abort, int* status) {
  *abort = 1;
  report_status(status, HYS_ERR_TIMEOUT);
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
  int* s_unit = reinterpret_cast<int*>(smem + C::kOffMisc + 32);
  float* s_lse = reinterpret_cast<float*>(smem + C::kOffLse);
  float* s_red = reinterpret_cast<float*>(smem + C::kOffRed);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int MT = p.G / 2;
  const int rounds = (MT + kMaxMT - 1) / kMaxMT;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(&bars->k_full[i], 1);
      tc::mbar_init(&bars->k_empty[i], 1);
    }
    tc::mbar_init(&bars->q_full, 1);
    tc::mbar_init(&bars->q_empty, 1);
    for (int i = 0; i < kBufs; ++i) {
      tc::mbar_init(&bars->s_full[i], 1);
      tc::mbar_init(&bars->s_free[i], 128);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&bars->rows_ready[i], 128);
      tc::mbar_init(&bars->comb_full[i], 128);
      tc::mbar_init(&bars->comb_empty[i], 128);
    }
    tc::mbar_init(&bars->mma_drain, 1);
    *abort = 0;
    tc::fence_barrier_init();
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

  // every role walks the same unit sequence (one thread claims, all read it back); counters of
  // rounds (rc), key-tile items (ni), K tiles (kc) and combines (cc) advance identically in all roles
  uint32_t rc = 0, ni = 0, kc = 0, cc = 0;
  for (;;) {
    if (threadIdx.x == 0) *s_unit = atomicAdd(p.counter, 1);
    __syncthreads();
    const int u = *s_unit;
    const bool stop = u >= p.num_units || *abort;
    __syncthreads();
    if (stop) break;
    int b, g, I;
    unit_coords(p, u, b, g, I);
    const int nkt = I / 2 + 1;
    float* srow = p.scores + (((size_t)b * p.Hkv + g) * p.T + I) * (size_t)p.N;

    for (int r = 0; r < rounds; ++r) {
      const int mt0 = kMaxMT * r;
      const int nm = min(kMaxMT, MT - mt0);
      if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
          bool ok = tc::mbar_wait(&bars->q_empty, (rc & 1u) ^ 1u, abort, p.wait_ns);
          // watchdog probe (tests only): the first unit's Q copies are never issued, so the MMA
          // warp's wait on them runs out and the kernel must end with HYS_ERR_TIMEOUT
          if (ok && !(p.probe && rc == 0)) {
            tc::mbar_arrive_expect_tx(&bars->q_full, nm * C::kQBytes);
            for (int m = 0; m < nm; ++m)
              for (int hh = 0; hh < 2; ++hh)
                for (int ch = 0; ch < C::kChunks; ++ch)
                  tc::tma_load_3d(&tmQ, &bars->q_full, smem + C::kOffQ + m * C::kQBytes + ch * 16384 + hh * 8192,
                                  ch * 64, 64 * I, b * p.Hq + g * p.G + 2 * (mt0 + m) + hh);
          }
          for (int j = 0; j < nkt && ok; ++j) {
            const uint32_t k = kc + j, st = k % kStages;
            if (!(ok = tc::mbar_wait(&bars->k_empty[st], ((k / kStages) & 1u) ^ 1u, abort, p.wait_ns))) break;
            tc::mbar_arrive_expect_tx(&bars->k_full[st], C::kKBytes);
            for (int ch = 0; ch < C::kChunks; ++ch)
              tc::tma_load_3d(&tmK, &bars->k_full[st], smem + C::kOffK + st * C::kKBytes + ch * 16384, ch * 64,
                              128 * j, b * p.Hkv + g);
          }
          if (!ok) fail(abort, p.status);
        }
      } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer: S^T = K Q^T
        if (lane == 0) {
          const uint32_t idS = tc::idesc_bf16_f32(128, 128, false);
          bool ok = tc::mbar_wait(&bars->q_full, rc & 1u, abort, p.wait_ns);
          for (int j = 0; j < nkt && ok; ++j) {
            const uint32_t k = kc + j, st = k % kStages;
            if (!(ok = tc::mbar_wait(&bars->k_full[st], (k / kStages) & 1u, abort, p.wait_ns))) break;
            const uint32_t kb = tc::smem_u32(smem + C::kOffK + st * C::kKBytes);
            for (int m = 0; m < nm && ok; ++m) {
              const uint32_t n = ni + j * nm + m, bf = n % kBufs, use = n / kBufs;
              if (use > 0 && !(ok = tc::mbar_wait(&bars->s_free[bf], (use - 1) & 1u, abort, p.wait_ns))) break;
              tc::fence_after_sync();
              const uint32_t qb = tc::smem_u32(smem + C::kOffQ + m * C::kQBytes);
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                tc::mma_ss(tmem_base + 128 * bf, tc::sdesc_sw128(kb + off, 16, 1024),
                           tc::sdesc_sw128(qb + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
              }
              tc::mma_commit(&bars->s_full[bf]);
            }
            tc::mma_commit(&bars->k_empty[st]);
          }
          if (ok) tc::mma_commit(&bars->q_empty);
          else fail(abort, p.status);
        }
      } else if (warp >= 4) {
        // ---------------------------------------------------------- softmax groups
        const int grp = (warp - 4) >> 2;                 // 0: even M-tiles, 1: odd M-tiles
        const int key = 32 * (warp & 3) + lane;          // TMEM lane = key of the tile
        const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
        const float sc = p.scale_log2;
        float* lse_r = s_lse + (rc & 1u) * kMaxMT * 128;
        bool ok = true;
        // this group's M-tiles' row LSEs (log2 units; rows past N never count)
        for (int m = grp; m < nm; m += 2) {
          const int h = g * p.G + 2 * (mt0 + m) + (key >> 6);
          const int t = 64 * I + (key & 63);
          lse_r[m * 128 + key] = t < p.N ? p.lse[((size_t)b * p.Hq + h) * p.N + t] * kLog2e : INFINITY;
        }
        if (grp == 0 && r == 0)
          for (int i = 128 * nkt + key; i < p.N; i += 128) srow[i] = 0.0f;   // keys past the last tile
        tc::mbar_arrive(&bars->rows_ready[grp]);
        ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->rows_ready[grp], rc & 1u, abort, p.wait_ns));
        const bool two = nm >= 2;
        for (int j = 0; j < nkt && ok; ++j) {
          float acc = 0.0f;
          const int kp = 128 * j + key;
          for (int m = grp; m < nm; m += 2) {
            const uint32_t n = ni + j * nm + m, bf = n % kBufs, use = n / kBufs;
            if (!(ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->s_full[bf], use & 1u, abort, p.wait_ns)))) break;
            tc::fence_after_sync();
            const float* lr = lse_r + m * 128;
            // causal: key kp counts for query column q when kp <= 64 I + (q & 63)
            const int lim = kp - 64 * I;   // columns with (q & 63) >= lim are visible
            float2 a2[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll 2
            for (int c = 0; c < 4; ++c) {
              uint32_t v[32];
              tc::tmem_ld32(tmem_base + 128 * bf + 32 * c + lane_off, v);
              tc::tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const int q = 32 * c + 2 * e;
                const float2 x = tc::ffma2(make_float2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1])),
                                           make_float2(sc, sc), make_float2(-lr[q], -lr[q + 1]));
                float2 pv = (16 * c + e) % 4 < kPolyPairs / 16 ? tc::exp2_poly3_x2(x)
                                                                : make_float2(exp2f(x.x), exp2f(x.y));
                if (lim > 0) {
                  pv.x = (q & 63) >= lim ? pv.x : 0.0f;
                  pv.y = ((q + 1) & 63) >= lim ? pv.y : 0.0f;
                }
                a2[e & 1] = tc::fadd2(a2[e & 1], pv);
              }
            }
            tc::fence_before_sync();
            tc::mbar_arrive(&bars->s_free[bf]);
            const float2 a = tc::fadd2(a2[0], a2[1]);
            acc += a.x + a.y;
          }
          if (!ok) break;
          // combine the two groups' partials of key kp and write the score once
          if (two) {
            const uint32_t slot = (cc + j) & 1u, use = (cc + j) >> 1;
            if (grp == 1) {
              if (use > 0 && !(ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->comb_empty[slot], (use - 1) & 1u, abort, p.wait_ns))))
                break;
              s_red[slot * 128 + key] = acc;
              tc::mbar_arrive(&bars->comb_full[slot]);
            } else {
              if (!(ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->comb_full[slot], use & 1u, abort, p.wait_ns)))) break;
              acc += s_red[slot * 128 + key];
              tc::mbar_arrive(&bars->comb_empty[slot]);
            }
          }
          if (grp == 0 && kp < p.N) srow[kp] = (r == 0 ? 0.0f : srow[kp]) + acc;
        }
        if (!ok) fail(abort, p.status);
      }
      ni += (uint32_t)(nkt * nm);
      kc += (uint32_t)nkt;
      cc += nm >= 2 ? (uint32_t)nkt : 0u;
      ++rc;
    }
    __syncthreads();   // every role finished the unit (a failed wait set abort)
  }

  // the MMAs and copies issued have completed before TMEM is released
  if (warp == 1 && lane == 0) {
    tc::mma_commit(&bars->mma_drain);
    tc::mbar_wait_drain(&bars->mma_drain, 0);
  }
  if (warp == 0 && lane == 0 && rc > 0) {
    tc::mbar_wait_drain(&bars->q_full, (rc - 1) & 1u);
    if (kc > 0) tc::mbar_wait_drain(&bars->k_full[(kc - 1) % kStages], ((kc - 1) / kStages) & 1u);
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
  // HYS_WATCHDOG_PROBE=1 (tests only) arms the probe above with a 0.2 s wait limit
  static const bool probe = [] {
    const char* e = getenv("HYS_WATCHDOG_PROBE");
    return e != nullptr && e[0] == '1';
  }();
  p.probe = probe ? 1 : 0;
  p.wait_ns = probe ? 200000000ull : 4000000000ull;
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
