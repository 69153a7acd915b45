// Token-sparse layer on the tensor cores (HySparse2 explainer, "Precise retrieval without a
// separate indexer"): row t of query tile I attends the tile's selected tokens united with its
// newest W tokens [t-W+1, t], each token once, over the shared K, V; no gate.
//
// The attended keys of a unit (b, g, I) split into two parts:
//   * part A: the selected tokens <= 64I - W.  They lie before every row's window and are
//     causal for every row, so no mask is needed.  They are gathered row by row with TMA
//     tile::gather4 (four 128-byte rows per instruction; the producer warp's 32 lanes each
//     issue one quad per chunk, 64 instructions per 128-key tile).
//   * part B: the contiguous extended window [w0, e_I], w0 = max(0, 64I-W+1), e_I the tile's
//     last row.  Row t sees key i there if i is in its own window, or if i was selected and
//     lies at or before t-W (selected, outside the window, causal).  The selected tokens in
//     part B travel as a bitmask published with the unit.
// The rest follows the full-layer kernel: 128-row M-tiles of two heads x 64 positions, two
// in flight, S and O in TMEM, P written back over S, one online softmax, O / l at the end.
//
// Gathers bound the layer (one TMA instruction per four 128-byte rows).  With four or more
// M-tiles per unit a single CTA needs two rounds over the unit's keys and gathers every tile
// twice, so such units run on a CTA pair (a cluster of two): both CTAs walk the same key
// tiles, each gathers half of every tile's rows (part B: half-tile boxes) and sends that half
// into the partner's stage with a shared-to-shared bulk copy, and each CTA computes two of the
// unit's M-tiles.  A stage is free again once both CTAs' MMAs have read it (the MMA warp's
// commit arrives on the stage barrier of both CTAs).  Every key row then crosses the TMA unit
// once per unit instead of once per round.
#include <cuda.h>

#include <algorithm>
#include <atomic>
#include <cstdlib>

#include "cluster_ptx.cuh"
#include "common.cuh"
#include "kernels.h"
#include "tma_host.h"
#include "tc_ptx.cuh"

namespace hys {

namespace {

constexpr int kThreads = 384;
#ifndef HYS_TOKEN_STAGES
#define HYS_TOKEN_STAGES 5
#endif
constexpr int kStages = HYS_TOKEN_STAGES;   // K / V stages of 128 keys (shared memory holds five)
constexpr int kMaxGrid = 148;
constexpr int kMaskWords = 16;     // extended window <= 512 keys  ->  W <= 449
constexpr float kRescaleLog2 = 8.0f;
#ifndef HYS_TOKEN_PAIR
#define HYS_TOKEN_PAIR 1
#endif
#ifndef HYS_TOKEN_POLY_PAIRS
#define HYS_TOKEN_POLY_PAIRS 0
#endif
// column pairs (of the 64 in a 128-key row) whose exp2 runs on the FMA pipe instead of MUFU
constexpr int kPolyPairs = HYS_TOKEN_POLY_PAIRS;
// Register split between the warpgroups (setmaxnreg): the launch gives every thread
// kLaunchRegs; the producer/MMA warpgroup drops to kLowRegs and each softmax warpgroup rises to
// kHighRegs.  The sum must equal three launch shares, or setmaxnreg.inc would wait forever;
// the host checks the compiled register count before every launch.
#ifndef HYS_TOKEN_LOW_REGS
#define HYS_TOKEN_LOW_REGS 88
#endif
constexpr int kLaunchRegs = 168, kLowRegs = HYS_TOKEN_LOW_REGS, kHighRegs = (3 * kLaunchRegs - kLowRegs) / 2;
static_assert(kLowRegs % 8 == 0 && kHighRegs % 8 == 0, "setmaxnreg takes multiples of 8");
static_assert(kLowRegs + 2 * kHighRegs == 3 * kLaunchRegs, "register split must match the launch allocation");

__device__ __forceinline__ float2 exp2_pair(float2 x, int i) {
  if ((i * kPolyPairs) % 64 < kPolyPairs) return tc::exp2_poly3_x2(x);
  return make_float2(exp2f(x.x), exp2f(x.y));
}

struct Params {
  int B, N, Hq, Hkv, G, T, kt, W;
  int num_units;
  const int* idx;     // [B,Hkv,T,kt]
  __nv_bfloat16* o;
  int o_v8;           // o is 32-byte aligned (256-bit stores)
  int* counter;
  int* status;
  float scale_log2;
};

struct Bars {
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t kv_half[kStages];   // CTA pair: this CTA's half of the stage has landed
  uint64_t q_full[2], q_empty[2], s_full[2], p_full[2], o_full[2], o_empty[2];
  uint64_t mma_drain, spare;
  tc::UnitQueue queue;
  uint32_t selmask[tc::kQueueSlots][kMaskWords];
};

template <int D>
struct Cfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kKVBytes = 128 * D * 2;
  static constexpr int kHalfBytes = kKVBytes / 2;   // 64 key rows
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kQBytes;
  static constexpr int kOffBar = kOffKV + kStages * kKVBytes;
  static constexpr int kOffMisc = kOffBar + (int)((sizeof(Bars) + 15) / 16 * 16);
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

struct Unit {
  int b, g, I, eI, w0;
  int nA;    // selected tokens in part A
  int n_sp;  // part-A tiles
  int n_w;   // part-B tiles
};

__device__ __forceinline__ Unit make_unit(const Params& p, int u, int nA) {
  Unit x;
  const int bg = u / p.T;
  x.I = p.T - 1 - u % p.T;
  x.b = bg / p.Hkv;
  x.g = bg % p.Hkv;
  x.eI = min(p.N, 64 * x.I + 64) - 1;
  x.w0 = max(0, 64 * x.I - p.W + 1);
  x.nA = nA;
  x.n_sp = (nA + 127) / 128;
  x.n_w = (x.eI - x.w0 + 128) / 128;
  return x;
}

__device__ __forceinline__ void fail(volatile int* abort, int* status) {
  *abort = 1;
  report_status(status, HYS_ERR_TIMEOUT);
}

// PAIR: the kernel runs as clusters of two CTAs, one unit per cluster at a time (see the top of
// the file); tmKb / tmVb are K and V with 64-row boxes (part B's half tiles).
template <int D, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    token_sparse_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
                           const __grid_constant__ CUtensorMap tmVb, const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int MT = p.G / 2;
  // M-tile mt = kRoundStride * r + mt0 + s (s = TMEM slot): two per CTA and round, four per pair
  constexpr int kRoundStride = PAIR ? 4 : 2;
  const int rounds = (MT + kRoundStride - 1) / kRoundStride;
  const uint32_t rank = PAIR ? tc::cluster_ctarank() : 0u;
  const int mt0 = 2 * (int)rank;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(&bars->kv_full[i], 1);
      tc::mbar_init(&bars->kv_empty[i], PAIR ? 2 : 1);   // pair: both CTAs' MMAs release a stage
      tc::mbar_init(&bars->kv_half[i], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->q_full[s], 1);
      tc::mbar_init(&bars->q_empty[s], 1);
      tc::mbar_init(&bars->s_full[s], 1);
      tc::mbar_init(&bars->p_full[s], 128);
      tc::mbar_init(&bars->o_full[s], 1);
      tc::mbar_init(&bars->o_empty[s], 128);
    }
    tc::mbar_init(&bars->mma_drain, 1);
    tc::queue_init(&bars->queue, 1 + 256 + (PAIR ? 1 : 0));   // MMA, softmax, pair: copier
    *abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tensormap(&tmQ);
    tc::prefetch_tensormap(&tmK);
    tc::prefetch_tensormap(&tmV);
    if (PAIR) {
      tc::prefetch_tensormap(&tmKb);
      tc::prefetch_tensormap(&tmVb);
    }
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (PAIR) tc::cluster_sync();   // the partner's barriers are initialised before any copy or commit reaches them
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ============================================================== producer warp (gathers)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kLowRegs));
    uint32_t kv_it = 0, q_cnt[2] = {0, 0};
    bool ok = true;
    // the next unit is claimed one unit ahead, so the counter's round trip overlaps a unit's work
    // (a CTA pair takes units in a fixed order instead: both CTAs must see the same sequence)
    int claim = 0;
    if (!PAIR && lane == 0) claim = atomicAdd(p.counter, 1);
    for (uint32_t n = 0; ok; ++n) {
      int u = 0;
      if (PAIR) {
        const int c = (int)(blockIdx.x >> 1) + (int)n * (int)(gridDim.x >> 1);
        u = c < p.num_units ? c : -1;
      } else if (lane == 0) {
        u = claim < p.num_units ? claim : -1;
        if (u >= 0) claim = atomicAdd(p.counter, 1);
      }
      u = __shfl_sync(0xffffffffu, u, 0);
      // wait for the queue slot before filling its mask
      if (lane == 0) ok = tc::mbar_wait(&bars->queue.empty[n % tc::kQueueSlots], ((n / tc::kQueueSlots) & 1u) ^ 1u, abort);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      int nA = 0;
      uint32_t* mask = bars->selmask[n % tc::kQueueSlots];
      const int* sel = nullptr;
      Unit x0;
      if (u >= 0) {
        x0 = make_unit(p, u, 0);
        sel = p.idx + (((size_t)x0.b * p.Hkv + x0.g) * p.T + x0.I) * p.kt;
        if (lane < kMaskWords) mask[lane] = 0u;
        __syncwarp();
        // eight 32-entry chunks in flight per step (the list's loads do not wait on each other);
        // the positions are kept in shared memory for the per-tile gathers
        bool stopped = false;
        for (int e0 = 0; e0 < p.kt && !stopped; e0 += 256) {
          int jv[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int e = e0 + 32 * c + lane;
            jv[c] = e < p.kt ? sel[e] : -1;
          }
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            if (stopped) break;
            const int e = e0 + 32 * c + lane;
            const int j = jv[c];
            const unsigned stop = __ballot_sync(0xffffffffu, j < 0);       // first -1 ends the list
            const int first_stop = stop ? __ffs(stop) - 1 : 32;
            const bool live = lane < first_stop;
            nA += __popc(__ballot_sync(0xffffffffu, live && j < x0.w0));
            if (live && j >= x0.w0 && j <= x0.eI) atomicOr(&mask[(j - x0.w0) >> 5], 1u << ((j - x0.w0) & 31));
            if (stop) stopped = true;
          }
        }
      }
      __syncwarp();
      __threadfence_block();
      if (lane == 0) {
        // the slot is free (waited above); publish the id and nA (the mask is already in place)
        const uint32_t sl = n % tc::kQueueSlots;
        bars->queue.unit[sl] = u;
        bars->queue.info[sl][0] = nA;
        tc::mbar_arrive(&bars->queue.full[sl]);
      }
      if (u < 0) break;
      const Unit x = make_unit(p, u, nA);
      const int ntiles = x.n_sp + x.n_w;
      const int head_row0 = (x.b * p.Hkv + x.g) * p.N;
      for (int r = 0; r < rounds && ok; ++r) {
        if (lane == 0) {
          for (int s = 0; s < 2 && ok; ++s) {
            const int mt = kRoundStride * r + mt0 + s;
            if (mt >= MT) continue;
            if (!(ok = tc::mbar_wait(&bars->q_empty[s], (q_cnt[s] & 1u) ^ 1u, abort))) break;
            ++q_cnt[s];
            tc::mbar_arrive_expect_tx(&bars->q_full[s], C::kQBytes);
            uint8_t* qdst = smem + C::kOffQ + s * C::kQBytes;
            const int h0 = x.g * p.G + 2 * mt;
            for (int hh = 0; hh < 2; ++hh)
              for (int ch = 0; ch < C::kChunks; ++ch)
                tc::tma_load_3d(&tmQ, &bars->q_full[s], qdst + ch * 16384 + hh * 8192, ch * 64, 64 * x.I,
                                x.b * p.Hq + h0 + hh);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        // part A positions of this lane's quad, read from the (L2-resident) index list one tile
        // ahead of their gathers
        auto positions = [&](int tau, int (&pos)[4]) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int e = PAIR ? 128 * tau + 64 * (int)rank + 4 * (lane & 15) + k : 128 * tau + 4 * lane + k;
            pos[k] = (tau < x.n_sp && e < x.nA) ? __ldg(sel + e) : 0;   // padding: row 0 (masked)
          }
        };
        int nxt[4];
        positions(0, nxt);
        for (int tau = 0; tau < ntiles && ok && PAIR; ++tau) {
          // this CTA's half of the tile: rows 64 rank .. 64 rank + 63.  Part A: lane = (column
          // chunk, quad of rows) gathers four rows; part B: one 64-row box per column chunk.
          const bool part_a = tau < x.n_sp;
          const int ch = lane >> 4, quad = lane & 15;
          int rows[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) rows[k] = head_row0 + nxt[k];
          positions(tau + 1, nxt);
          const int brow = head_row0 + x.w0 + 128 * (tau - x.n_sp) + 64 * (int)rank;  // past e_I: masked
          for (int kv = 0; kv < 2; ++kv) {
            const uint32_t st = kv_it % kStages;
            if (lane == 0) {
              ok = tc::mbar_wait(&bars->kv_empty[st], ((kv_it / kStages) & 1u) ^ 1u, abort);
              if (ok) tc::mbar_arrive_expect_tx(&bars->kv_half[st], C::kHalfBytes);
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            uint8_t* dst = smem + C::kOffKV + st * C::kKVBytes + 64 * (int)rank * 128;
            if (part_a) {
              if (ch < C::kChunks)
                tc::tma_gather4(kv ? &tmV : &tmK, &bars->kv_half[st], dst + ch * 16384 + 4 * quad * 128, ch * 64,
                                rows[0], rows[1], rows[2], rows[3]);
            } else if (lane == 0) {
              for (int c = 0; c < C::kChunks; ++c)
                tc::tma_load_2d(kv ? &tmVb : &tmKb, &bars->kv_half[st], dst + c * 16384, c * 64, brow);
            }
            ++kv_it;
          }
        }
        for (int tau = 0; tau < ntiles && ok && !PAIR; ++tau) {
          // key rows of this lane's quad (rows 4*lane .. 4*lane+3 of the tile)
          int rows[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int rr = 4 * lane + k;
            int pos = nxt[k];
            if (tau >= x.n_sp) {
              const int i = x.w0 + 128 * (tau - x.n_sp) + rr;
              pos = i <= x.eI ? i : 0;
            }
            rows[k] = head_row0 + pos;
          }
          positions(tau + 1, nxt);
          for (int kv = 0; kv < 2; ++kv) {
            const uint32_t st = kv_it % kStages;
            if (lane == 0) {
              ok = tc::mbar_wait(&bars->kv_empty[st], ((kv_it / kStages) & 1u) ^ 1u, abort);
              if (ok) tc::mbar_arrive_expect_tx(&bars->kv_full[st], C::kKVBytes);
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            uint8_t* dst = smem + C::kOffKV + st * C::kKVBytes;
            for (int ch = 0; ch < C::kChunks; ++ch)
              tc::tma_gather4(kv ? &tmV : &tmK, &bars->kv_full[st], dst + ch * 16384 + 4 * lane * 128, ch * 64,
                              rows[0], rows[1], rows[2], rows[3]);
            ++kv_it;
          }
        }
      }
    }
    if (lane == 0) {
      if (!ok) fail(abort, p.status);
      for (uint32_t i = (kv_it > kStages ? kv_it - kStages : 0); i < kv_it; ++i)
        tc::mbar_wait_drain(&bars->kv_full[i % kStages], (i / kStages) & 1u);
      for (int s = 0; s < 2; ++s)
        if (q_cnt[s] > 0) tc::mbar_wait_drain(&bars->q_full[s], (q_cnt[s] - 1) & 1u);
      // pair: this CTA's own gathers of the last uses, and each stage's last use released by
      // both MMAs, so every half this CTA sent has been read by the partner before either leaves
      if (PAIR)
        for (uint32_t i = (kv_it > kStages ? kv_it - kStages : 0); i < kv_it; ++i) {
          tc::mbar_wait_drain(&bars->kv_half[i % kStages], (i / kStages) & 1u);
          tc::mbar_wait_drain(&bars->kv_empty[i % kStages], (i / kStages) & 1u);
        }
    }
  } else if (warp == 1) {
    // ============================================================== MMA issuer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kLowRegs));
    if (lane == 0) {
      const uint32_t idS = tc::idesc_bf16_f32(128, 128, false);
      const uint32_t idO = tc::idesc_bf16_f32(128, D, true);
      const uint32_t tS[2] = {tmem_base, tmem_base + 128};
      const uint32_t tO[2] = {tmem_base + 256, tmem_base + 384};
      const uint32_t qaddr = tc::smem_u32(smem + C::kOffQ);
      const uint32_t kvaddr = tc::smem_u32(smem + C::kOffKV);
      uint32_t kv_it = 0, q_cnt[2] = {0, 0}, p_cnt[2] = {0, 0}, o_cnt[2] = {0, 0};
      bool ok = true;
      auto issue_S = [&](int s, uint32_t st) {
        const uint32_t qb = qaddr + s * C::kQBytes, kb = kvaddr + st * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          tc::mma_ss(tS[s], tc::sdesc_sw128(qb + off, 16, 1024), tc::sdesc_sw128(kb + off, 16, 1024), idS,
                     kk > 0 ? 1u : 0u);
        }
      };
      // a stage is released to both CTAs of a pair (each gathered half of it)
      auto release_kv = [&](uint32_t st) {
        if (PAIR)
          tc::mma_commit_cluster(&bars->kv_empty[st], 0x3);
        else
          tc::mma_commit(&bars->kv_empty[st]);
      };
      auto issue_PV = [&](int s, uint32_t st, bool acc) {
        const uint32_t vb = kvaddr + st * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_ts(tO[s], tS[s] + kk * 8, tc::sdesc_sw128(vb + kk * 2048, 16384, 1024), idO,
                     (acc || kk > 0) ? 1u : 0u);
      };
      for (uint32_t n = 0; ok; ++n) {
        int nA = 0, unused = 0;
        const int u = tc::queue_peek(&bars->queue, n, abort, ok, &nA, &unused);
        if (u < 0) break;
        const Unit x = make_unit(p, u, nA);
        const int ntiles = x.n_sp + x.n_w;
        for (int r = 0; r < rounds && ok; ++r) {
          bool act[2];
          for (int s = 0; s < 2; ++s) {
            act[s] = (kRoundStride * r + mt0 + s) < MT;
            if (act[s] && ok) {
              ok = tc::mbar_wait(&bars->q_full[s], q_cnt[s] & 1u, abort);
              ++q_cnt[s];
            }
          }
          if (!ok) break;
          uint32_t kst = kv_it % kStages;
          if (!(ok = tc::mbar_wait(&bars->kv_full[kst], (kv_it / kStages) & 1u, abort))) break;
          ++kv_it;
          tc::fence_after_sync();
          for (int s = 0; s < 2; ++s)
            if (act[s]) {
              issue_S(s, kst);
              tc::mma_commit(&bars->s_full[s]);
            }
          release_kv(kst);
          for (int tau = 1; tau <= ntiles && ok; ++tau) {
            const uint32_t vst = kv_it % kStages;
            if (!(ok = tc::mbar_wait(&bars->kv_full[vst], (kv_it / kStages) & 1u, abort))) break;
            ++kv_it;
            bool have_k = false;
            for (int s = 0; s < 2 && ok; ++s) {
              if (!act[s]) continue;
              if (!(ok = tc::mbar_wait(&bars->p_full[s], p_cnt[s] & 1u, abort))) break;
              ++p_cnt[s];
              if (tau == 1) {
                if (!(ok = tc::mbar_wait(&bars->o_empty[s], (o_cnt[s] & 1u) ^ 1u, abort))) break;
              }
              tc::fence_after_sync();
              issue_PV(s, vst, tau > 1);
              if (tau < ntiles) {
                if (!have_k) {
                  kst = kv_it % kStages;
                  if (!(ok = tc::mbar_wait(&bars->kv_full[kst], (kv_it / kStages) & 1u, abort))) break;
                  ++kv_it;
                  have_k = true;
                  tc::fence_after_sync();
                }
                issue_S(s, kst);
                tc::mma_commit(&bars->s_full[s]);
              } else {
                tc::mma_commit(&bars->o_full[s]);
                ++o_cnt[s];
              }
            }
            release_kv(vst);
            if (have_k) release_kv(kst);
          }
          for (int s = 0; s < 2; ++s)
            if (act[s]) tc::mma_commit(&bars->q_empty[s]);
        }
        tc::queue_release(&bars->queue, n);
      }
      if (!ok) fail(abort, p.status);
      tc::mma_commit(&bars->mma_drain);
      tc::mbar_wait_drain(&bars->mma_drain, 0);
    }
  } else if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kLowRegs));
    if (PAIR && warp == 2 && lane == 0) {
      // ============================================================== copier (CTA pair)
      // once this CTA's half of a stage has landed, send it into the partner's stage (its bytes
      // complete the partner's kv_full) and expect the partner's half on our own kv_full
      const uint32_t peer = rank ^ 1u;
      uint32_t kv_it = 0;
      bool ok = true;
      for (uint32_t n = 0; ok; ++n) {
        int nA = 0, unused = 0;
        const int u = tc::queue_peek(&bars->queue, n, abort, ok, &nA, &unused);
        if (u < 0) break;
        const Unit x = make_unit(p, u, nA);
        const int nkv = 2 * rounds * (x.n_sp + x.n_w);
        for (int i = 0; i < nkv && ok; ++i) {
          const uint32_t st = kv_it % kStages;
          if (!(ok = tc::mbar_wait(&bars->kv_half[st], (kv_it / kStages) & 1u, abort))) break;
          ++kv_it;
          tc::mbar_arrive_expect_tx(&bars->kv_full[st], C::kHalfBytes);
          const uint32_t bar_peer = tc::peer_addr(&bars->kv_full[st], peer);
          for (int c = 0; c < C::kChunks; ++c) {
            const uint8_t* src = smem + C::kOffKV + st * C::kKVBytes + c * 16384 + 64 * (int)rank * 128;
            tc::bulk_copy_to_peer(tc::peer_addr(src, peer), src, C::kHalfBytes / C::kChunks, bar_peer);
          }
        }
        tc::queue_release(&bars->queue, n);
      }
      if (!ok) fail(abort, p.status);
    }
  } else {
    // ============================================================== softmax / epilogue
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kHighRegs));
    const int s = (warp - 4) >> 2;
    const int row = 32 * (warp & 3) + lane;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tSrow = tmem_base + 128 * s + lane_off;
    const uint32_t tOrow = tmem_base + 256 + 128 * s + lane_off;
    const float sc = p.scale_log2;
    uint32_t s_cnt = 0, o_cnt = 0;
    bool ok = true;
    for (uint32_t n = 0; ok; ++n) {
      int nA = 0, unused = 0;
      const int u = tc::queue_peek(&bars->queue, n, abort, ok, &nA, &unused);
      ok = __all_sync(0xffffffffu, ok);   // warp-uniform: TMEM accesses are warp-collective
      if (__any_sync(0xffffffffu, u < 0)) break;
      const Unit x = make_unit(p, u, nA);
      const uint32_t* mask = bars->selmask[n % tc::kQueueSlots];
      const int ntiles = x.n_sp + x.n_w;
      for (int r = 0; r < rounds && ok; ++r) {
        const int mt = kRoundStride * r + mt0 + s;
        if (mt >= MT) continue;
        const int h = x.g * p.G + 2 * mt + (row >> 6);
        const int t = 64 * x.I + (row & 63);
        const bool valid = t < p.N;
        float m_used = -INFINITY, l = 0.0f;
        for (int tau = 0; tau < ntiles; ++tau) {
          if (!(ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->s_full[s], s_cnt & 1u, abort)))) break;
          ++s_cnt;
          tc::fence_after_sync();
          float sv[128];
          {
            uint32_t r0[32], r1[32], r2[32], r3[32];
            tc::tmem_ld32(tSrow + 0, r0);
            tc::tmem_ld32(tSrow + 32, r1);
            tc::tmem_ld32(tSrow + 64, r2);
            tc::tmem_ld32(tSrow + 96, r3);
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              sv[i] = __uint_as_float(r0[i]);
              sv[32 + i] = __uint_as_float(r1[i]);
              sv[64 + i] = __uint_as_float(r2[i]);
              sv[96 + i] = __uint_as_float(r3[i]);
            }
          }
          if (tau < x.n_sp) {
            const int nvis = x.nA - 128 * tau;  // part A: only padding columns are masked
            if (nvis < 128) {
#pragma unroll
              for (int i = 0; i < 128; ++i)
                if (i >= nvis) sv[i] = -INFINITY;
            }
          } else {
            // part B: key i = base + c; own window, or selected and at or before t - W
            const int base = x.w0 + 128 * (tau - x.n_sp);
            const int mw0 = (128 * (tau - x.n_sp)) >> 5;
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
              const uint32_t bits = (mw0 + wd < kMaskWords) ? mask[mw0 + wd] : 0u;
#pragma unroll
              for (int c = 0; c < 32; ++c) {
                const int i = base + 32 * wd + c;
                const bool win = i >= t - p.W + 1 && i <= t;
                const bool selected = ((bits >> c) & 1u) && i <= t - p.W;
                if (!((win || selected) && i <= x.eI)) sv[32 * wd + c] = -INFINITY;
              }
            }
          }
          const float2 sc2 = make_float2(sc, sc);
          // P = exp2(s sc - ms) written to TMEM as bf16 over S; returns the row sum and (three-
          // input max chains on the ALU, beside the MUFU work) the row max
          auto emit_p = [&](float ms, float& rmax) -> float {
            const float2 nm2 = make_float2(-ms, -ms);
            float2 acc[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
            float mk[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float s0 = sv[32 * c + 2 * i], s1 = sv[32 * c + 2 * i + 1];
                mk[i & 3] = tc::fmax3(mk[i & 3], s0, s1);
                const float2 pv = exp2_pair(tc::ffma2(make_float2(s0, s1), sc2, nm2), 16 * c + i);
                acc[i & 1] = tc::fadd2(acc[i & 1], pv);
                pk[i] = tc::pack_bf16x2(pv.x, pv.y);
              }
              tc::tmem_st16(tSrow + 16 * c, pk);
            }
            rmax = tc::fmax3(fmaxf(mk[0], mk[1]), mk[2], mk[3]);
            const float2 a = tc::fadd2(acc[0], acc[1]);
            return a.x + a.y;
          };
          // The row max is needed first only while the row has none: later tiles compute P with
          // the running max straight away and find the tile max beside it; a row whose max rose
          // by more than 2^kRescaleLog2 redoes the tile with the new max (rare), and O is
          // rescaled.  Warp-uniform branches only: TMEM loads and stores are warp-collective.
          if (m_used == -INFINITY) m_used = fmaxf(tc::max64(sv), tc::max64(sv + 64));
          float mx;
          float lt = emit_p(m_used == -INFINITY ? 0.0f : m_used * sc, mx);
          float alpha = 1.0f;
          const bool rescale = mx > -INFINITY && (mx - m_used) * sc > kRescaleLog2;
          if (__any_sync(0xffffffffu, rescale)) {
            if (rescale) {
              alpha = exp2f((m_used - mx) * sc);
              m_used = mx;
            }
            float unused;
            lt = emit_p(m_used * sc, unused);   // unchanged rows write the same P again
            if (tau > 0) {
              uint32_t ov[D];
#pragma unroll
              for (int c = 0; c < D / 32; ++c) tc::tmem_ld32(tOrow + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(ov + 32 * c));
              tc::tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < D; i += 2) {
                const float2 vv = tc::fmul2(make_float2(__uint_as_float(ov[i]), __uint_as_float(ov[i + 1])), make_float2(alpha, alpha));
                ov[i] = __float_as_uint(vv.x);
                ov[i + 1] = __float_as_uint(vv.y);
              }
#pragma unroll
              for (int c = 0; c < D / 32; ++c) tc::tmem_st32(tOrow + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(ov + 32 * c));
            }
          }
          l = l * alpha + lt;
          tc::tmem_wait_st();
          tc::fence_before_sync();
          tc::mbar_arrive(&bars->p_full[s]);
        }
        if (!ok) break;
        if (!(ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->o_full[s], o_cnt & 1u, abort)))) break;
        ++o_cnt;
        tc::fence_after_sync();
        const float il = l > 0.0f ? 1.0f / l : 0.0f;
        __nv_bfloat16* orow = p.o + (((size_t)x.b * p.Hq + h) * p.N + t) * D;
        uint32_t pk[D / 2];
        {
          uint32_t ov[D];
#pragma unroll
          for (int c = 0; c < D / 32; ++c) tc::tmem_ld32(tOrow + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(ov + 32 * c));
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < D / 2; ++i) {
            const float2 vv = tc::fmul2(make_float2(__uint_as_float(ov[2 * i]), __uint_as_float(ov[2 * i + 1])), make_float2(il, il));
            pk[i] = tc::pack_bf16x2(vv.x, vv.y);
          }
        }
        tc::fence_before_sync();
        tc::mbar_arrive(&bars->o_empty[s]);  // O may be overwritten by the next round from here on
        if (valid) {
          if (p.o_v8) {  // 32-byte aligned output: 256-bit stores, full sectors
#pragma unroll
            for (int i = 0; i < D / 16; ++i) tc::st_global_v8(orow + 16 * i, pk + 8 * i);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
            for (int i = 0; i < D / 8; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      }
      tc::queue_release(&bars->queue, n);
    }
    if (!ok) fail(abort, p.status);
  }

  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem_base, 512);
  }
  if (PAIR) tc::cluster_sync();   // neither CTA's shared memory goes away while the partner may use it
}

// Q: [heads][rows][D], box 64 columns x 64 rows x 1 head
bool make_q_map(CUtensorMap* m, const void* base, int D, int rows, int heads) {
  EncodeTiledFn fn = tma_encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K or V as a 2-D [B*Hkv*N][D] tensor with a box of 64 columns x box_rows rows (one row for
// tile::gather4, 64 for part B's half tiles)
bool make_kv_map(CUtensorMap* m, const void* base, int D, long long rows, int box_rows) {
  EncodeTiledFn fn = tma_encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_units(const PrefillDims& d) { return d.B * d.Hkv * d.T; }
int grid_size(const PrefillDims& d) { return num_units(d) < kMaxGrid ? num_units(d) : kMaxGrid; }

// The register split assumes exactly kLaunchRegs per thread at launch.
template <int D, bool PAIR>
cudaError_t check_regs() {
  static std::atomic<int> regs{-1};
  int r = regs.load(std::memory_order_relaxed);
  if (r < 0) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, token_sparse_tc_kernel<D, PAIR>);
    if (e != cudaSuccess) return e;
    r = fa.numRegs;
    regs.store(r, std::memory_order_relaxed);
  }
  return r == kLaunchRegs ? cudaSuccess : cudaErrorInvalidConfiguration;
}

// Clusters of two that fit on the device at once (per device; 0 = not known yet).
template <int D>
int pair_clusters(cudaStream_t s) {
  static std::atomic<int> known[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int n = known[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * kMaxGrid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Cfg<D>::kSmemBytes;
  cfg.stream = s;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  if (cudaOccupancyMaxActiveClusters(&n, token_sparse_tc_kernel<D, true>, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    return 0;
  }
  known[dev].store(n, std::memory_order_relaxed);
  return n;
}

template <int D>
cudaError_t launch_typed(const PrefillDims& d, const void* q, const void* k, const void* v, const int* idx, int kt,
                         int W, void* o, void* ws, cudaStream_t s) {
  CUtensorMap mq, mk, mv, mkb, mvb;
  const long long rows = (long long)d.B * d.Hkv * d.N;
  if (!make_q_map(&mq, q, D, d.N, d.B * d.Hq) || !make_kv_map(&mk, k, D, rows, 1) ||
      !make_kv_map(&mv, v, D, rows, 1) || !make_kv_map(&mkb, k, D, rows, 64) || !make_kv_map(&mvb, v, D, rows, 64))
    return cudaErrorInvalidValue;
  Params p;
  p.B = d.B;
  p.N = d.N;
  p.Hq = d.Hq;
  p.Hkv = d.Hkv;
  p.G = d.G();
  p.T = d.T;
  p.kt = kt;
  p.W = W;
  p.num_units = num_units(d);
  p.idx = idx;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.o_v8 = (reinterpret_cast<uintptr_t>(o) & 31u) == 0;
  p.counter = reinterpret_cast<int*>(ws);
  p.status = device_status_ptr();
  p.scale_log2 = kLog2e / sqrtf((float)D);
  const int smem = Cfg<D>::kSmemBytes;
  // four or more M-tiles per unit: a single CTA would gather every key tile once per round.
  // HYS_TOKEN_SINGLE_CTA=1 (tests only) keeps the single-CTA kernel, the path taken where no
  // cluster of two fits, so that its rounds are checked too
  static const bool single_forced = [] {
    const char* e = getenv("HYS_TOKEN_SINGLE_CTA");
    return e != nullptr && e[0] == '1';
  }();
  const bool pair = HYS_TOKEN_PAIR && p.G / 2 >= 3 && !single_forced;
  cudaError_t e = pair ? check_regs<D, true>() : check_regs<D, false>();
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(pair ? token_sparse_tc_kernel<D, true> : token_sparse_tc_kernel<D, false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int ncl = 0;
  if (pair) ncl = std::min(pair_clusters<D>(s), p.num_units);
  if (ncl > 0) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * ncl);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, token_sparse_tc_kernel<D, true>, mq, mk, mv, mkb, mvb, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  if (pair) {   // no cluster fits: the single-CTA kernel
    e = check_regs<D, false>();
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(token_sparse_tc_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
  }
  e = cudaMemsetAsync(p.counter, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  token_sparse_tc_kernel<D, false><<<grid_size(d), kThreads, smem, s>>>(mq, mk, mv, mkb, mvb, p);
  return cudaGetLastError();
}

}  // namespace

bool token_sparse_tc_supported(const PrefillDims& d, hys_dtype dt, int forced) {
  // the part-B mask covers at most 32 * kMaskWords keys: W + 63 of them
  return dt == HYS_BF16 && (d.D == 64 || d.D == 128) && d.G() % 2 == 0 && forced + 63 <= 32 * kMaskWords &&
         (long long)d.B * d.Hkv * d.N < (1ll << 31);
}

size_t token_sparse_tc_workspace() { return 256; }

cudaError_t launch_token_sparse_tc(const PrefillDims& d, const void* q, const void* k, const void* v, const int* idx,
                                   int kt, int forced, void* o, void* ws, cudaStream_t s) {
  if (ws == nullptr) return cudaErrorInvalidValue;
  return d.D == 64 ? launch_typed<64>(d, q, k, v, idx, kt, forced, o, ws, s)
                   : launch_typed<128>(d, q, k, v, idx, kt, forced, o, ws, s);
}

}  // namespace hys
