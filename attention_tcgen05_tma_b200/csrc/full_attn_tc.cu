// Full attention layer with fused block scores on the 5th-generation tensor cores.
//
// What it computes (HySparse 3.4.1): causal GQA attention o_t, and
//   score[b,g,I,j] = R_{h in g} R_{t in tile I} exp(m~_{t,j} - m_t) / l_t ,   j <= I,
// where m~_{t,j} is the row max logit of 64-key block j (clipped at t), m_t and l_t the
// final softmax max and normaliser of row t (the paper's two-pass rescale, with the
// exp), and R = sum (default) or max over the query heads of KV group g and the rows of
// 64-query tile I.
//
// How (B200-first):
//   * Persistent CTAs (one per SM) walk work units (b, g, I) longest-first.  A unit holds
//     the G query heads of KV group g for the 64 positions of tile I.  They are packed two
//     heads per 128-row M-tile (rows 0-63 head 2m, rows 64-127 head 2m+1, same positions),
//     so every K/V tile staged in shared memory serves two heads, the causal extent of all
//     rows of an M-tile is the same, and the whole score reduction of a unit stays in the
//     CTA (no per-head partials, no second kernel).
//   * Two M-tiles are in flight (ping-pong): S_s = Q_s K^T (tcgen05.mma, SS, fp32 in
//     TMEM), softmax warpgroup s turns S_s into P_s (bf16, written back into the same TMEM
//     columns) and O_s += P_s V (tcgen05.mma with A from TMEM).  TMEM: S0 S1 O0 O1 = 512
//     columns.  K/V tiles (128 keys) arrive by TMA (128-byte swizzle) into a 4-stage ring.
//   * The block max logits m~ fall out of the softmax row max for free: each thread owns
//     one row and takes the max of the two 64-column halves of the 128-key S tile.  They are
//     stashed (fp32, L2-resident per-CTA scratch) because m_t, l_t are final only after the
//     last key tile; the M-tile epilogue rescales them and reduces over the tile's rows
//     into a shared-memory accumulator per slot; the unit epilogue writes the scores.
//   * Conditional rescaling: O and l are rescaled only when the row max grows by more
//     than 2^8 (in exp2 units); the result is exact after the final normalisation.
//   * Every wait is a bounded mbarrier wait; on expiry the kernel records HYS_ERR_TIMEOUT,
//     drains its own TMA loads and MMAs, frees TMEM and returns.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tma_host.h"
#include "tc_ptx.cuh"

namespace hys {

namespace {

constexpr int kThreads = 384;      // warp 0 TMA, warp 1 MMA, warps 4-7 / 8-11 softmax slots 0 / 1
constexpr int kStages = 4;         // K/V ring depth (one stage = one 128-key K or V tile)
constexpr int kMaxNB = 2048;       // score accumulator capacity per slot (N <= 131072)
constexpr int kMaxGrid = 148;      // B200 SM count; the workspace is sized for this grid
constexpr float kRescaleLog2 = 8.0f;
#ifndef HYS_FULL_POLY_PAIRS
#define HYS_FULL_POLY_PAIRS 4
#endif
// column pairs (of the 64 in a 128-key row) whose exp2 runs on the FMA pipe instead of MUFU
constexpr int kPolyPairs = HYS_FULL_POLY_PAIRS;
// Register split between the warpgroups (setmaxnreg): the launch gives every thread
// kLaunchRegs; the producer/MMA warpgroup drops to kLowRegs and each softmax warpgroup rises to
// kHighRegs.  The sum must equal three launch shares, or setmaxnreg.inc would wait forever;
// the host checks the compiled register count before every launch.
#ifndef HYS_FULL_LOW_REGS
#define HYS_FULL_LOW_REGS 104
#endif
constexpr int kLaunchRegs = 168, kLowRegs = HYS_FULL_LOW_REGS, kHighRegs = (3 * kLaunchRegs - kLowRegs) / 2;
static_assert(kLowRegs % 8 == 0 && kHighRegs % 8 == 0, "setmaxnreg takes multiples of 8");
static_assert(kLowRegs + 2 * kHighRegs == 3 * kLaunchRegs, "register split must match the launch allocation");

__device__ __forceinline__ float2 exp2_pair(float2 x, int i) {
  if ((i * kPolyPairs) % 64 < kPolyPairs) return tc::exp2_poly3_x2(x);
  return make_float2(exp2f(x.x), exp2f(x.y));
}


struct Params {
  int B, N, Hq, Hkv, G, T, NB, NBpad;
  int num_units;
  __nv_bfloat16* o;
  int o_v8;       // o is 32-byte aligned (256-bit stores)
  float* lse;     // optional [B,Hq,N]
  float* scores;  // optional [B,Hkv,T,NB], or [B,Hkv,N,NB] per position (emitted iff non-null)
  int per_row;    // per-position scores: group max per (position, block), zeroed before the launch
  float* stash;   // [grid][2][128][NBpad]
  int* counter;   // work-unit counter (zeroed before the launch)
  int red_max;
  int* status;
  float scale_log2;  // log2(e) / sqrt(D)
};

struct Bars {
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t q_full[2], q_empty[2], s_full[2], p_full[2], o_full[2], o_empty[2], wg[2], all[2];
  uint64_t mma_drain, spare;
  tc::UnitQueue queue;
};

template <int D>
struct Cfg {
  static constexpr int kChunks = D / 64;             // 128-byte swizzle chunks per row
  static constexpr int kQBytes = 128 * D * 2;        // one M-tile of Q
  static constexpr int kKVBytes = 128 * D * 2;       // one K or V tile of 128 keys
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kQBytes;
  static constexpr int kOffAcc = kOffKV + kStages * kKVBytes;
  static constexpr int kOffRow = kOffAcc + 2 * kMaxNB * 4;
  static constexpr int kOffBar = kOffRow + 2 * 256 * 4;
  static constexpr int kOffMisc = kOffBar + (int)((sizeof(Bars) + 15) / 16 * 16);
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + slack for 1024-byte alignment
};

// Units are drawn from a counter in KV-group-major order, longest query tile first within a
// group: co-running CTAs then stream the same group's K/V (L2-resident), and the dynamic draw
// balances the causal lengths and leaves the shortest units for the tail.
__device__ __forceinline__ void unit_coords(const Params& p, int u, int& b, int& g, int& I) {
  const int bg = u / p.T;
  I = p.T - 1 - u % p.T;
  b = bg / p.Hkv;
  g = bg % p.Hkv;
}

// Group barrier on an mbarrier (count = group size); bounded, with acquire/release at CTA scope.
__device__ __forceinline__ bool group_sync(uint64_t* bar, uint32_t& phase, volatile int* abort) {
  tc::mbar_arrive(bar);
  const bool ok = tc::mbar_wait(bar, phase & 1u, abort);
  ++phase;
  return ok;
}

__device__ __forceinline__ void fail(volatile int* abort, int* status) {
  *abort = 1;
  report_status(status, HYS_ERR_TIMEOUT);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    full_attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 16);
  float* acc_all = reinterpret_cast<float*>(smem + C::kOffAcc);
  float* row_all = reinterpret_cast<float*>(smem + C::kOffRow);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool scores_on = p.scores != nullptr;
  const int MT = p.G / 2;              // M-tiles per unit
  const int rounds = (MT + 1) / 2;     // two M-tiles (slots) per round

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(&bars->kv_full[i], 1);
      tc::mbar_init(&bars->kv_empty[i], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->q_full[s], 1);
      tc::mbar_init(&bars->q_empty[s], 1);
      tc::mbar_init(&bars->s_full[s], 1);
      tc::mbar_init(&bars->p_full[s], 128);
      tc::mbar_init(&bars->o_full[s], 1);
      tc::mbar_init(&bars->o_empty[s], 128);
      tc::mbar_init(&bars->wg[s], 128);
      tc::mbar_init(&bars->all[s], 256);
    }
    tc::mbar_init(&bars->mma_drain, 1);
    tc::queue_init(&bars->queue, 1 + 256);  // MMA thread + both softmax warpgroups
    *abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tensormap(&tmQ);
    tc::prefetch_tensormap(&tmK);
    tc::prefetch_tensormap(&tmV);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, 512);
    tc::tmem_relinquish();
  }
  // zero the score accumulators
  for (int i = threadIdx.x; i < 2 * kMaxNB; i += kThreads) acc_all[i] = 0.0f;
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ============================================================== TMA producer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kLowRegs));
    if (lane == 0) {
      uint32_t kv_it = 0, q_cnt[2] = {0, 0};
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
            const int h0 = g * p.G + 2 * mt;
            uint8_t* qdst = smem + C::kOffQ + s * C::kQBytes;
            for (int hh = 0; hh < 2; ++hh)
              for (int c = 0; c < C::kChunks; ++c)
                tc::tma_load_3d(&tmQ, &bars->q_full[s], qdst + c * 16384 + hh * 8192, c * 64, 64 * I,
                                b * p.Hq + h0 + hh);
          }
          for (int tau = 0; tau < nkt && ok; ++tau) {
            for (int kv = 0; kv < 2; ++kv) {
              const uint32_t st = kv_it % kStages;
              if (!(ok = tc::mbar_wait(&bars->kv_empty[st], ((kv_it / kStages) & 1u) ^ 1u, abort))) break;
              tc::mbar_arrive_expect_tx(&bars->kv_full[st], C::kKVBytes);
              uint8_t* dst = smem + C::kOffKV + st * C::kKVBytes;
              for (int c = 0; c < C::kChunks; ++c)
                tc::tma_load_3d(kv ? &tmV : &tmK, &bars->kv_full[st], dst + c * 16384, c * 64, 128 * tau,
                                b * p.Hkv + g);
              ++kv_it;
            }
          }
        }
      }
      if (!ok) fail(abort, p.status);
      // drain: the last loads issued into each stage / Q slot must land before the CTA exits
      for (uint32_t i = (kv_it > kStages ? kv_it - kStages : 0); i < kv_it; ++i)
        tc::mbar_wait_drain(&bars->kv_full[i % kStages], (i / kStages) & 1u);
      for (int s = 0; s < 2; ++s)
        if (q_cnt[s] > 0) tc::mbar_wait_drain(&bars->q_full[s], (q_cnt[s] - 1) & 1u);
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
      auto issue_PV = [&](int s, uint32_t st, bool acc) {
        const uint32_t vb = kvaddr + st * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc::mma_ts(tO[s], tS[s] + kk * 8, tc::sdesc_sw128(vb + kk * 2048, 16384, 1024), idO,
                     (acc || kk > 0) ? 1u : 0u);
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
          // prologue: S_s(0) = Q_s K_0^T
          uint32_t kst = kv_it % kStages;
          if (!(ok = tc::mbar_wait(&bars->kv_full[kst], (kv_it / kStages) & 1u, abort))) break;
          ++kv_it;
          tc::fence_after_sync();
          for (int s = 0; s < 2; ++s)
            if (act[s]) {
              issue_S(s, kst);
              tc::mma_commit(&bars->s_full[s]);
            }
          tc::mma_commit(&bars->kv_empty[kst]);
          for (int tau = 1; tau <= nkt && ok; ++tau) {
            const uint32_t vst = kv_it % kStages;
            if (!(ok = tc::mbar_wait(&bars->kv_full[vst], (kv_it / kStages) & 1u, abort))) break;
            ++kv_it;
            bool have_k = false;
            for (int s = 0; s < 2 && ok; ++s) {
              if (!act[s]) continue;
              if (!(ok = tc::mbar_wait(&bars->p_full[s], p_cnt[s] & 1u, abort))) break;
              ++p_cnt[s];
              if (tau == 1) {  // the previous round's epilogue must have read O_s
                if (!(ok = tc::mbar_wait(&bars->o_empty[s], (o_cnt[s] & 1u) ^ 1u, abort))) break;
              }
              tc::fence_after_sync();
              issue_PV(s, vst, tau > 1);
              if (tau < nkt) {
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
            tc::mma_commit(&bars->kv_empty[vst]);
            if (have_k) tc::mma_commit(&bars->kv_empty[kst]);
          }
          for (int s = 0; s < 2; ++s)
            if (act[s]) tc::mma_commit(&bars->q_empty[s]);
        }
      }
      if (!ok) fail(abort, p.status);
      tc::mma_commit(&bars->mma_drain);
      tc::mbar_wait_drain(&bars->mma_drain, 0);
    }
  } else if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kLowRegs));
  } else {
    // ============================================================== softmax / epilogue
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kHighRegs));
    const int s = (warp - 4) >> 2;                 // slot
    const int row = 32 * (warp & 3) + lane;        // M-tile row == TMEM lane
    const int wtid = threadIdx.x - 128 - 128 * s;  // 0..127 within the warpgroup
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tSrow = tmem_base + 128 * s + lane_off;
    const uint32_t tOrow = tmem_base + 256 + 128 * s + lane_off;
    float* acc = acc_all + s * kMaxNB;
    float* row_m = row_all + 256 * s;
    float* row_il = row_m + 128;
    float* stash = p.stash + ((size_t)blockIdx.x * 2 + s) * 128 * (size_t)p.NBpad;
    const float sc = p.scale_log2;
    uint32_t s_cnt = 0, o_cnt = 0, wg_ph = 0, all_ph = 0;
    bool ok = true;
    for (uint32_t n = 0; ok; ++n) {
      const int u = tc::queue_pop(&bars->queue, n, abort, ok);
      // warp-uniform outcomes: the warp-collective TMEM accesses must not diverge
      ok = __all_sync(0xffffffffu, ok);
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
        float m_used = -INFINITY, l = 0.0f;
        for (int tau = 0; tau < nkt; ++tau) {
          if (!(ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->s_full[s], s_cnt & 1u, abort)))) break;
          ++s_cnt;
          tc::fence_after_sync();
          // S row from TMEM; keys past the row are masked on the causal diagonal
          const bool diag = tau == nkt - 1;
          const int cmax = t - 128 * tau;
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
            if (diag) {
#pragma unroll
              for (int i = 0; i < 128; ++i)
                if (i > cmax) sv[i] = -INFINITY;
            }
          }
          const float2 sc2 = make_float2(sc, sc);
          // P = exp2(s sc - ms) written to TMEM as bf16 over S; returns the row sum and (three-
          // input max chains on the ALU, beside the MUFU work) the maxima of the two 64-key
          // halves, which are the block maxima of blocks 2 tau and 2 tau + 1
          auto emit_p = [&](float ms, float& mlo, float& mhi) -> float {
            const float2 nm2 = make_float2(-ms, -ms);
            float2 acc[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
            float mk[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float s0 = sv[32 * c + 2 * i], s1 = sv[32 * c + 2 * i + 1];
                mk[2 * (c >> 1) + (i & 1)] = tc::fmax3(mk[2 * (c >> 1) + (i & 1)], s0, s1);
                const float2 pv = exp2_pair(tc::ffma2(make_float2(s0, s1), sc2, nm2), 16 * c + i);
                acc[i & 1] = tc::fadd2(acc[i & 1], pv);
                pk[i] = tc::pack_bf16x2(pv.x, pv.y);
              }
              tc::tmem_st16(tSrow + 16 * c, pk);
            }
            mlo = fmaxf(mk[0], mk[1]);
            mhi = fmaxf(mk[2], mk[3]);
            const float2 a = tc::fadd2(acc[0], acc[1]);
            return a.x + a.y;
          };
          // The row max is needed first only while the row has none: later tiles compute P
          // with the running max m_used straight away and find the tile maxima beside it; a row
          // whose max rose by more than 2^kRescaleLog2 redoes the tile with the new max (rare),
          // and O is rescaled.  Warp-uniform branches only: TMEM loads and stores are
          // warp-collective.
          if (m_used == -INFINITY) m_used = fmaxf(tc::max64(sv), tc::max64(sv + 64));
          float mlo, mhi;
          float lt = emit_p(m_used == -INFINITY ? 0.0f : m_used * sc, mlo, mhi);
          if (scores_on) *reinterpret_cast<float2*>(stash + (size_t)row * p.NBpad + 2 * tau) = make_float2(mlo, mhi);
          const float mt_ = fmaxf(mlo, mhi);
          float alpha = 1.0f;
          const bool rescale = (mt_ - m_used) * sc > kRescaleLog2;
          if (__any_sync(0xffffffffu, rescale)) {
            if (rescale) {
              alpha = exp2f((m_used - mt_) * sc);
              m_used = mt_;
            }
            float u0, u1;
            lt = emit_p(m_used * sc, u0, u1);   // unchanged rows write the same P again
            if (tau > 0) {
              // O_s holds the sum over the earlier key tiles; its last PV is complete because
              // S_s(tau), committed after it, is.  PV_s(tau) waits for p_full below.
              uint32_t ov[D];
#pragma unroll
              for (int c = 0; c < D / 32; ++c) tc::tmem_ld32(tOrow + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(ov + 32 * c));
              tc::tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < D; i += 2) {
                const float2 v = tc::fmul2(make_float2(__uint_as_float(ov[i]), __uint_as_float(ov[i + 1])), make_float2(alpha, alpha));
                ov[i] = __float_as_uint(v.x);
                ov[i + 1] = __float_as_uint(v.y);
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
        // ---- M-tile epilogue: O / l -> global, LSE, block-score contribution
        if (!(ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->o_full[s], o_cnt & 1u, abort)))) break;
        ++o_cnt;
        tc::fence_after_sync();
        const float il = 1.0f / l;
        __nv_bfloat16* orow = p.o + (((size_t)b * p.Hq + h) * p.N + t) * D;
        uint32_t pk[D / 2];
        {
          uint32_t ov[D];
#pragma unroll
          for (int c = 0; c < D / 32; ++c) tc::tmem_ld32(tOrow + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(ov + 32 * c));
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < D / 2; ++i) {
            const float2 v = tc::fmul2(make_float2(__uint_as_float(ov[2 * i]), __uint_as_float(ov[2 * i + 1])), make_float2(il, il));
            pk[i] = tc::pack_bf16x2(v.x, v.y);
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
        if (p.lse != nullptr && valid) p.lse[((size_t)b * p.Hq + h) * p.N + t] = (m_used * sc + log2f(l)) * 0.69314718055994531f;
        if (scores_on && p.per_row) {
          // per-position scores: rows r and r + 64 are the M-tile's two heads at one position;
          // their maximum joins the other heads' through an atomic max on the float bits (all
          // values are >= 0, so the bit patterns order like the floats; any order gives one result)
          row_m[row] = m_used;
          row_il[row] = valid ? il : 0.0f;
          if (!(ok = __all_sync(0xffffffffu, group_sync(&bars->wg[s], wg_ph, abort)))) break;
          const int nj = I + 1;
          unsigned int* out = reinterpret_cast<unsigned int*>(p.scores) + (((size_t)b * p.Hkv + g) * p.N + 64 * I) * p.NB;
          for (int e = wtid; e < 64 * nj; e += 128) {
            const int pos = e / nj, j = e - pos * nj;
            if (64 * I + pos >= p.N) break;
            const float x0 = exp2f((stash[(size_t)pos * p.NBpad + j] - row_m[pos]) * sc) * row_il[pos];
            const float x1 = exp2f((stash[(size_t)(pos + 64) * p.NBpad + j] - row_m[pos + 64]) * sc) * row_il[pos + 64];
            atomicMax(out + (size_t)pos * p.NB + j, __float_as_uint(fmaxf(x0, x1)));
          }
          if (!(ok = __all_sync(0xffffffffu, group_sync(&bars->wg[s], wg_ph, abort)))) break;
        } else if (scores_on) {
          row_m[row] = m_used;
          row_il[row] = valid ? il : 0.0f;
          if (!(ok = __all_sync(0xffffffffu, group_sync(&bars->wg[s], wg_ph, abort)))) break;
          for (int j = wtid; j <= I; j += 128) {
            float a = 0.0f;
            for (int rr = 0; rr < 128; ++rr) {
              const float x = exp2f((stash[(size_t)rr * p.NBpad + j] - row_m[rr]) * sc) * row_il[rr];
              a = p.red_max ? fmaxf(a, x) : a + x;
            }
            acc[j] = p.red_max ? fmaxf(acc[j], a) : acc[j] + a;
          }
          if (!(ok = __all_sync(0xffffffffu, group_sync(&bars->wg[s], wg_ph, abort)))) break;
        }
      }
      if (!ok) break;
      if (scores_on && !p.per_row) {
        // ---- unit epilogue: both slots' accumulators -> scores[b,g,I,:]
        if (!(ok = __all_sync(0xffffffffu, group_sync(&bars->all[0], all_ph, abort)))) break;
        float* out = p.scores + (((size_t)b * p.Hkv + g) * p.T + I) * p.NB;
        const int tid2 = wtid + 128 * s;
        for (int j = tid2; j < p.NB; j += 256) {
          float v = 0.0f;
          if (j <= I) v = p.red_max ? fmaxf(acc_all[j], acc_all[kMaxNB + j]) : acc_all[j] + acc_all[kMaxNB + j];
          out[j] = v;
        }
        if (!(ok = __all_sync(0xffffffffu, group_sync(&bars->all[0], all_ph, abort)))) break;
        for (int j = wtid; j <= I; j += 128) acc[j] = 0.0f;
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

// ------------------------------------------------------------------ host side
// [heads][rows][D] bf16, box = 64 columns x box_rows rows x 1 head, 128-byte swizzle
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

int nb_pad(int NB) { return (NB + 2 + 3) & ~3; }
int num_units(const PrefillDims& d) { return d.B * d.Hkv * d.T; }
int grid_size(const PrefillDims& d) { return num_units(d) < kMaxGrid ? num_units(d) : kMaxGrid; }

template <int D>
cudaError_t launch_typed(const PrefillDims& d, const void* q, const void* k, const void* v, void* o, float* lse,
                         float* scores, hys_reduce red, bool per_row, void* ws, cudaStream_t s) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, D, d.N, d.B * d.Hq, 64) || !make_map(&mk, k, D, d.N, d.B * d.Hkv, 128) ||
      !make_map(&mv, v, D, d.N, d.B * d.Hkv, 128))
    return cudaErrorInvalidValue;
  Params p;
  p.B = d.B;
  p.N = d.N;
  p.Hq = d.Hq;
  p.Hkv = d.Hkv;
  p.G = d.G();
  p.T = d.T;
  p.NB = d.NB;
  p.NBpad = nb_pad(d.NB);
  p.num_units = num_units(d);
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.o_v8 = (reinterpret_cast<uintptr_t>(o) & 31u) == 0;
  p.lse = lse;
  p.scores = scores;
  p.per_row = per_row ? 1 : 0;
  p.counter = reinterpret_cast<int*>(ws);
  p.stash = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + 256);
  p.red_max = red == HYS_REDUCE_MAX;
  p.status = device_status_ptr();
  p.scale_log2 = kLog2e / sqrtf((float)D);
  const int smem = Cfg<D>::kSmemBytes;
  static int regs = -1;   // the register split assumes exactly kLaunchRegs per thread at launch
  if (regs < 0) {
    cudaFuncAttributes fa;
    cudaError_t e0 = cudaFuncGetAttributes(&fa, full_attn_tc_kernel<D>);
    if (e0 != cudaSuccess) return e0;
    regs = fa.numRegs;
  }
  if (regs != kLaunchRegs) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(full_attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(p.counter, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  if (per_row && scores != nullptr) {
    e = cudaMemsetAsync(scores, 0, sizeof(float) * (size_t)d.B * d.Hkv * d.N * d.NB, s);
    if (e != cudaSuccess) return e;
  }
  full_attn_tc_kernel<D><<<grid_size(d), kThreads, smem, s>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace

bool full_attn_tc_supported(const PrefillDims& d, hys_dtype dt, bool want_scores) {
  if (dt != HYS_BF16 || (d.D != 64 && d.D != 128)) return false;
  if (d.G() % 2 != 0) return false;
  if (want_scores && d.NB > kMaxNB) return false;
  return true;
}

size_t full_attn_tc_workspace(const PrefillDims& d, bool want_scores) {
  return 256 + (want_scores ? sizeof(float) * (size_t)grid_size(d) * 2 * 128 * (size_t)nb_pad(d.NB) : 0);
}

cudaError_t launch_full_attn_tc(const PrefillDims& d, const void* q, const void* k, const void* v, void* o,
                                float* lse, float* scores, hys_reduce red, bool want_scores, void* ws, size_t ws_bytes,
                                cudaStream_t s, bool per_row) {
  if (!want_scores) scores = nullptr;
  if (ws == nullptr || ws_bytes < full_attn_tc_workspace(d, want_scores)) return cudaErrorInvalidValue;
  return d.D == 64 ? launch_typed<64>(d, q, k, v, o, lse, scores, red, per_row, ws, s)
                   : launch_typed<128>(d, q, k, v, o, lse, scores, red, per_row, ws, s);
}

}  // namespace hys
