// Sparse layer on the 5th-generation tensor cores: gathered block-sparse branch + SWA
// branch + sigmoid gate (HySparse 3.4.3).
//
//   o~_t = softmax attention of q'_t over {i <= t : floor(i/64) in Sel_I} of the shared K, V
//   o'_t = softmax attention of q'_t over [max(0, t-w+1), t] of the layer's own K', V'
//   o_t  = sigmoid(g0) o~_t + sigmoid(g1) o'_t
//
// Structure follows the full-layer kernel: persistent CTAs over units (b, g, I), two
// heads x 64 positions per 128-row M-tile, two M-tiles in flight, S and O in TMEM, P
// written back over S and fed to the P.V MMA from TMEM.  What differs:
//   * Gather: a 128-key tile holds two 64-key blocks.  Each block is one TMA box per
//     128-byte chunk at row 64*j of K (or V), so only the selected blocks are read; K~, V~
//     are never materialised.  A missing half (odd count, -1 padding) is loaded from a
//     row past the end of the tensor, which TMA fills with zeros.
//   * Both branches accumulate into the same O, with no scratch memory.  The tiles of a
//     round are: the selected blocks (online softmax into O); then the window tiles twice.
//     Before the first window pass the softmax warpgroup scales O in TMEM by sigmoid(g0)/l
//     (O becomes sigmoid(g0) o~, exactly); the first window pass only computes the window
//     branch's row max m' and sum l'; the second recomputes S and adds
//     P' = exp(s - m') * sigmoid(g1) / l' times V' to O, which then holds o_t.
//   * Masks: per 64-key half, the visible key range is [64j, min(t, 64j+63)] for a selected
//     block and [max(64j, t-w+1), min(t, 64j+63)] for a window block.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tma_host.h"
#include "tc_ptx.cuh"

namespace hys {

namespace {

constexpr int kThreads = 384;
// Register split between the warpgroups (setmaxnreg): the launch gives every thread
// kLaunchRegs; the producer/MMA warpgroup drops to kLowRegs and each softmax warpgroup rises to
// kHighRegs.  The sum must equal three launch shares, or setmaxnreg.inc would wait forever;
// the host checks the compiled register count before every launch.
#ifndef HYS_SPARSE_LOW_REGS
#define HYS_SPARSE_LOW_REGS 104
#endif
constexpr int kLaunchRegs = 168, kLowRegs = HYS_SPARSE_LOW_REGS, kHighRegs = (3 * kLaunchRegs - kLowRegs) / 2;
static_assert(kLowRegs % 8 == 0 && kHighRegs % 8 == 0, "setmaxnreg takes multiples of 8");
static_assert(kLowRegs + 2 * kHighRegs == 3 * kLaunchRegs, "register split must match the launch allocation");
constexpr int kStages = 4;
constexpr int kMaxGrid = 148;
constexpr int kMaxKb = 1024;
constexpr float kRescaleLog2 = 8.0f;
constexpr float kRescaleSum = 256.0f;   // 2^kRescaleLog2
#ifndef HYS_SPARSE_POLY_PAIRS
#define HYS_SPARSE_POLY_PAIRS 4
#endif
// column pairs (of the 64 in a 128-key row) whose exp2 runs on the FMA pipe instead of MUFU
constexpr int kPolyPairs = HYS_SPARSE_POLY_PAIRS;

__device__ __forceinline__ float2 exp2_pair(float2 x, int i) {
  if ((i * kPolyPairs) % 64 < kPolyPairs) return tc::exp2_poly3_x2(x);
  return make_float2(exp2f(x.x), exp2f(x.y));
}


constexpr int kRowWords = 16;   // per-position mode: union entries < 512 (N <= 32768)

struct Params {
  int B, N, Hq, Hkv, G, T, kb, window;
  int num_units;
  const int* idx;      // [B,Hkv,T,kb], or [B,Hkv,N,kb] per position
  const float* gate;   // [B,Hq,N,2]
  const float* sinks;  // [Hq,2] sink logits of the two branches, or null
  __nv_bfloat16* o;
  int o_v8;            // o is 32-byte aligned (256-bit stores)
  float* blse;         // training forward: [B,Hq,N,2] LSE of the sparse and window branches
  __nv_bfloat16* osp;  // training forward: [B,Hq,N,D] the gated sparse-branch part sigmoid(g0) o~
  int* counter;        // work-unit counter (zeroed before the launch)
  int* status;
  float scale_log2;
};

struct Bars {
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t q_full[2], q_empty[2], s_full[2], p_full[2], o_full[2], o_empty[2];
  uint64_t mma_drain, spare;
  tc::UnitQueue queue;
};

template <int D>
struct Cfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kKVBytes = 128 * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kQBytes;
  static constexpr int kOffList = kOffKV + kStages * kKVBytes;   // producer's copy of a unit's indices
  static constexpr int kOffBar = kOffList + kMaxKb * 4;
  static constexpr int kOffMisc = kOffBar + (int)((sizeof(Bars) + 15) / 16 * 16);
  // per-position mode: for each queue slot and each of the tile's 64 positions, the union
  // entries that position selected (bit e of row r), and the producer's union bitmap
  static constexpr int kOffRows = kOffMisc + 64;
  static constexpr int kOffUnion = kOffRows + tc::kQueueSlots * 64 * kRowWords * 4;
  static constexpr int kSmemBytes = kOffUnion + kRowWords * 4 + 1024;
};

struct Unit {
  int b, g, I;
  int nsel;    // leading valid selected entries (0 <= j <= I); later entries are ignored
  int diag;    // entry holding block I (causally masked per row), or -1
  int n_sp;    // sparse tiles
  int jw0;     // first window block
  int n_sw;    // window tiles (each appears twice: statistics pass, then P.V pass)
};

// tile kinds of a round: selected blocks, window statistics pass, window P.V pass
enum TileKind { kSparse = 0, kWinStats = 1, kWinPV = 2 };

__device__ __forceinline__ int tile_kind(const Unit& x, int tau) {
  return tau < x.n_sp ? kSparse : (tau < x.n_sp + x.n_sw ? kWinStats : kWinPV);
}
__device__ __forceinline__ int num_tiles(const Unit& x) { return x.n_sp + 2 * x.n_sw; }

// Units come from a counter in KV-group-major order, so co-running CTAs gather from the same
// group's K/V (L2-resident); within a group the order is longest-first.  nsel and diag are
// found once by the producer warp and published with the unit id.
__device__ __forceinline__ Unit make_unit(const Params& p, int u, int nsel, int diag) {
  Unit x;
  const int bg = u / p.T;
  x.I = p.T - 1 - u % p.T;
  x.b = bg / p.Hkv;
  x.g = bg % p.Hkv;
  x.nsel = nsel;
  x.diag = diag;
  x.n_sp = (nsel + 1) / 2;
  const int w_lo = 64 * x.I - p.window + 1;
  x.jw0 = w_lo > 0 ? w_lo / 64 : 0;
  x.n_sw = (x.I - x.jw0 + 2) / 2;
  return x;
}

// Per-position selection of a unit (warp-wide): the union of the 64 rows' blocks, in ascending
// order, goes to plist (nsel entries; diag = the entry of block I or -1); bit e of rb[r] is set
// when row r selected union entry e.  Blocks past I are never candidates of the tile's rows and,
// like padding entries (-1), are ignored.
__device__ __noinline__ void per_row_lists(const int* __restrict__ idx, int N, int Hkv, int kb, int b, int g, int I,
                                           int* plist, uint32_t* rb, uint32_t* ubits, int lane, int* out) {
  const int nw = (I >> 5) + 1;
  if (lane < kRowWords) ubits[lane] = 0u;
  for (int i = lane; i < 64 * kRowWords; i += 32) rb[i] = 0u;
  __syncwarp();
  const int rows = min(64, N - 64 * I);
  const int* base = idx + (((size_t)b * Hkv + g) * N + 64 * I) * kb;
  const int total = rows * kb;
  // pass 1: the union (eight 32-entry chunks in flight per step)
  for (int e0 = 0; e0 < total; e0 += 256) {
    int jv[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int e = e0 + 32 * c + lane;
      jv[c] = e < total ? base[e] : -1;
    }
#pragma unroll
    for (int c = 0; c < 8; ++c)
      if (jv[c] >= 0 && jv[c] <= I) atomicOr(&ubits[jv[c] >> 5], 1u << (jv[c] & 31));
  }
  __syncwarp();
  // lane w owns bitmap word w: its entries start at the exclusive prefix of the popcounts
  const uint32_t wv = lane < nw ? ubits[lane] : 0u;
  const int cnt = __popc(wv);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  const int excl = incl - cnt;
  const int nsel = __shfl_sync(0xffffffffu, incl, 31);
  {
    int pos = excl;
    for (uint32_t w = wv; w != 0u; w &= w - 1u) plist[pos++] = 32 * lane + __ffs(w) - 1;
  }
  const uint32_t wI = __shfl_sync(0xffffffffu, wv, I >> 5);
  const int xI = __shfl_sync(0xffffffffu, excl, I >> 5);
  const int diag = ((wI >> (I & 31)) & 1u) ? xI + __popc(wI & ((1u << (I & 31)) - 1u)) : -1;
  // pass 2: each row's selected blocks as union entries
  for (int e0 = 0; e0 < total; e0 += 256) {
    int jv[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int e = e0 + 32 * c + lane;
      jv[c] = e < total ? base[e] : -1;
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int j = jv[c];
      const bool in = j >= 0 && j <= I;
      const int w = in ? j >> 5 : 0;
      const int wp = __shfl_sync(0xffffffffu, excl, w);
      const uint32_t ww = __shfl_sync(0xffffffffu, wv, w);
      if (in) {
        const int ent = wp + __popc(ww & ((1u << (j & 31)) - 1u));
        const int r = (e0 + 32 * c + lane) / kb;
        atomicOr(&rb[r * kRowWords + (ent >> 5)], 1u << (ent & 31));
      }
    }
  }
  out[0] = nsel;
  out[1] = diag;
}

__device__ __forceinline__ void fail(volatile int* abort, int* status) {
  *abort = 1;
  report_status(status, HYS_ERR_TIMEOUT);
}

template <int D, bool PR, bool TR>   // PR: per-position selection (idx [B,Hkv,N,kb]); TR: training
                                     // forward (also writes the branch LSEs and sigmoid(g0) o~)
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKs,
                          const __grid_constant__ CUtensorMap tmVs, const Params p) {
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
    }
    tc::mbar_init(&bars->mma_drain, 1);
    tc::queue_init(&bars->queue, 1 + 256);
    *abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tensormap(&tmQ);
    tc::prefetch_tensormap(&tmK);
    tc::prefetch_tensormap(&tmV);
    tc::prefetch_tensormap(&tmKs);
    tc::prefetch_tensormap(&tmVs);
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
    // ============================================================== TMA producer (gather)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kLowRegs));
    // The whole warp reads a unit's index row (32 entries per step) and finds the leading
    // valid entries with a ballot; lane 0 then issues the Q and gathered K/V loads.
    int* plist = reinterpret_cast<int*>(smem + C::kOffList);
    uint32_t kv_it = 0, q_cnt[2] = {0, 0};
    bool ok = true;
    for (uint32_t n = 0; ok; ++n) {
      int u = 0;
      if (lane == 0) {
        const int c = atomicAdd(p.counter, 1);
        u = c < p.num_units ? c : -1;
      }
      u = __shfl_sync(0xffffffffu, u, 0);
      int nsel = 0, diag = -1;
      if (PR) {
        // the slot's row masks may be rewritten only after every consumer released the slot
        const uint32_t sl = n % tc::kQueueSlots;
        if (lane == 0) ok = tc::mbar_wait(&bars->queue.empty[sl], ((n / tc::kQueueSlots) & 1u) ^ 1u, abort);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        if (u >= 0) {
          const Unit x0 = make_unit(p, u, 0, -1);
          int nd[2];
          per_row_lists(p.idx, p.N, p.Hkv, p.kb, x0.b, x0.g, x0.I, plist,
                        reinterpret_cast<uint32_t*>(smem + C::kOffRows) + sl * 64 * kRowWords,
                        reinterpret_cast<uint32_t*>(smem + C::kOffUnion), lane, nd);
          nsel = nd[0];
          diag = nd[1];
        }
        __syncwarp();
        __threadfence_block();
        if (lane == 0) {
          bars->queue.unit[sl] = u;
          bars->queue.info[sl][0] = nsel;
          bars->queue.info[sl][1] = diag;
          tc::mbar_arrive(&bars->queue.full[sl]);
        }
      } else if (u >= 0) {
        const Unit x0 = make_unit(p, u, 0, -1);
        const int* sel = p.idx + (((size_t)x0.b * p.Hkv + x0.g) * p.T + x0.I) * p.kb;
        nsel = p.kb;
        for (int e0 = 0; e0 < p.kb; e0 += 32) {
          const int e = e0 + lane;
          const int j = e < p.kb ? sel[e] : -1;
          if (e < p.kb) plist[e] = j;
          const unsigned bad = __ballot_sync(0xffffffffu, e < p.kb && (j < 0 || j > x0.I));
          const unsigned dg = __ballot_sync(0xffffffffu, e < p.kb && j == x0.I);
          const int first_bad = bad ? e0 + __ffs(bad) - 1 : p.kb;
          if (diag < 0 && dg) {
            const int first_dg = e0 + __ffs(dg) - 1;
            if (first_dg < first_bad) diag = first_dg;
          }
          if (bad) {
            nsel = first_bad;
            break;
          }
        }
      }
      __syncwarp();
      if (lane == 0 && !PR) ok = tc::queue_push(&bars->queue, n, u, abort, nsel, diag);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok || u < 0) break;
      if (lane == 0) {
        const Unit x = make_unit(p, u, nsel, diag);
        const int ntiles = num_tiles(x);
        // part kv (0: K, 1: V) of tile tau into the next stage
        auto load_kv = [&](int tau, int kv) -> bool {
          const int kind = tile_kind(x, tau);
          const bool swa = kind != kSparse;
          const int wi = kind == kWinStats ? tau - x.n_sp : tau - x.n_sp - x.n_sw;  // window pair
          int jj[2];
          for (int hh = 0; hh < 2; ++hh) {
            if (!swa) {
              const int e = 2 * tau + hh;
              jj[hh] = e < x.nsel ? plist[e] : -1;
            } else {
              const int j = x.jw0 + 2 * wi + hh;
              jj[hh] = j <= x.I ? j : -1;
            }
          }
          const uint32_t st = kv_it % kStages;
          if (!tc::mbar_wait(&bars->kv_empty[st], ((kv_it / kStages) & 1u) ^ 1u, abort)) return false;
          tc::mbar_arrive_expect_tx(&bars->kv_full[st], C::kKVBytes);
          uint8_t* dst = smem + C::kOffKV + st * C::kKVBytes;
          const CUtensorMap* map = swa ? (kv ? &tmVs : &tmKs) : (kv ? &tmV : &tmK);
          for (int hh = 0; hh < 2; ++hh) {
            const int row = jj[hh] >= 0 ? 64 * jj[hh] : p.N;  // empty half: rows past the end read as zeros
            for (int ch = 0; ch < C::kChunks; ++ch)
              tc::tma_load_3d(map, &bars->kv_full[st], dst + ch * 16384 + hh * 8192, ch * 64, row,
                              x.b * p.Hkv + x.g);
          }
          ++kv_it;
          return true;
        };
        for (int r = 0; r < rounds && ok; ++r) {
          // The round's first K tile goes ahead of its Q tiles: its stage is free well before the
          // previous round's last MMA releases Q, and the Q tiles (HBM reads that the TMA unit
          // serves one after another) would otherwise hold it back.
          if (!(ok = load_kv(0, 0))) break;
          for (int s = 0; s < 2 && ok; ++s) {
            const int mt = 2 * r + s;
            if (mt >= MT) continue;
            if (!(ok = tc::mbar_wait(&bars->q_empty[s], (q_cnt[s] & 1u) ^ 1u, abort))) break;
            ++q_cnt[s];
            tc::mbar_arrive_expect_tx(&bars->q_full[s], C::kQBytes);
            const int h0 = x.g * p.G + 2 * mt;
            uint8_t* qdst = smem + C::kOffQ + s * C::kQBytes;
            for (int hh = 0; hh < 2; ++hh)
              for (int ch = 0; ch < C::kChunks; ++ch)
                tc::tma_load_3d(&tmQ, &bars->q_full[s], qdst + ch * 16384 + hh * 8192, ch * 64, 64 * x.I,
                                x.b * p.Hq + h0 + hh);
          }
          for (int tau = 0; tau < ntiles && ok; ++tau)
            for (int kv = (tau == 0 ? 1 : 0); kv < (tile_kind(x, tau) == kWinStats ? 1 : 2) && ok; ++kv)
              ok = load_kv(tau, kv);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    if (lane == 0) {
      if (!ok) fail(abort, p.status);
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
        int nsel = 0, diag = -1;
        const int u = tc::queue_pop(&bars->queue, n, abort, ok, &nsel, &diag);
        if (u < 0) break;
        const Unit x = make_unit(p, u, nsel, diag);
        const int ntiles = num_tiles(x);
        for (int r = 0; r < rounds && ok; ++r) {
          bool act[2];
          for (int s = 0; s < 2; ++s) act[s] = (2 * r + s) < MT;
          // the round's first K tile (loaded ahead of the Q tiles), then each slot's S as soon as
          // its Q has landed
          uint32_t kst = kv_it % kStages;
          if (!(ok = tc::mbar_wait(&bars->kv_full[kst], (kv_it / kStages) & 1u, abort))) break;
          ++kv_it;
          for (int s = 0; s < 2 && ok; ++s)
            if (act[s]) {
              if (!(ok = tc::mbar_wait(&bars->q_full[s], q_cnt[s] & 1u, abort))) break;
              ++q_cnt[s];
              tc::fence_after_sync();
              issue_S(s, kst);
              tc::mma_commit(&bars->s_full[s]);
            }
          if (!ok) break;
          tc::mma_commit(&bars->kv_empty[kst]);
          bool pv_started = false;  // O of this round already holds a P.V product
          for (int tau = 1; tau <= ntiles && ok; ++tau) {
            const bool prev_pv = tile_kind(x, tau - 1) != kWinStats;
            uint32_t vst = 0;
            if (prev_pv) {
              vst = kv_it % kStages;
              if (!(ok = tc::mbar_wait(&bars->kv_full[vst], (kv_it / kStages) & 1u, abort))) break;
              ++kv_it;
            }
            bool have_k = false;
            // the next K tile before the first slot's P.V, so that S follows P.V without a wait
            if (tau < ntiles) {
              kst = kv_it % kStages;
              if (!(ok = tc::mbar_wait(&bars->kv_full[kst], (kv_it / kStages) & 1u, abort))) break;
              ++kv_it;
              have_k = true;
              tc::fence_after_sync();
            }
            for (int s = 0; s < 2 && ok; ++s) {
              if (!act[s]) continue;
              // p_full: the softmax is done with S_s(tau-1) (and wrote P unless it was a statistics tile)
              if (!(ok = tc::mbar_wait(&bars->p_full[s], p_cnt[s] & 1u, abort))) break;
              ++p_cnt[s];
              if (prev_pv) {
                if (!pv_started) {  // the previous round's epilogue must have read O_s
                  if (!(ok = tc::mbar_wait(&bars->o_empty[s], (o_cnt[s] & 1u) ^ 1u, abort))) break;
                }
                tc::fence_after_sync();
                issue_PV(s, vst, pv_started);
              }
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
            if (prev_pv) {
              pv_started = true;
              tc::mma_commit(&bars->kv_empty[vst]);
            }
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
  } else if (warp >= 4) {
    // ============================================================== softmax / gate epilogue
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
      int nsel = 0, diag = -1;
      // the slot stays held until the unit is done: per-position masks live beside its id
      const int u = tc::queue_peek(&bars->queue, n, abort, ok, &nsel, &diag);
      // warp-uniform outcomes: the warp-collective TMEM accesses must not diverge
      ok = __all_sync(0xffffffffu, ok);
      if (__any_sync(0xffffffffu, u < 0)) break;
      const Unit x = make_unit(p, u, nsel, diag);
      const int ntiles = num_tiles(x);
      for (int r = 0; r < rounds && ok; ++r) {
        const int mt = 2 * r + s;
        if (mt >= MT) continue;
        const int h = x.g * p.G + 2 * mt + (row >> 6);
        const int t = 64 * x.I + (row & 63);
        const bool valid = t < p.N;
        // gate logits: loaded here, used at the branch switch and after the window statistics,
        // so the load latency hides behind the first tiles
        float2 gl = make_float2(-INFINITY, -INFINITY);
        if (valid) gl = *reinterpret_cast<const float2*>(p.gate + (((size_t)x.b * p.Hq + h) * p.N + t) * 2);
        // sink logits (a softmax entry with a zero value per branch), in log2 units
        float2 sk = make_float2(-INFINITY, -INFINITY);
        if (p.sinks != nullptr) {
          sk = *reinterpret_cast<const float2*>(p.sinks + 2 * h);
          sk.x *= kLog2e;
          sk.y *= kLog2e;
        }
        float m_used = -INFINITY, l = 0.0f;   // online state of the sparse branch
        float mw = -INFINITY, lw = 0.0f;      // window branch statistics
        float pw = 0.0f;                      // sigmoid(g1) / l' for the window P.V pass
        for (int tau = 0; tau < ntiles; ++tau) {
          const int kind = tile_kind(x, tau);
          if (!(ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->s_full[s], s_cnt & 1u, abort)))) break;
          ++s_cnt;
          tc::fence_after_sync();
          if (tau == x.n_sp && x.n_sp > 0) {
            // the sparse branch is complete in O (its last P.V finished before this S did):
            // scale O in place to sigmoid(g0) * o~
            const float lt = l + exp2f(sk.x - m_used * sc);   // + the sparse branch's sink
            const float f = lt > 0.0f ? sigmoidf_(gl.x) / lt : 0.0f;
            uint32_t ov[D];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) tc::tmem_ld32(tOrow + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(ov + 32 * c));
            tc::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < D; i += 2) {
              const float2 v = tc::fmul2(make_float2(__uint_as_float(ov[i]), __uint_as_float(ov[i + 1])), make_float2(f, f));
              ov[i] = __float_as_uint(v.x);
              ov[i + 1] = __float_as_uint(v.y);
            }
#pragma unroll
            for (int c = 0; c < D / 32; ++c) tc::tmem_st32(tOrow + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(ov + 32 * c));
            if (TR && valid) {
              uint4* dst = reinterpret_cast<uint4*>(p.osp + (((size_t)x.b * p.Hq + h) * p.N + t) * D);
#pragma unroll
              for (int i = 0; i < D / 8; ++i)
                dst[i] = make_uint4(tc::pack_bf16x2(__uint_as_float(ov[8 * i]), __uint_as_float(ov[8 * i + 1])),
                                    tc::pack_bf16x2(__uint_as_float(ov[8 * i + 2]), __uint_as_float(ov[8 * i + 3])),
                                    tc::pack_bf16x2(__uint_as_float(ov[8 * i + 4]), __uint_as_float(ov[8 * i + 5])),
                                    tc::pack_bf16x2(__uint_as_float(ov[8 * i + 6]), __uint_as_float(ov[8 * i + 7])));
            }
          }
          // visible columns of the two 64-key halves of this tile (empty by default)
          const int wi = kind == kWinStats ? tau - x.n_sp : tau - x.n_sp - x.n_sw;
          int clo[2], chi[2];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            clo[hh] = 64;
            chi[hh] = -1;
            if (kind == kSparse) {
              const int e = 2 * tau + hh;
              bool sel = e < x.nsel;
              if (PR && sel) {   // this position's own blocks among the unit's union
                const uint32_t* rbits = reinterpret_cast<const uint32_t*>(smem + C::kOffRows) +
                                        ((n % tc::kQueueSlots) * 64 + (row & 63)) * kRowWords;
                sel = (rbits[e >> 5] >> (e & 31)) & 1u;
              }
              if (sel) {
                clo[hh] = 0;
                chi[hh] = (e == x.diag) ? t - 64 * x.I : 63;  // only block I crosses the causal line
              }
            } else {
              const int j = x.jw0 + 2 * wi + hh;
              if (j <= x.I) {
                clo[hh] = max(64 * j, t - p.window + 1) - 64 * j;
                chi[hh] = min(t, 64 * j + 63) - 64 * j;
              }
            }
          }
          // S row from TMEM (masked per half)
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
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              if (clo[hh] > 0 || chi[hh] < 63) {
#pragma unroll
                for (int i = 0; i < 64; ++i)
                  if (i < clo[hh] || i > chi[hh]) sv[64 * hh + i] = -INFINITY;
              }
            }
          }
          const float2 sc2 = make_float2(sc, sc);
          // P = exp2(s sc - ms) for the whole row, written to TMEM as bf16 over S; returns the
          // row sum
          auto emit_p = [&](float ms) -> float {
            const float2 nm2 = make_float2(-ms, -ms);
            float2 acc[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float s0 = sv[32 * c + 2 * i], s1 = sv[32 * c + 2 * i + 1];
                const float2 pv = exp2_pair(tc::ffma2(make_float2(s0, s1), sc2, nm2), 16 * c + i);
                acc[i & 1] = tc::fadd2(acc[i & 1], pv);
                pk[i] = tc::pack_bf16x2(pv.x, pv.y);
              }
              tc::tmem_st16(tSrow + 16 * c, pk);
            }
            const float2 a = tc::fadd2(acc[0], acc[1]);
            return a.x + a.y;
          };
          if (kind == kWinPV) {
            // window P.V pass with the final statistics; pw holds the combined exponent offset
            emit_p(pw);
          } else if (kind == kWinStats) {
            // window statistics only: running max and sum, no P, no P.V
            const float mx = fmaxf(tc::max64(sv), tc::max64(sv + 64));
            if (mx > mw) {
              lw = (mw == -INFINITY) ? 0.0f : lw * exp2f((mw - mx) * sc);
              mw = mx;
            }
            const float ms = mw == -INFINITY ? 0.0f : mw * sc;
            const float2 nm2 = make_float2(-ms, -ms);
            float2 acc[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
            for (int i = 0; i < 64; ++i) {
              const float2 xv = tc::ffma2(make_float2(sv[2 * i], sv[2 * i + 1]), sc2, nm2);
              acc[i & 1] = tc::fadd2(acc[i & 1], exp2_pair(xv, i));
            }
            const float2 a = tc::fadd2(acc[0], acc[1]);
            lw += a.x + a.y;
            if (tau == x.n_sp + x.n_sw - 1) {
              // P' = exp2((s - m') sc) * sigmoid(g1) / l' = exp2(s sc - (m' sc - log2(sigmoid(g1) / l')))
              const float lwt = lw + exp2f(sk.y - (mw == -INFINITY ? 0.0f : mw * sc));   // + its sink
              pw = lwt > 0.0f ? sigmoidf_(gl.y) / lwt : 0.0f;
              pw = (mw == -INFINITY ? 0.0f : mw * sc) - __log2f(pw);
            }
          } else {
            // Sparse tile.  The row max is needed first only while the row has none: later
            // tiles compute P with the running max m_used straight away.  While no score
            // exceeds m_used every P is at most 1, so only a tile sum above 2^kRescaleLog2 can
            // hide a P above 2^kRescaleLog2: such a row takes its tile max, redoes the tile
            // with it (rare), and O is rescaled.  Warp-uniform branches only: the TMEM loads
            // and stores are warp-collective.
            if (m_used == -INFINITY) m_used = fmaxf(tc::max64(sv), tc::max64(sv + 64));
            float lt = emit_p(m_used == -INFINITY ? 0.0f : m_used * sc);
            float alpha = 1.0f;
            bool rescale = false;
            if (__any_sync(0xffffffffu, lt > kRescaleSum)) {
              const float mx = fmaxf(tc::max64(sv), tc::max64(sv + 64));
              rescale = lt > kRescaleSum && mx > m_used;
              if (rescale) {
                alpha = exp2f((m_used - mx) * sc);
                m_used = mx;
              }
            }
            if (__any_sync(0xffffffffu, rescale)) {
              lt = emit_p(m_used * sc);   // unchanged rows write the same P again
              if (tau > 0) {
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
          }
          tc::tmem_wait_st();
          tc::fence_before_sync();
          tc::mbar_arrive(&bars->p_full[s]);
        }
        if (!ok) break;
        if (TR && valid) {
          // LSE of each branch in natural-log units of the scaled logits, the sink term included
          // (a branch without keys: the sink alone, or -inf)
          const float a = m_used == -INFINITY ? sk.x : m_used * sc + __log2f(l + exp2f(sk.x - m_used * sc));
          const float c = mw == -INFINITY ? sk.y : mw * sc + __log2f(lw + exp2f(sk.y - mw * sc));
          *reinterpret_cast<float2*>(p.blse + (((size_t)x.b * p.Hq + h) * p.N + t) * 2) =
              make_float2(a * 0.6931471805599453f, c * 0.6931471805599453f);
          if (x.n_sp == 0) {   // no sparse tile: the gated sparse part is zero
            uint4* dst = reinterpret_cast<uint4*>(p.osp + (((size_t)x.b * p.Hq + h) * p.N + t) * D);
#pragma unroll
            for (int i = 0; i < D / 8; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        // ---- epilogue: O already holds sigmoid(g0) o~ + sigmoid(g1) o'
        if (!(ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->o_full[s], o_cnt & 1u, abort)))) break;
        ++o_cnt;
        tc::fence_after_sync();
        __nv_bfloat16* orow = p.o + (((size_t)x.b * p.Hq + h) * p.N + t) * D;
        uint32_t pk[D / 2];
        {
          uint32_t ov[D];
#pragma unroll
          for (int c = 0; c < D / 32; ++c) tc::tmem_ld32(tOrow + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(ov + 32 * c));
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < D / 2; ++i) pk[i] = tc::pack_bf16x2(__uint_as_float(ov[2 * i]), __uint_as_float(ov[2 * i + 1]));
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
}

bool make_map(CUtensorMap* m, const void* base, int D, int rows, int heads) {
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

int num_units(const PrefillDims& d) { return d.B * d.Hkv * d.T; }
int grid_size(const PrefillDims& d) { return num_units(d) < kMaxGrid ? num_units(d) : kMaxGrid; }

template <int D, bool PR, bool TR>
cudaError_t launch_typed(const PrefillDims& d, const void* q, const void* k, const void* v, const int* idx, int kb,
                         const void* ks, const void* vs, int window, const float* gate, const float* sinks,
                         void* o, void* ws, cudaStream_t s, float* blse, void* osp) {
  CUtensorMap mq, mk, mv, mks, mvs;
  if (!make_map(&mq, q, D, d.N, d.B * d.Hq) || !make_map(&mk, k, D, d.N, d.B * d.Hkv) ||
      !make_map(&mv, v, D, d.N, d.B * d.Hkv) || !make_map(&mks, ks, D, d.N, d.B * d.Hkv) ||
      !make_map(&mvs, vs, D, d.N, d.B * d.Hkv))
    return cudaErrorInvalidValue;
  Params p;
  p.B = d.B;
  p.N = d.N;
  p.Hq = d.Hq;
  p.Hkv = d.Hkv;
  p.G = d.G();
  p.T = d.T;
  p.kb = kb;
  p.window = window;
  p.num_units = num_units(d);
  p.idx = idx;
  p.gate = gate;
  p.sinks = sinks;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.o_v8 = (reinterpret_cast<uintptr_t>(o) & 31u) == 0;
  p.blse = blse;
  p.osp = reinterpret_cast<__nv_bfloat16*>(osp);
  p.counter = reinterpret_cast<int*>(ws);
  p.status = device_status_ptr();
  p.scale_log2 = kLog2e / sqrtf((float)D);
  const int smem = PR ? Cfg<D>::kSmemBytes : Cfg<D>::kOffRows + 1024;   // per-position masks only when used
  static int regs = -1;   // the register split assumes exactly kLaunchRegs per thread at launch
  if (regs < 0) {
    cudaFuncAttributes fa;
    cudaError_t e0 = cudaFuncGetAttributes(&fa, sparse_attn_tc_kernel<D, PR, TR>);
    if (e0 != cudaSuccess) return e0;
    regs = fa.numRegs;
  }
  if (regs != kLaunchRegs) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_tc_kernel<D, PR, TR>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(p.counter, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  sparse_attn_tc_kernel<D, PR, TR><<<grid_size(d), kThreads, smem, s>>>(mq, mk, mv, mks, mvs, p);
  return cudaGetLastError();
}

}  // namespace

bool sparse_attn_tc_supported(const PrefillDims& d, hys_dtype dt) {
  return dt == HYS_BF16 && (d.D == 64 || d.D == 128) && d.G() % 2 == 0;
}

size_t sparse_attn_tc_workspace(const PrefillDims&) { return 256; }

bool sparse_attn_rows_tc_supported(const PrefillDims& d, hys_dtype dt) {
  return sparse_attn_tc_supported(d, dt) && d.NB <= 32 * kRowWords;
}

cudaError_t launch_sparse_attn_tc(const PrefillDims& d, const void* q, const void* k, const void* v, const int* idx,
                                  int kb, const void* ks, const void* vs, int window, const float* gate,
                                  const float* sinks, void* o, void* ws, size_t ws_bytes, cudaStream_t s,
                                  bool per_row, float* blse, void* osp) {
  if (ws_bytes < sparse_attn_tc_workspace(d)) return cudaErrorInvalidValue;
  if (per_row && d.NB > 32 * kRowWords) return cudaErrorInvalidValue;
  if (per_row && blse != nullptr) return cudaErrorInvalidValue;   // training outputs: per-tile selection only
  if (per_row)
    return d.D == 64 ? launch_typed<64, true, false>(d, q, k, v, idx, kb, ks, vs, window, gate, sinks, o, ws, s,
                                                     nullptr, nullptr)
                     : launch_typed<128, true, false>(d, q, k, v, idx, kb, ks, vs, window, gate, sinks, o, ws, s,
                                                      nullptr, nullptr);
  if (blse != nullptr)
    return d.D == 64 ? launch_typed<64, false, true>(d, q, k, v, idx, kb, ks, vs, window, gate, sinks, o, ws, s, blse,
                                                     osp)
                     : launch_typed<128, false, true>(d, q, k, v, idx, kb, ks, vs, window, gate, sinks, o, ws, s,
                                                      blse, osp);
  return d.D == 64 ? launch_typed<64, false, false>(d, q, k, v, idx, kb, ks, vs, window, gate, sinks, o, ws, s,
                                                    nullptr, nullptr)
                   : launch_typed<128, false, false>(d, q, k, v, idx, kb, ks, vs, window, gate, sinks, o, ws, s,
                                                     nullptr, nullptr);
}

}  // namespace hys
