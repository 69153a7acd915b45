// Backward of grouped-query attention on the tcgen05 tensor cores (bf16, D = 128, even group
// size), key-major: one work unit is a 128-key tile j of one (batch, KV head) and all query
// M-tiles (two heads of the group x 64 positions) that attend any of its keys.  The same kernel
// serves the three key sets of the hybrid block ([HS] 3.4.1 and 3.4.3, gradients as in the
// training section 3.4.6, where the selection is a constant of the step):
//   kModeFull    causal attention over every earlier key (the full layer);
//   kModeWindow  the sliding window [t - w + 1, t] over the layer's own K', V';
//   kModeSparse  the selected 64-key blocks: a query tile visits the key tile when it selected
//                either of its two blocks (a two-bit mask says which), causal on the diagonal.
//
// Per M-tile (rows t = query positions of two heads, keys i of the tile), with the row's LSE
// from the forward pass, its D_t and a per-row factor sigma_t (the branch gate; 1 for the full
// layer):
//   S^T  = K_j Q_m^T,  dP^T = V_j dO_m^T                          (tcgen05, fp32 in TMEM)
//   P    = exp(tau s - LSE_t) on visible (i, t), 0 elsewhere      (softmax warps, one key row each)
//   dS   = P (sigma_t dP - D_t)
//   dV_j += (sigma P)^T dO_m,  dK_j += dS^T Q_m                   (A operand from TMEM, fp32 in TMEM)
//   dQ_m += dS K_j                                                (A = dS^T in shared memory)
// so that dV = sum_t sigma_t P_ti dO_t, dK = tau sum_t dS_ti q_t and dQ = tau sum_i dS_ti k_i are
// the gradients of o = sigma * softmax(tau q k^T) v with D_t = sigma_t dO_t . o_t.  dK_j and dV_j
// stay in TMEM for the whole unit and are written (or added) once (kModeSparse: a key tile's
// query tiles come in units of at most 16, whose parts are added atomically); every M-tile's dQ part goes
// from TMEM into shared memory over the M-tile's own Q and dO stage (free once its MMAs have read
// them), and a reduce warp sends it to an fp32 accumulator in global memory with TMA reduce-adds
// while the next M-tile runs; the stage goes back to the producer once the reduce has read it.
// dQ is scaled by tau and rounded to the output type afterwards.
//
// Warp roles (384 threads): warp 0 TMA producer (K_j, V_j once per unit; Q and dO of every
// M-tile, two stages), warp 1 MMA issuer (and TMEM owner), warp 2 dQ reducer, warps 4-7 and 8-11 two softmax and
// drain groups (thread = key row r of the tile = TMEM lane; each group takes half of the row's
// query columns, and half of the head-dim columns in the drains).  TMEM: tS (S^T, then sigma P^T as bf16), tP (dP^T, then
// dS^T as bf16, then the M-tile's dQ part), tdV, tdK: 4 x 128 columns.  The MMA order per M-tile
// is dV, dK, dQ (into tP), then S^T of the next M-tile into tS, then its dP^T once the dQ part
// has been read out of tP.
// Every mbarrier wait is bounded; a timeout records HYS_ERR_TIMEOUT, waits (bounded) for the
// copies and MMAs already issued and frees TMEM.
#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace hys {
namespace {

constexpr int kThreads = 384;   // warp 0 TMA, warp 1 MMA, warps 4-7 / 8-11 softmax groups
constexpr int kD = 128;
constexpr int kMaxGrid = 148;
#ifndef HYS_BWD_SPARSE_CHUNK
#define HYS_BWD_SPARSE_CHUNK 16
#endif
constexpr int kSparseChunk = HYS_BWD_SPARSE_CHUNK;   // query tiles per selected-block unit
constexpr int kTile = 128 * kD * 2;  // 128 rows x 128 bf16: two 64-column swizzled chunks of 16 KB
constexpr int kModeFull = 0, kModeWindow = 1, kModeSparse = 2;

// instruction descriptor of kind::f16 (bf16 A and B, fp32 D) with both major-ness bits
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

struct Params {
  int B, N, Hq, Hkv, G, MT, NK, T, num_units, window;
  int chunk;           // kModeSparse: query tiles per unit (a key tile's list is cut into pieces)
  const float* lse2;   // [B,Hq,N] row LSE in log2 units (includes any sink term)
  const float* dsum;   // [B,Hq,N] D_t of this key set
  const float* sig;    // [B,Hq,N] per-row factor sigma_t, or null (1)
  float* dq;           // [B,Hq,N,128] fp32 accumulator (red.add), unscaled
  float* dk;           // [B,Hkv,N,128] fp32
  float* dv;
  int accumulate;      // add dK, dV to the outputs instead of overwriting them
  const int* list;     // kModeSparse: per (b, g, j) T entries (i << 2 | mask) ...
  const int* list_cnt; // ... and their count
  int* counter;
  int* status;
  float sc;            // log2(e) / sqrt(D)
  float tau;           // 1 / sqrt(D)
};

struct Bars {
  uint64_t kv_full, kv_empty, q_full[2], q_red[2], s_full, p_full, dq_full, s_free, ds_free, acc_full, acc_free;
  uint64_t mma_drain, rows_ready[2];
  uint64_t dq_staged;   // an M-tile's dQ part is in its Q / dO stage (both groups)
};

constexpr int kOffK = 0, kOffV = kTile, kOffQ = 2 * kTile, kOffDO = 4 * kTile, kOffDS = 6 * kTile;
constexpr int kOffRow = 7 * kTile;                     // lse2, dsum, sig of the M-tile's 128 rows
constexpr int kOffBar = kOffRow + 3 * 128 * 4;
constexpr int kOffMisc = kOffBar + (int)((sizeof(Bars) + 15) / 16 * 16);
constexpr int kSmemBytes = kOffMisc + 64 + 1024;       // + alignment of the dynamic base to 1 KB
static_assert(kSmemBytes <= 232448, "shared memory of one CTA");

__device__ __forceinline__ void fail(volatile int* abort, int* status) {
  *abort = 1;
  report_status(status, HYS_ERR_TIMEOUT);
}


// four fp32 atomic adds in one vector reduction (relaxed, device scope)
__device__ __forceinline__ void red_add_v4(float4* dst, float4 x) {
  asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(x.x), "f"(x.y), "f"(x.z),
               "f"(x.w)
               : "memory");
}

// unit u -> (b, g, j), key tiles in increasing j across all (b, g) first: small j has the most
// query tiles in the full mode, so the longest units start first.  In the selected-block mode a
// key tile's query tiles come in pieces of at most p.chunk (piece `sub`, pieces outermost):
// how often a block is selected varies a lot, and one popular key tile as a single unit would
// outlast the rest of the launch.
template <int MODE>
__device__ __forceinline__ void unit_coords(const Params& p, int u, int& b, int& g, int& j, int& lu, int& sub) {
  const int per = p.B * p.Hkv * p.NK;
  sub = MODE == kModeSparse ? u / per : 0;
  const int v = MODE == kModeSparse ? u % per : u;
  const int bg = v % (p.B * p.Hkv);
  j = v / (p.B * p.Hkv);
  b = bg / p.Hkv;
  g = bg % p.Hkv;
  lu = bg * p.NK + j;
}

template <int MODE>
__device__ __forceinline__ int num_qtiles(const Params& p, int j, int lu, int sub) {
  if (MODE == kModeFull) return p.T - 2 * j;
  if (MODE == kModeWindow) {
    const int hi = min(p.T - 1, (128 * j + 127 + p.window - 1) / 64);
    return hi - 2 * j + 1;
  }
  return min(p.chunk, p.list_cnt[lu] - sub * p.chunk);
}

// query tile and key-half mask of the unit's M-tile m.  The query tiles run from the last one
// down: the units running at the same time then reach the same query tiles (and the same dQ
// accumulator rows) together, so the accumulator's reduce-adds mostly hit L2.
template <int MODE>
__device__ __forceinline__ void mtile(const Params& p, int j, int lu, int sub, int m, int nmt, int& i, int& hp,
                                      int& mask) {
  const int n = (nmt - 1 - m) / p.MT;
  hp = m % p.MT;
  if (MODE == kModeSparse) {
    const int e = p.list[(size_t)lu * p.T + sub * p.chunk + n];
    i = e >> 2;
    mask = e & 3;
  } else {
    i = 2 * j + n;
    mask = 3;
  }
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                       const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmDQ, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 16);
  int* s_unit = reinterpret_cast<int*>(smem + kOffMisc + 32);
  float* s_lse = reinterpret_cast<float*>(smem + kOffRow);
  float* s_dsum = s_lse + 128;
  float* s_sig = s_lse + 256;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    tc::mbar_init(&bars->kv_full, 1);
    tc::mbar_init(&bars->kv_empty, 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&bars->q_full[s], 1);
      tc::mbar_init(&bars->q_red[s], 1);   // the stage's dQ part has been read by the TMA reduce
    }
    tc::mbar_init(&bars->s_full, 1);
    tc::mbar_init(&bars->p_full, 256);
    tc::mbar_init(&bars->dq_full, 1);
    tc::mbar_init(&bars->s_free, 256);
    tc::mbar_init(&bars->ds_free, 1);
    tc::mbar_init(&bars->acc_full, 1);
    tc::mbar_init(&bars->acc_free, 256);
    tc::mbar_init(&bars->mma_drain, 1);
    tc::mbar_init(&bars->rows_ready[0], 128);
    tc::mbar_init(&bars->rows_ready[1], 128);
    tc::mbar_init(&bars->dq_staged, 256);
    *abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tensormap(&tmQ);
    tc::prefetch_tensormap(&tmDO);
    tc::prefetch_tensormap(&tmK);
    tc::prefetch_tensormap(&tmV);
    tc::prefetch_tensormap(&tmDQ);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, 512);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tS = tmem_base, tP = tmem_base + 128, tdV = tmem_base + 256, tdK = tmem_base + 384;

  // Every role walks the same unit sequence (one thread claims, all read it back).  Barriers that
  // complete once per unit take their parity from nu (units processed), the per-M-tile ones from
  // mc (M-tiles processed before this unit); units without M-tiles are skipped by every role.
  uint32_t mc = 0, nu = 0, q_issued = 0;
  for (;;) {
    if (threadIdx.x == 0) *s_unit = atomicAdd(p.counter, 1);
    __syncthreads();
    const int u = *s_unit;
    const bool stop = u >= p.num_units || *abort;
    __syncthreads();
    if (stop) break;
    int b, g, j, lu, sub;
    unit_coords<MODE>(p, u, b, g, j, lu, sub);
    const int nmt = num_qtiles<MODE>(p, j, lu, sub) * p.MT;
    if (nmt <= 0) continue;
    const uint32_t par = nu & 1u;

    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        bool ok = tc::mbar_wait(&bars->kv_empty, par ^ 1u, abort);
        const bool kv_issued = ok;
        if (ok) {
          tc::mbar_arrive_expect_tx(&bars->kv_full, 2 * kTile);
          for (int ch = 0; ch < 2; ++ch) {
            tc::tma_load_3d(&tmK, &bars->kv_full, smem + kOffK + ch * 16384, ch * 64, 128 * j, b * p.Hkv + g);
            tc::tma_load_3d(&tmV, &bars->kv_full, smem + kOffV + ch * 16384, ch * 64, 128 * j, b * p.Hkv + g);
          }
        }
        for (int m = 0; m < nmt && ok; ++m) {
          const uint32_t n = mc + m, st = n & 1u;
          int i, hp, mask;
          mtile<MODE>(p, j, lu, sub, m, nmt, i, hp, mask);
          // the stage is free once M-tile n - 2's MMAs and the TMA reduce of its dQ part (staged over
          // its Q and dO) have read it
          if (!(ok = tc::mbar_wait(&bars->q_red[st], ((n >> 1) & 1u) ^ 1u, abort))) break;
          tc::mbar_arrive_expect_tx(&bars->q_full[st], 2 * kTile);
          for (int hh = 0; hh < 2; ++hh)
            for (int ch = 0; ch < 2; ++ch) {
              const int head = b * p.Hq + g * p.G + 2 * hp + hh;
              const int off = st * kTile + ch * 16384 + hh * 8192;
              tc::tma_load_3d(&tmQ, &bars->q_full[st], smem + kOffQ + off, ch * 64, 64 * i, head);
              tc::tma_load_3d(&tmDO, &bars->q_full[st], smem + kOffDO + off, ch * 64, 64 * i, head);
            }
          q_issued = n + 1;
        }
        if (!ok) {
          fail(abort, p.status);
          // the copies already issued land before the kernel leaves
          if (kv_issued) tc::mbar_wait_drain(&bars->kv_full, par);
          if (q_issued > 0) {
            const uint32_t n = q_issued - 1;
            tc::mbar_wait_drain(&bars->q_full[n & 1u], (n >> 1) & 1u);
          }
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        const uint32_t idS = idesc_bf16(128, 128, false, false);  // K-major A and B
        const uint32_t idAcc = idesc_bf16(128, kD, false, true);  // A in TMEM, B MN-major
        const uint32_t idQ = idesc_bf16(128, kD, true, true);     // A and B MN-major
        const uint32_t kb = tc::smem_u32(smem + kOffK), vb = tc::smem_u32(smem + kOffV);
        const uint32_t dsb = tc::smem_u32(smem + kOffDS);
        auto issue_s = [&](uint32_t st) {   // S^T = K Q^T into tS
          const uint32_t qb = tc::smem_u32(smem + kOffQ + st * kTile);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            tc::mma_ss(tS, tc::sdesc_sw128(kb + off, 16, 1024), tc::sdesc_sw128(qb + off, 16, 1024), idS, kk > 0);
          }
        };
        auto issue_dp = [&](uint32_t st) {   // dP^T = V dO^T into tP
          const uint32_t dob = tc::smem_u32(smem + kOffDO + st * kTile);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            tc::mma_ss(tP, tc::sdesc_sw128(vb + off, 16, 1024), tc::sdesc_sw128(dob + off, 16, 1024), idS, kk > 0);
          }
        };
        bool ok = tc::mbar_wait(&bars->kv_full, par, abort);
        // M-tile 0: S^T and dP^T (tS and tP were released by the previous unit's last drain)
        if (ok) ok = tc::mbar_wait(&bars->q_full[mc & 1u], (mc >> 1) & 1u, abort);
        if (ok && mc > 0) ok = tc::mbar_wait(&bars->s_free, (mc - 1) & 1u, abort);
        if (ok) {
          tc::fence_after_sync();
          issue_s(mc & 1u);
          issue_dp(mc & 1u);
          tc::mma_commit(&bars->s_full);
        }
        for (int m = 0; m < nmt && ok; ++m) {
          const uint32_t n = mc + m, st = n & 1u;
          if (!(ok = tc::mbar_wait(&bars->p_full, n & 1u, abort))) break;
          // the previous unit's dK / dV must be drained before this unit's first update
          if (m == 0 && nu > 0 && !(ok = tc::mbar_wait(&bars->acc_free, par ^ 1u, abort))) break;
          tc::fence_after_sync();
          const uint32_t qb = tc::smem_u32(smem + kOffQ + st * kTile);
          const uint32_t dob = tc::smem_u32(smem + kOffDO + st * kTile);
          // A operands in TMEM: query rows 0-63 packed at columns 0-31, rows 64-127 at 64-95
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)   // dV += (sigma P)^T dO : K = 128 query rows, 16 per step
            tc::mma_ts(tdV, tS + kk * 8 + (kk >= 4 ? 32 : 0), tc::sdesc_sw128(dob + kk * 2048, 16384, 1024), idAcc,
                       (m > 0 || kk > 0));
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)   // dK += dS^T Q
            tc::mma_ts(tdK, tP + kk * 8 + (kk >= 4 ? 32 : 0), tc::sdesc_sw128(qb + kk * 2048, 16384, 1024), idAcc,
                       (m > 0 || kk > 0));
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)   // dQ part = dS K_j : K = 128 keys, 16 per step, into tP
            tc::mma_ss(tP, tc::sdesc_sw128(dsb + kk * 2048, 16384, 1024), tc::sdesc_sw128(kb + kk * 2048, 16384, 1024),
                       idQ, kk > 0);
          tc::mma_commit(&bars->ds_free);
          tc::mma_commit(&bars->dq_full);
          if (m + 1 < nmt) {
            const uint32_t n1 = n + 1, st1 = n1 & 1u;
            if (!(ok = tc::mbar_wait(&bars->q_full[st1], (n1 >> 1) & 1u, abort))) break;
            tc::fence_after_sync();
            issue_s(st1);                                             // overlaps the dQ drain
            if (!(ok = tc::mbar_wait(&bars->s_free, n & 1u, abort))) break;   // dQ part read from tP
            tc::fence_after_sync();
            issue_dp(st1);
            tc::mma_commit(&bars->s_full);
          }
        }
        if (ok) {
          tc::mma_commit(&bars->acc_full);
          tc::mma_commit(&bars->kv_empty);
        } else {
          fail(abort, p.status);
        }
        // every MMA of the unit has completed before the next unit (or the TMEM release)
        tc::mma_commit(&bars->mma_drain);
        tc::mbar_wait_drain(&bars->mma_drain, nu & 1u);
      }
    } else if (warp == 2) {
      // ------------------------------------------------------------ dQ reducer
      // every M-tile's staged dQ part (two 64-row boxes per 32-column chunk) into the fp32
      // accumulator with TMA reduce-adds; the stage goes back to the producer once read
      if (lane == 0) {
        bool ok = true;
        for (int m = 0; m < nmt && ok; ++m) {
          const uint32_t n = mc + m, st = n & 1u;
          int i, hp, mask;
          mtile<MODE>(p, j, lu, sub, m, nmt, i, hp, mask);
          if (!(ok = tc::mbar_wait(&bars->dq_staged, n & 1u, abort))) break;
          const int head0 = b * p.Hq + g * p.G + 2 * hp;
          for (int c = 0; c < 4; ++c) {
            const uint8_t* stg = smem + (c < 2 ? kOffQ : kOffDO) + st * kTile + (c & 1) * 16384;
            tc::tma_reduce_add_3d(&tmDQ, stg, 32 * c, 64 * i, head0);
            tc::tma_reduce_add_3d(&tmDQ, stg + 8192, 32 * c, 64 * i, head0 + 1);
          }
          tc::bulk_commit_group();
          tc::bulk_wait_group_read0();
          tc::mbar_arrive(&bars->q_red[st]);
        }
        if (!ok) fail(abort, p.status);
      }
    } else if (warp >= 4) {
      // ------------------------------------------------------------ softmax / drains
      // Two groups share every M-tile: group wg takes the query columns (and, in the drains, the
      // head-dim columns) [64 wg, 64 wg + 64) of the thread's TMEM lane.
      const int wg = (warp - 4) >> 2;
      const int r = 32 * (warp & 3) + lane;              // TMEM lane: key row, later query row
      const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
      const int kp = 128 * j + r;                        // this thread's key position
      bool ok = true;
      // the statistics of this group's 64 query rows of an M-tile (head 2hp + wg, positions 64i ..),
      // loaded one M-tile ahead so that their latency overlaps the previous M-tile
      float nl = INFINITY, nd = 0.0f, ns = 1.0f;
      auto load_rows = [&](int m) {
        int i, hp, mask;
        mtile<MODE>(p, j, lu, sub, m, nmt, i, hp, mask);
        const int head = b * p.Hq + g * p.G + 2 * hp + wg;
        const int pos = 64 * i + (r & 63);
        const size_t rix = (size_t)head * p.N + pos;
        nl = pos < p.N ? p.lse2[rix] : INFINITY;
        nd = pos < p.N ? p.dsum[rix] : 0.0f;
        ns = (pos < p.N && p.sig != nullptr) ? p.sig[rix] : 1.0f;
      };
      if (r < 64) load_rows(0);
      for (int m = 0; m < nmt && ok; ++m) {
        const uint32_t n = mc + m;
        int i, hp, mask;
        mtile<MODE>(p, j, lu, sub, m, nmt, i, hp, mask);
        if (r < 64) {
          const int q = 64 * wg + r;
          s_lse[q] = nl;
          s_dsum[q] = nd;
          s_sig[q] = ns;
          if (m + 1 < nmt) load_rows(m + 1);
        }
        // the group's rows written (a bounded wait: a warp that left on a failed wait cannot block
        // the others); the previous M-tile's values were read by every thread before its p_full
        // arrival, which the previous dq_full wait covered
        tc::mbar_arrive(&bars->rows_ready[wg]);
        if (!(ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->rows_ready[wg], n & 1u, abort)))) break;
        if (!(ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->s_full, n & 1u, abort)))) break;
        if (n > 0 && !(ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->ds_free, (n - 1) & 1u, abort)))) break;
        tc::fence_after_sync();
        // visibility of this key row: valid key, selected half (sparse), then per query column
        // the causal line (and the window's lower edge)
        const bool row_on = kp < p.N && (MODE != kModeSparse || ((mask >> (r >> 6)) & 1));
        // warp-uniform cases: every pair of the warp's rows visible (a key tile wholly before the
        // query tile, full and selected-block modes), or no visible pair (a key row past N or a
        // half the query tile did not select): the per-column tests and the exponentials go
        const int vis_mode = __all_sync(0xffffffffu, row_on && MODE != kModeWindow && 128 * j + 127 <= 64 * i) ? 1
                             : (__all_sync(0xffffffffu, !row_on) ? 2 : 0);
#pragma unroll 1
        for (int c = 2 * wg; c < 2 * wg + 2; ++c) {        // 32 query columns per chunk
          uint32_t sr[32], dr[32];
          tc::tmem_ld32(tS + 32 * c + lane_off, sr);
          tc::tmem_ld32(tP + 32 * c + lane_off, dr);
          tc::tmem_wait_ld();
          uint32_t pk[16], dk2[16];
          // P and dS for four query columns at a time (the row statistics as float4); ALL: every
          // pair visible
          auto pairs = [&](auto all_tag) {
            constexpr bool ALL = decltype(all_tag)::value;
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {
              const int q4 = 32 * c + 4 * e4;
              // (the full layer has no per-row factor: sigma = 1)
              const float4 l4 = *reinterpret_cast<const float4*>(s_lse + q4);
              const float4 g4 = MODE == kModeFull ? make_float4(1.0f, 1.0f, 1.0f, 1.0f)
                                                  : *reinterpret_cast<const float4*>(s_sig + q4);
              const float4 d4 = *reinterpret_cast<const float4*>(s_dsum + q4);
              const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, gv[4] = {g4.x, g4.y, g4.z, g4.w},
                          dsv[4] = {d4.x, d4.y, d4.z, d4.w};
              float pv[4], dv[4];
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                float pe;
                if (ALL) {
                  pe = exp2f(fmaf(__uint_as_float(sr[4 * e4 + h]), p.sc, -lv[h]));
                } else {
                  const int qpos = 64 * i + ((q4 + h) & 63);
                  bool vis = row_on && kp <= qpos;
                  if (MODE == kModeWindow) vis = vis && kp > qpos - p.window;
                  pe = vis ? exp2f(fmaf(__uint_as_float(sr[4 * e4 + h]), p.sc, -lv[h])) : 0.0f;
                }
                pv[h] = pe * gv[h];
                dv[h] = pe * fmaf(gv[h], __uint_as_float(dr[4 * e4 + h]), -dsv[h]);
              }
              pk[2 * e4] = tc::pack_bf16x2(pv[0], pv[1]);
              pk[2 * e4 + 1] = tc::pack_bf16x2(pv[2], pv[3]);
              dk2[2 * e4] = tc::pack_bf16x2(dv[0], dv[1]);
              dk2[2 * e4 + 1] = tc::pack_bf16x2(dv[2], dv[3]);
            }
          };
          if (vis_mode == 1) {
            pairs(std::true_type{});
          } else if (vis_mode == 2) {
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = dk2[e] = 0u;
          } else {
            pairs(std::false_type{});
          }
          // packed bf16 pairs over this group's own fp32 columns, behind its reads (the other group
          // is still reading its half): group wg's 32 packed columns start at column 64 wg
          tc::tmem_st16(tS + 64 * wg + 16 * (c - 2 * wg) + lane_off, pk);
          tc::tmem_st16(tP + 64 * wg + 16 * (c - 2 * wg) + lane_off, dk2);
          // dS^T into shared memory (the dQ MMA's MN-major A): 16-byte units of 8 query columns,
          // 128-byte swizzle by key row
#pragma unroll
          for (int uu = 0; uu < 4; ++uu) {
            const int q0 = 32 * c + 8 * uu;
            const int chunk = q0 >> 6, unit = (q0 & 63) >> 3;
            uint4* dst = reinterpret_cast<uint4*>(smem + kOffDS + chunk * 16384 + r * 128 + ((unit ^ (r & 7)) << 4));
            *dst = make_uint4(dk2[4 * uu], dk2[4 * uu + 1], dk2[4 * uu + 2], dk2[4 * uu + 3]);
          }
        }
        tc::tmem_wait_st();
        tc::fence_proxy_async_shared();   // dS^T shared-memory writes -> the MMA (async proxy)
        tc::fence_before_sync();
        tc::mbar_arrive(&bars->p_full);
        // dQ part (TMEM lane r of tP = query row r, 128 fp32 columns): the group's two 32-column
        // chunks are read out of TMEM (tP is free for the next dP^T from there on) and staged
        // over this M-tile's Q stage (group 0) or dO stage (group 1), which its MMAs have finished
        // reading; the reduce warp sends them to the fp32 accumulator while the next M-tile runs
        if (!(ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->dq_full, n & 1u, abort)))) break;
        tc::fence_after_sync();
        {
          uint32_t v0[32], v1[32];
          tc::tmem_ld32(tP + 64 * wg + lane_off, v0);
          tc::tmem_ld32(tP + 64 * wg + 32 + lane_off, v1);
          tc::tmem_wait_ld();
          tc::fence_before_sync();
          tc::mbar_arrive(&bars->s_free);
          uint8_t* stg = smem + (wg == 0 ? kOffQ : kOffDO) + (n & 1u) * kTile;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int o = r * 128 + ((u ^ (r & 7)) << 4);
            *reinterpret_cast<uint4*>(stg + o) = make_uint4(v0[4 * u], v0[4 * u + 1], v0[4 * u + 2], v0[4 * u + 3]);
            *reinterpret_cast<uint4*>(stg + 16384 + o) =
                make_uint4(v1[4 * u], v1[4 * u + 1], v1[4 * u + 2], v1[4 * u + 3]);
          }
          tc::fence_proxy_async_shared();   // generic shared-memory writes -> the TMA (async proxy)
          tc::mbar_arrive(&bars->dq_staged);
        }
      }
      // unit epilogue: dK (scaled by tau) and dV of key row r, written or added once
      if (ok && (ok = __all_sync(0xffffffffu, tc::mbar_wait(&bars->acc_full, par, abort)))) {
        tc::fence_after_sync();
        for (int t2 = 0; t2 < 2; ++t2) {
          const uint32_t tsrc = t2 ? tdV : tdK;
          float* dst = (t2 ? p.dv : p.dk) + (((size_t)b * p.Hkv + g) * p.N + kp) * kD;
          const float f = t2 ? 1.0f : p.tau;
#pragma unroll 1
          for (int c = 2 * wg; c < 2 * wg + 2; ++c) {
            uint32_t v[32];
            tc::tmem_ld32(tsrc + 32 * c + lane_off, v);
            tc::tmem_wait_ld();
            if (kp < p.N) {
              float4* d4 = reinterpret_cast<float4*>(dst + 32 * c);
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                float4 x = make_float4(__uint_as_float(v[4 * e]) * f, __uint_as_float(v[4 * e + 1]) * f,
                                       __uint_as_float(v[4 * e + 2]) * f, __uint_as_float(v[4 * e + 3]) * f);
                if (MODE == kModeSparse) {   // pieces of one key tile may run at the same time
                  red_add_v4(d4 + e, x);
                  continue;
                }
                if (p.accumulate) {
                  const float4 y = d4[e];
                  x.x += y.x;
                  x.y += y.y;
                  x.z += y.z;
                  x.w += y.w;
                }
                d4[e] = x;
              }
            }
          }
        }
        tc::fence_before_sync();
        tc::mbar_arrive(&bars->acc_free);
      }
      if (!ok) fail(abort, p.status);
    }
    mc += (uint32_t)nmt;
    ++nu;
    __syncthreads();   // every role finished the unit (a failed wait set abort)
  }

  if (warp == 2 && lane == 0) tc::bulk_wait_group0();   // the dQ reductions have landed
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem_base, 512);
  }
}

// ------------------------------------------------------------------------------ helpers
// Per row of the full layer: lse2 = LSE * log2(e) and D_t = dO_t . o_t (one warp per row).
__global__ void bwd_rows_full_kernel(const float* __restrict__ lse, const __nv_bfloat16* __restrict__ o,
                                     const __nv_bfloat16* __restrict__ d_o, float* __restrict__ lse2,
                                     float* __restrict__ dsum, long long rows) {
  const long long r = (long long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const uint2 a = reinterpret_cast<const uint2*>(o + r * kD)[lane];
  const uint2 c = reinterpret_cast<const uint2*>(d_o + r * kD)[lane];
  const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
  const __nv_bfloat162* c2 = reinterpret_cast<const __nv_bfloat162*>(&c);
  float acc = 0.0f;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const float2 x = __bfloat1622float2(a2[e]), y = __bfloat1622float2(c2[e]);
    acc = fmaf(x.x, y.x, fmaf(x.y, y.y, acc));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    dsum[r] = acc;
    lse2[r] = lse[r] * kLog2e;
  }
}

// out (bf16) = tau * acc (fp32), 8 elements per thread
__global__ void bwd_dq_out_kernel(const float4* __restrict__ acc, uint4* __restrict__ out, float tau, long long n8) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = acc[2 * i], b = acc[2 * i + 1];
  out[i] = make_uint4(tc::pack_bf16x2(a.x * tau, a.y * tau), tc::pack_bf16x2(a.z * tau, a.w * tau),
                      tc::pack_bf16x2(b.x * tau, b.y * tau), tc::pack_bf16x2(b.z * tau, b.w * tau));
}

// [heads][rows][128] bf16, box = 64 columns x box_rows rows x 1 head, 128-byte swizzle
bool make_map(CUtensorMap* m, const void* base, int rows, int heads, int box_rows) {
  EncodeTiledFn fn = tma_encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)rows, (cuuint64_t)heads};
  cuuint64_t strides[2] = {256, (cuuint64_t)rows * 256};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [heads][rows][128] fp32 (the dQ accumulator), box = 32 columns x 64 rows x 1 head, 128-byte
// swizzle: the target of the TMA reduce-adds
bool make_map_f32(CUtensorMap* m, const void* base, int rows, int heads) {
  EncodeTiledFn fn = tma_encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)rows, (cuuint64_t)heads};
  cuuint64_t strides[2] = {512, (cuuint64_t)rows * 512};
  cuuint32_t box[3] = {32, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE>
cudaError_t launch_mode(const PrefillDims& d, const void* q, const void* d_o, const void* k, const void* v,
                        const float* lse2, const float* dsum, const float* sig, float* dq_acc, float* dk, float* dv,
                        int accumulate, int window, const int* list, const int* list_cnt, int* counter,
                        cudaStream_t s) {
  CUtensorMap mq, mdo, mk, mv, mdq;
  if (!make_map(&mq, q, d.N, d.B * d.Hq, 64) || !make_map(&mdo, d_o, d.N, d.B * d.Hq, 64) ||
      !make_map(&mk, k, d.N, d.B * d.Hkv, 128) || !make_map(&mv, v, d.N, d.B * d.Hkv, 128) ||
      !make_map_f32(&mdq, dq_acc, d.N, d.B * d.Hq))
    return cudaErrorInvalidValue;
  Params p;
  p.B = d.B;
  p.N = d.N;
  p.Hq = d.Hq;
  p.Hkv = d.Hkv;
  p.G = d.G();
  p.MT = p.G / 2;
  p.NK = (d.N + 127) / 128;
  p.T = d.T;
  p.chunk = kSparseChunk;
  p.num_units = d.B * d.Hkv * p.NK * (MODE == kModeSparse ? (d.T + kSparseChunk - 1) / kSparseChunk : 1);
  p.window = window;
  p.lse2 = lse2;
  p.dsum = dsum;
  p.sig = sig;
  p.dq = dq_acc;
  p.dk = dk;
  p.dv = dv;
  p.accumulate = accumulate;
  p.list = list;
  p.list_cnt = list_cnt;
  p.counter = counter;
  p.status = device_status_ptr();
  p.sc = kLog2e / sqrtf((float)kD);
  p.tau = 1.0f / sqrtf((float)kD);
  cudaError_t e = cudaMemsetAsync(counter, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_bwd_tc_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const int grid = p.num_units < kMaxGrid ? p.num_units : kMaxGrid;
  attn_bwd_tc_kernel<MODE><<<grid, kThreads, kSmemBytes, s>>>(mq, mdo, mk, mv, mdq, p);
  return cudaGetLastError();
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

bool attn_bwd_tc_supported(const PrefillDims& d, hys_dtype dt) {
  return dt == HYS_BF16 && d.D == kD && d.G() % 2 == 0 && d.G() <= 64;
}

// workspace: [256: unit counter][lse2 rows][dsum rows][dq accumulator rows x 128] (fp32)
size_t full_bwd_tc_workspace(const PrefillDims& d) {
  const size_t rows = (size_t)d.B * d.Hq * d.N;
  return 256 + 2 * align256(rows * 4) + rows * kD * 4;
}

cudaError_t launch_full_bwd_tc(const PrefillDims& d, const void* q, const void* k, const void* v, const void* o,
                               const void* d_o, const float* lse, void* dq, float* dk, float* dv, int accumulate,
                               void* ws, cudaStream_t s) {
  const size_t rows = (size_t)d.B * d.Hq * d.N;
  uint8_t* w = reinterpret_cast<uint8_t*>(ws);
  int* counter = reinterpret_cast<int*>(w);
  float* lse2 = reinterpret_cast<float*>(w + 256);
  float* dsum = reinterpret_cast<float*>(w + 256 + align256(rows * 4));
  float* acc = reinterpret_cast<float*>(w + 256 + 2 * align256(rows * 4));
  cudaError_t e = cudaMemsetAsync(acc, 0, rows * kD * 4, s);
  if (e != cudaSuccess) return e;
  bwd_rows_full_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(
      lse, reinterpret_cast<const __nv_bfloat16*>(o), reinterpret_cast<const __nv_bfloat16*>(d_o), lse2, dsum,
      (long long)rows);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_mode<kModeFull>(d, q, d_o, k, v, lse2, dsum, nullptr, acc, dk, dv, accumulate, 0, nullptr, nullptr,
                             counter, s);
  if (e != cudaSuccess) return e;
  return launch_bwd_dq_out(acc, dq, rows * kD, s);
}

cudaError_t launch_bwd_dq_out(const float* acc, void* dq, size_t n, cudaStream_t s) {
  const long long n8 = (long long)(n / 8);
  bwd_dq_out_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, s>>>(reinterpret_cast<const float4*>(acc),
                                                                  reinterpret_cast<uint4*>(dq),
                                                                  1.0f / sqrtf((float)kD), n8);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_tc_window(const PrefillDims& d, const void* q, const void* d_o, const void* k,
                                      const void* v, const float* lse2, const float* dsum, const float* sig,
                                      float* dq_acc, float* dk, float* dv, int window, int* counter, cudaStream_t s) {
  return launch_mode<kModeWindow>(d, q, d_o, k, v, lse2, dsum, sig, dq_acc, dk, dv, 0, window, nullptr, nullptr,
                                  counter, s);
}

cudaError_t launch_attn_bwd_tc_sparse(const PrefillDims& d, const void* q, const void* d_o, const void* k,
                                      const void* v, const float* lse2, const float* dsum, const float* sig,
                                      float* dq_acc, float* dk, float* dv, const int* list, const int* list_cnt,
                                      int* counter, cudaStream_t s) {
  return launch_mode<kModeSparse>(d, q, d_o, k, v, lse2, dsum, sig, dq_acc, dk, dv, 1, 0, list, list_cnt, counter,
                                  s);
}

}  // namespace hys
