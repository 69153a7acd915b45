// Single-token decode, bf16: split-KV kernels that stream the cache at HBM speed.
// (HySparse2 explainer, "Twenty lines of algorithmic intuition": scores of the new query
// against the cache, top-k of the old blocks, then the sparse followers; HySparse 3.4.1
// block scores and 3.4.3 sparse/SWA/gate for one query row.)
//
// One CTA = (split, KV group g, sequence b): C consumer warps + 1 TMA producer warp (C = 3,
// so two CTAs share an SM and one's start-up and drain overlap the other's streaming).  The
// producer streams 64-key blocks of K and V (two 128-byte-swizzled TMA boxes each per
// tensor, 32 KB per block) into C stages; consumer warp w owns stage w and takes blocks
// w, w+C, ... of the split, so every stage's barrier phases are consumed by one warp in
// order (a parity wait cannot be fooled by a phase two ahead) and the max logit of a
// block (HySparse's m~) is a warp-local reduction.  A sparse layer's split holds 32 of the
// selected blocks; its SWA ring is a split of its own.  A token-sparse layer's split holds up
// to 2048 selected tokens, copied row by row with cp.async into the same stage layout, and the
// forced newest tokens are a split of contiguous boxes.
// The G <= 16 query heads of the group form the 16 rows of mma.sync.m16n8k16 tiles
// (zero-padded): S = Q K^T (64 mma per block), online softmax in registers, O += P V (64
// mma per block).  The warps' partial (m, l, O) are merged in shared memory (reusing the stages) and the
// split's partial goes to the workspace; a combine kernel merges the splits, writes o and
// (full layer) the block scores exp(m~ - m)/l aggregated over the group's heads, or
// (sparse layer) the gated sum of the sparse-branch and SWA-ring branches.  In the token
// variant the full layer also writes every key's logit and a wide kernel turns them into the
// token scores.  An FP8 (E4M3) cache runs in its own instance: 16 KB blocks, six stages
// (warp w owns stages w and w + C), codes converted to f16 inside the MMA fragments.
#include <cuda.h>
#include <cuda_fp16.h>
#include <math.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "tma_host.h"
#include "tc_ptx.cuh"

namespace hys {

namespace {

#ifndef HYS_DECODE_CONSUMERS
#define HYS_DECODE_CONSUMERS 3
#endif
constexpr int kConsumers = HYS_DECODE_CONSUMERS;
constexpr int kCtasPerSm = kConsumers <= 3 ? 2 : 1;   // two CTAs share an SM when they fit
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int kStages = kConsumers;              // bf16: stage w belongs to consumer warp w
constexpr int kStageBytes = 2 * 64 * 128 * 2;   // K + V of one 64-key block, D = 128, bf16
constexpr int kMaxStages = 2 * kConsumers;
// Stage geometry per cache format.  An FP8 block is half the bytes, so the same shared memory
// holds twice the stages: consumer warp w owns stages w and w + C (entries w, w + C, ...
// alternate between them), so each stage's barrier phases are still consumed by one warp in order.
template <bool F8>
struct Stg {
  static constexpr int kHalf = F8 ? 64 * 128 : 64 * 128 * 2;   // K at 0, V at kHalf
  static constexpr int kBytes = 2 * kHalf;
  static constexpr int kCount = kStages * kStageBytes / kBytes;
  static_assert(kCount % kConsumers == 0 && kCount <= kMaxStages, "stages per consumer warp");
};
constexpr int kMaxList = 72;                     // blocks per split (incl. padding)
#ifndef HYS_DECODE_TOK_SPLIT
#define HYS_DECODE_TOK_SPLIT 2048
#endif
constexpr int kTokSplit = HYS_DECODE_TOK_SPLIT;  // selected tokens per token-sparse split (stages of 64)
static_assert(kTokSplit % 32 == 0 && kTokSplit <= 4096 && kTokSplit / 64 <= 72, "a split's list fits the entry list");
constexpr int kPartBytes = kConsumers * 16 * (128 + 2) * 4;
static_assert(kPartBytes <= kStages * kStageBytes, "partials reuse the stage buffers");
constexpr int kSmemBytes = kStages * kStageBytes + kMaxList * 16 + 256 + kTokSplit * 4 + 1024;
constexpr int kTargetCtas = 4 * 148;
#ifndef HYS_DECODE_SPARSE_BPS
#define HYS_DECODE_SPARSE_BPS 32
#endif
#ifndef HYS_DECODE_SPLIT_MAJOR
#define HYS_DECODE_SPLIT_MAJOR 1
#endif
// grid of the split kernel: (splits, Hkv, B), or (Hkv, B, splits) with HYS_DECODE_SPLIT_MAJOR
__host__ __forceinline__ dim3 split_grid(int nsplit, int Hkv, int B) {
  return HYS_DECODE_SPLIT_MAJOR ? dim3(Hkv, B, nsplit) : dim3(nsplit, Hkv, B);
}
constexpr int kSparseBps = HYS_DECODE_SPARSE_BPS;   // selected blocks per sparse-layer split (<= 32)
static_assert(kSparseBps <= 32 && kSparseBps <= kMaxList, "one warp gathers a split's entries");

struct Params {
  int B, L, Hq, Hkv, G, NB;
  const int* seqlens;
  int mode;         // 0: full layer (contiguous blocks), 1: sparse layer (selected blocks + ring),
                    // 2: token-sparse layer (selected tokens + the newest W of the cache)
  int bps;          // blocks per split
  int nsplit;       // splits per (b, g)
  int nsp;          // sparse-mode splits over the selected list (the ring is split nsp)
  const int* idx;   // [B,Hkv,kb] (mode 1)
  int kb;
  int W;            // ring capacity (mode 1)
  const int* swa_len;
  const float* sinks;      // [Hq,2] sink logits of the two branches (mode 1), or null
  float* logits;           // [B,Hq,L] raw logits of every cached key (mode 0, token scores), or null
  float* tok_scores;       // [B,Hkv,L] token scores written by the merge (mode 0), or null
  int forced;              // newest tokens always attended (mode 2)
  const __nv_bfloat16* q;  // [B,Hq,D]
  const uint8_t* kc;       // [B,Hkv,L,D] shared cache, bf16 or FP8 (mode 2 gathers rows from it)
  const uint8_t* vc;
  const float* k_scale;    // [Hkv] FP8 cache scales (value = code * scale), or null for bf16
  const float* v_scale;
  float* pm;        // [B,Hq,nsplit]
  float* pl;
  float* po;        // [B,Hq,nsplit,D]
  float* bmax;      // [B,Hq,NB] raw max logit of each block (mode 0)
  int* status;
  float scale_log2;
};

struct Entry {  // 16 bytes
  int row;    // first key row in its tensor (src 2: first position in the split's token list)
  int valid;  // valid keys (1..64)
  int src;    // 0: shared cache, 1: SWA ring, 2: gathered tokens of the shared cache
  int blk;    // block id (for the block max)
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma16816_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// two E4M3 codes (low byte -> low half) to two f16 values; every E4M3 value is exact in f16
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t v) {
  uint32_t r;
  const unsigned short h = static_cast<unsigned short>(v & 0xffffu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(h));
  return r;
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
  return pack_f16x2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}

// byte offset of (row, 16-byte unit) inside a [64 rows][128 B] 128-byte-swizzled box
__device__ __forceinline__ uint32_t sw128(int row, int unit) { return row * 128 + ((unit ^ (row & 7)) << 4); }

// 16-byte global -> shared copy on the load/store path (kept in L2 only), and an arrival on a
// stage barrier that fires once every earlier copy of this thread has landed (the barrier's
// expected count is raised for it, so it adds no arrival of its own)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_bar_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(tc::smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

template <bool F8>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmKr, const __grid_constant__ CUtensorMap tmVr,
                        const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* part = reinterpret_cast<float*>(smem);  // after the pipeline has drained
  Entry* list = reinterpret_cast<Entry*>(smem + kStages * kStageBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes + kMaxList * 16);
  uint64_t* empty = full + kMaxStages;
  int* s_nlist = reinterpret_cast<int*>(empty + kMaxStages);
  constexpr int NS = Stg<F8>::kCount, SB = Stg<F8>::kBytes, HALF = Stg<F8>::kHalf;
  volatile int* abort = s_nlist + 1;
  int* tok = reinterpret_cast<int*>(smem + kStages * kStageBytes + kMaxList * 16 + 256);   // mode 2 token rows

#if HYS_DECODE_SPLIT_MAJOR
  const int sp = blockIdx.z, g = blockIdx.x, b = blockIdx.y;   // every (b, g)'s first split launches first
#else
  const int sp = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
#endif
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Lb = p.seqlens ? max(1, min(p.seqlens[b], p.L)) : p.L;

  if (p.mode == 1 && sp < p.nsp) {
    // this split's selected blocks: warp 0 reads the index entries at once and keeps the
    // valid ones in order (ballot + prefix count)
    if (warp == 0) {
      const int nb = (Lb + 63) / 64;
      const int* sel = p.idx + ((size_t)b * p.Hkv + g) * p.kb;
      const int e = sp * p.bps + lane;
      const int j = (lane < p.bps && e < p.kb) ? sel[e] : -1;
      const bool keep = j >= 0 && j < nb;
      const unsigned m = __ballot_sync(0xffffffffu, keep);
      if (keep) list[__popc(m & ((1u << lane) - 1u))] = Entry{64 * j, min(64, Lb - 64 * j), 0, j};
      if (lane == 0) *s_nlist = __popc(m);
    }
  }
  if (p.mode == 2 && sp < p.nsp && warp == 0) {
    // this split's selected tokens (older than the forced window), compacted in order; stage i
    // gathers tokens 64i .. 64i+63 of the list
    // (all of the split's entries are loaded before the first ballot, so their latencies overlap)
    const int lim = Lb - p.forced;
    const int* sel = p.idx + ((size_t)b * p.Hkv + g) * p.kb;
    const int e_lo = sp * kTokSplit, e_hi = min(p.kb, e_lo + kTokSplit);
    constexpr int kPass = kTokSplit < 1024 ? kTokSplit : 1024;   // entries loaded per pass (32 per lane)
    int cnt = 0;
    for (int e_pass = e_lo; e_pass < e_hi; e_pass += kPass) {
      int jv[kPass / 32];
#pragma unroll
      for (int c = 0; c < kPass / 32; ++c) {
        const int e = e_pass + 32 * c + lane;
        jv[c] = e < e_hi ? sel[e] : -1;
      }
#pragma unroll
      for (int c = 0; c < kPass / 32; ++c) {
        const bool keep = jv[c] >= 0 && jv[c] < lim;
        const unsigned m = __ballot_sync(0xffffffffu, keep);
        if (keep) tok[cnt + __popc(m & ((1u << lane) - 1u))] = jv[c];
        cnt += __popc(m);
      }
    }
    if (lane == 0) {
      int n = 0;
      for (int i = 0; 64 * i < cnt; ++i) list[n++] = Entry{64 * i, min(64, cnt - 64 * i), 2, 0};
      *s_nlist = n;
    }
  }
  if (threadIdx.x == 0) {
    // this split's block list
    int n = 0;
    if (p.mode == 0) {
      const int nb = (Lb + 63) / 64;
      for (int j = sp * p.bps; j < min(nb, (sp + 1) * p.bps); ++j) list[n++] = Entry{64 * j, min(64, Lb - 64 * j), 0, j};
      *s_nlist = n;
    } else if (p.mode == 1 && sp >= p.nsp) {
      const int nring = p.swa_len ? max(0, min(p.swa_len[b], p.W)) : p.W;
      for (int j = 0; 64 * j < nring; ++j) list[n++] = Entry{64 * j, min(64, nring - 64 * j), 1, j};
      *s_nlist = n;
    } else if (p.mode == 2 && sp >= p.nsp) {
      // the forced newest tokens [L_b - forced, L_b - 1]: contiguous rows of the cache
      const int w0 = max(0, Lb - p.forced);
      for (int r = w0; r < Lb; r += 64) list[n++] = Entry{r, min(64, Lb - r), 0, 0};
      *s_nlist = n;
    }

    for (int i = 0; i < NS; ++i) {
      tc::mbar_init(&full[i], 1);
      tc::mbar_init(&empty[i], 1);
    }
    *abort = 0;
    tc::fence_barrier_init();
  }
  __syncthreads();
  const int nlist = *s_nlist;
  // FP8: logits are kept in code units (q . code); the K scale joins the softmax scale
  const float sc = F8 ? p.scale_log2 * p.k_scale[g] : p.scale_log2;

  if (warp == kConsumers) {
    // ---------------------------------------------------------------- producer
    // Lane 0 waits for the stage and issues contiguous blocks (one TMA box per 64 rows and
    // 128-byte chunk).  Gathered tokens go through the load/store path instead (scattered
    // 256-byte rows are too small for TMA's per-request rate): the warp's 32 lanes copy 16-byte
    // units, two token rows per instruction, into the same swizzled layout as the boxes.
    bool ok = true;
    const int head = b * p.Hkv + g;
    for (int i = 0; i < nlist; ++i) {
      const int st = i % NS;
      if (lane == 0) ok = tc::mbar_wait(&empty[st], ((i / NS) & 1) ^ 1, abort);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      uint8_t* dst = smem + st * SB;
      const Entry e = list[i];
      if (e.src == 2) {
        // 16-byte unit u of a row (bf16: 256-byte rows, units 0-7 in the low box, 8-15 the
        // high one; FP8: 128-byte rows, one box)
        constexpr int kRow = F8 ? 128 : 256, kUpr = kRow / 16, kRpi = 32 / kUpr;
        const int u = lane % kUpr;
        const uint32_t sdst = tc::smem_u32(dst) + (u >> 3) * 8192;
        const uint8_t* kh = p.kc + (size_t)head * p.L * kRow + u * 16;
        const uint8_t* vh = p.vc + (size_t)head * p.L * kRow + u * 16;
#pragma unroll 4
        for (int j = 0; j < 64 / kRpi; ++j) {
          const int q = kRpi * j + lane / kUpr;   // rows past the stage's count repeat its first token (masked)
          const size_t r = (size_t)tok[e.row + (q < e.valid ? q : 0)] * kRow;
          const uint32_t so = sdst + sw128(q, u & 7);
          cp_async16(so, kh + r);
          cp_async16(so + HALF, vh + r);
        }
        cp_async_bar_arrive(&full[st]);
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&full[st]);
      } else if (lane == 0) {
        const CUtensorMap* mk = e.src ? &tmKr : &tmK;
        const CUtensorMap* mv = e.src ? &tmVr : &tmV;
        tc::mbar_arrive_expect_tx(&full[st], SB);
        if (F8) {
          tc::tma_load_3d(mk, &full[st], dst, 0, e.row, head);
          tc::tma_load_3d(mv, &full[st], dst + HALF, 0, e.row, head);
        } else {
          tc::tma_load_3d(mk, &full[st], dst, 0, e.row, head);
          tc::tma_load_3d(mk, &full[st], dst + 8192, 64, e.row, head);
          tc::tma_load_3d(mv, &full[st], dst + 16384, 0, e.row, head);
          tc::tma_load_3d(mv, &full[st], dst + 24576, 64, e.row, head);
        }
      }
    }
    if (lane == 0) {
      if (!ok) {
        *abort = 1;
        report_status(p.status, HYS_ERR_TIMEOUT);
      }
      for (int i = max(0, nlist - NS); i < nlist; ++i)
        tc::mbar_wait_drain(&full[i % NS], (i / NS) & 1);
    }
    cp_async_wait_all();
    __syncwarp();
    tc::named_bar_sync(1, kThreads);
  } else {
    // ---------------------------------------------------------------- consumers
    const int r = lane >> 2, cq = lane & 3;
    const int h_lo = r, h_hi = r + 8;
    // Q as A fragments (rows = heads, zero past G)
    uint32_t qa[8][4];
    const __nv_bfloat16* qg = p.q + ((size_t)b * p.Hq + g * p.G) * 128;
    if (F8) {
      // f16 fragments in the dim order of the FP8 K fragments below: k-step ks covers dims
      // 16ks .. 16ks+15 and its k slots (2c, 2c+1 | 2c+8, 2c+9) hold dims 16ks + 4c + (0, 1 | 2, 3)
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int d0 = 16 * ks + 4 * cq;
        const uint2 lo = h_lo < p.G ? *reinterpret_cast<const uint2*>(qg + h_lo * 128 + d0) : make_uint2(0u, 0u);
        const uint2 hi = h_hi < p.G ? *reinterpret_cast<const uint2*>(qg + h_hi * 128 + d0) : make_uint2(0u, 0u);
        qa[ks][0] = bf16x2_to_f16x2(lo.x);
        qa[ks][1] = bf16x2_to_f16x2(hi.x);
        qa[ks][2] = bf16x2_to_f16x2(lo.y);
        qa[ks][3] = bf16x2_to_f16x2(hi.y);
      }
    } else {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int c0 = 16 * ks + 2 * cq;
        qa[ks][0] = h_lo < p.G ? *reinterpret_cast<const uint32_t*>(qg + h_lo * 128 + c0) : 0u;
        qa[ks][1] = h_hi < p.G ? *reinterpret_cast<const uint32_t*>(qg + h_hi * 128 + c0) : 0u;
        qa[ks][2] = h_lo < p.G ? *reinterpret_cast<const uint32_t*>(qg + h_lo * 128 + c0 + 8) : 0u;
        qa[ks][3] = h_hi < p.G ? *reinterpret_cast<const uint32_t*>(qg + h_hi * 128 + c0 + 8) : 0u;
      }
    }
    float o[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
    float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.0f, l_hi = 0.0f;
    bool ok = true;
    const uint32_t sbase = tc::smem_u32(smem);
    for (int i = warp; i < nlist; i += kConsumers) {
      const int st = i % NS;   // bf16: == warp; FP8: warp or warp + C
      if (!(ok = tc::mbar_wait(&full[st], (i / NS) & 1, abort))) break;
      const Entry e = list[i];
      const uint32_t kb = sbase + st * SB, vb = kb + HALF;
      // ---- S = Q K^T : 8 key tiles x 8 dim steps
      float s[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
        const int key = 8 * nt + (lane & 7);
        const int mtx = lane >> 3;
        if (F8) {
          // an 8 x 16-byte matrix of codes read as 16-bit pairs: lane gets key 8nt + lane/4 and
          // dims 16sg + 4c .. +3 (c = lane % 4), i.e. both B registers of k-step sg
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            uint32_t r[4];
            ldsm_x4(kb + sw128(key, 4 * hf + mtx), r[0], r[1], r[2], r[3]);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              const int ks = 4 * hf + m;
              mma16816_f16(s[nt], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], e4m3x2_to_f16x2(r[m]),
                           e4m3x2_to_f16x2(r[m] >> 16));
            }
          }
        } else {
#pragma unroll
          for (int kp = 0; kp < 4; ++kp) {  // pairs of 16-dim steps
            const int ks = 2 * kp;
            const int chunk = ks >> 2;
            const int unit = 2 * (ks & 3) + mtx;
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kb + chunk * 8192 + sw128(key, unit), b0, b1, b2, b3);
            mma16816(s[nt], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
            mma16816(s[nt], qa[ks + 1][0], qa[ks + 1][1], qa[ks + 1][2], qa[ks + 1][3], b2, b3);
          }
        }
      }
      // ---- mask keys past the valid count, block max, online softmax
      float bm_lo = -INFINITY, bm_hi = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int key = 8 * nt + 2 * cq + c;
          if (key >= e.valid) {
            s[nt][c] = -INFINITY;
            s[nt][2 + c] = -INFINITY;
          }
          bm_lo = fmaxf(bm_lo, s[nt][c]);
          bm_hi = fmaxf(bm_hi, s[nt][2 + c]);
        }
      }
      bm_lo = fmaxf(bm_lo, __shfl_xor_sync(0xffffffffu, bm_lo, 1));
      bm_lo = fmaxf(bm_lo, __shfl_xor_sync(0xffffffffu, bm_lo, 2));
      bm_hi = fmaxf(bm_hi, __shfl_xor_sync(0xffffffffu, bm_hi, 1));
      bm_hi = fmaxf(bm_hi, __shfl_xor_sync(0xffffffffu, bm_hi, 2));
      if (p.mode == 0 && cq == 0) {
        if (h_lo < p.G) p.bmax[((size_t)b * p.Hq + g * p.G + h_lo) * p.NB + e.blk] = bm_lo;
        if (h_hi < p.G) p.bmax[((size_t)b * p.Hq + g * p.G + h_hi) * p.NB + e.blk] = bm_hi;
      }
      if (p.logits != nullptr) {
        // token scores need every key's logit under the final max and sum: keep them
        float* lrow_lo = p.logits + ((size_t)b * p.Hq + g * p.G + h_lo) * p.L + e.row;
        float* lrow_hi = p.logits + ((size_t)b * p.Hq + g * p.G + h_hi) * p.L + e.row;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int key = 8 * nt + 2 * cq + c;
            if (key < e.valid) {
              if (h_lo < p.G) lrow_lo[key] = s[nt][c];
              if (h_hi < p.G) lrow_hi[key] = s[nt][2 + c];
            }
          }
        }
      }
      const float mn_lo = fmaxf(m_lo, bm_lo), mn_hi = fmaxf(m_hi, bm_hi);
      const float a_lo = exp2f((m_lo - mn_lo) * sc), a_hi = exp2f((m_hi - mn_hi) * sc);
      m_lo = mn_lo;
      m_hi = mn_hi;
      l_lo *= a_lo;
      l_hi *= a_hi;
#pragma unroll
      for (int dt = 0; dt < 16; ++dt) {
        o[dt][0] *= a_lo;
        o[dt][1] *= a_lo;
        o[dt][2] *= a_hi;
        o[dt][3] *= a_hi;
      }
      const float ms_lo = m_lo * sc, ms_hi = m_hi * sc;
      uint32_t pa[8][2];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float p0 = exp2f(fmaf(s[nt][0], sc, -ms_lo));
        const float p1 = exp2f(fmaf(s[nt][1], sc, -ms_lo));
        const float p2 = h_hi < p.G ? exp2f(fmaf(s[nt][2], sc, -ms_hi)) : 0.0f;
        const float p3 = h_hi < p.G ? exp2f(fmaf(s[nt][3], sc, -ms_hi)) : 0.0f;
        l_lo += p0 + p1;
        l_hi += p2 + p3;
        pa[nt][0] = F8 ? pack_f16x2(p0, p1) : tc::pack_bf16x2(p0, p1);
        pa[nt][1] = F8 ? pack_f16x2(p2, p3) : tc::pack_bf16x2(p2, p3);
      }
      // ---- O += P V : 4 key steps x 16 dim tiles
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int mtx = lane >> 3;
        const int key = 16 * kk + 8 * (mtx & 1) + (lane & 7);
        if (F8) {
          // transposed 8 x 8 matrices of 16-bit pairs: lane gets keys 2c, 2c+1 x dims 2n, 2n+1 of
          // segment sg (n = lane / 4); regrouping the bytes by dim gives the B registers of
          // output tile 2sg (dims 16sg + 2n) and 2sg+1 (dims 16sg + 2n + 1)
#pragma unroll
          for (int sp = 0; sp < 4; ++sp) {
            uint32_t r[4];
            ldsm_x4_t(vb + sw128(key, 2 * sp + (mtx >> 1)), r[0], r[1], r[2], r[3]);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const uint32_t x0 = __byte_perm(r[2 * j], 0u, 0x3120), x1 = __byte_perm(r[2 * j + 1], 0u, 0x3120);
              const int ot = 2 * (2 * sp + j);
              mma16816_f16(o[ot], pa[2 * kk][0], pa[2 * kk][1], pa[2 * kk + 1][0], pa[2 * kk + 1][1],
                           e4m3x2_to_f16x2(x0), e4m3x2_to_f16x2(x1));
              mma16816_f16(o[ot + 1], pa[2 * kk][0], pa[2 * kk][1], pa[2 * kk + 1][0], pa[2 * kk + 1][1],
                           e4m3x2_to_f16x2(x0 >> 16), e4m3x2_to_f16x2(x1 >> 16));
            }
          }
        } else {
#pragma unroll
          for (int dp = 0; dp < 8; ++dp) {  // pairs of 8-dim tiles
            const int dt = 2 * dp + (mtx >> 1);
            const int chunk = dt >> 3;
            const int unit = dt & 7;
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(vb + chunk * 8192 + sw128(key, unit), b0, b1, b2, b3);
            mma16816(o[2 * dp], pa[2 * kk][0], pa[2 * kk][1], pa[2 * kk + 1][0], pa[2 * kk + 1][1], b0, b1);
            mma16816(o[2 * dp + 1], pa[2 * kk][0], pa[2 * kk][1], pa[2 * kk + 1][0], pa[2 * kk + 1][1], b2, b3);
          }
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&empty[st]);
    }
    if (!ok) {
      *abort = 1;
      report_status(p.status, HYS_ERR_TIMEOUT);
    }
    // ---- this warp's partial (m, l, O) -> shared memory, once no warp reads a stage
    //      any more and the producer has drained its loads (all consumer + producer warps)
    tc::named_bar_sync(1, kThreads);
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
    float* wp = part + warp * 16 * 130;  // [16 heads][m, l, O[128]]
    if (cq == 0) {
      wp[h_lo * 130 + 0] = m_lo;
      wp[h_lo * 130 + 1] = l_lo;
      wp[h_hi * 130 + 0] = m_hi;
      wp[h_hi * 130 + 1] = l_hi;
    }
#pragma unroll
    for (int dt = 0; dt < 16; ++dt) {
      // bf16: tile dt holds dims 8dt + (2c, 2c+1); FP8: tile 2sg+j holds dims 16sg + 4c + j + (0, 2)
      const int d0 = F8 ? 16 * (dt >> 1) + 4 * cq + (dt & 1) : 8 * dt + 2 * cq;
      const int d1 = F8 ? d0 + 2 : d0 + 1;
      wp[h_lo * 130 + 2 + d0] = o[dt][0];
      wp[h_lo * 130 + 2 + d1] = o[dt][1];
      wp[h_hi * 130 + 2 + d0] = o[dt][2];
      wp[h_hi * 130 + 2 + d1] = o[dt][3];
    }
  }
  __syncthreads();
  // ---- merge the warps' partials into the split's partial
  for (int e = threadIdx.x; e < p.G * 128; e += kThreads) {
    const int hh = e >> 7, d = e & 127;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, part[(w * 16 + hh) * 130]);
    float lsum = 0.0f, acc = 0.0f;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) {
      const float mw = part[(w * 16 + hh) * 130];
      const float f = mw == -INFINITY ? 0.0f : exp2f((mw - M) * sc);
      lsum += part[(w * 16 + hh) * 130 + 1] * f;
      acc += part[(w * 16 + hh) * 130 + 2 + d] * f;
    }
    const size_t ph = ((size_t)b * p.Hq + g * p.G + hh) * p.nsplit + sp;
    p.po[ph * 128 + d] = acc;
    if (d == 0) {
      p.pm[ph] = M;
      p.pl[ph] = lsum;
    }
  }
}

// Merge the splits of one (b, g).  mode 0: o and block scores; mode 1: gated two-branch output.
__global__ void __launch_bounds__(256) decode_merge_kernel(const Params p, const float* __restrict__ gate,
                                                           __nv_bfloat16* __restrict__ o, float* __restrict__ scores,
                                                           int red_max) {
  __shared__ float sM[2][16], sInv[2][16], sVw[2][16];
  const int g = blockIdx.x, b = blockIdx.y;
  const int Lb = p.seqlens ? max(1, min(p.seqlens[b], p.L)) : p.L;
  const float sc = p.k_scale ? p.scale_log2 * p.k_scale[g] : p.scale_log2;   // FP8: logits in code units
  const float vsc = p.v_scale ? p.v_scale[g] : 1.0f;
  const bool two = p.mode == 1;   // the sparse layer merges two branches under the gate
  const int nbr = two ? 2 : 1;
  if (threadIdx.x < p.G * nbr) {
    const int hh = threadIdx.x % p.G, br = threadIdx.x / p.G;
    const int s0 = !two ? 0 : (br == 0 ? 0 : p.nsp);
    const int s1 = !two ? p.nsplit : (br == 0 ? p.nsp : p.nsplit);
    const size_t ph = ((size_t)b * p.Hq + g * p.G + hh) * p.nsplit;
    float M = -INFINITY;
    for (int s = s0; s < s1; ++s) M = fmaxf(M, p.pm[ph + s]);
    float L = 0.0f;
    for (int s = s0; s < s1; ++s)
      if (p.pm[ph + s] != -INFINITY) L += p.pl[ph + s] * exp2f((p.pm[ph + s] - M) * sc);
    // the branch's sink logit: a softmax entry with a zero value
    if (p.mode == 1 && p.sinks != nullptr) L += exp2f(p.sinks[2 * (g * p.G + hh) + br] * kLog2e - M * sc);
    sM[br][hh] = M;
    sInv[br][hh] = L > 0.0f ? 1.0f / L : 0.0f;
    sVw[br][hh] = L > 0.0f ? vsc / L : 0.0f;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < p.G * 128; e += blockDim.x) {
    const int hh = e >> 7, d = e & 127;
    const size_t ph = ((size_t)b * p.Hq + g * p.G + hh) * p.nsplit;
    float out = 0.0f;
    for (int br = 0; br < nbr; ++br) {
      const int s0 = !two ? 0 : (br == 0 ? 0 : p.nsp);
      const int s1 = !two ? p.nsplit : (br == 0 ? p.nsp : p.nsplit);
      float acc = 0.0f;
      for (int s = s0; s < s1; ++s) {
        const float m = p.pm[ph + s];
        if (m != -INFINITY) acc = fmaf(p.po[(ph + s) * 128 + d], exp2f((m - sM[br][hh]) * sc), acc);
      }
      float w = sVw[br][hh];   // 1/l, times the V scale of an FP8 cache
      if (two) w *= sigmoidf_(gate[((size_t)b * p.Hq + g * p.G + hh) * 2 + br]);
      out = fmaf(acc, w, out);
    }
    o[((size_t)b * p.Hq + g * p.G + hh) * 128 + d] = __float2bfloat16_rn(out);
  }
  if (p.mode == 0 && scores != nullptr) {
    const int nb = (Lb + 63) / 64;
    for (int j = threadIdx.x; j < p.NB; j += blockDim.x) {
      float a = 0.0f;
      if (j < nb) {
        for (int hh = 0; hh < p.G; ++hh) {
          const float x = exp2f((p.bmax[((size_t)b * p.Hq + g * p.G + hh) * p.NB + j] - sM[0][hh]) * sc) * sInv[0][hh];
          a = hh == 0 ? x : (red_max ? fmaxf(a, x) : a + x);
        }
      }
      scores[((size_t)b * p.Hkv + g) * p.NB + j] = a;
    }
  }
}

// Token scores of the full layer (token-variant decode): sum over the group's heads of
// exp(s - m) / l under the merged statistics, for the positions [1024 x, 1024 x + 1024) of
// (b, g).  Many CTAs per sequence so the logit stream (G fp32 per cached token) runs at HBM speed.
constexpr int kTokScoreSpan = 1024;
__global__ void __launch_bounds__(256) decode_token_scores_kernel(const Params p) {
  __shared__ float sM[16], sInv[16];
  const int g = blockIdx.y, b = blockIdx.z;
  const int Lb = p.seqlens ? max(1, min(p.seqlens[b], p.L)) : p.L;
  const float sc = p.k_scale ? p.scale_log2 * p.k_scale[g] : p.scale_log2;
  if (threadIdx.x < p.G) {
    const size_t ph = ((size_t)b * p.Hq + g * p.G + threadIdx.x) * p.nsplit;
    float M = -INFINITY;
    for (int s = 0; s < p.nsplit; ++s) M = fmaxf(M, p.pm[ph + s]);
    float L = 0.0f;
    for (int s = 0; s < p.nsplit; ++s)
      if (p.pm[ph + s] != -INFINITY) L += p.pl[ph + s] * exp2f((p.pm[ph + s] - M) * sc);
    sM[threadIdx.x] = M * sc;
    sInv[threadIdx.x] = L > 0.0f ? 1.0f / L : 0.0f;
  }
  __syncthreads();
  float* trow = p.tok_scores + ((size_t)b * p.Hkv + g) * p.L;
  const float* lg = p.logits + ((size_t)b * p.Hq + g * p.G) * p.L;
  const int i0 = blockIdx.x * kTokScoreSpan, i1 = min(p.L, i0 + kTokScoreSpan);
  if ((p.L & 3) == 0) {
    // four positions per thread: 16-byte loads of each head's logits, one 16-byte store
    for (int i = i0 + 4 * threadIdx.x; i < i1; i += 4 * blockDim.x) {
      float4 a = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      if (i < Lb) {
        for (int hh = 0; hh < p.G; ++hh) {
          const float4 x = *reinterpret_cast<const float4*>(lg + (size_t)hh * p.L + i);
          const float m = sM[hh], w = sInv[hh];
          a.x += exp2f(fmaf(x.x, sc, -m)) * w;
          a.y += exp2f(fmaf(x.y, sc, -m)) * w;
          a.z += exp2f(fmaf(x.z, sc, -m)) * w;
          a.w += exp2f(fmaf(x.w, sc, -m)) * w;
        }
        if (i + 1 >= Lb) a.y = 0.0f;
        if (i + 2 >= Lb) a.z = 0.0f;
        if (i + 3 >= Lb) a.w = 0.0f;
      }
      *reinterpret_cast<float4*>(trow + i) = a;
    }
  } else {
    for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
      float a = 0.0f;
      if (i < Lb)
        for (int hh = 0; hh < p.G; ++hh) a += exp2f(fmaf(lg[(size_t)hh * p.L + i], sc, -sM[hh])) * sInv[hh];
      trow[i] = a;
    }
  }
}

bool make_map(CUtensorMap* m, const void* base, int rows, int heads) {
  EncodeTiledFn fn = tma_encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)rows, (cuuint64_t)heads};
  cuuint64_t strides[2] = {256, (cuuint64_t)rows * 256};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// FP8 codes: [heads][rows][128] bytes, box 128 bytes x 64 rows x 1 head
bool make_map8(CUtensorMap* m, const void* base, int rows, int heads) {
  EncodeTiledFn fn = tma_encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)rows, (cuuint64_t)heads};
  cuuint64_t strides[2] = {128, (cuuint64_t)rows * 128};
  cuuint32_t box[3] = {128, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_cache_maps(bool f8, CUtensorMap* mk, CUtensorMap* mv, const void* kc, const void* vc, const DecodeDims& d) {
  if (f8) return make_map8(mk, kc, d.L, d.B * d.Hkv) && make_map8(mv, vc, d.L, d.B * d.Hkv);
  return make_map(mk, kc, d.L, d.B * d.Hkv) && make_map(mv, vc, d.L, d.B * d.Hkv);
}

int full_bps(const DecodeDims& d) {
  const long long work = (long long)d.NB * d.B * d.Hkv;
  long long bps = (work + kTargetCtas - 1) / kTargetCtas;
  if (bps < 4) bps = 4;
  if (bps > 64) bps = 64;
  return (int)bps;
}

void fill_common(Params& p, const DecodeDims& d, const void* q, const int* seqlens, void* ws, int nsplit) {
  p.B = d.B;
  p.L = d.L;
  p.Hq = d.Hq;
  p.Hkv = d.Hkv;
  p.G = d.G();
  p.NB = d.NB;
  p.seqlens = seqlens;
  p.nsplit = nsplit;
  p.q = reinterpret_cast<const __nv_bfloat16*>(q);
  float* w = reinterpret_cast<float*>(ws);
  const size_t np = (size_t)d.B * d.Hq * nsplit;
  p.pm = w;
  p.pl = w + np;
  p.po = w + 2 * np;
  p.bmax = w + 2 * np + np * 128;
  p.status = device_status_ptr();
  p.scale_log2 = kLog2e / sqrtf(128.0f);
  p.idx = nullptr;
  p.kb = 0;
  p.W = 0;
  p.swa_len = nullptr;
  p.sinks = nullptr;
  p.kc = p.vc = nullptr;
  p.k_scale = p.v_scale = nullptr;
  p.logits = nullptr;
  p.tok_scores = nullptr;
  p.forced = 0;
  p.nsp = 0;
}

// The shared-memory opt-in is a per-device attribute: remember it per device (one bit each).
template <bool F8>
cudaError_t set_smem() {
  static std::atomic<unsigned long long> done{0ull};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
  if (bit != 0ull && (done.load(std::memory_order_relaxed) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(decode_split_kernel<F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_relaxed);
  return e;
}

}  // namespace

bool decode_mma_supported(const DecodeDims& d, hys_dtype dt) { return dt == HYS_BF16 && d.D == 128 && d.G() <= 16; }

size_t decode_mma_full_workspace(const DecodeDims& d) {
  const size_t nsplit = (d.NB + full_bps(d) - 1) / full_bps(d);
  const size_t np = (size_t)d.B * d.Hq * nsplit;
  return sizeof(float) * (np * (2 + 128) + (size_t)d.B * d.Hq * d.NB);
}

int decode_sparse_splits(int kb) { return (kb + kSparseBps - 1) / kSparseBps; }

size_t decode_mma_sparse_workspace(const DecodeDims& d, int kb) {
  const size_t nsplit = decode_sparse_splits(kb) + 1;
  return sizeof(float) * ((size_t)d.B * d.Hq * nsplit * (2 + 128));
}

cudaError_t launch_decode_full_mma(const DecodeDims& d, const void* q, const void* kc, const void* vc,
                                   const int* seqlens, void* o, float* scores, hys_reduce red, void* ws,
                                   cudaStream_t s) {
  CUtensorMap mk, mv;
  if (!make_map(&mk, kc, d.L, d.B * d.Hkv) || !make_map(&mv, vc, d.L, d.B * d.Hkv)) return cudaErrorInvalidValue;
  cudaError_t e = set_smem<false>();
  if (e != cudaSuccess) return e;
  Params p;
  const int bps = full_bps(d);
  const int nsplit = (d.NB + bps - 1) / bps;
  fill_common(p, d, q, seqlens, ws, nsplit);
  p.mode = 0;
  p.bps = bps;
  decode_split_kernel<false><<<split_grid(nsplit, d.Hkv, d.B), kThreads, kSmemBytes, s>>>(mk, mv, mk, mv, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_merge_kernel<<<dim3(d.Hkv, d.B), 256, 0, s>>>(p, nullptr, reinterpret_cast<__nv_bfloat16*>(o), scores,
                                                      red == HYS_REDUCE_MAX);
  return cudaGetLastError();
}

cudaError_t launch_decode_sparse_mma(const DecodeDims& d, const void* q, const void* kc, const void* vc,
                                     const int* seqlens, const int* idx, int kb, const void* kr, const void* vr, int W,
                                     const int* swa_len, const float* gate, const float* sinks, void* o, void* ws,
                                     cudaStream_t s) {
  CUtensorMap mk, mv, mkr, mvr;
  if (!make_map(&mk, kc, d.L, d.B * d.Hkv) || !make_map(&mv, vc, d.L, d.B * d.Hkv) ||
      !make_map(&mkr, kr, W, d.B * d.Hkv) || !make_map(&mvr, vr, W, d.B * d.Hkv))
    return cudaErrorInvalidValue;
  cudaError_t e = set_smem<false>();
  if (e != cudaSuccess) return e;
  Params p;
  const int nsp = decode_sparse_splits(kb);
  fill_common(p, d, q, seqlens, ws, nsp + 1);
  p.mode = 1;
  p.bps = kSparseBps;
  p.nsp = nsp;
  p.idx = idx;
  p.kb = kb;
  p.W = W;
  p.swa_len = swa_len;
  p.sinks = sinks;
  decode_split_kernel<false><<<split_grid(nsp + 1, d.Hkv, d.B), kThreads, kSmemBytes, s>>>(mk, mv, mkr, mvr, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_merge_kernel<<<dim3(d.Hkv, d.B), 256, 0, s>>>(p, gate, reinterpret_cast<__nv_bfloat16*>(o), nullptr, 0);
  return cudaGetLastError();
}

// the logits follow the split partials at a 256-byte boundary (the token-score kernel reads
// them with 16-byte loads)
static size_t logits_offset(const DecodeDims& d) { return (decode_mma_full_workspace(d) + 255) & ~size_t(255); }

size_t decode_mma_full_tokens_workspace(const DecodeDims& d) {
  return logits_offset(d) + sizeof(float) * (size_t)d.B * d.Hq * d.L;
}

namespace {

template <bool F8>
cudaError_t full_tokens(const DecodeDims& d, const void* q, const void* kc, const void* vc, const float* k_scale,
                        const float* v_scale, const int* seqlens, void* o, float* tok_scores, void* ws, cudaStream_t s) {
  CUtensorMap mk, mv;
  if (!make_cache_maps(F8, &mk, &mv, kc, vc, d)) return cudaErrorInvalidValue;
  cudaError_t e = set_smem<F8>();
  if (e != cudaSuccess) return e;
  Params p;
  const int bps = full_bps(d);
  const int nsplit = (d.NB + bps - 1) / bps;
  fill_common(p, d, q, seqlens, ws, nsplit);
  p.mode = 0;
  p.bps = bps;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.logits = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + logits_offset(d));
  p.tok_scores = tok_scores;
  decode_split_kernel<F8><<<split_grid(nsplit, d.Hkv, d.B), kThreads, kSmemBytes, s>>>(mk, mv, mk, mv, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_merge_kernel<<<dim3(d.Hkv, d.B), 256, 0, s>>>(p, nullptr, reinterpret_cast<__nv_bfloat16*>(o), nullptr, 0);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_token_scores_kernel<<<dim3((d.L + kTokScoreSpan - 1) / kTokScoreSpan, d.Hkv, d.B), 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_full_tokens_mma(const DecodeDims& d, const void* q, const void* kc, const void* vc,
                                          const int* seqlens, void* o, float* tok_scores, void* ws, cudaStream_t s) {
  return full_tokens<false>(d, q, kc, vc, nullptr, nullptr, seqlens, o, tok_scores, ws, s);
}

cudaError_t launch_decode_full_tokens_mma_fp8(const DecodeDims& d, const void* q, const void* kc, const void* vc,
                                              const float* k_scale, const float* v_scale, const int* seqlens, void* o,
                                              float* tok_scores, void* ws, cudaStream_t s) {
  return full_tokens<true>(d, q, kc, vc, k_scale, v_scale, seqlens, o, tok_scores, ws, s);
}

int decode_token_splits(int kt) { return (kt + kTokSplit - 1) / kTokSplit; }

size_t decode_mma_sparse_tokens_workspace(const DecodeDims& d, int kt) {
  const size_t nsplit = decode_token_splits(kt) + 1;
  return sizeof(float) * ((size_t)d.B * d.Hq * nsplit * (2 + 128));
}

namespace {

template <bool F8>
cudaError_t sparse_tokens(const DecodeDims& d, const void* q, const void* kc, const void* vc, const float* k_scale,
                          const float* v_scale, const int* seqlens, const int* idx, int kt, int forced, void* o,
                          void* ws, cudaStream_t s) {
  CUtensorMap mk, mv;
  if (!make_cache_maps(F8, &mk, &mv, kc, vc, d)) return cudaErrorInvalidValue;
  cudaError_t e = set_smem<F8>();
  if (e != cudaSuccess) return e;
  Params p;
  const int nsp = decode_token_splits(kt);
  fill_common(p, d, q, seqlens, ws, nsp + 1);
  p.mode = 2;
  p.bps = kTokSplit;
  p.nsp = nsp;
  p.idx = idx;
  p.kb = kt;
  p.forced = forced;
  p.kc = reinterpret_cast<const uint8_t*>(kc);
  p.vc = reinterpret_cast<const uint8_t*>(vc);
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  decode_split_kernel<F8><<<split_grid(nsp + 1, d.Hkv, d.B), kThreads, kSmemBytes, s>>>(mk, mv, mk, mv, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_merge_kernel<<<dim3(d.Hkv, d.B), 256, 0, s>>>(p, nullptr, reinterpret_cast<__nv_bfloat16*>(o), nullptr, 0);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_sparse_tokens_mma(const DecodeDims& d, const void* q, const void* kc, const void* vc,
                                            const int* seqlens, const int* idx, int kt, int forced, void* o, void* ws,
                                            cudaStream_t s) {
  return sparse_tokens<false>(d, q, kc, vc, nullptr, nullptr, seqlens, idx, kt, forced, o, ws, s);
}

cudaError_t launch_decode_sparse_tokens_mma_fp8(const DecodeDims& d, const void* q, const void* kc, const void* vc,
                                                const float* k_scale, const float* v_scale, const int* seqlens,
                                                const int* idx, int kt, int forced, void* o, void* ws, cudaStream_t s) {
  return sparse_tokens<true>(d, q, kc, vc, k_scale, v_scale, seqlens, idx, kt, forced, o, ws, s);
}

}  // namespace hys
