// Internal launchers of the HySparse kernels (C++; the public C ABI lives in abi.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "../../include/hysparse.h"

namespace hys {

// Device address of this device's status word (nullptr if it cannot be resolved).
int* device_status_ptr();

struct PrefillDims {
  int B, N, Hq, Hkv, D;
  int T;   // query tiles = ceil(N / 64)
  int NB;  // key blocks  = ceil(N / 64)
  __host__ __device__ int G() const { return Hq / Hkv; }
};

struct DecodeDims {
  int B, L, Hq, Hkv, D;
  int NB;  // ceil(L / 64)
  __host__ __device__ int G() const { return Hq / Hkv; }
};

// ---- full layer, SIMT fp32-accumulate path (any supported dtype / D / G) -------------
// Writes o, lse (always) and, in block mode, per-head partial block scores
// part[B,Hq,T,NB] (reduced over the tile's rows with `red`).
cudaError_t launch_full_attn_simt(const PrefillDims& d, hys_dtype dt, const void* q, const void* k,
                                  const void* v, void* o, float* lse, float* part, bool want_scores,
                                  hys_reduce red, cudaStream_t s);
// scores[B,Hkv,T,NB] = R over the group's heads (fixed head order) of part.
cudaError_t launch_head_reduce(const PrefillDims& d, const float* part, float* scores, hys_reduce red,
                               cudaStream_t s);
// Token scores [B,Hkv,T,N] from q, k and the rows' LSE.
cudaError_t launch_token_scores_simt(const PrefillDims& d, hys_dtype dt, const void* q, const void* k,
                                     const float* lse, float* scores, cudaStream_t s);

// ---- full layer, tcgen05 path (bf16, D=128, even G) ----------------------------------------
bool full_attn_tc_supported(const PrefillDims& d, hys_dtype dt, bool want_scores);
size_t full_attn_tc_workspace(const PrefillDims& d, bool want_scores);
// per_row: scores [B,Hkv,N,NB] per position, the group max (zeroed by the launch)
cudaError_t launch_full_attn_tc(const PrefillDims& d, const void* q, const void* k, const void* v,
                                void* o, float* lse, float* scores, hys_reduce red, bool want_scores,
                                void* ws, size_t ws_bytes, cudaStream_t s, bool per_row = false);

// Token scores (second pass) on the tensor cores; ws holds the 256-byte unit counter.
bool token_scores_tc_supported(const PrefillDims& d, hys_dtype dt);
cudaError_t launch_token_scores_tc(const PrefillDims& d, const void* q, const void* k, const float* lse,
                                   float* scores, void* ws, cudaStream_t s);

// Token-sparse layer on the tensor cores; ws holds the 256-byte unit counter.
bool token_sparse_tc_supported(const PrefillDims& d, hys_dtype dt, int forced);
size_t token_sparse_tc_workspace();
cudaError_t launch_token_sparse_tc(const PrefillDims& d, const void* q, const void* k, const void* v, const int* idx,
                                   int kt, int forced, void* o, void* ws, cudaStream_t s);

// ---- top-k -------------------------------------------------------------------------------
// rows = B*Hkv*T (prefill) or B*Hkv (decode); row r has n_cand(r) candidates.
cudaError_t launch_topk_blocks(const float* scores, int* idx, int B, int Hkv, int T, int NB, int k,
                               const int* seqlens, int L, bool decode, cudaStream_t s);
// per-position rows: B*Hkv*N rows of NB scores; row (b, g, t) has floor(t/64) + 1 candidates
cudaError_t launch_topk_blocks_rows(const float* scores, int* idx, int B, int Hkv, int N, int NB, int k,
                                    cudaStream_t s);
cudaError_t launch_topk_tokens(const PrefillDims& d, const float* scores, int k_tokens, int forced,
                               int* idx, cudaStream_t s);
cudaError_t launch_topk_decode_tokens(const float* scores, int* idx, int B, int Hkv, int L, int k_tokens, int forced,
                                      const int* seqlens, cudaStream_t s);

// ---- sparse layer ----------------------------------------------------------------------------
cudaError_t launch_sparse_attn_simt(const PrefillDims& d, hys_dtype dt, const void* q, const void* k,
                                    const void* v, const int* idx, int kb, const void* ks,
                                    const void* vs, int window, const float* gate, const float* sinks, void* o,
                                    cudaStream_t s, float* blse = nullptr, void* osp = nullptr);
cudaError_t launch_sparse_tokens_simt(const PrefillDims& d, hys_dtype dt, const void* q, const void* k,
                                      const void* v, const int* idx, int kt, int forced, void* o,
                                      cudaStream_t s);

bool sparse_attn_tc_supported(const PrefillDims& d, hys_dtype dt);
size_t sparse_attn_tc_workspace(const PrefillDims& d);
// per_row: idx is [B,Hkv,N,kb], one block list per query position (NB <= 512)
bool sparse_attn_rows_tc_supported(const PrefillDims& d, hys_dtype dt);
// blse / osp (training forward, per-tile selection only): [B,Hq,N,2] branch LSEs and [B,Hq,N,D] the
// gated sparse-branch part sigmoid(g0) o~
cudaError_t launch_sparse_attn_tc(const PrefillDims& d, const void* q, const void* k, const void* v, const int* idx,
                                  int kb, const void* ks, const void* vs, int window, const float* gate,
                                  const float* sinks, void* o, void* ws, size_t ws_bytes, cudaStream_t s,
                                  bool per_row = false, float* blse = nullptr, void* osp = nullptr);

// ---- backward (tcgen05, key-major; bf16, D = 128, even G) ----------------------------------
bool attn_bwd_tc_supported(const PrefillDims& d, hys_dtype dt);
size_t full_bwd_tc_workspace(const PrefillDims& d);
// full layer: dq (bf16) from lse [B,Hq,N] and o; dk, dv fp32, overwritten or (accumulate) added to
cudaError_t launch_full_bwd_tc(const PrefillDims& d, const void* q, const void* k, const void* v, const void* o,
                               const void* d_o, const float* lse, void* dq, float* dk, float* dv, int accumulate,
                               void* ws, cudaStream_t s);
// one key set of a sparse layer into the fp32 dq accumulator: the window over K', V' (dk, dv
// overwritten) or the selected blocks over the shared K, V (dk, dv added to; list/list_cnt per
// (b, g, 128-key tile): query tiles << 2 | block-half mask).  lse2 in log2 units, dsum = D_t,
// sig = the branch's gate sigma_t per row
cudaError_t launch_attn_bwd_tc_window(const PrefillDims& d, const void* q, const void* d_o, const void* k,
                                      const void* v, const float* lse2, const float* dsum, const float* sig,
                                      float* dq_acc, float* dk, float* dv, int window, int* counter, cudaStream_t s);
cudaError_t launch_attn_bwd_tc_sparse(const PrefillDims& d, const void* q, const void* d_o, const void* k,
                                      const void* v, const float* lse2, const float* dsum, const float* sig,
                                      float* dq_acc, float* dk, float* dv, const int* list, const int* list_cnt,
                                      int* counter, cudaStream_t s);
// dq (bf16) = acc / sqrt(128); n a multiple of 8
cudaError_t launch_bwd_dq_out(const float* acc, void* dq, size_t n, cudaStream_t s);

// ---- backward, any supported dtype / D / G (tcgen05 where it applies, SIMT otherwise) --------
size_t full_bwd_workspace(const PrefillDims& d, hys_dtype dt);
cudaError_t launch_full_bwd(const PrefillDims& d, hys_dtype dt, const void* q, const void* k, const void* v,
                            const void* o, const void* d_o, const float* lse, void* dq, float* dk, float* dv,
                            int accumulate, void* ws, cudaStream_t s);
size_t sparse_bwd_workspace(const PrefillDims& d);
cudaError_t launch_sparse_bwd(const PrefillDims& d, hys_dtype dt, const void* q, const void* k, const void* v,
                              const int* idx, int kb, const void* ks, const void* vs, int window, const float* gate,
                              const float* sinks, const void* o, const void* osp, const float* blse, const void* d_o,
                              void* dq, float* dk, float* dv, float* dks, float* dvs, float* dgate, float* dsinks,
                              void* ws, cudaStream_t s);

// ---- decode ----------------------------------------------------------------------------------
size_t decode_full_workspace(const DecodeDims& d);
cudaError_t launch_decode_full(const DecodeDims& d, hys_dtype dt, const void* q, const void* kc,
                               const void* vc, const int* seqlens, void* o, float* scores,
                               hys_reduce red, void* ws, cudaStream_t s);
cudaError_t launch_decode_sparse(const DecodeDims& d, hys_dtype dt, const void* q, const void* kc,
                                 const void* vc, const int* seqlens, const int* idx, int kb,
                                 const void* kr, const void* vr, int W, const int* swa_len,
                                 const float* gate, const float* sinks, void* o, cudaStream_t s);

// bf16, D = 128, G <= 16: tensor-core split-KV kernels
bool decode_mma_supported(const DecodeDims& d, hys_dtype dt);
size_t decode_mma_full_workspace(const DecodeDims& d);
size_t decode_mma_sparse_workspace(const DecodeDims& d, int kb);
cudaError_t launch_decode_full_mma(const DecodeDims& d, const void* q, const void* kc, const void* vc,
                                   const int* seqlens, void* o, float* scores, hys_reduce red, void* ws,
                                   cudaStream_t s);
// token-variant decode (bf16, D = 128, G <= 16)
size_t decode_mma_full_tokens_workspace(const DecodeDims& d);
cudaError_t launch_decode_full_tokens_mma(const DecodeDims& d, const void* q, const void* kc, const void* vc,
                                          const int* seqlens, void* o, float* tok_scores, void* ws, cudaStream_t s);
size_t decode_mma_sparse_tokens_workspace(const DecodeDims& d, int kt);
cudaError_t launch_decode_sparse_tokens_mma(const DecodeDims& d, const void* q, const void* kc, const void* vc,
                                            const int* seqlens, const int* idx, int kt, int forced, void* o, void* ws,
                                            cudaStream_t s);
// FP8 (E4M3) cache variants of the token-variant decode: k_cache/v_cache hold codes, value =
// code * scale[g] with k_scale/v_scale [Hkv]; workspaces as for the bf16 calls
cudaError_t launch_decode_full_tokens_mma_fp8(const DecodeDims& d, const void* q, const void* kc, const void* vc,
                                              const float* k_scale, const float* v_scale, const int* seqlens, void* o,
                                              float* tok_scores, void* ws, cudaStream_t s);
cudaError_t launch_decode_sparse_tokens_mma_fp8(const DecodeDims& d, const void* q, const void* kc, const void* vc,
                                                const float* k_scale, const float* v_scale, const int* seqlens,
                                                const int* idx, int kt, int forced, void* o, void* ws, cudaStream_t s);
cudaError_t launch_decode_sparse_mma(const DecodeDims& d, const void* q, const void* kc, const void* vc,
                                     const int* seqlens, const int* idx, int kb, const void* kr, const void* vr, int W,
                                     const int* swa_len, const float* gate, const float* sinks, void* o, void* ws,
                                     cudaStream_t s);

}  // namespace hys
