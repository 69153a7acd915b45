/*
 * hysparse.h -- C ABI of the HySparse hybrid-block attention hot path (B200, sm_100a).
 *
 * Sources of the operations (cited per entry point below):
 *   [HS]  "HySparse: A Hybrid Sparse Attention Architecture with Oracle Token Selection
 *         and KV Cache Sharing" (paper-graph long-form summary), section 3.4.1 (full
 *         attention o_t, block-level max score S_t^i, two-pass rescale, GQA aggregation),
 *         3.4.2 (TopK block selection), 3.4.3 (gather, sparse branch, SWA branch,
 *         sigmoid gated fusion), 3.4.4 (cross-layer KV sharing).
 *   [HS2] HySparse2 explainer (deep-reads): "Precise retrieval without a separate
 *         indexer" (token-level selection, newest 128 tokens forced in) and "Twenty
 *         lines of algorithmic intuition" (decode step).
 *
 * Conventions shared by every entry point
 *   - Every pointer argument is a DEVICE pointer owned by the caller, unless stated.
 *     The library never allocates device memory inside a call; scratch memory comes
 *     from a caller-provided workspace whose size the matching *_workspace_size()
 *     query returns (a NULL workspace with size 0 is accepted when the query says 0).
 *   - Work is enqueued asynchronously on the caller's CUDA stream; no call
 *     synchronises the host.  Inputs must stay valid until the work completes.
 *   - Tensors are contiguous row-major:
 *        Q, O (prefill)            [B, Hq, N, D]
 *        K, V, K', V' (prefill)    [B, Hkv, N, D]
 *        gate logits (prefill)     [B, Hq, N, 2] fp32 (index 0: sparse branch, 1: SWA)
 *        block scores              [B, Hkv, T, NB] fp32, T = NB = ceil(N / block)
 *        token scores              [B, Hkv, T, N] fp32
 *        block indices             [B, Hkv, T, k] int32, ascending, padded with -1
 *        token indices             [B, Hkv, T, k_tokens] int32, ascending, padded with -1
 *     Query head h reads KV head h / (Hq / Hkv) (grouped-query attention).
 *   - Element type: HYS_BF16 or HYS_F32 for Q/K/V/O (outputs take the input type);
 *     arithmetic accumulates in fp32.  Scores are always fp32.
 *   - block must be 64; D must be 64 or 128; Hq % Hkv == 0; every pointer 16-byte
 *     aligned.  Violations return HYS_ERR_INVALID_ARG and launch nothing.
 *   - No exception crosses the ABI.  A CUDA launch error returns HYS_ERR_CUDA.
 *     Kernels whose waits are bounded record HYS_ERR_TIMEOUT in a device status
 *     word that hysparse_get_device_status() reads.
 */
#ifndef HYSPARSE_H_
#define HYSPARSE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HYS_API __attribute__((visibility("default")))
#else
#define HYS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* hys_stream_t; /* same type as cudaStream_t; NULL = legacy default stream */

typedef enum {
  HYS_OK = 0,
  HYS_ERR_INVALID_ARG = 1,
  HYS_ERR_UNSUPPORTED = 2,
  HYS_ERR_CUDA = 3,
  HYS_ERR_TIMEOUT = 4,
  HYS_ERR_WORKSPACE = 5 /* workspace missing or smaller than the size query returned */
} hys_status;

typedef enum { HYS_F32 = 0, HYS_BF16 = 1 } hys_dtype;

/* Granularity of the importance scores the full layer emits. */
typedef enum { HYS_GRAN_BLOCK = 0, HYS_GRAN_TOKEN = 1, HYS_GRAN_BLOCK_ROW = 2 } hys_gran;

/* Aggregation R over the query heads of a KV group and the rows of a 64-query tile.
 * SUM is the default; MAX is the paper's conservative group-wise maximum. */
typedef enum { HYS_REDUCE_SUM = 0, HYS_REDUCE_MAX = 1 } hys_reduce;

typedef struct {
  int B;     /* batch */
  int N;     /* sequence length, >= 1 */
  int Hq;    /* query heads */
  int Hkv;   /* key/value heads, divides Hq */
  int D;     /* head dim, 64 or 128 */
  int block; /* KV block = query tile = 64 */
} hys_shape;

typedef struct {
  int B;     /* sequences */
  int L;     /* cache capacity per sequence (tokens), >= 1 */
  int Hq;
  int Hkv;
  int D;
  int block; /* 64 */
} hys_decode_shape;

/* Library version as "major.minor.patch". Host pointer, static storage. */
HYS_API const char* hysparse_version(void);

/* Human-readable name of a status code. Host pointer, static storage. */
HYS_API const char* hysparse_status_string(hys_status s);

/* Reads (and with reset != 0 clears) the device status word of the current device:
 * HYS_OK, or HYS_ERR_TIMEOUT when a bounded wait inside a kernel ran out.
 * *out is a HOST pointer. Synchronises the given stream. */
HYS_API hys_status hysparse_get_device_status(hys_stream_t stream, int reset, int* out);

/* ------------------------------------------------------------------------------------
 * Full attention layer with fused importance scores.
 *
 * o_t = sum_{i<=t} softmax_i(tau q_t.k_i) v_i, tau = 1/sqrt(D)            [HS] 3.4.1, o_t
 *
 * gran = HYS_GRAN_BLOCK: scores [B,Hkv,T,NB] with
 *   scores[b,g,I,j] = R_{h in g} R_{t in tile I} S^h_{t,j}   for j <= I, 0 for j > I,
 *   S^h_{t,j} = max over keys i of block j with i <= t of the probability P^h_{t,i}
 *   ([HS] 3.4.1, S_t^i and the two-pass rescale exp(m~ - m)/l; GQA aggregation with R
 *   = sum (default) or max).
 * gran = HYS_GRAN_TOKEN: scores [B,Hkv,T,N] with
 *   scores[b,g,I,i] = sum_{h in g} sum_{t in tile I, t >= i} P^h_{t,i}   ([HS2], token
 *   selection; red must be HYS_REDUCE_SUM).
 * gran = HYS_GRAN_BLOCK_ROW: scores [B,Hkv,N,NB] per query position with
 *   scores[b,g,t,j] = max_{h in g} S^h_{t,j}   for j <= floor(t/64), 0 beyond
 *   ([HS] 3.4.1 group-wise maximum per (query position, key block) entry; 3.4.2 selection
 *   per query position).  red must be HYS_REDUCE_MAX; bf16 with D in {64, 128}, an even
 *   group size and NB <= 2048 (N <= 131072) only (HYS_ERR_UNSUPPORTED otherwise).  The
 *   workspace is the HYS_GRAN_BLOCK one.
 * lse_opt: NULL or [B,Hq,N] fp32, receives LSE_t = log sum_i exp(tau q_t.k_i).
 * ------------------------------------------------------------------------------------ */
HYS_API hys_status hysparse_full_attn_select_workspace_size(const hys_shape* shape, hys_dtype dtype,
                                                    hys_gran gran, size_t* bytes);
HYS_API hys_status hysparse_full_attn_select(const hys_shape* shape, hys_dtype dtype, const void* q,
                                     const void* k, const void* v, void* o, float* scores,
                                     hys_gran gran, hys_reduce red, float* lse_opt,
                                     void* workspace, size_t workspace_bytes,
                                     hys_stream_t stream);

/* ------------------------------------------------------------------------------------
 * TopK block selection ([HS] 3.4.2).  For each (b, g, I) the k largest of
 * scores[b,g,I,0..I] (I+1 candidates), ties to the lower block index; fewer than k
 * candidates selects all of them.  idx [B,Hkv,T,k] int32, ascending, padded with -1.
 * 1 <= k <= 1024.  No workspace.
 * ------------------------------------------------------------------------------------ */
HYS_API hys_status hysparse_topk(const hys_shape* shape, const float* scores, int k, int* idx,
                         hys_stream_t stream);

/* Per-position TopK ([HS] 3.4.2, for each query position t and group): the k largest of
 * scores[b,g,t,0..floor(t/64)] from HYS_GRAN_BLOCK_ROW, ties to the lower block index,
 * fewer candidates than k selects all; idx [B,Hkv,N,k] int32, ascending, padded with -1.
 * 1 <= k <= 1024, NB <= 8192.  No workspace. */
HYS_API hys_status hysparse_topk_rows(const hys_shape* shape, const float* scores, int k, int* idx,
                              hys_stream_t stream);

/* ------------------------------------------------------------------------------------
 * TopK token selection with a forced recent window ([HS2]).  Candidates of tile I are
 * positions [0, e_I - forced_window], e_I = min(64I+63, N-1); the k_tokens largest of
 * scores[b,g,I,i] over them, ties to the lower position; ascending, padded with -1.
 * The forced window is not part of the budget.  1 <= k_tokens <= 16384.
 * ------------------------------------------------------------------------------------ */
HYS_API hys_status hysparse_topk_tokens_workspace_size(const hys_shape* shape, int k_tokens,
                                               size_t* bytes);
HYS_API hys_status hysparse_topk_tokens(const hys_shape* shape, const float* tok_scores, int k_tokens,
                                int forced_window, int* idx, void* workspace,
                                size_t workspace_bytes, hys_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Sparse layer: block-sparse branch + sliding-window branch + sigmoid gate
 * ([HS] 3.4.3, the gather K~,V~ = concat of the selected blocks, o~_t, o'_t, and
 * o_t = sigmoid(g0) o~_t + sigmoid(g1) o'_t).
 *   Row t of tile I attends {i <= t : floor(i/64) in idx[b,g,I,:]} of the shared K, V
 *   (the full layer's cache, [HS] 3.4.4) and [max(0, t-window+1), t] of its own K', V'.
 *   k_swa/v_swa may alias k_shared/v_shared (the "share both" ablation).
 *   idx entries are ascending block ids <= I or -1 (ignored); 1 <= k <= 1024.
 *   sinks: NULL, or [Hq, 2] fp32 per-head sink logits ([HSP] 4.1: per-head learnable sink
 *   biases in the sparse and sliding-window branches, as in gpt-oss), index 0 for the sparse
 *   branch and 1 for the window branch, in the units of the scaled logits tau q.k: each joins
 *   its branch's softmax as an entry with a zero value (the denominator gains exp(sink - m)).
 *   workspace: at least hysparse_sparse_attn_workspace_size() bytes (the tensor-core kernel's
 *   work-unit counter; no scratch rows: both branches accumulate into one output tile).
 * ------------------------------------------------------------------------------------ */
HYS_API hys_status hysparse_sparse_attn_workspace_size(const hys_shape* shape, hys_dtype dtype,
                                                     size_t* bytes);
HYS_API hys_status hysparse_sparse_attn(const hys_shape* shape, hys_dtype dtype, const void* q_sparse,
                                const void* k_shared, const void* v_shared, const int* idx,
                                int k, const void* k_swa, const void* v_swa, int window,
                                const float* gate_logits, const float* sinks, void* o,
                                void* workspace, size_t workspace_bytes, hys_stream_t stream);

/* The sparse layer with per-position selection ([HS] 3.4.2 'computed per query position'):
 * as hysparse_sparse_attn, but idx is [B,Hkv,N,k] and row t's sparse branch attends
 * {i <= t : floor(i/64) in idx[b,g,t,:]} (entries past floor(t/64) and -1 are ignored).
 * bf16 with D in {64, 128}, an even group size, k <= 256 and N <= 32768 only
 * (HYS_ERR_UNSUPPORTED otherwise).  workspace: hysparse_sparse_attn_workspace_size() bytes. */
HYS_API hys_status hysparse_sparse_attn_rows(const hys_shape* shape, hys_dtype dtype, const void* q_sparse,
                                     const void* k_shared, const void* v_shared, const int* idx,
                                     int k, const void* k_swa, const void* v_swa, int window,
                                     const float* gate_logits, const float* sinks, void* o,
                                     void* workspace, size_t workspace_bytes, hys_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Training: the sparse layer's forward with saved statistics, and the backward of the full
 * and sparse layers ([HS] 3.4.6, training pipeline: no auxiliary loss for the selection, the
 * selected indices are constants of the step; the sparse layers' gradients reach the full
 * layer's K and V through the shared cache of 3.4.4).  Gradients of attention over a key set
 * with p = softmax(tau q.k) and o = sum_i p_i v_i: dV_i = sum_t p_ti dO_t, dK_i = tau sum_t
 * dS_ti q_t, dQ_t = tau sum_i dS_ti k_i, dS_ti = p_ti (dO_t.v_i - dO_t.o_t); for the gated layer
 * ([HS] 3.4.3) each branch b sees dO scaled by sigmoid(g_b), and d g_b = sigmoid(g_b)
 * (1 - sigmoid(g_b)) dO.o_b; a sink logit's gradient is -sum_t p_sink,t sigmoid(g_b) dO_t.o_b,t.
 * Key and value gradients are fp32 (they are sums over layers and heads); dq takes the input
 * type.  bf16 with D = 128 and an even group size runs on the tensor cores (key-major tcgen05
 * kernel, dQ accumulated in fp32 by TMA reduce-adds); other shapes and fp32 run SIMT
 * fp32-accumulate kernels.
 * ------------------------------------------------------------------------------------ */

/* The sparse layer of a training step: hysparse_sparse_attn (same arguments, limits and
 * workspace) that also saves
 *   o_sparse    [B,Hq,N,D] input type: the gated sparse-branch part sigmoid(g0) o~ of o;
 *   branch_lse  [B,Hq,N,2] fp32: log of each branch's softmax normaliser in units of the
 *               scaled logits, LSE = log(sum_i exp(tau q.k_i) + exp(sink)), index 0 the sparse
 *               branch and 1 the window branch (a branch without keys: the sink, or -inf). */
HYS_API hys_status hysparse_sparse_attn_train(const hys_shape* shape, hys_dtype dtype, const void* q_sparse,
                                              const void* k_shared, const void* v_shared, const int* idx, int k,
                                              const void* k_swa, const void* v_swa, int window,
                                              const float* gate_logits, const float* sinks, void* o, void* o_sparse,
                                              float* branch_lse, void* workspace, size_t workspace_bytes,
                                              hys_stream_t stream);

/* Backward of the full layer (causal GQA attention, [HS] 3.4.1).  Inputs q, k, v, o and the
 * output gradient d_o as for hysparse_full_attn_select, lse [B,Hq,N] fp32 the forward's lse_opt.
 * Outputs: dq [B,Hq,N,D] (input type); dk, dv [B,Hkv,N,D] fp32, summed over the group's heads,
 * overwritten (accumulate_kv == 0) or added to (accumulate_kv != 0).  workspace: at least
 * hysparse_full_attn_backward_workspace_size() bytes. */
HYS_API hys_status hysparse_full_attn_backward_workspace_size(const hys_shape* shape, hys_dtype dtype,
                                                              size_t* bytes);
HYS_API hys_status hysparse_full_attn_backward(const hys_shape* shape, hys_dtype dtype, const void* q, const void* k,
                                               const void* v, const void* o, const void* d_o, const float* lse,
                                               void* dq, float* dk, float* dv, int accumulate_kv, void* workspace,
                                               size_t workspace_bytes, hys_stream_t stream);

/* Backward of one sparse layer (per-tile selection, [HS] 3.4.3).  Inputs as for
 * hysparse_sparse_attn_train, plus its outputs o, o_sparse and branch_lse, and d_o [B,Hq,N,D].
 * Outputs:
 *   dq                 [B,Hq,N,D] input type, both branches;
 *   dk_shared,
 *   dv_shared          [B,Hkv,N,D] fp32, the sparse branch's gradient of the shared cache, ADDED
 *                      to the buffers (pass the full layer's gradient, or zeros, and call the
 *                      block's sparse layers one after another to sum the block);
 *   dk_swa, dv_swa     [B,Hkv,N,D] fp32, the window branch's gradient of K', V', overwritten;
 *   dgate              [B,Hq,N,2] fp32, overwritten;
 *   dsinks             [Hq,2] fp32 (required when sinks is given, else ignored), overwritten.
 * The gradient buffers must not alias one another (inputs may: K'/V' may be K/V).  workspace:
 * at least hysparse_sparse_attn_backward_workspace_size() bytes. */
HYS_API hys_status hysparse_sparse_attn_backward_workspace_size(const hys_shape* shape, hys_dtype dtype,
                                                                size_t* bytes);
HYS_API hys_status hysparse_sparse_attn_backward(const hys_shape* shape, hys_dtype dtype, const void* q_sparse,
                                                 const void* k_shared, const void* v_shared, const int* idx, int k,
                                                 const void* k_swa, const void* v_swa, int window,
                                                 const float* gate_logits, const float* sinks, const void* o,
                                                 const void* o_sparse, const float* branch_lse, const void* d_o,
                                                 void* dq, float* dk_shared, float* dv_shared, float* dk_swa,
                                                 float* dv_swa, float* dgate, float* dsinks, void* workspace,
                                                 size_t workspace_bytes, hys_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Token-sparse layer ([HS2]): row t of tile I attends idx[b,g,I,:] (token positions,
 * ascending, -1 padded, all <= t) united with [max(0, t-forced_window+1), t], each
 * token once, over the shared K, V; no gate.  sinks must be NULL.  workspace: at least
 * hysparse_sparse_attn_tokens_workspace_size() bytes.
 * ------------------------------------------------------------------------------------ */
HYS_API hys_status hysparse_sparse_attn_tokens_workspace_size(const hys_shape* shape, hys_dtype dtype,
                                                            int forced_window, size_t* bytes);
HYS_API hys_status hysparse_sparse_attn_tokens(const hys_shape* shape, hys_dtype dtype,
                                       const void* q_sparse, const void* k_shared,
                                       const void* v_shared, const int* idx, int k_tokens,
                                       int forced_window, const float* sinks, void* o,
                                       void* workspace, size_t workspace_bytes, hys_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Decode, full layer ([HS2] decode step; [HS] 3.4.1).  One new token per sequence at
 * position L_b - 1 of its cache (L_b = seqlens[b], or L when seqlens is NULL).
 *   q [B,Hq,D]; k_cache, v_cache [B,Hkv,L,D]; o [B,Hq,D];
 *   scores [B,Hkv,NB] fp32, NB = ceil(L/64): R_{h in g} S^h_j, 0 past the sequence end.
 *   seqlens: NULL or [B] int32 in [1, L].
 * ------------------------------------------------------------------------------------ */
HYS_API hys_status hysparse_full_attn_select_decode_workspace_size(const hys_decode_shape* shape,
                                                           hys_dtype dtype, size_t* bytes);
HYS_API hys_status hysparse_full_attn_select_decode(const hys_decode_shape* shape, hys_dtype dtype,
                                            const void* q, const void* k_cache,
                                            const void* v_cache, const int* seqlens, void* o,
                                            float* scores, hys_reduce red, void* workspace,
                                            size_t workspace_bytes, hys_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Allocation-free decode full layer.  The paper has no counterpart: this entry point
 * exists for callers that cannot allocate device memory when they run a decode step
 * (an engine that plans all of its device memory up front and forbids later
 * cudaMalloc, which may synchronise the device; a host integration with no
 * allocator).  Same operation, arguments and layouts as
 * hysparse_full_attn_select_decode, minus the workspace: the split-KV scratch lives in
 * a fixed 16 MiB array inside the library, held in device memory by every GPU that
 * loads the library until the process exits.
 *   - Shapes whose scratch (the value hysparse_full_attn_select_decode_workspace_size
 *     returns) exceeds 16 MiB return HYS_ERR_WORKSPACE and launch nothing.
 *   - The call makes no cudaMalloc/cudaFree and no allocating library call.
 *   - The first call on a device is the set-up: with that device current it resolves the
 *     array's device address, and under the CUDA driver's lazy module loading (the default)
 *     that is also when the driver loads the array onto the device, so this first call may
 *     allocate the array's 16 MiB and synchronise.  Make it during set-up, before any
 *     stream capture; later calls on that device allocate nothing.
 *   - All calls share the one array: calls whose work overlaps on the GPU (different
 *     streams, or different host threads on the same device) race and must be ordered
 *     by the caller.  Nothing in the array needs clearing between calls.
 * ------------------------------------------------------------------------------------ */
HYS_API hys_status hysparse_full_attn_select_decode_noalloc(const hys_decode_shape* shape,
                                                          hys_dtype dtype, const void* q,
                                                          const void* k_cache, const void* v_cache,
                                                          const int* seqlens, void* o, float* scores,
                                                          hys_reduce red, hys_stream_t stream);

/* TopK over the decode scores: idx [B,Hkv,k]; candidates are the blocks holding
 * cached tokens (ceil(L_b/64)); ties to the lower index; ascending, -1 padded. */
HYS_API hys_status hysparse_topk_decode(const hys_decode_shape* shape, const float* scores, int k,
                                const int* seqlens, int* idx, hys_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Decode, sparse layer ([HS] 3.4.3 for one query row).  The sparse branch attends every
 * cached token (< L_b) of the selected blocks of the shared cache; the SWA branch attends
 * the layer's own ring k_swa_ring/v_swa_ring [B,Hkv,W,D] (swa_len[b] valid entries, or W
 * when swa_len is NULL; order is irrelevant); gate_logits [B,Hq,2]; o [B,Hq,D].
 * W = window, 1 <= window <= 1024.  sinks: NULL or [Hq, 2] fp32 sink logits, as for
 * hysparse_sparse_attn.  workspace: at least
 * hysparse_sparse_attn_decode_workspace_size() bytes (per-split partial softmax states).
 * ------------------------------------------------------------------------------------ */
HYS_API hys_status hysparse_sparse_attn_decode_workspace_size(const hys_decode_shape* shape,
                                                            hys_dtype dtype, int k, size_t* bytes);
HYS_API hys_status hysparse_sparse_attn_decode(const hys_decode_shape* shape, hys_dtype dtype,
                                       const void* q, const void* k_cache,
                                       const void* v_cache, const int* seqlens,
                                       const int* idx, int k, const void* k_swa_ring,
                                       const void* v_swa_ring, int window, const int* swa_len,
                                       const float* gate_logits, const float* sinks, void* o,
                                       void* workspace, size_t workspace_bytes, hys_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Token-variant decode ([HS2] "Twenty lines of algorithmic intuition", with the token
 * granularity of "Precise retrieval without a separate indexer").  bf16, D = 128 and
 * Hq/Hkv <= 16 (the tensor-core decode path); other shapes and types return
 * HYS_ERR_UNSUPPORTED.
 *
 * hysparse_full_attn_select_decode_tokens: the full layer for the new token (position
 *   L_b - 1 of an L_b-token cache), o [B,Hq,D], and its token scores tok_scores [B,Hkv,L]
 *   fp32: score[b,g,i] = sum over the group's heads of the new token's attention probability
 *   of cached token i (0 for i >= L_b).  workspace: at least
 *   hysparse_full_attn_select_decode_tokens_workspace_size() bytes (per-split partial softmax
 *   states and every key's logit, B*Hq*L fp32).
 * hysparse_topk_decode_tokens: idx [B,Hkv,k_tokens] int32, the k_tokens highest scores among
 *   the tokens older than the forced newest window, positions [0, L_b - 1 - forced_window];
 *   ties to the lower position; ascending, padded with -1.  1 <= k_tokens <= 16384.
 * hysparse_sparse_attn_decode_tokens: the token-sparse layer for the new token: the selected
 *   cached tokens idx[b,g,:] (entries outside [0, L_b - 1 - forced_window] are ignored) united
 *   with the newest forced_window tokens [L_b - forced_window, L_b - 1], each token once, over
 *   the shared cache; no gate.  1 <= forced_window <= 4096.  workspace: at least
 *   hysparse_sparse_attn_decode_tokens_workspace_size() bytes.
 * ------------------------------------------------------------------------------------ */
HYS_API hys_status hysparse_full_attn_select_decode_tokens_workspace_size(const hys_decode_shape* shape,
                                                                      hys_dtype dtype, size_t* bytes);
HYS_API hys_status hysparse_full_attn_select_decode_tokens(const hys_decode_shape* shape, hys_dtype dtype,
                                                       const void* q, const void* k_cache,
                                                       const void* v_cache, const int* seqlens, void* o,
                                                       float* tok_scores, void* workspace,
                                                       size_t workspace_bytes, hys_stream_t stream);
HYS_API hys_status hysparse_topk_decode_tokens(const hys_decode_shape* shape, const float* tok_scores,
                                           int k_tokens, int forced_window, const int* seqlens, int* idx,
                                           hys_stream_t stream);
HYS_API hys_status hysparse_sparse_attn_decode_tokens_workspace_size(const hys_decode_shape* shape,
                                                                 hys_dtype dtype, int k_tokens,
                                                                 size_t* bytes);
HYS_API hys_status hysparse_sparse_attn_decode_tokens(const hys_decode_shape* shape, hys_dtype dtype,
                                                  const void* q, const void* k_cache,
                                                  const void* v_cache, const int* seqlens,
                                                  const int* idx, int k_tokens, int forced_window,
                                                  void* o, void* workspace, size_t workspace_bytes,
                                                  hys_stream_t stream);


/* ------------------------------------------------------------------------------------
 * Token-variant decode over an FP8 KV cache (HySparse2 explainer, "What actually improved?":
 * the cache is sized in FP8).  The pages fix neither the FP8 format nor its scaling; these
 * calls take OCP E4M3 codes ("fn" variant: bias 7, no infinities) with one float32 scale per
 * KV head for K and one for V: the cached value is code * scale[g].
 *
 * Same operations, layouts, limits and errors as hysparse_full_attn_select_decode_tokens and
 * hysparse_sparse_attn_decode_tokens, with:
 *   q, o         [B,Hq,128] bf16 (D = 128 and G <= 16 only; other shapes: HYS_ERR_UNSUPPORTED);
 *   k_cache,
 *   v_cache      [B,Hkv,L,128] E4M3 codes, one byte each, 16-byte aligned;
 *   k_scale,
 *   v_scale      [Hkv] float32 device arrays, 4-byte aligned, finite and positive;
 *   workspace    sized by the bf16 queries (hysparse_full_attn_select_decode_tokens_workspace_size
 *                / hysparse_sparse_attn_decode_tokens_workspace_size with HYS_BF16).
 * Token scores are the probabilities under the scaled logits, exactly as for a bf16 cache
 * holding the decoded values; hysparse_topk_decode_tokens selects from them unchanged.
 * ------------------------------------------------------------------------------------ */
HYS_API hys_status hysparse_full_attn_select_decode_tokens_fp8(const hys_decode_shape* shape, const void* q,
                                                           const void* k_cache, const void* v_cache,
                                                           const float* k_scale, const float* v_scale,
                                                           const int* seqlens, void* o, float* tok_scores,
                                                           void* workspace, size_t workspace_bytes,
                                                           hys_stream_t stream);
HYS_API hys_status hysparse_sparse_attn_decode_tokens_fp8(const hys_decode_shape* shape, const void* q,
                                                      const void* k_cache, const void* v_cache,
                                                      const float* k_scale, const float* v_scale,
                                                      const int* seqlens, const int* idx, int k_tokens,
                                                      int forced_window, void* o, void* workspace,
                                                      size_t workspace_bytes, hys_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HYSPARSE_H_ */
