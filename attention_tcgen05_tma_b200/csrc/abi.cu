// C ABI of the HySparse hot path: argument validation, workspace carving and dispatch.
// Every entry point enqueues on the caller's stream and never allocates.
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tma_host.h"

namespace hys {
__device__ int g_device_status = 0;

// Device address of g_device_status on the current device, resolved once per device under a
// lock (host threads may make their first calls concurrently).
int* device_status_ptr() {
  static std::mutex mu;
  static int* cached[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!cached[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    cached[dev] = static_cast<int*>(p);
  }
  return cached[dev];
}

EncodeTiledFn tma_encode_fn() {
  // a function-local static is initialised exactly once, even under concurrent first calls
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(ptr);
    return nullptr;
  }();
  return fn;
}
}  // namespace hys

using namespace hys;

namespace {

constexpr int kBlock = 64;

bool aligned16(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

hys_status check_prefill(const hys_shape* s, PrefillDims* d) {
  if (!s) return HYS_ERR_INVALID_ARG;
  if (s->B <= 0 || s->N <= 0 || s->Hq <= 0 || s->Hkv <= 0) return HYS_ERR_INVALID_ARG;
  if (s->Hq % s->Hkv != 0) return HYS_ERR_INVALID_ARG;
  if (s->D != 64 && s->D != 128) return HYS_ERR_INVALID_ARG;
  if (s->block != kBlock) return HYS_ERR_INVALID_ARG;
  if (s->N > (1 << 20)) return HYS_ERR_UNSUPPORTED;
  if (s->Hq / s->Hkv > 64) return HYS_ERR_UNSUPPORTED;
  d->B = s->B;
  d->N = s->N;
  d->Hq = s->Hq;
  d->Hkv = s->Hkv;
  d->D = s->D;
  d->T = (s->N + kBlock - 1) / kBlock;
  d->NB = d->T;
  return HYS_OK;
}

hys_status check_decode(const hys_decode_shape* s, DecodeDims* d) {
  if (!s) return HYS_ERR_INVALID_ARG;
  if (s->B <= 0 || s->L <= 0 || s->Hq <= 0 || s->Hkv <= 0) return HYS_ERR_INVALID_ARG;
  if (s->Hq % s->Hkv != 0) return HYS_ERR_INVALID_ARG;
  if (s->D != 64 && s->D != 128) return HYS_ERR_INVALID_ARG;
  if (s->block != kBlock) return HYS_ERR_INVALID_ARG;
  if (s->Hq / s->Hkv > 16) return HYS_ERR_UNSUPPORTED;
  if (s->L > (1 << 23)) return HYS_ERR_UNSUPPORTED;
  d->B = s->B;
  d->L = s->L;
  d->Hq = s->Hq;
  d->Hkv = s->Hkv;
  d->D = s->D;
  d->NB = (s->L + kBlock - 1) / kBlock;
  return HYS_OK;
}

bool dtype_ok(hys_dtype dt) { return dt == HYS_F32 || dt == HYS_BF16; }

hys_status from_cuda(cudaError_t e) { return e == cudaSuccess ? HYS_OK : HYS_ERR_CUDA; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace of hysparse_full_attn_select.  Block scores: the tensor-core kernel's counter and
// m~ stash, or the SIMT path's per-head partial scores.  Token scores: the tensor-core
// kernel's counter (256 B) followed by room for the LSE of every row (used when the caller
// passes no lse buffer).
size_t full_ws_bytes(const PrefillDims& d, hys_dtype dt, hys_gran gran) {
  if (gran == HYS_GRAN_TOKEN) return 256 + align256(sizeof(float) * (size_t)d.B * d.Hq * d.N);
  if (full_attn_tc_supported(d, dt, true)) return align256(full_attn_tc_workspace(d, true));
  return align256(sizeof(float) * (size_t)d.B * d.Hq * d.T * d.NB);
}

}  // namespace

extern "C" {

const char* hysparse_version(void) { return "0.1.0"; }

const char* hysparse_status_string(hys_status s) {
  switch (s) {
    case HYS_OK: return "HYS_OK";
    case HYS_ERR_INVALID_ARG: return "HYS_ERR_INVALID_ARG";
    case HYS_ERR_UNSUPPORTED: return "HYS_ERR_UNSUPPORTED";
    case HYS_ERR_CUDA: return "HYS_ERR_CUDA";
    case HYS_ERR_TIMEOUT: return "HYS_ERR_TIMEOUT";
    case HYS_ERR_WORKSPACE: return "HYS_ERR_WORKSPACE";
  }
  return "HYS_ERR_UNKNOWN";
}

hys_status hysparse_get_device_status(hys_stream_t stream, int reset, int* out) {
  if (!out) return HYS_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_device_status, sizeof(int), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return HYS_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return HYS_ERR_CUDA;
  if (reset) {
    const int zero = 0;
    if (cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s) != cudaSuccess)
      return HYS_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return HYS_ERR_CUDA;
  }
  *out = v;
  return HYS_OK;
}

// ----------------------------------------------------------------------------- full layer
hys_status hysparse_full_attn_select_workspace_size(const hys_shape* shape, hys_dtype dtype, hys_gran gran,
                                                    size_t* bytes) {
  PrefillDims d;
  hys_status st = check_prefill(shape, &d);
  if (st != HYS_OK) return st;
  if (!bytes || !dtype_ok(dtype) || (gran != HYS_GRAN_BLOCK && gran != HYS_GRAN_TOKEN && gran != HYS_GRAN_BLOCK_ROW))
    return HYS_ERR_INVALID_ARG;
  *bytes = full_ws_bytes(d, dtype, gran == HYS_GRAN_BLOCK_ROW ? HYS_GRAN_BLOCK : gran);
  return HYS_OK;
}

hys_status hysparse_full_attn_select(const hys_shape* shape, hys_dtype dtype, const void* q, const void* k,
                                     const void* v, void* o, float* scores, hys_gran gran, hys_reduce red,
                                     float* lse_opt, void* workspace, size_t workspace_bytes,
                                     hys_stream_t stream) {
  PrefillDims d;
  hys_status st = check_prefill(shape, &d);
  if (st != HYS_OK) return st;
  if (!dtype_ok(dtype) || (gran != HYS_GRAN_BLOCK && gran != HYS_GRAN_TOKEN && gran != HYS_GRAN_BLOCK_ROW))
    return HYS_ERR_INVALID_ARG;
  if (red != HYS_REDUCE_SUM && red != HYS_REDUCE_MAX) return HYS_ERR_INVALID_ARG;
  if (gran == HYS_GRAN_TOKEN && red != HYS_REDUCE_SUM) return HYS_ERR_UNSUPPORTED;
  if (gran == HYS_GRAN_BLOCK_ROW && (red != HYS_REDUCE_MAX || !full_attn_tc_supported(d, dtype, true)))
    return HYS_ERR_UNSUPPORTED;
  if (!q || !k || !v || !o || !scores) return HYS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(scores) ||
      !aligned16(lse_opt) || !aligned16(workspace))
    return HYS_ERR_INVALID_ARG;
  const size_t need = full_ws_bytes(d, dtype, gran == HYS_GRAN_BLOCK_ROW ? HYS_GRAN_BLOCK : gran);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return HYS_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (gran == HYS_GRAN_BLOCK_ROW)
    return from_cuda(launch_full_attn_tc(d, q, k, v, o, lse_opt, scores, red, true, workspace, workspace_bytes, s,
                                         true));
  if (gran == HYS_GRAN_BLOCK) {
    if (full_attn_tc_supported(d, dtype, true))
      return from_cuda(launch_full_attn_tc(d, q, k, v, o, lse_opt, scores, red, true, workspace, workspace_bytes, s));
    float* part = reinterpret_cast<float*>(workspace);
    cudaError_t e = launch_full_attn_simt(d, dtype, q, k, v, o, lse_opt, part, true, red, s);
    if (e != cudaSuccess) return HYS_ERR_CUDA;
    return from_cuda(launch_head_reduce(d, part, scores, red, s));
  }
  float* lse = lse_opt ? lse_opt : reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) + 256);
  cudaError_t e;
  if (full_attn_tc_supported(d, dtype, false))
    e = launch_full_attn_tc(d, q, k, v, o, lse, nullptr, HYS_REDUCE_SUM, false, workspace, 256, s);
  else
    e = launch_full_attn_simt(d, dtype, q, k, v, o, lse, nullptr, false, HYS_REDUCE_SUM, s);
  if (e != cudaSuccess) return HYS_ERR_CUDA;
  if (token_scores_tc_supported(d, dtype)) return from_cuda(launch_token_scores_tc(d, q, k, lse, scores, workspace, s));
  return from_cuda(launch_token_scores_simt(d, dtype, q, k, lse, scores, s));
}

// ----------------------------------------------------------------------------- top-k
hys_status hysparse_topk(const hys_shape* shape, const float* scores, int k, int* idx, hys_stream_t stream) {
  PrefillDims d;
  hys_status st = check_prefill(shape, &d);
  if (st != HYS_OK) return st;
  if (!scores || !idx || k < 1 || k > 1024) return HYS_ERR_INVALID_ARG;
  if (!aligned16(scores) || !aligned16(idx)) return HYS_ERR_INVALID_ARG;
  if (d.NB > 8192) return HYS_ERR_UNSUPPORTED;
  return from_cuda(launch_topk_blocks(scores, idx, d.B, d.Hkv, d.T, d.NB, k, nullptr, 0, false,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

hys_status hysparse_topk_rows(const hys_shape* shape, const float* scores, int k, int* idx, hys_stream_t stream) {
  PrefillDims d;
  hys_status st = check_prefill(shape, &d);
  if (st != HYS_OK) return st;
  if (!scores || !idx || k < 1 || k > 1024) return HYS_ERR_INVALID_ARG;
  if (!aligned16(scores) || !aligned16(idx)) return HYS_ERR_INVALID_ARG;
  if (d.NB > 8192) return HYS_ERR_UNSUPPORTED;
  if ((long long)d.B * d.Hkv * d.N >= (1ll << 31)) return HYS_ERR_UNSUPPORTED;
  return from_cuda(launch_topk_blocks_rows(scores, idx, d.B, d.Hkv, d.N, d.NB, k,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

hys_status hysparse_topk_tokens_workspace_size(const hys_shape* shape, int k_tokens, size_t* bytes) {
  PrefillDims d;
  hys_status st = check_prefill(shape, &d);
  if (st != HYS_OK) return st;
  if (!bytes || k_tokens < 1 || k_tokens > 16384) return HYS_ERR_INVALID_ARG;
  *bytes = 0;
  return HYS_OK;
}

hys_status hysparse_topk_tokens(const hys_shape* shape, const float* tok_scores, int k_tokens, int forced_window,
                                int* idx, void* workspace, size_t workspace_bytes, hys_stream_t stream) {
  (void)workspace;
  (void)workspace_bytes;
  PrefillDims d;
  hys_status st = check_prefill(shape, &d);
  if (st != HYS_OK) return st;
  if (!tok_scores || !idx || k_tokens < 1 || k_tokens > 16384 || forced_window < 0) return HYS_ERR_INVALID_ARG;
  if (!aligned16(tok_scores) || !aligned16(idx)) return HYS_ERR_INVALID_ARG;
  return from_cuda(launch_topk_tokens(d, tok_scores, k_tokens, forced_window, idx,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

// ----------------------------------------------------------------------------- sparse layer
hys_status hysparse_sparse_attn_workspace_size(const hys_shape* shape, hys_dtype dtype, size_t* bytes) {
  PrefillDims d;
  hys_status st = check_prefill(shape, &d);
  if (st != HYS_OK) return st;
  if (!bytes || !dtype_ok(dtype)) return HYS_ERR_INVALID_ARG;
  *bytes = sparse_attn_tc_supported(d, dtype) ? align256(sparse_attn_tc_workspace(d)) : 0;
  return HYS_OK;
}

hys_status hysparse_sparse_attn(const hys_shape* shape, hys_dtype dtype, const void* q_sparse, const void* k_shared,
                                const void* v_shared, const int* idx, int k, const void* k_swa, const void* v_swa,
                                int window, const float* gate_logits, const float* sinks, void* o, void* workspace,
                                size_t workspace_bytes, hys_stream_t stream) {
  PrefillDims d;
  hys_status st = check_prefill(shape, &d);
  if (st != HYS_OK) return st;
  if (!dtype_ok(dtype)) return HYS_ERR_INVALID_ARG;
  if (!q_sparse || !k_shared || !v_shared || !idx || !k_swa || !v_swa || !gate_logits || !o) return HYS_ERR_INVALID_ARG;
  if (!aligned16(sinks)) return HYS_ERR_INVALID_ARG;
  if (k < 1 || k > 1024 || window < 1) return HYS_ERR_INVALID_ARG;
  if (!aligned16(q_sparse) || !aligned16(k_shared) || !aligned16(v_shared) || !aligned16(idx) || !aligned16(k_swa) ||
      !aligned16(v_swa) || !aligned16(gate_logits) || !aligned16(o) || !aligned16(workspace))
    return HYS_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (sparse_attn_tc_supported(d, dtype) && k <= 256) {
    const size_t need = align256(sparse_attn_tc_workspace(d));
    if (workspace == nullptr || workspace_bytes < need) return HYS_ERR_WORKSPACE;
    return from_cuda(launch_sparse_attn_tc(d, q_sparse, k_shared, v_shared, idx, k, k_swa, v_swa, window,
                                           gate_logits, sinks, o, workspace, workspace_bytes, s));
  }
  return from_cuda(launch_sparse_attn_simt(d, dtype, q_sparse, k_shared, v_shared, idx, k, k_swa, v_swa, window,
                                           gate_logits, sinks, o, s));
}

// ----------------------------------------------------------------------------- training
hys_status hysparse_sparse_attn_train(const hys_shape* shape, hys_dtype dtype, const void* q_sparse,
                                      const void* k_shared, const void* v_shared, const int* idx, int k,
                                      const void* k_swa, const void* v_swa, int window, const float* gate_logits,
                                      const float* sinks, void* o, void* o_sparse, float* branch_lse, void* workspace,
                                      size_t workspace_bytes, hys_stream_t stream) {
  PrefillDims d;
  hys_status st = check_prefill(shape, &d);
  if (st != HYS_OK) return st;
  if (!dtype_ok(dtype)) return HYS_ERR_INVALID_ARG;
  if (!q_sparse || !k_shared || !v_shared || !idx || !k_swa || !v_swa || !gate_logits || !o || !o_sparse ||
      !branch_lse)
    return HYS_ERR_INVALID_ARG;
  if (k < 1 || k > 1024 || window < 1) return HYS_ERR_INVALID_ARG;
  if (!aligned16(q_sparse) || !aligned16(k_shared) || !aligned16(v_shared) || !aligned16(idx) || !aligned16(k_swa) ||
      !aligned16(v_swa) || !aligned16(gate_logits) || !aligned16(sinks) || !aligned16(o) || !aligned16(o_sparse) ||
      !aligned16(branch_lse) || !aligned16(workspace))
    return HYS_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (sparse_attn_tc_supported(d, dtype) && k <= 256) {
    if (workspace == nullptr || workspace_bytes < align256(sparse_attn_tc_workspace(d))) return HYS_ERR_WORKSPACE;
    return from_cuda(launch_sparse_attn_tc(d, q_sparse, k_shared, v_shared, idx, k, k_swa, v_swa, window, gate_logits,
                                           sinks, o, workspace, workspace_bytes, s, false, branch_lse, o_sparse));
  }
  return from_cuda(launch_sparse_attn_simt(d, dtype, q_sparse, k_shared, v_shared, idx, k, k_swa, v_swa, window,
                                           gate_logits, sinks, o, s, branch_lse, o_sparse));
}

hys_status hysparse_full_attn_backward_workspace_size(const hys_shape* shape, hys_dtype dtype, size_t* bytes) {
  PrefillDims d;
  hys_status st = check_prefill(shape, &d);
  if (st != HYS_OK) return st;
  if (!dtype_ok(dtype) || !bytes) return HYS_ERR_INVALID_ARG;
  *bytes = align256(full_bwd_workspace(d, dtype));
  return HYS_OK;
}

hys_status hysparse_full_attn_backward(const hys_shape* shape, hys_dtype dtype, const void* q, const void* k,
                                       const void* v, const void* o, const void* d_o, const float* lse, void* dq,
                                       float* dk, float* dv, int accumulate_kv, void* workspace,
                                       size_t workspace_bytes, hys_stream_t stream) {
  PrefillDims d;
  hys_status st = check_prefill(shape, &d);
  if (st != HYS_OK) return st;
  if (!dtype_ok(dtype)) return HYS_ERR_INVALID_ARG;
  if (!q || !k || !v || !o || !d_o || !lse || !dq || !dk || !dv) return HYS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(d_o) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
    return HYS_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < align256(full_bwd_workspace(d, dtype))) return HYS_ERR_WORKSPACE;
  return from_cuda(launch_full_bwd(d, dtype, q, k, v, o, d_o, lse, dq, dk, dv, accumulate_kv != 0, workspace,
                                   reinterpret_cast<cudaStream_t>(stream)));
}

hys_status hysparse_sparse_attn_backward_workspace_size(const hys_shape* shape, hys_dtype dtype, size_t* bytes) {
  PrefillDims d;
  hys_status st = check_prefill(shape, &d);
  if (st != HYS_OK) return st;
  if (!dtype_ok(dtype) || !bytes) return HYS_ERR_INVALID_ARG;
  *bytes = align256(sparse_bwd_workspace(d));
  return HYS_OK;
}

hys_status hysparse_sparse_attn_backward(const hys_shape* shape, hys_dtype dtype, const void* q_sparse,
                                         const void* k_shared, const void* v_shared, const int* idx, int k,
                                         const void* k_swa, const void* v_swa, int window, const float* gate_logits,
                                         const float* sinks, const void* o, const void* o_sparse,
                                         const float* branch_lse, const void* d_o, void* dq, float* dk_shared,
                                         float* dv_shared, float* dk_swa, float* dv_swa, float* dgate, float* dsinks,
                                         void* workspace, size_t workspace_bytes, hys_stream_t stream) {
  PrefillDims d;
  hys_status st = check_prefill(shape, &d);
  if (st != HYS_OK) return st;
  if (!dtype_ok(dtype)) return HYS_ERR_INVALID_ARG;
  if (!q_sparse || !k_shared || !v_shared || !idx || !k_swa || !v_swa || !gate_logits || !o || !o_sparse ||
      !branch_lse || !d_o || !dq || !dk_shared || !dv_shared || !dk_swa || !dv_swa || !dgate)
    return HYS_ERR_INVALID_ARG;
  if (sinks != nullptr && dsinks == nullptr) return HYS_ERR_INVALID_ARG;
  if (k < 1 || k > 1024 || window < 1) return HYS_ERR_INVALID_ARG;
  // gradient outputs are distinct buffers (the window branch's are overwritten, the shared ones added to)
  if (dk_swa == dk_shared || dv_swa == dv_shared || dk_swa == dv_shared || dv_swa == dk_shared)
    return HYS_ERR_INVALID_ARG;
  const void* ptrs[] = {q_sparse, k_shared, v_shared, idx, k_swa, v_swa, gate_logits, sinks, o, o_sparse, branch_lse,
                        d_o, dq, dk_shared, dv_shared, dk_swa, dv_swa, dgate, dsinks, workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return HYS_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < align256(sparse_bwd_workspace(d))) return HYS_ERR_WORKSPACE;
  return from_cuda(launch_sparse_bwd(d, dtype, q_sparse, k_shared, v_shared, idx, k, k_swa, v_swa, window, gate_logits,
                                     sinks, o, o_sparse, branch_lse, d_o, dq, dk_shared, dv_shared, dk_swa, dv_swa,
                                     dgate, dsinks, workspace, reinterpret_cast<cudaStream_t>(stream)));
}

hys_status hysparse_sparse_attn_rows(const hys_shape* shape, hys_dtype dtype, const void* q_sparse,
                                     const void* k_shared, const void* v_shared, const int* idx, int k,
                                     const void* k_swa, const void* v_swa, int window, const float* gate_logits,
                                     const float* sinks, void* o, void* workspace, size_t workspace_bytes,
                                     hys_stream_t stream) {
  PrefillDims d;
  hys_status st = check_prefill(shape, &d);
  if (st != HYS_OK) return st;
  if (!dtype_ok(dtype)) return HYS_ERR_INVALID_ARG;
  if (!q_sparse || !k_shared || !v_shared || !idx || !k_swa || !v_swa || !gate_logits || !o) return HYS_ERR_INVALID_ARG;
  if (k < 1 || k > 1024 || window < 1) return HYS_ERR_INVALID_ARG;
  if (!aligned16(q_sparse) || !aligned16(k_shared) || !aligned16(v_shared) || !aligned16(idx) || !aligned16(k_swa) ||
      !aligned16(v_swa) || !aligned16(gate_logits) || !aligned16(sinks) || !aligned16(o) || !aligned16(workspace))
    return HYS_ERR_INVALID_ARG;
  if (!sparse_attn_rows_tc_supported(d, dtype) || k > 256) return HYS_ERR_UNSUPPORTED;
  if (workspace == nullptr || workspace_bytes < align256(sparse_attn_tc_workspace(d))) return HYS_ERR_WORKSPACE;
  return from_cuda(launch_sparse_attn_tc(d, q_sparse, k_shared, v_shared, idx, k, k_swa, v_swa, window, gate_logits,
                                         sinks, o, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream),
                                         true));
}

hys_status hysparse_sparse_attn_tokens_workspace_size(const hys_shape* shape, hys_dtype dtype, int forced_window,
                                                      size_t* bytes) {
  PrefillDims d;
  hys_status st = check_prefill(shape, &d);
  if (st != HYS_OK) return st;
  if (!bytes || !dtype_ok(dtype) || forced_window < 1) return HYS_ERR_INVALID_ARG;
  *bytes = token_sparse_tc_supported(d, dtype, forced_window) ? align256(token_sparse_tc_workspace()) : 0;
  return HYS_OK;
}

hys_status hysparse_sparse_attn_tokens(const hys_shape* shape, hys_dtype dtype, const void* q_sparse,
                                       const void* k_shared, const void* v_shared, const int* idx, int k_tokens,
                                       int forced_window, const float* sinks, void* o, void* workspace,
                                       size_t workspace_bytes, hys_stream_t stream) {
  PrefillDims d;
  hys_status st = check_prefill(shape, &d);
  if (st != HYS_OK) return st;
  if (!dtype_ok(dtype)) return HYS_ERR_INVALID_ARG;
  if (sinks) return HYS_ERR_UNSUPPORTED;
  if (!q_sparse || !k_shared || !v_shared || !idx || !o) return HYS_ERR_INVALID_ARG;
  if (k_tokens < 1 || k_tokens > 16384 || forced_window < 1) return HYS_ERR_INVALID_ARG;
  if (!aligned16(q_sparse) || !aligned16(k_shared) || !aligned16(v_shared) || !aligned16(idx) || !aligned16(o) ||
      !aligned16(workspace))
    return HYS_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (token_sparse_tc_supported(d, dtype, forced_window)) {
    if (workspace == nullptr || workspace_bytes < align256(token_sparse_tc_workspace())) return HYS_ERR_WORKSPACE;
    return from_cuda(launch_token_sparse_tc(d, q_sparse, k_shared, v_shared, idx, k_tokens, forced_window, o,
                                            workspace, s));
  }
  return from_cuda(launch_sparse_tokens_simt(d, dtype, q_sparse, k_shared, v_shared, idx, k_tokens, forced_window, o,
                                             s));
}

// ----------------------------------------------------------------------------- decode
hys_status hysparse_full_attn_select_decode_workspace_size(const hys_decode_shape* shape, hys_dtype dtype,
                                                           size_t* bytes) {
  DecodeDims d;
  hys_status st = check_decode(shape, &d);
  if (st != HYS_OK) return st;
  if (!bytes || !dtype_ok(dtype)) return HYS_ERR_INVALID_ARG;
  *bytes = align256(decode_mma_supported(d, dtype) ? decode_mma_full_workspace(d) : decode_full_workspace(d));
  return HYS_OK;
}

hys_status hysparse_full_attn_select_decode(const hys_decode_shape* shape, hys_dtype dtype, const void* q,
                                            const void* k_cache, const void* v_cache, const int* seqlens, void* o,
                                            float* scores, hys_reduce red, void* workspace, size_t workspace_bytes,
                                            hys_stream_t stream) {
  DecodeDims d;
  hys_status st = check_decode(shape, &d);
  if (st != HYS_OK) return st;
  if (!dtype_ok(dtype) || (red != HYS_REDUCE_SUM && red != HYS_REDUCE_MAX)) return HYS_ERR_INVALID_ARG;
  if (!q || !k_cache || !v_cache || !o || !scores) return HYS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) || !aligned16(scores) ||
      !aligned16(seqlens) || !aligned16(workspace))
    return HYS_ERR_INVALID_ARG;
  const bool mma = decode_mma_supported(d, dtype);
  const size_t need = align256(mma ? decode_mma_full_workspace(d) : decode_full_workspace(d));
  if (workspace == nullptr || workspace_bytes < need) return HYS_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (mma) return from_cuda(launch_decode_full_mma(d, q, k_cache, v_cache, seqlens, o, scores, red, workspace, s));
  return from_cuda(launch_decode_full(d, dtype, q, k_cache, v_cache, seqlens, o, scores, red, workspace, s));
}

hys_status hysparse_topk_decode(const hys_decode_shape* shape, const float* scores, int k, const int* seqlens,
                                int* idx, hys_stream_t stream) {
  DecodeDims d;
  hys_status st = check_decode(shape, &d);
  if (st != HYS_OK) return st;
  if (!scores || !idx || k < 1 || k > 1024) return HYS_ERR_INVALID_ARG;
  if (!aligned16(scores) || !aligned16(idx) || !aligned16(seqlens)) return HYS_ERR_INVALID_ARG;
  if (d.NB > 8192) return HYS_ERR_UNSUPPORTED;
  return from_cuda(launch_topk_blocks(scores, idx, d.B, d.Hkv, 1, d.NB, k, seqlens, d.L, true,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

hys_status hysparse_sparse_attn_decode_workspace_size(const hys_decode_shape* shape, hys_dtype dtype, int k,
                                                      size_t* bytes) {
  DecodeDims d;
  hys_status st = check_decode(shape, &d);
  if (st != HYS_OK) return st;
  if (!bytes || !dtype_ok(dtype) || k < 1 || k > 1024) return HYS_ERR_INVALID_ARG;
  *bytes = decode_mma_supported(d, dtype) ? align256(decode_mma_sparse_workspace(d, k)) : 0;
  return HYS_OK;
}

hys_status hysparse_sparse_attn_decode(const hys_decode_shape* shape, hys_dtype dtype, const void* q,
                                       const void* k_cache, const void* v_cache, const int* seqlens, const int* idx,
                                       int k, const void* k_swa_ring, const void* v_swa_ring, int window,
                                       const int* swa_len, const float* gate_logits, const float* sinks, void* o,
                                       void* workspace, size_t workspace_bytes, hys_stream_t stream) {
  DecodeDims d;
  hys_status st = check_decode(shape, &d);
  if (st != HYS_OK) return st;
  if (!dtype_ok(dtype)) return HYS_ERR_INVALID_ARG;
  if (!q || !k_cache || !v_cache || !idx || !k_swa_ring || !v_swa_ring || !gate_logits || !o) return HYS_ERR_INVALID_ARG;
  if (!aligned16(sinks)) return HYS_ERR_INVALID_ARG;
  if (k < 1 || k > 1024 || window < 1 || window > 1024) return HYS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(seqlens) || !aligned16(idx) ||
      !aligned16(k_swa_ring) || !aligned16(v_swa_ring) || !aligned16(swa_len) || !aligned16(gate_logits) ||
      !aligned16(o) || !aligned16(workspace))
    return HYS_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (decode_mma_supported(d, dtype)) {
    if (workspace == nullptr || workspace_bytes < align256(decode_mma_sparse_workspace(d, k))) return HYS_ERR_WORKSPACE;
    return from_cuda(launch_decode_sparse_mma(d, q, k_cache, v_cache, seqlens, idx, k, k_swa_ring, v_swa_ring, window,
                                              swa_len, gate_logits, sinks, o, workspace, s));
  }
  return from_cuda(launch_decode_sparse(d, dtype, q, k_cache, v_cache, seqlens, idx, k, k_swa_ring, v_swa_ring,
                                        window, swa_len, gate_logits, sinks, o, s));
}

// ----------------------------------------------------------------------------- token-variant decode
hys_status hysparse_full_attn_select_decode_tokens_workspace_size(const hys_decode_shape* shape, hys_dtype dtype,
                                                                  size_t* bytes) {
  DecodeDims d;
  hys_status st = check_decode(shape, &d);
  if (st != HYS_OK) return st;
  if (!bytes || !dtype_ok(dtype)) return HYS_ERR_INVALID_ARG;
  if (!decode_mma_supported(d, dtype)) return HYS_ERR_UNSUPPORTED;
  *bytes = align256(decode_mma_full_tokens_workspace(d));
  return HYS_OK;
}

hys_status hysparse_full_attn_select_decode_tokens(const hys_decode_shape* shape, hys_dtype dtype, const void* q,
                                                   const void* k_cache, const void* v_cache, const int* seqlens,
                                                   void* o, float* tok_scores, void* workspace,
                                                   size_t workspace_bytes, hys_stream_t stream) {
  DecodeDims d;
  hys_status st = check_decode(shape, &d);
  if (st != HYS_OK) return st;
  if (!dtype_ok(dtype)) return HYS_ERR_INVALID_ARG;
  if (!q || !k_cache || !v_cache || !o || !tok_scores) return HYS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(seqlens) || !aligned16(o) ||
      !aligned16(tok_scores) || !aligned16(workspace))
    return HYS_ERR_INVALID_ARG;
  if (!decode_mma_supported(d, dtype)) return HYS_ERR_UNSUPPORTED;
  if (workspace == nullptr || workspace_bytes < align256(decode_mma_full_tokens_workspace(d))) return HYS_ERR_WORKSPACE;
  return from_cuda(launch_decode_full_tokens_mma(d, q, k_cache, v_cache, seqlens, o, tok_scores, workspace,
                                                 reinterpret_cast<cudaStream_t>(stream)));
}

hys_status hysparse_topk_decode_tokens(const hys_decode_shape* shape, const float* tok_scores, int k_tokens,
                                       int forced_window, const int* seqlens, int* idx, hys_stream_t stream) {
  DecodeDims d;
  hys_status st = check_decode(shape, &d);
  if (st != HYS_OK) return st;
  if (!tok_scores || !idx || k_tokens < 1 || k_tokens > 16384 || forced_window < 1) return HYS_ERR_INVALID_ARG;
  if (!aligned16(tok_scores) || !aligned16(idx) || !aligned16(seqlens)) return HYS_ERR_INVALID_ARG;
  return from_cuda(launch_topk_decode_tokens(tok_scores, idx, d.B, d.Hkv, d.L, k_tokens, forced_window, seqlens,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

hys_status hysparse_sparse_attn_decode_tokens_workspace_size(const hys_decode_shape* shape, hys_dtype dtype,
                                                             int k_tokens, size_t* bytes) {
  DecodeDims d;
  hys_status st = check_decode(shape, &d);
  if (st != HYS_OK) return st;
  if (!bytes || !dtype_ok(dtype) || k_tokens < 1 || k_tokens > 16384) return HYS_ERR_INVALID_ARG;
  if (!decode_mma_supported(d, dtype)) return HYS_ERR_UNSUPPORTED;
  *bytes = align256(decode_mma_sparse_tokens_workspace(d, k_tokens));
  return HYS_OK;
}

hys_status hysparse_sparse_attn_decode_tokens(const hys_decode_shape* shape, hys_dtype dtype, const void* q,
                                              const void* k_cache, const void* v_cache, const int* seqlens,
                                              const int* idx, int k_tokens, int forced_window, void* o,
                                              void* workspace, size_t workspace_bytes, hys_stream_t stream) {
  DecodeDims d;
  hys_status st = check_decode(shape, &d);
  if (st != HYS_OK) return st;
  if (!dtype_ok(dtype)) return HYS_ERR_INVALID_ARG;
  if (!q || !k_cache || !v_cache || !idx || !o) return HYS_ERR_INVALID_ARG;
  if (k_tokens < 1 || k_tokens > 16384 || forced_window < 1 || forced_window > 4096) return HYS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(seqlens) || !aligned16(idx) ||
      !aligned16(o) || !aligned16(workspace))
    return HYS_ERR_INVALID_ARG;
  if (!decode_mma_supported(d, dtype)) return HYS_ERR_UNSUPPORTED;
  if ((long long)d.B * d.Hkv * d.L >= (1ll << 31)) return HYS_ERR_UNSUPPORTED;
  if (workspace == nullptr || workspace_bytes < align256(decode_mma_sparse_tokens_workspace(d, k_tokens)))
    return HYS_ERR_WORKSPACE;
  return from_cuda(launch_decode_sparse_tokens_mma(d, q, k_cache, v_cache, seqlens, idx, k_tokens, forced_window, o,
                                                   workspace, reinterpret_cast<cudaStream_t>(stream)));
}

namespace {
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
}  // namespace

hys_status hysparse_full_attn_select_decode_tokens_fp8(const hys_decode_shape* shape, const void* q,
                                                       const void* k_cache, const void* v_cache,
                                                       const float* k_scale, const float* v_scale,
                                                       const int* seqlens, void* o, float* tok_scores,
                                                       void* workspace, size_t workspace_bytes,
                                                       hys_stream_t stream) {
  DecodeDims d;
  hys_status st = check_decode(shape, &d);
  if (st != HYS_OK) return st;
  if (!q || !k_cache || !v_cache || !k_scale || !v_scale || !o || !tok_scores) return HYS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned4(k_scale) || !aligned4(v_scale) ||
      !aligned16(seqlens) || !aligned16(o) || !aligned16(tok_scores) || !aligned16(workspace))
    return HYS_ERR_INVALID_ARG;
  if (!decode_mma_supported(d, HYS_BF16)) return HYS_ERR_UNSUPPORTED;
  if (workspace == nullptr || workspace_bytes < align256(decode_mma_full_tokens_workspace(d))) return HYS_ERR_WORKSPACE;
  return from_cuda(launch_decode_full_tokens_mma_fp8(d, q, k_cache, v_cache, k_scale, v_scale, seqlens, o, tok_scores,
                                                     workspace, reinterpret_cast<cudaStream_t>(stream)));
}

hys_status hysparse_sparse_attn_decode_tokens_fp8(const hys_decode_shape* shape, const void* q, const void* k_cache,
                                                  const void* v_cache, const float* k_scale, const float* v_scale,
                                                  const int* seqlens, const int* idx, int k_tokens, int forced_window,
                                                  void* o, void* workspace, size_t workspace_bytes,
                                                  hys_stream_t stream) {
  DecodeDims d;
  hys_status st = check_decode(shape, &d);
  if (st != HYS_OK) return st;
  if (!q || !k_cache || !v_cache || !k_scale || !v_scale || !idx || !o) return HYS_ERR_INVALID_ARG;
  if (k_tokens < 1 || k_tokens > 16384 || forced_window < 1 || forced_window > 4096) return HYS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned4(k_scale) || !aligned4(v_scale) ||
      !aligned16(seqlens) || !aligned16(idx) || !aligned16(o) || !aligned16(workspace))
    return HYS_ERR_INVALID_ARG;
  if (!decode_mma_supported(d, HYS_BF16)) return HYS_ERR_UNSUPPORTED;
  if ((long long)d.B * d.Hkv * d.L >= (1ll << 31)) return HYS_ERR_UNSUPPORTED;
  if (workspace == nullptr || workspace_bytes < align256(decode_mma_sparse_tokens_workspace(d, k_tokens)))
    return HYS_ERR_WORKSPACE;
  return from_cuda(launch_decode_sparse_tokens_mma_fp8(d, q, k_cache, v_cache, k_scale, v_scale, seqlens, idx,
                                                       k_tokens, forced_window, o, workspace,
                                                       reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
