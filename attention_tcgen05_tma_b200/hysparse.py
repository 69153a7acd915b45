"""Thin ctypes binding of libhysparse.so (the C ABI declared in include/hysparse.h).

The ``hysparse_*`` functions mirror the C entry points one to one and take raw
integers for pointers and the stream.  The short-named helpers below them only
marshal torch tensors (device pointers, the current stream, output allocation); every
step of the computation runs in the library's CUDA kernels.  There is no fallback:
loading fails loudly when the library is missing or was not built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libhysparse.so")

HYS_OK, HYS_ERR_INVALID_ARG, HYS_ERR_UNSUPPORTED, HYS_ERR_CUDA, HYS_ERR_TIMEOUT, HYS_ERR_WORKSPACE = range(6)
HYS_F32, HYS_BF16 = 0, 1
HYS_GRAN_BLOCK, HYS_GRAN_TOKEN, HYS_GRAN_BLOCK_ROW = 0, 1, 2
HYS_REDUCE_SUM, HYS_REDUCE_MAX = 0, 1

# every symbol include/hysparse.h declares
EXPORTED = (
    "hysparse_version", "hysparse_status_string", "hysparse_get_device_status",
    "hysparse_full_attn_select_workspace_size", "hysparse_full_attn_select",
    "hysparse_topk", "hysparse_topk_tokens_workspace_size", "hysparse_topk_tokens",
    "hysparse_sparse_attn_workspace_size", "hysparse_sparse_attn",
    "hysparse_sparse_attn_tokens_workspace_size", "hysparse_sparse_attn_tokens",
    "hysparse_full_attn_select_decode_workspace_size", "hysparse_full_attn_select_decode",
    "hysparse_topk_decode", "hysparse_sparse_attn_decode_workspace_size", "hysparse_sparse_attn_decode",
    "hysparse_full_attn_select_decode_noalloc",
    "hysparse_full_attn_select_decode_tokens_workspace_size", "hysparse_full_attn_select_decode_tokens",
    "hysparse_topk_decode_tokens", "hysparse_sparse_attn_decode_tokens_workspace_size",
    "hysparse_sparse_attn_decode_tokens",
    "hysparse_full_attn_select_decode_tokens_fp8", "hysparse_sparse_attn_decode_tokens_fp8",
    "hysparse_topk_rows", "hysparse_sparse_attn_rows",
    "hysparse_sparse_attn_train", "hysparse_full_attn_backward_workspace_size", "hysparse_full_attn_backward",
    "hysparse_sparse_attn_backward_workspace_size", "hysparse_sparse_attn_backward",
)


class HysparseError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


class hys_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("N", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("D", ctypes.c_int), ("block", ctypes.c_int)]


class hys_decode_shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("L", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("D", ctypes.c_int), ("block", ctypes.c_int)]


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
_SH = ctypes.POINTER(hys_shape)
_DSH = ctypes.POINTER(hys_decode_shape)

_SIGS = {
    "hysparse_version": ([], ctypes.c_char_p),
    "hysparse_status_string": ([_I], ctypes.c_char_p),
    "hysparse_get_device_status": ([_P, _I, ctypes.POINTER(_I)], _I),
    "hysparse_full_attn_select_workspace_size": ([_SH, _I, _I, ctypes.POINTER(_SZ)], _I),
    "hysparse_full_attn_select": ([_SH, _I, _P, _P, _P, _P, _P, _I, _I, _P, _P, _SZ, _P], _I),
    "hysparse_topk": ([_SH, _P, _I, _P, _P], _I),
    "hysparse_topk_rows": ([_SH, _P, _I, _P, _P], _I),
    "hysparse_topk_tokens_workspace_size": ([_SH, _I, ctypes.POINTER(_SZ)], _I),
    "hysparse_topk_tokens": ([_SH, _P, _I, _I, _P, _P, _SZ, _P], _I),
    "hysparse_sparse_attn_workspace_size": ([_SH, _I, ctypes.POINTER(_SZ)], _I),
    "hysparse_sparse_attn": ([_SH, _I, _P, _P, _P, _P, _I, _P, _P, _I, _P, _P, _P, _P, _SZ, _P], _I),
    "hysparse_sparse_attn_rows": ([_SH, _I, _P, _P, _P, _P, _I, _P, _P, _I, _P, _P, _P, _P, _SZ, _P], _I),
    "hysparse_sparse_attn_tokens_workspace_size": ([_SH, _I, _I, ctypes.POINTER(_SZ)], _I),
    "hysparse_sparse_attn_tokens": ([_SH, _I, _P, _P, _P, _P, _I, _I, _P, _P, _P, _SZ, _P], _I),
    "hysparse_full_attn_select_decode_workspace_size": ([_DSH, _I, ctypes.POINTER(_SZ)], _I),
    "hysparse_full_attn_select_decode": ([_DSH, _I, _P, _P, _P, _P, _P, _P, _I, _P, _SZ, _P], _I),
    "hysparse_topk_decode": ([_DSH, _P, _I, _P, _P, _P], _I),
    "hysparse_full_attn_select_decode_noalloc": ([_DSH, _I, _P, _P, _P, _P, _P, _P, _I, _P], _I),
    "hysparse_sparse_attn_decode_workspace_size": ([_DSH, _I, _I, ctypes.POINTER(_SZ)], _I),
    "hysparse_sparse_attn_decode": ([_DSH, _I, _P, _P, _P, _P, _P, _I, _P, _P, _I, _P, _P, _P, _P, _P, _SZ, _P],
                                    _I),
    "hysparse_full_attn_select_decode_tokens_workspace_size": ([_DSH, _I, ctypes.POINTER(_SZ)], _I),
    "hysparse_full_attn_select_decode_tokens": ([_DSH, _I, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], _I),
    "hysparse_topk_decode_tokens": ([_DSH, _P, _I, _I, _P, _P, _P], _I),
    "hysparse_sparse_attn_decode_tokens_workspace_size": ([_DSH, _I, _I, ctypes.POINTER(_SZ)], _I),
    "hysparse_sparse_attn_decode_tokens": ([_DSH, _I, _P, _P, _P, _P, _P, _I, _I, _P, _P, _SZ, _P], _I),
    "hysparse_full_attn_select_decode_tokens_fp8": ([_DSH, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], _I),
    "hysparse_sparse_attn_decode_tokens_fp8": ([_DSH, _P, _P, _P, _P, _P, _P, _P, _I, _I, _P, _P, _SZ, _P], _I),
    "hysparse_sparse_attn_train": ([_SH, _I, _P, _P, _P, _P, _I, _P, _P, _I, _P, _P, _P, _P, _P, _P, _SZ, _P], _I),
    "hysparse_full_attn_backward_workspace_size": ([_SH, _I, ctypes.POINTER(_SZ)], _I),
    "hysparse_full_attn_backward": ([_SH, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _SZ, _P], _I),
    "hysparse_sparse_attn_backward_workspace_size": ([_SH, _I, ctypes.POINTER(_SZ)], _I),
    "hysparse_sparse_attn_backward": ([_SH, _I, _P, _P, _P, _P, _I, _P, _P, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                       _P, _P, _P, _P, _P, _SZ, _P], _I),
}

_lib: Optional[ctypes.CDLL] = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library (once) and declare the signatures.  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libhysparse.so not found at {path}; build it with "
                           "`python -m attention_tcgen05_tma_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (args, res) in _SIGS.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def status_string(s: int) -> str:
    return load().hysparse_status_string(int(s)).decode()


def _check(s: int, where: str):
    if s != HYS_OK:
        raise HysparseError(s, where)


# ----------------------------------------------------------------------------- raw C mirrors
def hysparse_version() -> str:
    return load().hysparse_version().decode()


def hysparse_get_device_status(stream: int = 0, reset: bool = False) -> int:
    out = _I(0)
    _check(load().hysparse_get_device_status(stream, int(reset), ctypes.byref(out)), "hysparse_get_device_status")
    return out.value


def hysparse_full_attn_select_workspace_size(shape: hys_shape, dtype: int, gran: int) -> int:
    n = _SZ(0)
    _check(load().hysparse_full_attn_select_workspace_size(ctypes.byref(shape), dtype, gran, ctypes.byref(n)),
           "hysparse_full_attn_select_workspace_size")
    return n.value


def hysparse_full_attn_select(shape, dtype, q, k, v, o, scores, gran, red, lse, ws, ws_bytes, stream) -> int:
    return load().hysparse_full_attn_select(ctypes.byref(shape), dtype, q, k, v, o, scores, gran, red, lse, ws,
                                            ws_bytes, stream)


def hysparse_topk(shape, scores, k, idx, stream) -> int:
    return load().hysparse_topk(ctypes.byref(shape), scores, k, idx, stream)


def hysparse_topk_rows(shape, scores, k, idx, stream) -> int:
    return load().hysparse_topk_rows(ctypes.byref(shape), scores, k, idx, stream)


def hysparse_topk_tokens_workspace_size(shape: hys_shape, k_tokens: int) -> int:
    n = _SZ(0)
    _check(load().hysparse_topk_tokens_workspace_size(ctypes.byref(shape), k_tokens, ctypes.byref(n)),
           "hysparse_topk_tokens_workspace_size")
    return n.value


def hysparse_topk_tokens(shape, scores, k_tokens, forced, idx, ws, ws_bytes, stream) -> int:
    return load().hysparse_topk_tokens(ctypes.byref(shape), scores, k_tokens, forced, idx, ws, ws_bytes, stream)


def hysparse_sparse_attn_workspace_size(shape: hys_shape, dtype: int) -> int:
    n = _SZ(0)
    _check(load().hysparse_sparse_attn_workspace_size(ctypes.byref(shape), dtype, ctypes.byref(n)),
           "hysparse_sparse_attn_workspace_size")
    return n.value


def hysparse_sparse_attn(shape, dtype, q, k, v, idx, kb, ks, vs, window, gate, sinks, o, ws, ws_bytes,
                         stream) -> int:
    return load().hysparse_sparse_attn(ctypes.byref(shape), dtype, q, k, v, idx, kb, ks, vs, window, gate, sinks,
                                       o, ws, ws_bytes, stream)


def hysparse_sparse_attn_rows(shape, dtype, q, k, v, idx, kb, ks, vs, window, gate, sinks, o, ws, ws_bytes,
                              stream) -> int:
    return load().hysparse_sparse_attn_rows(ctypes.byref(shape), dtype, q, k, v, idx, kb, ks, vs, window, gate,
                                            sinks, o, ws, ws_bytes, stream)


def hysparse_sparse_attn_tokens_workspace_size(shape: hys_shape, dtype: int, forced: int) -> int:
    n = _SZ(0)
    _check(load().hysparse_sparse_attn_tokens_workspace_size(ctypes.byref(shape), dtype, forced, ctypes.byref(n)),
           "hysparse_sparse_attn_tokens_workspace_size")
    return n.value


def hysparse_sparse_attn_tokens(shape, dtype, q, k, v, idx, kt, forced, sinks, o, ws, ws_bytes, stream) -> int:
    return load().hysparse_sparse_attn_tokens(ctypes.byref(shape), dtype, q, k, v, idx, kt, forced, sinks, o, ws,
                                              ws_bytes, stream)


def hysparse_full_attn_select_decode_workspace_size(shape: hys_decode_shape, dtype: int) -> int:
    n = _SZ(0)
    _check(load().hysparse_full_attn_select_decode_workspace_size(ctypes.byref(shape), dtype, ctypes.byref(n)),
           "hysparse_full_attn_select_decode_workspace_size")
    return n.value


def hysparse_full_attn_select_decode(shape, dtype, q, kc, vc, seqlens, o, scores, red, ws, ws_bytes, stream) -> int:
    return load().hysparse_full_attn_select_decode(ctypes.byref(shape), dtype, q, kc, vc, seqlens, o, scores, red,
                                                   ws, ws_bytes, stream)


def hysparse_full_attn_select_decode_noalloc(shape, dtype, q, kc, vc, seqlens, o, scores, red, stream) -> int:
    """Decode full layer without a workspace (scratch in a fixed 16 MiB array inside the
    library); for callers that cannot allocate device memory during a decode step."""
    return load().hysparse_full_attn_select_decode_noalloc(ctypes.byref(shape), dtype, q, kc, vc, seqlens, o,
                                                           scores, red, stream)


def hysparse_topk_decode(shape, scores, k, seqlens, idx, stream) -> int:
    return load().hysparse_topk_decode(ctypes.byref(shape), scores, k, seqlens, idx, stream)


def hysparse_sparse_attn_decode_workspace_size(shape: hys_decode_shape, dtype: int, k: int) -> int:
    n = _SZ(0)
    _check(load().hysparse_sparse_attn_decode_workspace_size(ctypes.byref(shape), dtype, k, ctypes.byref(n)),
           "hysparse_sparse_attn_decode_workspace_size")
    return n.value


def hysparse_sparse_attn_decode(shape, dtype, q, kc, vc, seqlens, idx, kb, kr, vr, window, swa_len, gate, sinks, o,
                                ws, ws_bytes, stream) -> int:
    return load().hysparse_sparse_attn_decode(ctypes.byref(shape), dtype, q, kc, vc, seqlens, idx, kb, kr, vr, window,
                                              swa_len, gate, sinks, o, ws, ws_bytes, stream)


def hysparse_full_attn_select_decode_tokens_workspace_size(shape: hys_decode_shape, dtype: int) -> int:
    n = _SZ(0)
    _check(load().hysparse_full_attn_select_decode_tokens_workspace_size(ctypes.byref(shape), dtype, ctypes.byref(n)),
           "hysparse_full_attn_select_decode_tokens_workspace_size")
    return n.value


def hysparse_full_attn_select_decode_tokens(shape, dtype, q, kc, vc, seqlens, o, tok_scores, ws, ws_bytes,
                                            stream) -> int:
    return load().hysparse_full_attn_select_decode_tokens(ctypes.byref(shape), dtype, q, kc, vc, seqlens, o,
                                                          tok_scores, ws, ws_bytes, stream)


def hysparse_topk_decode_tokens(shape, tok_scores, k_tokens, forced, seqlens, idx, stream) -> int:
    return load().hysparse_topk_decode_tokens(ctypes.byref(shape), tok_scores, k_tokens, forced, seqlens, idx, stream)


def hysparse_sparse_attn_decode_tokens_workspace_size(shape: hys_decode_shape, dtype: int, k_tokens: int) -> int:
    n = _SZ(0)
    _check(load().hysparse_sparse_attn_decode_tokens_workspace_size(ctypes.byref(shape), dtype, k_tokens,
                                                                    ctypes.byref(n)),
           "hysparse_sparse_attn_decode_tokens_workspace_size")
    return n.value


def hysparse_sparse_attn_decode_tokens(shape, dtype, q, kc, vc, seqlens, idx, k_tokens, forced, o, ws, ws_bytes,
                                       stream) -> int:
    return load().hysparse_sparse_attn_decode_tokens(ctypes.byref(shape), dtype, q, kc, vc, seqlens, idx, k_tokens,
                                                     forced, o, ws, ws_bytes, stream)


def hysparse_full_attn_select_decode_tokens_fp8(shape, q, kc, vc, k_scale, v_scale, seqlens, o, tok_scores, ws,
                                                ws_bytes, stream) -> int:
    return load().hysparse_full_attn_select_decode_tokens_fp8(ctypes.byref(shape), q, kc, vc, k_scale, v_scale,
                                                              seqlens, o, tok_scores, ws, ws_bytes, stream)


def hysparse_sparse_attn_decode_tokens_fp8(shape, q, kc, vc, k_scale, v_scale, seqlens, idx, k_tokens, forced, o, ws,
                                           ws_bytes, stream) -> int:
    return load().hysparse_sparse_attn_decode_tokens_fp8(ctypes.byref(shape), q, kc, vc, k_scale, v_scale, seqlens,
                                                         idx, k_tokens, forced, o, ws, ws_bytes, stream)


def hysparse_sparse_attn_train(shape, dtype, q, k, v, idx, kb, ks, vs, window, gate, sinks, o, o_sparse, blse, ws,
                               ws_bytes, stream) -> int:
    return load().hysparse_sparse_attn_train(ctypes.byref(shape), dtype, q, k, v, idx, kb, ks, vs, window, gate,
                                             sinks, o, o_sparse, blse, ws, ws_bytes, stream)


def hysparse_full_attn_backward_workspace_size(shape: hys_shape, dtype: int) -> int:
    n = _SZ(0)
    _check(load().hysparse_full_attn_backward_workspace_size(ctypes.byref(shape), dtype, ctypes.byref(n)),
           "hysparse_full_attn_backward_workspace_size")
    return n.value


def hysparse_full_attn_backward(shape, dtype, q, k, v, o, d_o, lse, dq, dk, dv, accumulate, ws, ws_bytes,
                                stream) -> int:
    return load().hysparse_full_attn_backward(ctypes.byref(shape), dtype, q, k, v, o, d_o, lse, dq, dk, dv,
                                              accumulate, ws, ws_bytes, stream)


def hysparse_sparse_attn_backward_workspace_size(shape: hys_shape, dtype: int) -> int:
    n = _SZ(0)
    _check(load().hysparse_sparse_attn_backward_workspace_size(ctypes.byref(shape), dtype, ctypes.byref(n)),
           "hysparse_sparse_attn_backward_workspace_size")
    return n.value


def hysparse_sparse_attn_backward(shape, dtype, q, k, v, idx, kb, ks, vs, window, gate, sinks, o, o_sparse, blse,
                                  d_o, dq, dk, dv, dks, dvs, dgate, dsinks, ws, ws_bytes, stream) -> int:
    return load().hysparse_sparse_attn_backward(ctypes.byref(shape), dtype, q, k, v, idx, kb, ks, vs, window, gate,
                                                sinks, o, o_sparse, blse, d_o, dq, dk, dv, dks, dvs, dgate, dsinks,
                                                ws, ws_bytes, stream)


# ----------------------------------------------------------------------------- torch helpers
def _torch():
    import torch
    return torch


def _dt(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return HYS_BF16
    if t.dtype == torch.float32:
        return HYS_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream) -> int:
    torch = _torch()
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def prefill_shape(q, k) -> hys_shape:
    B, Hq, N, D = q.shape
    return hys_shape(B, N, Hq, k.shape[1], D, 64)


def decode_shape(q, k_cache) -> hys_decode_shape:
    B, Hq, D = q.shape
    return hys_decode_shape(B, k_cache.shape[2], Hq, k_cache.shape[1], D, 64)


def workspace_for(nbytes: int, device):
    torch = _torch()
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)


def full_attn_select(q, k, v, *, gran: str = "block", reduce: str = "sum", o=None, scores=None, lse=None,
                     workspace=None, stream=None) -> Tuple[object, object]:
    """Full causal GQA attention plus importance scores. Returns (o, scores).

    gran "block": [B,Hkv,T,NB] per 64-query tile; "token": [B,Hkv,T,N]; "block_row":
    [B,Hkv,N,NB] per query position (group maximum, reduce must be "max")."""
    torch = _torch()
    sh = prefill_shape(q, k)
    g = {"token": HYS_GRAN_TOKEN, "block_row": HYS_GRAN_BLOCK_ROW}.get(gran, HYS_GRAN_BLOCK)
    T = (sh.N + 63) // 64
    if o is None:
        o = torch.empty_like(q)
    if scores is None:
        rows = sh.N if g == HYS_GRAN_BLOCK_ROW else T
        cols = sh.N if g == HYS_GRAN_TOKEN else T
        scores = torch.empty((sh.B, sh.Hkv, rows, cols), dtype=torch.float32, device=q.device)
    nws = hysparse_full_attn_select_workspace_size(sh, _dt(q), g)
    if workspace is None and nws > 0:
        workspace = workspace_for(nws, q.device)
    st = hysparse_full_attn_select(sh, _dt(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(scores), g,
                                   HYS_REDUCE_MAX if reduce == "max" else HYS_REDUCE_SUM, _ptr(lse),
                                   _ptr(workspace), workspace.numel() if workspace is not None else 0,
                                   _stream(stream))
    _check(st, "hysparse_full_attn_select")
    return o, scores


def topk(scores, k: int, *, idx=None, stream=None):
    torch = _torch()
    B, Hkv, T, NB = scores.shape
    sh = hys_shape(B, NB * 64, Hkv, Hkv, 64, 64)
    if idx is None:
        idx = torch.empty((B, Hkv, T, k), dtype=torch.int32, device=scores.device)
    _check(hysparse_topk(sh, _ptr(scores), k, _ptr(idx), _stream(stream)), "hysparse_topk")
    return idx


def topk_tokens(scores, k_tokens: int, forced_window: int, *, idx=None, stream=None):
    torch = _torch()
    B, Hkv, T, N = scores.shape
    sh = hys_shape(B, N, Hkv, Hkv, 64, 64)
    if idx is None:
        idx = torch.empty((B, Hkv, T, k_tokens), dtype=torch.int32, device=scores.device)
    _check(hysparse_topk_tokens(sh, _ptr(scores), k_tokens, forced_window, _ptr(idx), None, 0, _stream(stream)),
           "hysparse_topk_tokens")
    return idx


def sparse_attn(q_sparse, k, v, idx, k_swa, v_swa, window: int, gate_logits, *, sinks=None, o=None,
                workspace=None, stream=None):
    torch = _torch()
    sh = prefill_shape(q_sparse, k)
    if o is None:
        o = torch.empty_like(q_sparse)
    if workspace is None:
        workspace = workspace_for(hysparse_sparse_attn_workspace_size(sh, _dt(q_sparse)), q_sparse.device)
    _check(hysparse_sparse_attn(sh, _dt(q_sparse), _ptr(q_sparse), _ptr(k), _ptr(v), _ptr(idx), idx.shape[-1],
                                _ptr(k_swa), _ptr(v_swa), window, _ptr(gate_logits), _ptr(sinks), _ptr(o),
                                _ptr(workspace), workspace.numel(), _stream(stream)), "hysparse_sparse_attn")
    return o


def topk_rows(scores, k: int, *, idx=None, stream=None):
    """Per-position top-k of [B,Hkv,N,NB] scores -> idx [B,Hkv,N,k]."""
    torch = _torch()
    B, Hkv, N, NB = scores.shape
    sh = hys_shape(B, N, Hkv, Hkv, 64, 64)
    if idx is None:
        idx = torch.empty((B, Hkv, N, k), dtype=torch.int32, device=scores.device)
    _check(hysparse_topk_rows(sh, _ptr(scores), k, _ptr(idx), _stream(stream)), "hysparse_topk_rows")
    return idx


def sparse_attn_rows(q_sparse, k, v, idx, k_swa, v_swa, window: int, gate_logits, *, sinks=None, o=None,
                     workspace=None, stream=None):
    """The sparse layer with per-position selection (idx [B,Hkv,N,k])."""
    torch = _torch()
    sh = prefill_shape(q_sparse, k)
    if o is None:
        o = torch.empty_like(q_sparse)
    if workspace is None:
        workspace = workspace_for(hysparse_sparse_attn_workspace_size(sh, _dt(q_sparse)), q_sparse.device)
    _check(hysparse_sparse_attn_rows(sh, _dt(q_sparse), _ptr(q_sparse), _ptr(k), _ptr(v), _ptr(idx), idx.shape[-1],
                                     _ptr(k_swa), _ptr(v_swa), window, _ptr(gate_logits), _ptr(sinks), _ptr(o),
                                     _ptr(workspace), workspace.numel(), _stream(stream)), "hysparse_sparse_attn_rows")
    return o


def sparse_attn_tokens(q_sparse, k, v, idx, forced_window: int, *, o=None, workspace=None, stream=None):
    torch = _torch()
    sh = prefill_shape(q_sparse, k)
    if o is None:
        o = torch.empty_like(q_sparse)
    if workspace is None:
        workspace = workspace_for(hysparse_sparse_attn_tokens_workspace_size(sh, _dt(q_sparse), forced_window),
                                  q_sparse.device)
    _check(hysparse_sparse_attn_tokens(sh, _dt(q_sparse), _ptr(q_sparse), _ptr(k), _ptr(v), _ptr(idx),
                                       idx.shape[-1], forced_window, None, _ptr(o), _ptr(workspace),
                                       workspace.numel(), _stream(stream)),
           "hysparse_sparse_attn_tokens")
    return o


def full_attn_select_decode(q, k_cache, v_cache, *, seqlens=None, reduce: str = "sum", o=None, scores=None,
                            workspace=None, stream=None):
    torch = _torch()
    sh = decode_shape(q, k_cache)
    nb = (sh.L + 63) // 64
    if o is None:
        o = torch.empty_like(q)
    if scores is None:
        scores = torch.empty((sh.B, sh.Hkv, nb), dtype=torch.float32, device=q.device)
    nws = hysparse_full_attn_select_decode_workspace_size(sh, _dt(q))
    if workspace is None:
        workspace = workspace_for(nws, q.device)
    _check(hysparse_full_attn_select_decode(sh, _dt(q), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens),
                                            _ptr(o), _ptr(scores), HYS_REDUCE_MAX if reduce == "max" else
                                            HYS_REDUCE_SUM, _ptr(workspace), workspace.numel(), _stream(stream)),
           "hysparse_full_attn_select_decode")
    return o, scores


def topk_decode(scores, k: int, L: int, *, seqlens=None, idx=None, stream=None):
    torch = _torch()
    B, Hkv, NB = scores.shape
    sh = hys_decode_shape(B, L, Hkv, Hkv, 64, 64)
    if idx is None:
        idx = torch.empty((B, Hkv, k), dtype=torch.int32, device=scores.device)
    _check(hysparse_topk_decode(sh, _ptr(scores), k, _ptr(seqlens), _ptr(idx), _stream(stream)), "hysparse_topk_decode")
    return idx


def sparse_attn_decode(q, k_cache, v_cache, idx, k_ring, v_ring, gate_logits, *, seqlens=None, swa_len=None,
                       sinks=None, o=None, workspace=None, stream=None):
    torch = _torch()
    sh = decode_shape(q, k_cache)
    if o is None:
        o = torch.empty_like(q)
    if workspace is None:
        workspace = workspace_for(hysparse_sparse_attn_decode_workspace_size(sh, _dt(q), idx.shape[-1]), q.device)
    _check(hysparse_sparse_attn_decode(sh, _dt(q), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), _ptr(idx),
                                       idx.shape[-1], _ptr(k_ring), _ptr(v_ring), k_ring.shape[2], _ptr(swa_len),
                                       _ptr(gate_logits), _ptr(sinks), _ptr(o), _ptr(workspace), workspace.numel(),
                                       _stream(stream)),
           "hysparse_sparse_attn_decode")
    return o


def full_attn_select_decode_tokens(q, k_cache, v_cache, *, seqlens=None, o=None, tok_scores=None, workspace=None,
                                   stream=None):
    """Token-variant decode full layer: o [B,Hq,D] and token scores [B,Hkv,L]."""
    torch = _torch()
    sh = decode_shape(q, k_cache)
    if o is None:
        o = torch.empty_like(q)
    if tok_scores is None:
        tok_scores = torch.empty((sh.B, sh.Hkv, sh.L), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = workspace_for(hysparse_full_attn_select_decode_tokens_workspace_size(sh, _dt(q)), q.device)
    _check(hysparse_full_attn_select_decode_tokens(sh, _dt(q), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens),
                                                   _ptr(o), _ptr(tok_scores), _ptr(workspace), workspace.numel(),
                                                   _stream(stream)),
           "hysparse_full_attn_select_decode_tokens")
    return o, tok_scores


def topk_decode_tokens(tok_scores, k_tokens: int, forced_window: int, *, seqlens=None, idx=None, stream=None):
    torch = _torch()
    B, Hkv, L = tok_scores.shape
    sh = hys_decode_shape(B, L, Hkv, Hkv, 64, 64)
    if idx is None:
        idx = torch.empty((B, Hkv, k_tokens), dtype=torch.int32, device=tok_scores.device)
    _check(hysparse_topk_decode_tokens(sh, _ptr(tok_scores), k_tokens, forced_window, _ptr(seqlens), _ptr(idx),
                                       _stream(stream)), "hysparse_topk_decode_tokens")
    return idx


def sparse_attn_decode_tokens(q, k_cache, v_cache, idx, forced_window: int, *, seqlens=None, o=None, workspace=None,
                              stream=None):
    """Token-variant sparse decode layer: the selected tokens plus the newest forced_window."""
    torch = _torch()
    sh = decode_shape(q, k_cache)
    if o is None:
        o = torch.empty_like(q)
    if workspace is None:
        workspace = workspace_for(hysparse_sparse_attn_decode_tokens_workspace_size(sh, _dt(q), idx.shape[-1]),
                                  q.device)
    _check(hysparse_sparse_attn_decode_tokens(sh, _dt(q), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens),
                                              _ptr(idx), idx.shape[-1], forced_window, _ptr(o), _ptr(workspace),
                                              workspace.numel(), _stream(stream)),
           "hysparse_sparse_attn_decode_tokens")
    return o


def _fp8_cache_ok(q, k_cache, v_cache, k_scale, v_scale):
    torch = _torch()
    if q.dtype != torch.bfloat16:
        raise TypeError("the FP8-cache decode takes a bf16 query")
    for t in (k_cache, v_cache):
        if t.element_size() != 1:
            raise TypeError("the FP8 cache holds one-byte E4M3 codes (torch.uint8 or torch.float8_e4m3fn)")
    for t in (k_scale, v_scale):
        if t.dtype != torch.float32 or t.numel() != k_cache.shape[1]:
            raise TypeError("k_scale / v_scale are float32 [Hkv]")


def full_attn_select_decode_tokens_fp8(q, k_cache, v_cache, k_scale, v_scale, *, seqlens=None, o=None,
                                       tok_scores=None, workspace=None, stream=None):
    """Token-variant decode full layer over an E4M3 cache (value = code * scale[g]):
    o [B,Hq,D] bf16 and token scores [B,Hkv,L]."""
    torch = _torch()
    _fp8_cache_ok(q, k_cache, v_cache, k_scale, v_scale)
    sh = decode_shape(q, k_cache)
    if o is None:
        o = torch.empty_like(q)
    if tok_scores is None:
        tok_scores = torch.empty((sh.B, sh.Hkv, sh.L), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = workspace_for(hysparse_full_attn_select_decode_tokens_workspace_size(sh, HYS_BF16), q.device)
    _check(hysparse_full_attn_select_decode_tokens_fp8(sh, _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale),
                                                       _ptr(v_scale), _ptr(seqlens), _ptr(o), _ptr(tok_scores),
                                                       _ptr(workspace), workspace.numel(), _stream(stream)),
           "hysparse_full_attn_select_decode_tokens_fp8")
    return o, tok_scores


def sparse_attn_decode_tokens_fp8(q, k_cache, v_cache, k_scale, v_scale, idx, forced_window: int, *, seqlens=None,
                                  o=None, workspace=None, stream=None):
    """Token-variant sparse decode layer over an E4M3 cache: the selected tokens plus the newest
    forced_window."""
    torch = _torch()
    _fp8_cache_ok(q, k_cache, v_cache, k_scale, v_scale)
    sh = decode_shape(q, k_cache)
    if o is None:
        o = torch.empty_like(q)
    if workspace is None:
        workspace = workspace_for(hysparse_sparse_attn_decode_tokens_workspace_size(sh, HYS_BF16, idx.shape[-1]),
                                  q.device)
    _check(hysparse_sparse_attn_decode_tokens_fp8(sh, _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale),
                                                  _ptr(v_scale), _ptr(seqlens), _ptr(idx), idx.shape[-1],
                                                  forced_window, _ptr(o), _ptr(workspace), workspace.numel(),
                                                  _stream(stream)),
           "hysparse_sparse_attn_decode_tokens_fp8")
    return o


# ----------------------------------------------------------------------------- training
def sparse_attn_train(q_sparse, k_shared, v_shared, idx, k_swa, v_swa, window: int, gate_logits, *, sinks=None,
                      o=None, o_sparse=None, branch_lse=None, workspace=None, stream=None):
    """Sparse layer forward of a training step. Returns (o, o_sparse, branch_lse): the layer
    output, its gated sparse-branch part sigmoid(g0) o~ and the two branches' LSE [B,Hq,N,2]."""
    torch = _torch()
    sh = prefill_shape(q_sparse, k_shared)
    o = torch.empty_like(q_sparse) if o is None else o
    o_sparse = torch.empty_like(q_sparse) if o_sparse is None else o_sparse
    if branch_lse is None:
        branch_lse = torch.empty((sh.B, sh.Hq, sh.N, 2), dtype=torch.float32, device=q_sparse.device)
    if workspace is None:
        workspace = workspace_for(hysparse_sparse_attn_workspace_size(sh, _dt(q_sparse)), q_sparse.device)
    _check(hysparse_sparse_attn_train(sh, _dt(q_sparse), _ptr(q_sparse), _ptr(k_shared), _ptr(v_shared), _ptr(idx),
                                      idx.shape[-1], _ptr(k_swa), _ptr(v_swa), window, _ptr(gate_logits), _ptr(sinks),
                                      _ptr(o), _ptr(o_sparse), _ptr(branch_lse), _ptr(workspace), workspace.numel(),
                                      _stream(stream)),
           "hysparse_sparse_attn_train")
    return o, o_sparse, branch_lse


def full_attn_backward(q, k, v, o, d_o, lse, *, dq=None, dk=None, dv=None, accumulate: bool = False,
                       workspace=None, stream=None):
    """Gradients of the full layer. Returns (dq [input type], dk fp32, dv fp32); with
    accumulate, dk and dv (given) receive the gradient added to their contents."""
    torch = _torch()
    sh = prefill_shape(q, k)
    dq = torch.empty_like(q) if dq is None else dq
    if dk is None:
        dk = torch.empty(k.shape, dtype=torch.float32, device=k.device)
    if dv is None:
        dv = torch.empty(v.shape, dtype=torch.float32, device=v.device)
    if workspace is None:
        workspace = workspace_for(hysparse_full_attn_backward_workspace_size(sh, _dt(q)), q.device)
    _check(hysparse_full_attn_backward(sh, _dt(q), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(d_o), _ptr(lse), _ptr(dq),
                                       _ptr(dk), _ptr(dv), int(accumulate), _ptr(workspace), workspace.numel(),
                                       _stream(stream)),
           "hysparse_full_attn_backward")
    return dq, dk, dv


def sparse_attn_backward(q_sparse, k_shared, v_shared, idx, k_swa, v_swa, window: int, gate_logits, o, o_sparse,
                         branch_lse, d_o, dk_shared, dv_shared, *, sinks=None, dq=None, dk_swa=None, dv_swa=None,
                         dgate=None, dsinks=None, workspace=None, stream=None):
    """Gradients of one sparse layer. dk_shared / dv_shared (fp32, given) receive the sparse
    branch's gradient of the shared cache ADDED to their contents. Returns
    (dq, dk_swa, dv_swa, dgate, dsinks)."""
    torch = _torch()
    sh = prefill_shape(q_sparse, k_shared)
    dev = q_sparse.device
    dq = torch.empty_like(q_sparse) if dq is None else dq
    if dk_swa is None:
        dk_swa = torch.empty(k_swa.shape, dtype=torch.float32, device=dev)
    if dv_swa is None:
        dv_swa = torch.empty(v_swa.shape, dtype=torch.float32, device=dev)
    if dgate is None:
        dgate = torch.empty((sh.B, sh.Hq, sh.N, 2), dtype=torch.float32, device=dev)
    if sinks is not None and dsinks is None:
        dsinks = torch.empty((sh.Hq, 2), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = workspace_for(hysparse_sparse_attn_backward_workspace_size(sh, _dt(q_sparse)), dev)
    _check(hysparse_sparse_attn_backward(sh, _dt(q_sparse), _ptr(q_sparse), _ptr(k_shared), _ptr(v_shared), _ptr(idx),
                                         idx.shape[-1], _ptr(k_swa), _ptr(v_swa), window, _ptr(gate_logits),
                                         _ptr(sinks), _ptr(o), _ptr(o_sparse), _ptr(branch_lse), _ptr(d_o), _ptr(dq),
                                         _ptr(dk_shared), _ptr(dv_shared), _ptr(dk_swa), _ptr(dv_swa), _ptr(dgate),
                                         _ptr(dsinks), _ptr(workspace), workspace.numel(), _stream(stream)),
           "hysparse_sparse_attn_backward")
    return dq, dk_swa, dv_swa, dgate, dsinks
