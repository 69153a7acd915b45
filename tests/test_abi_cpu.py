"""Host-only checks of the C ABI library: it builds, loads, exports every symbol the
header declares, and rejects bad arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

from attention_tcgen05_tma_b200 import build as B
from attention_tcgen05_tma_b200 import hysparse as H

HEADER = os.path.join(B.ROOT, "include", "hysparse.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return H.load()


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"HYS_API\s+[\w\s\*]+?\b(hysparse_\w+)\s*\(", txt)))


def test_header_and_binding_agree():
    assert declared_symbols() == sorted(H.EXPORTED)


def test_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_version_and_status_strings(lib):
    assert re.match(r"^\d+\.\d+\.\d+$", H.hysparse_version())
    assert H.status_string(H.HYS_ERR_INVALID_ARG) == "HYS_ERR_INVALID_ARG"
    assert H.status_string(H.HYS_ERR_TIMEOUT) == "HYS_ERR_TIMEOUT"


def test_workspace_queries_and_validation(lib):
    good = H.hys_shape(1, 1000, 8, 2, 128, 64)
    assert H.hysparse_full_attn_select_workspace_size(good, H.HYS_BF16, H.HYS_GRAN_BLOCK) >= 0
    assert H.hysparse_full_attn_select_workspace_size(good, H.HYS_BF16, H.HYS_GRAN_TOKEN) >= 4 * 8 * 1000
    for bad in (H.hys_shape(1, 1000, 8, 3, 128, 64), H.hys_shape(1, 1000, 8, 2, 96, 64),
                H.hys_shape(1, 0, 8, 2, 128, 64), H.hys_shape(1, 1000, 8, 2, 128, 32)):
        with pytest.raises(H.HysparseError) as e:
            H.hysparse_full_attn_select_workspace_size(bad, H.HYS_BF16, H.HYS_GRAN_BLOCK)
        assert e.value.status == H.HYS_ERR_INVALID_ARG
    dsh = H.hys_decode_shape(4, 5000, 32, 4, 128, 64)
    assert H.hysparse_full_attn_select_decode_workspace_size(dsh, H.HYS_BF16) > 0


def test_entry_points_reject_bad_arguments_without_launching(lib):
    sh = H.hys_shape(1, 256, 4, 1, 64, 64)
    # null pointers / misaligned pointers / bad k are rejected on the host
    assert H.hysparse_full_attn_select(sh, H.HYS_F32, None, None, None, None, None, 0, 0, None, None, 0, None) \
        == H.HYS_ERR_INVALID_ARG
    assert H.hysparse_topk(sh, 16, 0, 16, None) == H.HYS_ERR_INVALID_ARG
    assert H.hysparse_topk(sh, 17, 4, 16, None) == H.HYS_ERR_INVALID_ARG
    # sink logits are accepted, but like every pointer must be 16-byte aligned (checked before
    # anything launches); the token variant has no sink biases
    assert H.hysparse_sparse_attn(sh, H.HYS_F32, 16, 16, 16, 16, 4, 16, 16, 128, 16, 8, 16, None, 0, None) \
        == H.HYS_ERR_INVALID_ARG
    assert H.hysparse_sparse_attn_tokens(sh, H.HYS_F32, 16, 16, 16, 16, 4, 128, 16, 16, None, 0, None) \
        == H.HYS_ERR_UNSUPPORTED
    dsh1 = H.hys_decode_shape(2, 1000, 8, 2, 128, 64)
    assert H.hysparse_sparse_attn_decode(dsh1, H.HYS_BF16, 16, 16, 16, None, 16, 4, 16, 16, 128, None, 16, 8, 16,
                                         16, 1 << 20, None) == H.HYS_ERR_INVALID_ARG
    bsh = H.hys_shape(1, 256, 4, 2, 128, 64)
    assert H.hysparse_sparse_attn_workspace_size(bsh, H.HYS_BF16) > 0
    assert H.hysparse_sparse_attn(bsh, H.HYS_BF16, 16, 16, 16, 16, 4, 16, 16, 128, 16, None, 16, None, 0, None) \
        == H.HYS_ERR_WORKSPACE
    assert H.hysparse_sparse_attn_tokens(sh, H.HYS_F32, 16, 16, 16, 16, 0, 128, None, 16, None, 0, None) \
        == H.HYS_ERR_INVALID_ARG
    tsh = H.hys_shape(1, 512, 8, 2, 128, 64)
    assert H.hysparse_sparse_attn_tokens_workspace_size(tsh, H.HYS_BF16, 128) > 0
    assert H.hysparse_sparse_attn_tokens(tsh, H.HYS_BF16, 16, 16, 16, 16, 64, 128, None, 16, None, 0, None) \
        == H.HYS_ERR_WORKSPACE
    assert H.hysparse_full_attn_select(sh, H.HYS_F32, 16, 16, 16, 16, 16, 0, 7, None, None, 0, None) \
        == H.HYS_ERR_INVALID_ARG
    # token scores with max aggregation are not defined
    assert H.hysparse_full_attn_select(sh, H.HYS_F32, 16, 16, 16, 16, 16, H.HYS_GRAN_TOKEN, H.HYS_REDUCE_MAX,
                                       None, 16, 1 << 20, None) == H.HYS_ERR_UNSUPPORTED
    # workspace too small
    assert H.hysparse_full_attn_select(sh, H.HYS_F32, 16, 16, 16, 16, 16, 0, 0, None, 16, 4, None) \
        == H.HYS_ERR_WORKSPACE
    dsh = H.hys_decode_shape(2, 100, 4, 1, 64, 64)
    assert H.hysparse_sparse_attn_decode(dsh, H.HYS_F32, 16, 16, 16, None, 16, 4, 16, 16, 2000, None, 16, None,
                                         16, None, 0, None) == H.HYS_ERR_INVALID_ARG
    bdsh = H.hys_decode_shape(2, 1000, 16, 2, 128, 64)
    assert H.hysparse_sparse_attn_decode_workspace_size(bdsh, H.HYS_BF16, 32) > 0
    assert H.hysparse_sparse_attn_decode(bdsh, H.HYS_BF16, 16, 16, 16, None, 16, 32, 16, 16, 128, None, 16, None,
                                         16, None, 0, None) == H.HYS_ERR_WORKSPACE
    assert H.hysparse_full_attn_select_decode(dsh, H.HYS_F32, 16, 16, 16, None, 16, 16, 0, None, 0, None) \
        == H.HYS_ERR_WORKSPACE


def test_token_decode_entry_points_validate(lib):
    dsh = H.hys_decode_shape(2, 1000, 16, 2, 128, 64)
    assert H.hysparse_full_attn_select_decode_tokens_workspace_size(dsh, H.HYS_BF16) > 0
    assert H.hysparse_sparse_attn_decode_tokens_workspace_size(dsh, H.HYS_BF16, 256) > 0
    # fp32 / D = 64 have no token-variant decode path: unsupported, nothing launched
    fsh = H.hys_decode_shape(2, 1000, 16, 2, 64, 64)
    assert H.hysparse_full_attn_select_decode_tokens(fsh, H.HYS_F32, 16, 16, 16, None, 16, 16, 16, 1 << 20, None) \
        == H.HYS_ERR_UNSUPPORTED
    # null output, bad budget / window, misaligned pointers, short workspace
    assert H.hysparse_full_attn_select_decode_tokens(dsh, H.HYS_BF16, 16, 16, 16, None, 16, None, 16, 1 << 20, None) \
        == H.HYS_ERR_INVALID_ARG
    assert H.hysparse_topk_decode_tokens(dsh, 16, 0, 64, None, 16, None) == H.HYS_ERR_INVALID_ARG
    assert H.hysparse_topk_decode_tokens(dsh, 16, 64, 0, None, 16, None) == H.HYS_ERR_INVALID_ARG
    assert H.hysparse_topk_decode_tokens(dsh, 8, 64, 64, None, 16, None) == H.HYS_ERR_INVALID_ARG
    assert H.hysparse_sparse_attn_decode_tokens(dsh, H.HYS_BF16, 16, 16, 16, None, 16, 64, 5000, 16, 16, 1 << 20,
                                                None) == H.HYS_ERR_INVALID_ARG
    assert H.hysparse_sparse_attn_decode_tokens(dsh, H.HYS_BF16, 16, 16, 16, None, 16, 64, 64, 16, 16, 64,
                                                None) == H.HYS_ERR_WORKSPACE


def test_per_position_entry_points_validate(lib):
    """Per-position selection: group max only, tensor-core shapes only, N <= 32768 for the
    sparse layer; every check fails before a launch."""
    sh = H.hys_shape(1, 1000, 8, 2, 128, 64)
    # HYS_GRAN_BLOCK_ROW needs the max aggregation, bf16 and an even group
    assert H.hysparse_full_attn_select(sh, H.HYS_BF16, 16, 16, 16, 16, 16, H.HYS_GRAN_BLOCK_ROW, H.HYS_REDUCE_SUM,
                                       None, 16, 1 << 20, None) == H.HYS_ERR_UNSUPPORTED
    assert H.hysparse_full_attn_select(sh, H.HYS_F32, 16, 16, 16, 16, 16, H.HYS_GRAN_BLOCK_ROW, H.HYS_REDUCE_MAX,
                                       None, 16, 1 << 20, None) == H.HYS_ERR_UNSUPPORTED
    assert H.hysparse_full_attn_select_workspace_size(sh, H.HYS_BF16, H.HYS_GRAN_BLOCK_ROW) == \
        H.hysparse_full_attn_select_workspace_size(sh, H.HYS_BF16, H.HYS_GRAN_BLOCK)
    assert H.hysparse_topk_rows(sh, 16, 0, 16, None) == H.HYS_ERR_INVALID_ARG
    assert H.hysparse_topk_rows(sh, 8, 4, 16, None) == H.HYS_ERR_INVALID_ARG
    rows = H.hysparse_sparse_attn_rows
    assert rows(sh, H.HYS_F32, 16, 16, 16, 16, 4, 16, 16, 128, 16, None, 16, 16, 1 << 20, None) \
        == H.HYS_ERR_UNSUPPORTED
    long_sh = H.hys_shape(1, 40000, 8, 2, 128, 64)
    assert rows(long_sh, H.HYS_BF16, 16, 16, 16, 16, 4, 16, 16, 128, 16, None, 16, 16, 1 << 20, None) \
        == H.HYS_ERR_UNSUPPORTED
    assert rows(sh, H.HYS_BF16, 16, 16, 16, 16, 300, 16, 16, 128, 16, None, 16, 16, 1 << 20, None) \
        == H.HYS_ERR_UNSUPPORTED
    assert rows(sh, H.HYS_BF16, 16, 16, 16, 16, 4, 16, 16, 128, 16, None, 16, 16, 0, None) == H.HYS_ERR_WORKSPACE
    assert rows(sh, H.HYS_BF16, 16, 16, 16, 16, 4, 16, 16, 128, 16, 8, 16, 16, 1 << 20, None) \
        == H.HYS_ERR_INVALID_ARG


def test_fp8_token_decode_entry_points_validate(lib):
    """FP8-cache token decode: the scales are required (4-byte aligned), D must be 128, and the
    workspace is the bf16 call's; every check fails before a launch."""
    dsh = H.hys_decode_shape(2, 1000, 16, 2, 128, 64)
    full = H.hysparse_full_attn_select_decode_tokens_fp8
    sparse = H.hysparse_sparse_attn_decode_tokens_fp8
    # missing scales / output, misaligned scale
    assert full(dsh, 16, 16, 16, None, 16, None, 16, 16, 16, 1 << 20, None) == H.HYS_ERR_INVALID_ARG
    assert full(dsh, 16, 16, 16, 16, 16, None, None, 16, 16, 1 << 20, None) == H.HYS_ERR_INVALID_ARG
    assert full(dsh, 16, 16, 16, 18, 16, None, 16, 16, 16, 1 << 20, None) == H.HYS_ERR_INVALID_ARG
    # D = 64: no FP8 path
    d64 = H.hys_decode_shape(2, 1000, 16, 2, 64, 64)
    assert full(d64, 16, 16, 16, 16, 16, None, 16, 16, 16, 1 << 20, None) == H.HYS_ERR_UNSUPPORTED
    # short workspace
    need = H.hysparse_full_attn_select_decode_tokens_workspace_size(dsh, H.HYS_BF16)
    assert full(dsh, 16, 16, 16, 16, 16, None, 16, 16, 16, need - 256, None) == H.HYS_ERR_WORKSPACE
    assert sparse(dsh, 16, 16, 16, 16, None, None, 16, 64, 64, 16, 16, 1 << 20, None) == H.HYS_ERR_INVALID_ARG
    assert sparse(dsh, 16, 16, 16, 16, 16, None, 16, 64, 5000, 16, 16, 1 << 20, None) == H.HYS_ERR_INVALID_ARG
    assert sparse(dsh, 16, 16, 16, 16, 16, None, 16, 64, 64, 16, 16, 64, None) == H.HYS_ERR_WORKSPACE


def test_training_entry_points_reject_bad_arguments_without_launching(lib):
    sh = H.hys_shape(1, 256, 4, 2, 128, 64)
    assert H.hysparse_full_attn_backward_workspace_size(sh, H.HYS_BF16) > 0
    assert H.hysparse_sparse_attn_backward_workspace_size(sh, H.HYS_BF16) > 0
    P = 256   # an aligned stand-in pointer: every call below fails validation before any launch
    # missing inputs / outputs
    assert H.hysparse_full_attn_backward(sh, H.HYS_BF16, P, P, P, P, P, None, P, P, P, 0, P, 1 << 30, None) \
        == H.HYS_ERR_INVALID_ARG
    # misaligned gradient output
    assert H.hysparse_full_attn_backward(sh, H.HYS_BF16, P, P, P, P, P, P, P + 4, P, P, 0, P, 1 << 30, None) \
        == H.HYS_ERR_INVALID_ARG
    # workspace too small
    assert H.hysparse_full_attn_backward(sh, H.HYS_BF16, P, P, P, P, P, P, P, P, P, 0, P, 16, None) \
        == H.HYS_ERR_WORKSPACE
    args = [P] * 4 + [2, P, P, 128, P, None, P, P, P, P]   # q, k, v, idx, k, ks, vs, window, gate, sinks, o, osp, lse, do
    outs = [512, 768, 1024, 1280, 1536, 1792, None]         # dq, dk, dv, dk_swa, dv_swa, dgate, dsinks
    ok = H.hysparse_sparse_attn_backward(sh, H.HYS_BF16, *args, *outs, P, 16, None)
    assert ok == H.HYS_ERR_WORKSPACE                        # valid arguments, workspace too small
    alias = list(outs)
    alias[3] = alias[1]                                     # dk_swa aliases dk_shared
    assert H.hysparse_sparse_attn_backward(sh, H.HYS_BF16, *args, *alias, P, 1 << 30, None) == H.HYS_ERR_INVALID_ARG
    with_sinks = list(args)
    with_sinks[9] = P                                       # sinks given without a dsinks output
    assert H.hysparse_sparse_attn_backward(sh, H.HYS_BF16, *with_sinks, *outs, P, 1 << 30, None) \
        == H.HYS_ERR_INVALID_ARG
    # the training forward needs both saved outputs
    assert H.hysparse_sparse_attn_train(sh, H.HYS_BF16, P, P, P, P, 2, P, P, 128, P, None, P, None, P, P, 1 << 20,
                                        None) == H.HYS_ERR_INVALID_ARG
