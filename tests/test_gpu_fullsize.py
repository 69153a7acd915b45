"""Parity at the full sizes the benchmark times, in its launch configuration (same workloads,
same calls through the C ABI, one sparse layer), checked on sampled outputs that the oracle
computes one query tile (prefill) or one sequence (decode) at a time: every output row of the
sampled tiles, their block or token scores, the selection rules, and the sparse layer's rows
recomputed by the oracle on the GPU's own indices."""
import numpy as np
import pytest
import torch

import oracle as O
from attention_tcgen05_tma_b200 import hysparse as H
from attention_tcgen05_tma_b200 import inputs as I
from tests.gpu_support import TOL, check_selection, device_fill, score_rel_err, to_np

pytestmark = pytest.mark.gpu


def _keys(w, heads):
    return [(b, h) for b in range(w.B) for h in range(heads)]


def test_prefill_fullsize_sampled():
    """moe80b: B2 N32768, 32/4 heads, D128, top-32 blocks, SWA 128."""
    w = I.scaled(I.WORKLOADS["moe80b"], layers=1)
    pl = I.plants(w)
    qsh, kvsh = (w.B, w.Hq, w.N, w.D), (w.B, w.Hkv, w.N, w.D)
    bq, bk = _keys(w, w.Hq), _keys(w, w.Hkv)
    q = device_fill(qsh, lambda b, h: I.q_slice(w, b, h), bq)
    k = device_fill(kvsh, lambda b, g: I.k_slice(w, b, g, pl), bk)
    v = device_fill(kvsh, lambda b, g: I.v_slice(w, b, g), bk)
    qs = device_fill(qsh, lambda b, h: I.sparse_q_slice(w, 0, b, h), bq)
    ks = device_fill(kvsh, lambda b, g: I.swa_k_slice(w, 0, b, g), bk)
    vs = device_fill(kvsh, lambda b, g: I.swa_v_slice(w, 0, b, g), bk)
    gate = device_fill((w.B, w.Hq, w.N, 2), lambda b, h: I.gate_slice(w, 0, b, h), bq, bf16=False)
    o, sc = H.full_attn_select(q, k, v)
    idx = H.topk(sc, w.topk)
    osp = H.sparse_attn(qs, k, v, idx, ks, vs, w.window, gate)
    torch.cuda.synchronize()
    assert H.hysparse_get_device_status() == 0
    G = w.G
    for b, g, I_ in I.sampled_tiles(w, 4):
        rows = O.tile_rows(I_, w.N)
        heads = list(range(g * G, (g + 1) * G))
        kk, vv = I.k_slice(w, b, g, pl), I.v_slice(w, b, g)
        qg = np.stack([I.q_slice(w, b, h) for h in heads])
        for j, h in enumerate(heads):
            o_ref, _ = O.attention_rows(qg[j][rows], rows, kk, vv)
            assert np.max(np.abs(to_np(o[b, h, I_ * 64:I_ * 64 + len(rows)]) - o_ref)) <= TOL["bf16"]
        s_ref = O.block_scores_tile(qg, kk, I_)
        s_gpu = to_np(sc[b, g, I_])
        assert score_rel_err(s_ref, s_gpu) <= 1e-3
        assert np.all(s_gpu[I_ + 1:] == 0)
        sel = idx[b, g, I_].cpu().numpy().astype(np.int64)
        check_selection(s_ref, s_gpu, sel, I_ + 1, w.topk)
        kss, vss = I.swa_k_slice(w, 0, b, g), I.swa_v_slice(w, 0, b, g)
        for h in heads:
            ref = O.gated_sparse_rows(I.sparse_q_slice(w, 0, b, h)[rows], rows, kk, vv, sel, kss, vss, w.window,
                                      I.gate_slice(w, 0, b, h)[rows])
            assert np.max(np.abs(to_np(osp[b, h, I_ * 64:I_ * 64 + len(rows)]) - ref)) <= TOL["bf16"]


def test_decode_fullsize_sampled():
    """decode: B64 sequences of L131072 cached tokens, 32/4 heads, D128, top-32 blocks, ring 128."""
    w = I.scaled(I.WORKLOADS["decode"], layers=1)
    bq, bk = _keys(w, w.Hq), _keys(w, w.Hkv)
    q = device_fill((w.B, w.Hq, w.D), lambda b, h: I.decode_q_slice(w, b, h), bq)
    k = device_fill((w.B, w.Hkv, w.N, w.D), lambda b, g: I.decode_k_slice(w, b, g), bk)
    v = device_fill((w.B, w.Hkv, w.N, w.D), lambda b, g: I.decode_v_slice(w, b, g), bk)
    qs = device_fill((w.B, w.Hq, w.D), lambda b, h: I.decode_sparse_q_slice(w, 0, b, h), bq)
    kr = device_fill((w.B, w.Hkv, w.window, w.D), lambda b, g: I.swa_k_slice(w, 0, b, g), bk)
    vr = device_fill((w.B, w.Hkv, w.window, w.D), lambda b, g: I.swa_v_slice(w, 0, b, g), bk)
    gate = device_fill((w.B, w.Hq, 2), lambda b, h: I.gate_slice(w, 0, b, h), bq, bf16=False)
    o, sc = H.full_attn_select_decode(q, k, v)
    idx = H.topk_decode(sc, w.topk, w.N)
    osp = H.sparse_attn_decode(qs, k, v, idx, kr, vr, gate)
    torch.cuda.synchronize()
    assert H.hysparse_get_device_status() == 0
    for b in (0, 37, w.B - 1):
        qb = np.stack([I.decode_q_slice(w, b, h) for h in range(w.Hq)])[None]
        kb = np.stack([I.decode_k_slice(w, b, g) for g in range(w.Hkv)])[None]
        vb = np.stack([I.decode_v_slice(w, b, g) for g in range(w.Hkv)])[None]
        o_ref, s_ref = O.decode_full(qb, kb, vb)
        assert np.max(np.abs(to_np(o[b]) - o_ref[0])) <= TOL["bf16"]
        s_gpu = to_np(sc[b])
        assert score_rel_err(s_ref[0], s_gpu) <= 1e-3
        sel = idx[b].cpu().numpy().astype(np.int64)
        for g in range(w.Hkv):
            check_selection(s_ref[0, g], s_gpu[g], sel[g], w.NB, w.topk)
        qsb = np.stack([I.decode_sparse_q_slice(w, 0, b, h) for h in range(w.Hq)])[None]
        krb = np.stack([I.swa_k_slice(w, 0, b, g) for g in range(w.Hkv)])[None]
        vrb = np.stack([I.swa_v_slice(w, 0, b, g) for g in range(w.Hkv)])[None]
        gb = np.stack([I.gate_slice(w, 0, b, h) for h in range(w.Hq)])[None]
        ref = O.decode_sparse(qsb, kb, vb, sel[None], krb, vrb, gb)
        assert np.max(np.abs(to_np(osp[b]) - ref[0])) <= TOL["bf16"]


def test_token_fullsize_sampled():
    """token variant: B1 N131072, 32/4 heads, D128, top-2048 tokens + newest 128 forced."""
    w = I.scaled(I.WORKLOADS["token"], layers=1)
    pl = I.plants(w)
    qsh, kvsh = (w.B, w.Hq, w.N, w.D), (w.B, w.Hkv, w.N, w.D)
    bq, bk = _keys(w, w.Hq), _keys(w, w.Hkv)
    q = device_fill(qsh, lambda b, h: I.q_slice(w, b, h), bq)
    k = device_fill(kvsh, lambda b, g: I.k_slice(w, b, g, pl), bk)
    v = device_fill(kvsh, lambda b, g: I.v_slice(w, b, g), bk)
    qs = device_fill(qsh, lambda b, h: I.sparse_q_slice(w, 0, b, h), bq)
    o, ts = H.full_attn_select(q, k, v, gran="token")
    idx = H.topk_tokens(ts, w.topk, w.window)
    osp = H.sparse_attn_tokens(qs, k, v, idx, w.window)
    torch.cuda.synchronize()
    assert H.hysparse_get_device_status() == 0
    G = w.G
    for b, g, I_ in I.sampled_tiles(w, 3):
        rows = O.tile_rows(I_, w.N)
        heads = list(range(g * G, (g + 1) * G))
        kk, vv = I.k_slice(w, b, g, pl), I.v_slice(w, b, g)
        qg = np.stack([I.q_slice(w, b, h) for h in heads])
        o_ref, _ = O.attention_rows(qg[0][rows], rows, kk, vv)
        assert np.max(np.abs(to_np(o[b, heads[0], I_ * 64:I_ * 64 + len(rows)]) - o_ref)) <= TOL["bf16"]
        s_ref = O.token_scores_tile(qg, kk, I_)
        s_gpu = to_np(ts[b, g, I_])
        assert score_rel_err(s_ref, s_gpu) <= 1e-3
        sel = idx[b, g, I_].cpu().numpy().astype(np.int64)
        check_selection(s_ref, s_gpu, sel, O.token_candidates(I_, w.N, w.window), w.topk)
        for h in (heads[0], heads[-1]):
            ref = O.token_sparse_rows(I.sparse_q_slice(w, 0, b, h)[rows], rows, kk, vv, sel, w.window)
            assert np.max(np.abs(to_np(osp[b, h, I_ * 64:I_ * 64 + len(rows)]) - ref)) <= TOL["bf16"]


def _fp8_fill(w, which):
    """The decode workload's FP8 cache codes, generated slice by slice on the host and copied in."""
    from concurrent.futures import ThreadPoolExecutor
    fn = I.decode_k_fp8_slice if which == "k" else I.decode_v_fp8_slice
    out = torch.empty((w.B, w.Hkv, w.N, w.D), dtype=torch.uint8, device="cuda")
    keys = _keys(w, w.Hkv)
    with ThreadPoolExecutor(16) as ex:
        for key, arr in ex.map(lambda key: (key, fn(w, *key)), keys):
            out[key].copy_(torch.from_numpy(arr))
    return out


@pytest.mark.parametrize("cache", ["bf16", "fp8"])
def test_token_decode_fullsize_sampled(cache):
    """Token-variant decode at the bench's size: B64 sequences of L131072, 32/4 heads, D128,
    top-2048 tokens older than the forced newest 128, over a bf16 or an E4M3 cache."""
    w = I.scaled(I.WORKLOADS["decode"], layers=1)
    kt, W = 2048, 128
    bq = _keys(w, w.Hq)
    q = device_fill((w.B, w.Hq, w.D), lambda b, h: I.decode_q_slice(w, b, h), bq)
    qs = device_fill((w.B, w.Hq, w.D), lambda b, h: I.decode_sparse_q_slice(w, 0, b, h), bq)
    if cache == "bf16":
        bk = _keys(w, w.Hkv)
        k = device_fill((w.B, w.Hkv, w.N, w.D), lambda b, g: I.decode_k_slice(w, b, g), bk)
        v = device_fill((w.B, w.Hkv, w.N, w.D), lambda b, g: I.decode_v_slice(w, b, g), bk)
        o, ts = H.full_attn_select_decode_tokens(q, k, v)
        idx = H.topk_decode_tokens(ts, kt, W)
        osp = H.sparse_attn_decode_tokens(qs, k, v, idx, W)
    else:
        k8, v8 = _fp8_fill(w, "k"), _fp8_fill(w, "v")
        ks_np, vs_np = I.fp8_kv_scales(w)
        ks, vs = torch.from_numpy(ks_np).cuda(), torch.from_numpy(vs_np).cuda()
        o, ts = H.full_attn_select_decode_tokens_fp8(q, k8, v8, ks, vs)
        idx = H.topk_decode_tokens(ts, kt, W)
        osp = H.sparse_attn_decode_tokens_fp8(qs, k8, v8, ks, vs, idx, W)
    torch.cuda.synchronize()
    assert H.hysparse_get_device_status() == 0
    for b in (0, 37, w.B - 1):
        qb = np.stack([I.decode_q_slice(w, b, h) for h in range(w.Hq)])[None]
        if cache == "bf16":
            kb = np.stack([I.decode_k_slice(w, b, g) for g in range(w.Hkv)])[None]
            vb = np.stack([I.decode_v_slice(w, b, g) for g in range(w.Hkv)])[None]
        else:
            kb = O.dequant_kv_fp8(np.stack([I.decode_k_fp8_slice(w, b, g) for g in range(w.Hkv)])[None], ks_np)
            vb = O.dequant_kv_fp8(np.stack([I.decode_v_fp8_slice(w, b, g) for g in range(w.Hkv)])[None], vs_np)
        o_ref, _ = O.decode_full(qb, kb, vb)
        assert np.max(np.abs(to_np(o[b]) - o_ref[0])) <= TOL["bf16"]
        s_ref = O.decode_token_scores(qb, kb)[0]
        s_gpu = to_np(ts[b])
        assert score_rel_err(s_ref, s_gpu) <= 1e-3
        sel = idx[b].cpu().numpy().astype(np.int64)
        for g in range(w.Hkv):
            check_selection(s_ref[g], s_gpu[g], sel[g], w.N - W, kt)
        qsb = np.stack([I.decode_sparse_q_slice(w, 0, b, h) for h in range(w.Hq)])[None]
        ref = O.decode_token_sparse(qsb, kb, vb, sel[None], W)
        assert np.max(np.abs(to_np(osp[b]) - ref[0])) <= TOL["bf16"]


def test_rows_fullsize_sampled():
    """Per-position selection at the headline size (moe80b: B2 N32768, 32/4, D128, top-32 blocks
    per query position, SWA 128): sampled tiles' per-row group-max scores, each row's selection,
    and the sparse rows on the GPU's indices."""
    w = I.scaled(I.WORKLOADS["moe80b"], layers=1)
    pl = I.plants(w)
    qsh, kvsh = (w.B, w.Hq, w.N, w.D), (w.B, w.Hkv, w.N, w.D)
    bq, bk = _keys(w, w.Hq), _keys(w, w.Hkv)
    q = device_fill(qsh, lambda b, h: I.q_slice(w, b, h), bq)
    k = device_fill(kvsh, lambda b, g: I.k_slice(w, b, g, pl), bk)
    v = device_fill(kvsh, lambda b, g: I.v_slice(w, b, g), bk)
    qs = device_fill(qsh, lambda b, h: I.sparse_q_slice(w, 0, b, h), bq)
    ks = device_fill(kvsh, lambda b, g: I.swa_k_slice(w, 0, b, g), bk)
    vs = device_fill(kvsh, lambda b, g: I.swa_v_slice(w, 0, b, g), bk)
    gate = device_fill((w.B, w.Hq, w.N, 2), lambda b, h: I.gate_slice(w, 0, b, h), bq, bf16=False)
    _, sc = H.full_attn_select(q, k, v, gran="block_row", reduce="max")
    idx = H.topk_rows(sc, w.topk)
    osp = H.sparse_attn_rows(qs, k, v, idx, ks, vs, w.window, gate)
    torch.cuda.synchronize()
    assert H.hysparse_get_device_status() == 0
    G = w.G
    for b, g, I_ in I.sampled_tiles(w, 3):
        rows = O.tile_rows(I_, w.N)
        heads = list(range(g * G, (g + 1) * G))
        kk, vv = I.k_slice(w, b, g, pl), I.v_slice(w, b, g)
        s_ref = np.zeros((len(rows), w.NB))
        for h in heads:
            p, _, _ = O.causal_softmax(I.q_slice(w, b, h)[rows], rows, kk)
            s_ref = np.maximum(s_ref, O.block_max_probs(p, rows))
        s_gpu = to_np(sc[b, g, I_ * 64:I_ * 64 + len(rows)])
        assert score_rel_err(s_ref, s_gpu) <= 1e-3
        sel = idx[b, g, I_ * 64:I_ * 64 + len(rows)].cpu().numpy().astype(np.int64)
        kss, vss = I.swa_k_slice(w, 0, b, g), I.swa_v_slice(w, 0, b, g)
        for r, t in enumerate(rows):
            assert np.all(s_gpu[r, t // 64 + 1:] == 0)
            check_selection(s_ref[r], s_gpu[r], sel[r], t // 64 + 1, w.topk)
        for h in (heads[0], heads[-1]):
            qh, gh = I.sparse_q_slice(w, 0, b, h), I.gate_slice(w, 0, b, h)
            ref = np.stack([O.gated_sparse_rows(qh[[t]], np.array([t]), kk, vv, sel[r], kss, vss, w.window,
                                                gh[[t]])[0] for r, t in enumerate(rows)])
            assert np.max(np.abs(to_np(osp[b, h, I_ * 64:I_ * 64 + len(rows)]) - ref)) <= TOL["bf16"]
