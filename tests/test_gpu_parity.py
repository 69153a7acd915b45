"""GPU parity of every entry point against the float64 oracle on small seeded cases
(several tiles and a ragged tail), called through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as O
from attention_tcgen05_tma_b200 import hysparse as H
from attention_tcgen05_tma_b200 import inputs as I
from tests.gpu_support import TOL, check_selection, score_rel_err, to_dev, to_np

pytestmark = pytest.mark.gpu

PREFILL_CASES = [
    # name, dtype, B, N, Hq, Hkv, D, k, window
    ("tiny_fp32", "f32", 1, 1024, 4, 1, 64, 4, 128),
    ("bf16_d128_g4_ragged", "bf16", 2, 1000, 8, 2, 128, 4, 128),
    ("bf16_d64_g8", "bf16", 1, 333, 8, 1, 64, 3, 100),
    ("bf16_d128_g2_k_large", "bf16", 1, 700, 4, 2, 128, 16, 64),
    ("f32_d128_g1", "f32", 1, 200, 2, 2, 128, 2, 300),
    ("bf16_d128_g16", "bf16", 1, 200, 16, 1, 128, 2, 128),
    ("bf16_d128_g8_many_units", "bf16", 2, 2048, 32, 4, 128, 8, 128),
]


def _workload(dtype, B, N, Hq, Hkv, D, k, window, seed=11):
    base = I.WORKLOADS["tiny"] if dtype == "f32" else I.WORKLOADS["dense7b"]
    return I.scaled(base, B=B, N=N, Hq=Hq, Hkv=Hkv, D=D, topk=k, window=window, layers=1, seed=seed,
                    scale_std=1.0 if dtype == "f32" else 1.0 / np.sqrt(D), n_plants=min(8, N // 64))


@pytest.mark.parametrize("case", PREFILL_CASES, ids=[c[0] for c in PREFILL_CASES])
@pytest.mark.parametrize("reduce", ["sum", "max"])
def test_hybrid_block_prefill(case, reduce):
    name, dt, B, N, Hq, Hkv, D, k, window = case
    w = _workload(dt, B, N, Hq, Hkv, D, k, window)
    a = I.prefill_arrays(w, layers=1)
    q, kk, vv = (to_dev(a[x], dt) for x in ("q", "k", "v"))
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
    o, sc = H.full_attn_select(q, kk, vv, reduce=reduce, lse=lse)
    idx = H.topk(sc, k)
    qs, ks, vs = (to_dev(a[x][0], dt) for x in ("q_sparse", "k_swa", "v_swa"))
    gate = to_dev(a["gate"][0], "f32")
    osp = H.sparse_attn(qs, kk, vv, idx, ks, vs, window, gate)
    torch.cuda.synchronize()

    o_ref, lse_ref = O.full_attention(a["q"], a["k"], a["v"])
    assert np.max(np.abs(to_np(o) - o_ref)) <= TOL[dt]
    assert np.max(np.abs(to_np(lse) - lse_ref)) <= 1e-3
    sc_ref = O.block_scores(a["q"], a["k"], reduce)
    sc_gpu = to_np(sc)
    assert score_rel_err(sc_ref, sc_gpu) <= 1e-3
    assert np.all(sc_gpu >= 0)
    T = sc_ref.shape[2]
    for I_ in range(T):
        assert np.all(sc_gpu[:, :, I_, I_ + 1:] == 0)
    gidx = idx.cpu().numpy().astype(np.int64)
    for b in range(B):
        for g in range(Hkv):
            for I_ in range(T):
                check_selection(sc_ref[b, g, I_], sc_gpu[b, g, I_], gidx[b, g, I_], I_ + 1, k)
    ref = O.sparse_attention(a["q_sparse"][0], a["k"], a["v"], gidx, a["k_swa"][0], a["v_swa"][0], window,
                             a["gate"][0])
    assert np.max(np.abs(to_np(osp) - ref)) <= TOL[dt]


@pytest.mark.parametrize("N", [1, 63, 64, 65, 129])
def test_edge_lengths(N):
    w = _workload("bf16", 1, N, 4, 2, 128, 2, 128, seed=N)
    a = I.prefill_arrays(w, layers=1)
    q, kk, vv = (to_dev(a[x], "bf16") for x in ("q", "k", "v"))
    o, sc = H.full_attn_select(q, kk, vv)
    idx = H.topk(sc, 2)
    qs, ks, vs = (to_dev(a[x][0], "bf16") for x in ("q_sparse", "k_swa", "v_swa"))
    osp = H.sparse_attn(qs, kk, vv, idx, ks, vs, 128, to_dev(a["gate"][0], "f32"))
    torch.cuda.synchronize()
    o_ref, _ = O.full_attention(a["q"], a["k"], a["v"])
    assert np.max(np.abs(to_np(o) - o_ref)) <= TOL["bf16"]
    gidx = idx.cpu().numpy().astype(np.int64)
    assert np.all(gidx[..., 0] == 0)    # block 0 is always a candidate
    ref = O.sparse_attention(a["q_sparse"][0], a["k"], a["v"], gidx, a["k_swa"][0], a["v_swa"][0], 128,
                             a["gate"][0])
    assert np.max(np.abs(to_np(osp) - ref)) <= TOL["bf16"]


def test_share_both_ablation_aliasing():
    """K'/V' may alias the shared K/V ("share both" ablation)."""
    w = _workload("bf16", 1, 300, 4, 1, 64, 2, 64)
    a = I.prefill_arrays(w, layers=1)
    q, kk, vv = (to_dev(a[x], "bf16") for x in ("q", "k", "v"))
    _, sc = H.full_attn_select(q, kk, vv)
    idx = H.topk(sc, 2)
    qs = to_dev(a["q_sparse"][0], "bf16")
    osp = H.sparse_attn(qs, kk, vv, idx, kk, vv, 64, to_dev(a["gate"][0], "f32"))
    torch.cuda.synchronize()
    gidx = idx.cpu().numpy().astype(np.int64)
    ref = O.sparse_attention(a["q_sparse"][0], a["k"], a["v"], gidx, a["k"], a["v"], 64, a["gate"][0])
    assert np.max(np.abs(to_np(osp) - ref)) <= TOL["bf16"]


def test_output_alignment_16_bytes():
    """Output rows at a 16-byte (not 32-byte) aligned address take the 128-bit store path of the
    tensor-core kernels; the values match the aligned call's exactly."""
    w = _workload("bf16", 1, 700, 8, 2, 128, 4, 128)
    a = I.prefill_arrays(w, layers=1)
    q, kk, vv = (to_dev(a[x], "bf16") for x in ("q", "k", "v"))
    o_al, sc = H.full_attn_select(q, kk, vv)
    buf = torch.empty(q.numel() + 8, dtype=q.dtype, device=q.device)
    o_un = buf[8:].view(q.shape)                      # 16 bytes past a 256-byte aligned base
    assert o_un.data_ptr() % 32 == 16
    H.full_attn_select(q, kk, vv, o=o_un, scores=torch.empty_like(sc))
    idx = H.topk(sc, 4)
    qs, gate = to_dev(a["q_sparse"][0], "bf16"), to_dev(a["gate"][0], "f32")
    ks, vs = to_dev(a["k_swa"][0], "bf16"), to_dev(a["v_swa"][0], "bf16")
    s_al = H.sparse_attn(qs, kk, vv, idx, ks, vs, 128, gate)
    buf2 = torch.empty(qs.numel() + 8, dtype=qs.dtype, device=qs.device)
    s_un = buf2[8:].view(qs.shape)
    H.sparse_attn(qs, kk, vv, idx, ks, vs, 128, gate, o=s_un)
    torch.cuda.synchronize()
    assert torch.equal(o_al, o_un) and torch.equal(s_al, s_un)


TOKEN_CASES = [
    ("bf16_d128", "bf16", 1, 700, 8, 2, 128, 100, 128),
    ("bf16_d64_small_forced", "bf16", 1, 300, 4, 1, 64, 40, 16),
    ("f32_d64", "f32", 1, 400, 4, 1, 64, 64, 128),
    ("bf16_d128_g8_rounds", "bf16", 1, 1500, 16, 2, 128, 300, 128),
    # four or more M-tiles per unit run on CTA pairs: D 64, three M-tiles (one idle slot), two
    # rounds of four, fewer units than the device holds clusters
    ("bf16_d64_g8_pair", "bf16", 1, 900, 8, 1, 64, 120, 128),
    ("bf16_d128_g6_pair_b2", "bf16", 2, 1000, 12, 2, 128, 200, 64),
    ("bf16_d128_g16_pair_2rounds", "bf16", 1, 700, 16, 1, 128, 150, 128),
]


@pytest.mark.parametrize("case", TOKEN_CASES, ids=[c[0] for c in TOKEN_CASES])
def test_token_variant(case):
    name, dt, B, N, Hq, Hkv, D, kt, forced = case
    w = _workload(dt, B, N, Hq, Hkv, D, kt, forced)
    a = I.prefill_arrays(w, layers=1)
    q, kk, vv = (to_dev(a[x], dt) for x in ("q", "k", "v"))
    o, ts = H.full_attn_select(q, kk, vv, gran="token")
    idx = H.topk_tokens(ts, kt, forced)
    qs = to_dev(a["q_sparse"][0], dt)
    osp = H.sparse_attn_tokens(qs, kk, vv, idx, forced)
    torch.cuda.synchronize()
    o_ref, _ = O.full_attention(a["q"], a["k"], a["v"])
    assert np.max(np.abs(to_np(o) - o_ref)) <= TOL[dt]
    ts_gpu = to_np(ts)
    gidx = idx.cpu().numpy().astype(np.int64)
    G = Hq // Hkv
    T = (N + 63) // 64
    for b in range(B):
        for g in range(Hkv):
            qg = a["q"][b, g * G:(g + 1) * G]
            for I_ in range(T):
                ref_ts = O.token_scores_tile(qg, a["k"][b, g], I_)
                assert score_rel_err(ref_ts, ts_gpu[b, g, I_]) <= 1e-3
                nc = O.token_candidates(I_, N, forced)
                check_selection(ref_ts, ts_gpu[b, g, I_], gidx[b, g, I_], nc, kt)
                rows = O.tile_rows(I_, N)
                for h in range(g * G, (g + 1) * G):
                    ref = O.token_sparse_rows(a["q_sparse"][0][b, h, rows], rows, a["k"][b, g], a["v"][b, g],
                                              gidx[b, g, I_], forced)
                    assert np.max(np.abs(to_np(osp[b, h, rows]) - ref)) <= TOL[dt]


DECODE_CASES = [
    ("bf16_d128_g8", "bf16", 3, 1500, 16, 2, 128, 4, 128, True),
    ("bf16_d64_g4", "bf16", 2, 700, 4, 1, 64, 8, 32, False),
    ("f32_d64_g4", "f32", 2, 300, 8, 2, 64, 2, 16, True),
    ("bf16_d128_g16_long", "bf16", 2, 9000, 16, 1, 128, 8, 128, True),
    ("bf16_d128_g4_ring100", "bf16", 2, 3000, 8, 2, 128, 4, 100, False),
    ("bf16_d128_g8_stage_reuse", "bf16", 64, 40000, 8, 1, 128, 32, 128, True),
]


@pytest.mark.parametrize("case", DECODE_CASES, ids=[c[0] for c in DECODE_CASES])
def test_decode(case):
    name, dt, B, L, Hq, Hkv, D, k, W, ragged = case
    w = I.scaled(I.WORKLOADS["decode"], B=B, N=L, Hq=Hq, Hkv=Hkv, D=D, topk=k, window=W, layers=1, seed=5,
                 scale_std=1.0 / np.sqrt(D))
    a = I.decode_arrays(w, layers=1)
    seqlens = np.array([L - 37 * b for b in range(B)], dtype=np.int32) if ragged else None
    # ragged rings, including an empty one (a sequence with no window tokens yet)
    swa_len = np.array([(W - 3 * b) % (W + 1) for b in range(B)], dtype=np.int32) if ragged else None
    q, kc, vc = (to_dev(a[x], dt) for x in ("q", "k", "v"))
    sl = torch.from_numpy(seqlens).cuda() if ragged else None
    o, sc = H.full_attn_select_decode(q, kc, vc, seqlens=sl)
    idx = H.topk_decode(sc, k, L, seqlens=sl)
    qs, kr, vr = (to_dev(a[x][0], dt) for x in ("q_sparse", "k_swa", "v_swa"))
    gate = to_dev(a["gate"][0], "f32")
    swl = torch.from_numpy(swa_len).cuda() if ragged else None
    osp = H.sparse_attn_decode(qs, kc, vc, idx, kr, vr, gate, seqlens=sl, swa_len=swl)
    torch.cuda.synchronize()
    o_ref, sc_ref = O.decode_full(a["q"], a["k"], a["v"], seqlens)
    assert np.max(np.abs(to_np(o) - o_ref)) <= TOL[dt]
    sc_gpu = to_np(sc)
    assert score_rel_err(sc_ref, sc_gpu) <= 1e-3
    gidx = idx.cpu().numpy().astype(np.int64)
    for b in range(B):
        nb = ((int(seqlens[b]) if seqlens is not None else L) + 63) // 64
        for g in range(Hkv):
            check_selection(sc_ref[b, g], sc_gpu[b, g], gidx[b, g], nb, k)
    ref = O.decode_sparse(a["q_sparse"][0], a["k"], a["v"], gidx, a["k_swa"][0], a["v_swa"][0], a["gate"][0],
                          seqlens, swa_len)
    assert np.max(np.abs(to_np(osp) - ref)) <= TOL[dt]


ROW_PREFILL_CASES = [
    # name, B, N, Hq, Hkv, D, k, window, with sinks
    ("d128_g4_ragged", 2, 1000, 8, 2, 128, 4, 128, False),
    ("d64_g8", 1, 333, 8, 1, 64, 3, 100, True),
    ("d128_g2_k_all", 1, 700, 4, 2, 128, 16, 64, False),     # k covers every block: dense branch
    ("d128_g8_many_units", 1, 2048, 16, 2, 128, 6, 128, False),
]


@pytest.mark.parametrize("case", ROW_PREFILL_CASES, ids=[c[0] for c in ROW_PREFILL_CASES])
def test_per_position_selection(case):
    """Per-position selection ([HS] 3.4.1-3.4.2 as printed): group-max scores [B,Hkv,N,NB], the
    top k of each row's floor(t/64)+1 blocks, and the sparse layer with each row's own blocks,
    against the oracle (the sparse rows on the GPU's own indices)."""
    name, B, N, Hq, Hkv, D, k, window, with_sinks = case
    w = _workload("bf16", B, N, Hq, Hkv, D, k, window, seed=17)
    a = I.prefill_arrays(w, layers=1)
    q, kk, vv = (to_dev(a[x], "bf16") for x in ("q", "k", "v"))
    o, sc = H.full_attn_select(q, kk, vv, gran="block_row", reduce="max")
    idx = H.topk_rows(sc, k)
    qs, ks, vs = (to_dev(a[x][0], "bf16") for x in ("q_sparse", "k_swa", "v_swa"))
    gate = to_dev(a["gate"][0], "f32")
    sinks = I.sink_logits(w, 0) if with_sinks else None
    osp = H.sparse_attn_rows(qs, kk, vv, idx, ks, vs, window, gate,
                             sinks=torch.from_numpy(sinks).cuda() if with_sinks else None)
    torch.cuda.synchronize()
    assert H.hysparse_get_device_status() == 0
    o_ref, _ = O.full_attention(a["q"], a["k"], a["v"])
    assert np.max(np.abs(to_np(o) - o_ref)) <= TOL["bf16"]
    sc_ref = O.block_scores_rows(a["q"], a["k"])
    sc_gpu = to_np(sc)
    assert sc_gpu.shape == sc_ref.shape
    assert score_rel_err(sc_ref, sc_gpu) <= 1e-3
    NB = sc_ref.shape[3]
    gidx = idx.cpu().numpy().astype(np.int64)
    for b in range(B):
        for g in range(Hkv):
            for t in range(N):
                assert np.all(sc_gpu[b, g, t, t // 64 + 1:] == 0)
                check_selection(sc_ref[b, g, t], sc_gpu[b, g, t], gidx[b, g, t], min(NB, t // 64 + 1), k)
    ref = O.sparse_attention_rows(a["q_sparse"][0], a["k"], a["v"], gidx, a["k_swa"][0], a["v_swa"][0], window,
                                  a["gate"][0], sinks=sinks)
    assert np.max(np.abs(to_np(osp) - ref)) <= TOL["bf16"]
    if name.endswith("k_all"):   # every row keeps all its blocks: the per-tile layer with all blocks
        tidx = H.topk(H.full_attn_select(q, kk, vv)[1], k)
        otile = H.sparse_attn(qs, kk, vv, tidx, ks, vs, window, gate)
        torch.cuda.synchronize()
        assert np.max(np.abs(to_np(osp) - to_np(otile))) <= TOL["bf16"]


SINK_PREFILL_CASES = [
    # name, dtype, B, N, Hq, Hkv, D, k, window  (tensor-core path for bf16 D in {64,128}, even G)
    ("bf16_d128_g4_tc", "bf16", 1, 700, 8, 2, 128, 4, 128),
    ("bf16_d64_g8_tc", "bf16", 1, 333, 8, 1, 64, 3, 100),
    ("f32_d64_g4_simt", "f32", 1, 300, 4, 1, 64, 3, 64),
]


@pytest.mark.parametrize("case", SINK_PREFILL_CASES, ids=[c[0] for c in SINK_PREFILL_CASES])
def test_sparse_layer_sinks(case):
    """Per-head sink logits of both branches ([HSP] 4.1): parity with the oracle, and sinks of
    -inf reproduce the call without sinks exactly."""
    name, dt, B, N, Hq, Hkv, D, k, window = case
    w = _workload(dt, B, N, Hq, Hkv, D, k, window)
    a = I.prefill_arrays(w, layers=1)
    q, kk, vv = (to_dev(a[x], dt) for x in ("q", "k", "v"))
    _, sc = H.full_attn_select(q, kk, vv)
    idx = H.topk(sc, k)
    qs, ks, vs = (to_dev(a[x][0], dt) for x in ("q_sparse", "k_swa", "v_swa"))
    gate = to_dev(a["gate"][0], "f32")
    sinks = I.sink_logits(w, 0)
    osp = H.sparse_attn(qs, kk, vv, idx, ks, vs, window, gate, sinks=torch.from_numpy(sinks).cuda())
    none = H.sparse_attn(qs, kk, vv, idx, ks, vs, window, gate)
    neg = H.sparse_attn(qs, kk, vv, idx, ks, vs, window, gate,
                        sinks=torch.full((Hq, 2), float("-inf"), device="cuda"))
    torch.cuda.synchronize()
    gidx = idx.cpu().numpy().astype(np.int64)
    ref = O.sparse_attention(a["q_sparse"][0], a["k"], a["v"], gidx, a["k_swa"][0], a["v_swa"][0], window,
                             a["gate"][0], sinks=sinks.astype(np.float64))
    assert np.max(np.abs(to_np(osp) - ref)) <= TOL[dt]
    assert torch.equal(none, neg)


@pytest.mark.parametrize("dt,D,Hq,Hkv", [("bf16", 128, 16, 2), ("f32", 64, 8, 2)], ids=["mma", "simt"])
def test_decode_sinks(dt, D, Hq, Hkv):
    B, L, k, W = 3, 1500, 4, 128
    w = I.scaled(I.WORKLOADS["decode"], B=B, N=L, Hq=Hq, Hkv=Hkv, D=D, topk=k, window=W, layers=1, seed=8,
                 scale_std=1.0 / np.sqrt(D))
    a = I.decode_arrays(w, layers=1)
    swa_len = np.array([W, 0, 37], dtype=np.int32)          # an empty ring: its branch gives zero
    q, kc, vc = (to_dev(a[x], dt) for x in ("q", "k", "v"))
    _, sc = H.full_attn_select_decode(q, kc, vc)
    idx = H.topk_decode(sc, k, L)
    qs, kr, vr = (to_dev(a[x][0], dt) for x in ("q_sparse", "k_swa", "v_swa"))
    gate = to_dev(a["gate"][0], "f32")
    sinks = I.sink_logits(w, 0)
    osp = H.sparse_attn_decode(qs, kc, vc, idx, kr, vr, gate, swa_len=torch.from_numpy(swa_len).cuda(),
                               sinks=torch.from_numpy(sinks).cuda())
    torch.cuda.synchronize()
    gidx = idx.cpu().numpy().astype(np.int64)
    ref = O.decode_sparse(a["q_sparse"][0], a["k"], a["v"], gidx, a["k_swa"][0], a["v_swa"][0], a["gate"][0],
                          None, swa_len, sinks=sinks.astype(np.float64))
    assert np.max(np.abs(to_np(osp) - ref)) <= TOL[dt]


TOKEN_DECODE_CASES = [
    # name, B, L, Hq, Hkv, k_tokens, forced, ragged
    ("g8_ragged", 3, 1500, 16, 2, 100, 64, True),
    ("g16_long", 2, 5000, 16, 1, 700, 128, False),
    ("g8_keep_all", 2, 600, 16, 2, 4096, 64, True),    # every candidate kept: dense decode
    ("g8_odd_L", 2, 1001, 16, 2, 90, 64, True),        # cache length not a multiple of 4
]


@pytest.mark.parametrize("case", TOKEN_DECODE_CASES, ids=[c[0] for c in TOKEN_DECODE_CASES])
def test_token_decode(case):
    name, B, L, Hq, Hkv, kt, W, ragged = case
    D = 128
    w = I.scaled(I.WORKLOADS["decode"], B=B, N=L, Hq=Hq, Hkv=Hkv, D=D, topk=kt, window=W, layers=1, seed=12,
                 scale_std=1.0 / np.sqrt(D))
    a = I.decode_arrays(w, layers=1)
    seqlens = np.array([L - 211 * b for b in range(B)], dtype=np.int32) if ragged else None
    q, kc, vc = (to_dev(a[x], "bf16") for x in ("q", "k", "v"))
    sl = torch.from_numpy(seqlens).cuda() if ragged else None
    o, ts = H.full_attn_select_decode_tokens(q, kc, vc, seqlens=sl)
    idx = H.topk_decode_tokens(ts, kt, W, seqlens=sl)
    qs = to_dev(a["q_sparse"][0], "bf16")
    osp = H.sparse_attn_decode_tokens(qs, kc, vc, idx, W, seqlens=sl)
    torch.cuda.synchronize()
    assert H.hysparse_get_device_status() == 0
    o_ref, _ = O.decode_full(a["q"], a["k"], a["v"], seqlens)
    assert np.max(np.abs(to_np(o) - o_ref)) <= TOL["bf16"]
    ts_ref = O.decode_token_scores(a["q"], a["k"], seqlens)
    ts_gpu = to_np(ts)
    assert score_rel_err(ts_ref, ts_gpu) <= 1e-3
    gidx = idx.cpu().numpy().astype(np.int64)
    for b in range(B):
        Lb = int(seqlens[b]) if ragged else L
        assert np.all(ts_gpu[b, :, Lb:] == 0)
        for g in range(Hkv):
            check_selection(ts_ref[b, g], ts_gpu[b, g], gidx[b, g], max(0, Lb - W), kt)
    ref = O.decode_token_sparse(a["q_sparse"][0], a["k"], a["v"], gidx, W, seqlens)
    assert np.max(np.abs(to_np(osp) - ref)) <= TOL["bf16"]
    if name == "g8_keep_all":   # every candidate selected: the sparse layer is dense decode of q'
        dense, _ = O.decode_full(a["q_sparse"][0], a["k"], a["v"], seqlens)
        assert np.max(np.abs(to_np(osp) - dense)) <= TOL["bf16"]


@pytest.mark.parametrize("case", TOKEN_DECODE_CASES, ids=[c[0] for c in TOKEN_DECODE_CASES])
def test_token_decode_fp8(case):
    """Token-variant decode over an E4M3 cache with per-KV-head K and V scales, against the
    oracle run on the decoded cache values."""
    name, B, L, Hq, Hkv, kt, W, ragged = case
    D = 128
    w = I.scaled(I.WORKLOADS["decode"], B=B, N=L, Hq=Hq, Hkv=Hkv, D=D, topk=kt, window=W, layers=1, seed=13,
                 scale_std=1.0 / np.sqrt(D))
    a = I.decode_arrays(w, layers=1)
    c = I.decode_fp8_cache(w)
    kd, vd = O.dequant_kv_fp8(c["k8"], c["k_scale"]), O.dequant_kv_fp8(c["v8"], c["v_scale"])
    seqlens = np.array([L - 211 * b for b in range(B)], dtype=np.int32) if ragged else None
    q, qs = to_dev(a["q"], "bf16"), to_dev(a["q_sparse"][0], "bf16")
    k8, v8 = torch.from_numpy(c["k8"]).cuda(), torch.from_numpy(c["v8"]).cuda()
    ks, vs = torch.from_numpy(c["k_scale"]).cuda(), torch.from_numpy(c["v_scale"]).cuda()
    sl = torch.from_numpy(seqlens).cuda() if ragged else None
    o, ts = H.full_attn_select_decode_tokens_fp8(q, k8, v8, ks, vs, seqlens=sl)
    idx = H.topk_decode_tokens(ts, kt, W, seqlens=sl)
    osp = H.sparse_attn_decode_tokens_fp8(qs, k8, v8, ks, vs, idx, W, seqlens=sl)
    torch.cuda.synchronize()
    assert H.hysparse_get_device_status() == 0
    o_ref, _ = O.decode_full(a["q"], kd, vd, seqlens)
    assert np.max(np.abs(to_np(o) - o_ref)) <= TOL["bf16"]
    ts_ref = O.decode_token_scores(a["q"], kd, seqlens)
    ts_gpu = to_np(ts)
    assert score_rel_err(ts_ref, ts_gpu) <= 1e-3
    gidx = idx.cpu().numpy().astype(np.int64)
    for b in range(B):
        Lb = int(seqlens[b]) if ragged else L
        assert np.all(ts_gpu[b, :, Lb:] == 0)
        for g in range(Hkv):
            check_selection(ts_ref[b, g], ts_gpu[b, g], gidx[b, g], max(0, Lb - W), kt)
    ref = O.decode_token_sparse(a["q_sparse"][0], kd, vd, gidx, W, seqlens)
    assert np.max(np.abs(to_np(osp) - ref)) <= TOL["bf16"]
    if name == "g8_keep_all":
        dense, _ = O.decode_full(a["q_sparse"][0], kd, vd, seqlens)
        assert np.max(np.abs(to_np(osp) - dense)) <= TOL["bf16"]
