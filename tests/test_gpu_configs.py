"""Parity of the stated workloads exactly as configured, through the C ABI, against the oracle.

* tiny fp32 hybrid block (seed 0): B1 N1024, 4 query heads / 1 KV head, D64, 8 planted keys,
  one full layer and 3 sparse layers (each with its own Q', K', V' and gate logits), top-4 blocks,
  SWA 128; checked in full (every output element, every tile's scores and selection).
* 7B-dense-shaped 1:3 block, bf16: B1 N8192, 32/8 heads, D128, 64 planted key blocks, one full
  layer and 3 sparse layers, top-16 blocks, SWA 128, run in full on the GPU exactly as the
  benchmark's dense7b leg runs it; checked on every query tile of KV group 0, the tile of every
  planted block's query and the last tile of every group.

Selection: rules 1/2 per tile, and per block the candidates that clear the k-th/(k+1)-th boundary
by more than the gap plus the GPU's own score error are decided exactly (tests/gpu_support.py).
On the bf16 workloads the unplanted blocks' scores are near ties (query-key logits have a
standard deviation of about 0.008), so most tiles fall under rule 2 while every planted block is
decided in its query's tile."""
import numpy as np
import pytest
import torch

import oracle as O
from attention_tcgen05_tma_b200 import hysparse as H
from attention_tcgen05_tma_b200 import inputs as I
from tests.gpu_support import TOL, check_selection, device_fill, score_rel_err, to_dev, to_np

pytestmark = pytest.mark.gpu


def test_tiny_fp32_config_as_stated():
    w = I.WORKLOADS["tiny"]
    assert (w.dtype, w.seed, w.B, w.N, w.Hq, w.Hkv, w.D, w.layers, w.topk, w.window) == \
        ("f32", 0, 1, 1024, 4, 1, 64, 3, 4, 128)
    a = I.prefill_arrays(w)
    q, kk, vv = (to_dev(a[x], "f32") for x in ("q", "k", "v"))
    o, sc = H.full_attn_select(q, kk, vv)
    idx = H.topk(sc, w.topk)
    outs = []
    for l in range(w.layers):
        qs, ks, vs = (to_dev(a[x][l], "f32") for x in ("q_sparse", "k_swa", "v_swa"))
        outs.append(H.sparse_attn(qs, kk, vv, idx, ks, vs, w.window, to_dev(a["gate"][l], "f32")))
    torch.cuda.synchronize()
    assert H.hysparse_get_device_status() == 0

    o_ref, _ = O.full_attention(a["q"], a["k"], a["v"])
    assert np.max(np.abs(to_np(o) - o_ref)) <= TOL["f32"]
    sc_ref = O.block_scores(a["q"], a["k"])
    sc_gpu = to_np(sc)
    assert score_rel_err(sc_ref, sc_gpu) <= 1e-3
    gidx = idx.cpu().numpy().astype(np.int64)
    rules = [check_selection(sc_ref[0, 0, t], sc_gpu[0, 0, t], gidx[0, 0, t], t + 1, w.topk)["rule"]
             for t in range(w.T)]
    # the fp32 workload's logits have unit scale: clear gaps, so rule 1 decides most tiles (14 of 16 on the oracle)
    assert rules.count("rule1") >= 0.75 * w.T, rules.count("rule1")
    for l in range(w.layers):
        ref = O.sparse_attention(a["q_sparse"][l], a["k"], a["v"], gidx, a["k_swa"][l], a["v_swa"][l], w.window,
                                 a["gate"][l])
        assert np.max(np.abs(to_np(outs[l]) - ref)) <= TOL["f32"], l


def _keys(w, heads):
    return [(b, h) for b in range(w.B) for h in range(heads)]


def test_dense7b_config_fullsize():
    w = I.WORKLOADS["dense7b"]
    assert (w.dtype, w.B, w.N, w.Hq, w.Hkv, w.D, w.layers, w.topk, w.window, w.n_plants) == \
        ("bf16", 1, 8192, 32, 8, 128, 3, 16, 128, 64)
    pl = I.plants(w)
    qsh, kvsh = (w.B, w.Hq, w.N, w.D), (w.B, w.Hkv, w.N, w.D)
    bq, bk = _keys(w, w.Hq), _keys(w, w.Hkv)
    q = device_fill(qsh, lambda b, h: I.q_slice(w, b, h), bq)
    k = device_fill(kvsh, lambda b, g: I.k_slice(w, b, g, pl), bk)
    v = device_fill(kvsh, lambda b, g: I.v_slice(w, b, g), bk)
    o, sc = H.full_attn_select(q, k, v)
    idx = H.topk(sc, w.topk)
    outs = []
    for l in range(w.layers):
        qs = device_fill(qsh, lambda b, h: I.sparse_q_slice(w, l, b, h), bq)
        ks = device_fill(kvsh, lambda b, g: I.swa_k_slice(w, l, b, g), bk)
        vs = device_fill(kvsh, lambda b, g: I.swa_v_slice(w, l, b, g), bk)
        gate = device_fill((w.B, w.Hq, w.N, 2), lambda b, h: I.gate_slice(w, l, b, h), bq, bf16=False)
        outs.append(H.sparse_attn(qs, k, v, idx, ks, vs, w.window, gate))
        del qs, ks, vs, gate
    torch.cuda.synchronize()
    assert H.hysparse_get_device_status() == 0
    o_np = o.float().cpu().numpy()
    outs_np = [x.float().cpu().numpy() for x in outs]
    sc_np = sc.cpu().numpy().astype(np.float64)
    idx_np = idx.cpu().numpy().astype(np.int64)

    planted = {}                                           # (b, g, query tile) -> planted blocks
    for p in pl:
        planted.setdefault((p.b, p.g, p.t // 64), []).append(p.pos // 64)
    tiles = {(0, 0, t) for t in range(w.T)} | set(planted) | {(0, g, w.T - 1) for g in range(w.Hkv)}
    G = w.G
    rules, n_planted_checked = {"rule1": 0, "rule2": 0}, 0
    for b, g in sorted({(b, g) for b, g, _ in tiles}):
        heads = list(range(g * G, (g + 1) * G))
        kk, vv = I.k_slice(w, b, g, pl), I.v_slice(w, b, g)
        qg = np.stack([I.q_slice(w, b, h) for h in heads])
        layer_in = [(np.stack([I.sparse_q_slice(w, l, b, h) for h in heads]), I.swa_k_slice(w, l, b, g),
                     I.swa_v_slice(w, l, b, g), np.stack([I.gate_slice(w, l, b, h) for h in heads]))
                    for l in range(w.layers)]
        for I_ in sorted(t for bb, gg, t in tiles if (bb, gg) == (b, g)):
            rows = O.tile_rows(I_, w.N)
            sl = slice(I_ * 64, I_ * 64 + len(rows))
            for j, h in enumerate(heads):
                o_ref, _ = O.attention_rows(qg[j][rows], rows, kk, vv)
                assert np.max(np.abs(o_np[b, h, sl] - o_ref)) <= TOL["bf16"], (b, h, I_)
            s_ref = O.block_scores_tile(qg, kk, I_)
            s_gpu = sc_np[b, g, I_]
            assert score_rel_err(s_ref, s_gpu) <= 1e-3
            assert np.all(s_gpu[I_ + 1:] == 0)
            sel = idx_np[b, g, I_]
            dec = check_selection(s_ref, s_gpu, sel, I_ + 1, w.topk)
            rules[dec["rule"]] += 1
            for j in planted.get((b, g, I_), []):
                assert j in dec["decided_in"] and j in sel, (b, g, I_, j)
                n_planted_checked += 1
            for l, (qs_l, ks_l, vs_l, gt_l) in enumerate(layer_in):
                for j, h in enumerate(heads):
                    ref = O.gated_sparse_rows(qs_l[j][rows], rows, kk, vv, sel, ks_l, vs_l, w.window, gt_l[j][rows])
                    assert np.max(np.abs(outs_np[l][b, h, sl] - ref)) <= TOL["bf16"], (l, b, h, I_)
    assert n_planted_checked == sum(len(v) for v in planted.values())
    assert rules["rule1"] + rules["rule2"] == len(tiles)
    print(f"dense7b: {len(tiles)} tiles checked, rule1 {rules['rule1']}, rule2 {rules['rule2']}, "
          f"{n_planted_checked} planted blocks decided in their query's tile")
