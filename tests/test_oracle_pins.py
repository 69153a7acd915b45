"""Pins of the float64 oracle against facts fixed outside the oracle itself.

* a hand-worked example with exact fractions (tests/golden/worked_example_block2.txt);
* a library routine: torch's CPU scaled_dot_product_attention in float64;
* closed forms (zero queries, one dominant key, saturated gates);
* invariants stated by the pages (k covering every block -> dense attention,
  window >= N -> dense attention, selected indices never past the causal
  position, forced tokens always attended);
* brute force: a scalar pure-Python transcription on N <= 256.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
from tests import brute_force as BF

GOLD = os.path.join(os.path.dirname(__file__), "golden", "worked_example_block2.txt")


def _gold():
    vals = {}
    with open(GOLD) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rest = line.split(":", 1)
            vals[key.strip()] = np.array([float(Fraction(x)) for x in rest.split()])
    return vals


def _sdpa(q, k, v):
    """torch float64 causal SDPA with GQA by repeating K/V heads. q [Hq,N,D], k/v [Hkv,N,D]."""
    G = q.shape[0] // k.shape[0]
    kk = torch.from_numpy(np.repeat(k, G, axis=0)).double()
    vv = torch.from_numpy(np.repeat(v, G, axis=0)).double()
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).double(), kk, vv, is_causal=True).numpy()


def _rand(rng, *shape):
    return rng.standard_normal(shape)


# ----------------------------------------------------------------------------- worked example
class TestWorkedExample:
    g = _gold()
    q = np.ones((1, 1, 4, 1))
    k = np.array([0.0, math.log(2.0), 0.0, math.log(3.0)]).reshape(1, 1, 4, 1)
    v = np.array([1.0, 2.0, 3.0, 4.0]).reshape(1, 1, 4, 1)

    def test_dense(self):
        o, lse = O.full_attention(self.q, self.k, self.v)
        np.testing.assert_allclose(o[0, 0, :, 0], self.g["o"], rtol=0, atol=1e-13)
        np.testing.assert_allclose(np.exp(lse[0, 0]), self.g["lse_exp"], rtol=1e-13)

    def test_block_max(self):
        rows = np.arange(4)
        p, _, _ = O.causal_softmax(self.q[0, 0], rows, self.k[0, 0])
        s = O.block_max_probs(p, rows, block=2)
        for t in range(4):
            np.testing.assert_allclose(s[t], self.g[f"smax_t{t}"], atol=1e-13)

    @pytest.mark.parametrize("red", ["sum", "max"])
    def test_scores_and_topk(self, red):
        sc = O.block_scores(self.q, self.k, red, block=2)
        for I in range(2):
            np.testing.assert_allclose(sc[0, 0, I], self.g[f"score_{red}_tile{I}"], atol=1e-13)
        idx = O.topk_blocks(sc, 1)
        assert idx[0, 0, 0, 0] == self.g["topk1_tile0"][0]
        assert idx[0, 0, 1, 0] == self.g["topk1_tile1"][0]

    def test_sparse_layer(self):
        sel = np.zeros((1, 1, 2, 1), dtype=np.int64)
        rows = np.arange(4)
        o_sp = np.concatenate([O.sparse_branch_rows(self.q[0, 0][r], r, self.k[0, 0], self.v[0, 0], [0], 2)
                               for r in (rows[:2], rows[2:])])[:, 0]
        np.testing.assert_allclose(o_sp, self.g["sparse_branch"], atol=1e-13)
        o_sw = O.swa_branch_rows(self.q[0, 0], rows, self.k[0, 0], self.v[0, 0], 1)[:, 0]
        np.testing.assert_allclose(o_sw, self.g["swa_branch"], atol=1e-13)
        gate = np.zeros((1, 1, 4, 2))
        o = O.sparse_attention(self.q, self.k, self.v, sel, self.k, self.v, 1, gate, block=2)
        np.testing.assert_allclose(o[0, 0, :, 0], self.g["gated"], atol=1e-13)

    def test_token_variant(self):
        for I in range(2):
            ts = O.token_scores_tile(self.q[0], self.k[0, 0], I, block=2)
            np.testing.assert_allclose(ts, self.g[f"token_score_tile{I}"], atol=1e-13)
            sel = O.topk_tokens_tile(ts, I, 4, 1, 1, block=2)
            assert sel[0] == self.g[f"token_top1_tile{I}"][0]
            rows = O.tile_rows(I, 4, 2)
            o = O.token_sparse_rows(self.q[0, 0][rows], rows, self.k[0, 0], self.v[0, 0], sel, 1)[:, 0]
            np.testing.assert_allclose(o, self.g["token_sparse"][rows], atol=1e-13)

    def test_per_position(self):
        sc = O.block_scores_rows(self.q, self.k, block=2)
        for t in range(4):
            np.testing.assert_allclose(sc[0, 0, t], self.g[f"smax_t{t}"], atol=1e-13)
        idx = O.topk_blocks_rows(sc, 1, block=2)
        assert idx[0, 0, :, 0].tolist() == self.g["rows_top1"].tolist()
        rows = np.arange(4)
        o_sp = np.concatenate([O.sparse_branch_rows(self.q[0, 0][[t]], np.array([t]), self.k[0, 0], self.v[0, 0],
                                                    idx[0, 0, t], 2) for t in rows])[:, 0]
        np.testing.assert_allclose(o_sp, self.g["rows_sparse_branch"], atol=1e-13)
        gate = np.zeros((1, 1, 4, 2))
        o = O.sparse_attention_rows(self.q, self.k, self.v, idx, self.k, self.v, 1, gate, block=2)
        np.testing.assert_allclose(o[0, 0, :, 0], self.g["rows_gated"], atol=1e-13)

    def test_token_decode(self):
        q = np.ones((1, 1, 1))
        ts = O.decode_token_scores(q, self.k)
        np.testing.assert_allclose(ts[0, 0], self.g["decode_token_scores"], atol=1e-13)
        idx = O.topk_decode_tokens(ts, 1, 1)
        assert idx[0, 0, 0] == self.g["decode_token_top1"][0]
        o = O.decode_token_sparse(q, self.k, self.v, idx, 1)
        np.testing.assert_allclose(o[0, 0], self.g["decode_token_sparse"], atol=1e-13)

    def test_gradients(self):
        dq, dk, dv = O.backward.full_attention_backward(self.q, self.k, self.v, np.ones((1, 1, 4, 1)))
        np.testing.assert_allclose(dv[0, 0, :, 0], self.g["grad_dv"], atol=1e-13)
        np.testing.assert_allclose(dk[0, 0, :, 0], self.g["grad_dk"], atol=1e-13)
        want = self.g["grad_dq_ln2"] * math.log(2.0) + self.g["grad_dq_ln3"] * math.log(3.0)
        np.testing.assert_allclose(dq[0, 0, :, 0], want, atol=1e-13)

    def test_decode(self):
        q = np.ones((1, 1, 1))
        o, sc = O.decode_full(q, self.k, self.v, block=2)
        np.testing.assert_allclose(o[0, 0], self.g["decode_o"], atol=1e-13)
        np.testing.assert_allclose(sc[0, 0], self.g["decode_scores"], atol=1e-13)
        idx = O.topk_decode(sc, 1, block=2)
        assert idx[0, 0, 0] == self.g["decode_top1"][0]
        kr = np.array([math.log(3.0)]).reshape(1, 1, 1, 1)
        vr = np.array([4.0]).reshape(1, 1, 1, 1)
        gate = np.zeros((1, 1, 2))
        o = O.decode_sparse(q, self.k, self.v, idx, kr, vr, gate, block=2)
        np.testing.assert_allclose(o[0, 0], self.g["decode_gated"], atol=1e-13)


# ----------------------------------------------------------------------------- library routine
@pytest.mark.parametrize("N,D,Hq,Hkv", [(64, 64, 4, 1), (200, 128, 8, 2), (257, 64, 4, 4)])
def test_dense_matches_torch_sdpa(N, D, Hq, Hkv):
    rng = np.random.default_rng(N + D)
    q, k, v = _rand(rng, 1, Hq, N, D), _rand(rng, 1, Hkv, N, D), _rand(rng, 1, Hkv, N, D)
    o, _ = O.full_attention(q, k, v, chunk=97)
    np.testing.assert_allclose(o[0], _sdpa(q[0], k[0], v[0]), rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- closed forms
def test_zero_queries_closed_form():
    """Q = 0: P_{t,i} = 1/(t+1), o_t = prefix mean of V, S_{t,j} = 1/(t+1) for 64j <= t,
    every candidate of a tile ties and TopK must return {0..k-1} (lower index wins)."""
    N, D, G = 200, 64, 4
    rng = np.random.default_rng(1)
    q = np.zeros((1, G, N, D))
    k, v = _rand(rng, 1, 1, N, D), _rand(rng, 1, 1, N, D)
    o, _ = O.full_attention(q, k, v)
    prefix_mean = np.cumsum(v[0, 0], axis=0) / np.arange(1, N + 1)[:, None]
    for h in range(G):
        np.testing.assert_allclose(o[0, h], prefix_mean, atol=1e-13)
    sc = O.block_scores(q, k, "sum")
    for I in range(sc.shape[2]):
        rows = O.tile_rows(I, N)
        expect = G * np.sum(1.0 / (rows + 1.0))
        np.testing.assert_allclose(sc[0, 0, I, :I + 1], expect, rtol=1e-13)
        assert np.all(sc[0, 0, I, I + 1:] == 0)
    idx = O.topk_blocks(sc, 2)
    assert idx[0, 0, 0].tolist() == [0, -1]
    assert idx[0, 0, 3].tolist() == [0, 1]


def test_dominant_key():
    """One key with a huge logit for every query that can see it: o_t -> v_p for t >= p."""
    N, D, p = 150, 64, 70
    rng = np.random.default_rng(2)
    u = rng.standard_normal(D)
    u /= np.linalg.norm(u)
    q = np.tile(u, (1, 1, N, 1))
    k = 0.01 * _rand(rng, 1, 1, N, D)
    k[0, 0, p] = 80.0 * math.sqrt(D) * u
    v = _rand(rng, 1, 1, N, D)
    o, _ = O.full_attention(q, k, v)
    np.testing.assert_allclose(o[0, 0, p:], np.tile(v[0, 0, p], (N - p, 1)), atol=1e-12)
    # block max: the block holding p scores ~1 for the rows after p
    rows = np.arange(p, N)
    pr, _, _ = O.causal_softmax(q[0, 0, p:], rows, k[0, 0])
    s = O.block_max_probs(pr, rows)
    np.testing.assert_allclose(s[:, p // 64], 1.0, atol=1e-12)


def test_gate_saturation():
    """Gate logits +-40 select one branch; 0 gives the average of both branches."""
    rng = np.random.default_rng(3)
    N, D = 130, 64
    q, k, v = _rand(rng, 1, 2, N, D), _rand(rng, 1, 1, N, D), _rand(rng, 1, 1, N, D)
    ks, vs = _rand(rng, 1, 1, N, D), _rand(rng, 1, 1, N, D)
    idx = O.topk_blocks(O.block_scores(q, k), 1)
    only_sp = O.sparse_attention(q, k, v, idx, ks, vs, 16, np.tile([40.0, -40.0], (1, 2, N, 1)))
    only_sw = O.sparse_attention(q, k, v, idx, ks, vs, 16, np.tile([-40.0, 40.0], (1, 2, N, 1)))
    half = O.sparse_attention(q, k, v, idx, ks, vs, 16, np.zeros((1, 2, N, 2)))
    for h in range(2):
        for I in range(3):
            rows = O.tile_rows(I, N)
            sp = O.sparse_branch_rows(q[0, h, rows], rows, k[0, 0], v[0, 0], idx[0, 0, I])
            sw = O.swa_branch_rows(q[0, h, rows], rows, ks[0, 0], vs[0, 0], 16)
            np.testing.assert_allclose(only_sp[0, h, rows], sp, atol=1e-12)
            np.testing.assert_allclose(only_sw[0, h, rows], sw, atol=1e-12)
            np.testing.assert_allclose(half[0, h, rows], 0.5 * (sp + sw), atol=1e-12)


# ----------------------------------------------------------------------------- invariants
@pytest.mark.parametrize("N,D,G", [(256, 64, 4), (200, 128, 2)])
def test_score_invariants(N, D, G):
    rng = np.random.default_rng(N * G)
    q, k = _rand(rng, 1, G, N, D), _rand(rng, 1, 1, N, D)
    rows = np.arange(N)
    for h in range(G):
        p, _, _ = O.causal_softmax(q[0, h], rows, k[0, 0])
        s = O.block_max_probs(p, rows)
        assert np.all(s >= 0) and np.all(s <= 1)
        np.testing.assert_allclose(s.max(axis=1), p.max(axis=1), rtol=0, atol=0)
        assert np.all(s[np.arange(s.shape[1])[None, :] * 64 > rows[:, None]] == 0)
    smax = O.block_scores(q, k, "max")
    assert np.all(smax <= 1.0)
    ssum = O.block_scores(q, k, "sum")
    assert np.all(ssum >= smax - 1e-15)
    k_sel = 3
    idx = O.topk_blocks(ssum, k_sel)
    for I in range(ssum.shape[2]):
        sel = [j for j in idx[0, 0, I] if j >= 0]
        assert len(sel) == min(k_sel, I + 1) and len(set(sel)) == len(sel)
        assert all(0 <= j <= I for j in sel) and sel == sorted(sel)
        rest = [j for j in range(I + 1) if j not in sel]
        if rest:
            assert min(ssum[0, 0, I, sel]) >= max(ssum[0, 0, I, rest])


def test_k_covering_all_blocks_is_dense():
    """With every block selected the sparse branch equals dense causal attention."""
    rng = np.random.default_rng(4)
    N, D, Hq = 200, 64, 4
    qs, k, v = _rand(rng, 1, Hq, N, D), _rand(rng, 1, 1, N, D), _rand(rng, 1, 1, N, D)
    nb = 4
    idx = O.topk_blocks(O.block_scores(qs, k), nb)
    gate = np.tile([40.0, -40.0], (1, Hq, N, 1))
    o = O.sparse_attention(qs, k, v, idx, k, v, 128, gate)
    np.testing.assert_allclose(o[0], _sdpa(qs[0], k[0], v[0]), atol=1e-12)


def test_window_covering_all_is_dense():
    rng = np.random.default_rng(5)
    N, D, Hq = 190, 64, 2
    qs, k, v = _rand(rng, 1, Hq, N, D), _rand(rng, 1, 1, N, D), _rand(rng, 1, 1, N, D)
    ks, vs = _rand(rng, 1, 1, N, D), _rand(rng, 1, 1, N, D)
    idx = O.topk_blocks(O.block_scores(qs, k), 1)
    gate = np.tile([-40.0, 40.0], (1, Hq, N, 1))
    o = O.sparse_attention(qs, k, v, idx, ks, vs, N, gate)
    np.testing.assert_allclose(o[0], _sdpa(qs[0], ks[0], vs[0]), atol=1e-12)


def test_selection_order_irrelevant():
    rng = np.random.default_rng(6)
    N, D = 256, 64
    q, k, v = _rand(rng, 1, 1, N, D), _rand(rng, 1, 1, N, D), _rand(rng, 1, 1, N, D)
    rows = O.tile_rows(3, N)
    a = O.sparse_branch_rows(q[0, 0, rows], rows, k[0, 0], v[0, 0], [0, 2, 3])
    b = O.sparse_branch_rows(q[0, 0, rows], rows, k[0, 0], v[0, 0], [3, -1, 0, 2])
    np.testing.assert_allclose(a, b, atol=1e-14)


def test_token_variant_invariants():
    rng = np.random.default_rng(7)
    N, D, G, forced, kt = 256, 64, 2, 16, 20
    q, k, v = _rand(rng, 1, G, N, D), _rand(rng, 1, 1, N, D), _rand(rng, 1, 1, N, D)
    for I in range(4):
        ts = O.token_scores_tile(q[0], k[0, 0], I)
        rows = O.tile_rows(I, N)
        # every row's probabilities sum to 1
        np.testing.assert_allclose(ts.sum(), G * len(rows), rtol=1e-12)
        assert np.all(ts[rows[-1] + 1:] == 0)
        sel = O.topk_tokens_tile(ts, I, N, kt, forced)
        real = [i for i in sel if i >= 0]
        assert all(i <= rows[-1] - forced for i in real)
        assert len(real) == min(kt, O.token_candidates(I, N, forced))
        # forced tokens are always attended: make the window keys dominant and compare
        o = O.token_sparse_rows(q[0, 0, rows], rows, k[0, 0], v[0, 0], sel, forced)
        o_win = O.swa_branch_rows(q[0, 0, rows], rows, k[0, 0], v[0, 0], forced)
        if not real:
            np.testing.assert_allclose(o, o_win, atol=1e-12)
    # when the budget covers every candidate, each row sees every earlier token: dense
    kt_all = N
    I = 3
    rows = O.tile_rows(I, N)
    ts = O.token_scores_tile(q[0], k[0, 0], I)
    sel = O.topk_tokens_tile(ts, I, N, kt_all, forced)
    o = O.token_sparse_rows(q[0, 0, rows], rows, k[0, 0], v[0, 0], sel, forced)
    np.testing.assert_allclose(o, _sdpa(q[0, :1], k[0], v[0])[0, rows], atol=1e-12)


def test_decode_is_last_row_of_dense():
    rng = np.random.default_rng(8)
    L, D, Hq, Hkv = 300, 64, 4, 2
    q, k, v = _rand(rng, 2, Hq, D), _rand(rng, 2, Hkv, L, D), _rand(rng, 2, Hkv, L, D)
    seqlens = np.array([300, 129])
    o, sc = O.decode_full(q, k, v, seqlens)
    for b in range(2):
        Lb = seqlens[b]
        qq = np.zeros((Hq, Lb, D))
        qq[:, -1] = q[b]
        ref = _sdpa(qq, k[b, :, :Lb], v[b, :, :Lb])[:, -1]
        np.testing.assert_allclose(o[b], ref, atol=1e-12)
        assert np.all(sc[b, :, (Lb + 63) // 64:] == 0)
    idx = O.topk_decode(sc, 4, seqlens)
    assert all(0 <= j < 3 for j in idx[1].ravel() if j >= 0)
    assert np.sum(idx[1] >= 0) == 2 * 3


def test_decode_empty_branch_contributes_zero():
    """An empty SWA ring (swa_len 0) leaves only the gated sparse branch."""
    rng = np.random.default_rng(10)
    L, D, G = 200, 8, 2
    q, k, v = _rand(rng, 1, G, D), _rand(rng, 1, 1, L, D), _rand(rng, 1, 1, L, D)
    kr, vr, gate = _rand(rng, 1, 1, 4, D), _rand(rng, 1, 1, 4, D), _rand(rng, 1, G, 2)
    idx = np.array([[[0, 2]]])
    o = O.decode_sparse(q, k, v, idx, kr, vr, gate, swa_len=np.array([0]))
    keys = list(range(0, 64)) + list(range(128, 192))
    for h in range(G):
        want = BF.attend(q[0, h].tolist(), keys, k[0, 0].tolist(), v[0, 0].tolist())
        g0 = 1 / (1 + math.exp(-gate[0, h, 0]))
        np.testing.assert_allclose(o[0, h], [g0 * x for x in want], atol=1e-12)


# ----------------------------------------------------------------------------- brute force
@pytest.mark.parametrize("seed,N,D,G", [(0, 64, 16, 1), (1, 65, 16, 2), (2, 130, 8, 2), (3, 200, 8, 1)])
def test_brute_force(seed, N, D, G):
    rng = np.random.default_rng(100 + seed)
    q, k, v = _rand(rng, 1, G, N, D), _rand(rng, 1, 1, N, D), _rand(rng, 1, 1, N, D)
    ks, vs = _rand(rng, 1, 1, N, D), _rand(rng, 1, 1, N, D)
    gate = _rand(rng, 1, G, N, 2)
    kk, vv, kl, vl = k[0, 0].tolist(), v[0, 0].tolist(), ks[0, 0].tolist(), vs[0, 0].tolist()
    qg = [q[0, h].tolist() for h in range(G)]
    T = (N + 63) // 64
    for red in ("sum", "max"):
        sc = O.block_scores(q, k, red)
        for I in range(T):
            for j in range(T):
                want = BF.block_score(qg, kk, I, j, N, 64, red) if j <= I else 0.0
                assert abs(sc[0, 0, I, j] - want) <= 1e-12 * max(1.0, abs(want))
    sc = O.block_scores(q, k, "sum")
    kb = 2
    idx = O.topk_blocks(sc, kb)
    window = 24
    o = O.sparse_attention(q, k, v, idx, ks, vs, window, gate)
    for I in range(T):
        assert idx[0, 0, I].tolist() == BF.topk(sc[0, 0, I].tolist(), I + 1, kb)
        for t in O.tile_rows(I, N)[::7]:
            for h in range(G):
                want = BF.gated_row(qg[h][t], t, kk, vv, idx[0, 0, I].tolist(), kl, vl, window,
                                    gate[0, h, t].tolist(), 64)
                np.testing.assert_allclose(o[0, h, t], want, atol=1e-12)
    # token variant
    forced, kt = 8, 10
    for I in range(T):
        ts = O.token_scores_tile(q[0], k[0, 0], I)
        for i in range(0, N, 5):
            assert abs(ts[i] - BF.token_score(qg, kk, I, i, N, 64)) <= 1e-12
        sel = O.topk_tokens_tile(ts, I, N, kt, forced)
        rows = O.tile_rows(I, N)
        assert sel.tolist() == BF.topk(ts.tolist(), O.token_candidates(I, N, forced), kt)
        ot = O.token_sparse_rows(q[0, 0, rows], rows, k[0, 0], v[0, 0], sel, forced)
        for r, t in list(enumerate(rows))[::9]:
            np.testing.assert_allclose(ot[r], BF.token_row(qg[0][t], t, kk, vv, sel.tolist(), forced),
                                       atol=1e-12)


@pytest.mark.parametrize("seed,N,D,G,Hkv", [(10, 65, 128, 8, 2), (11, 256, 64, 4, 2), (12, 200, 128, 4, 1),
                                             (13, 129, 64, 8, 1)])
def test_brute_force_gqa(seed, N, D, G, Hkv):
    """The head dims and group sizes of the workloads (D 64/128, G 4/8), with two KV groups where
    the head-to-group mapping matters: block scores under both reductions, the top-k, gated
    sparse rows and token scores against the scalar transcription, group by group."""
    rng = np.random.default_rng(200 + seed)
    Hq = G * Hkv
    q, k, v = _rand(rng, 1, Hq, N, D), _rand(rng, 1, Hkv, N, D), _rand(rng, 1, Hkv, N, D)
    ks, vs = _rand(rng, 1, Hkv, N, D), _rand(rng, 1, Hkv, N, D)
    gate = _rand(rng, 1, Hq, N, 2)
    T = (N + 63) // 64
    sc = {red: O.block_scores(q, k, red) for red in ("sum", "max")}
    kb, window = 2, 40
    idx = O.topk_blocks(sc["sum"], kb)
    o = O.sparse_attention(q, k, v, idx, ks, vs, window, gate)
    for g in range(Hkv):
        kk, vv, kl, vl = k[0, g].tolist(), v[0, g].tolist(), ks[0, g].tolist(), vs[0, g].tolist()
        heads = list(range(g * G, (g + 1) * G))
        qg = [q[0, h].tolist() for h in heads]
        memo = {}
        for red in ("sum", "max"):
            for I in range(T):
                for j in range(I + 1):
                    want = BF.block_score(qg, kk, I, j, N, 64, red, memo)
                    assert abs(sc[red][0, g, I, j] - want) <= 1e-12 * max(1.0, abs(want))
                assert np.all(sc[red][0, g, I, I + 1:] == 0)
        for I in range(T):
            assert idx[0, g, I].tolist() == BF.topk(sc["sum"][0, g, I].tolist(), I + 1, kb)
            for t in O.tile_rows(I, N)[::13]:
                for h in (heads[0], heads[-1]):
                    want = BF.gated_row(q[0, h, t].tolist(), t, kk, vv, idx[0, g, I].tolist(), kl, vl, window,
                                        gate[0, h, t].tolist(), 64)
                    np.testing.assert_allclose(o[0, h, t], want, atol=1e-12)
            ts = O.token_scores_tile(q[0, g * G:(g + 1) * G], k[0, g], I)
            for i in range(0, N, 11):
                assert abs(ts[i] - BF.token_score(qg, kk, I, i, N, 64, memo)) <= 1e-12


def test_brute_force_decode():
    rng = np.random.default_rng(9)
    L, D, G = 190, 8, 2
    q, k, v = _rand(rng, 1, G, D), _rand(rng, 1, 1, L, D), _rand(rng, 1, 1, L, D)
    kr, vr = _rand(rng, 1, 1, 5, D), _rand(rng, 1, 1, 5, D)
    gate = _rand(rng, 1, G, 2)
    o, sc = O.decode_full(q, k, v)
    kk, vv = k[0, 0].tolist(), v[0, 0].tolist()
    for j in range(3):
        want = sum(max(p for i, p in BF.softmax_over(q[0, h].tolist(), list(range(L)), kk)
                       if j * 64 <= i < (j + 1) * 64) for h in range(G))
        assert abs(sc[0, 0, j] - want) < 1e-12
    for h in range(G):
        np.testing.assert_allclose(o[0, h], BF.attend(q[0, h].tolist(), list(range(L)), kk, vv), atol=1e-12)
    idx = O.topk_decode(sc, 2)
    assert idx[0, 0].tolist() == BF.topk(sc[0, 0].tolist(), 3, 2)
    swa_len = np.array([3])
    od = O.decode_sparse(q, k, v, idx, kr, vr, gate, swa_len=swa_len)
    for h in range(G):
        keys = [i for j in idx[0, 0] for i in range(j * 64, min(L, (j + 1) * 64))]
        a = BF.attend(q[0, h].tolist(), keys, kk, vv)
        b = BF.attend(q[0, h].tolist(), [0, 1, 2], kr[0, 0].tolist(), vr[0, 0].tolist())
        g0, g1 = 1 / (1 + math.exp(-gate[0, h, 0])), 1 / (1 + math.exp(-gate[0, h, 1]))
        np.testing.assert_allclose(od[0, h], [g0 * x + g1 * y for x, y in zip(a, b)], atol=1e-12)


# ----------------------------------------------------------------------------- planted mistakes
def test_sink_closed_forms():
    """A sink logit b joins the softmax as an extra entry with zero value ([HSP] §4.1, gpt-oss
    sinks): one visible key gives o = v * sigmoid(s - b); n keys with equal logits give
    o = mean(v) * n / (n + exp(b - s)); b = -inf is no sink at all."""
    rng = np.random.default_rng(5)
    D = 16
    k = rng.standard_normal((4, D))
    v = rng.standard_normal((4, D))
    q = rng.standard_normal((1, D))
    s0 = float(q[0] @ k[0]) / math.sqrt(D)
    for b in (-2.0, 0.0, 1.5, 7.0):
        o, _ = O.attention_rows(q, np.array([0]), k, v, sink=b)
        want = v[0] / (1.0 + math.exp(b - s0))
        np.testing.assert_allclose(o[0], want, rtol=1e-12, atol=1e-14)
    qz = np.zeros((1, D))
    for b in (-1.0, 0.5, 3.0):
        o, _ = O.attention_rows(qz, np.array([3]), k, v, sink=b)
        want = v.mean(axis=0) * 4.0 / (4.0 + math.exp(b))
        np.testing.assert_allclose(o[0], want, rtol=1e-12, atol=1e-14)
    o_none, _ = O.attention_rows(q, np.array([3]), k, v)
    o_inf, _ = O.attention_rows(q, np.array([3]), k, v, sink=-np.inf)
    np.testing.assert_array_equal(o_none, o_inf)


def test_sink_per_branch_and_decode():
    """sinks[h] = (sparse-branch, SWA-branch) logits: each branch's output shrinks by exactly its
    own factor l / (l + exp(b - m)); a huge sink silences its branch; decode agrees with the
    prefill rows of the same keys."""
    rng = np.random.default_rng(6)
    N, D = 128, 16
    k, v, ks, vs = (rng.standard_normal((N, D)) for _ in range(4))
    q = rng.standard_normal((64, D))
    rows = np.arange(64, 128)
    gate = rng.standard_normal((64, 2))
    base = O.gated_sparse_rows(q, rows, k, v, [0], ks, vs, 32, gate)
    # huge sparse-branch sink: only the SWA branch remains
    only_swa = O.gated_sparse_rows(q, rows, k, v, [0], ks, vs, 32, gate, sinks=(1e3, -np.inf))
    want = O.sigmoid(gate[:, 1:2]) * O.swa_branch_rows(q, rows, ks, vs, 32)
    np.testing.assert_allclose(only_swa, want, rtol=1e-12, atol=1e-14)
    # huge SWA sink: only the sparse branch remains
    only_sp = O.gated_sparse_rows(q, rows, k, v, [0], ks, vs, 32, gate, sinks=(-np.inf, 1e3))
    want = O.sigmoid(gate[:, 0:1]) * O.sparse_branch_rows(q, rows, k, v, [0])
    np.testing.assert_allclose(only_sp, want, rtol=1e-12, atol=1e-14)
    np.testing.assert_array_equal(O.gated_sparse_rows(q, rows, k, v, [0], ks, vs, 32, gate,
                                                      sinks=(-np.inf, -np.inf)), base)
    # decode: the new token at L-1 = the last prefill row, sink factors included
    L = 128
    kc, vc = k[None, None], v[None, None]
    kr, vr = ks[None, None, L - 32:], vs[None, None, L - 32:]
    qd = q[-1][None, None]
    g = gate[-1][None, None]
    sk = np.array([[0.7, -0.3]])
    od = O.decode_sparse(qd, kc, vc, np.array([[[0, 1]]]), kr, vr, g, sinks=sk)
    op = O.gated_sparse_rows(q[-1:], np.array([L - 1]), k, v, [0, 1], ks, vs, 32, gate[-1:], sinks=sk[0])
    np.testing.assert_allclose(od[0, 0], op[0], rtol=1e-12, atol=1e-14)


def test_token_decode_pins():
    """Token-variant decode: the scores are torch's float64 softmax of the new token's logits
    summed over the group's heads (they sum to G); every candidate selected gives dense decode;
    the layer equals the prefill token-sparse row of position L-1 with the same selection; the
    selection never enters the forced window and breaks ties to the lower index."""
    rng = np.random.default_rng(9)
    B, Hq, Hkv, D, L, W = 2, 4, 2, 16, 300, 32
    G = Hq // Hkv
    q = rng.standard_normal((B, Hq, D))
    kc = rng.standard_normal((B, Hkv, L, D))
    vc = rng.standard_normal((B, Hkv, L, D))
    seqlens = np.array([L, 211])
    sc = O.decode_token_scores(q, kc, seqlens)
    for b in range(B):
        Lb = int(seqlens[b])
        for g in range(Hkv):
            kk = torch.from_numpy(kc[b, g, :Lb]).double()
            want = np.zeros(L)
            for h in range(g * G, (g + 1) * G):
                lg = (torch.from_numpy(q[b, h]).double() @ kk.T) / math.sqrt(D)
                want[:Lb] += torch.softmax(lg, dim=0).numpy()
            np.testing.assert_allclose(sc[b, g], want, rtol=1e-12, atol=1e-15)
            assert abs(sc[b, g].sum() - G) < 1e-12
    # all candidates selected -> dense decode
    idx_all = O.topk_decode_tokens(sc, L, W, seqlens)
    o_all = O.decode_token_sparse(q, kc, vc, idx_all, W, seqlens)
    o_dense, _ = O.decode_full(q, kc, vc, seqlens)
    np.testing.assert_allclose(o_all, o_dense, rtol=1e-12, atol=1e-13)
    # a small budget: the prefill token-sparse row of position L_b - 1 agrees
    kt = 20
    idx = O.topk_decode_tokens(sc, kt, W, seqlens)
    o = O.decode_token_sparse(q, kc, vc, idx, W, seqlens)
    for b in range(B):
        Lb = int(seqlens[b])
        for g in range(Hkv):
            sel = idx[b, g]
            assert np.all(sel[sel >= 0] <= Lb - 1 - W) and np.all(np.diff(sel[sel >= 0]) > 0)
            for h in range(g * G, (g + 1) * G):
                ref = O.token_sparse_rows(q[b, h][None, :], np.array([Lb - 1]), kc[b, g, :Lb], vc[b, g, :Lb], sel, W)
                np.testing.assert_allclose(o[b, h], ref[0], rtol=1e-12, atol=1e-13)
    # ties: equal scores pick the lowest indices
    flat = np.zeros((1, 1, 100))
    got = O.topk_decode_tokens(flat, 5, 10)
    assert got[0, 0].tolist() == [0, 1, 2, 3, 4]


def test_e4m3_decode_pins():
    """FP8 E4M3 codes: every one of the 256 codes equals torch's float8_e4m3fn -> float64
    conversion (NaN exactly at S.1111.111), and hand values of the format (1.0, the largest
    finite 448, the smallest subnormal 2^-9, the smallest normal 2^-6, the largest subnormal
    7/8 * 2^-6, -1.0, both zeros); positive codes increase strictly up to 448."""
    codes = np.arange(256, dtype=np.uint8)
    got = O.e4m3_to_float(codes)
    want = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(got), np.isnan(want))
    assert np.nonzero(np.isnan(got))[0].tolist() == [0x7F, 0xFF]
    fin = ~np.isnan(want)
    assert np.array_equal(got[fin], want[fin])
    hand = {0x38: 1.0, 0x7E: 448.0, 0x01: 2.0 ** -9, 0x08: 2.0 ** -6, 0x07: 7 / 8 * 2.0 ** -6, 0xB8: -1.0,
            0x00: 0.0, 0x80: -0.0, 0x40: 2.0, 0x3C: 1.5}
    for c, v in hand.items():
        assert got[c] == v and math.copysign(1.0, got[c]) == math.copysign(1.0, v), hex(c)
    assert np.all(np.diff(got[:0x7F]) > 0)


def test_fp8_token_decode_pins():
    """FP8 cache: each KV head's values are its codes times that head's scale (K and V scaled
    separately); the token-variant decode on them equals torch's float64 attention over the
    values torch decodes from the same codes, and with every candidate selected it equals dense
    decode over those values."""
    rng = np.random.default_rng(21)
    B, Hq, Hkv, D, L, W = 2, 4, 2, 16, 260, 32
    G = Hq // Hkv
    kx = rng.standard_normal((B, Hkv, L, D)) * 40.0
    vx = rng.standard_normal((B, Hkv, L, D)) * 40.0
    kcode = torch.from_numpy(kx.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    vcode = torch.from_numpy(vx.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ks, vs = np.array([0.01, 0.02]), np.array([0.03, 0.005])
    kd, vd = O.dequant_kv_fp8(kcode, ks), O.dequant_kv_fp8(vcode, vs)
    tk = torch.from_numpy(kcode).view(torch.float8_e4m3fn).to(torch.float64)
    tv = torch.from_numpy(vcode).view(torch.float8_e4m3fn).to(torch.float64)
    for g in range(Hkv):
        assert np.array_equal(kd[:, g], tk[:, g].numpy() * ks[g])
        assert np.array_equal(vd[:, g], tv[:, g].numpy() * vs[g])
    q = rng.standard_normal((B, Hq, D))
    seqlens = np.array([L, 190])
    sc = O.decode_token_scores(q, kd, seqlens)
    idx = O.topk_decode_tokens(sc, 24, W, seqlens)
    o = O.decode_token_sparse(q, kd, vd, idx, W, seqlens)
    for b in range(B):
        Lb = int(seqlens[b])
        for g in range(Hkv):
            sel = [int(i) for i in idx[b, g] if i >= 0]
            keys = sorted(set(sel) | set(range(Lb - W, Lb)))
            kk = tk[b, g, keys] * ks[g]
            vv = tv[b, g, keys] * vs[g]
            for h in range(g * G, (g + 1) * G):
                qq = torch.from_numpy(q[b, h]).double()[None, None, None, :]
                ref = torch.nn.functional.scaled_dot_product_attention(qq, kk[None, None], vv[None, None])
                np.testing.assert_allclose(o[b, h], ref[0, 0, 0].numpy(), rtol=1e-12, atol=1e-13)
    idx_all = O.topk_decode_tokens(sc, L, W, seqlens)
    o_all = O.decode_token_sparse(q, kd, vd, idx_all, W, seqlens)
    o_dense, _ = O.decode_full(q, kd, vd, seqlens)
    np.testing.assert_allclose(o_all, o_dense, rtol=1e-12, atol=1e-13)


def test_per_position_selection_pins():
    """Per-position selection: the scores equal a torch float64 causal softmax, reshaped into
    64-key blocks and maxed over the block and the group's heads; the top k of row t never
    passes block floor(t/64), breaks ties low and matches the brute-force selection; each row's
    sparse branch equals torch attention under a mask built from that row's own blocks; rows
    that share one selection reproduce the per-tile layer; k covering every block is dense."""
    rng = np.random.default_rng(31)
    B, Hq, Hkv, N, D, k, win = 1, 4, 2, 300, 16, 2, 20
    G = Hq // Hkv
    q = rng.standard_normal((B, Hq, N, D))
    kk = rng.standard_normal((B, Hkv, N, D))
    vv = rng.standard_normal((B, Hkv, N, D))
    sc = O.block_scores_rows(q, kk)
    nb = (N + 63) // 64
    causal = torch.ones(N, N, dtype=torch.bool).tril()
    for g in range(Hkv):
        want = torch.zeros(N, nb, dtype=torch.float64)
        for h in range(g * G, (g + 1) * G):
            lg = (torch.from_numpy(q[0, h]) @ torch.from_numpy(kk[0, g]).T) / math.sqrt(D)
            p = torch.softmax(lg.masked_fill(~causal, float("-inf")), dim=1)
            pad = torch.zeros(N, nb * 64, dtype=torch.float64)
            pad[:, :N] = p
            want = torch.maximum(want, pad.view(N, nb, 64).amax(dim=2))
        np.testing.assert_allclose(sc[0, g], want.numpy(), rtol=1e-12, atol=1e-15)
    idx = O.topk_blocks_rows(sc, k)
    for g in range(Hkv):
        for t in range(N):
            sel = idx[0, g, t]
            assert sel.tolist() == BF.topk(sc[0, g, t].tolist(), t // 64 + 1, k)
            assert np.all(sel[sel >= 0] <= t // 64)
    ties = O.topk_blocks_rows(np.zeros((1, 1, 200, 4)), 2)
    assert ties[0, 0, 199].tolist() == [0, 1] and ties[0, 0, 10].tolist() == [0, -1]
    # sparse branch of each row vs torch under the row's own mask (gate saturated to the sparse branch)
    gate = np.zeros((B, Hq, N, 2))
    gate[..., 0], gate[..., 1] = 60.0, -60.0
    ks, vs = rng.standard_normal((B, Hkv, N, D)), rng.standard_normal((B, Hkv, N, D))
    o = O.sparse_attention_rows(q, kk, vv, idx, ks, vs, win, gate)
    for h in range(Hq):
        g = h // G
        mask = torch.zeros(N, N, dtype=torch.bool)
        for t in range(N):
            for j in idx[0, g, t]:
                if j >= 0:
                    mask[t, 64 * j:min(N, 64 * j + 64)] = True
        mask &= causal
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[0, h])[None, None], torch.from_numpy(kk[0, g])[None, None],
            torch.from_numpy(vv[0, g])[None, None], attn_mask=mask[None, None])
        np.testing.assert_allclose(o[0, h], ref[0, 0].numpy(), rtol=1e-9, atol=1e-12)
    # one selection per tile -> the per-tile layer
    tile_idx = O.topk_blocks(O.block_scores(q, kk, "max"), k)
    rows_idx = np.repeat(tile_idx, 64, axis=2)[:, :, :N]
    gate2 = rng.standard_normal((B, Hq, N, 2))
    np.testing.assert_allclose(O.sparse_attention_rows(q, kk, vv, rows_idx, ks, vs, win, gate2),
                               O.sparse_attention(q, kk, vv, tile_idx, ks, vs, win, gate2), rtol=1e-12, atol=1e-13)
    # k covering every block: dense causal attention
    full_idx = O.topk_blocks_rows(sc, nb)
    o_all = O.sparse_attention_rows(q, kk, vv, full_idx, ks, vs, win, gate)
    for h in range(Hq):
        g = h // G
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[0, h])[None, None], torch.from_numpy(kk[0, g])[None, None],
            torch.from_numpy(vv[0, g])[None, None], is_causal=True)
        np.testing.assert_allclose(o_all[0, h], ref[0, 0].numpy(), rtol=1e-9, atol=1e-12)


def test_pins_catch_planted_mistakes(monkeypatch):
    """Plant plausible mistakes in the oracle and check that a pin above fails."""
    g = _gold()
    q = np.ones((1, 1, 4, 1))
    k = np.array([0.0, math.log(2.0), 0.0, math.log(3.0)]).reshape(1, 1, 4, 1)
    # 1) ties broken toward the higher index
    monkeypatch.setattr(O.hysparse_oracle, "select_topk",
                        lambda s, n, kk: np.concatenate([np.sort(np.lexsort((-np.arange(n), -s[:n]))[:kk]),
                                                         -np.ones(max(0, kk - n), np.int64)]))
    sc = np.zeros((1, 1, 4, 4))
    idx = O.hysparse_oracle.topk_blocks(sc, 2)
    assert idx[0, 0, 3].tolist() != [0, 1]
    monkeypatch.undo()
    # 2) forgetting to clip the block at t changes nothing (P is zero past t), but
    #    dropping the 1/sqrt(d) scale breaks the SDPA pin
    rng = np.random.default_rng(0)
    qq, kk2, vv = _rand(rng, 1, 1, 40, 16), _rand(rng, 1, 1, 40, 16), _rand(rng, 1, 1, 40, 16)
    o_ok, _ = O.full_attention(qq, kk2, vv)
    o_bad, _ = O.full_attention(qq * 4.0, kk2, vv)   # == no 1/sqrt(16) scaling
    ref = _sdpa(qq[0], kk2[0], vv[0])
    assert np.allclose(o_ok[0], ref, atol=1e-12) and not np.allclose(o_bad[0], ref, atol=1e-6)
    # 3) an off-by-one window ([t-w, t]) breaks the worked SWA example
    rows = np.arange(4)
    o_sw_bad = O.swa_branch_rows(q[0, 0], rows, k[0, 0], np.arange(1.0, 5.0)[:, None], 2)[:, 0]
    assert not np.allclose(o_sw_bad, g["swa_branch"])
