"""Pins of the float64 gradient oracle (oracle/hysparse_backward.py) against torch's float64
autograd of the forward definitions, plus closed forms and invariants of the softmax gradient."""
import math

import numpy as np
import torch

import oracle as O

BW = O.backward


def _t(x, grad=True):
    return torch.tensor(np.asarray(x, np.float64), dtype=torch.float64, requires_grad=grad)


def _torch_attention(q, k, v, visible, sink=None):
    """Masked softmax attention in torch (rows x keys), with an optional zero-value sink entry."""
    s = (q @ k.T) / math.sqrt(q.shape[1])
    s = s.masked_fill(~visible, float("-inf"))
    if sink is not None:
        s = torch.cat([s, sink.expand(s.shape[0], 1)], dim=1)
    p = torch.softmax(s, dim=1)
    return p[:, :k.shape[0]] @ v


def test_rows_backward_matches_autograd():
    rng = np.random.default_rng(41)
    R, N, D = 7, 23, 8
    q, k, v, do = (rng.standard_normal(s) for s in ((R, D), (N, D), (N, D), (R, D)))
    rows = np.array([3, 5, 9, 12, 15, 20, 22])
    vis = rng.random((R, N)) < 0.7
    vis[np.arange(R), rows] = True          # every row sees itself
    for sink in (None, 0.7):
        dq, dk, dv, dsink = BW.attention_rows_backward(q, rows, k, v, do, vis, sink)
        tq, tk, tv = _t(q), _t(k), _t(v)
        ts = None if sink is None else _t(np.array([sink]))
        causal = torch.from_numpy(np.arange(N)[None, :] <= rows[:, None])
        o = _torch_attention(tq, tk, tv, causal & torch.from_numpy(vis), ts)
        (o * torch.from_numpy(do)).sum().backward()
        np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-10, atol=1e-12)
        if sink is not None:
            assert abs(dsink - ts.grad.item()) <= 1e-10


def test_full_backward_matches_sdpa_autograd():
    """torch's float64 scaled_dot_product_attention (causal, GQA by repeating the KV heads)."""
    rng = np.random.default_rng(42)
    B, Hq, Hkv, N, D = 1, 4, 2, 40, 16
    q, do = rng.standard_normal((B, Hq, N, D)), rng.standard_normal((B, Hq, N, D))
    k, v = rng.standard_normal((B, Hkv, N, D)), rng.standard_normal((B, Hkv, N, D))
    dq, dk, dv = BW.full_attention_backward(q, k, v, do)
    tq, tk, tv = _t(q), _t(k), _t(v)
    G = Hq // Hkv
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk.repeat_interleave(G, 1), tv.repeat_interleave(G, 1),
                                                         is_causal=True)
    (o * torch.from_numpy(do)).sum().backward()
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-9, atol=1e-11)


def _torch_sparse_layer(q_s, k, v, sel_sets, k_swa, v_swa, window, gate, sinks, rows_of):
    """The gated two-branch layer in torch, for autograd; sel_sets[(b, g, key)] lists the blocks of
    a row group (key = tile or position)."""
    B, Hq, N, D = q_s.shape
    G = Hq // k.shape[1]
    outs = []
    kpos = torch.arange(N)
    for b in range(B):
        heads = []
        for h in range(Hq):
            g = h // G
            o_h = torch.zeros(N, D, dtype=torch.float64)
            for key, rows in rows_of:
                rows_t = torch.from_numpy(rows)
                in_sel = torch.zeros(N, dtype=torch.bool)
                for j in sel_sets[(b, g, key)]:
                    if j >= 0:
                        in_sel[64 * j:min(N, 64 * j + 64)] = True
                causal = kpos[None, :] <= rows_t[:, None]
                vis_sp = causal & in_sel[None, :]
                vis_sw = causal & (kpos[None, :] >= rows_t[:, None] - window + 1)
                s0 = None if sinks is None else sinks[h, 0:1]
                s1 = None if sinks is None else sinks[h, 1:2]
                o_sp = _torch_attention(q_s[b, h, rows_t], k[b, g], v[b, g], vis_sp, s0)
                o_sw = _torch_attention(q_s[b, h, rows_t], k_swa[b, g], v_swa[b, g], vis_sw, s1)
                gt = torch.sigmoid(gate[b, h, rows_t])
                o_h = o_h.index_put((rows_t,), gt[:, 0:1] * o_sp + gt[:, 1:2] * o_sw)
            heads.append(o_h)
        outs.append(torch.stack(heads))
    return torch.stack(outs)


def test_sparse_backward_matches_autograd():
    """Tile and per-position selection, with and without sinks: every gradient of the layer
    (q', shared k and v through the selected blocks, the window's k' and v', the gate logits and
    the sinks) against torch's float64 autograd."""
    rng = np.random.default_rng(43)
    B, Hq, Hkv, N, D, win = 1, 4, 2, 150, 8, 20
    T = (N + 63) // 64
    q_s, do = rng.standard_normal((B, Hq, N, D)), rng.standard_normal((B, Hq, N, D))
    k, v, ks, vs = (rng.standard_normal((B, Hkv, N, D)) for _ in range(4))
    gate = rng.standard_normal((B, Hq, N, 2))
    for per_row in (False, True):
        if per_row:
            idx = np.full((B, Hkv, N, 2), -1)
            for g in range(Hkv):
                for t in range(N):
                    c = rng.permutation(t // 64 + 1)[:2]
                    idx[0, g, t, :len(c)] = np.sort(c)
            rows_of = [(t, np.array([t])) for t in range(N)]
        else:
            idx = np.full((B, Hkv, T, 2), -1)
            for g in range(Hkv):
                for I_ in range(T):
                    c = rng.permutation(I_ + 1)[:2]
                    idx[0, g, I_, :len(c)] = np.sort(c)
            rows_of = [(I_, O.tile_rows(I_, N)) for I_ in range(T)]
        sel_sets = {(0, g, key): idx[0, g, key].tolist() for g in range(Hkv) for key, _ in rows_of}
        for sinks in (None, rng.standard_normal((Hq, 2))):
            got = BW.sparse_attention_backward(q_s, k, v, idx, ks, vs, win, gate, do, sinks=sinks, per_row=per_row)
            tq, tk, tv, tks, tvs, tg = _t(q_s), _t(k), _t(v), _t(ks), _t(vs), _t(gate)
            tsk = None if sinks is None else _t(sinks)
            o = _torch_sparse_layer(tq, tk, tv, sel_sets, tks, tvs, win, tg, tsk, rows_of)
            (o * torch.from_numpy(do)).sum().backward()
            for name, ten in (("dq", tq), ("dk", tk), ("dv", tv), ("dk_swa", tks), ("dv_swa", tvs), ("dgate", tg)):
                np.testing.assert_allclose(got[name], ten.grad.numpy(), rtol=1e-9, atol=1e-11, err_msg=name)
            if sinks is not None:
                np.testing.assert_allclose(got["dsinks"], tsk.grad.numpy(), rtol=1e-9, atol=1e-11)


def test_backward_closed_forms_and_invariants():
    rng = np.random.default_rng(44)
    D = 8
    # a row that sees one key: p = 1, so dq = dk = 0 and dv = dO
    q, k, v, do = (rng.standard_normal((1, D)) for _ in range(4))
    dq, dk, dv, _ = BW.attention_rows_backward(q, np.array([0]), k, v, do)
    assert np.max(np.abs(dq)) <= 1e-14 and np.max(np.abs(dk)) <= 1e-14   # zero up to rounding
    np.testing.assert_allclose(dv, do, rtol=0, atol=1e-15)
    # without a sink each row's dS sums to zero, so the key gradients sum to zero over the keys
    R, N = 6, 30
    q, do = rng.standard_normal((R, D)), rng.standard_normal((R, D))
    k, v = rng.standard_normal((N, D)), rng.standard_normal((N, D))
    rows = np.array([5, 9, 14, 20, 25, 29])
    _, dk, dv, _ = BW.attention_rows_backward(q, rows, k, v, do)
    assert np.max(np.abs(dk.sum(axis=0))) <= 1e-12
    # dV sums the output gradients: sum_i dv_i = sum_t dO_t (each row's probabilities sum to 1)
    np.testing.assert_allclose(dv.sum(axis=0), do.sum(axis=0), rtol=1e-12, atol=1e-12)
    # saturated gate on the window branch: its logit gets no gradient, nor do K', V'
    B, Hq, Hkv, Nn = 1, 2, 1, 80
    q_s, dO = rng.standard_normal((B, Hq, Nn, D)), rng.standard_normal((B, Hq, Nn, D))
    kk, vv, ks, vs = (rng.standard_normal((B, Hkv, Nn, D)) for _ in range(4))
    gate = np.zeros((B, Hq, Nn, 2))
    gate[..., 1] = -800.0
    idx = np.array([[[[0], [1]]]])
    with np.errstate(over="ignore"):   # sigmoid(-800) underflows to exactly 0
        got = BW.sparse_attention_backward(q_s, kk, vv, idx, ks, vs, 16, gate, dO)
    assert np.all(got["dgate"][..., 1] == 0) and np.all(got["dk_swa"] == 0) and np.all(got["dv_swa"] == 0)


def test_hybrid_block_backward_sums_the_shared_cache_gradients():
    """Shared K, V of the block: the full layer's gradient plus each sparse layer's, as autograd
    gives for the sum of the layers' losses."""
    rng = np.random.default_rng(45)
    B, Hq, Hkv, N, D, win = 1, 2, 1, 130, 8, 16
    T = (N + 63) // 64
    q, d_full = rng.standard_normal((B, Hq, N, D)), rng.standard_normal((B, Hq, N, D))
    k, v = rng.standard_normal((B, Hkv, N, D)), rng.standard_normal((B, Hkv, N, D))
    layers = []
    for _ in range(2):
        idx = np.full((B, Hkv, T, 1), -1)
        for I_ in range(T):
            idx[0, 0, I_, 0] = rng.integers(0, I_ + 1)
        layers.append({"q_s": rng.standard_normal((B, Hq, N, D)), "idx": idx,
                       "k_swa": rng.standard_normal((B, Hkv, N, D)), "v_swa": rng.standard_normal((B, Hkv, N, D)),
                       "gate": rng.standard_normal((B, Hq, N, 2)), "d_o": rng.standard_normal((B, Hq, N, D))})
    got = BW.hybrid_block_backward(q, k, v, d_full, layers, win)
    tk, tv = _t(k), _t(v)
    o_full = torch.nn.functional.scaled_dot_product_attention(_t(q, False), tk.repeat_interleave(Hq // Hkv, 1),
                                                              tv.repeat_interleave(Hq // Hkv, 1), is_causal=True)
    loss = (o_full * torch.from_numpy(d_full)).sum()
    rows_of = [(I_, O.tile_rows(I_, N)) for I_ in range(T)]
    for L in layers:
        sel_sets = {(0, 0, I_): L["idx"][0, 0, I_].tolist() for I_ in range(T)}
        o = _torch_sparse_layer(_t(L["q_s"], False), tk, tv, sel_sets, _t(L["k_swa"], False), _t(L["v_swa"], False),
                                win, _t(L["gate"], False), None, rows_of)
        loss = loss + (o * torch.from_numpy(L["d_o"])).sum()
    loss.backward()
    np.testing.assert_allclose(got["dk"], tk.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(got["dv"], tv.grad.numpy(), rtol=1e-9, atol=1e-11)


def test_token_sparse_backward_matches_autograd():
    """Token-sparse layer: the selected tokens united with the forced newest window, each once."""
    rng = np.random.default_rng(47)
    B, Hq, Hkv, N, D, W, kt = 1, 4, 2, 150, 8, 16, 10
    T = (N + 63) // 64
    q_s, do = rng.standard_normal((B, Hq, N, D)), rng.standard_normal((B, Hq, N, D))
    k, v = rng.standard_normal((B, Hkv, N, D)), rng.standard_normal((B, Hkv, N, D))
    idx = np.full((B, Hkv, T, kt), -1)
    for g in range(Hkv):
        for I_ in range(T):
            n = max(0, min(N, 64 * I_ + 64) - W)
            c = np.sort(rng.permutation(n)[:kt])
            idx[0, g, I_, :len(c)] = c
    got = BW.token_sparse_backward(q_s, k, v, idx, W, do)
    tq, tk, tv = _t(q_s), _t(k), _t(v)
    kpos = torch.arange(N)
    outs = []
    for h in range(Hq):
        g = h // (Hq // Hkv)
        o_h = torch.zeros(N, D, dtype=torch.float64)
        for I_ in range(T):
            rows = torch.from_numpy(O.tile_rows(I_, N))
            in_sel = torch.zeros(N, dtype=torch.bool)
            for i in idx[0, g, I_]:
                if i >= 0:
                    in_sel[i] = True
            vis = (kpos[None, :] <= rows[:, None]) & (in_sel[None, :] | (kpos[None, :] >= rows[:, None] - W + 1))
            o_h = o_h.index_put((rows,), _torch_attention(tq[0, h, rows], tk[0, g], tv[0, g], vis))
        outs.append(o_h)
    (torch.stack(outs)[None] * torch.from_numpy(do)).sum().backward()
    for name, ten in (("dq", tq), ("dk", tk), ("dv", tv)):
        np.testing.assert_allclose(got[name], ten.grad.numpy(), rtol=1e-9, atol=1e-11, err_msg=name)


def test_backward_pins_catch_planted_mistakes(monkeypatch):
    """Plant plausible mistakes in the gradient oracle (a dropped D_t term, a missing scale, the
    gate derivative without the 1 - sigmoid factor) and check that a pin above fails."""
    import pytest
    orig = BW.attention_rows_backward

    def no_d_term(q_rows, t_rows, k, v, d_o, keys_visible=None, sink=None):
        q_rows, k, v, d_o = (np.asarray(x, np.float64) for x in (q_rows, k, v, d_o))
        tau = 1.0 / math.sqrt(q_rows.shape[1])
        p, _, _ = O.causal_softmax(q_rows, t_rows, k, keys_visible, sink)
        ds = p * (d_o @ v.T)                    # D_t dropped
        return tau * (ds @ k), tau * (ds.T @ q_rows), p.T @ d_o, 0.0

    monkeypatch.setattr(BW, "attention_rows_backward", no_d_term)
    with pytest.raises(AssertionError):
        test_rows_backward_matches_autograd()
    with pytest.raises(AssertionError):
        test_full_backward_matches_sdpa_autograd()

    def no_scale(*a, **kw):
        dq, dk, dv, ds = orig(*a, **kw)
        return dq * math.sqrt(np.asarray(a[0]).shape[1]), dk, dv, ds

    monkeypatch.setattr(BW, "attention_rows_backward", no_scale)
    with pytest.raises(AssertionError):
        test_rows_backward_matches_autograd()
    monkeypatch.undo()

    # the gate derivative without the (1 - sigmoid) factor differs from autograd's
    rng = np.random.default_rng(46)
    B, Hq, Hkv, N, D, win = 1, 2, 1, 70, 8, 12
    q_s, do = rng.standard_normal((B, Hq, N, D)), rng.standard_normal((B, Hq, N, D))
    k, v, ks, vs = (rng.standard_normal((B, Hkv, N, D)) for _ in range(4))
    gate = rng.standard_normal((B, Hq, N, 2))
    idx = np.array([[[[0], [1]]]])
    good = BW.sparse_attention_backward(q_s, k, v, idx, ks, vs, win, gate, do)
    bad = good["dgate"] / (1.0 - BW.sigmoid(gate))
    tg = _t(gate)
    sel_sets = {(0, 0, 0): [0], (0, 0, 1): [1]}
    o = _torch_sparse_layer(_t(q_s, False), _t(k, False), _t(v, False), sel_sets, _t(ks, False), _t(vs, False), win,
                            tg, None, [(0, O.tile_rows(0, N)), (1, O.tile_rows(1, N))])
    (o * torch.from_numpy(do)).sum().backward()
    np.testing.assert_allclose(good["dgate"], tg.grad.numpy(), rtol=1e-9, atol=1e-11)
    assert not np.allclose(bad, tg.grad.numpy(), rtol=1e-6, atol=1e-9)
