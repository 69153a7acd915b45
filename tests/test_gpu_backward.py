"""GPU parity of the training path against the float64 gradient oracle, through the C ABI: the
sparse layer's training forward (its saved branch statistics), the full layer's backward, the
sparse layer's backward (both branches, gate and sink gradients) and the hybrid block's shared
K/V gradient summed over its layers.  The selection is a constant of the step, so the oracle
runs on the GPU's own indices."""
import numpy as np
import pytest
import torch

import oracle as O
from oracle import hysparse_backward as OB
from attention_tcgen05_tma_b200 import hysparse as H
from attention_tcgen05_tma_b200 import inputs as I
from tests.gpu_support import DQ_TOL, GRAD_TOL, TOL, grad_err, to_dev, to_np

pytestmark = pytest.mark.gpu

CASES = [
    # name, dtype, B, N, Hq, Hkv, D, k, window
    ("bf16_d128_g4_ragged", "bf16", 2, 300, 8, 2, 128, 2, 64),       # tensor cores, ragged tail
    ("bf16_d128_g8_tiles", "bf16", 1, 1000, 16, 2, 128, 4, 128),     # tensor cores, many key tiles
    ("bf16_d64_g2", "bf16", 1, 200, 4, 2, 64, 2, 100),               # SIMT (D = 64)
    ("bf16_d128_g1", "bf16", 1, 130, 2, 2, 128, 2, 64),              # SIMT (odd group)
    ("f32_d64_g4", "f32", 1, 256, 4, 1, 64, 2, 128),                 # SIMT fp32
]


def _workload(dt, B, N, Hq, Hkv, D, k, window, layers=1, seed=21):
    base = I.WORKLOADS["tiny"] if dt == "f32" else I.WORKLOADS["dense7b"]
    return I.scaled(base, B=B, N=N, Hq=Hq, Hkv=Hkv, D=D, topk=k, window=window, layers=layers, seed=seed,
                    scale_std=1.0 if dt == "f32" else 1.0 / np.sqrt(D), n_plants=min(8, N // 64))


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_full_layer_backward(case):
    name, dt, B, N, Hq, Hkv, D, k, window = case
    w = _workload(dt, B, N, Hq, Hkv, D, k, window, layers=0)
    a = I.prefill_arrays(w, grads=True)
    q, kk, vv, do = (to_dev(a[x], dt) for x in ("q", "k", "v", "d_o"))
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
    o, _ = H.full_attn_select(q, kk, vv, lse=lse)
    dq, dk, dv = H.full_attn_backward(q, kk, vv, o, do, lse)
    # accumulate: added to what the buffers hold
    base_k = torch.randn(kk.shape, device="cuda")
    base_v = torch.randn(vv.shape, device="cuda")
    dk2, dv2 = base_k.clone(), base_v.clone()
    H.full_attn_backward(q, kk, vv, o, do, lse, dk=dk2, dv=dv2, accumulate=True)
    torch.cuda.synchronize()
    assert H.hysparse_get_device_status() == 0
    ref_q, ref_k, ref_v = OB.full_attention_backward(a["q"], a["k"], a["v"], a["d_o"])
    tol = GRAD_TOL[dt]
    assert grad_err(to_np(dq), ref_q) <= DQ_TOL[dt], grad_err(to_np(dq), ref_q)
    assert grad_err(to_np(dk), ref_k) <= tol, grad_err(to_np(dk), ref_k)
    assert grad_err(to_np(dv), ref_v) <= tol, grad_err(to_np(dv), ref_v)
    # the kernels are deterministic: the accumulated result is the buffer plus the same gradient, up
    # to the rounding of that one fp32 addition (a fused multiply-add may skip the product's rounding)
    ulp = 1.2e-7
    assert torch.allclose(dk2, base_k + dk, rtol=0, atol=4 * ulp * float(base_k.abs().max()))
    assert torch.allclose(dv2, base_v + dv, rtol=0, atol=4 * ulp * float(base_v.abs().max()))


def _branch_lse(q_s, k, v, idx, k_swa, window, sinks, G, block=64):
    """The oracle's per-branch log normaliser (sink included), [B,Hq,N,2]."""
    B, Hq, N, D = q_s.shape
    out = np.zeros((B, Hq, N, 2))
    kpos = np.arange(N)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            for I_ in range((N + block - 1) // block):
                rows = O.tile_rows(I_, N, block)
                in_sel = np.zeros(N, dtype=bool)
                for j in idx[b, g, I_]:
                    if j >= 0:
                        in_sel[j * block:(j + 1) * block] = True
                s0 = None if sinks is None else float(sinks[h][0])
                s1 = None if sinks is None else float(sinks[h][1])
                _, m0, l0 = O.causal_softmax(q_s[b, h, rows], rows, k[b, g], np.broadcast_to(in_sel, (len(rows), N)), s0)
                vis = kpos[None, :] >= rows[:, None] - window + 1
                _, m1, l1 = O.causal_softmax(q_s[b, h, rows], rows, k_swa[b, g], vis, s1)
                out[b, h, rows, 0] = m0 + np.log(l0)
                out[b, h, rows, 1] = m1 + np.log(l1)
    return out


def _sparse_inputs(a, l, dt):
    return [to_dev(a[x][l], dt) for x in ("q_sparse", "k_swa", "v_swa")] + [to_dev(a["gate"][l], "f32")]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("with_sinks", [False, True], ids=["nosink", "sinks"])
def test_sparse_layer_train_and_backward(case, with_sinks):
    name, dt, B, N, Hq, Hkv, D, k, window = case
    w = _workload(dt, B, N, Hq, Hkv, D, k, window, layers=1)
    a = I.prefill_arrays(w, grads=True)
    q, kk, vv = (to_dev(a[x], dt) for x in ("q", "k", "v"))
    _, sc = H.full_attn_select(q, kk, vv)
    idx = H.topk(sc, k)
    qs, ks, vs, gate = _sparse_inputs(a, 0, dt)
    sinks_np = I.sink_logits(w, 0) if with_sinks else None
    sinks = torch.from_numpy(sinks_np).cuda() if with_sinks else None
    o_inf = H.sparse_attn(qs, kk, vv, idx, ks, vs, window, gate, sinks=sinks)
    o, osp, blse = H.sparse_attn_train(qs, kk, vv, idx, ks, vs, window, gate, sinks=sinks)
    do = to_dev(a["d_o_sparse"][0], dt)
    dk_sh = torch.randn(kk.shape, device="cuda")      # the shared gradient is added to what the buffer holds
    dv_sh = torch.randn(vv.shape, device="cuda")
    base_k, base_v = dk_sh.clone(), dv_sh.clone()
    dq, dks, dvs, dgate, dsinks = H.sparse_attn_backward(qs, kk, vv, idx, ks, vs, window, gate, o, osp, blse, do,
                                                         dk_sh, dv_sh, sinks=sinks)
    torch.cuda.synchronize()
    assert H.hysparse_get_device_status() == 0
    assert torch.equal(o, o_inf)                      # the training forward computes the same output
    gidx = idx.cpu().numpy().astype(np.int64)
    G = Hq // Hkv
    # saved statistics: the gated sparse part and each branch's LSE
    o_sp_ref = np.zeros(a["q"].shape)
    for b in range(B):
        for h in range(Hq):
            for I_ in range(w.T):
                rows = O.tile_rows(I_, N)
                s0 = None if sinks_np is None else float(sinks_np[h][0])
                part = O.sparse_branch_rows(a["q_sparse"][0][b, h, rows], rows, a["k"][b, h // G], a["v"][b, h // G],
                                            gidx[b, h // G, I_], 64, s0)
                o_sp_ref[b, h, rows] = O.sigmoid(a["gate"][0][b, h, rows, 0])[:, None] * part
    assert np.max(np.abs(to_np(osp) - o_sp_ref)) <= TOL[dt]
    lse_ref = _branch_lse(a["q_sparse"][0], a["k"], a["v"], gidx, a["k_swa"][0], window, sinks_np, G)
    assert np.max(np.abs(to_np(blse) - lse_ref)) <= (2e-3 if dt == "bf16" else 1e-5)
    # gradients
    ref = OB.sparse_attention_backward(a["q_sparse"][0], a["k"], a["v"], gidx, a["k_swa"][0], a["v_swa"][0], window,
                                       a["gate"][0], a["d_o_sparse"][0], sinks=sinks_np)
    tol = GRAD_TOL[dt]
    checks = {"dq": to_np(dq), "dk": to_np(dk_sh - base_k), "dv": to_np(dv_sh - base_v), "dk_swa": to_np(dks),
              "dv_swa": to_np(dvs), "dgate": to_np(dgate)}
    if with_sinks:
        checks["dsinks"] = to_np(dsinks)
    for key, val in checks.items():
        e = grad_err(val, ref[key])
        assert e <= (DQ_TOL[dt] if key == "dq" else tol), (key, e)


def test_hybrid_block_backward():
    """Full layer + 2 sparse layers (tensor-core path): the shared K, V gradient is the full
    layer's plus every sparse layer's, accumulated in the same fp32 buffers."""
    dt = "bf16"
    w = _workload(dt, 1, 512, 8, 2, 128, 3, 128, layers=2, seed=23)
    a = I.prefill_arrays(w, grads=True)
    q, kk, vv, do = (to_dev(a[x], dt) for x in ("q", "k", "v", "d_o"))
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device="cuda")
    o, sc = H.full_attn_select(q, kk, vv, lse=lse)
    idx = H.topk(sc, w.topk)
    dq, dk, dv = H.full_attn_backward(q, kk, vv, o, do, lse)
    layers = []
    for l in range(w.layers):
        qs, ks, vs, gate = _sparse_inputs(a, l, dt)
        ol, osp, blse = H.sparse_attn_train(qs, kk, vv, idx, ks, vs, w.window, gate)
        dol = to_dev(a["d_o_sparse"][l], dt)
        layers.append(H.sparse_attn_backward(qs, kk, vv, idx, ks, vs, w.window, gate, ol, osp, blse, dol, dk, dv))
    torch.cuda.synchronize()
    assert H.hysparse_get_device_status() == 0
    gidx = idx.cpu().numpy().astype(np.int64)
    ref = OB.hybrid_block_backward(a["q"], a["k"], a["v"], a["d_o"],
                                   [dict(q_s=a["q_sparse"][l], idx=gidx, k_swa=a["k_swa"][l], v_swa=a["v_swa"][l],
                                         gate=a["gate"][l], d_o=a["d_o_sparse"][l]) for l in range(w.layers)],
                                   w.window)
    tol = GRAD_TOL[dt]
    assert grad_err(to_np(dq), ref["dq"]) <= DQ_TOL[dt]
    assert grad_err(to_np(dk), ref["dk"]) <= tol
    assert grad_err(to_np(dv), ref["dv"]) <= tol
    for l in range(w.layers):
        assert grad_err(to_np(layers[l][0]), ref["layers"][l]["dq"]) <= DQ_TOL[dt]
        assert grad_err(to_np(layers[l][3]), ref["layers"][l]["dgate"]) <= tol
