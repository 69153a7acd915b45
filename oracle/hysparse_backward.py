"""Plain float64 CPU oracle for the gradients of the HySparse hybrid block.

TEST INFRASTRUCTURE ONLY.  Only tests may import this module; the product path (the CUDA
library and its Python binding) never calls it and shares no code with it.

What it computes ([HS] §3.4.6, training pipeline: no auxiliary loss for the selection; the
selected indices come from the full layer and are constants of the step, and the sparse layers'
gradients reach the full layer's K and V through the shared cache):

* attention over a set of visible keys with scale tau = 1/sqrt(D), p = softmax(tau q.k), and an
  optional sink logit that joins the softmax as an entry with a zero value:
      dV_i = sum_t p_ti dO_t,  dP_ti = dO_t . v_i,  D_t = dO_t . o_t,
      dS_ti = p_ti (dP_ti - D_t),  dQ_t = tau sum_i dS_ti k_i,  dK_i = tau sum_t dS_ti q_t,
      d(sink) = -sum_t p_sink,t D_t;
* the gated sparse layer o = sigmoid(g0) o~ + sigmoid(g1) o' ([HS] §3.4.3):
      d o~ = sigmoid(g0) dO,  d o' = sigmoid(g1) dO,
      d g_b = sigmoid(g_b) (1 - sigmoid(g_b)) (dO . o_b) for the two branches;
  the sparse branch's dK, dV land on the shared cache at the selected blocks' keys, the window
  branch's on the layer's own K', V';
* the hybrid block: the shared K, V gradient is the full layer's plus every sparse layer's.

Each formula is the derivative of the forward definition in oracle/hysparse_oracle.py, written
out; the pins in tests/test_oracle_backward.py check them against torch's float64 autograd.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence

import numpy as np

from .hysparse_oracle import causal_softmax, sigmoid, tile_rows


def attention_rows_backward(q_rows, t_rows, k, v, d_o, keys_visible=None, sink: Optional[float] = None):
    """Gradients of o_t = sum_i p_ti v_i for some rows of one head.

    q_rows [R, D], t_rows [R], k, v [N, D], d_o [R, D]; keys_visible as in causal_softmax.
    Returns dq [R, D], dk [N, D], dv [N, D] and d(sink) (0.0 without a sink)."""
    q_rows = np.asarray(q_rows, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    d_o = np.asarray(d_o, np.float64)
    tau = 1.0 / math.sqrt(q_rows.shape[1])
    p, m, l = causal_softmax(q_rows, t_rows, k, keys_visible, sink)
    o = p @ v
    dv = p.T @ d_o
    dp = d_o @ v.T
    dd = np.sum(d_o * o, axis=1)
    ds = p * (dp - dd[:, None])
    dq = tau * (ds @ k)
    dk = tau * (ds.T @ q_rows)
    dsink = 0.0
    if sink is not None:
        p_sink = np.exp(sink - m) / l
        dsink = float(-np.sum(p_sink * dd))
    return dq, dk, dv, dsink


def full_attention_backward(q, k, v, d_o):
    """Causal GQA full layer. q, d_o [B,Hq,N,D]; k, v [B,Hkv,N,D] -> dq, dk, dv."""
    B, Hq, N, D = q.shape
    G = Hq // k.shape[1]
    dq = np.zeros((B, Hq, N, D))
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    rows = np.arange(N)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            dq[b, h], dk_h, dv_h, _ = attention_rows_backward(q[b, h], rows, k[b, g], v[b, g], d_o[b, h])
            dk[b, g] += dk_h
            dv[b, g] += dv_h
    return dq, dk, dv


def sparse_attention_backward(q_s, k, v, idx, k_swa, v_swa, window: int, gate, d_o, block: int = 64,
                              sinks=None, per_row: bool = False) -> Dict[str, np.ndarray]:
    """Gradients of one sparse layer.  Arguments as sparse_attention (idx [B,Hkv,T,k]) or, with
    per_row, as sparse_attention_rows (idx [B,Hkv,N,k]); d_o [B,Hq,N,D].

    Returns dq, dk, dv (shared cache), dk_swa, dv_swa, dgate [B,Hq,N,2] and dsinks [Hq,2]
    (zeros without sinks)."""
    B, Hq, N, D = q_s.shape
    G = Hq // k.shape[1]
    T = (N + block - 1) // block
    out = {"dq": np.zeros((B, Hq, N, D)), "dk": np.zeros(k.shape), "dv": np.zeros(v.shape),
           "dk_swa": np.zeros(k_swa.shape), "dv_swa": np.zeros(v_swa.shape), "dgate": np.zeros((B, Hq, N, 2)),
           "dsinks": np.zeros((Hq, 2))}
    kpos = np.arange(N)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            s0 = None if sinks is None else float(sinks[h][0])
            s1 = None if sinks is None else float(sinks[h][1])
            groups = [(np.array([t]), idx[b, g, t]) for t in range(N)] if per_row else \
                [(tile_rows(I, N, block), idx[b, g, I]) for I in range(T)]
            for rows, sel in groups:
                in_sel = np.zeros(N, dtype=bool)
                for j in sel:
                    if j >= 0:
                        in_sel[j * block:min(N, (j + 1) * block)] = True
                vis_sp = np.broadcast_to(in_sel, (len(rows), N))
                vis_sw = kpos[None, :] >= (rows[:, None] - window + 1)
                qr = np.asarray(q_s[b, h, rows], np.float64)
                gr = sigmoid(gate[b, h, rows])
                dor = np.asarray(d_o[b, h, rows], np.float64)
                # branch outputs (for the gate gradient) and the branch backward passes
                p_sp, _, _ = causal_softmax(qr, rows, k[b, g], vis_sp, s0)
                o_sp = p_sp @ np.asarray(v[b, g], np.float64)
                p_sw, _, _ = causal_softmax(qr, rows, k_swa[b, g], vis_sw, s1)
                o_sw = p_sw @ np.asarray(v_swa[b, g], np.float64)
                out["dgate"][b, h, rows, 0] = gr[:, 0] * (1.0 - gr[:, 0]) * np.sum(dor * o_sp, axis=1)
                out["dgate"][b, h, rows, 1] = gr[:, 1] * (1.0 - gr[:, 1]) * np.sum(dor * o_sw, axis=1)
                dq0, dk0, dv0, ds0 = attention_rows_backward(qr, rows, k[b, g], v[b, g], gr[:, 0:1] * dor, vis_sp, s0)
                dq1, dk1, dv1, ds1 = attention_rows_backward(qr, rows, k_swa[b, g], v_swa[b, g], gr[:, 1:2] * dor,
                                                             vis_sw, s1)
                out["dq"][b, h, rows] = dq0 + dq1
                out["dk"][b, g] += dk0
                out["dv"][b, g] += dv0
                out["dk_swa"][b, g] += dk1
                out["dv_swa"][b, g] += dv1
                if sinks is not None:
                    out["dsinks"][h, 0] += ds0
                    out["dsinks"][h, 1] += ds1
    return out


def token_sparse_backward(q_s, k, v, idx, forced: int, d_o, block: int = 64) -> Dict[str, np.ndarray]:
    """Gradients of one token-sparse layer ([HS2] "Precise retrieval without a separate indexer":
    row t of tile I attends Sel_I united with [max(0, t-forced+1), t] over the shared K, V, no
    gate).  idx [B,Hkv,T,k_tokens]; returns dq, dk, dv."""
    B, Hq, N, D = q_s.shape
    G = Hq // k.shape[1]
    T = (N + block - 1) // block
    out = {"dq": np.zeros((B, Hq, N, D)), "dk": np.zeros(k.shape), "dv": np.zeros(v.shape)}
    kpos = np.arange(N)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            for I in range(T):
                rows = tile_rows(I, N, block)
                in_sel = np.zeros(N, dtype=bool)
                sel = np.asarray([i for i in idx[b, g, I] if i >= 0], dtype=np.int64)
                in_sel[sel] = True
                vis = in_sel[None, :] | (kpos[None, :] >= rows[:, None] - forced + 1)
                dq, dk, dv, _ = attention_rows_backward(q_s[b, h, rows], rows, k[b, g], v[b, g], d_o[b, h, rows], vis)
                out["dq"][b, h, rows] = dq
                out["dk"][b, g] += dk
                out["dv"][b, g] += dv
    return out


def hybrid_block_backward(q, k, v, d_o_full, sparse_layers: Sequence[dict], window: int, block: int = 64):
    """The hybrid block's gradients: the full layer plus the sparse layers, whose gradients of the
    shared K, V are added to the full layer's.  Each sparse layer is a dict with q_s, idx, k_swa,
    v_swa, gate, d_o (and optionally sinks, per_row).  Returns the full layer's dq, the shared
    dk, dv, and the per-layer gradient dicts."""
    dq, dk, dv = full_attention_backward(q, k, v, d_o_full)
    layers = []
    for L in sparse_layers:
        gL = sparse_attention_backward(L["q_s"], k, v, L["idx"], L["k_swa"], L["v_swa"], window, L["gate"], L["d_o"],
                                       block, L.get("sinks"), L.get("per_row", False))
        dk = dk + gL["dk"]
        dv = dv + gL["dv"]
        layers.append(gL)
    return {"dq": dq, "dk": dk, "dv": dv, "layers": layers}
