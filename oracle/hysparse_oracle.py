"""Plain float64 CPU oracle for the HySparse hybrid-block attention hot path.

TEST INFRASTRUCTURE ONLY.  Only tests, the smoke check and the benchmark's CPU
baseline leg may import this module; the product path (the CUDA library and its
Python binding) never calls it and shares no code with it.

Every function follows the equations of

* [HS]  "HySparse: A Hybrid Sparse Attention Architecture with Oracle Token
        Selection and KV Cache Sharing" (paper-graph long-form summary), §3.4.1
        (full attention o_t, block-level max score S_t^i, the two-pass rescale,
        GQA group aggregation), §3.4.2 (TopK block selection), §3.4.3 (sparse
        branch gather and attention, SWA branch, sigmoid gated fusion);
* [HSP] the HySparse paper text (paperpeel extraction), §3.1-§3.3;
* [HS2] the HySparse2 explainer (deep-reads), sections "Precise retrieval
        without a separate indexer" (token-level selection, forced newest 128
        tokens) and "Twenty lines of algorithmic intuition" (decode step).

Readings where the pages leave a step open (each is listed in the design notes):

* The block score of a (KV group g, 64-query tile I, key block j) is
  R_{h in g} R_{t in tile I} S^h_{t,j}, with R = sum by default (the summed
  hardware-tile aggregation) or R = max (the paper's conservative group max).
* S_{t,j} is the max over keys of block j that are <= t of the post-softmax
  probability (the rescale step is exp(m~ - m)/l; the printed formula lost the exp).
* TopK: candidates j in [0, I]; order by (score descending, index ascending);
  fewer than k candidates -> all of them; emitted ascending, padded with -1.
* Per-position selection ([HS] §3.4.1-§3.4.2 as printed): S_g[t, j] = max over the
  group's heads of S^h_{t,j}; row t selects the top k of its floor(t/64) + 1 blocks and its
  sparse branch attends {i <= t : floor(i/64) in Sel_t}.
* Sparse row t of tile I attends {i <= t : floor(i/64) in Sel_I}; the SWA branch
  attends [max(0, t-w+1), t]; o = sigmoid(g0) * o_sparse + sigmoid(g1) * o_swa.
* Token variant: token score = sum over the group's heads and the tile's rows
  t >= i of P_{t,i}; candidates [0, e_I - W] with e_I the tile's last row and W
  the forced window; row t attends Sel_I united with [max(0, t-W+1), t], each
  token once, no gate.
* Decode: the new token sits at position L-1 of an L-token cache; it is its own
  tile; candidates are all blocks (block variant).
* Token-variant decode ([HS2] "Twenty lines of algorithmic intuition" with the token
  granularity of "Precise retrieval without a separate indexer"): the new token at
  position L-1 scores every cached token i < L by sum over the group's heads of P_i;
  candidates are the tokens older than the forced newest W, [0, L-1-W]; row L-1
  attends the top-k candidates united with [L-W, L-1], each token once, no gate.
* FP8 KV cache ([HS2] "What actually improved?", the KV-cache-at-1M-tokens row, which
  sizes the cache in FP8; the pages fix neither the FP8 format nor the scaling): each
  cached K or V element is an OCP E4M3 code (the "fn" variant: bias 7, no infinities,
  S.1111.111 is NaN), and its value is the decoded code times a float32 scale of its
  KV head, one scale for K and one for V.  The decode step then runs on these values.
* Sink biases ([HSP] §4.1, per-head learnable sinks in the sparse and SWA branches,
  following gpt-oss): one logit per (head, branch), sinks [Hq, 2] with index 0 for
  the sparse branch and 1 for the SWA branch; it joins the branch's softmax as an
  extra entry with a zero value, so the denominator gains exp(sink - m).

All arithmetic is float64; inputs are converted exactly (bf16 and fp32 values are
exactly representable in float64).
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

NEG_INF = -np.inf


# -----------------------------------------------------------------------------
# dense causal attention  ([HS] §3.4.1, equation for o_t)
# -----------------------------------------------------------------------------
def causal_softmax(q_rows: np.ndarray, t_rows: np.ndarray, k: np.ndarray,
                   keys_visible: Optional[np.ndarray] = None, sink: Optional[float] = None
                   ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Softmax attention probabilities of some query rows against the keys of one head.

    q_rows [R, D], t_rows [R] (absolute query positions), k [N, D].
    keys_visible, if given, is a boolean [R, N] mask of the keys each row may see
    (it is intersected with causality i <= t).  sink, if given, is a logit that joins
    every row's softmax as an extra entry with a zero value.
    Returns P [R, N] (zero where a key is not visible), the row max m [R] of the
    scaled logits (and the sink) and the normaliser l [R] = sum_i exp(s_i - m)
    (+ exp(sink - m)).
    """
    q_rows = np.asarray(q_rows, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    d = q_rows.shape[1]
    tau = 1.0 / math.sqrt(d)
    s = tau * (q_rows @ k.T)
    visible = np.arange(k.shape[0])[None, :] <= np.asarray(t_rows)[:, None]
    if keys_visible is not None:
        visible = visible & keys_visible
    s = np.where(visible, s, NEG_INF)
    m = s.max(axis=1)
    if sink is not None:
        m = np.maximum(m, sink)
    e = np.where(visible, np.exp(s - m[:, None]), 0.0)
    l = e.sum(axis=1)
    if sink is not None:
        l = l + np.exp(sink - m)
    return e / l[:, None], m, l


def attention_rows(q_rows, t_rows, k, v, keys_visible=None, sink=None):
    """o_t = sum_i P_{t,i} v_i for the given rows; also returns LSE_t = m_t + log l_t."""
    p, m, l = causal_softmax(q_rows, t_rows, k, keys_visible, sink)
    o = p @ np.asarray(v, dtype=np.float64)
    return o, m + np.log(l)


def full_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, chunk: int = 1024
                   ) -> Tuple[np.ndarray, np.ndarray]:
    """Causal GQA attention over all rows. q [B,Hq,N,D]; k, v [B,Hkv,N,D].

    Query head h reads KV head h // (Hq // Hkv).  Returns o [B,Hq,N,D] and LSE [B,Hq,N]
    (natural-log units of the scaled logits)."""
    B, Hq, N, D = q.shape
    G = Hq // k.shape[1]
    o = np.zeros((B, Hq, N, D))
    lse = np.zeros((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            kk = np.asarray(k[b, h // G], dtype=np.float64)
            vv = np.asarray(v[b, h // G], dtype=np.float64)
            for r0 in range(0, N, chunk):
                rows = np.arange(r0, min(N, r0 + chunk))
                o[b, h, rows], lse[b, h, rows] = attention_rows(q[b, h, rows], rows, kk, vv)
    return o, lse


# -----------------------------------------------------------------------------
# block-level max scores  ([HS] §3.4.1, equation for S_t^i and the rescale pass)
# -----------------------------------------------------------------------------
def block_max_probs(p: np.ndarray, t_rows: np.ndarray, block: int = 64) -> np.ndarray:
    """S[r, j] = max over keys i of block j with i <= t_r of P[r, i]; 0 when the block
    starts after t_r (the block is then empty for that row)."""
    R, N = p.shape
    nb = (N + block - 1) // block
    s = np.zeros((R, nb))
    for j in range(nb):
        s[:, j] = p[:, j * block:min(N, (j + 1) * block)].max(axis=1)
    # P is zero beyond t, so the max over the whole block equals the max over the
    # part clipped at t; a block that starts after t holds only zeros.
    s[np.arange(nb)[None, :] * block > np.asarray(t_rows)[:, None]] = 0.0
    return s


def tile_rows(I: int, N: int, block: int = 64) -> np.ndarray:
    return np.arange(I * block, min(N, (I + 1) * block))


def block_scores_tile(q_group: np.ndarray, k: np.ndarray, I: int, reduce: str = "sum",
                      block: int = 64) -> np.ndarray:
    """Aggregated block scores of one (KV group, query tile I): a vector over key blocks.

    q_group [G, N, D] holds the group's query heads; k [N, D] its KV head.
    score[j] = R_h R_{t in tile I} S^h_{t,j} for j <= I (0 for j > I), R = sum or max
    ([HS] §3.4.1 'GQA aggregation' with the reading above)."""
    N = k.shape[0]
    nb = (N + block - 1) // block
    rows = tile_rows(I, N, block)
    acc = np.zeros(nb)
    for h in range(q_group.shape[0]):
        p, _, _ = causal_softmax(q_group[h][rows], rows, k)
        s = block_max_probs(p, rows, block)
        part = s.sum(axis=0) if reduce == "sum" else s.max(axis=0)
        acc = acc + part if reduce == "sum" else np.maximum(acc, part)
    acc[I + 1:] = 0.0
    return acc


def block_scores(q: np.ndarray, k: np.ndarray, reduce: str = "sum", block: int = 64) -> np.ndarray:
    """All block scores: [B, Hkv, T, NB]."""
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    T = (N + block - 1) // block
    out = np.zeros((B, Hkv, T, T))
    for b in range(B):
        for g in range(Hkv):
            qg = np.asarray(q[b, g * G:(g + 1) * G], dtype=np.float64)
            kk = np.asarray(k[b, g], dtype=np.float64)
            for I in range(T):
                out[b, g, I] = block_scores_tile(qg, kk, I, reduce, block)
    return out


def block_scores_rows(q: np.ndarray, k: np.ndarray, block: int = 64) -> np.ndarray:
    """Per-position group scores ([HS] §3.4.1 group-wise maximum over the group's heads, taken
    per (query position, key block) entry; §3.4.2 selection per query position):
    S_g[t, j] = max_h S^h_{t,j}, with S^h_{t,j} the largest probability of row t inside block j
    (keys <= t); 0 for blocks that start after t.  Returns [B, Hkv, N, NB]."""
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    nb = (N + block - 1) // block
    out = np.zeros((B, Hkv, N, nb))
    for b in range(B):
        for g in range(Hkv):
            kk = np.asarray(k[b, g], dtype=np.float64)
            for I in range(nb):
                rows = tile_rows(I, N, block)
                acc = np.zeros((len(rows), nb))
                for h in range(g * G, (g + 1) * G):
                    p, _, _ = causal_softmax(np.asarray(q[b, h, rows], np.float64), rows, kk)
                    acc = np.maximum(acc, block_max_probs(p, rows, block))
                out[b, g, rows] = acc
    return out


# -----------------------------------------------------------------------------
# TopK  ([HS] §3.4.2; tie and padding rules are the reading above)
# -----------------------------------------------------------------------------
def select_topk(scores: np.ndarray, n_candidates: int, k: int) -> np.ndarray:
    """Indices of the k largest among scores[0:n_candidates], ties to the lower index,
    returned ascending and padded with -1 to length k."""
    cand = np.arange(n_candidates)
    order = np.lexsort((cand, -np.asarray(scores[:n_candidates], dtype=np.float64)))
    chosen = np.sort(order[:k])
    out = np.full(k, -1, dtype=np.int64)
    out[:len(chosen)] = chosen
    return out


def topk_blocks(scores: np.ndarray, k: int) -> np.ndarray:
    """[B, Hkv, T, NB] scores -> [B, Hkv, T, k] block indices; tile I has I+1 candidates."""
    B, Hkv, T, NB = scores.shape
    out = np.full((B, Hkv, T, k), -1, dtype=np.int64)
    for b in range(B):
        for g in range(Hkv):
            for I in range(T):
                out[b, g, I] = select_topk(scores[b, g, I], min(I + 1, NB), k)
    return out


def topk_blocks_rows(scores: np.ndarray, k: int, block: int = 64) -> np.ndarray:
    """[B, Hkv, N, NB] per-position scores -> [B, Hkv, N, k] block indices ([HS] §3.4.2: for each
    query position t and group, the k highest of the floor(t/64) + 1 blocks holding keys <= t);
    ties to the lower index, ascending, padded with -1."""
    B, Hkv, N, NB = scores.shape
    out = np.full((B, Hkv, N, k), -1, dtype=np.int64)
    for b in range(B):
        for g in range(Hkv):
            for t in range(N):
                out[b, g, t] = select_topk(scores[b, g, t], min(t // block + 1, NB), k)
    return out


# -----------------------------------------------------------------------------
# sparse layer  ([HS] §3.4.3: gather, sparse branch, SWA branch, gated fusion)
# -----------------------------------------------------------------------------
def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-np.asarray(x, dtype=np.float64)))


def sparse_branch_rows(q_rows, t_rows, k, v, sel_blocks: Sequence[int], block: int = 64, sink=None):
    """Sparse-branch output of rows of one tile: keys i <= t with floor(i/64) in Sel."""
    N = k.shape[0]
    in_sel = np.zeros(N, dtype=bool)
    for j in sel_blocks:
        if j >= 0:
            in_sel[j * block:min(N, (j + 1) * block)] = True
    o, _ = attention_rows(q_rows, t_rows, k, v, np.broadcast_to(in_sel, (len(t_rows), N)), sink)
    return o


def swa_branch_rows(q_rows, t_rows, k_swa, v_swa, window: int, sink=None):
    """SWA-branch output: keys in [max(0, t-w+1), t] of the layer's own K', V'."""
    N = k_swa.shape[0]
    i = np.arange(N)[None, :]
    vis = i >= (np.asarray(t_rows)[:, None] - window + 1)
    o, _ = attention_rows(q_rows, t_rows, k_swa, v_swa, vis, sink)
    return o


def gated_sparse_rows(q_rows, t_rows, k, v, sel_blocks, k_swa, v_swa, window, gate_rows,
                      block: int = 64, sinks=None):
    """o_t = sigmoid(g0) * o~_t + sigmoid(g1) * o'_t for rows of one tile; sinks, if given,
    is this head's (sparse-branch, SWA-branch) sink logit pair."""
    s0, s1 = (None, None) if sinks is None else (float(sinks[0]), float(sinks[1]))
    o_sp = sparse_branch_rows(q_rows, t_rows, k, v, sel_blocks, block, s0)
    o_sw = swa_branch_rows(q_rows, t_rows, k_swa, v_swa, window, s1)
    g = sigmoid(gate_rows)
    return g[:, 0:1] * o_sp + g[:, 1:2] * o_sw


def sparse_attention(q_s, k, v, idx, k_swa, v_swa, window: int, gate, block: int = 64, sinks=None):
    """Whole sparse layer. q_s [B,Hq,N,D]; k, v, k_swa, v_swa [B,Hkv,N,D];
    idx [B,Hkv,T,k]; gate [B,Hq,N,2]; sinks None or [Hq,2].  Returns o [B,Hq,N,D]."""
    B, Hq, N, D = q_s.shape
    G = Hq // k.shape[1]
    T = (N + block - 1) // block
    o = np.zeros((B, Hq, N, D))
    for b in range(B):
        for h in range(Hq):
            g = h // G
            kk, vv = np.asarray(k[b, g], np.float64), np.asarray(v[b, g], np.float64)
            ks, vs = np.asarray(k_swa[b, g], np.float64), np.asarray(v_swa[b, g], np.float64)
            for I in range(T):
                rows = tile_rows(I, N, block)
                o[b, h, rows] = gated_sparse_rows(q_s[b, h, rows], rows, kk, vv, idx[b, g, I],
                                                  ks, vs, window, gate[b, h, rows], block,
                                                  None if sinks is None else sinks[h])
    return o


def sparse_attention_rows(q_s, k, v, idx_rows, k_swa, v_swa, window: int, gate, block: int = 64, sinks=None):
    """Whole sparse layer with per-position selection ([HS] §3.4.2 'computed per query position';
    §3.4.3 branches and gate): row t's sparse branch attends {i <= t : floor(i/64) in Sel_t} with
    Sel_t = idx_rows[b, g, t].  idx_rows [B,Hkv,N,k]; other arguments as sparse_attention."""
    B, Hq, N, D = q_s.shape
    G = Hq // k.shape[1]
    o = np.zeros((B, Hq, N, D))
    for b in range(B):
        for h in range(Hq):
            g = h // G
            kk, vv = np.asarray(k[b, g], np.float64), np.asarray(v[b, g], np.float64)
            ks, vs = np.asarray(k_swa[b, g], np.float64), np.asarray(v_swa[b, g], np.float64)
            for t in range(N):
                rows = np.array([t])
                o[b, h, t] = gated_sparse_rows(q_s[b, h, rows], rows, kk, vv, idx_rows[b, g, t], ks, vs, window,
                                               gate[b, h, rows], block, None if sinks is None else sinks[h])[0]
    return o


# -----------------------------------------------------------------------------
# token-granularity variant  ([HS2] "Precise retrieval without a separate indexer")
# -----------------------------------------------------------------------------
def token_scores_tile(q_group: np.ndarray, k: np.ndarray, I: int, block: int = 64) -> np.ndarray:
    """score_tok[i] = sum_{h in g} sum_{t in tile I, t >= i} P^h_{t,i}, over all keys i < N."""
    N = k.shape[0]
    rows = tile_rows(I, N, block)
    acc = np.zeros(N)
    for h in range(q_group.shape[0]):
        p, _, _ = causal_softmax(q_group[h][rows], rows, k)
        acc += p.sum(axis=0)
    return acc


def token_candidates(I: int, N: int, forced: int, block: int = 64) -> int:
    """Number of candidates of tile I: positions [0, e_I - forced], e_I the tile's last row."""
    e = min(N, (I + 1) * block) - 1
    return max(0, e - forced + 1)


def topk_tokens_tile(score_tok: np.ndarray, I: int, N: int, k_tokens: int, forced: int,
                     block: int = 64) -> np.ndarray:
    return select_topk(score_tok, token_candidates(I, N, forced, block), k_tokens)


def token_sparse_rows(q_rows, t_rows, k, v, sel_tokens: Sequence[int], forced: int):
    """Row t attends Sel united with [max(0, t-forced+1), t], each token once; no gate."""
    N = k.shape[0]
    in_sel = np.zeros(N, dtype=bool)
    sel = np.asarray([i for i in sel_tokens if i >= 0], dtype=np.int64)
    in_sel[sel] = True
    i = np.arange(N)[None, :]
    vis = in_sel[None, :] | (i >= (np.asarray(t_rows)[:, None] - forced + 1))
    o, _ = attention_rows(q_rows, t_rows, k, v, vis)
    return o


# -----------------------------------------------------------------------------
# decode  ([HS2] "Twenty lines of algorithmic intuition"; [HS] §3.4.1-§3.4.3)
# -----------------------------------------------------------------------------
def decode_full(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray, seqlens=None,
                reduce: str = "sum", block: int = 64):
    """One new token per sequence at position L_b - 1 against an L_b-token cache.

    q [B,Hq,D]; k_cache, v_cache [B,Hkv,L,D]. Returns o [B,Hq,D] and block scores
    [B,Hkv,NB] = R_{h in g} S^h_j (blocks past the sequence end score 0)."""
    B, Hq, D = q.shape
    Hkv, L = k_cache.shape[1], k_cache.shape[2]
    G = Hq // Hkv
    nb = (L + block - 1) // block
    o = np.zeros((B, Hq, D))
    sc = np.zeros((B, Hkv, nb))
    for b in range(B):
        Lb = L if seqlens is None else int(seqlens[b])
        for g in range(Hkv):
            kk = np.asarray(k_cache[b, g, :Lb], np.float64)
            vv = np.asarray(v_cache[b, g, :Lb], np.float64)
            for h in range(g * G, (g + 1) * G):
                t = np.array([Lb - 1])
                p, _, _ = causal_softmax(q[b, h][None, :], t, kk)
                o[b, h] = (p @ vv)[0]
                s = block_max_probs(p, t, block)[0]
                part = np.zeros(nb)
                part[:len(s)] = s
                sc[b, g] = sc[b, g] + part if reduce == "sum" else np.maximum(sc[b, g], part)
    return o, sc


def topk_decode(scores: np.ndarray, k: int, seqlens=None, L: Optional[int] = None, block: int = 64):
    """[B,Hkv,NB] -> [B,Hkv,k]; the candidates are the blocks that hold cached tokens."""
    B, Hkv, NB = scores.shape
    out = np.full((B, Hkv, k), -1, dtype=np.int64)
    for b in range(B):
        n = NB if seqlens is None else (int(seqlens[b]) + block - 1) // block
        for g in range(Hkv):
            out[b, g] = select_topk(scores[b, g], n, k)
    return out


def decode_token_scores(q: np.ndarray, k_cache: np.ndarray, seqlens=None) -> np.ndarray:
    """score[b,g,i] = sum_{h in g} P^h_i of the new token (at L_b - 1) over the cached tokens
    i < L_b (0 past the sequence end).  q [B,Hq,D]; k_cache [B,Hkv,L,D] -> [B,Hkv,L]."""
    B, Hq, D = q.shape
    Hkv, L = k_cache.shape[1], k_cache.shape[2]
    G = Hq // Hkv
    sc = np.zeros((B, Hkv, L))
    for b in range(B):
        Lb = L if seqlens is None else int(seqlens[b])
        for g in range(Hkv):
            kk = np.asarray(k_cache[b, g, :Lb], np.float64)
            for h in range(g * G, (g + 1) * G):
                p, _, _ = causal_softmax(np.asarray(q[b, h], np.float64)[None, :], np.array([Lb - 1]), kk)
                sc[b, g, :Lb] += p[0]
    return sc


def topk_decode_tokens(scores: np.ndarray, k_tokens: int, forced: int, seqlens=None) -> np.ndarray:
    """[B,Hkv,L] -> [B,Hkv,k_tokens]: the top k of the candidates [0, L_b - 1 - forced]
    (the tokens older than the forced newest window), ties to the lower index, ascending,
    padded with -1."""
    B, Hkv, L = scores.shape
    out = np.full((B, Hkv, k_tokens), -1, dtype=np.int64)
    for b in range(B):
        Lb = L if seqlens is None else int(seqlens[b])
        n = max(0, Lb - forced)
        for g in range(Hkv):
            out[b, g] = select_topk(scores[b, g], n, k_tokens)
    return out


def decode_token_sparse(q: np.ndarray, k_cache, v_cache, idx, forced: int, seqlens=None) -> np.ndarray:
    """Token-sparse layer for the new token: the selected cached tokens idx[b,g,:] united
    with the forced newest window [L_b - forced, L_b - 1], each token once; no gate."""
    B, Hq, D = q.shape
    Hkv, L = k_cache.shape[1], k_cache.shape[2]
    G = Hq // Hkv
    o = np.zeros((B, Hq, D))
    for b in range(B):
        Lb = L if seqlens is None else int(seqlens[b])
        for g in range(Hkv):
            keep = np.zeros(Lb, dtype=bool)
            sel = np.asarray([i for i in idx[b, g] if 0 <= i < Lb], dtype=np.int64)
            keep[sel] = True
            keep[max(0, Lb - forced):] = True
            keys = np.nonzero(keep)[0]
            ks = np.asarray(k_cache[b, g, keys], np.float64)
            vs = np.asarray(v_cache[b, g, keys], np.float64)
            for h in range(g * G, (g + 1) * G):
                qq = np.asarray(q[b, h], np.float64)[None, :]
                o[b, h] = attention_rows(qq, np.array([len(keys)]), ks, vs)[0][0]
    return o


def e4m3_to_float(codes) -> np.ndarray:
    """OCP 8-bit floating point, E4M3 ("fn": no infinities), code -> float64 value: sign bit 7,
    exponent bits 6..3 with bias 7, mantissa bits 2..0; exponent 0 is subnormal (m/8 * 2^-6),
    exponent 15 with mantissa 7 is NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2((e - 7).astype(np.float64)))
    mag = np.where((e == 15) & ((c & 0x7) == 7), np.nan, mag)
    return sign * mag


def dequant_kv_fp8(codes, scale) -> np.ndarray:
    """FP8 cache [B,Hkv,L,D] of E4M3 codes with one float32 scale per KV head [Hkv] -> the
    float64 cache values code * scale[g] the decode step attends over."""
    v = e4m3_to_float(codes)
    sc = np.asarray(scale, np.float64).reshape(1, -1, 1, 1)
    return v * sc


def decode_sparse(q: np.ndarray, k_cache, v_cache, idx, k_ring, v_ring, gate, seqlens=None,
                  swa_len=None, block: int = 64, sinks=None):
    """One sparse layer for the new token: selected blocks of the shared cache (all keys
    of a selected block that hold cached tokens) plus the layer's own SWA ring of
    swa_len[b] tokens (ring order does not matter: softmax is permutation invariant),
    merged by the sigmoid gate [B,Hq,2].  A branch with no keys (an empty ring, or no
    selected block holding cached tokens) contributes zero; sinks None or [Hq,2] as in
    gated_sparse_rows."""
    B, Hq, D = q.shape
    Hkv, L = k_cache.shape[1], k_cache.shape[2]
    G = Hq // Hkv
    o = np.zeros((B, Hq, D))
    for b in range(B):
        Lb = L if seqlens is None else int(seqlens[b])
        nring = k_ring.shape[2] if swa_len is None else int(swa_len[b])
        for g in range(Hkv):
            keys = np.concatenate([np.arange(j * block, min(Lb, (j + 1) * block))
                                   for j in idx[b, g] if j >= 0] or [np.zeros(0, np.int64)])
            ks = np.asarray(k_cache[b, g, keys], np.float64)
            vs = np.asarray(v_cache[b, g, keys], np.float64)
            kr = np.asarray(k_ring[b, g, :nring], np.float64)
            vr = np.asarray(v_ring[b, g, :nring], np.float64)
            for h in range(g * G, (g + 1) * G):
                qq = np.asarray(q[b, h], np.float64)[None, :]
                s0, s1 = (None, None) if sinks is None else (float(sinks[h][0]), float(sinks[h][1]))
                o_sp = attention_rows(qq, np.array([len(keys)]), ks, vs, None, s0)[0] if len(keys) else np.zeros((1, D))
                o_sw = attention_rows(qq, np.array([nring]), kr, vr, None, s1)[0] if nring else np.zeros((1, D))
                gg = sigmoid(gate[b, h])
                o[b, h] = gg[0] * o_sp[0] + gg[1] * o_sw[0]
    return o
