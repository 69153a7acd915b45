"""Scalar pure-Python transcription of the hybrid-block path, for tiny inputs only.

It is written independently of the vectorised oracle: plain loops over rows,
keys and blocks, math.exp, explicit key lists built by concatenating the
selected blocks (the gather of HySparse §3.4.3) and a full sort for TopK.  It
pins the oracle on N <= 256.
"""
import math


def _dot(a, b):
    s = 0.0
    for x, y in zip(a, b):
        s += float(x) * float(y)
    return s


def softmax_over(q, keys, kmat):
    """Probabilities of query q over the listed key positions (list of (pos, prob))."""
    tau = 1.0 / math.sqrt(len(q))
    logits = [tau * _dot(q, kmat[i]) for i in keys]
    m = max(logits)
    ex = [math.exp(s - m) for s in logits]
    z = sum(ex)
    return [(i, e / z) for i, e in zip(keys, ex)]


def attend(q, keys, kmat, vmat):
    probs = softmax_over(q, keys, kmat)
    d = len(vmat[0])
    out = [0.0] * d
    for i, p in probs:
        row = vmat[i]
        for c in range(d):
            out[c] += p * float(row[c])
    return out


def _row_probs(q_head, t, kmat, memo, h):
    """Probabilities of row t over keys 0..t; memo (a dict or None) keeps them per (head, row)."""
    if memo is not None and (h, t) in memo:
        return memo[(h, t)]
    probs = dict(softmax_over(q_head[t], list(range(t + 1)), kmat))
    if memo is not None:
        memo[(h, t)] = probs
    return probs


def block_score(qs_group, kmat, tile, j, n, block, reduce="sum", memo=None):
    """R_h R_{t in tile} max_{i in block j, i <= t} P_{t,i}."""
    vals = []
    for h, q_head in enumerate(qs_group):
        for t in range(tile * block, min(n, (tile + 1) * block)):
            probs = _row_probs(q_head, t, kmat, memo, h)
            in_block = [probs[i] for i in range(j * block, min(n, (j + 1) * block)) if i <= t]
            vals.append(max(in_block) if in_block else 0.0)
    return sum(vals) if reduce == "sum" else max(vals)


def topk(scores, n_candidates, k):
    ranked = sorted(range(n_candidates), key=lambda j: (-scores[j], j))
    chosen = sorted(ranked[:k])
    return chosen + [-1] * (k - len(chosen))


def sparse_row(q, t, kmat, vmat, sel_blocks, block):
    keys = []
    for j in sel_blocks:            # concatenation of the selected blocks
        if j < 0:
            continue
        for i in range(j * block, (j + 1) * block):
            if i <= t and i < len(kmat):
                keys.append(i)
    return attend(q, keys, kmat, vmat)


def swa_row(q, t, kmat, vmat, window):
    return attend(q, list(range(max(0, t - window + 1), t + 1)), kmat, vmat)


def gated_row(q, t, k, v, sel, ks, vs, window, gate, block):
    a = sparse_row(q, t, k, v, sel, block)
    b = swa_row(q, t, ks, vs, window)
    g0 = 1.0 / (1.0 + math.exp(-gate[0]))
    g1 = 1.0 / (1.0 + math.exp(-gate[1]))
    return [g0 * x + g1 * y for x, y in zip(a, b)]


def token_score(qs_group, kmat, tile, i, n, block, memo=None):
    s = 0.0
    for h, q_head in enumerate(qs_group):
        for t in range(max(i, tile * block), min(n, (tile + 1) * block)):
            probs = _row_probs(q_head, t, kmat, memo, h)
            s += probs[i]
    return s


def token_row(q, t, kmat, vmat, sel_tokens, forced):
    keys = set(i for i in sel_tokens if 0 <= i <= t)     # causal: never past the row
    keys |= set(range(max(0, t - forced + 1), t + 1))
    return attend(q, sorted(keys), kmat, vmat)
