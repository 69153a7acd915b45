"""Helpers of the GPU parity tests: device tensors from the seeded generator, the
hybrid-block path through the C ABI, and the two acceptance rules.

Rule 1: where the oracle's k-th and (k+1)-th scores of a tile differ by more than
1e-3 relative, the GPU's selected set equals the oracle's.  Rule 2: elsewhere it
equals the oracle's selection routine applied to the GPU's own emitted scores.
Outputs are then compared with the oracle run on the GPU's indices: max-abs error
<= 1e-4 for fp32 inputs and <= 2e-2 for bf16 inputs (fp32 accumulation)."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from attention_tcgen05_tma_b200 import hysparse as H

TOL = {"f32": 1e-4, "bf16": 2e-2}
GAP = 1e-3


def to_dev(x: np.ndarray, dtype: str, device="cuda"):
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)   # exact: the generator already rounded to bf16
    return t.to(device)


def device_fill(shape, fn, keys, bf16: bool = True, device="cuda"):
    """A device tensor filled slice by slice from the seeded generator (slices drawn by a
    thread pool), the way the benchmark builds its full-size inputs."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    out = torch.empty(shape, dtype=torch.bfloat16 if bf16 else torch.float32, device=device)
    with ThreadPoolExecutor(min(32, os.cpu_count() or 8)) as ex:
        for key, arr in ex.map(lambda key: (key, fn(*key)), keys):
            t = torch.from_numpy(np.ascontiguousarray(arr))
            out[key].copy_(t.to(torch.bfloat16) if bf16 else t)
    return out


def to_np(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_selection(oracle_scores: np.ndarray, gpu_scores: np.ndarray, gpu_idx: np.ndarray, n_cand: int, k: int):
    """Apply rules 1/2 to one tile (raises on a violation) and return what decided it:

    * ``rule``: 'rule1' (the oracle's k-th and (k+1)-th scores differ by more than the gap, or
      there are at most k candidates: the GPU set equals the oracle's) or 'rule2' (near tie: the
      GPU set equals the oracle's selection routine on the GPU's own scores);
    * ``decided_in`` / ``decided_out``: candidates whose oracle score clears the k-th/(k+1)-th
      boundary by more than the gap plus twice the GPU's largest score error on this tile, which
      no correct selection on the GPU's scores can move: each must be selected / left out, on
      rule-2 tiles too (a planted block far above the boundary is always decided in)."""
    s = oracle_scores[:n_cand]
    order = np.lexsort((np.arange(n_cand), -s))
    want_oracle = O.select_topk(oracle_scores, n_cand, k)
    if n_cand <= k:
        assert np.array_equal(gpu_idx, want_oracle), (gpu_idx, want_oracle)
        return {"rule": "rule1", "decided_in": list(range(n_cand)), "decided_out": []}
    sk, sk1 = s[order[k - 1]], s[order[k]]
    if sk > 0 and (sk - sk1) / sk > GAP:
        assert np.array_equal(gpu_idx, want_oracle), (gpu_idx, want_oracle)
        rule = "rule1"
    else:
        want_gpu = O.select_topk(gpu_scores.astype(np.float64), n_cand, k)
        assert np.array_equal(gpu_idx, want_gpu), (gpu_idx, want_gpu)
        rule = "rule2"
    g = gpu_scores[:n_cand].astype(np.float64)
    pos = s > 0
    err = float(np.max(np.abs(g[pos] - s[pos]) / s[pos])) if pos.any() else 0.0
    margin = GAP + 3.0 * err
    chosen = set(int(j) for j in gpu_idx if j >= 0)
    d_in = [int(j) for j in range(n_cand) if s[j] > sk1 * (1.0 + margin)]
    d_out = [int(j) for j in range(n_cand) if s[j] < sk * (1.0 - margin)]
    assert all(j in chosen for j in d_in), ("decided-in block not selected", d_in, sorted(chosen))
    assert not any(j in chosen for j in d_out), ("decided-out block selected", sorted(chosen))
    return {"rule": rule, "decided_in": d_in, "decided_out": d_out}


def score_rel_err(oracle_scores: np.ndarray, gpu_scores: np.ndarray, floor: float = 1e-6) -> float:
    mask = np.abs(oracle_scores) > floor
    if not mask.any():
        return 0.0
    return float(np.max(np.abs(gpu_scores[mask] - oracle_scores[mask]) / np.abs(oracle_scores[mask])))


# Gradients: the largest error relative to the gradient's largest element.  bf16 inputs: 2e-2 (the
# bound set for bf16 attention outputs; P and dS are rounded to bf16 before the contractions and dq is
# stored in bf16, each a relative 2^-9 per term); fp32 inputs (fp32 kernels throughout): 1e-4.
# dq of bf16 inputs: 5e-2.  The backward forms D_t = dO_t . o_t from the forward's stored bf16 output
# o; its rounding (2^-9 relative per element) shifts D_t by dD_t and dq_t by tau dD_t sum_i P_ti k_i,
# which the planted keys (norm 3 sqrt(D), far above the others) carry to 2.5% of max|dq| with every
# other step exact (a float64 emulation of just that step on the 2 x 300 ragged case).
GRAD_TOL = {"f32": 1e-4, "bf16": 2e-2}
DQ_TOL = {"f32": 1e-4, "bf16": 5e-2}


def grad_err(gpu: np.ndarray, ref: np.ndarray) -> float:
    scale = float(np.max(np.abs(ref)))
    if scale == 0.0:
        return float(np.max(np.abs(gpu)))
    return float(np.max(np.abs(np.asarray(gpu, np.float64) - ref))) / scale
