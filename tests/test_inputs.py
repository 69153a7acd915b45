"""Host-side checks of the seeded input generator (no GPU)."""
import math

import numpy as np
import torch

from attention_tcgen05_tma_b200 import inputs as I


def test_round_bf16_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.array([1.00390625, 1.01171875, -2.5e-39, 3e38], np.float32)])
    ours = I.round_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


def test_slices_are_reproducible_and_independent():
    w = I.scaled(I.WORKLOADS["dense7b"], N=256, Hq=4, Hkv=2, layers=1)
    a = I.q_slice(w, 0, 1)
    b = I.q_slice(w, 0, 1)
    c = I.q_slice(w, 0, 2)
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    full = I.prefill_arrays(w, threads=4)
    assert np.array_equal(full["q"][0, 1], a)
    assert np.array_equal(full["k"][0, 1], I.k_slice(w, 0, 1))
    assert full["gate"][0].shape == (1, 4, 256, 2)


def test_block_plants_raise_the_target_logit():
    w = I.scaled(I.WORKLOADS["dense7b"], N=1024, Hq=8, Hkv=2, n_plants=6, layers=0)
    pl = I.plants(w)
    assert len(pl) == 6 and len({(p.b, p.g, p.pos) for p in pl}) == 6
    for p in pl:
        assert p.pos // 64 < w.NB - 1 and p.t >= p.pos + 64
        q = I.q_slice(w, p.b, p.h)[p.t].astype(np.float64)
        k = I.k_slice(w, p.b, p.g)[p.pos:p.pos + 64].astype(np.float64)
        logits = k @ q / math.sqrt(w.D)
        assert logits.min() > 2.0, logits.min()


def test_position_plants_tiny():
    w = I.WORKLOADS["tiny"]
    pl = I.plants(w)
    assert len(pl) == 8 and all(p.length == 1 and p.t > p.pos for p in pl)
    for p in pl:
        q = I.q_slice(w, 0, p.h)[p.t].astype(np.float64)
        k = I.k_slice(w, 0, p.g)[p.pos].astype(np.float64)
        assert abs(k @ q / 8.0 - 3.0 * np.linalg.norm(q) / 8.0) < 1e-5


def test_sampled_tiles_include_last():
    for name in ("moe80b", "token"):
        w = I.WORKLOADS[name]
        t = I.sampled_tiles(w, 8)
        assert (0, 0, w.T - 1) in t and len(t) == 8
