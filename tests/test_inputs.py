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


def test_fp8_cache_codes():
    """The FP8 decode cache: per-KV-head scales in the stated range, no NaN codes, and every code
    within E4M3's rounding of the seeded value / scale (half a unit in the last place: 2^-4
    relative for normal codes, 2^-10 absolute below the smallest normal 2^-6)."""
    import oracle as O
    w = I.scaled(I.WORKLOADS["decode"], B=2, N=300, layers=1)
    c = I.decode_fp8_cache(w)
    base = w.scale_std / 32.0
    for sc in (c["k_scale"], c["v_scale"]):
        assert sc.dtype == np.float32 and sc.shape == (w.Hkv,)
        assert np.all(sc >= 0.75 * base * (1 - 1e-6)) and np.all(sc <= 1.25 * base * (1 + 1e-6))
    for name, sc in (("k8", c["k_scale"]), ("v8", c["v_scale"])):
        codes = c[name]
        assert codes.dtype == np.uint8 and codes.shape == (w.B, w.Hkv, w.N, w.D)
        assert not np.any((codes & 0x7F) == 0x7F)             # no NaN codes
        vals = O.e4m3_to_float(codes)
        for b in range(w.B):
            for g in range(w.Hkv):
                x = I.normal_slice(w.seed, I.TID_K if name == "k8" else I.TID_V, b, g, (w.N, w.D), w.scale_std,
                                   False).astype(np.float64) / np.float64(np.float32(sc[g]))
                err = np.abs(vals[b, g] - x)
                bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10)
                assert np.all(err <= bound * (1 + 1e-6))
