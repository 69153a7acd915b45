"""Host-side pieces of bench.py that need no GPU: the recorded DRAM traffic of the dominant
kernel is only reported while the kernel's sources are the ones it was captured from, and it
scales with the work units."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_record_matches_current_sources():
    rec = bench.NCU_TRAFFIC["sparse_attn"]
    t = bench.ncu_traffic("sparse_attn", rec["units"])
    # a kernel source changed since the capture: re-capture the DRAM bytes and update the record
    assert t is not None, "sparse_attn_tc DRAM traffic is stale: re-run the ncu capture"
    assert t == rec["bytes"]
    assert bench.ncu_traffic("sparse_attn", 4 * rec["units"]) == 4 * rec["bytes"]


def test_traffic_is_null_for_unknown_kernels():
    assert bench.ncu_traffic("no_such_kernel", 1) is None


def test_reference_arm_json_contract():
    """`bench.py --impl reference` (the float64 oracle on the host cores) prints one JSON line with
    the contract's keys, its own cpu_baseline and an e2e block without host-device traffic."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [x for x in r.stdout.splitlines() if x.startswith("{")][-1]
    d = json.loads(line)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1 and d["warmup"] == 3
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    # the same config object as our arm prints, and a step time that is the sample's own
    from attention_tcgen05_tma_b200 import inputs as I
    assert d["config"] == bench.workload_config(I.WORKLOADS["tiny"], 1)
    assert d["ms_per_step"] > 0 and "extrapolated" in d["ms_per_step_kind"]


def test_cpu_baseline_is_unbiased_over_tile_position():
    """The baseline's estimate is mean time per sampled tile x all tiles, with tiles stratified
    over the tile index: two samples of different sizes give the same order of magnitude."""
    from attention_tcgen05_tma_b200 import inputs as I
    w = I.WORKLOADS["tiny"]
    a = bench.cpu_baseline(w, budget_s=0.0, n_tiles=4, seed=1)
    b = bench.cpu_baseline(w, budget_s=60.0, n_tiles=16, seed=2)
    assert a["tiles"] == 1 and b["tiles"] == 16
    assert 0.2 < a["value"] / b["value"] < 5.0


def _brute_attended(idx, N, W, block):
    """Per (b, g, row): |Sel_I ∪ [max(0, t-W+1), t]| by explicit sets."""
    B, Hkv, T, _ = idx.shape
    n = 0
    for b in range(B):
        for g in range(Hkv):
            for t in range(N):
                sel = {int(i) for i in idx[b, g, t // block] if i >= 0}
                n += len(sel | set(range(max(0, t - W + 1), t + 1)))
    return n


def test_token_sparse_flops_count_each_attended_key_once():
    """The token-sparse layer's algorithmic flops: 4*D per (row, head, key of the union of the
    tile's selected tokens and the row's newest W), checked against explicit sets on a small
    ragged case whose selections reach up to the window."""
    import numpy as np
    rng = np.random.default_rng(5)
    B, Hkv, G, D, N, W, block, kt = 1, 2, 3, 16, 333, 128, 64, 24
    T = (N + block - 1) // block
    idx = np.full((B, Hkv, T, kt), -1, dtype=np.int32)
    for b in range(B):
        for g in range(Hkv):
            for I in range(T):
                e_I = min(64 * I + 63, N - 1)
                cand = np.arange(0, e_I - W + 1)
                if cand.size == 0:
                    continue
                pick = np.sort(rng.choice(cand, size=min(kt, cand.size), replace=False))
                pick[-1] = cand[-1]   # the last candidate sits inside every row's window but the tile's last
                idx[b, g, I, :pick.size] = pick
    want = 4.0 * D * G * _brute_attended(idx, N, W, block)
    assert bench.token_sparse_flops(idx, N, G, D, W, block) == want


def test_block_sparse_flops_count_visible_keys_of_both_branches():
    """The block-sparse layer's algorithmic flops: 4*D per (row, head) for each causally visible
    key of the selected blocks plus each key of the row's window branch, against explicit counts
    on a small ragged case."""
    import numpy as np
    rng = np.random.default_rng(7)
    B, Hkv, G, D, N, W, block, kb = 2, 1, 2, 8, 300, 100, 64, 3
    T = (N + block - 1) // block
    idx = np.full((B, Hkv, T, kb), -1, dtype=np.int32)
    for b in range(B):
        for I in range(T):
            pick = np.sort(rng.choice(I + 1, size=min(kb, I + 1), replace=False))
            idx[b, 0, I, :pick.size] = pick
    n = 0
    for b in range(B):
        for t in range(N):
            for j in idx[b, 0, t // block]:
                if j >= 0:
                    n += len([i for i in range(64 * j, 64 * j + 64) if i <= t])
            n += len(range(max(0, t - W + 1), t + 1))
    assert bench.sparse_flops(idx, N, G, D, W, block) == 4.0 * D * G * n
