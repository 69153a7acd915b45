"""Benchmark of the HySparse hybrid-block hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one hybrid block of the MoE-shaped prefill workload (B=2, N=32768, 32 query
heads / 4 KV heads, D=128, bf16): the full-attention layer with fused block scores,
the top-k block selector (k=32) and 11 sparse layers (block-sparse + SWA(128) + gate),
each with its own Q', K', V' and gate logits.  ``value`` is prefill tokens/s over the
whole job.  The decode workload (64 sequences x 131072 cached tokens, 1 full + 11
sparse layers) is timed in the same run and reported as ``decode`` (us/token).

Further legs, each outside the headline's timed region and reported under its own key:
``rows`` (per-position selection on the prefill inputs, one layer), ``dense7b`` (the 7B-dense-shaped
1:3 block: B1 N8192, 32/8 heads, top-16 blocks, 3 sparse layers), ``backward`` (the training
backward of the full layer and of one sparse layer on the headline inputs), ``decode_tokens`` (the
token-variant decode step over the decode cache, bf16 and FP8 E4M3, us/token), ``token`` (the
token-variant prefill, N=131072), ``e2e`` (the headline through the C ABI with host buffers
copied in and out every step) and ``cpu_baseline`` (the float64 oracle on a bounded sample).
Flags ``--no-rows``, ``--no-dense7b``, ``--no-backward``, ``--no-decode``, ``--no-decode-tokens``, ``--no-token``,
``--no-e2e`` and ``--no-cpu`` skip them.

Multi-GPU (torchrun): every rank runs its own independent batch (weak scaling, no
data-path collective); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from attention_tcgen05_tma_b200.distributed import max_over_ranks  # noqa: E402

# DRAM traffic of the dominant prefill kernel from one ncu capture (profiles/
# sparse_attn_tc_moe80b_small.md): dram__bytes_read.sum + dram__bytes_write.sum of one launch on
# the moe80b_small workload, the work units (batch, KV group, 64-query tile) that launch
# processed, and a digest of the kernel's sources at capture time.  Every term of the traffic
# (Q', O, gate, K'/V', the gathered blocks) grows with the units, so the bench scales the bytes
# to its own units; it reports null once the sources differ from the captured ones.
NCU_TRAFFIC = {
    "sparse_attn": {"bytes": 199150848 + 103134208, "units": 1024,
                    "sources": ("sparse_attn_tc.cu", "tc_ptx.cuh", "common.cuh"),
                    "sha256": "3c6fb1605ffd7117f5f3d405b1cda39f09ee089aefa9957ea2ac071a4a6fbbad"},
}


def ncu_traffic(kernel, units):
    """Bytes per launch from the recorded capture scaled to `units`, or None when the kernel's
    sources changed since the counters were taken."""
    rec = NCU_TRAFFIC.get(kernel)
    if rec is None:
        return None
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "attention_tcgen05_tma_b200", "csrc")
    h = hashlib.sha256()
    try:
        for f in rec["sources"]:
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(fh.read())
    except OSError:
        return None
    if h.hexdigest() != rec["sha256"]:
        return None
    return round(rec["bytes"] * units / rec["units"])


METRIC = "hybrid-block prefill tokens/s @32K and decode µs/token; % of tensor/HBM roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def workload_config(w, world):
    """The `config` object of the JSON line; both arms print the same one."""
    return {"workload": f"{w.name}: B={w.B} N={w.N} Hq={w.Hq} Hkv={w.Hkv} D={w.D} 1 full + {w.layers} "
                        f"sparse layers, top-{w.topk} blocks, SWA {w.window}",
            "global_batch": w.B * world, "seq_len": w.N, "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (Q 512 MiB per layer)" if w.N * w.B >= 32768 else
                  "step inputs larger than L2"}


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def wait_ready(self, timeout_s: float = 3.0):
        """Block until the sampler has printed its first line, so that it runs for the whole
        timed region; the samples taken before the region are dropped."""
        t_end = time.time() + timeout_s
        while self.proc is not None and not self.lines and time.time() < t_end:
            time.sleep(0.01)
        self.lines.clear()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- inputs
def _device_tensor(torch, dev, shape, fn, keys, bf16=True):
    """Allocate a device tensor and fill it slice by slice from the seeded generator
    (slices are drawn by a thread pool; each is copied into its place)."""
    from concurrent.futures import ThreadPoolExecutor
    out = torch.empty(shape, dtype=torch.bfloat16 if bf16 else torch.float32, device=dev)

    def one(key):
        return key, fn(*key)

    with ThreadPoolExecutor(min(32, os.cpu_count() or 8)) as ex:
        for key, arr in ex.map(one, keys):
            t = torch.from_numpy(arr)
            out[key].copy_(t.to(torch.bfloat16) if bf16 else t)
    return out


def make_prefill_inputs(w, torch, dev, layers, seed_offset=0):
    from attention_tcgen05_tma_b200 import inputs as I
    if seed_offset:
        w = I.scaled(w, seed=w.seed + seed_offset)
    t0 = time.time()
    bq = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    bk = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    qs, kvs, gs = (w.B, w.Hq, w.N, w.D), (w.B, w.Hkv, w.N, w.D), (w.B, w.Hq, w.N, 2)
    pl = I.plants(w)
    d = {"q": _device_tensor(torch, dev, qs, lambda b, h: I.q_slice(w, b, h), bq),
         "k": _device_tensor(torch, dev, kvs, lambda b, g: I.k_slice(w, b, g, pl), bk),
         "v": _device_tensor(torch, dev, kvs, lambda b, g: I.v_slice(w, b, g), bk),
         "q_sparse": [], "k_swa": [], "v_swa": [], "gate": []}
    for l in range(layers):
        d["q_sparse"].append(_device_tensor(torch, dev, qs, lambda b, h: I.sparse_q_slice(w, l, b, h), bq))
        d["k_swa"].append(_device_tensor(torch, dev, kvs, lambda b, g: I.swa_k_slice(w, l, b, g), bk))
        d["v_swa"].append(_device_tensor(torch, dev, kvs, lambda b, g: I.swa_v_slice(w, l, b, g), bk))
        d["gate"].append(_device_tensor(torch, dev, gs, lambda b, h: I.gate_slice(w, l, b, h), bq, bf16=False))
    log(f"prefill inputs ready in {time.time() - t0:.1f}s")
    return d


def make_decode_inputs(w, torch, dev, layers, seed_offset=0):
    from attention_tcgen05_tma_b200 import inputs as I
    if seed_offset:
        w = I.scaled(w, seed=w.seed + seed_offset)
    t0 = time.time()
    bq = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    bk = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    d = {"q": _device_tensor(torch, dev, (w.B, w.Hq, w.D), lambda b, h: I.decode_q_slice(w, b, h), bq),
         "k": _device_tensor(torch, dev, (w.B, w.Hkv, w.N, w.D), lambda b, g: I.decode_k_slice(w, b, g), bk),
         "v": _device_tensor(torch, dev, (w.B, w.Hkv, w.N, w.D), lambda b, g: I.decode_v_slice(w, b, g), bk),
         "q_sparse": [], "k_swa": [], "v_swa": [], "gate": []}
    for l in range(layers):
        d["q_sparse"].append(_device_tensor(torch, dev, (w.B, w.Hq, w.D),
                                            lambda b, h: I.decode_sparse_q_slice(w, l, b, h), bq))
        d["k_swa"].append(_device_tensor(torch, dev, (w.B, w.Hkv, w.window, w.D),
                                         lambda b, g: I.swa_k_slice(w, l, b, g), bk))
        d["v_swa"].append(_device_tensor(torch, dev, (w.B, w.Hkv, w.window, w.D),
                                         lambda b, g: I.swa_v_slice(w, l, b, g), bk))
        d["gate"].append(_device_tensor(torch, dev, (w.B, w.Hq, 2), lambda b, h: I.gate_slice(w, l, b, h), bq,
                                        bf16=False))
    log(f"decode inputs ready in {time.time() - t0:.1f}s")
    return d


# ----------------------------------------------------------------------------- our arm
class PrefillStep:
    """One hybrid block through the C ABI with preallocated outputs/workspace."""

    def __init__(self, w, x, torch, dev):
        from attention_tcgen05_tma_b200 import hysparse as H
        self.H, self.w, self.x, self.torch = H, w, x, torch
        T = w.T
        self.o_full = torch.empty_like(x["q"])
        self.scores = torch.empty((w.B, w.Hkv, T, w.NB), dtype=torch.float32, device=dev)
        self.idx = torch.empty((w.B, w.Hkv, T, w.topk), dtype=torch.int32, device=dev)
        # every layer's output in its own buffer (the block's result is all twelve layers' outputs)
        self.o_sp = [torch.empty_like(x["q"]) for _ in range(w.layers)]
        sh = H.prefill_shape(x["q"], x["k"])
        nws = H.hysparse_full_attn_select_workspace_size(sh, H.HYS_BF16, H.HYS_GRAN_BLOCK)
        self.ws = H.workspace_for(nws, dev)
        self.ws_sp = H.workspace_for(H.hysparse_sparse_attn_workspace_size(sh, H.HYS_BF16), dev)
        self.events = None

    def run(self, timing=None):
        H, x, w = self.H, self.x, self.w
        ev = timing
        if ev is not None:
            ev["full"][0].record()
        H.full_attn_select(x["q"], x["k"], x["v"], o=self.o_full, scores=self.scores, workspace=self.ws)
        if ev is not None:
            ev["full"][1].record()
        H.topk(self.scores, w.topk, idx=self.idx)
        if ev is not None:
            ev["topk"][1].record()
        for l in range(w.layers):
            H.sparse_attn(x["q_sparse"][l], x["k"], x["v"], self.idx, x["k_swa"][l], x["v_swa"][l], w.window,
                          x["gate"][l], o=self.o_sp[l], workspace=self.ws_sp)
        if ev is not None:
            ev["sparse"][1].record()


def sparse_flops(idx_np, N, G, D, window, block=64):
    """Algorithmic flops of one sparse layer: 4*D per (row, head, attended key)."""
    B, Hkv, T, k = idx_np.shape
    total = 0
    for I_ in range(T):
        rows = np.arange(I_ * block, min(N, (I_ + 1) * block))
        sel = idx_np[:, :, I_, :]
        full_blocks = ((sel >= 0) & (sel < I_)).sum(axis=-1)          # fully visible blocks
        diag = (sel == I_).sum(axis=-1)                                 # causal diagonal block
        vis_sparse = full_blocks[..., None] * block + diag[..., None] * (rows - I_ * block + 1)[None, None, :]
        vis_win = np.minimum(rows + 1, window)
        total += int(vis_sparse.sum()) * G + int(vis_win.sum()) * B * Hkv * G
    return 4.0 * D * total


def time_call(torch, fn, n=5, warm=2):
    """Mean device time of fn() over n calls (CUDA events on the current stream, after warm-up)."""
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / n


def run_ours(args, torch, dist, rank, world, dev):
    from attention_tcgen05_tma_b200 import build as Bld
    from attention_tcgen05_tma_b200 import hysparse as H
    from attention_tcgen05_tma_b200 import inputs as I
    if rank == 0:
        Bld.build()
    if dist is not None:
        dist.barrier()
    H.load()
    peaks, peak_src = load_peaks()
    w = I.WORKLOADS[args.workload]
    x = make_prefill_inputs(w, torch, dev, w.layers, seed_offset=1000 * rank)
    step = PrefillStep(w, x, torch, dev)
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    idx_np = step.idx.cpu().numpy()
    sp_flops = sparse_flops(idx_np, w.N, w.G, w.D, w.window)
    full_flops = 4.0 * w.D * w.Hq * w.B * w.N * (w.N + 1) / 2

    # timed region: K steps, per-kernel events on the launching stream
    stream = torch.cuda.current_stream()
    evs = [{k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for k in ("full", "topk", "sparse")} for _ in range(args.steps)]
    for e in evs:
        e["topk"] = (e["full"][1], e["topk"][1])
        e["sparse"] = (e["topk"][1], e["sparse"][1])
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    clocks.wait_ready()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step.run(evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms_total = t0.elapsed_time(t1)
    per = {k: sum(e[k][0].elapsed_time(e[k][1]) for e in evs) / args.steps for k in ("full", "topk", "sparse")}
    ms_step = max_over_ranks(ms_total / args.steps, dist, dev)
    tokens_job = w.B * w.N * world
    value = tokens_job / (ms_step / 1e3)

    # roofline of the dominant kernel
    full_ms = per["full"]
    sparse_ms_layer = per["sparse"] / w.layers
    peak_tf = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    full_tf = full_flops / (full_ms / 1e3) / 1e12
    sp_tf = sp_flops / (sparse_ms_layer / 1e3) / 1e12
    dominant = "full_attn_select" if full_ms >= per["sparse"] else "sparse_attn"
    if dominant == "full_attn_select":
        roof = {"kernel": "full_attn_select", "bound": "tensor", "achieved": round(full_tf, 2), "peak": peak_tf,
                "unit": "TFLOP/s", "frac": round(full_tf / peak_tf, 4), "traffic": None}
    else:
        roof = {"kernel": "sparse_attn", "bound": "tensor", "achieved": round(sp_tf, 2), "peak": peak_tf,
                "unit": "TFLOP/s", "frac": round(sp_tf / peak_tf, 4),
                "traffic": ncu_traffic("sparse_attn", w.B * w.Hkv * w.T)}
        if roof["traffic"] is not None:
            roof["traffic_source"] = "ncu dram bytes of one moe80b_small launch, scaled by work units"
    roof["peak_source"] = f"{peak_src} bf16_tflops_sustained"
    kernels = {
        "full_attn_select_ms": round(full_ms, 4), "full_attn_select_tflops": round(full_tf, 2),
        "full_attn_select_frac": round(full_tf / peak_tf, 4),
        "topk_ms": round(per["topk"], 4),
        "sparse_attn_ms_per_layer": round(sparse_ms_layer, 4), "sparse_attn_tflops": round(sp_tf, 2),
        "sparse_attn_frac": round(sp_tf / peak_tf, 4),
        "full_flops": full_flops, "sparse_flops_per_layer": sp_flops,
    }
    launches_full = 1 if step.ws.numel() <= 1 or _uses_tc(H, w) else 2
    launches = args.steps * (launches_full + 1 + w.layers)
    # the same sparse layer with per-head sink logits of both branches (outside the timed step)
    sinks = torch.from_numpy(I.sink_logits(w, 0)).to(dev)
    ms_sinks = time_call(torch, lambda: H.sparse_attn(x["q_sparse"][0], x["k"], x["v"], step.idx, x["k_swa"][0],
                                                      x["v_swa"][0], w.window, x["gate"][0], sinks=sinks,
                                                      o=step.o_sp[0], workspace=step.ws_sp))
    ms_plain = time_call(torch, lambda: H.sparse_attn(x["q_sparse"][0], x["k"], x["v"], step.idx, x["k_swa"][0],
                                                      x["v_swa"][0], w.window, x["gate"][0], o=step.o_sp[0],
                                                      workspace=step.ws_sp))
    kernels["sparse_attn_sinks_ms"] = round(ms_sinks, 4)
    kernels["sparse_attn_same_layer_no_sinks_ms"] = round(ms_plain, 4)   # same repeated-call timing
    kernels["sparse_attn_sinks_tflops"] = round(sp_flops / (ms_sinks / 1e3) / 1e12, 2)
    rows = None if args.no_rows else run_rows(torch, H, w, x, step, peak_tf)
    backward = None if args.no_backward else run_backward(torch, H, w, x, step, peak_tf)

    res = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1/128) Q/K/V with 64 planted blocks)",
           "config": workload_config(w, world),
           "kernels": kernels, "roofline": roof, "clocks": clk, "gpu_launches": launches}
    if rows is not None:
        res["rows"] = rows
    if backward is not None:
        res["backward"] = backward
    if not args.no_e2e:
        res["e2e"] = run_e2e(args, torch, dist, world, w, x, step, dev)
    del x, step
    torch.cuda.empty_cache()

    if not args.no_dense7b and args.workload != "dense7b":
        res["dense7b"] = run_dense7b(args, torch, dist, rank, world, dev, peaks, peak_src)
    if not args.no_decode:
        res["decode"] = run_decode(args, torch, dist, rank, world, dev, peaks, peak_src)
    if not args.no_decode_tokens:
        res["decode_tokens"] = run_decode_tokens(args, torch, dist, rank, world, dev, peaks, peak_src)
    if not args.no_token:
        res["token"] = run_token(args, torch, dist, rank, world, dev, peaks, peak_src)
    if rank == 0 and world == 1 and not args.no_cpu:
        res["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_budget)
    return res


def run_rows(torch, H, w, x, step, peak_tf):
    """Per-position selection ([HS] 3.4.2 per query position, group max) on the same inputs, one
    sparse layer, each call timed on its own: full layer with [B,Hkv,N,NB] scores, per-row top-k,
    and the sparse layer over each tile's union of its rows' blocks (every row masked to its own)."""
    o = torch.empty_like(x["q"])
    sc = torch.empty((w.B, w.Hkv, w.N, w.NB), dtype=torch.float32, device=x["q"].device)
    idx = torch.empty((w.B, w.Hkv, w.N, w.topk), dtype=torch.int32, device=x["q"].device)
    full = lambda: H.full_attn_select(x["q"], x["k"], x["v"], gran="block_row", reduce="max", o=o, scores=sc,
                                      workspace=step.ws)
    topk = lambda: H.topk_rows(sc, w.topk, idx=idx)
    sparse = lambda: H.sparse_attn_rows(x["q_sparse"][0], x["k"], x["v"], idx, x["k_swa"][0], x["v_swa"][0],
                                        w.window, x["gate"][0], o=step.o_sp[0], workspace=step.ws_sp)
    ms_full = time_call(torch, full, n=3, warm=1)
    ms_topk = time_call(torch, topk, n=3, warm=1)
    ms_sparse = time_call(torch, sparse, n=3, warm=1)
    # attended keys per row (selected blocks up to t, then the window) and the tiles' union sizes
    t = torch.arange(w.N, device=idx.device)
    jt = (t // 64).view(1, 1, w.N, 1)
    valid = (idx >= 0) & (idx <= jt)
    keys = torch.where(idx < jt, 64, (t % 64 + 1).view(1, 1, w.N, 1)) * valid
    attended = keys.sum(dim=3).double() + torch.clamp(t + 1, max=w.window).double().view(1, 1, w.N)
    alg_flops = 4.0 * w.D * (w.Hq // w.Hkv) * attended.sum().item()
    tiles = idx.view(w.B, w.Hkv, w.T, 64 * w.topk).sort(dim=3).values
    distinct = ((tiles[..., 1:] != tiles[..., :-1]) & (tiles[..., 1:] >= 0)).sum(dim=3) + (tiles[..., 0] >= 0).long()
    union = distinct.double().mean().item()
    res = {"config": f"{w.name}, one sparse layer, top-{w.topk} blocks per query position (group max)",
           "full_ms": round(ms_full, 4), "topk_ms": round(ms_topk, 4), "sparse_ms": round(ms_sparse, 4),
           "sparse_alg_tflops": round(alg_flops / (ms_sparse / 1e3) / 1e12, 2),
           "sparse_alg_frac": round(alg_flops / (ms_sparse / 1e3) / 1e12 / peak_tf, 4),
           "mean_union_blocks_per_tile": round(union, 1)}
    del o, sc, idx
    torch.cuda.empty_cache()
    return res


def run_backward(torch, H, w, x, step, peak_tf):
    """Training backward on the headline inputs, each call timed on its own: the full layer's
    gradients (dq, and fp32 dk, dv of the shared cache) and one sparse layer's (dq, its share of the
    shared dk, dv, dk', dv', gate gradients) after its training forward.  Algorithmic work: five
    contractions of 2*D flops per attended (row, head, key) = 10*D, i.e. 2.5x the forward's."""
    gen = torch.Generator(device=x["q"].device)
    gen.manual_seed(1234)
    d_o = (torch.randn(x["q"].shape, generator=gen, device=x["q"].device) / math.sqrt(w.D)).to(torch.bfloat16)
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=x["q"].device)
    o = torch.empty_like(x["q"])
    H.full_attn_select(x["q"], x["k"], x["v"], o=o, scores=step.scores, lse=lse, workspace=step.ws)
    H.topk(step.scores, w.topk, idx=step.idx)
    dq = torch.empty_like(x["q"])
    dk = torch.empty(x["k"].shape, dtype=torch.float32, device=x["q"].device)
    dv = torch.empty_like(dk)
    ws_f = H.workspace_for(H.hysparse_full_attn_backward_workspace_size(H.prefill_shape(x["q"], x["k"]), H.HYS_BF16),
                           x["q"].device)
    full = lambda: H.full_attn_backward(x["q"], x["k"], x["v"], o, d_o, lse, dq=dq, dk=dk, dv=dv, workspace=ws_f)
    ms_full = time_call(torch, full, n=3, warm=1)
    del ws_f
    lx = [x[key][0] for key in ("q_sparse", "k_swa", "v_swa", "gate")]
    o_l, osp, blse = H.sparse_attn_train(lx[0], x["k"], x["v"], step.idx, lx[1], lx[2], w.window, lx[3],
                                         workspace=step.ws_sp)
    dks = torch.empty(x["k"].shape, dtype=torch.float32, device=x["q"].device)
    dvs = torch.empty_like(dks)
    dgate = torch.empty((w.B, w.Hq, w.N, 2), dtype=torch.float32, device=x["q"].device)
    ws_s = H.workspace_for(H.hysparse_sparse_attn_backward_workspace_size(H.prefill_shape(x["q"], x["k"]),
                                                                         H.HYS_BF16), x["q"].device)
    sparse = lambda: H.sparse_attn_backward(lx[0], x["k"], x["v"], step.idx, lx[1], lx[2], w.window, lx[3], o_l, osp,
                                            blse, d_o, dk, dv, dq=dq, dk_swa=dks, dv_swa=dvs, dgate=dgate,
                                            workspace=ws_s)
    ms_sparse = time_call(torch, sparse, n=3, warm=1)
    full_flops = 2.5 * 4.0 * w.D * w.Hq * w.B * w.N * (w.N + 1) / 2
    sp_flops = 2.5 * sparse_flops(step.idx.cpu().numpy(), w.N, w.G, w.D, w.window)
    res = {"config": f"{w.name}: full layer and one sparse layer, bf16 inputs, fp32 K/V gradients",
           "full_bwd_ms": round(ms_full, 3), "full_bwd_tflops": round(full_flops / ms_full / 1e9, 1),
           "full_bwd_frac": round(full_flops / ms_full / 1e9 / peak_tf, 4),
           "sparse_bwd_ms": round(ms_sparse, 3), "sparse_bwd_tflops": round(sp_flops / ms_sparse / 1e9, 1),
           "sparse_bwd_frac": round(sp_flops / ms_sparse / 1e9 / peak_tf, 4),
           "full_bwd_flops": full_flops, "sparse_bwd_flops": sp_flops}
    del d_o, lse, o, dq, dk, dv, dks, dvs, dgate, ws_s, o_l, osp, blse
    torch.cuda.empty_cache()
    return res


def run_dense7b(args, torch, dist, rank, world, dev, peaks, peak_src):
    """The 7B-dense-shaped 1:3 block (B1 N8192, 32/8 heads, D128, top-16 blocks, SWA 128, 3 sparse
    layers, bf16) through the same step as the headline, per-kernel CUDA events over the steps;
    the targets are 60% (full layer + scores) and 50% (sparse layer, on its selected flops) of the
    sustained bf16 peak."""
    from attention_tcgen05_tma_b200 import inputs as I
    w = I.WORKLOADS["dense7b"]
    x = make_prefill_inputs(w, torch, dev, w.layers, seed_offset=1000 * rank)
    step = PrefillStep(w, x, torch, dev)
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    sp_flops = sparse_flops(step.idx.cpu().numpy(), w.N, w.G, w.D, w.window)
    full_flops = 4.0 * w.D * w.Hq * w.B * w.N * (w.N + 1) / 2
    steps = max(5, args.steps)
    evs = [{k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for k in ("full", "topk", "sparse")} for _ in range(steps)]
    for e in evs:
        e["topk"] = (e["full"][1], e["topk"][1])
        e["sparse"] = (e["topk"][1], e["sparse"][1])
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(steps):
        step.run(evs[i])
    torch.cuda.synchronize()
    per = {k: sum(e[k][0].elapsed_time(e[k][1]) for e in evs) / steps for k in ("full", "topk", "sparse")}
    ms_step = max_over_ranks(per["full"] + per["topk"] + per["sparse"], dist, dev)
    peak_tf = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    full_tf = full_flops / (per["full"] / 1e3) / 1e12
    sp_ms = per["sparse"] / w.layers
    sp_tf = sp_flops / (sp_ms / 1e3) / 1e12
    res = {"config": workload_config(w, world)["workload"], "steps": steps,
           "tokens_per_s": round(w.B * w.N * world / (ms_step / 1e3), 1), "ms_per_step": round(ms_step, 4),
           "full_attn_select_ms": round(per["full"], 4), "full_attn_select_tflops": round(full_tf, 2),
           "full_attn_select_frac": round(full_tf / peak_tf, 4), "full_target_ms": round(full_flops / (0.6 * peak_tf * 1e9), 4),
           "topk_ms": round(per["topk"], 4),
           "sparse_attn_ms_per_layer": round(sp_ms, 4), "sparse_attn_tflops": round(sp_tf, 2),
           "sparse_attn_frac": round(sp_tf / peak_tf, 4), "sparse_target_ms": round(sp_flops / (0.5 * peak_tf * 1e9), 4),
           "full_flops": full_flops, "sparse_flops_per_layer": sp_flops,
           "peak_source": f"{peak_src} bf16_tflops_sustained"}
    del x, step
    torch.cuda.empty_cache()
    return res


def _uses_tc(H, w):
    sh = H.hys_shape(w.B, w.N, w.Hq, w.Hkv, w.D, 64)
    return H.hysparse_full_attn_select_workspace_size(sh, H.HYS_BF16, H.HYS_GRAN_BLOCK) != \
        4 * w.B * w.Hq * w.T * w.NB


def run_decode_tokens(args, torch, dist, rank, world, dev, peaks, peak_src):
    """Token-variant decode step on the decode workload's cache: full layer with token scores,
    top-2048 tokens older than the forced newest 128, and the token-sparse layers; timed over the
    bf16 cache and again over its FP8 (E4M3, per-KV-head scales) copy."""
    from attention_tcgen05_tma_b200 import hysparse as H
    from attention_tcgen05_tma_b200 import inputs as I
    w = I.WORKLOADS[args.decode_workload]
    kt, W = 2048, 128
    x = make_decode_inputs(w, torch, dev, w.layers, seed_offset=1000 * rank)
    for key in ("k_swa", "v_swa", "gate"):
        x[key] = []   # the token variant has no SWA ring and no gate
    torch.cuda.empty_cache()
    o = torch.empty_like(x["q"])
    ts = torch.empty((w.B, w.Hkv, w.N), dtype=torch.float32, device=dev)
    idx = torch.empty((w.B, w.Hkv, kt), dtype=torch.int32, device=dev)
    osp = torch.empty_like(x["q"])
    sh = H.decode_shape(x["q"], x["k"])
    ws = H.workspace_for(H.hysparse_full_attn_select_decode_tokens_workspace_size(sh, H.HYS_BF16), dev)
    ws_sp = H.workspace_for(H.hysparse_sparse_attn_decode_tokens_workspace_size(sh, H.HYS_BF16, kt), dev)
    hbm = peaks["hbm_gbs"]

    def timed(full, sparse, elem_bytes):
        def step(ev=None):
            if ev:
                ev[0].record()
            full()
            if ev:
                ev[1].record()
            H.topk_decode_tokens(ts, kt, W, idx=idx)
            if ev:
                ev[2].record()
            for l in range(w.layers):
                sparse(l)
            if ev:
                ev[3].record()

        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        for i in range(args.steps):
            step(evs[i])
        torch.cuda.synchronize()
        full_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
        topk_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
        sp_ms = sum(e[2].elapsed_time(e[3]) for e in evs) / args.steps
        ms_step = max_over_ranks(sum(e[0].elapsed_time(e[3]) for e in evs) / args.steps, dist, dev)
        # full layer: K and V once, plus every key's logit written and read back for the scores
        full_bytes = 2.0 * w.B * w.Hkv * w.N * w.D * elem_bytes + 2.0 * w.B * w.Hq * w.N * 4
        sp_bytes = 2.0 * w.B * w.Hkv * (kt + W) * w.D * elem_bytes
        full_gbs = full_bytes / (full_ms / 1e3) / 1e9
        sp_gbs = sp_bytes / (sp_ms / w.layers / 1e3) / 1e9
        return {"us_per_token": round(ms_step * 1e3 / (w.B * world), 3),
                "ms_per_step": round(ms_step, 4),
                "full_ms": round(full_ms, 4), "topk_ms": round(topk_ms, 4),
                "sparse_ms_per_layer": round(sp_ms / w.layers, 4),
                "roofline": {"kernel": "full_attn_select_decode_tokens", "bound": "hbm", "achieved": round(full_gbs, 1),
                             "peak": hbm, "unit": "GB/s", "frac": round(full_gbs / hbm, 4), "traffic": None,
                             "peak_source": f"{peak_src} hbm_gbs"},
                "sparse_roofline": {"bound": "hbm", "achieved": round(sp_gbs, 1), "peak": hbm, "unit": "GB/s",
                                    "frac": round(sp_gbs / hbm, 4)}}

    res = timed(lambda: H.full_attn_select_decode_tokens(x["q"], x["k"], x["v"], o=o, tok_scores=ts, workspace=ws),
                lambda l: H.sparse_attn_decode_tokens(x["q_sparse"][l], x["k"], x["v"], idx, W, o=osp,
                                                      workspace=ws_sp), 2)
    res["config"] = (f"B={w.B} L={w.N} Hq={w.Hq} Hkv={w.Hkv} D={w.D}, 1 full + {w.layers} token-sparse, top-{kt} "
                     f"tokens + forced newest {W}")
    # the same cache as E4M3 codes of value / scale (one scale per KV head for K and for V),
    # converted on the device a sequence at a time
    ks_np, vs_np = I.fp8_kv_scales(w)
    ks, vs = torch.from_numpy(ks_np).to(dev), torch.from_numpy(vs_np).to(dev)
    k8 = torch.empty(x["k"].shape, dtype=torch.uint8, device=dev)
    v8 = torch.empty(x["v"].shape, dtype=torch.uint8, device=dev)
    for b in range(w.B):
        k8[b] = (x["k"][b].float() / ks[:, None, None]).to(torch.float8_e4m3fn).view(torch.uint8)
        v8[b] = (x["v"][b].float() / vs[:, None, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    del x["k"], x["v"]
    torch.cuda.empty_cache()
    res["fp8"] = timed(lambda: H.full_attn_select_decode_tokens_fp8(x["q"], k8, v8, ks, vs, o=o, tok_scores=ts,
                                                                    workspace=ws),
                       lambda l: H.sparse_attn_decode_tokens_fp8(x["q_sparse"][l], k8, v8, ks, vs, idx, W, o=osp,
                                                                 workspace=ws_sp), 1)
    res["fp8"]["cache"] = "E4M3 codes, per-KV-head K and V scales"
    del x, ts, ws, ws_sp, k8, v8
    torch.cuda.empty_cache()
    return res


def run_decode(args, torch, dist, rank, world, dev, peaks, peak_src):
    from attention_tcgen05_tma_b200 import hysparse as H
    from attention_tcgen05_tma_b200 import inputs as I
    w = I.WORKLOADS[args.decode_workload]
    x = make_decode_inputs(w, torch, dev, w.layers, seed_offset=1000 * rank)
    o = torch.empty_like(x["q"])
    sc = torch.empty((w.B, w.Hkv, w.NB), dtype=torch.float32, device=dev)
    idx = torch.empty((w.B, w.Hkv, w.topk), dtype=torch.int32, device=dev)
    osp = torch.empty_like(x["q"])
    sh = H.decode_shape(x["q"], x["k"])
    ws = H.workspace_for(H.hysparse_full_attn_select_decode_workspace_size(sh, H.HYS_BF16), dev)
    ws_sp = H.workspace_for(H.hysparse_sparse_attn_decode_workspace_size(sh, H.HYS_BF16, w.topk), dev)

    def step(ev=None):
        if ev:
            ev[0].record()
        H.full_attn_select_decode(x["q"], x["k"], x["v"], o=o, scores=sc, workspace=ws)
        if ev:
            ev[1].record()
        H.topk_decode(sc, w.topk, w.N, idx=idx)
        if ev:
            ev[2].record()
        for l in range(w.layers):
            H.sparse_attn_decode(x["q_sparse"][l], x["k"], x["v"], idx, x["k_swa"][l], x["v_swa"][l], x["gate"][l],
                                 o=osp, workspace=ws_sp)
        if ev:
            ev[3].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize()
    full_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    topk_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    sp_ms = sum(e[2].elapsed_time(e[3]) for e in evs) / args.steps
    ms_step = max_over_ranks(sum(e[0].elapsed_time(e[3]) for e in evs) / args.steps, dist, dev)
    full_bytes = 2.0 * w.B * w.Hkv * w.N * w.D * 2
    sp_bytes = 2.0 * w.B * w.Hkv * (w.topk * 64 + w.window) * w.D * 2
    hbm = peaks["hbm_gbs"]
    full_gbs = full_bytes / (full_ms / 1e3) / 1e9
    sp_gbs = sp_bytes / (sp_ms / w.layers / 1e3) / 1e9
    res = {"us_per_token": round(ms_step * 1e3 / (w.B * world), 3),
           "ms_per_step": round(ms_step, 4),
           "config": f"B={w.B} L={w.N} Hq={w.Hq} Hkv={w.Hkv} D={w.D}, 1 full + {w.layers} sparse, top-{w.topk} "
                     f"blocks + SWA ring {w.window}",
           "full_ms": round(full_ms, 4), "topk_ms": round(topk_ms, 4), "sparse_ms_per_layer": round(sp_ms / w.layers, 4),
           "roofline": {"kernel": "full_attn_select_decode", "bound": "hbm", "achieved": round(full_gbs, 1),
                        "peak": hbm, "unit": "GB/s", "frac": round(full_gbs / hbm, 4), "traffic": None,
                        "peak_source": f"{peak_src} hbm_gbs"},
           "sparse_roofline": {"bound": "hbm", "achieved": round(sp_gbs, 1), "peak": hbm, "unit": "GB/s",
                               "frac": round(sp_gbs / hbm, 4)}}
    del x
    torch.cuda.empty_cache()
    return res


def token_sparse_flops(idx_np, N, G, D, W, block=64):
    """Algorithmic flops of one token-sparse layer: 4*D per (row, head, attended key).  Row t of
    tile I attends Sel_I and its newest W tokens [max(0, t-W+1), t], each key once.  Every
    selected token is at most e_I - W < 64 I <= t, so the selected tokens at or after t - W + 1
    are the ones the two sets share."""
    B, Hkv, T, k = idx_np.shape
    win = np.minimum(np.arange(N) + 1, W)
    total = 0
    for b in range(B):
        for g in range(Hkv):
            for I in range(T):
                sel = idx_np[b, g, I]
                sel = np.sort(sel[sel >= 0])
                t = np.arange(I * block, min(N, (I + 1) * block))
                shared = sel.size - np.searchsorted(sel, t - W + 1, side="left")
                total += int((sel.size + win[t] - shared).sum())
    return 4.0 * D * total * G


def run_token(args, torch, dist, rank, world, dev, peaks, peak_src):
    """Token-granularity variant: full layer with token scores (two passes), top-k tokens with
    the forced newest window, and its token-sparse layers."""
    from attention_tcgen05_tma_b200 import hysparse as H
    from attention_tcgen05_tma_b200 import inputs as I
    w = I.WORKLOADS[args.token_workload]
    x = make_prefill_inputs(w, torch, dev, w.layers, seed_offset=1000 * rank)
    for key in ("k_swa", "v_swa", "gate"):
        x[key] = []   # the token variant has no SWA branch and no gate
    torch.cuda.empty_cache()
    T = w.T
    sh = H.prefill_shape(x["q"], x["k"])
    ws = H.workspace_for(H.hysparse_full_attn_select_workspace_size(sh, H.HYS_BF16, H.HYS_GRAN_TOKEN), dev)
    wst = H.workspace_for(H.hysparse_sparse_attn_tokens_workspace_size(sh, H.HYS_BF16, w.window), dev)
    o = torch.empty_like(x["q"])
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
    ts = torch.empty((w.B, w.Hkv, T, w.N), dtype=torch.float32, device=dev)
    idx = torch.empty((w.B, w.Hkv, T, w.topk), dtype=torch.int32, device=dev)
    osp = torch.empty_like(x["q"])

    def step(ev=None):
        if ev:
            ev[0].record()
        H.full_attn_select(x["q"], x["k"], x["v"], gran="token", o=o, scores=ts, lse=lse, workspace=ws)
        if ev:
            ev[1].record()
        H.topk_tokens(ts, w.topk, w.window, idx=idx)
        if ev:
            ev[2].record()
        for l in range(w.layers):
            H.sparse_attn_tokens(x["q_sparse"][l], x["k"], x["v"], idx, w.window, o=osp, workspace=wst)
        if ev:
            ev[3].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 3))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(steps):
        step(evs[i])
    torch.cuda.synchronize()
    full_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / steps
    topk_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / steps
    sp_ms = sum(e[2].elapsed_time(e[3]) for e in evs) / steps / w.layers
    ms_step = max_over_ranks(sum(e[0].elapsed_time(e[3]) for e in evs) / steps, dist, dev)
    peak_tf = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    full_alg = 4.0 * w.D * w.Hq * w.B * w.N * (w.N + 1) / 2
    full_exec = 1.5 * full_alg      # pass 2 recomputes Q.K^T (2.D of the 4.D flops per causal pair)
    sp_fl = token_sparse_flops(idx.cpu().numpy(), w.N, w.G, w.D, w.window)
    res = {"tokens_per_s": round(w.B * w.N * world / (ms_step / 1e3), 1), "ms_per_step": round(ms_step, 3),
           "steps": steps,
           "config": f"B={w.B} N={w.N} Hq={w.Hq} Hkv={w.Hkv} D={w.D}: full layer + token scores, top-{w.topk} "
                     f"tokens + forced newest {w.window}, {w.layers} token-sparse layers",
           "full_token_ms": round(full_ms, 3),
           "full_token_alg_tflops": round(full_alg / full_ms / 1e9, 1),
           "full_token_exec_tflops": round(full_exec / full_ms / 1e9, 1),
           "full_token_frac_exec": round(full_exec / full_ms / 1e9 / peak_tf, 4),
           "full_token_frac_alg": round(full_alg / full_ms / 1e9 / peak_tf, 4),
           "topk_tokens_ms": round(topk_ms, 3),
           "sparse_tokens_ms_per_layer": round(sp_ms, 3),
           "sparse_tokens_tflops": round(sp_fl / sp_ms / 1e9, 1),
           "sparse_tokens_frac": round(sp_fl / sp_ms / 1e9 / peak_tf, 4),
           "peak_source": f"{peak_src} bf16_tflops_sustained"}
    del x, o, lse, ts, idx, osp, ws, wst
    torch.cuda.empty_cache()
    return res


def run_e2e(args, torch, dist, world, w, x, step, dev=None):
    """Same step through the public API with the inputs and outputs in pinned HOST memory:
    every step copies its inputs host->device and every layer's output (the full layer's O and
    each sparse layer's O) device->host.  Input copies run on a stream of their own in layer order
    (Q, K, V first, then each sparse layer's Q', K', V', gate) and every layer starts once its own
    inputs have landed; each layer's output goes back on a third stream as soon as the layer
    ends, so both transfer directions overlap the compute of other layers.  A copy of the next
    step waits until the kernels of this step that read the same buffer are done (the shared K, V:
    the last sparse layer; a layer's own inputs: that layer), and a layer does not overwrite its
    output buffer before the previous step's copy of it has left."""
    H = step.H
    host = {k: (v.cpu().pin_memory() if not isinstance(v, list) else [t.cpu().pin_memory() for t in v])
            for k, v in x.items()}
    outs_dev = [step.o_full] + list(step.o_sp)
    outs_host = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs_dev]
    h2d = sum(t.numel() * t.element_size() for k, v in host.items() for t in (v if isinstance(v, list) else [v]))
    d2h = sum(t.numel() * t.element_size() for t in outs_host)
    groups = [[(x[k], host[k]) for k in ("q", "k", "v")]]
    groups += [[(x[k][l], host[k][l]) for k in ("q_sparse", "k_swa", "v_swa", "gate")] for l in range(w.layers)]
    main = torch.cuda.current_stream()
    copy_stream, back_stream = torch.cuda.Stream(), torch.cuda.Stream()
    copied = [torch.cuda.Event() for _ in groups]
    done = [None] * len(groups)          # event after the last kernel reading each group (previous step)
    sent = [None] * len(outs_dev)        # event after each output's device->host copy (previous step)

    def send(i):
        ev = torch.cuda.Event()
        ev.record(main)
        back_stream.wait_event(ev)
        with torch.cuda.stream(back_stream):
            outs_host[i].copy_(outs_dev[i], non_blocking=True)
            sent[i] = torch.cuda.Event()
            sent[i].record(back_stream)

    def one():
        with torch.cuda.stream(copy_stream):
            if done[0] is None:            # first step: after whatever the main stream holds
                copy_stream.wait_stream(main)
            for gi, grp in enumerate(groups):
                if done[gi] is not None:
                    copy_stream.wait_event(done[gi])
                for dst, src in grp:
                    dst.copy_(src, non_blocking=True)
                copied[gi].record(copy_stream)
        main.wait_event(copied[0])
        if sent[0] is not None:
            main.wait_event(sent[0])
        H.full_attn_select(x["q"], x["k"], x["v"], o=step.o_full, scores=step.scores, workspace=step.ws)
        send(0)
        H.topk(step.scores, w.topk, idx=step.idx)
        for l in range(w.layers):
            main.wait_event(copied[l + 1])
            if sent[l + 1] is not None:
                main.wait_event(sent[l + 1])
            H.sparse_attn(x["q_sparse"][l], x["k"], x["v"], step.idx, x["k_swa"][l], x["v_swa"][l], w.window,
                          x["gate"][l], o=step.o_sp[l], workspace=step.ws_sp)
            done[l + 1] = torch.cuda.Event()
            done[l + 1].record(main)
            send(l + 1)
        done[0] = torch.cuda.Event()
        done[0].record(main)

    for _ in range(max(1, args.warmup // 2)):
        one()
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 3))
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    copy_stream.wait_event(e0)
    back_stream.wait_event(e0)
    for _ in range(steps):
        one()
    main.wait_stream(back_stream)          # the last outputs are on the host when the region ends
    e1.record(main)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, dist, dev)
    del host, outs_host
    return {"value": round(w.B * w.N * world / (ms / 1e3), 1), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "ms_per_step": round(ms, 3), "steps": steps,
            "outputs_back": f"full layer O and all {w.layers} sparse layers' O, each its own buffer",
            "overlap": "per-layer host->device copies and per-layer device->host copies on their own streams, "
                       "overlapped with other layers' compute"}


# ----------------------------------------------------------------------------- CPU oracle
_CPU_CACHE = {}


def _group_inputs(w, b, g):
    """All slices one KV group needs (full layer + every sparse layer), drawn once."""
    from concurrent.futures import ThreadPoolExecutor

    from attention_tcgen05_tma_b200 import inputs as I
    key = (w.name, w.seed, b, g)
    if key in _CPU_CACHE:
        return _CPU_CACHE[key]
    _CPU_CACHE.clear()
    G = w.G
    heads = list(range(g * G, (g + 1) * G))
    jobs = {("q", h): (lambda h=h: I.q_slice(w, b, h)) for h in heads}
    jobs[("k",)] = lambda: I.k_slice(w, b, g)
    jobs[("v",)] = lambda: I.v_slice(w, b, g)
    for l in range(w.layers):
        jobs[("ks", l)] = lambda l=l: I.swa_k_slice(w, l, b, g)
        jobs[("vs", l)] = lambda l=l: I.swa_v_slice(w, l, b, g)
        for h in heads:
            jobs[("qs", l, h)] = lambda l=l, h=h: I.sparse_q_slice(w, l, b, h)
            jobs[("gate", l, h)] = lambda l=l, h=h: I.gate_slice(w, l, b, h)
    with ThreadPoolExecutor(min(32, os.cpu_count() or 8)) as ex:
        futs = {k: ex.submit(f) for k, f in jobs.items()}
        data = {k: f.result() for k, f in futs.items()}
    _CPU_CACHE[key] = data
    return data


def oracle_hybrid_tile(w, g, I_, data):
    """The oracle's hybrid block restricted to one (b, g, query tile): the full layer's rows
    for the group's heads, the tile's block scores, top-k, and every sparse layer's rows."""
    import oracle as O
    G = w.G
    rows = O.tile_rows(I_, w.N)
    heads = list(range(g * G, (g + 1) * G))
    kk, vv = data[("k",)], data[("v",)]
    qg = np.stack([data[("q", h)] for h in heads])
    for h in range(G):
        O.attention_rows(qg[h][rows], rows, kk, vv)
    sc = O.block_scores_tile(qg, kk, I_)
    sel = O.select_topk(sc, I_ + 1, w.topk)
    for l in range(w.layers):
        for h in heads:
            O.gated_sparse_rows(data[("qs", l, h)][rows], rows, kk, vv, sel, data[("ks", l)], data[("vs", l)],
                                w.window, data[("gate", l, h)][rows])


def cpu_baseline(w, budget_s=15.0, n_tiles=64, seed=1234):
    """Time the oracle (as it stands) on a bounded sample of query tiles of one KV group and
    extrapolate to the whole workload.  Each sampled unit is one (b, KV group, 64-query tile)
    through the full layer (all heads of the group), the top-k and every sparse layer.  The
    tiles are stratified over the tile index (one per equal slice of [0, T), a seeded random
    offset in each), and the whole workload's time is the mean time per tile times the number
    of tiles B * Hkv * T: the oracle's cost per tile does not depend on the tile's position (it
    forms every row's logits over all N keys), so this is the same estimate whatever the sample
    size."""
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    rng = np.random.default_rng(seed)
    b, g = 0, 0
    data = _group_inputs(w, b, g)        # input generation is not timed
    width = w.T / n_tiles
    order = rng.permutation(n_tiles)     # visit the strata in random order, so a cut-off sample is spread too
    t_total, done = 0.0, 0
    for s_ in order:
        if t_total >= budget_s and done > 0:
            break
        I_ = min(w.T - 1, int((s_ + rng.random()) * width))
        t0 = time.perf_counter()
        oracle_hybrid_tile(w, g, I_, data)
        t_total += time.perf_counter() - t0
        done += 1
    n_all = w.B * w.Hkv * w.T
    est_s = t_total / done * n_all
    tokens_per_s = (w.B * w.N) / est_s
    return {"value": round(tokens_per_s, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} query tiles of (b=0, kv-head 0), stratified over the tile index: 64 rows x {w.G} "
                      f"heads through the full layer, top-k and {w.layers} sparse layers in {t_total:.1f}s; "
                      f"whole workload = mean time per tile x {n_all} tiles (extrapolated)",
            "sample_s": round(t_total, 2), "tiles": done}


def run_reference(args, rank, world):
    """Reference arm: the float64 oracle on the host cores.  Each step is one bounded sample of
    the workload (stratified query tiles, the cpu_baseline estimator); ms_per_step is the time
    the sample took, and value is the whole workload's throughput extrapolated from it."""
    from attention_tcgen05_tma_b200 import inputs as I
    w = I.WORKLOADS[args.workload]
    if rank != 0:
        return None
    per_step_budget = max(2.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup):
        cpu_baseline(w, budget_s=per_step_budget / 4, n_tiles=1, seed=i)
    vals, sample_ms = [], []
    t0 = time.perf_counter()
    last = None
    for i in range(args.steps):
        t1 = time.perf_counter()
        last = cpu_baseline(w, budget_s=per_step_budget, n_tiles=64, seed=100 + i)
        sample_ms.append((time.perf_counter() - t1) * 1e3)
        vals.append(last["value"])
    wall = time.perf_counter() - t0
    value = statistics.median(vals)
    return {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(statistics.mean(sample_ms), 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)", "impl": "reference",
            "ms_per_step_kind": "measured time of one step's bounded sample; value is extrapolated from it",
            "whole_workload_s_extrapolated": round((w.B * w.N) / value, 1),
            "config": workload_config(w, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": last["cores"], "kind": "oracle",
                             "sample": last["sample"]},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s": round(wall, 1)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="moe80b", help="prefill workload (moe80b, dense7b, ...)")
    ap.add_argument("--decode-workload", default="decode", help="decode workload (decode, decode_small)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-decode-tokens", action="store_true", help="skip the token-variant decode leg")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-token", action="store_true")
    ap.add_argument("--no-rows", action="store_true", help="skip the per-position selection leg")
    ap.add_argument("--no-dense7b", action="store_true", help="skip the 7B-dense-shaped block leg")
    ap.add_argument("--no-backward", action="store_true", help="skip the training backward leg")
    ap.add_argument("--token-workload", default="token", help="token-variant workload")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    import torch
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist_mod
        torch.cuda.set_device(local)
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
        dist = dist_mod
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    res = run_ours(args, torch, dist, rank, world, dev)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
