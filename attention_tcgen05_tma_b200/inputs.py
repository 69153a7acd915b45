"""Seeded synthetic inputs for the HySparse hybrid-block hot path.

This module is shared by the CPU oracle side (tests, CPU baseline) and the GPU
side (tests, bench).  It holds no attention arithmetic: it only draws random
tensors, rounds them to bf16 (a storage-format conversion) and applies the
"planted block" recipe that makes the block scores non-uniform.

Every tensor is produced slice by slice, one ``(tensor id, batch, head)`` slice
at a time, from its own PCG64 stream ``SeedSequence(seed, spawn_key=(tid, b, h))``.
Any slice can therefore be regenerated on its own, which lets the oracle check
sampled query tiles of the full-size workloads without materialising them.

Workloads (paper: HySparse, Table 1 / Section 4.1 for the head counts and the
64-token block, 1024-token budget and 128-token window; HySparse2 explainer for
the token-level variant and the forced newest-128 window):

* ``tiny``     fp32, B1 N1024, 4 query heads / 1 KV head, D64, k=4 blocks, 3 sparse layers
* ``dense7b``  bf16, B1 N8192, 32/8, D128, k=16 blocks, 3 sparse layers
* ``moe80b``   bf16, B2 N32768, 32/4, D128, k=32 blocks, 11 sparse layers
* ``moe80b_small``  the same per-unit shape at B1 N16384 with 2 sparse layers (profiling)
* ``decode``   bf16, B64, L131072 cached tokens, 32/4, D128, k=32 blocks, 11 sparse layers
* ``token``    bf16, B1 N131072, 32/4, D128, top-2048 tokens + forced 128, 3 sparse layers
* ``token_small``  the token variant at N32768 with 1 sparse layer (profiling)

An FP8 cache (the token-variant decode's FP8 option) stores the same normal draws as OCP E4M3
codes of value / scale, with one seeded scale per KV head for K and one for V (the conversion
to E4M3 is a storage-format rounding, like the bf16 one, done by torch).
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, List, Optional, Tuple

import numpy as np

# ----------------------------------------------------------------------------
# tensor ids (stream keys).  Per sparse layer l the ids are 16 + 8*l + {0..3}.
# ----------------------------------------------------------------------------
TID_Q, TID_K, TID_V = 0, 1, 2
TID_DO = 12          # output gradient of the full layer (training workloads)
TID_FP8_SCALE = 14
TID_PLANT = 15
_TID_LAYER0 = 16
SPARSE_Q, SPARSE_KSWA, SPARSE_VSWA, SPARSE_GATE, SPARSE_SINK, SPARSE_DO = 0, 1, 2, 3, 4, 5


def layer_tid(layer: int, which: int) -> int:
    return _TID_LAYER0 + 8 * layer + which


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    mode: str            # "prefill_block" | "prefill_token" | "decode"
    dtype: str           # "f32" | "bf16"
    B: int
    N: int               # sequence length (prefill) or cached length L (decode)
    Hq: int
    Hkv: int
    D: int
    layers: int          # sparse layers following the full layer
    topk: int            # blocks (block variant / decode) or tokens (token variant)
    window: int          # SWA window (block variant) or forced window (token variant)
    block: int = 64
    seed: int = 0
    scale_std: float = 1.0   # standard deviation of q/k/v draws
    plant: str = "none"      # "none" | "positions" | "blocks"
    n_plants: int = 0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def NB(self) -> int:
        return (self.N + self.block - 1) // self.block

    @property
    def T(self) -> int:
        return (self.N + self.block - 1) // self.block


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", "prefill_block", "f32", 1, 1024, 4, 1, 64, 3, 4, 128,
                     seed=0, scale_std=1.0, plant="positions", n_plants=8),
    "dense7b": Workload("dense7b", "prefill_block", "bf16", 1, 8192, 32, 8, 128, 3, 16, 128,
                        seed=1, scale_std=1.0 / math.sqrt(128), plant="blocks", n_plants=64),
    "moe80b": Workload("moe80b", "prefill_block", "bf16", 2, 32768, 32, 4, 128, 11, 32, 128,
                       seed=2, scale_std=1.0 / math.sqrt(128), plant="blocks", n_plants=64),
    "decode": Workload("decode", "decode", "bf16", 64, 131072, 32, 4, 128, 11, 32, 128,
                       seed=3, scale_std=1.0 / math.sqrt(128)),
    "token": Workload("token", "prefill_token", "bf16", 1, 131072, 32, 4, 128, 3, 2048, 128,
                      seed=4, scale_std=1.0 / math.sqrt(128), plant="blocks", n_plants=64),
    # the moe80b per-unit shape (G=8, k=32) at one sequence of 16K (profiling captures, < 1 GiB)
    "moe80b_small": Workload("moe80b_small", "prefill_block", "bf16", 1, 16384, 32, 4, 128, 2, 32, 128,
                             seed=6, scale_std=1.0 / math.sqrt(128), plant="blocks", n_plants=64),
    # the token variant at one sequence of 32K (profiling captures: token scores 256 MiB)
    "token_small": Workload("token_small", "prefill_token", "bf16", 1, 32768, 32, 4, 128, 1, 2048, 128,
                            seed=7, scale_std=1.0 / math.sqrt(128), plant="blocks", n_plants=64),
    # smaller decode batch with the same per-sequence shape (profiling captures: 2 GiB of cache)
    "decode_small": Workload("decode_small", "decode", "bf16", 8, 131072, 32, 4, 128, 11, 32, 128,
                             seed=5, scale_std=1.0 / math.sqrt(128)),
}


def scaled(w: Workload, **changes) -> Workload:
    """A copy of a workload with some fields replaced (smaller parity cases)."""
    return dataclasses.replace(w, **changes)


# ----------------------------------------------------------------------------
# bf16 storage rounding (round to nearest, ties to even), done on the bit pattern
# ----------------------------------------------------------------------------
def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 value (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32)
    bias = np.uint32(0x7FFF) + ((bits >> np.uint32(16)) & np.uint32(1))
    out = ((bits + bias) & np.uint32(0xFFFF0000)).astype(np.uint32)
    return out.view(np.float32)


def _stream(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=tuple(key))))


def normal_slice(seed: int, tid: int, b: int, h: int, shape: Tuple[int, ...], std: float,
                 bf16: bool) -> np.ndarray:
    """One (tensor, batch, head) slice: fp32 N(0, std^2) draws, optionally bf16-rounded."""
    x = _stream(seed, tid, b, h).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x = x * np.float32(std)
    return round_bf16(x) if bf16 else x


# ----------------------------------------------------------------------------
# planting
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Plant:
    b: int
    g: int          # KV head
    pos: int        # first key position that is overwritten
    length: int     # 1 (position plant) or block size (block plant)
    h: int          # query head whose query is copied
    t: int          # query position whose query is copied
    additive: bool  # block plants add the planted direction to the existing key


def plants(w: Workload) -> List[Plant]:
    """The planted keys of a workload, in application order.

    * ``positions`` (tiny fp32 workload): 8 distinct positions p in [0, N-2]; each gets
      a random query head h of its KV group and a later query position t in (p, N);
      the key at p is replaced by 3 * q_t / |q_t|.
    * ``blocks``: n distinct (b, g, j) with j < NB-1; a random query head h of group g
      and a query position t in [64(j+1), N); every key of block j becomes
      3 * sqrt(D) * q_t / |q_t| plus its own drawn value.
    """
    if w.plant == "none" or w.n_plants == 0:
        return []
    rng = _stream(w.seed, TID_PLANT)
    out: List[Plant] = []
    if w.plant == "positions":
        ps = rng.choice(w.N - 1, size=min(w.n_plants, w.N - 1), replace=False)
        for p in ps:
            b = int(rng.integers(w.B))
            g = int(rng.integers(w.Hkv))
            h = g * w.G + int(rng.integers(w.G))
            t = int(rng.integers(int(p) + 1, w.N))
            out.append(Plant(b, g, int(p), 1, h, t, False))
    elif w.plant == "blocks":
        nbl = w.NB - 1
        if nbl <= 0:
            return []
        n = min(w.n_plants, w.B * w.Hkv * nbl)
        flat = rng.choice(w.B * w.Hkv * nbl, size=n, replace=False)
        for f in flat:
            f = int(f)
            b, rem = divmod(f, w.Hkv * nbl)
            g, j = divmod(rem, nbl)
            h = g * w.G + int(rng.integers(w.G))
            t = int(rng.integers(w.block * (j + 1), w.N))
            out.append(Plant(b, g, w.block * j, w.block, h, t, True))
    else:
        raise ValueError(w.plant)
    return out


def _plant_direction(w: Workload, p: Plant, q_row: np.ndarray) -> np.ndarray:
    qn = q_row.astype(np.float64)
    unit = qn / np.sqrt(np.dot(qn, qn))
    gain = 3.0 * (math.sqrt(w.D) if p.additive else 1.0)
    return (gain * unit).astype(np.float32)


# ----------------------------------------------------------------------------
# slices of the prefill workloads
# ----------------------------------------------------------------------------
def _bf16(w: Workload) -> bool:
    return w.dtype == "bf16"


def q_slice(w: Workload, b: int, h: int) -> np.ndarray:
    return normal_slice(w.seed, TID_Q, b, h, (w.N, w.D), w.scale_std, _bf16(w))


def k_slice(w: Workload, b: int, g: int, _plants: Optional[List[Plant]] = None) -> np.ndarray:
    k = normal_slice(w.seed, TID_K, b, g, (w.N, w.D), w.scale_std, False)
    pl = plants(w) if _plants is None else _plants
    qcache: Dict[int, np.ndarray] = {}
    for p in pl:
        if p.b != b or p.g != g:
            continue
        if p.h not in qcache:
            qcache[p.h] = q_slice(w, b, p.h)
        d = _plant_direction(w, p, qcache[p.h][p.t])
        if p.additive:
            k[p.pos:p.pos + p.length] += d[None, :]
        else:
            k[p.pos:p.pos + p.length] = d[None, :]
    return round_bf16(k) if _bf16(w) else k


def v_slice(w: Workload, b: int, g: int) -> np.ndarray:
    return normal_slice(w.seed, TID_V, b, g, (w.N, w.D), w.scale_std, _bf16(w))


def sparse_q_slice(w: Workload, layer: int, b: int, h: int) -> np.ndarray:
    return normal_slice(w.seed, layer_tid(layer, SPARSE_Q), b, h, (w.N, w.D), w.scale_std, _bf16(w))


def swa_k_slice(w: Workload, layer: int, b: int, g: int) -> np.ndarray:
    n = w.window if w.mode == "decode" else w.N
    return normal_slice(w.seed, layer_tid(layer, SPARSE_KSWA), b, g, (n, w.D), w.scale_std, _bf16(w))


def swa_v_slice(w: Workload, layer: int, b: int, g: int) -> np.ndarray:
    n = w.window if w.mode == "decode" else w.N
    return normal_slice(w.seed, layer_tid(layer, SPARSE_VSWA), b, g, (n, w.D), w.scale_std, _bf16(w))


def gate_slice(w: Workload, layer: int, b: int, h: int) -> np.ndarray:
    """Gate logits (fp32, standard normal): [N, 2] for prefill, [2] for decode."""
    shape = (2,) if w.mode == "decode" else (w.N, 2)
    return normal_slice(w.seed, layer_tid(layer, SPARSE_GATE), b, h, shape, 1.0, False)


def d_o_slice(w: Workload, b: int, h: int) -> np.ndarray:
    """Output gradient of the full layer (training): N(0, std^2) draws like Q, [N, D]."""
    return normal_slice(w.seed, TID_DO, b, h, (w.N, w.D), w.scale_std, _bf16(w))


def sparse_d_o_slice(w: Workload, layer: int, b: int, h: int) -> np.ndarray:
    """Output gradient of a sparse layer (training), [N, D]."""
    return normal_slice(w.seed, layer_tid(layer, SPARSE_DO), b, h, (w.N, w.D), w.scale_std, _bf16(w))


def sink_logits(w: Workload, layer: int, std: float = 2.0) -> np.ndarray:
    """Per-head sink logits of a sparse layer, [Hq, 2] fp32 (index 0: sparse branch, 1: SWA
    branch); standard deviation 2 so that sinks range from negligible to dominant."""
    return np.stack([normal_slice(w.seed, layer_tid(layer, SPARSE_SINK), 0, h, (2,), std, False)
                     for h in range(w.Hq)]).astype(np.float32)


# decode: the query of the new token, the shared cache and the SWA rings
def decode_q_slice(w: Workload, b: int, h: int) -> np.ndarray:
    return normal_slice(w.seed, TID_Q, b, h, (w.D,), w.scale_std, True)


def decode_k_slice(w: Workload, b: int, g: int) -> np.ndarray:
    return normal_slice(w.seed, TID_K, b, g, (w.N, w.D), w.scale_std, True)


def decode_v_slice(w: Workload, b: int, g: int) -> np.ndarray:
    return normal_slice(w.seed, TID_V, b, g, (w.N, w.D), w.scale_std, True)


def decode_sparse_q_slice(w: Workload, layer: int, b: int, h: int) -> np.ndarray:
    return normal_slice(w.seed, layer_tid(layer, SPARSE_Q), b, h, (w.D,), w.scale_std, True)


# FP8 (E4M3) decode cache: codes of value / scale, one scale per KV head for K and for V
def fp8_kv_scales(w: Workload) -> Tuple[np.ndarray, np.ndarray]:
    """[Hkv] float32 scales for K and for V: the cache's std / 32 times a seeded factor in
    [0.75, 1.25], so the codes stay well inside E4M3's range (|code| <= 448)."""
    u = _stream(w.seed, TID_FP8_SCALE).uniform(0.75, 1.25, size=(2, w.Hkv))
    base = w.scale_std / 32.0
    return (base * u[0]).astype(np.float32), (base * u[1]).astype(np.float32)


def e4m3_codes(x: np.ndarray) -> np.ndarray:
    """float32 values -> OCP E4M3 ("fn") codes as uint8, rounded to nearest (torch's conversion)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def decode_k_fp8_slice(w: Workload, b: int, g: int) -> np.ndarray:
    x = normal_slice(w.seed, TID_K, b, g, (w.N, w.D), w.scale_std, False)
    return e4m3_codes(x / fp8_kv_scales(w)[0][g])


def decode_v_fp8_slice(w: Workload, b: int, g: int) -> np.ndarray:
    x = normal_slice(w.seed, TID_V, b, g, (w.N, w.D), w.scale_std, False)
    return e4m3_codes(x / fp8_kv_scales(w)[1][g])


# ----------------------------------------------------------------------------
# whole tensors (small workloads, or bulk fill with threads)
# ----------------------------------------------------------------------------
def _fill(shape, fn, keys, threads: int = 8) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)

    def one(key):
        out[key] = fn(*key)

    if threads <= 1 or len(keys) <= 1:
        for key in keys:
            one(key)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, keys))
    return out


def prefill_arrays(w: Workload, layers: Optional[int] = None, threads: int = 8,
                   grads: bool = False) -> Dict[str, object]:
    """All prefill tensors of a workload as float32 numpy arrays ([B, H, N, D] layout).

    Keys: q, k, v, and per sparse layer l: q_sparse[l], k_swa[l], v_swa[l], gate[l]
    (gate is [B, Hq, N, 2]); with grads, also the output gradients d_o (full layer) and
    d_o_sparse[l].
    """
    L = w.layers if layers is None else layers
    bq = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    bk = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    pl = plants(w)
    out: Dict[str, object] = {
        "q": _fill((w.B, w.Hq, w.N, w.D), lambda b, h: q_slice(w, b, h), bq, threads),
        "k": _fill((w.B, w.Hkv, w.N, w.D), lambda b, g: k_slice(w, b, g, pl), bk, threads),
        "v": _fill((w.B, w.Hkv, w.N, w.D), lambda b, g: v_slice(w, b, g), bk, threads),
        "q_sparse": [], "k_swa": [], "v_swa": [], "gate": [],
    }
    for l in range(L):
        out["q_sparse"].append(_fill((w.B, w.Hq, w.N, w.D), lambda b, h: sparse_q_slice(w, l, b, h), bq, threads))
        out["k_swa"].append(_fill((w.B, w.Hkv, w.N, w.D), lambda b, g: swa_k_slice(w, l, b, g), bk, threads))
        out["v_swa"].append(_fill((w.B, w.Hkv, w.N, w.D), lambda b, g: swa_v_slice(w, l, b, g), bk, threads))
        out["gate"].append(_fill((w.B, w.Hq, w.N, 2), lambda b, h: gate_slice(w, l, b, h), bq, threads))
    if grads:
        out["d_o"] = _fill((w.B, w.Hq, w.N, w.D), lambda b, h: d_o_slice(w, b, h), bq, threads)
        out["d_o_sparse"] = [_fill((w.B, w.Hq, w.N, w.D), lambda b, h: sparse_d_o_slice(w, l, b, h), bq, threads)
                             for l in range(L)]
    return out


def decode_fp8_cache(w: Workload, threads: int = 8) -> Dict[str, np.ndarray]:
    """The FP8 decode cache: k8/v8 uint8 codes [B,Hkv,L,D] and k_scale/v_scale [Hkv] float32."""
    bk = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    out = {"k8": np.empty((w.B, w.Hkv, w.N, w.D), np.uint8), "v8": np.empty((w.B, w.Hkv, w.N, w.D), np.uint8)}

    def one(key):
        out["k8"][key] = decode_k_fp8_slice(w, *key)
        out["v8"][key] = decode_v_fp8_slice(w, *key)

    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(one, bk))
    out["k_scale"], out["v_scale"] = fp8_kv_scales(w)
    return out


def decode_arrays(w: Workload, layers: Optional[int] = None, threads: int = 8) -> Dict[str, object]:
    """All decode tensors: q [B,Hq,D], k/v cache [B,Hkv,L,D]; per layer q_sparse [B,Hq,D],
    k_swa/v_swa rings [B,Hkv,W,D], gate [B,Hq,2]."""
    L = w.layers if layers is None else layers
    bq = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    bk = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    out: Dict[str, object] = {
        "q": _fill((w.B, w.Hq, w.D), lambda b, h: decode_q_slice(w, b, h), bq, threads),
        "k": _fill((w.B, w.Hkv, w.N, w.D), lambda b, g: decode_k_slice(w, b, g), bk, threads),
        "v": _fill((w.B, w.Hkv, w.N, w.D), lambda b, g: decode_v_slice(w, b, g), bk, threads),
        "q_sparse": [], "k_swa": [], "v_swa": [], "gate": [],
    }
    for l in range(L):
        out["q_sparse"].append(_fill((w.B, w.Hq, w.D), lambda b, h: decode_sparse_q_slice(w, l, b, h), bq, threads))
        out["k_swa"].append(_fill((w.B, w.Hkv, w.window, w.D), lambda b, g: swa_k_slice(w, l, b, g), bk, threads))
        out["v_swa"].append(_fill((w.B, w.Hkv, w.window, w.D), lambda b, g: swa_v_slice(w, l, b, g), bk, threads))
        out["gate"].append(_fill((w.B, w.Hq, 2), lambda b, h: gate_slice(w, l, b, h), bq, threads))
    return out


def sampled_tiles(w: Workload, count: int = 8) -> List[Tuple[int, int, int]]:
    """Seeded sample of (b, kv-head, query tile) triples for full-size parity checks.

    Always includes the last tile and, for the token variant, tile ceil((topk+window)/64)
    (the first tile whose rows cannot see every earlier token)."""
    rng = _stream(w.seed, 99)
    tiles = {(0, 0, w.T - 1)}
    if w.mode == "prefill_token":
        tiles.add((0, 0, min(w.T - 1, -(-(w.topk + w.window) // w.block))))
    while len(tiles) < min(count, w.B * w.Hkv * w.T):
        tiles.add((int(rng.integers(w.B)), int(rng.integers(w.Hkv)), int(rng.integers(w.T))))
    return sorted(tiles)
