"""The allocation-free decode entry point, through the C ABI.

Some callers cannot allocate device memory while they run a decode step: a serving engine
that sizes all of its device memory at start-up and forbids later cudaMalloc calls (which
may synchronise the device), or a host integration with no allocator of its own.  For them
hysparse_full_attn_select_decode_noalloc takes its split-KV scratch from a fixed array inside
the library.  These tests check it against the regular entry point (which takes a caller
workspace) and against the float64 oracle, on several calls in a row that reuse the array.

Collected last on purpose: if it fails, a run that stops at the first failure has already run
every other test.  It passes both alone in a fresh process and after the other tests (the
array keeps the previous call's contents, and the entry point must not depend on them)."""
import numpy as np
import pytest
import torch

import oracle as O
from attention_tcgen05_tma_b200 import hysparse as H
from attention_tcgen05_tma_b200 import inputs as I
from tests.gpu_support import TOL, to_np

pytestmark = pytest.mark.gpu


def _case(B, L, Hq, Hkv, D, seed, dtype):
    w = I.scaled(I.WORKLOADS["decode"], B=B, N=L, Hq=Hq, Hkv=Hkv, D=D, layers=0, seed=seed,
                 scale_std=1.0 / np.sqrt(D))
    a = I.decode_arrays(w, layers=0)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    dev = lambda x: torch.from_numpy(x).to(tdt).cuda()  # noqa: E731  (exact: bf16 draws are pre-rounded)
    return a, dev(a["q"]), dev(a["k"]), dev(a["v"])


def _noalloc_into(q, kc, vc, seqlens, o, sc, dtype):
    sh = H.decode_shape(q, kc)
    st = H.hysparse_full_attn_select_decode_noalloc(sh, H.HYS_BF16 if dtype == "bf16" else H.HYS_F32,
                                                    q.data_ptr(), kc.data_ptr(), vc.data_ptr(),
                                                    seqlens.data_ptr() if seqlens is not None else None,
                                                    o.data_ptr(), sc.data_ptr(), H.HYS_REDUCE_SUM,
                                                    torch.cuda.current_stream().cuda_stream)
    assert st == H.HYS_OK, H.status_string(st)


# (B, L, Hq, Hkv, D, seed, dtype, seqlens): a large tensor-core case with many splits per
# sequence, then a small one with short sequences on the same path (the second call runs over
# the first call's leftover scratch in the same layout), then the fp32 path.
CASES = [
    (8, 16384, 32, 4, 128, 1, "bf16", [16384, 15000, 9001, 16383, 4097, 12000, 700, 16320]),
    (2, 300, 8, 1, 128, 2, "bf16", [300, 65]),
    (2, 4100, 8, 1, 64, 3, "f32", [4100, 1000]),
]


def test_noalloc_matches_regular_entry_point_and_oracle_on_calls_in_a_row():
    for B, L, Hq, Hkv, D, seed, dt, lens in CASES:
        a, q, kc, vc = _case(B, L, Hq, Hkv, D, seed, dt)
        sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        o_ref, sc_ref = H.full_attn_select_decode(q, kc, vc, seqlens=sl)
        o, sc = torch.empty_like(q), torch.empty_like(sc_ref)
        _noalloc_into(q, kc, vc, sl, o, sc, dt)
        torch.cuda.synchronize()
        tol = TOL[dt]
        assert torch.max(torch.abs(o.float() - o_ref.float())).item() <= tol
        rel = torch.abs(sc - sc_ref) / torch.clamp(sc_ref.abs(), min=1e-6)
        assert rel.max().item() <= 1e-3
        o_or, sc_or = O.decode_full(a["q"], a["k"], a["v"], seqlens=np.array(lens))
        assert np.max(np.abs(to_np(o) - o_or)) <= tol
        mask = sc_or > 1e-6
        assert np.max(np.abs(to_np(sc)[mask] - sc_or[mask]) / sc_or[mask]) <= 1e-3
        assert np.all(to_np(sc)[~mask] <= 1e-6)


def test_noalloc_second_call_leaves_device_memory_unchanged():
    """The first call on a device is its set-up (the driver may place the array on the device
    then); a later call allocates nothing, so the device's free memory does not move."""
    B, L, Hq, Hkv, D, seed, dt, lens = CASES[0]
    _, q, kc, vc = _case(B, L, Hq, Hkv, D, seed, dt)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o = torch.empty_like(q)
    sc = torch.empty((B, Hkv, (L + 63) // 64), dtype=torch.float32, device="cuda")
    _noalloc_into(q, kc, vc, sl, o, sc, dt)      # set-up call
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    _noalloc_into(q, kc, vc, sl, o, sc, dt)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before


def test_noalloc_rejects_shapes_beyond_capacity():
    sh = H.hys_decode_shape(64, 131072, 32, 4, 128, 64)   # needs far more than the fixed scratch
    assert H.hysparse_full_attn_select_decode_workspace_size(sh, H.HYS_BF16) > (16 << 20)
    st = H.hysparse_full_attn_select_decode_noalloc(sh, H.HYS_BF16, 16, 16, 16, None, 16, 16, H.HYS_REDUCE_SUM,
                                                    torch.cuda.current_stream().cuda_stream)
    assert st == H.HYS_ERR_WORKSPACE
