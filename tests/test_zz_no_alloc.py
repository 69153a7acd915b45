"""The allocation-free decode entry point (for callers that cannot allocate device
memory during a decode step) against the regular decode entry point, through the C ABI.

Collected last on purpose: if it fails, a run that stops at the first failure has
already run every other test.  It passes both alone in a fresh process and after the
other tests (the library's fixed scratch array keeps the previous call's contents, and
the entry point must not depend on them)."""
import numpy as np
import pytest
import torch

from attention_tcgen05_tma_b200 import hysparse as H
from attention_tcgen05_tma_b200 import inputs as I
from tests.gpu_support import TOL

pytestmark = pytest.mark.gpu


def _case(B, L, Hq, Hkv, D, seed):
    w = I.scaled(I.WORKLOADS["decode"], B=B, N=L, Hq=Hq, Hkv=Hkv, D=D, layers=0, seed=seed,
                 scale_std=1.0 / np.sqrt(D))
    a = I.decode_arrays(w, layers=0)
    dev = lambda x: torch.from_numpy(x).to(torch.bfloat16).cuda()  # noqa: E731
    return dev(a["q"]), dev(a["k"]), dev(a["v"])


def _noalloc(q, kc, vc, seqlens):
    sh = H.decode_shape(q, kc)
    o = torch.empty_like(q)
    sc = torch.empty((sh.B, sh.Hkv, (sh.L + 63) // 64), dtype=torch.float32, device="cuda")
    st = H.hysparse_full_attn_select_decode_noalloc(sh, H.HYS_BF16, q.data_ptr(), kc.data_ptr(), vc.data_ptr(),
                                                    seqlens.data_ptr() if seqlens is not None else None,
                                                    o.data_ptr(), sc.data_ptr(), H.HYS_REDUCE_SUM,
                                                    torch.cuda.current_stream().cuda_stream)
    assert st == H.HYS_OK, H.status_string(st)
    return o, sc


def test_noalloc_matches_regular_entry_point_on_two_calls():
    # two calls in a row with different shapes and lengths: the second must not see the first's scratch
    cases = [(3, 2000, 16, 2, 128, 1, [2000, 1500, 77]), (2, 4100, 8, 1, 64, 2, None)]
    for B, L, Hq, Hkv, D, seed, lens in cases:
        q, kc, vc = _case(B, L, Hq, Hkv, D, seed)
        sl = torch.tensor(lens, dtype=torch.int32, device="cuda") if lens else None
        o_ref, sc_ref = H.full_attn_select_decode(q, kc, vc, seqlens=sl)
        o, sc = _noalloc(q, kc, vc, sl)
        torch.cuda.synchronize()
        assert torch.max(torch.abs(o.float() - o_ref.float())).item() <= TOL["bf16"]
        rel = torch.abs(sc - sc_ref) / torch.clamp(sc_ref.abs(), min=1e-6)
        assert rel.max().item() <= 1e-3


def test_noalloc_rejects_shapes_beyond_capacity():
    sh = H.hys_decode_shape(64, 131072, 32, 4, 128, 64)   # needs far more than the fixed scratch
    assert H.hysparse_full_attn_select_decode_workspace_size(sh, H.HYS_BF16) > (16 << 20)
    st = H.hysparse_full_attn_select_decode_noalloc(sh, H.HYS_BF16, 16, 16, 16, None, 16, 16, H.HYS_REDUCE_SUM,
                                                    torch.cuda.current_stream().cuda_stream)
    assert st == H.HYS_ERR_WORKSPACE
