"""The watchdog path of the bounded waits, without faulting or hanging the GPU: in a child
process the token-score kernel runs with its test-only probe armed (HYS_WATCHDOG_PROBE=1: the
producer never issues the first unit's Q copies and every wait is limited to 0.2 s).  The MMA
warp's wait runs out, the kernel records HYS_ERR_TIMEOUT in the device status word, waits
(bounded) for the copies it did issue, frees TMEM and returns; the context stays usable for the
next launches.  A code read of that kernel shows every role reaches the per-unit block barrier
and the TMEM release on this path (all waits are mbarrier waits with a limit; no named
barriers)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys, torch
sys.path.insert(0, %r)
from attention_tcgen05_tma_b200 import hysparse as H
q = torch.randn(1, 4, 512, 128, device="cuda").to(torch.bfloat16)
k = torch.randn(1, 2, 512, 128, device="cuda").to(torch.bfloat16)
v = torch.randn(1, 2, 512, 128, device="cuda").to(torch.bfloat16)
H.hysparse_get_device_status(reset=True)
o, ts = H.full_attn_select(q, k, v, gran="token")
torch.cuda.synchronize()
st = H.hysparse_get_device_status(reset=True)
assert st == H.HYS_ERR_TIMEOUT, st
# the context is still usable: the block-score layer, a top-k and torch work normally
o2, sc = H.full_attn_select(q, k, v)
idx = H.topk(sc, 2)
torch.cuda.synchronize()
assert H.hysparse_get_device_status() == H.HYS_OK
assert torch.isfinite(o2.float()).all() and int(idx[0, 0, -1, 0]) >= 0
print("WATCHDOG_OK")
""" % ROOT


def test_bounded_wait_runs_out_and_reports_timeout():
    env = dict(os.environ, HYS_WATCHDOG_PROBE="1")
    r = subprocess.run([sys.executable, "-c", CHILD], capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0 and "WATCHDOG_OK" in r.stdout, (r.stdout[-2000:], r.stderr[-2000:])
