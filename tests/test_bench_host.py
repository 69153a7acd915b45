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
