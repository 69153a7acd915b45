"""The FMA-pipe exp2 used for part of the softmax exponentials, emulated in fp32 on the
host, against numpy's exp2: relative error within the fitted bound wherever the result is a
normal float, and non-negative tiny values below."""
import numpy as np
import pytest


def exp2_poly3_fp32(x):
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0)).astype(np.float32)).astype(np.float32)
    p = (np.float32(0.0551716685) * f + np.float32(0.2426111251)).astype(np.float32)
    p = (p * f + np.float32(0.6932609677)).astype(np.float32)
    p = (p * f + np.float32(0.9999280572)).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.astype(np.int32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-124.0, 9.0, 2_000_001).astype(np.float32)
    y = exp2_poly3_fp32(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 8e-5, rel.max()


def test_tiny_and_masked_inputs():
    y = exp2_poly3_fp32(np.array([-np.inf, -1000.0, -127.0, -126.5, -125.0], np.float32))
    assert np.all(np.isfinite(y)) and np.all(y > 0) and np.all(y < 2.0 ** -124)


def _header_coefficients():
    """The four constants of exp2_poly3 and exp2_poly3_x2 in the kernels' PTX helper header."""
    import os
    import re
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "attention_tcgen05_tma_b200",
                        "csrc", "tc_ptx.cuh")
    src = open(path).read()
    out = []
    for fn in ("exp2_poly3", "exp2_poly3_x2"):
        body = src[src.index(f"__device__ __forceinline__ {'float2' if fn.endswith('x2') else 'float'} {fn}("):]
        body = body[:body.index("\n}\n")]
        consts = [float(v) for v in re.findall(r"(\d+\.\d+)f", body)
                  if float(v) not in (125.0, 12582912.0, 1.0)]
        out.append(sorted(set(consts)))
    return out


def test_coefficients_are_the_remez_fit():
    """Regenerate the polynomial by the Remez exchange method and compare with the header."""
    from tests.remez_exp2 import remez_exp2_rel
    c, E, emax = remez_exp2_rel(3)
    assert abs(emax - E) < 1e-9 and 7.4e-5 < E < 7.6e-5          # levelled: the fit converged
    want = sorted(c.tolist())
    for consts in _header_coefficients():
        assert len(consts) == 4, consts
        # the constants are compiled as fp32: agreement to about one fp32 ulp
        np.testing.assert_allclose(consts, want, rtol=1.2e-7, atol=0)


def test_remez_fit_beats_taylor():
    """Sanity of the fit itself: its worst relative error is well below the degree-3 Taylor
    polynomial's on the same interval, and it equioscillates (5 extrema of equal size)."""
    from tests.remez_exp2 import remez_exp2_rel
    import math
    c, E, _ = remez_exp2_rel(3)
    f = np.linspace(-0.5, 0.5, 100001)
    ln2 = math.log(2.0)
    taylor = 1 + ln2 * f + (ln2 * f) ** 2 / 2 + (ln2 * f) ** 3 / 6
    assert np.max(np.abs(taylor / np.exp2(f) - 1)) > 2 * E
    err = np.polyval(c[::-1], f) / np.exp2(f) - 1
    assert abs(err[0]) == pytest.approx(E, rel=1e-6) and abs(err[-1]) == pytest.approx(E, rel=1e-6)
