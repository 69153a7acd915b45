"""The FMA-pipe exp2 used for part of the softmax exponentials, emulated in fp32 on the
host, against numpy's exp2: relative error within the fitted bound wherever the result is a
normal float, and non-negative tiny values below."""
import numpy as np


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
