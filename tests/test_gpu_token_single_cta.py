"""The token-sparse layer's single-CTA kernel for units of four or more M-tiles (two rounds over
the unit's keys), the path taken where no cluster of two CTAs fits on the device: the token
variant's parity cases with eight and sixteen heads per KV head run again in a child process
with HYS_TOKEN_SINGLE_CTA=1 (read once per process by the library), against the oracle."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_token_variant_single_cta_rounds():
    env = dict(os.environ, HYS_TOKEN_SINGLE_CTA="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-m", "gpu", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_gpu_parity.py"),
                        "-k", "token_variant and (g8_rounds or g6_pair or g16_pair or d64_g8)"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert " passed" in r.stdout and "4 passed" in r.stdout, r.stdout[-2000:]
