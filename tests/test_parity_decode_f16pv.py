"""The tensor-core kernel's f16 P.V path for ternary pages against the fp64
oracle.

At GQA <= 4 the library runs the ternary pages' P.V on int8 MMAs (P as two
exact unsigned digits) by default; KVC_DECODE_TERNARY_PV=f16, read once per
process, selects the f16 MMAs with P as an f16 hi + lo pair instead (the
path every GQA > 4 layout takes).  This test re-runs the decode parity file
and the outlier-query cases in a child process with that selection, so both
paths stay checked against the oracle."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_decode_parity_with_f16_ternary_pv(cuda_device):
    env = dict(os.environ, KVC_DECODE_TERNARY_PV="f16")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_parity_decode.py"),
                        os.path.join(ROOT, "tests", "test_parity_q_range.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
