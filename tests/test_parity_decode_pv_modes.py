"""The tensor-core kernel's other ternary P.V paths against the fp64 oracle.

At GQA <= 4 the library runs the ternary pages' P.V on int8 MMAs (P as two
exact unsigned digits) and tests the running maximum once per full entry of
8 pages by default.  KVC_DECODE_TERNARY_PV, read once per process, selects
instead "pair" (the same products, the maximum tested per page pair, as
entries shorter than 8 pages always run) or "f16" (f16 MMAs with P as an
f16 hi + lo pair, the path every GQA > 4 layout takes).  This test re-runs
the decode parity file and the outlier-query and moving-maximum cases in a
child process with each selection, so every path stays checked against the
oracle."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("mode", ["f16", "pair"])
def test_decode_parity_with_other_ternary_pv(cuda_device, mode):
    env = dict(os.environ, KVC_DECODE_TERNARY_PV=mode)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_parity_decode.py"),
                        os.path.join(ROOT, "tests", "test_parity_q_range.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
