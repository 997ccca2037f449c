"""The tensor-memory (tcgen05) decode kernel against the fp64 oracle.

The library runs its register-sourced tensor-core kernel by default; the
tcgen05 kernel (int8 MMAs with accumulators in tensor memory, one MMA-issuer
warp per warpgroup) is selected by KVC_DECODE_KERNEL=tcgen05, read once per
process.  This test re-runs the whole decode parity file in a child process
with that selection, so both implementations stay checked against the oracle
(head_dim 256, which the tcgen05 kernel does not take, falls back to the
default kernel there)."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_decode_parity_with_tcgen05_kernel(cuda_device):
    env = dict(os.environ, KVC_DECODE_KERNEL="tcgen05")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_parity_decode.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
