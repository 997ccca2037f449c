"""Failure detection of the decode kernel: a bounded wait that runs out.

Every wait of the tensor-core decode kernel on its shared-memory ring is
bounded; when one gives up the kernel raises device flag 8, lets its copies
in flight land and returns, so the call ends and the CUDA context stays
usable.  KVC_TEST_DECODE_TIMEOUT=1 (read once per process) arms the first
ring slot of every CTA for 16 bytes that no copy delivers, which makes that
wait run out after a few short tries.  A child process decodes a small
batch in that mode and checks the flag, then that the device still runs
the library's kernels correctly (a dequantise of oracle-packed pages,
bit-exact against the oracle)."""

import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import sys
    sys.path.insert(0, sys.argv[1]); sys.path.insert(0, sys.argv[1] + "/tests")
    import numpy as np, torch
    import oracle as O, synth
    import compressed_decode_attention_kvc_b200 as K
    from kvc_testlib import HP, bits, lib_older_fmt, oracle_build_from_inputs, run_decode, upload_oracle_cache
    dev = torch.device("cuda:0")
    inp = synth.make_decode_inputs("tiny", seed=4, batch=3, context=16 * 12 + 5)
    cfg = inp["cfg"]
    cache, bt, fmt, older = oracle_build_from_inputs(inp, HP["bf16"])
    _, struct = upload_oracle_cache(cache, dev)
    B, max_pages = bt.shape
    assert K.kvc_decode_plan_info(B, cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"], max_pages)[0] \\
        == K.KVC_DECODE_KERNEL_MMA
    out, ws = run_decode(inp["q"].to(dev), struct, torch.from_numpy(bt).to(dev), lib_older_fmt(older, dev),
                         inp["context_lens"].to(dev), cfg["n_kv_heads"], max_pages, cfg["sink"], cfg["window"],
                         HP["bf16"])
    torch.cuda.synchronize()
    flags = K.kvc_decode_read_error(ws, B, cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"], max_pages)
    assert flags & K.ERR_TIMEOUT, flags
    # the context is still usable: dequantise oracle-packed ternary pages, bit-exact
    pages = bits(inp["k_pages"].reshape(-1, cfg["n_kv_heads"], 16, cfg["head_dim"])[:20].contiguous())
    codes_o, gamma_o = O.quantize_pack_ternary(pages)
    n, hkv, _, d = pages.shape
    back = torch.empty((n, hkv, 16, d), dtype=torch.bfloat16, device=dev)
    K.kvc_dequantize_pages(torch.from_numpy(codes_o).to(dev), torch.from_numpy(gamma_o).to(dev), None, n, 16,
                           hkv, d, K.KVC_FMT_TERNARY2, back)
    torch.cuda.synchronize()
    assert np.array_equal(bits(back), O.dequantize_ternary(codes_o, gamma_o))
    print("TIMEOUT-FLAG-OK")
""")


def test_decode_wait_timeout_sets_flag_and_context_survives(cuda_device):
    env = dict(os.environ, KVC_TEST_DECODE_TIMEOUT="1")
    r = subprocess.run([sys.executable, "-c", CHILD, ROOT], env=env, cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and "TIMEOUT-FLAG-OK" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]
