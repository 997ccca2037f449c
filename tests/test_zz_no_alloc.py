"""kvc_decode_attention_paged_noalloc: decode attention for callers that
cannot allocate device memory (their allocations all go through a
framework's pool, or they run under a fixed memory budget), so they cannot
hand the library a workspace.  The entry point uses a fixed device array
inside the library instead.

Checked through the C ABI against the regular entry point (which gets a
workspace from the caller), on two calls in a row: the second call finds
the array as the first left it and must still give the same answer.  This
file is collected last so that a run stopping at its first failure has
already run every other test; it passes alone in a fresh process too."""

import numpy as np
import pytest
import torch

import synth
import compressed_decode_attention_kvc_b200 as K
from kvc_testlib import (HP, assert_attention_close, lib_older_fmt, oracle_build_from_inputs,
                         run_decode, upload_oracle_cache)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,over", [
    ("qwen3b", dict(batch=3, context=1024 + 7)),
    ("longctx", dict(batch=2, context=(300, 2000), window=300)),
])
def test_noalloc_matches_regular_entry_point_twice(cuda_device, name, over):
    inp = synth.make_decode_inputs(name, seed=11, **over)
    cfg = inp["cfg"]
    hp = HP[cfg["hp"]]
    cache, bt, fmt, older = oracle_build_from_inputs(inp, hp)
    pools, struct = upload_oracle_cache(cache, cuda_device)
    q = inp["q"].to(cuda_device)
    B, hq, d = q.shape
    bt_d = torch.from_numpy(bt).to(cuda_device)
    older_d = lib_older_fmt(older, cuda_device)
    lens = inp["context_lens"].to(cuda_device)
    max_pages = bt.shape[1]
    hkv = cfg["n_kv_heads"]
    assert K.kvc_decode_workspace_size(B, hq, hkv, d, max_pages) <= K.NOALLOC_SCRATCH_BYTES

    ref, _ = run_decode(q, struct, bt_d, older_d, lens, hkv, max_pages, cfg["sink"], cfg["window"], hp)
    for call in range(2):
        out = torch.full((B, hq, d), float("nan"), dtype=torch.float32, device=cuda_device)
        K.kvc_decode_attention_paged_noalloc(q, struct, bt_d, older_d, lens, B, hq, hkv, d,
                                             K.PAGE_SIZE, max_pages, cfg["sink"], cfg["window"],
                                             hp, 0.0, out)
        torch.cuda.synchronize()
        assert_attention_close(out.cpu().numpy(), ref.cpu().numpy().astype(np.float64),
                               f"{name} no-alloc call {call}")


def _setup(name, dev, seed, **over):
    inp = synth.make_decode_inputs(name, seed=seed, **over)
    cfg = inp["cfg"]
    hp = HP[cfg["hp"]]
    cache, bt, fmt, older = oracle_build_from_inputs(inp, hp)
    pools, struct = upload_oracle_cache(cache, dev)
    args = dict(q=inp["q"].to(dev), struct=struct, bt=torch.from_numpy(bt).to(dev),
                older=lib_older_fmt(older, dev), lens=inp["context_lens"].to(dev), hkv=cfg["n_kv_heads"],
                max_pages=bt.shape[1], sink=cfg["sink"], window=cfg["window"], hp=hp)
    return args, pools


def _noalloc(a):
    B, hq, d = a["q"].shape
    out = torch.full((B, hq, d), float("nan"), dtype=torch.float32, device=a["q"].device)
    K.kvc_decode_attention_paged_noalloc(a["q"], a["struct"], a["bt"], a["older"], a["lens"], B, hq, a["hkv"], d,
                                         K.PAGE_SIZE, a["max_pages"], a["sink"], a["window"], a["hp"], 0.0, out)
    return out


def test_noalloc_small_then_large_call(cuda_device):
    # the first call (4 (sequence, KV head) pairs) leaves partial states at
    # the start of the array that the second call (96 pairs) uses for its
    # merge tickets: the second call must clear them before it runs
    small, ps = _setup("tiny", cuda_device, seed=3)
    large, pl = _setup("qwen3b", cuda_device, seed=4, batch=48, context=16 * 12 + 5)
    assert small["q"].shape[0] * small["hkv"] <= 8 and large["q"].shape[0] * large["hkv"] > 64
    for a in (small, large, small, large):
        out = _noalloc(a)
        torch.cuda.synchronize()
        ref, _ = run_decode(a["q"], a["struct"], a["bt"], a["older"], a["lens"], a["hkv"], a["max_pages"],
                            a["sink"], a["window"], a["hp"])
        torch.cuda.synchronize()
        assert_attention_close(out.cpu().numpy(), ref.cpu().numpy().astype(np.float64), "no-alloc sequence")


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_device):
    # a workspace larger than the fixed array is refused before any work
    B, hq, hkv, d, max_pages = 4096, 64, 8, 256, 1 << 15
    assert K.kvc_decode_workspace_size(B, hq, hkv, d, max_pages) > K.NOALLOC_SCRATCH_BYTES
    fake = torch.zeros(16, dtype=torch.uint8, device=cuda_device)
    struct = K.make_paged_cache(k_tern=fake, v_tern=fake, k_gamma=fake, v_gamma=fake, n_pages=(0, 0, 1))
    with pytest.raises(K.KvcError) as e:
        K.kvc_decode_attention_paged_noalloc(fake, struct, fake, None, fake, B, hq, hkv, d, K.PAGE_SIZE,
                                             max_pages, 4, 16, K.KVC_FMT_BF16, 0.0, fake)
    assert e.value.status == K.KVC_ERR_WORKSPACE
