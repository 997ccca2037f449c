"""kvc_decode_attention_paged_layers (all attention layers of one decode step
in one launch) against the fp64 oracle, layer by layer: each layer's cache
is built by the oracle from its own data with the shared page placement
(same lengths, tags and slot order, so one block table), the pools are
stacked layer after layer, and every layer's output must match the oracle's
attention over that layer's pages (max-abs 2e-3, relative-L2 1e-3).  The
tensor-core kernel is compared in the GQA <= 4 and wider layouts and with
FP8 / BF16 windows and anchors; a large virtual batch covers the CUDA-core
kernel."""

import numpy as np
import pytest
import torch

import oracle as O
import synth
import compressed_decode_attention_kvc_b200 as K
from kvc_testlib import (HP, assert_attention_close, bits, lib_older_fmt, oracle_build_from_inputs,
                         upload_oracle_cache)

pytestmark = pytest.mark.gpu


def _stack(caches):
    c0 = caches[0]
    out = O.PagedCache(**{f: np.concatenate([getattr(c, f) for c in caches])
                          for f in c0.__dataclass_fields__})
    return out


def _run(name, over, n_layers, dev):
    inps = [synth.make_decode_inputs(name, seed=100 + l, **over) for l in range(n_layers)]
    cfg = inps[0]["cfg"]
    hp = HP[cfg["hp"]]
    built = []
    for l, inp in enumerate(inps):
        # shared placement: the first layer's lengths, tags and slot order
        inp["context_lens"] = inps[0]["context_lens"]
        inp["anchor"] = inps[0]["anchor"]
        inp["slot_key"] = inps[0]["slot_key"]
        built.append(oracle_build_from_inputs(inp, hp))
    bt, fmt, older = built[0][1], built[0][2], built[0][3]
    for c, b2, f2, _ in built[1:]:
        assert np.array_equal(b2, bt) and np.array_equal(f2, fmt)
    stacked = _stack([b[0] for b in built])
    t, struct = upload_oracle_cache(stacked, dev)
    # the struct's page counts are per layer
    struct.n_pages[0] = built[0][0].k_bf16.shape[0]
    struct.n_pages[1] = built[0][0].k_fp8.shape[0]
    struct.n_pages[2] = built[0][0].k_tern.shape[0]
    B, max_pages = bt.shape
    hq, hkv, d = cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    q = torch.stack([inp["q"] for inp in inps]).to(dev)          # [layers][B][Hq][D]
    lens = inps[0]["context_lens"].to(dev)
    ws_bytes = K.kvc_decode_workspace_size(n_layers * B, hq, hkv, d, max_pages)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    out = torch.full((n_layers, B, hq, d), float("nan"), dtype=torch.float32, device=dev)
    K.kvc_decode_attention_paged_layers(q, struct, torch.from_numpy(bt).to(dev), lib_older_fmt(older, dev),
                                        lens, n_layers, B, hq, hkv, d, K.PAGE_SIZE, max_pages, cfg["sink"],
                                        cfg["window"], hp, 0.0, out, ws, ws_bytes)
    torch.cuda.synchronize()
    assert K.kvc_decode_read_error(ws, n_layers * B, hq, hkv, d, max_pages) == 0
    got = out.cpu().numpy()
    for l, (cache, _, _, _) in enumerate(built):
        ref = O.decode_attention(bits(inps[l]["q"]), cache, bt, fmt, inps[0]["context_lens"].numpy(), hkv)
        assert_attention_close(got[l], ref, f"{name} layer {l}")


@pytest.mark.parametrize("name,over,n_layers", [
    ("llama8b", dict(batch=2, context=700), 3),                                  # GQA 4, BF16 window
    ("qwen3b", dict(batch=3, context=1031), 4),                                  # GQA 8, FP8 window
    ("longctx", dict(batch=2, context=(300, 1500), window=300), 2),              # D 256, anchors
    ("tiny", dict(batch=2), 3),
])
def test_layers_match_oracle_per_layer(cuda_device, name, over, n_layers):
    _run(name, over, n_layers, cuda_device)


def test_layers_large_virtual_batch_cuda_core_kernel(cuda_device):
    # layers * batch above the tensor-core kernel's batch limit (1024)
    _run("tiny", dict(batch=260, context=64, window=16), 4, cuda_device)
