"""kvc_decode_attention_paged_layers (all attention layers of one decode step
in one launch) against the fp64 oracle, layer by layer: each layer's cache
is built by the oracle from its own data with the shared page placement
(same lengths, tags and slot order, so one block table), the pools are
stacked layer after layer, and every layer's output must match the oracle's
attention over that layer's pages (max-abs 2e-3, relative-L2 1e-3).  The
tensor-core kernel is compared in the GQA <= 4 and wider layouts and with
FP8 / BF16 windows and anchors; virtual batches above one launch's 1024
sequences cover the consecutive launches."""

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


@pytest.mark.parametrize("batch,n_layers,launches", [
    (260, 4, 2),      # 1040 entries: the second launch starts inside layer 3 (row 244)
    (512, 4, 2),      # 2048 entries
    (700, 3, 3),      # 2100 entries: launches start inside layers 1 and 2
])
def test_layers_large_virtual_batch_tensor_core_kernel(cuda_device, batch, n_layers, launches):
    # layers * batch above one launch's 1024 virtual sequences: the
    # tensor-core kernel runs in consecutive launches
    kern, n = K.kvc_decode_plan_info(n_layers * batch, 8, 4, 64, 4)
    assert (kern, n) == (K.KVC_DECODE_KERNEL_MMA, launches)
    _run("tiny", dict(batch=batch, context=64, window=16), n_layers, cuda_device)


def test_qwen3b_36_layers_full_size_sampled(cuda_device):
    """The launch the benchmark times for the Qwen2.5-3B-shaped workload: 36
    layers of the full-size layer (B = 8, L = 4096) packed by the library and
    decoded in one launch.  For sampled (layer, sequence) pairs the library's
    pages are checked against the oracle's codec and then replaced by the
    oracle's bytes; those rows must match the oracle's attention.  Every row
    is finite and a convex combination of its layer's values."""
    from compressed_decode_attention_kvc_b200 import paged_cache as PC
    from kvc_testlib import check_ternary
    dev = cuda_device
    n_layers, P = 36, 16
    inps = [synth.make_decode_inputs("qwen3b", seed=1000 + l, device=dev) for l in range(n_layers)]
    cfg = inps[0]["cfg"]
    hp = HP[cfg["hp"]]
    B, max_pages, hkv, _, D = inps[0]["k_pages"].shape
    hq = cfg["n_q_heads"]
    lens_h = inps[0]["context_lens"].cpu()
    layout = PC.plan_paged_cache(lens_h, max_pages, cfg["sink"], cfg["window"], hp)
    cache = PC.allocate_device_cache(layout, hkv, D, dev, n_layers=n_layers)
    kf = torch.cat([i["k_pages"] for i in inps]).view(n_layers * B * max_pages, hkv, P, D)
    vf = torch.cat([i["v_pages"] for i in inps]).view(n_layers * B * max_pages, hkv, P, D)
    PC.compress_into(cache, kf, vf)
    torch.cuda.synchronize()
    bt, pf = layout.block_table.numpy(), layout.page_fmt.numpy()
    per_layer = layout.pool_pages
    pools = cache.pools
    refs = {}
    for l, b in [(0, 0), (17, 5), (35, 7)]:
        L = int(lens_h[b])
        sub = {"k_pages": inps[l]["k_pages"][b:b + 1].cpu(), "v_pages": inps[l]["v_pages"][b:b + 1].cpu(),
               "context_lens": lens_h[b:b + 1], "anchor": inps[l]["anchor"][b:b + 1].cpu(), "slot_key": None,
               "cfg": cfg}
        oc, obt, ofmt, _ = oracle_build_from_inputs(sub, hp)
        npg = O.num_pages(L)
        assert np.array_equal(ofmt[0, :npg], pf[b, :npg])
        for f, (kn, vn, ks, vs) in ((O.FP8_E4M3, ("k_fp8", "v_fp8", "k_fp8_scale", "v_fp8_scale")),
                                    (O.TERNARY, ("k_tern", "v_tern", "k_gamma", "v_gamma"))):
            js = np.nonzero(pf[b, :npg] == f)[0]
            if len(js) == 0:
                continue
            gslots = torch.from_numpy(l * per_layer[f] + bt[b, js].astype(np.int64)).to(dev)
            oslots = obt[0, js]
            for nm, sn, src in ((kn, ks, kf), (vn, vs, vf)):
                o_pool = getattr(oc, nm)[oslots]
                if f == O.TERNARY:
                    rows = torch.from_numpy(((l * B + b) * max_pages + js).astype(np.int64)).to(dev)
                    check_ternary(pools[nm][gslots].cpu().numpy(), pools[sn][gslots].cpu().numpy(),
                                  bits(src[rows]))
                else:
                    assert np.array_equal(pools[nm][gslots].cpu().numpy(), o_pool)
                    assert np.array_equal(pools[sn][gslots].cpu().numpy(), getattr(oc, sn)[oslots])
                pools[nm][gslots] = torch.from_numpy(o_pool).to(dev)
                pools[sn][gslots] = torch.from_numpy(getattr(oc, sn)[oslots]).to(dev)
        refs[(l, b)] = O.decode_attention(bits(inps[l]["q"][b:b + 1]), oc, obt, ofmt, [L], hkv)[0]

    q = torch.cat([i["q"] for i in inps])                       # [layers * B][Hq][D]
    ws_bytes = K.kvc_decode_workspace_size(n_layers * B, hq, hkv, D, max_pages)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    out = torch.full((n_layers * B, hq, D), float("nan"), device=dev)
    K.kvc_decode_attention_paged_layers(q, cache.struct, cache.block_table, None, inps[0]["context_lens"],
                                        n_layers, B, hq, hkv, D, P, max_pages, cfg["sink"], cfg["window"], hp,
                                        0.0, out, ws, ws_bytes)
    assert K.kvc_decode_read_error(ws, n_layers * B, hq, hkv, D, max_pages) == 0
    out_h = out.cpu().numpy().reshape(n_layers, B, hq, D)
    for (l, b), ref in refs.items():
        assert_attention_close(out_h[l, b], ref, f"qwen3b layer {l} b={b}")
    assert np.isfinite(out_h).all()
    G = hq // hkv
    for l in range(n_layers):
        vmax = inps[l]["v_pages"].abs().amax(dim=(1, 3, 4)).float().cpu().numpy()     # [B][Hkv]
        bound = np.repeat(vmax, G, axis=1)[:, :, None] * (1 + 1e-3) + 1e-6
        assert np.all(np.abs(out_h[l]) <= bound), l
