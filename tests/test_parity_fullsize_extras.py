"""Stale-to-anchor promotion and the lossless BF16 codec in the launch
configuration the benchmark times: the Llama-3-8B-shaped layer at full size
(B = 32, L = 32768), 32 promotions per sequence and all 4160 BF16 window
pages coded in one launch.  Sampled outputs are compared with the oracle
bit for bit; the oracle's inputs are the generator's bf16 pages (and, for
promotion, the oracle's own ternary bytes placed in the sampled slots)."""

import numpy as np
import pytest
import torch

import oracle as O
import oracle.exans as X
import synth
import compressed_decode_attention_kvc_b200 as K
from compressed_decode_attention_kvc_b200 import paged_cache as PC
from kvc_testlib import bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def llama_cache(cuda_device):
    dev = cuda_device
    inp = synth.make_decode_inputs("llama8b", seed=0, device=dev)
    cfg = inp["cfg"]
    B, max_pages, hkv, P, D = inp["k_pages"].shape
    lens_h = inp["context_lens"].cpu()
    layout = PC.plan_paged_cache(lens_h, max_pages, cfg["sink"], cfg["window"], K.KVC_FMT_BF16,
                                 slot_key=inp["slot_key"].cpu())
    cache = PC.allocate_device_cache(layout, hkv, D, dev)
    kf = inp["k_pages"].view(B * max_pages, hkv, P, D)
    vf = inp["v_pages"].view(B * max_pages, hkv, P, D)
    PC.compress_into(cache, kf, vf)
    torch.cuda.synchronize()
    yield dict(inp=inp, cfg=cfg, layout=layout, cache=cache, kf=kf, vf=vf, lens_h=lens_h, dims=(B, max_pages, hkv, P, D))
    del cache, inp
    torch.cuda.empty_cache()


def test_codec_full_size_sampled(llama_cache, cuda_device):
    c = llama_cache
    B, max_pages, hkv, P, D = c["dims"]
    pools = c["cache"].pools
    src = torch.cat([pools["k_bf16"], pools["v_bf16"]])
    n = src.shape[0]
    N = hkv * P * D
    ws_bytes = K.kvc_exans_workspace_size(n, P, hkv, D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=cuda_device)
    dst_bytes = n * (64 + 2 * N)
    dst = torch.empty(dst_bytes, dtype=torch.uint8, device=cuda_device)
    off = torch.empty(n + 1, dtype=torch.int64, device=cuda_device)
    K.kvc_exans_encode(src, None, n, P, hkv, D, ws, ws_bytes, dst, dst_bytes, off)
    back = torch.empty_like(src)
    flags = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    K.kvc_exans_decode(dst, dst_bytes, off, n, None, n, P, hkv, D, back, flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    assert torch.equal(back.view(torch.int16), src.view(torch.int16))        # lossless at full size
    off_h = off.cpu().numpy()
    assert off_h[0] == 0 and (np.diff(off_h) % 16 == 0).all() and (np.diff(off_h) >= 64).all()
    ids = c["layout"].pool_src_ids[0].numpy()           # logical page of each BF16 slot
    n_bf = len(ids)
    for i in (0, 1234, n_bf - 1, n_bf, n - 1):
        which, slot = ("k", i) if i < n_bf else ("v", i - n_bf)
        logical = ids[slot]
        page = bits((c["inp"]["k_pages"] if which == "k" else c["inp"]["v_pages"]).view(-1, hkv, P, D)[logical])
        want = X.encode_group(page.reshape(-1))
        got = dst[off_h[i]:off_h[i + 1]].cpu().numpy().tobytes()
        assert got == want, i


def test_promote_full_size_sampled(llama_cache, cuda_device):
    c = llama_cache
    dev = cuda_device
    B, max_pages, hkv, P, D = c["dims"]
    cfg, cache = c["cfg"], c["cache"]
    L = c["lens_h"].tolist()
    per_seq = 32
    reqs = []
    for b in range(B):
        first = -(-cfg["sink"] // P)
        last = max(0, (L[b] - cfg["window"]) // P)
        step = (last - first) // per_seq
        reqs += [(b, first + i * step) for i in range(per_seq)]
    n = len(reqs)
    assert n == 1024
    bt = cache.block_table.cpu().numpy()
    sample = [0, 517, n - 1]
    # the sampled pages' ternary slots get the oracle's own encoding of their bf16 pages
    expect = {}
    for r in sample:
        b, j = reqs[r]
        t = int(bt[b, j])
        for which, src in (("k", c["kf"]), ("v", c["vf"])):
            page = bits(src[b * max_pages + j])[None]                  # [1][Hkv][P][D]
            codes, gam = O.quantize_pack_ternary(page)
            cache.pools[which + "_tern"][t] = torch.from_numpy(codes[0]).to(dev)
            cache.pools[which + "_gamma"][t] = torch.from_numpy(gam[0]).to(dev)
            expect[(r, which)] = O.dequantize_ternary(codes, gam)[0]
    anchors = {w: torch.full((n, hkv, P, D), 0x7FC0, dtype=torch.int16, device=dev).view(torch.bfloat16)
               for w in ("k", "v")}
    st = K.kvc_paged_cache()
    for name, _ in st._fields_:
        if name != "n_pages":
            setattr(st, name, getattr(cache.struct, name))
    st.k_bf16, st.v_bf16 = anchors["k"].data_ptr(), anchors["v"].data_ptr()
    st.n_pages[0], st.n_pages[1], st.n_pages[2] = n, cache.struct.n_pages[1], cache.struct.n_pages[2]
    bt_d = cache.block_table.clone()
    tags = torch.full((B, max_pages), K.KVC_FMT_TERNARY2, dtype=torch.uint8, device=dev)
    seq = torch.tensor([r[0] for r in reqs], dtype=torch.int32, device=dev)
    page = torch.tensor([r[1] for r in reqs], dtype=torch.int32, device=dev)
    slot = torch.arange(n, dtype=torch.int32, device=dev)
    freed = torch.full((n,), -5, dtype=torch.int32, device=dev)
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    K.kvc_promote_pages(st, bt_d, tags, c["inp"]["context_lens"], seq, page, slot, n, freed, flags, B, hkv, D, P,
                        max_pages, cfg["sink"], cfg["window"], K.KVC_FMT_BF16, K.KVC_FMT_BF16)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    bt2, tags2, fr = bt_d.cpu().numpy(), tags.cpu().numpy(), freed.cpu().numpy()
    for i, (b, j) in enumerate(reqs):
        assert fr[i] == bt[b, j] and bt2[b, j] == i and tags2[b, j] == K.KVC_FMT_BF16
    moved = np.zeros_like(bt, dtype=bool)
    for b, j in reqs:
        moved[b, j] = True
    assert np.array_equal(bt2[~moved], bt[~moved])
    for (r, which), want in expect.items():
        assert np.array_equal(bits(anchors[which][r]), want), (r, which)
