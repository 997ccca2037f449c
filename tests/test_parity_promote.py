"""kvc_promote_pages (stale-to-anchor promotion: re-expand ternary pages into
BF16 or FP8 anchors) against the oracle, through the C ABI.

Bar: block table, tags, freed slots, flags and anchor pools (BF16 bits, FP8
bytes and scales) bit-exact -- both sides take the same float32 steps on
the same packed bytes and gammas; the ternary pools untouched; decode over
the promoted cache within the attention tolerance."""

import numpy as np
import pytest
import torch

import oracle as O
import compressed_decode_attention_kvc_b200 as K
from kvc_testlib import HP, assert_attention_close, bits, run_decode, upload_oracle_cache

pytestmark = pytest.mark.gpu

ANCHOR = {"bf16": (O.BF16, K.KVC_FMT_BF16), "fp8": (O.FP8_E4M3, K.KVC_FMT_FP8_E4M3)}


def _inputs(rng, B, max_pages, hkv, d, lens):
    """bf16 bits [B][max_pages][Hkv][P][D]: N(0,1) with 2% of the (head, dim)
    channels x10; every fourth (page, head) group all zero, so that some
    anchor pages have heads that add nothing to the FP8 amax."""
    x = rng.standard_normal((B, max_pages, hkv, O.PAGE_SIZE, d)).astype(np.float32)
    ch = rng.random((hkv, d)) < 0.02
    x[:, :, ch[:, None, :].repeat(O.PAGE_SIZE, 1)] *= 10.0
    x.reshape(-1, O.PAGE_SIZE, d)[::4] = 0.0
    return torch.tensor(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _grow_anchor(cache, anchor, n, hkv, d):
    P = O.PAGE_SIZE
    if anchor == O.BF16:
        for w in ("k", "v"):
            a = getattr(cache, w + "_bf16")
            setattr(cache, w + "_bf16", np.concatenate([a, np.full((n, hkv, P, d), 0x7FC0, np.uint16)]))
    else:
        for w in ("k", "v"):
            a = getattr(cache, w + "_fp8")
            setattr(cache, w + "_fp8", np.concatenate([a, np.full((n, hkv, P, d), 0x55, np.uint8)]))
            s = getattr(cache, w + "_fp8_scale")
            setattr(cache, w + "_fp8_scale", np.concatenate([s, np.full(n, 3.0, np.float32)]))


def _setup(rng, d, hkv, hp, anchor, B=5, max_pages=14, sink=4, window=40):
    lens = np.array([16 * 14, 16 * 9 + 5, 16 * 3, 16 * 12 + 1, 16 * 7], dtype=np.int32)[:B]
    k = _inputs(rng, B, max_pages, hkv, d, lens)
    v = _inputs(rng, B, max_pages, hkv, d, lens)
    tags = np.where(rng.random((B, max_pages)) < 0.15, anchor, O.TERNARY).astype(np.uint8)
    cache, bt, fmt = O.build_paged_cache(k, v, lens, sink, window, hp, older_fmt=tags)
    stale = [(b, j) for b in range(B) for j in range(max_pages) if fmt[b, j] == O.TERNARY]
    return lens, tags, cache, bt, fmt, stale


def _upload_tables(bt, tags, lens, dev):
    return (torch.from_numpy(bt.copy()).to(dev), torch.from_numpy(tags.copy()).to(dev),
            torch.from_numpy(lens).to(dev))


def _promote_gpu(struct, bt_d, tags_d, lens_d, reqs, slots, B, hkv, d, max_pages, sink, window, hp_lib,
                 anchor_lib, dev):
    n = len(reqs)
    seq = torch.tensor([r[0] for r in reqs], dtype=torch.int32, device=dev)
    page = torch.tensor([r[1] for r in reqs], dtype=torch.int32, device=dev)
    slot = torch.tensor(slots, dtype=torch.int32, device=dev)
    freed = torch.full((n,), 12345, dtype=torch.int32, device=dev)
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    K.kvc_promote_pages(struct, bt_d, tags_d, lens_d, seq, page, slot, n, freed, flags, B, hkv, d,
                        K.PAGE_SIZE, max_pages, sink, window, hp_lib, anchor_lib)
    torch.cuda.synchronize()
    return freed.cpu().numpy(), int(flags.item())


@pytest.mark.parametrize("d,hkv,hp_name,anchor_name", [
    (64, 4, "bf16", "bf16"), (128, 2, "fp8", "fp8"), (128, 8, "bf16", "fp8"), (256, 4, "fp8", "bf16"),
    (256, 1, "bf16", "fp8")])
def test_promote_matches_oracle(cuda_device, d, hkv, hp_name, anchor_name):
    hp_lib = HP[hp_name]
    hp = O.BF16 if hp_name == "bf16" else O.FP8_E4M3
    anchor, anchor_lib = ANCHOR[anchor_name]
    rng = np.random.default_rng(d + 7 * hkv)
    B, max_pages, sink, window = 5, 14, 4, 40
    lens, tags, cache, bt, fmt, stale = _setup(rng, d, hkv, hp, anchor)
    pick = [stale[i] for i in rng.choice(len(stale), size=min(12, len(stale)), replace=False)]
    n_anchor = (cache.k_bf16 if anchor == O.BF16 else cache.k_fp8).shape[0]
    _grow_anchor(cache, anchor, len(pick) + 2, hkv, d)
    slots = list(n_anchor + rng.permutation(len(pick) + 2)[:len(pick)])
    # requests the kernel must skip: a sink page, a window page, an out-of-range
    # page, an out-of-range sequence, a slot past the pool
    bad = [(0, 0), (0, 13), (2, 3), (B, 1), pick[0]]
    bad_slots = [n_anchor, n_anchor, n_anchor, n_anchor, n_anchor + len(pick) + 2]
    reqs, req_slots = pick[1:] + bad, slots[1:] + bad_slots
    c_ref, bt_ref, tags_ref, freed_ref, flags_ref = O.promote_pages(
        cache, bt, tags, lens, [r[0] for r in reqs], [r[1] for r in reqs], req_slots, sink, window, hp, anchor)
    assert flags_ref == O.PROMOTE_SLOT | O.PROMOTE_NOT_STALE | O.PROMOTE_RANGE
    assert (freed_ref[:len(pick) - 1] >= 0).all() and (freed_ref[len(pick) - 1:] == -1).all()
    t, struct = upload_oracle_cache(cache, cuda_device)
    bt_d, tags_d, lens_d = _upload_tables(bt, tags, lens, cuda_device)
    freed, flags = _promote_gpu(struct, bt_d, tags_d, lens_d, reqs, req_slots, B, hkv, d, max_pages, sink,
                                window, hp_lib, anchor_lib, cuda_device)
    assert flags == flags_ref
    assert np.array_equal(freed, freed_ref)
    assert np.array_equal(bt_d.cpu().numpy(), bt_ref) and np.array_equal(tags_d.cpu().numpy(), tags_ref)
    for w in ("k", "v"):
        if anchor == O.BF16:
            assert np.array_equal(bits(t[w + "_bf16"].cpu()), getattr(c_ref, w + "_bf16"))
        else:
            assert np.array_equal(t[w + "_fp8"].cpu().numpy(), getattr(c_ref, w + "_fp8"))
            assert np.array_equal(t[w + "_fp8_scale"].cpu().numpy(), getattr(c_ref, w + "_fp8_scale"))
        assert np.array_equal(t[w + "_tern"].cpu().numpy(), getattr(cache, w + "_tern"))
        assert np.array_equal(t[w + "_gamma"].cpu().numpy(), getattr(cache, w + "_gamma"))


@pytest.mark.parametrize("anchor_name", ["bf16", "fp8"])
def test_promote_then_decode(cuda_device, anchor_name):
    """Promote a third of the stale pages, then decode over the promoted
    cache on both sides (the tags now route those pages to the anchor
    format)."""
    anchor, anchor_lib = ANCHOR[anchor_name]
    rng = np.random.default_rng(5 if anchor == O.BF16 else 6)
    d, hkv, hq, max_pages, sink, window = 128, 4, 16, 14, 4, 40
    hp, hp_lib = O.FP8_E4M3, K.KVC_FMT_FP8_E4M3
    lens, tags, cache, bt, fmt, stale = _setup(rng, d, hkv, hp, anchor)
    pick = stale[::3]
    n_anchor = (cache.k_bf16 if anchor == O.BF16 else cache.k_fp8).shape[0]
    _grow_anchor(cache, anchor, len(pick), hkv, d)
    slots = [n_anchor + i for i in range(len(pick))]
    c_ref, bt_ref, tags_ref, freed_ref, flags_ref = O.promote_pages(
        cache, bt, tags, lens, [r[0] for r in pick], [r[1] for r in pick], slots, sink, window, hp, anchor)
    assert flags_ref == 0
    t, struct = upload_oracle_cache(cache, cuda_device)
    bt_d, tags_d, lens_d = _upload_tables(bt, tags, lens, cuda_device)
    freed, flags = _promote_gpu(struct, bt_d, tags_d, lens_d, pick, slots, len(lens), hkv, d, max_pages, sink,
                                window, hp_lib, anchor_lib, cuda_device)
    assert flags == 0 and np.array_equal(freed, freed_ref)
    B = len(lens)
    fmt2 = np.full((B, max_pages), 255, np.uint8)
    for b in range(B):
        for j in range(O.num_pages(int(lens[b]))):
            fmt2[b, j] = O.page_format(j, int(lens[b]), sink, window, hp, int(tags_ref[b, j]))
    assert sum(int(fmt2[b, j] == anchor) for b, j in pick) == len(pick)
    q = (torch.randn(B, hq, d) * 2).to(torch.bfloat16)
    ref = O.decode_attention(bits(q), c_ref, bt_ref, fmt2, lens, hkv)
    older_d = tags_d
    out, _ = run_decode(q.to(cuda_device), struct, bt_d, older_d, lens_d, hkv, max_pages, sink, window, hp_lib)
    torch.cuda.synchronize()
    assert_attention_close(out.cpu().numpy(), ref, f"decode after promotion to {anchor_name}")
