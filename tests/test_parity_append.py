"""kvc_append_retier (one decode step's cache update: append one token per
sequence, move the page that leaves the high-precision window to the
ternary pool) against the oracle, through the C ABI.

Bar: block table, freed slots and high-precision pages (BF16 bits, FP8
bytes and scales) bit-exact; the retiered ternary pages by the codec rule
(bit-exact outside the gamma/2 threshold band, gamma within 1e-6)."""

import numpy as np
import pytest
import torch

import oracle as O
import compressed_decode_attention_kvc_b200 as K
from kvc_testlib import (HP, assert_attention_close, bits, check_ternary, from_bits, run_decode,
                         upload_oracle_cache)

pytestmark = pytest.mark.gpu


def _pages_up_to(rng, B, max_pages, hkv, d, upto):
    x = rng.standard_normal((B, max_pages, hkv, O.PAGE_SIZE, d)).astype(np.float32)
    tok = np.arange(max_pages)[:, None] * O.PAGE_SIZE + np.arange(O.PAGE_SIZE)[None, :]
    for b in range(B):
        x[b][(tok >= upto[b])[:, None, :, None].repeat(hkv, 1).repeat(d, 3)] = 0.0
    return torch.tensor(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _grow(cache, hp, n_hp, n_t, hkv, d):
    """Room for the new pages and retiered pages; new slots hold junk."""
    P = O.PAGE_SIZE
    if hp == O.BF16:
        for w in ("k", "v"):
            a = getattr(cache, w + "_bf16")
            setattr(cache, w + "_bf16", np.concatenate([a, np.full((n_hp, hkv, P, d), 0x7FC0, np.uint16)]))
    else:
        for w in ("k", "v"):
            a = getattr(cache, w + "_fp8")
            setattr(cache, w + "_fp8", np.concatenate([a, np.full((n_hp, hkv, P, d), 0x55, np.uint8)]))
            s = getattr(cache, w + "_fp8_scale")
            setattr(cache, w + "_fp8_scale", np.concatenate([s, np.full(n_hp, 3.0, np.float32)]))
    for w in ("k", "v"):
        a = getattr(cache, w + "_tern")
        setattr(cache, w + "_tern", np.concatenate([a, np.full((n_t, hkv, P, d // 4), 0xAA, np.uint8)]))
        g = getattr(cache, w + "_gamma")
        setattr(cache, w + "_gamma", np.concatenate([g, np.full((n_t, hkv), -1.0, np.float32)]))


def _state(t, hp):
    name = "bf16" if hp == O.BF16 else "fp8"
    out = {w: t[f"{w}_{name}"].cpu() for w in ("k", "v")}
    if hp != O.BF16:
        out.update({w + "s": t[f"{w}_fp8_scale"].cpu().numpy() for w in ("k", "v")})
    out.update({w + "t": t[f"{w}_tern"].cpu().numpy() for w in ("k", "v")})
    out.update({w + "g": t[f"{w}_gamma"].cpu().numpy() for w in ("k", "v")})
    return out


@pytest.mark.parametrize("d,hkv,hp_name", [(64, 4, "bf16"), (128, 2, "fp8"), (128, 8, "bf16"), (256, 4, "fp8")])
def test_append_retier_matches_oracle(cuda_device, d, hkv, hp_name):
    hp_lib = HP[hp_name]
    hp = O.BF16 if hp_name == "bf16" else O.FP8_E4M3
    rng = np.random.default_rng(d * 10 + hkv)
    B, max_pages, sink, window = 6, 12, 4, 40
    lens = np.array([71, 64, 31, 87, 20, 135], dtype=np.int32)
    assert [O.leaving_page(int(L), sink, window) for L in lens] == [1, -1, -1, 2, -1, 5]
    k = _pages_up_to(rng, B, max_pages, hkv, d, lens)
    v = _pages_up_to(rng, B, max_pages, hkv, d, lens)
    cache, bt, fmt = O.build_paged_cache(k, v, lens, sink, window, hp)
    n_hp = (cache.k_bf16 if hp == O.BF16 else cache.k_fp8).shape[0]
    n_t = cache.k_tern.shape[0]
    _grow(cache, hp, B, B, hkv, d)
    for b, L in enumerate(lens):
        if L % 16 == 0:
            bt[b, L // 16] = n_hp + b
    tern_slot = (n_t + np.arange(B)).astype(np.int32)
    kn = _pages_up_to(rng, B, 1, hkv, d, [16] * B)[:, 0, :, 0]        # [B][Hkv][D]
    vn = _pages_up_to(rng, B, 1, hkv, d, [16] * B)[:, 0, :, 0]
    c_ref, bt_ref, freed_ref, _ = O.append_retier(cache, bt, lens, kn, vn, tern_slot, sink, window, hp)

    t, struct = upload_oracle_cache(cache, cuda_device)
    bt_d = torch.from_numpy(bt.copy()).to(cuda_device)
    freed = torch.full((B,), 12345, dtype=torch.int32, device=cuda_device)
    flags = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    K.kvc_append_retier(from_bits(kn, cuda_device), from_bits(vn, cuda_device), struct, bt_d, None,
                        torch.from_numpy(lens).to(cuda_device), torch.from_numpy(tern_slot).to(cuda_device),
                        freed, flags, B, hkv, d, K.PAGE_SIZE, max_pages, sink, window, hp_lib)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    assert np.array_equal(freed.cpu().numpy(), freed_ref)
    assert np.array_equal(bt_d.cpu().numpy(), bt_ref)
    got = _state(t, hp)
    if hp == O.BF16:
        assert np.array_equal(bits(got["k"]), c_ref.k_bf16) and np.array_equal(bits(got["v"]), c_ref.v_bf16)
    else:
        assert np.array_equal(got["k"].numpy(), c_ref.k_fp8) and np.array_equal(got["v"].numpy(), c_ref.v_fp8)
        assert np.array_equal(got["ks"], c_ref.k_fp8_scale) and np.array_equal(got["vs"], c_ref.v_fp8_scale)
    for w in ("k", "v"):
        codes, gam = got[w + "t"], got[w + "g"]
        untouched = [s for s in range(codes.shape[0]) if s < n_t or s - n_t not in np.where(freed_ref >= 0)[0]]
        assert np.array_equal(codes[untouched], getattr(cache, w + "_tern")[untouched])
        assert np.array_equal(gam[untouched], getattr(cache, w + "_gamma")[untouched])
        for b in np.where(freed_ref >= 0)[0]:
            phys, ts = int(freed_ref[b]), int(tern_slot[b])
            if hp == O.BF16:
                src = getattr(cache, w + "_bf16")[phys:phys + 1]
            else:
                src = O.dequantize_fp8(getattr(cache, w + "_fp8")[phys:phys + 1],
                                       getattr(cache, w + "_fp8_scale")[phys:phys + 1])
            check_ternary(codes[ts:ts + 1], gam[ts:ts + 1], src)


def test_append_retier_steps_then_decode(cuda_device):
    """Forty steps of append + retier on the GPU and in the oracle (fresh
    slots handed out as pages start and leave), states compared after every
    step, then decode attention over each side's final cache."""
    rng = np.random.default_rng(77)
    B, hkv, d, hq, max_pages, sink, window = 3, 2, 64, 8, 10, 4, 24
    hp_lib, hp = K.KVC_FMT_BF16, O.BF16
    lens = np.array([30, 44, 16], dtype=np.int32)
    k = _pages_up_to(rng, B, max_pages, hkv, d, lens)
    v = _pages_up_to(rng, B, max_pages, hkv, d, lens)
    cache, bt, fmt = O.build_paged_cache(k, v, lens, sink, window, hp)
    steps = 40
    n_hp, n_t = cache.k_bf16.shape[0], cache.k_tern.shape[0]
    _grow(cache, hp, B * 4, B * 4, hkv, d)
    t, struct = upload_oracle_cache(cache, cuda_device)
    bt_d = torch.from_numpy(bt.copy()).to(cuda_device)
    next_hp, next_t = n_hp, n_t
    free_hp = []
    freed = torch.empty(B, dtype=torch.int32, device=cuda_device)
    flags = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    for step in range(steps):
        for b, L in enumerate(lens):
            if L % 16 == 0:
                slot = free_hp.pop(0) if free_hp else next_hp
                if slot == next_hp:
                    next_hp += 1
                bt[b, L // 16] = slot
        bt_d.copy_(torch.from_numpy(bt))
        tern_slot = np.full(B, -1, np.int32)
        for b, L in enumerate(lens):
            if O.leaving_page(int(L), sink, window) >= 0:
                tern_slot[b] = next_t
                next_t += 1
        kn = _pages_up_to(rng, B, 1, hkv, d, [16] * B)[:, 0, :, 0]
        vn = _pages_up_to(rng, B, 1, hkv, d, [16] * B)[:, 0, :, 0]
        cache, bt, freed_ref, _ = O.append_retier(cache, bt, lens, kn, vn, tern_slot, sink, window, hp)
        K.kvc_append_retier(from_bits(kn, cuda_device), from_bits(vn, cuda_device), struct, bt_d, None,
                            torch.from_numpy(lens).to(cuda_device), torch.from_numpy(tern_slot).to(cuda_device),
                            freed, flags, B, hkv, d, K.PAGE_SIZE, max_pages, sink, window, hp_lib)
        torch.cuda.synchronize()
        assert np.array_equal(freed.cpu().numpy(), freed_ref), step
        assert np.array_equal(bt_d.cpu().numpy(), bt), step
        assert np.array_equal(bits(t["k_bf16"].cpu()), cache.k_bf16), step
        free_hp += [int(f) for f in freed_ref if f >= 0]
        lens = lens + 1
    assert int(flags.item()) == 0
    assert next_hp <= n_hp + B * 4 and next_t <= n_t + B * 4
    # the retiered pages: codec rule against the oracle's own retier output
    got_codes, got_gamma = t["k_tern"].cpu().numpy(), t["k_gamma"].cpu().numpy()
    assert np.array_equal(got_gamma[:n_t], cache.k_gamma[:n_t])
    # decode over each side's cache: both follow the same formats
    fmt = np.full((B, max_pages), 255, np.uint8)
    for b in range(B):
        for j in range(O.num_pages(int(lens[b]))):
            fmt[b, j] = O.page_format(j, int(lens[b]), sink, window, O.BF16, O.TERNARY)
    q = torch.randn(B, hq, d).to(torch.bfloat16)
    ref = O.decode_attention(bits(q), cache, bt, fmt, lens, hkv)
    out, _ = run_decode(q.to(cuda_device), struct, bt_d, None, torch.from_numpy(lens).to(cuda_device),
                        hkv, max_pages, sink, window, hp_lib)
    torch.cuda.synchronize()
    assert_attention_close(out.cpu().numpy(), ref, "decode after 40 append steps")
