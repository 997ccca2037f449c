"""Pins of the oracle against facts fixed outside it: figures printed on the
pages (tests/golden/page_figures.json), hand-derived encodings of the
formats, library routines (torch's bf16 and float8_e4m3fn conversions and
scaled_dot_product_attention), closed forms and brute force on tiny inputs.
Each pin is chosen so that a plausible slip in the oracle (a wrong bit order,
a dropped term, a transposed operand, an off-by-one page, a wrong GQA index)
fails at least one of them.  CPU only."""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(vals):
    t = torch.tensor(np.asarray(vals, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------- bf16 helpers

def test_bf16_conversions_match_torch():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(20000).astype(np.float32) * np.float32(3.0)
    # exact ties: low half 0x8000, both parities of the kept LSB
    u = rng.integers(0, 2**31, 2000, dtype=np.uint64).astype(np.uint32)
    ties = ((u & np.uint32(0x7F7F0000)) | np.uint32(0x8000)).view(np.float32)
    x = np.concatenate([x, ties, -ties, np.float32([0.0, -0.0, 1e-40, -1e-40])])
    ours = O.f32_to_bf16_rne(x)
    ref = torch.tensor(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = O.bf16_to_f64(ref)
    assert np.array_equal(back, torch.tensor(x).to(torch.bfloat16).double().numpy())


# ------------------------------------------------------------------ packing

def test_pack_literal_bytes():
    # 00 -> 0, 01 -> +1, 11 -> -1, element i at bits 2*(i % 4) of byte i // 4
    cases = {
        (1, 0, 0, 0): 0x01, (-1, 0, 0, 0): 0x03, (0, 1, 0, 0): 0x04,
        (0, 0, 0, -1): 0xC0, (-1, -1, -1, -1): 0xFF, (1, 1, 1, 1): 0x55,
        (1, -1, 0, 1): 0x4D, (0, 0, 0, 0): 0x00, (0, 0, 1, 0): 0x10,
    }
    for codes, byte in cases.items():
        assert O.pack_ternary(np.array(codes, np.int8))[0] == byte, codes


def test_pack_roundtrip_exhaustive_and_no_field_10():
    combos = np.array(list(itertools.product((-1, 0, 1), repeat=4)), dtype=np.int8)
    assert len(combos) == 81
    packed = O.pack_ternary(combos)                      # [81][1]
    assert packed.shape == (81, 1)
    assert len(set(packed[:, 0].tolist())) == 81          # injective
    for b in packed[:, 0]:
        for j in range(4):
            assert (int(b) >> (2 * j)) & 3 != 0b10
    assert np.array_equal(O.unpack_ternary(packed), combos)


def test_unpack_rejects_field_10():
    with pytest.raises(ValueError):
        O.unpack_ternary(np.array([0x02], np.uint8))
    with pytest.raises(ValueError):
        O.pack_ternary(np.array([2, 0, 0, 0], np.int8))


def test_group_element_order_row_major():
    P, D = 16, 64
    for (t, d) in [(0, 0), (0, 5), (3, 17), (15, 63)]:
        x = np.zeros((1, 1, P, D), np.float32)
        x[0, 0, t, d] = 1.0
        codes, gamma = O.quantize_pack_ternary(bf16_bits(x))
        flat = codes.reshape(-1)
        i = t * D + d
        nz = np.nonzero(flat)[0]
        assert list(nz) == [i // 4]
        assert flat[i // 4] == 1 << (2 * (i % 4))
        assert gamma[0, 0] == np.float32(1.0 / (P * D))


def test_storage_figures_vantage():
    fig = json.load(open(os.path.join(GOLDEN, "page_figures.json")))
    P = 16
    for D in (64, 128, 256):
        codes, _ = O.quantize_pack_ternary(bf16_bits(np.ones((1, 1, P, D))))
        assert codes.nbytes * 8 / (P * D) == fig["ternary_bits_per_element"]["value"]
    # one fp32 gamma per 16 x 256 group: 16 / 2.0078 -> 7.97x (as printed)
    r = 16.0 / O.ternary_bits_per_element(P, 256)
    assert round(r, fig["ternary_reduction_vs_fp16"]["decimals"]) == fig["ternary_reduction_vs_fp16"]["value"]
    assert O.ternary_group_bytes(16, 128) == 516


def test_storage_figures_minima():
    fig = json.load(open(os.path.join(GOLDEN, "page_figures.json")))
    f = fig["minima_bf16_kib_per_token"]
    bf = O.kv_bytes_per_token(f["layers"], f["n_kv_heads"], f["head_dim"], 2)
    f8 = O.kv_bytes_per_token(f["layers"], f["n_kv_heads"], f["head_dim"], 1)
    assert bf == f["value"] * 1024
    assert f8 == fig["minima_fp8_kib_per_token"]["value"] * 1024
    g = fig["minima_gib_at_32k"]
    assert bf * g["tokens"] / 2**30 == g["bf16"] and f8 * g["tokens"] / 2**30 == g["fp8"]
    dep = fig["minima_deployed"]
    assert round(bf / 1024 / dep["kib_per_token"], dep["decimals"]) == dep["reduction_vs_bf16"]
    assert round(f8 / 1024 / dep["kib_per_token"], dep["decimals"]) == dep["reduction_vs_fp8"]
    m = fig["minima_gib_per_million_tokens"]
    assert round(bf * 1e6 / 2**30, m["decimals"]) == m["bf16"]
    assert round(f8 * 1e6 / 2**30, m["decimals"]) == m["fp8"]
    assert round(dep["kib_per_token"] * 1024 * 1e6 / 2**30, m["decimals"]) == m["deployed"]


# ------------------------------------------------------------- gamma, codes

def test_gamma_closed_forms():
    rng = np.random.default_rng(1)
    P, D = 16, 128
    signs = rng.choice([-1.0, 1.0], size=(P, D))
    assert O.ternary_gamma(O.bf16_to_f64(bf16_bits(0.375 * signs))) == np.float32(0.375)
    two = np.where(rng.random((P, D)) < 0.5, 1.5, 0.25)
    two[0, 0], two[0, 1] = 1.5, 0.25
    k = (two == 1.5).sum()
    expect = (1.5 * k + 0.25 * (P * D - k)) / (P * D)
    assert O.ternary_gamma(two) == np.float32(expect)
    assert O.ternary_gamma(np.zeros((P, D))) == 0.0
    x = O.bf16_to_f64(bf16_bits(rng.standard_normal((P, D))))
    assert O.ternary_gamma(4.0 * x) == 4.0 * O.ternary_gamma(x)          # exact scaling
    assert O.ternary_gamma(x[::-1, ::-1]) == O.ternary_gamma(x)           # order-free


def test_gamma_is_per_page_and_head():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((3, 2, 16, 64)).astype(np.float32)
    x[:, 1] = 4.0 * x[:, 0]
    x[2] *= 0.5
    codes, gamma = O.quantize_pack_ternary(bf16_bits(x))
    assert np.array_equal(gamma[:, 1], 4.0 * gamma[:, 0])
    assert np.array_equal(codes[:, 1], codes[:, 0])
    xb = O.bf16_to_f64(bf16_bits(x))
    for p in range(3):
        for h in range(2):
            assert gamma[p, h] == np.float32(np.abs(xb[p, h]).mean())
    # page selection and order
    c2, g2 = O.quantize_pack_ternary(bf16_bits(x), page_ids=[2, 0])
    assert np.array_equal(c2, codes[[2, 0]]) and np.array_equal(g2, gamma[[2, 0]])


def test_codes_equal_literal_roundclip():
    rng = np.random.default_rng(3)
    for dist in ("normal", "laplace", "outlier"):
        x = rng.standard_normal((16, 128))
        if dist == "laplace":
            x = rng.laplace(size=(16, 128))
        if dist == "outlier":
            x[:, :3] *= 10
        x = O.bf16_to_f64(bf16_bits(x))
        g = O.ternary_gamma(x)
        c = O.ternary_codes(x, g)
        literal = np.clip(np.round(x / float(g)), -1, 1)   # RoundClip, half-to-even
        assert np.array_equal(c, literal.astype(np.int8))
        assert set(np.unique(c).tolist()) <= {-1, 0, 1}


def test_codes_at_threshold_ties():
    # gamma = 1 exactly: half the group 1.5, half 0.5; threshold 0.5
    P, D = 16, 64
    x = np.full((P, D), 1.5)
    x[:, D // 2:] = 0.5
    x[0, 0], x[0, D // 2] = 1.49609375, 0.50390625   # sum unchanged; bf16 neighbours
    x[1, 0], x[1, D // 2] = -1.5, -0.5
    g = O.ternary_gamma(x)
    assert g == np.float32(1.0)
    c = O.ternary_codes(x, g)
    assert c[0, D // 2] == 1          # just above the threshold
    assert c[2, D // 2] == 0          # exactly at gamma / 2 -> tie -> 0
    assert c[1, D // 2] == 0 and c[1, 0] == -1
    assert c[2, 0] == 1


def test_zero_group():
    codes, gamma = O.quantize_pack_ternary(bf16_bits(np.zeros((1, 1, 16, 64))))
    assert gamma[0, 0] == 0 and not codes.any()


# ------------------------------------------------------------------- FP8

def test_e4m3_known_codes():
    # hand-derived from the OCP 8-bit floating point definition (E4M3: bias 7,
    # max normal 448 = S.1111.110, min normal 2^-6, min subnormal 2^-9)
    cases = [
        (1.0, 0x38), (448.0, 0x7E), (-2.0, 0xC0), (0.5, 0x30), (2.0**-9, 0x01),
        (2.0**-6, 0x08), (7 / 8 * 2.0**-6, 0x07), (1.125, 0x39),
        (1.0625, 0x38),            # tie between 1.0 (even) and 1.125
        (1.1875, 0x3A),            # tie between 1.125 and 1.25 (even)
        (3 * 2.0**-10, 0x02),      # tie between 2^-9 and 2^-8 (even)
        (2.0**-10, 0x00),          # tie between 0 (even) and 2^-9
        (2.0**-10 * 1.0001, 0x01),
        (-(2.0**-11), 0x80),       # negative underflow keeps its sign
        (500.0, 0x7E), (-1e6, 0xFE), (464.0, 0x7E), (240.0, 0x77), (-0.0, 0x80),
    ]
    for v, code in cases:
        got = O.f32_to_e4m3_rne_satfinite(np.float32([v]))[0]
        assert got == code, (v, hex(got), hex(code))
    assert np.array_equal(O.e4m3_to_f64(np.uint8([0x38, 0x7E, 0xC0, 0x01, 0x08])),
                          [1.0, 448.0, -2.0, 2.0**-9, 2.0**-6])


def test_e4m3_matches_torch_on_every_bf16():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):          # the NaN bit patterns
        x = O.bf16_to_f64(bits).astype(np.float32)
    ok = np.isfinite(x) & (np.abs(x) <= 448.0)
    ours = O.f32_to_e4m3_rne_satfinite(x[ok])
    ref = torch.tensor(x[ok]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)
    big = np.isfinite(x) & (np.abs(x) > 448.0)
    sat = O.f32_to_e4m3_rne_satfinite(x[big])
    assert np.all((sat & 0x7F) == 0x7E)


def test_e4m3_decode_matches_torch():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    ref = torch.tensor(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(O.e4m3_to_f64(codes), ref)
    assert np.array_equal(O.f32_to_e4m3_rne_satfinite(O.e4m3_to_f64(codes).astype(np.float32)), codes)


def test_fp8_page_scale():
    x = np.zeros((1, 2, 16, 64), np.float32)
    x[0, 0, 0, 0], x[0, 1, 5, 7] = 1.0, -8.0          # amax over all heads = 8
    q, s = O.quantize_fp8_pages(bf16_bits(x))
    assert s[0] == np.float32(8.0 / 448.0)
    assert q[0, 1, 5, 7] == 0xFE                       # -8 * (448/8) = -448
    assert q[0, 0, 0, 0] == O.f32_to_e4m3_rne_satfinite(np.float32([np.float32(1.0) * np.float32(448.0 / 8.0)]))[0]
    q0, s0 = O.quantize_fp8_pages(bf16_bits(np.zeros((1, 1, 16, 64))))
    assert s0[0] == 1.0 and not q0.any()


# ------------------------------------------------------------- dequantise

def test_dequantize_ternary_closed_form():
    codes = O.pack_ternary(np.array([[1, 0, -1, 1] * 16] * 16, np.int8)).reshape(1, 1, 16, 16)
    for g in (0.75, 1.0 / 3.0):
        out = O.dequantize_ternary(codes, np.float32([[g]]))
        row = np.array([g, 0.0, -g, g] * 16, np.float32)
        assert np.array_equal(out[0, 0, 0], bf16_bits(row))


def test_dequantize_fp8_closed_form():
    e = np.zeros((1, 1, 16, 16), np.uint8)
    e[0, 0, 0, :4] = [0x38, 0xC0, 0x7E, 0x01]          # 1, -2, 448, 2^-9
    out = O.dequantize_fp8(e, np.float32([0.1]))
    s = np.float32(0.1)
    want = np.float32([s * np.float32(1), s * np.float32(-2), s * np.float32(448), s * np.float32(2.0**-9)])
    assert np.array_equal(out[0, 0, 0, :4], bf16_bits(want))


# -------------------------------------------------------------- attention

def test_softmax_weights_sum_to_one_and_simple_cases():
    rng = np.random.default_rng(4)
    for L in (1, 7, 300):
        q = rng.standard_normal(8)
        k = rng.standard_normal((L, 8)) * 3
        w = O.attention_full(q, k, np.eye(L), 0.5)        # V = I exposes the weights
        assert abs(w.sum() - 1.0) < 1e-12 and (w >= 0).all()
    v = rng.standard_normal((1, 8))
    assert np.allclose(O.attention_full(rng.standard_normal(8), rng.standard_normal((1, 8)), v, 1.0), v[0], rtol=0, atol=1e-15)
    vv = rng.standard_normal((50, 8))
    kc = np.tile(rng.standard_normal(8), (50, 1))
    assert np.allclose(O.attention_full(rng.standard_normal(8), kc, vv, 1.0), vv.mean(0), rtol=0, atol=1e-12)


def test_attention_matches_sdpa():
    rng = np.random.default_rng(5)
    for L, D in ((5, 4), (333, 64), (1000, 256)):
        q = rng.standard_normal(D)
        k = rng.standard_normal((L, D))
        v = rng.standard_normal((L, D))
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.tensor(q)[None, None, None], torch.tensor(k)[None, None], torch.tensor(v)[None, None])
        ours = O.attention_full(q, k, v, 1.0 / math.sqrt(D))
        assert np.abs(ours - ref.numpy().reshape(-1)).max() < 1e-12


def test_brute_force_tiny_long_double():
    rng = np.random.default_rng(6)
    for L in range(1, 9):
        q = rng.standard_normal(4)
        k = rng.standard_normal((L, 4))
        v = rng.standard_normal((L, 4))
        s = [np.longdouble(0.5) * sum(np.longdouble(q[d]) * np.longdouble(k[t, d]) for d in range(4)) for t in range(L)]
        e = [np.exp(x) for x in s]
        z = sum(e)
        want = [sum(e[t] * np.longdouble(v[t, d]) for t in range(L)) / z for d in range(4)]
        assert np.abs(O.attention_full(q, k, v, 0.5) - np.array(want, dtype=np.float64)).max() < 1e-13


def test_split_merge_equals_full():
    rng = np.random.default_rng(7)
    L, D = 997, 32
    q, k, v = rng.standard_normal(D), rng.standard_normal((L, D)) * 2, rng.standard_normal((L, D))
    full = O.attention_full(q, k, v, 0.3)
    for cuts in ([16], [1, 5, 400], [64 * i for i in range(1, 15)]):
        edges = [0] + cuts + [L]
        parts = [O.attention_partial(q, k[a:b], v[a:b], 0.3) for a, b in zip(edges, edges[1:])]
        assert np.abs(O.merge_partials(parts) - full).max() < 1e-12
        assert np.abs(O.merge_partials(parts[::-1]) - full).max() < 1e-12


# ------------------------------------------------------- page classification

def hp_pages(L, sink, window):
    return [j for j in range(O.num_pages(L)) if O.page_format(j, L, sink, window, O.BF16, O.TERNARY) == O.BF16]


def test_page_classification_hand_counts():
    assert hp_pages(512, 4, 64) == [0, 28, 29, 30, 31]
    assert hp_pages(4096, 4, 256) == [0] + list(range(240, 256))
    assert len(hp_pages(32768, 4, 1024)) == 65
    # ragged: L = 8200, window 2048 -> tokens 6152..8199 -> pages 384..512
    assert hp_pages(8200, 4, 2048) == [0] + list(range(384, 513))
    assert hp_pages(100, 0, 1) == [6]                  # only the (partial) last page
    assert hp_pages(100, 17, 0) == [0, 1]              # sink spans two pages, no window
    assert hp_pages(100, 0, 0) == []
    assert hp_pages(100, 0, 500) == list(range(7))     # window longer than the context


# ----------------------------------------------- decode over a hand-built cache

def _hand_cache(D=16, hkv=2):
    """Pools written directly from the encodings (no oracle quantiser): one
    ternary page whose token rows are all +1 (0x55 bytes) or all -1 (0xFF),
    one FP8 page of 1.0 (0x38) at scale s, one BF16 page of known values."""
    P = 16
    tern = np.zeros((1, hkv, P, D // 4), np.uint8)
    for t in range(P):
        tern[0, :, t, :] = 0x55 if t % 3 else 0xFF
    gam = np.float32([[1.0 / 3.0, 0.75]])
    fp8 = np.full((1, hkv, P, D), 0x38, np.uint8)
    fp8[0, 1] = 0xC0                                    # -2.0 on KV head 1
    s = np.float32([0.1])
    rng = np.random.default_rng(8)
    bfv = rng.standard_normal((1, hkv, P, D)).astype(np.float32)
    bfb = bf16_bits(bfv)
    cache = O.PagedCache(k_bf16=bfb, v_bf16=bfb[:, ::-1].copy(), k_fp8=fp8, v_fp8=fp8.copy(),
                         k_fp8_scale=s, v_fp8_scale=np.float32([0.5]), k_tern=tern,
                         v_tern=tern[:, :, ::-1].copy(), k_gamma=gam, v_gamma=gam[:, ::-1].copy())
    # expected dense values, written from the encodings above
    def dense(which, h):
        t_rows = np.array([1.0 if t % 3 else -1.0 for t in range(P)])
        if which == "v":
            t_rows = t_rows[::-1]
        g = float(gam[0, h]) if which == "k" else float(gam[0, ::-1][h])
        tern_d = g * np.repeat(t_rows[:, None], D, axis=1)
        f8v = (1.0 if h == 0 else -2.0) * float(s[0] if which == "k" else 0.5)
        f8_d = np.full((P, D), f8v)
        bf_d = O.bf16_to_f64(bfb[0, h] if which == "k" else bfb[0, ::-1][h])
        return tern_d, f8_d, bf_d
    return cache, dense


@pytest.mark.parametrize("order", [(O.TERNARY, O.FP8_E4M3, O.BF16), (O.BF16, O.TERNARY, O.FP8_E4M3)])
def test_decode_over_hand_built_cache_matches_sdpa(order):
    D, hkv, G = 16, 2, 2
    cache, dense = _hand_cache(D, hkv)
    L = 16 * 3 - 5                                     # ragged last page
    fmt = np.array([list(order) + [255]], np.uint8)
    bt = np.zeros((1, 4), np.int32)
    rng = np.random.default_rng(9)
    qf = rng.standard_normal((1, hkv * G, D)).astype(np.float32)
    qb = bf16_bits(qf)
    out = O.decode_attention(qb, cache, bt, fmt, [L], hkv)
    pos = {O.TERNARY: 0, O.FP8_E4M3: 1, O.BF16: 2}
    for h in range(hkv * G):
        g = h // G
        ks, vs = [], []
        for f in order:
            ks.append(dense("k", g)[pos[f]])
            vs.append(dense("v", g)[pos[f]])
        k = torch.tensor(np.concatenate(ks)[:L])
        v = torch.tensor(np.concatenate(vs)[:L])
        qq = torch.tensor(O.bf16_to_f64(qb[0, h]))
        ref = torch.nn.functional.scaled_dot_product_attention(qq[None, None, None], k[None, None], v[None, None])
        assert np.abs(out[0, h] - ref.numpy().reshape(-1)).max() < 1e-12


def test_decode_all_bf16_matches_sdpa_gqa_and_ignores_masked_slots():
    rng = np.random.default_rng(10)
    B, hq, hkv, D, L = 2, 6, 2, 32, 16 * 5 - 3
    maxp = 5
    k = rng.standard_normal((B, maxp, hkv, 16, D)).astype(np.float32)
    v = rng.standard_normal((B, maxp, hkv, 16, D)).astype(np.float32)
    q = rng.standard_normal((B, hq, D)).astype(np.float32)
    lens = [L, 16 * 2 + 1]
    kb, vb, qb = bf16_bits(k), bf16_bits(v), bf16_bits(q)
    cache, bt, fmt = O.build_paged_cache(kb, vb, lens, sink=0, window=10**6, hp_fmt=O.BF16)
    out = O.decode_attention(qb, cache, bt, fmt, lens, hkv)
    for b in range(B):
        Lb = lens[b]
        kk = torch.tensor(O.bf16_to_f64(kb[b]).transpose(1, 0, 2, 3).reshape(hkv, -1, D)[:, :Lb])
        vv = torch.tensor(O.bf16_to_f64(vb[b]).transpose(1, 0, 2, 3).reshape(hkv, -1, D)[:, :Lb])
        kk = kk.repeat_interleave(hq // hkv, dim=0)    # HF repeat_kv grouping
        vv = vv.repeat_interleave(hq // hkv, dim=0)
        qq = torch.tensor(O.bf16_to_f64(qb[b]))[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(qq[None], kk[None], vv[None])[0, :, 0]
        assert np.abs(out[b] - ref.numpy()).max() < 1e-12
    # garbage in the slots past each context length changes nothing
    k2, v2 = k.copy(), v.copy()
    k2[0, 4, :, 13:] = 1e4
    v2[0, 4, :, 13:] = -1e4
    k2[1, 2, :, 1:] = 7e3
    c2, bt2, f2 = O.build_paged_cache(bf16_bits(k2), bf16_bits(v2), lens, sink=0, window=10**6, hp_fmt=O.BF16)
    assert np.array_equal(O.decode_attention(qb, c2, bt2, f2, lens, hkv), out)


def test_physical_placement_is_invisible():
    rng = np.random.default_rng(11)
    B, hkv, D, maxp = 3, 2, 64, 12
    k = bf16_bits(rng.standard_normal((B, maxp, hkv, 16, D)))
    v = bf16_bits(rng.standard_normal((B, maxp, hkv, 16, D)))
    q = bf16_bits(rng.standard_normal((B, 4, D)))
    lens = [16 * 12, 16 * 9 + 4, 40]
    older = np.where(rng.random((B, maxp)) < 0.3, O.BF16, O.TERNARY).astype(np.uint8)
    c1, bt1, f1 = O.build_paged_cache(k, v, lens, 4, 20, O.FP8_E4M3, older_fmt=older)
    c2, bt2, f2 = O.build_paged_cache(k, v, lens, 4, 20, O.FP8_E4M3, older_fmt=older, slot_key=rng.random((B, maxp)))
    assert np.array_equal(f1, f2) and not np.array_equal(bt1, bt2)
    o1 = O.decode_attention(q, c1, bt1, f1, lens, hkv)
    o2 = O.decode_attention(q, c2, bt2, f2, lens, hkv)
    assert np.abs(o1 - o2).max() < 1e-13
    assert {O.BF16, O.FP8_E4M3, O.TERNARY} <= set(np.unique(f1).tolist())


# ------------------------------------------------------- append and retier

def _pages_up_to(rng, B, max_pages, hkv, d, upto):
    """bf16 bits [B][max_pages][Hkv][P][D]: N(0,1) for tokens < upto[b],
    zero after (a page that is being filled has zero rows past its end)."""
    x = rng.standard_normal((B, max_pages, hkv, O.PAGE_SIZE, d)).astype(np.float32)
    tok = (np.arange(max_pages)[:, None] * O.PAGE_SIZE + np.arange(O.PAGE_SIZE)[None, :])
    for b in range(B):
        x[b][(tok >= upto[b])[:, None, :, None].repeat(hkv, 1).repeat(d, 3)] = 0.0
    return bf16_bits(x)


def _decoded_logical(cache, bt, fmt, lens, hkv):
    out = {}
    for b in range(bt.shape[0]):
        for j in range(O.num_pages(int(lens[b]))):
            for h in range(hkv):
                for w in ("k", "v"):
                    out[(b, j, h, w)] = O.decoded_page_f64(cache, w, int(fmt[b, j]), int(bt[b, j]), h)
    return out


def test_leaving_page_matches_page_format():
    # the page that leaves is exactly the one whose format flips from hp to older
    for sink, window in [(4, 64), (4, 1024), (0, 16), (40, 33), (4, 1)]:
        for L in range(0, 400):
            before = [O.page_format(j, L, sink, window, O.BF16, O.TERNARY) for j in range(O.num_pages(L))]
            after = [O.page_format(j, L + 1, sink, window, O.BF16, O.TERNARY) for j in range(O.num_pages(L))]
            flips = [j for j in range(len(before)) if before[j] == O.BF16 and after[j] == O.TERNARY]
            j0 = O.leaving_page(L, sink, window)
            assert flips == ([j0] if j0 >= 0 else []), (sink, window, L)


def test_append_retier_bf16_equals_building_the_longer_cache():
    """Appending token L to a cache built for L tokens gives the same logical
    pages as building the cache for L + 1 tokens from scratch (BF16 window;
    retiered pages go through the same ternary codec on the same bf16 data)."""
    rng = np.random.default_rng(5)
    B, max_pages, hkv, d, sink, window = 5, 9, 2, 16, 4, 40
    # lengths hit a retier (L - window + 1 = 16k: L = 71, 87), a fresh page
    # (L % 16 == 0: L = 64) and neither
    lens = np.array([71, 64, 31, 87, 20], dtype=np.int32)
    assert [O.leaving_page(int(L), sink, window) for L in lens] == [1, -1, -1, 2, -1]
    k_full = _pages_up_to(rng, B, max_pages, hkv, d, lens + 1)
    v_full = _pages_up_to(rng, B, max_pages, hkv, d, lens + 1)
    k_old, v_old = k_full.copy(), v_full.copy()
    for b, L in enumerate(lens):                      # token L not yet in the cache
        k_old[b, L // 16, :, L % 16] = 0
        v_old[b, L // 16, :, L % 16] = 0
    cache, bt, fmt = O.build_paged_cache(k_old, v_old, lens, sink, window, O.BF16)
    # the caller provides the new page's hp slot and a ternary slot for the retier
    n_bf, n_t = cache.k_bf16.shape[0], cache.k_tern.shape[0]
    extra = 2 * B
    grow = lambda a, n: np.concatenate([a, np.zeros((n,) + a.shape[1:], a.dtype)])
    cache.k_bf16, cache.v_bf16 = grow(cache.k_bf16, extra), grow(cache.v_bf16, extra)
    cache.k_tern, cache.v_tern = grow(cache.k_tern, extra), grow(cache.v_tern, extra)
    cache.k_gamma, cache.v_gamma = grow(cache.k_gamma, extra), grow(cache.v_gamma, extra)
    cache.k_bf16[n_bf:] = 0x7FC0                      # stale NaN-looking slots must be zeroed
    cache.v_bf16[n_bf:] = 0x7FC0
    for b, L in enumerate(lens):
        if L % 16 == 0:
            bt[b, L // 16] = n_bf + b
    tern_slot = n_t + np.arange(B, dtype=np.int32)
    kn = np.stack([k_full[b, L // 16, :, L % 16] for b, L in enumerate(lens)])
    vn = np.stack([v_full[b, L // 16, :, L % 16] for b, L in enumerate(lens)])
    c2, bt2, freed, _ = O.append_retier(cache, bt, lens, kn, vn, tern_slot, sink, window, O.BF16)
    fmt2 = np.full_like(fmt, 255)
    for b in range(B):
        for j in range(O.num_pages(int(lens[b]) + 1)):
            fmt2[b, j] = O.page_format(j, int(lens[b]) + 1, sink, window, O.BF16, O.TERNARY)
    ref_cache, ref_bt, ref_fmt = O.build_paged_cache(k_full, v_full, lens + 1, sink, window, O.BF16)
    assert np.array_equal(fmt2, ref_fmt)
    got = _decoded_logical(c2, bt2, fmt2, lens + 1, hkv)
    ref = _decoded_logical(ref_cache, ref_bt, ref_fmt, lens + 1, hkv)
    assert got.keys() == ref.keys()
    for key in ref:
        assert np.array_equal(got[key], ref[key]), key
    for b, L in enumerate(lens):
        j0 = O.leaving_page(int(L), sink, window)
        assert freed[b] == (bt[b, j0] if j0 >= 0 else -1)
        if j0 >= 0:
            assert bt2[b, j0] == tern_slot[b]
    # the inputs are not modified
    assert np.array_equal(cache.k_bf16[n_bf:], np.full_like(cache.k_bf16[n_bf:], 0x7FC0))


def test_append_retier_fp8_rows_and_untouched_codes():
    """FP8 window: the new row decodes to the new values within e4m3 rounding,
    rows past it stay zero, and when the new row does not raise the page's
    amax the codes of the other rows are unchanged (re-encoding bf16(s*e)
    with the same scale returns e); a fresh page starts from zeros."""
    rng = np.random.default_rng(9)
    hkv, d, sink, window = 2, 32, 4, 64
    L = 37                                             # row 5 of page 2
    k = _pages_up_to(rng, 1, 4, hkv, d, [L])
    v = _pages_up_to(rng, 1, 4, hkv, d, [L])
    cache, bt, fmt = O.build_paged_cache(k, v, [L], sink, window, O.FP8_E4M3)
    phys = int(bt[0, 2])
    small = bf16_bits(0.25 * np.clip(rng.standard_normal((1, hkv, d)), -1, 1))   # below amax
    c2, bt2, freed, _ = O.append_retier(cache, bt, [L], small, small, [0], sink, window, O.FP8_E4M3)
    assert freed[0] == -1 and np.array_equal(bt2, bt)
    old, new = cache.k_fp8[phys], c2.k_fp8[phys]
    assert c2.k_fp8_scale[phys] == cache.k_fp8_scale[phys]
    rows = [r for r in range(16) if r != 5]
    assert np.array_equal(old[:, rows], new[:, rows])
    dec = c2.k_fp8_scale[phys] * O.e4m3_to_f64(new[:, 5])
    x = O.bf16_to_f64(small[0])
    assert np.all(np.abs(dec - x) <= np.abs(x) * 2.0 ** -4 + c2.k_fp8_scale[phys] * 2.0 ** -10)
    # a larger row raises amax and the scale
    big = bf16_bits(8.0 * np.ones((1, hkv, d)))
    c3, _, _, _ = O.append_retier(cache, bt, [L], big, big, [0], sink, window, O.FP8_E4M3)
    assert c3.v_fp8_scale[phys] == np.float32(8.0 / 448.0)
    assert np.all(O.e4m3_to_f64(c3.v_fp8[phys][:, 5]) == 448.0)
    # fresh page: everything but the new row is zero
    L2 = 48
    k2 = _pages_up_to(rng, 1, 4, hkv, d, [L2])
    cache2, bt2b, _ = O.build_paged_cache(k2, k2, [L2], sink, window, O.FP8_E4M3)
    cache2.k_fp8 = np.concatenate([cache2.k_fp8, np.full((1, hkv, 16, d), 0x55, np.uint8)])
    cache2.v_fp8 = np.concatenate([cache2.v_fp8, np.full((1, hkv, 16, d), 0x55, np.uint8)])
    cache2.k_fp8_scale = np.concatenate([cache2.k_fp8_scale, np.float32([3.0])])
    cache2.v_fp8_scale = np.concatenate([cache2.v_fp8_scale, np.float32([3.0])])
    bt2b[0, 3] = cache2.k_fp8.shape[0] - 1
    c4, _, _, _ = O.append_retier(cache2, bt2b, [L2], small, small, [0], sink, window, O.FP8_E4M3)
    pg = c4.k_fp8[-1]
    assert np.all(pg[:, 1:] == 0) and np.any(pg[:, 0] != 0)


def test_append_retier_keeps_sinks_and_anchors():
    rng = np.random.default_rng(3)
    hkv, d = 1, 8
    # window 16: at L = 47, page 1 (tokens 16..31) leaves -- unless it holds
    # sink tokens (sink 20); page 0 always holds sink tokens
    assert O.leaving_page(47, 20, 16) == -1
    assert O.leaving_page(47, 4, 16) == 1
    assert O.leaving_page(31, 4, 16) == -1
    L = 31
    k = _pages_up_to(rng, 1, 3, hkv, d, [L])
    cache, bt, fmt = O.build_paged_cache(k, k, [L], 4, 16, O.BF16)
    # a page tagged as a BF16 anchor stays where it is
    tags = np.full((1, 3), O.TERNARY, np.uint8)
    tags[0, 1] = O.BF16
    L3 = 47                                            # page 1 leaves
    k3 = _pages_up_to(rng, 1, 3, hkv, d, [L3])
    c3, bt3, _ = O.build_paged_cache(k3, k3, [L3], 4, 16, O.BF16)
    assert c3.k_tern.shape[0] == 0                     # room for the retiered page
    for w in ("k", "v"):
        setattr(c3, w + "_tern", np.zeros((1, hkv, 16, d // 4), np.uint8))
        setattr(c3, w + "_gamma", np.zeros((1, hkv), np.float32))
    nz = bf16_bits(np.ones((1, hkv, d)))
    out, bt_out, freed, tags_out = O.append_retier(c3, bt3, [L3], nz, nz, [0], 4, 16, O.BF16, older_fmt=tags)
    assert freed[0] == -1 and bt_out[0, 1] == bt3[0, 1]
    out2, bt_out2, freed2, _ = O.append_retier(c3, bt3, [L3], nz, nz, [0], 4, 16, O.BF16)
    assert freed2[0] == bt3[0, 1] and bt_out2[0, 1] == 0


# ------------------------------------------------- stale -> anchor promotion

def _one_stale_page_cache(codes, gammas, n_anchor=2, d=8):
    """A cache whose only ternary page holds the given literal packed bytes
    ([Hkv][P][D/4]) and gammas, plus empty BF16 / FP8 anchor pools of
    n_anchor slots; sequence 0 has 3 pages, page 1 is the stale one."""
    hkv = codes.shape[0]
    z16 = np.zeros((n_anchor, hkv, 16, d), np.uint16)
    z8 = np.zeros((n_anchor, hkv, 16, d), np.uint8)
    cache = O.PagedCache(k_bf16=z16, v_bf16=z16.copy(), k_fp8=z8, v_fp8=z8.copy(),
                         k_fp8_scale=np.zeros(n_anchor, np.float32), v_fp8_scale=np.zeros(n_anchor, np.float32),
                         k_tern=codes[None].copy(), v_tern=codes[None, :, ::-1].copy(),
                         k_gamma=np.float32(gammas)[None], v_gamma=np.float32(gammas)[None].copy())
    bt = np.array([[0, 0, 0]], np.int32)
    tags = np.full((1, 3), O.TERNARY, np.uint8)
    return cache, bt, tags


def _literal_codes(hkv=4, d=8):
    # row t of every head: bytes 0x55 (+1 +1 +1 +1), 0xFF (-1 x4), 0x1D (+1 -1 +1 0)
    # and 0x00, rotating with t; head 3 is all zero
    pat = [0x55, 0xFF, 0x1D, 0x00]
    c = np.zeros((hkv, 16, d // 4), np.uint8)
    for h in range(hkv - 1):
        for t in range(16):
            for w in range(d // 4):
                c[h, t, w] = pat[(t + w + h) % 4]
    return c


def test_promote_bf16_literal_values():
    # gamma 1, 0.5, 0.25 (bf16-exact) and 2.0 on an all-zero head: the anchor
    # page holds +-gamma as bf16 bit patterns written out by hand
    codes = _literal_codes()
    cache, bt, tags = _one_stale_page_cache(codes, [1.0, 0.5, 0.25, 2.0])
    out, bt2, tags2, freed, flags = O.promote_pages(cache, bt, tags, [40], [0], [1], [1], 4, 8, O.BF16, O.BF16)
    assert flags == 0 and freed.tolist() == [0] and bt2[0, 1] == 1 and tags2[0, 1] == O.BF16
    assert bt2[0, 0] == 0 and tags2[0, 0] == O.TERNARY and bt2[0, 2] == 0
    pos = {0: 0x3F80, 1: 0x3F00, 2: 0x3E80, 3: 0x4000}      # 1.0, 0.5, 0.25, 2.0
    val = {0x55: [1, 1, 1, 1], 0xFF: [-1, -1, -1, -1], 0x1D: [1, -1, 1, 0], 0x00: [0, 0, 0, 0]}
    for h in range(4):
        for t in range(16):
            row = [c for w in range(2) for c in val[int(codes[h, t, w])]]
            want = [0 if c == 0 else (pos[h] | (0x8000 if c < 0 else 0)) for c in row]
            assert out.k_bf16[1, h, t].tolist() == want, (h, t)
    assert np.all(out.k_bf16[0] == 0)                 # the other anchor slot untouched
    assert np.array_equal(out.k_tern, cache.k_tern)   # the stale copy stays (freed, not erased)


def test_promote_fp8_literal_codes_and_zero_head_excluded_from_amax():
    # amax over the decoded page is 1.0 (the all-zero head's gamma 2.0 does not
    # count): s = fl32(1/448); +-1, +-0.5, +-0.25 map to +-448, +-224, +-112,
    # e4m3 0x7E, 0x76, 0x6E (sign bit 0x80), zero to 0x00
    codes = _literal_codes()
    cache, bt, tags = _one_stale_page_cache(codes, [1.0, 0.5, 0.25, 2.0])
    out, bt2, tags2, freed, flags = O.promote_pages(cache, bt, tags, [40], [0], [1], [0], 4, 8, O.BF16,
                                                    O.FP8_E4M3)
    assert flags == 0 and freed.tolist() == [0] and bt2[0, 1] == 0 and tags2[0, 1] == O.FP8_E4M3
    assert out.k_fp8_scale[0] == np.float32(1.0 / 448.0)
    mag = {0: 0x7E, 1: 0x76, 2: 0x6E, 3: 0x00}
    val = {0x55: [1, 1, 1, 1], 0xFF: [-1, -1, -1, -1], 0x1D: [1, -1, 1, 0], 0x00: [0, 0, 0, 0]}
    for h in range(4):
        for t in range(16):
            row = [c for w in range(2) for c in val[int(codes[h, t, w])]]
            want = [0 if c == 0 else (mag[h] | (0x80 if c < 0 else 0)) for c in row]
            assert out.k_fp8[0, h, t].tolist() == want, (h, t)
    # V was built from the row-reversed codes: same magnitudes, same scale
    assert out.v_fp8_scale[0] == np.float32(1.0 / 448.0)


def test_promote_skips_sinks_window_anchors_and_bad_indices():
    codes = _literal_codes()
    cache, bt, tags = _one_stale_page_cache(codes, [1.0, 0.5, 0.25, 2.0])
    tags_anchor = tags.copy()
    tags_anchor[0, 1] = O.BF16
    cases = [
        (dict(req_page=[0]), tags, O.PROMOTE_NOT_STALE),        # sink page
        (dict(req_page=[2]), tags, O.PROMOTE_NOT_STALE),        # window page (L = 40, window 8)
        (dict(req_page=[1]), tags_anchor, O.PROMOTE_NOT_STALE),  # already an anchor
        (dict(req_page=[3]), tags, O.PROMOTE_RANGE),            # beyond the sequence's 3 pages
        (dict(req_seq=[1]), tags, O.PROMOTE_RANGE),             # beyond the batch
        (dict(slot=[2]), tags, O.PROMOTE_SLOT),                 # anchor pool has 2 slots
    ]
    for over, tg, flag in cases:
        a = dict(req_seq=[0], req_page=[1], slot=[0])
        a.update(over)
        out, bt2, tags2, freed, flags = O.promote_pages(cache, bt, tg, [40], a["req_seq"], a["req_page"],
                                                        a["slot"], 4, 8, O.BF16, O.BF16)
        assert flags == flag and freed.tolist() == [-1], over
        assert np.array_equal(bt2, bt) and np.array_equal(tags2, tg)
        assert np.all(out.k_bf16 == 0) and np.all(out.v_bf16 == 0)


@pytest.mark.parametrize("anchor_fmt", [O.BF16, O.FP8_E4M3])
def test_promote_keeps_attention_when_values_are_exact(anchor_fmt):
    """Groups whose |x| is one bf16 value a per (page, head) have gamma = a
    and decode exactly to +-a; promoting such pages must leave decode
    attention unchanged (BF16: the same values; FP8: s*e = a up to the fp32
    rounding of s when a / amax is a power of two)."""
    rng = np.random.default_rng(21)
    B, maxp, hkv, d, hq = 2, 6, 2, 16, 4
    lens = [16 * 6, 16 * 5 + 3]
    mag = np.float32(2.0) ** rng.integers(-2, 2, size=(B, maxp, hkv))[..., None, None]
    x = np.sign(rng.standard_normal((B, maxp, hkv, 16, d))).astype(np.float32) * mag
    kb = bf16_bits(x)
    vb = bf16_bits(x[:, :, ::-1])
    q = bf16_bits(rng.standard_normal((B, hq, d)))
    tags = np.full((B, maxp), O.TERNARY, np.uint8)
    cache, bt, fmt = O.build_paged_cache(kb, vb, lens, 4, 20, O.BF16, older_fmt=tags)
    ref = O.decode_attention(q, cache, bt, fmt, lens, hkv)
    stale = [(b, j) for b in range(B) for j in range(maxp) if fmt[b, j] == O.TERNARY]
    assert len(stale) >= 4
    pick = stale[::2]
    for w in ("k", "v"):                                 # room for the anchors
        if anchor_fmt == O.BF16:
            setattr(cache, w + "_bf16", np.concatenate([getattr(cache, w + "_bf16"),
                                                        np.zeros((len(pick), hkv, 16, d), np.uint16)]))
        else:
            setattr(cache, w + "_fp8", np.zeros((len(pick), hkv, 16, d), np.uint8))
            setattr(cache, w + "_fp8_scale", np.zeros(len(pick), np.float32))
    base = 0 if anchor_fmt == O.FP8_E4M3 else cache.k_bf16.shape[0] - len(pick)
    slots = [base + i for i in range(len(pick))]
    out, bt2, tags2, freed, flags = O.promote_pages(cache, bt, tags, lens, [b for b, _ in pick],
                                                    [j for _, j in pick], slots, 4, 20, O.BF16, anchor_fmt)
    assert flags == 0 and sorted(freed.tolist()) == sorted(int(bt[b, j]) for b, j in pick)
    fmt2 = np.array([[O.page_format(j, lens[b], 4, 20, O.BF16, int(tags2[b, j])) if j < O.num_pages(lens[b])
                      else 255 for j in range(maxp)] for b in range(B)], np.uint8)
    assert all(fmt2[b, j] == anchor_fmt for b, j in pick)
    got = O.decode_attention(q, out, bt2, fmt2, lens, hkv)
    assert np.abs(got - ref).max() < (1e-12 if anchor_fmt == O.BF16 else 1e-6)


def test_promote_fp8_within_e4m3_rounding_of_the_stale_values():
    """An FP8 anchor decodes (s * e) to the stale page's bf16(gamma * c)
    within half an e4m3 step: relative 2^-4 for normal e4m3 values, and the
    head with the largest gamma maps to +-448 exactly."""
    rng = np.random.default_rng(31)
    hkv, d = 4, 16
    codes = rng.choice(np.array([0x55, 0xFF, 0x1D, 0x00, 0x7D], np.uint8), size=(hkv, 16, d // 4))
    codes[0] = 0x55                                          # head 0: all +1
    gam = np.float32([2.5, 0.37, 0.011, 1.9])
    cache, bt, tags = _one_stale_page_cache(codes, gam, d=d)
    out, _, _, _, flags = O.promote_pages(cache, bt, tags, [40], [0], [1], [0], 4, 8, O.BF16, O.FP8_E4M3)
    assert flags == 0
    want = O.bf16_to_f64(O.dequantize_ternary(codes[None], gam[None])[0])          # [Hkv][P][D]
    got = float(out.k_fp8_scale[0]) * O.e4m3_to_f64(out.k_fp8[0])
    amax = np.abs(want).max()
    assert np.all(np.abs(out.k_fp8[0][0]) == 0x7E)                  # +448 (the largest gamma is head 0)
    nz = want != 0
    assert np.all(np.sign(got[nz]) == np.sign(want[nz])) and np.all(got[~nz] == 0)
    normal = np.abs(want) >= amax / 448 * 2.0 ** -6                # e4m3 normal range after scaling
    assert np.all(np.abs(got - want)[normal] <= np.abs(want)[normal] * 2.0 ** -4 + 1e-12)
    sub = nz & ~normal
    assert np.all(np.abs(got - want)[sub] <= amax / 448 * 2.0 ** -10 + 1e-12)   # half a subnormal step
