"""Pins of the exponent-split lossless codec oracle (oracle/exans.py) against
what the page and the mathematics fix: losslessness, the exponent /
sign+mantissa split of the bf16 format, the ANS size (the cross-entropy of
the symbols under the coded table), the table rules, and hand-derived
bytes for a single-exponent group."""

import math

import numpy as np
import torch

import oracle.exans as X


def _bf16(vals):
    return torch.tensor(np.asarray(vals, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _groups():
    rng = np.random.default_rng(0)
    n = 8 * 16 * 128
    x = rng.standard_normal(n).astype(np.float32)
    outl = x.reshape(8, 16, 128).copy()
    outl[:, :, rng.random(128) < 0.02] *= 10.0
    lap = rng.laplace(size=4 * 16 * 64).astype(np.float32)
    tiny = (rng.standard_normal(1024) * 1e-30).astype(np.float32)      # subnormal-heavy
    every = np.arange(65536, dtype=np.uint32).astype(np.uint16)          # every bf16 pattern
    return {"normal": _bf16(x), "outlier_channels": _bf16(outl.reshape(-1)), "laplace": _bf16(lap),
            "tiny": _bf16(tiny), "zeros": np.zeros(2048, np.uint16), "every_pattern": every,
            "signed_zeros": np.tile(np.array([0x0000, 0x8000], np.uint16), 512)}


def test_round_trip_is_lossless():
    for name, g in _groups().items():
        blob = X.encode_group(g)
        assert len(blob) % 16 == 0 and X.parse_header(blob)["total"] == len(blob), name
        assert np.array_equal(X.decode_group(blob), g), name
    # every bf16 pattern: nearly all exponents escape, so the group is stored raw
    h = X.parse_header(X.encode_group(_groups()["every_pattern"]))
    assert h["mode"] == 0 and h["total"] == X.HEADER + 2 * 65536


def test_split_follows_the_bf16_layout():
    # bf16 = sign(1) | exponent(8) | mantissa(7); values written from that definition
    vals = {0x3F80: (127, 0x00), 0xBF80: (127, 0x80), 0x4049: (128, 0x49), 0xC2F7: (133, 0xF7),
            0x0001: (0, 0x01), 0x8000: (0, 0x80), 0x7F80: (255, 0x00), 0xFFC1: (255, 0xC1)}
    bits = np.array(list(vals), np.uint16)
    exp, sm = X.split_streams(bits)
    assert exp.tolist() == [v[0] for v in vals.values()]
    assert sm.tolist() == [v[1] for v in vals.values()]
    assert np.array_equal(X.join_streams(exp, sm), bits)
    # the coded blob carries the sign+mantissa bytes raw, in element order
    g = _groups()["normal"]
    blob = X.encode_group(g)
    assert blob[X.HEADER:X.HEADER + len(g)] == X.split_streams(g)[1].tobytes()


def test_centre_and_table_rules():
    exps = np.array([5] * 10 + [3] * 10 + [9] * 4, np.uint8)
    assert X.centre(exps) == 3                                          # tie 3 / 5 -> smaller
    assert X.symbols(np.array([3, 4, 9, 0, 200], np.uint8), 3).tolist() == [8, 9, 14, 5, 15]
    assert X.symbols(np.array([10, 11], np.uint8), 3).tolist() == [15, 15]   # +7 and beyond escape
    assert X.symbols(np.array([0], np.uint8), 9).tolist() == [15]          # -9 escapes
    n = 16384
    f = X.normalise(np.array([n // 2, n // 4, n // 4] + [0] * 13), n)
    assert f.tolist() == [2048, 1024, 1024] + [0] * 13
    counts = np.zeros(16, np.int64)
    counts[[0, 7, 8, 15]] = [1, 9000, 7382, 1]                          # two symbols below 1/4096
    f = X.normalise(counts, n)
    assert f.sum() == X.M and f[0] == 1 and f[15] == 1 and (f[counts == 0] == 0).all()
    assert f[7] == 9000 * 4096 // n + (X.M - (1 + 9000 * 4096 // n + 7382 * 4096 // n + 1))


def test_single_exponent_group_hand_bytes():
    # every value in [1, 2): exponent 127 for all -> one symbol with f = 4096;
    # each rANS state stays at 2^23, so the stream is 32 x (00 00 80 00)
    rng = np.random.default_rng(3)
    n = 1024
    g = ((127 << 7) | rng.integers(0, 128, n) | (rng.integers(0, 2, n) << 15)).astype(np.uint16)
    blob = X.encode_group(g)
    h = X.parse_header(blob)
    assert (h["mode"], h["n"], h["centre"], h["escapes"], h["stream"]) == (1, n, 127, 0, 128)
    assert h["f"].tolist() == [0] * 8 + [4096] + [0] * 7
    assert h["total"] == X.HEADER + n + 128 == len(blob)
    assert blob[:4] == (X.HEADER + n + 128).to_bytes(4, "little")
    assert blob[X.HEADER + n:] == bytes([0x00, 0x00, 0x80, 0x00]) * 32


def test_stream_size_is_the_cross_entropy():
    """ANS spends -log2(f_s / 4096) bits per symbol; over a group the stream
    is that sum plus at most the 32 flushed states (4 bytes each) and one
    partial byte per lane."""
    rng = np.random.default_rng(4)
    for scale in (1.0, 0.3, 30.0):
        x = _bf16(rng.standard_normal(16384) * scale)
        exp, _ = X.split_streams(x)
        sym = X.symbols(exp, X.centre(exp))
        f = X.normalise(np.bincount(sym, minlength=16), len(sym))
        bits = float(sum(-math.log2(f[s] / X.M) for s in sym))
        n_stream = X.parse_header(X.encode_group(x))["stream"]
        assert bits / 8 - 4 <= n_stream <= bits / 8 + 32 * 5, (scale, n_stream, bits / 8)


def test_escapes_in_element_order():
    g = _bf16(np.ones(1024, np.float32))                              # exponent 127
    pos = [5, 130, 131, 900]
    far = [0x7000, 0x0080, 0xFF00, 0x2000]                             # exponents 224, 1, 254, 64
    g[pos] = np.array(far, np.uint16)
    blob = X.encode_group(g)
    h = X.parse_header(blob)
    assert h["escapes"] == 4
    assert list(blob[X.HEADER + 1024:X.HEADER + 1028]) == [224, 1, 254, 64]
    assert np.array_equal(X.decode_group(blob), g)


def test_ratio_on_normal_data_is_near_the_page():
    # context, not a target: the page reports 1.51x on real KV caches
    g = _groups()["normal"]
    r = 2 * len(g) / len(X.encode_group(g))
    assert 1.45 < r < 1.56


def test_pages_round_trip():
    rng = np.random.default_rng(5)
    pages = _bf16(rng.standard_normal((6, 2, 16, 64))).reshape(6, 2, 16, 64)
    pool, off = X.encode_pages(pages, [4, 0, 2])
    assert off[0] == 0 and off[-1] == len(pool) and (np.diff(off) % 16 == 0).all()
    back = X.decode_pages(pool, off, (2, 16, 64))
    assert np.array_equal(back, pages[[4, 0, 2]])


def test_rans_round_trip_on_adversarial_tables():
    """The coder on its own, with tables the exponent data rarely produces:
    symbols of frequency 1 used often (two renormalisation bytes per
    symbol), a table of one symbol, and uniform tables.  Decoding gives
    the symbols back and the size stays at the cross-entropy."""
    rng = np.random.default_rng(9)
    n = 4096
    cases = []
    f = np.zeros(16, np.int64); f[0] = 1; f[1] = 1; f[2] = X.M - 2
    cases.append((rng.choice([0, 1, 2], size=n, p=[0.45, 0.45, 0.10]), f))          # rare-by-table symbols dominate
    f = np.zeros(16, np.int64); f[7] = X.M
    cases.append((np.full(n, 7), f))                                                 # one symbol
    cases.append((rng.integers(0, 16, n), np.full(16, X.M // 16, np.int64)))         # uniform, 4 bits each
    f = np.full(16, 1, np.int64); f[15] = X.M - 15
    cases.append((rng.integers(0, 15, n), f))                                        # 15 symbols at 1/4096
    for sym, f in cases:
        assert f.sum() == X.M and (f[np.unique(sym)] > 0).all()
        stream = X.rans_encode(sym, f)
        assert np.array_equal(X.rans_decode(stream, f, n), sym)
        bits = float(sum(-math.log2(f[s] / X.M) for s in sym))
        assert bits / 8 - 4 <= len(stream) <= bits / 8 + 32 * 5, (len(stream), bits / 8)


def test_normalise_properties():
    rng = np.random.default_rng(10)
    for _ in range(300):
        n = int(rng.integers(128, 1 << 16)) // 128 * 128 or 128
        k = int(rng.integers(1, 17))
        probs = rng.dirichlet(np.full(k, float(rng.choice([0.05, 1.0, 20.0]))))
        counts = np.zeros(16, np.int64)
        idx = rng.choice(16, size=k, replace=False)
        counts[idx] = rng.multinomial(n, probs)
        f = X.normalise(counts, n)
        assert f.sum() == X.M
        assert np.array_equal(f > 0, counts > 0) and (f >= 0).all()
