"""Oracle: a plain, slow, CPU restatement of the compressed paged KV cache and
of single-token decode attention over it.

TEST INFRASTRUCTURE ONLY.  Nothing in the product package
(``compressed_decode_attention_kvc_b200``) imports, links or runs this file.
The only callers are ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / ``--impl reference`` legs.  It shares no code, header, table
or constant generator with the CUDA path; the two meet only in the seeded
input generators of ``synth/``, which hold none of the method's arithmetic.

Every array is numpy.  bf16 values travel as their uint16 bit patterns and
e4m3 values as their uint8 bit patterns, so that the byte-level outputs can be
compared bit for bit.  Attention runs in float64 on the exactly decoded cache.

Sources, cited by page title and section:

* [Vantage] "Show HN: Vantage-V-AI - 2-bit ternary KV cache with attention
  sinks" (newshot.cc), section "Core architecture": keys and values quantised
  to ternary {-1, 0, +1} with gamma = mean(|X|) ("inspired by BitNet b1.58"),
  4 elements per uint8 byte = 2.0 bit/element, 7.97x smaller than FP16;
  attention-sink retention (sink_tokens=4, after StreamingLLM).  Section
  "Quick start": the knobs ``max_active_tokens`` (the recent window),
  ``sink_tokens`` and ``quant_mode="fp8"`` (dynamic FP8 streaming mode).
* [Minima] "Minima-KV: more memory for long-context AI without deleting old
  context" (twodots.gr), section "Recent, Anchor and Stale": recent pages in
  FP8, older critical pages (system prompt, initial sinks) kept at higher
  fidelity as anchors, stale pages compressed yet still addressable; section
  "How mixed-format attention works": format-specific branches read each
  page's format directly, each branch emits a partial state (max score, sum
  of exponentials, normalised output) and the partial states are merged by a
  common online-softmax normalisation that keeps logical page order and the
  causal mask; section "Why the KV cache becomes a bottleneck": paged,
  non-contiguous KV blocks addressed through a block table, and the 64 KiB /
  32 KiB per-token figures; section "What the memory measurements showed":
  the 18.3 KiB/token accounting.

Readings taken where the pages are silent (each is also listed in the design
notes of the repository):

* gamma is per (page, KV head), K and V separately, not per tensor as the
  Vantage page says; the sum of |x| is taken in float64 and rounded once to
  float32.  gamma == 0 (an all-zero group) gives all-zero codes and a stored
  gamma of 0.
* RoundClip(x / gamma, -1, +1) with round-half-to-even: code +1 iff
  x > gamma/2, -1 iff x < -gamma/2, else 0 (so |x| == gamma/2 maps to 0).
* 2-bit fields: 00 -> 0, 01 -> +1, 11 -> -1 (two's complement); 10 is never
  written.  Element i of a group's row-major [token][dim] order sits in byte
  i // 4 at bits 2*(i % 4) .. 2*(i % 4) + 1.
* FP8 e4m3 (OCP 8-bit float, bias 7, max 448, no infinities) with one float32
  scale per (page, K or V) over all KV heads: s = amax / 448,
  e = RNE-satfinite(x * (448 / amax)), both products and quotients in
  float32; amax == 0 gives s = 1.  Negative values that round to zero keep
  their sign (0x80).
* Pages are 16 tokens; a page is high precision (the caller's hp format) iff
  it overlaps the first ``sink`` tokens or the last ``window`` tokens;
  otherwise its format is the caller's per-page tag (ternary for stale
  pages, BF16 / FP8 for anchors).  Tokens at or beyond the context length are
  masked.  The query token's own K/V is already in the cache.
* Query head h reads KV head h // (Hq / Hkv).  The softmax scale defaults to
  1 / sqrt(head_dim).

Parity status: every function below is pinned by ``tests/test_oracle_pins.py``
against closed forms, library routines (torch's bf16 / float8_e4m3fn
conversions and scaled_dot_product_attention) or brute force, except the
*approximation quality* of ternary attention against dense attention, which
the pages measure only end to end with trained weights: parity unpinned
there, and nothing here claims it.
"""

from __future__ import annotations

from dataclasses import dataclass
import math

import numpy as np

PAGE_SIZE = 16  # tokens per page

# Page formats (the oracle's own names; the tests map them to the library's).
BF16 = 0
FP8_E4M3 = 1
TERNARY = 2

E4M3_MAX = 448.0


# ---------------------------------------------------------------------------
# bf16 <-> float helpers (bit patterns in uint16)
# ---------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64 (exact: bf16 is the top half of a float32)."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


def f32_to_bf16_rne(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest, ties to even (finite x)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    return ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)


# ---------------------------------------------------------------------------
# Ternary codec  [Vantage, "Core architecture"]
# ---------------------------------------------------------------------------

def ternary_gamma(group: np.ndarray) -> np.float32:
    """gamma = mean(|X|) of one (page, KV head) group, summed in float64 and
    rounded once to float32.  [Vantage, "Core architecture": the absmean
    scale of BitNet b1.58.]"""
    g = np.asarray(group, dtype=np.float64)
    return np.float32(np.abs(g).sum() / g.size)


def ternary_codes(group: np.ndarray, gamma: np.float32) -> np.ndarray:
    """RoundClip(x / gamma, -1, +1) with ties to even, as int8 codes in
    {-1, 0, +1}.  [Vantage, "Core architecture"]

    round(x / gamma) is +1 exactly when x / gamma > 1/2 and -1 exactly when
    x / gamma < -1/2 (a tie at +-1/2 rounds to the even value 0); clipping to
    [-1, 1] changes nothing else.  The comparison is made against
    gamma / 2 in float64, where both x (a bf16 value) and gamma / 2 (a float32
    value halved) are exact, so the decision carries no rounding."""
    x = np.asarray(group, dtype=np.float64)
    t = 0.5 * float(gamma)
    c = np.zeros(x.shape, dtype=np.int8)
    c[x > t] = 1
    c[x < -t] = -1
    return c


_FIELD_OF_CODE = {0: 0b00, 1: 0b01, -1: 0b11}
_CODE_OF_FIELD = {0b00: 0, 0b01: 1, 0b11: -1}


def pack_ternary(codes: np.ndarray) -> np.ndarray:
    """Pack int8 codes (last axis a multiple of 4) into bytes, 4 per byte.
    Code i of the last axis goes to byte i // 4, bits 2*(i % 4)..+1, with
    00 -> 0, 01 -> +1, 11 -> -1.  [Vantage, "Core architecture": 4 elements
    per uint8 byte = 2.0 bit/element.]"""
    c = np.asarray(codes, dtype=np.int8)
    if c.shape[-1] % 4:
        raise ValueError("last axis must be a multiple of 4")
    if not np.isin(c, (-1, 0, 1)).all():
        raise ValueError("codes must be in {-1, 0, +1}")
    fields = np.zeros(c.shape, dtype=np.uint8)
    for code, field in _FIELD_OF_CODE.items():
        fields[c == code] = field
    f = fields.reshape(c.shape[:-1] + (c.shape[-1] // 4, 4))
    out = np.zeros(f.shape[:-1], dtype=np.uint8)
    for j in range(4):
        out |= (f[..., j] << np.uint8(2 * j)).astype(np.uint8)
    return out


def unpack_ternary(packed: np.ndarray) -> np.ndarray:
    """Inverse of pack_ternary.  Raises on the unused field 10."""
    p = np.asarray(packed, dtype=np.uint8)
    fields = np.stack([(p >> np.uint8(2 * j)) & np.uint8(3) for j in range(4)], axis=-1)
    if (fields == 0b10).any():
        raise ValueError("invalid 2-bit field 10 in packed ternary data")
    codes = np.zeros(fields.shape, dtype=np.int8)
    for field, code in _CODE_OF_FIELD.items():
        codes[fields == field] = code
    return codes.reshape(p.shape[:-1] + (p.shape[-1] * 4,))


def quantize_pack_ternary(src_pages: np.ndarray, page_ids=None):
    """Ternary-quantise and pack whole pages.

    src_pages: bf16 bits [n_src][Hkv][P][D].  page_ids: which source pages,
    in output order (None = all).  Returns (codes uint8 [n][Hkv][P][D/4],
    gamma float32 [n][Hkv]).  Each (page, KV head) group is quantised on its
    own: gamma over its P*D values, then codes, then packing in row-major
    [token][dim] order."""
    src = np.asarray(src_pages, dtype=np.uint16)
    ids = np.arange(src.shape[0]) if page_ids is None else np.asarray(page_ids)
    n, (_, hkv, p, d) = len(ids), src.shape
    codes = np.zeros((n, hkv, p, d // 4), dtype=np.uint8)
    gamma = np.zeros((n, hkv), dtype=np.float32)
    for i, pid in enumerate(ids):
        for h in range(hkv):
            x = bf16_to_f64(src[pid, h])           # [P][D]
            gamma[i, h] = ternary_gamma(x)
            c = ternary_codes(x, gamma[i, h])
            codes[i, h] = pack_ternary(c.reshape(p, d)).reshape(p, d // 4)
    return codes, gamma


def ternary_decoded_f64(codes: np.ndarray, gamma) -> np.ndarray:
    """Exact value of a ternary group: gamma * c in float64."""
    return float(gamma) * unpack_ternary(codes).astype(np.float64)


def dequantize_ternary(codes: np.ndarray, gamma: np.ndarray) -> np.ndarray:
    """Packed pages [n][Hkv][P][D/4] + gamma [n][Hkv] -> bf16 bits
    [n][Hkv][P][D]: bf16(RN(gamma * c)), the product taken in float32 (it is
    exact: c is -1, 0 or +1)."""
    c = unpack_ternary(codes).astype(np.float32)            # [n][Hkv][P][D]
    prod = (np.asarray(gamma, np.float32)[:, :, None, None] * c).astype(np.float32)
    return f32_to_bf16_rne(prod)


# ---------------------------------------------------------------------------
# FP8 e4m3 codec  [Vantage, "Quick start" quant_mode="fp8" and "Core
# architecture" FP8 streaming mode; Minima, "Recent, Anchor and Stale"]
# ---------------------------------------------------------------------------

def e4m3_table():
    """All non-negative finite e4m3 values and their codes, in increasing
    order, from the format's definition: sign | 4-bit exponent (bias 7) |
    3-bit mantissa; exponent 0 is subnormal (m/8 * 2^-6); the code with all
    exponent and mantissa bits set is NaN; there is no infinity."""
    vals, codes = [], []
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
            vals.append(v)
            codes.append((e << 3) | m)
    return np.array(vals, dtype=np.float64), np.array(codes, dtype=np.uint8)


_E4M3_VALS, _E4M3_CODES = e4m3_table()


def e4m3_to_f64(bits: np.ndarray) -> np.ndarray:
    """e4m3 bit patterns -> float64 (exact).  NaN codes are rejected."""
    b = np.asarray(bits, dtype=np.uint8)
    mag = b & np.uint8(0x7F)
    if (mag == 0x7F).any():
        raise ValueError("e4m3 NaN code in data")
    lut = np.zeros(128, dtype=np.float64)
    lut[_E4M3_CODES] = _E4M3_VALS
    v = lut[mag]
    return np.where(b & np.uint8(0x80), -v, v)


def f32_to_e4m3_rne_satfinite(y: np.ndarray) -> np.ndarray:
    """float32 -> e4m3 bit patterns: round to the nearest finite e4m3 value,
    ties to the even code (mantissa LSB 0), magnitudes beyond 448 saturate to
    448, and the sign bit follows the input's (so a negative value that
    rounds to zero gives 0x80)."""
    y32 = np.asarray(y, dtype=np.float32)
    a = np.minimum(np.abs(y32).astype(np.float64), E4M3_MAX)
    hi = np.searchsorted(_E4M3_VALS, a, side="left")            # first value >= a
    hi = np.minimum(hi, len(_E4M3_VALS) - 1)
    lo = np.maximum(hi - 1, 0)
    d_hi = _E4M3_VALS[hi] - a
    d_lo = a - _E4M3_VALS[lo]
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ((_E4M3_CODES[hi] & 1) == 0))
    pick_hi |= (d_hi == 0)
    mag_code = np.where(pick_hi, _E4M3_CODES[hi], _E4M3_CODES[lo])
    sign = np.signbit(y32).astype(np.uint8) << np.uint8(7)
    return (mag_code | sign).astype(np.uint8)


def fp8_page_scale(page_f32: np.ndarray):
    """(amax, s, inv) of one page over all its KV heads: s = fl32(amax/448),
    inv = fl32(448/amax); amax == 0 gives s = inv = 1."""
    amax = np.float32(np.abs(page_f32).max()) if page_f32.size else np.float32(0)
    if amax == 0:
        return amax, np.float32(1.0), np.float32(1.0)
    return amax, np.float32(amax / np.float32(E4M3_MAX)), np.float32(np.float32(E4M3_MAX) / amax)


def quantize_fp8_pages(src_pages: np.ndarray, page_ids=None):
    """FP8-quantise whole pages: one scale per page (over all KV heads).
    src bf16 bits [n_src][Hkv][P][D] -> (e4m3 bits [n][Hkv][P][D],
    scale float32 [n]).  y = fl32(x * inv), e = RNE-satfinite(y)."""
    src = np.asarray(src_pages, dtype=np.uint16)
    ids = np.arange(src.shape[0]) if page_ids is None else np.asarray(page_ids)
    out = np.zeros((len(ids),) + src.shape[1:], dtype=np.uint8)
    scale = np.zeros(len(ids), dtype=np.float32)
    for i, pid in enumerate(ids):
        x = bf16_to_f64(src[pid]).astype(np.float32)             # exact
        _, s, inv = fp8_page_scale(x)
        y = (x * inv).astype(np.float32)                          # one fp32 rounding
        out[i] = f32_to_e4m3_rne_satfinite(y)
        scale[i] = s
    return out, scale


def dequantize_fp8(e4m3: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """e4m3 pages [n][Hkv][P][D] + scale [n] -> bf16 bits: bf16(RN(fl32(s*e)))."""
    e = e4m3_to_f64(e4m3).astype(np.float32)                      # exact
    prod = (np.asarray(scale, np.float32)[:, None, None, None] * e).astype(np.float32)
    return f32_to_bf16_rne(prod)


def copy_bf16_pages(src_pages: np.ndarray, page_ids=None) -> np.ndarray:
    """The high-precision BF16 format keeps the page as it is."""
    src = np.asarray(src_pages, dtype=np.uint16)
    ids = np.arange(src.shape[0]) if page_ids is None else np.asarray(page_ids)
    return src[ids].copy()


# ---------------------------------------------------------------------------
# Paged mixed-format cache  [Minima, "Why the KV cache becomes a bottleneck"
# (paged blocks), "Recent, Anchor and Stale" (tiers); Vantage, "Quick start"
# and "Core architecture" (sinks, window)]
# ---------------------------------------------------------------------------

def num_pages(context_len: int) -> int:
    return -(-int(context_len) // PAGE_SIZE)


def page_format(j: int, context_len: int, sink: int, window: int,
                hp_fmt: int, older_fmt: int) -> int:
    """Format of logical page j: the high-precision format if the page holds
    any of the first ``sink`` tokens or any of the last ``window`` tokens,
    otherwise the caller's tag for that older page (ternary = stale, BF16 or
    FP8 = anchor)."""
    first = j * PAGE_SIZE
    last_valid = min((j + 1) * PAGE_SIZE, context_len) - 1   # last token held
    if first < sink or last_valid >= context_len - window:
        return hp_fmt
    return older_fmt


@dataclass
class PagedCache:
    """Per-format page pools (K and V separately), HND layout per page:
    bf16 / fp8 pools [n][Hkv][P][D], ternary pool [n][Hkv][P][D/4]."""
    k_bf16: np.ndarray
    v_bf16: np.ndarray
    k_fp8: np.ndarray
    v_fp8: np.ndarray
    k_fp8_scale: np.ndarray
    v_fp8_scale: np.ndarray
    k_tern: np.ndarray
    v_tern: np.ndarray
    k_gamma: np.ndarray
    v_gamma: np.ndarray


def build_paged_cache(k_pages, v_pages, context_lens, sink, window, hp_fmt,
                      older_fmt=None, slot_key=None):
    """Compress logical bf16 pages into per-format pools.

    k_pages, v_pages: bf16 bits [B][max_pages][Hkv][P][D] (logical pages).
    older_fmt: per-page tag [B][max_pages] for pages outside sink/window
    (None = all ternary).  slot_key: optional [B][max_pages] sort key; within
    each format pool, pages take physical slots in increasing key order (a
    random key gives a random physical placement).
    Returns (cache, block_table int32 [B][max_pages], fmt uint8 [B][max_pages]);
    unused block-table entries are 0 and their fmt is 255."""
    k_pages = np.asarray(k_pages, np.uint16)
    v_pages = np.asarray(v_pages, np.uint16)
    B, max_pages, hkv, p, d = k_pages.shape
    fmt = np.full((B, max_pages), 255, dtype=np.uint8)
    members = {BF16: [], FP8_E4M3: [], TERNARY: []}
    for b in range(B):
        L = int(context_lens[b])
        for j in range(num_pages(L)):
            tag = TERNARY if older_fmt is None else int(older_fmt[b][j])
            f = page_format(j, L, sink, window, hp_fmt, tag)
            fmt[b, j] = f
            members[f].append((b, j))
    block_table = np.zeros((B, max_pages), dtype=np.int32)
    for f, lst in members.items():
        if slot_key is not None:
            lst.sort(key=lambda bj: (float(slot_key[bj[0]][bj[1]]), bj))
        for slot, (b, j) in enumerate(lst):
            block_table[b, j] = slot
    flat_k = k_pages.reshape(B * max_pages, hkv, p, d)
    flat_v = v_pages.reshape(B * max_pages, hkv, p, d)

    def sorted_ids(f):
        # logical page id held by each physical slot of format f's pool
        out = np.zeros(len(members[f]), dtype=np.int64)
        for b, j in members[f]:
            out[block_table[b, j]] = b * max_pages + j
        return out

    i_bf, i_f8, i_t = sorted_ids(BF16), sorted_ids(FP8_E4M3), sorted_ids(TERNARY)
    k_f8, k_s = quantize_fp8_pages(flat_k, i_f8)
    v_f8, v_s = quantize_fp8_pages(flat_v, i_f8)
    k_t, k_g = quantize_pack_ternary(flat_k, i_t)
    v_t, v_g = quantize_pack_ternary(flat_v, i_t)
    cache = PagedCache(
        k_bf16=copy_bf16_pages(flat_k, i_bf), v_bf16=copy_bf16_pages(flat_v, i_bf),
        k_fp8=k_f8, v_fp8=v_f8, k_fp8_scale=k_s, v_fp8_scale=v_s,
        k_tern=k_t, v_tern=v_t, k_gamma=k_g, v_gamma=v_g)
    return cache, block_table, fmt


def decoded_page_f64(cache: PagedCache, which: str, fmt: int, phys: int, h: int) -> np.ndarray:
    """Exact float64 value [P][D] of KV head h of physical page ``phys`` of
    the given format: the bf16 value, s * e for FP8, gamma * c for ternary
    (no rounding of the product)."""
    if fmt == BF16:
        return bf16_to_f64(getattr(cache, which + "_bf16")[phys, h])
    if fmt == FP8_E4M3:
        s = float(getattr(cache, which + "_fp8_scale")[phys])
        return s * e4m3_to_f64(getattr(cache, which + "_fp8")[phys, h])
    if fmt == TERNARY:
        g = getattr(cache, which + "_gamma")[phys, h]
        return ternary_decoded_f64(getattr(cache, which + "_tern")[phys, h], g)
    raise ValueError(f"unknown page format {fmt}")


def gather_sequence_f64(cache, block_table_row, fmt_row, context_len, h):
    """Logical K-hat, V-hat [L][D] (float64) of one sequence and KV head,
    read page by page through the block table in logical page order; tokens
    at or beyond the context length are dropped (the causal mask)."""
    L = int(context_len)
    ks, vs = [], []
    for j in range(num_pages(L)):
        f, phys = int(fmt_row[j]), int(block_table_row[j])
        ks.append(decoded_page_f64(cache, "k", f, phys, h))
        vs.append(decoded_page_f64(cache, "v", f, phys, h))
    if not ks:
        d = cache.k_bf16.shape[-1] if cache.k_bf16.size else cache.k_fp8.shape[-1]
        return np.zeros((0, d)), np.zeros((0, d))
    return np.concatenate(ks)[:L], np.concatenate(vs)[:L]


# ---------------------------------------------------------------------------
# Attention  [Minima, "How mixed-format attention works"]
# ---------------------------------------------------------------------------

def attention_full(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * q K^T) V for one query vector, float64 throughout."""
    s = scale * (k @ q)
    w = np.exp(s - s.max())
    w /= w.sum()
    return w @ v


def attention_partial(q, k, v, scale):
    """Partial state of one chunk of tokens: (max score m, sum of
    exponentials l = sum exp(s - m), normalised output o = sum exp(s - m) v / l)."""
    s = scale * (k @ q)
    m = s.max()
    e = np.exp(s - m)
    l = e.sum()
    return m, l, (e @ v) / l


def merge_partials(parts):
    """Online-softmax merge of partial states (m_i, l_i, o_i):
    m* = max m_i, l* = sum l_i e^{m_i - m*}, o = sum l_i e^{m_i - m*} o_i / l*."""
    m_star = max(m for m, _, _ in parts)
    wts = [l * math.exp(m - m_star) for m, l, _ in parts]
    l_star = sum(wts)
    return sum(w * o for w, (_, _, o) in zip(wts, parts)) / l_star


def decode_attention(q_bits, cache: PagedCache, block_table, fmt, context_lens,
                     n_kv_heads: int, softmax_scale: float = 0.0, pairs=None):
    """Single-token decode attention over the mixed-format paged cache.

    q_bits: bf16 bits [B][Hq][D].  fmt: the per-page formats the cache was
    built with (as returned by build_paged_cache).  Returns float64
    [B][Hq][D]; with ``pairs`` (a list of (b, kv_head)), only those rows are
    computed and the rest are NaN.  A sequence of length 0 gives zeros."""
    q = bf16_to_f64(q_bits)
    B, hq, d = q.shape
    G = hq // n_kv_heads
    scale = softmax_scale if softmax_scale > 0 else 1.0 / math.sqrt(d)
    out = np.full((B, hq, d), np.nan)
    todo = pairs if pairs is not None else [(b, g) for b in range(B) for g in range(n_kv_heads)]
    for b, g in todo:
        k, v = gather_sequence_f64(cache, block_table[b], fmt[b], context_lens[b], g)
        for r in range(G):
            h = g * G + r
            out[b, h] = attention_full(q[b, h], k, v, scale) if len(k) else 0.0
    return out


# ---------------------------------------------------------------------------
# Append one token and retier  [Vantage, "Core architecture" (sinks kept,
# the window slides); Minima, "Recent, Anchor and Stale" (recent pages move
# to the compressed stale tier as they age)]
# ---------------------------------------------------------------------------

def leaving_page(context_len: int, sink: int, window: int) -> int:
    """The page that leaves the high-precision window when token
    ``context_len`` (0-based) is appended, or -1.  With page-granular
    windows a page j stops being high precision when its last token
    (j+1)*P - 1 falls below L' - window, L' = context_len + 1, i.e. when
    (j+1)*P == context_len - window + 1; sink pages never leave."""
    if window < 1:
        return -1
    x = context_len - window + 1
    if x <= 0 or x % PAGE_SIZE:
        return -1
    j = x // PAGE_SIZE - 1
    return j if j * PAGE_SIZE >= sink else -1


def append_retier(cache: PagedCache, block_table, context_lens, k_new, v_new, tern_slot,
                  sink: int, window: int, hp_fmt: int, older_fmt=None):
    """One decode step's cache update, per sequence b (lengths before the
    append; requires window >= 1, so the newest page is high precision):

    1. retier: if a page j0 leaves the window (``leaving_page``) and its tag
       is ternary (``older_fmt`` None, or older_fmt[b][j0] == TERNARY), its
       high-precision content -- the bf16 page, or bf16(s*e) of an FP8 page --
       is quantised to ternary (the ternary codec) into ternary-pool slot
       tern_slot[b]; block_table[b][j0] becomes that slot and the old
       high-precision slot is reported as freed.  A tag equal to hp_fmt keeps
       the page where it is (an anchor).
    2. append: token L = context_lens[b] goes to row L % P of page L // P,
       whose high-precision slot block_table[b][L // P] the caller has set;
       a page starting at row 0 is zeroed first.  BF16 pages take the bf16
       row as it is; FP8 pages are re-quantised as a whole: decode every row
       to bf16(s*e), put the new row in, quantise the page again.

    k_new, v_new: bf16 bits [B][Hkv][D].  Returns (cache', block_table',
    freed int32 [B] with -1 for none, older_fmt' or None); the inputs are not
    modified."""
    import copy
    c = copy.deepcopy(cache)
    bt = np.array(block_table, dtype=np.int32, copy=True)
    tags = None if older_fmt is None else np.array(older_fmt, dtype=np.uint8, copy=True)
    B = bt.shape[0]
    freed = np.full(B, -1, dtype=np.int32)
    k_new = np.asarray(k_new, np.uint16)
    v_new = np.asarray(v_new, np.uint16)
    for b in range(B):
        L = int(context_lens[b])
        j0 = leaving_page(L, sink, window)
        tag = TERNARY if (tags is None or j0 < 0) else int(tags[b, j0])
        if j0 >= 0 and tag == TERNARY:
            phys, ts = int(bt[b, j0]), int(tern_slot[b])
            for which in ("k", "v"):
                if hp_fmt == BF16:
                    page = getattr(c, which + "_bf16")[phys]
                else:
                    page = dequantize_fp8(getattr(c, which + "_fp8")[phys:phys + 1],
                                          getattr(c, which + "_fp8_scale")[phys:phys + 1])[0]
                codes, gam = quantize_pack_ternary(page[None])
                getattr(c, which + "_tern")[ts] = codes[0]
                getattr(c, which + "_gamma")[ts] = gam[0]
            bt[b, j0] = ts
            freed[b] = phys
        j, r = L // PAGE_SIZE, L % PAGE_SIZE
        phys = int(bt[b, j])
        for which, new in (("k", k_new[b]), ("v", v_new[b])):
            if hp_fmt == BF16:
                pool = getattr(c, which + "_bf16")
                if r == 0:
                    pool[phys] = 0
                pool[phys][:, r, :] = new
            else:
                pool = getattr(c, which + "_fp8")
                scl = getattr(c, which + "_fp8_scale")
                if r == 0:
                    page = np.zeros(pool.shape[1:], dtype=np.uint16)
                else:
                    page = dequantize_fp8(pool[phys:phys + 1], scl[phys:phys + 1])[0]
                page[:, r, :] = new
                e, sc = quantize_fp8_pages(page[None])
                pool[phys] = e[0]
                scl[phys] = sc[0]
    return c, bt, freed, tags


# ---------------------------------------------------------------------------
# Stale -> Anchor promotion  [Minima, "Recent, Anchor and Stale": critical
# older pages are kept at higher fidelity as anchors, stale pages stay
# addressable in compressed form and can be reconstructed]
# ---------------------------------------------------------------------------

PROMOTE_SLOT = 1        # flag: a ternary or anchor slot outside its pool
PROMOTE_NOT_STALE = 2   # flag: the page is not a ternary page (sink, window or anchor)
PROMOTE_RANGE = 4       # flag: sequence or page index outside the batch / the sequence


def promote_pages(cache: PagedCache, block_table, older_fmt, context_lens, req_seq, req_page,
                  anchor_slot, sink: int, window: int, hp_fmt: int, anchor_fmt: int):
    """Re-expand selected stale (ternary) pages into anchors of format
    ``anchor_fmt`` (BF16 or FP8), K and V alike.  Request i names logical
    page req_page[i] of sequence req_seq[i] and the anchor-pool slot
    anchor_slot[i] it moves to.  The page's content is its dequantised value
    bf16(gamma * c) per KV head (the only content a stale page has); a BF16
    anchor stores those bf16 values, an FP8 anchor quantises the bf16 page
    with the FP8 page codec (one scale over all KV heads).  The page's
    block-table entry becomes the anchor slot, its tag becomes anchor_fmt and
    the ternary slot is reported as freed.

    Requests that name a page outside the batch or beyond the sequence's
    pages (PROMOTE_RANGE), a page that is not ternary by the page
    classification (PROMOTE_NOT_STALE) or a slot outside its pool
    (PROMOTE_SLOT) are skipped with freed = -1 and the flag OR-ed into the
    returned word.  Requests name distinct pages.

    Returns (cache', block_table', older_fmt', freed int32 [n], flags); the
    inputs are not modified."""
    import copy
    c = copy.deepcopy(cache)
    bt = np.array(block_table, dtype=np.int32, copy=True)
    tags = np.array(older_fmt, dtype=np.uint8, copy=True)
    n = len(req_seq)
    freed = np.full(n, -1, dtype=np.int32)
    flags = 0
    n_tern = c.k_tern.shape[0]
    n_anchor = (c.k_bf16 if anchor_fmt == BF16 else c.k_fp8).shape[0]
    for i in range(n):
        b, j = int(req_seq[i]), int(req_page[i])
        if not (0 <= b < bt.shape[0]):
            flags |= PROMOTE_RANGE
            continue
        L = int(context_lens[b])
        if not (0 <= j < num_pages(L)) or L > bt.shape[1] * PAGE_SIZE:
            flags |= PROMOTE_RANGE
            continue
        if page_format(j, L, sink, window, hp_fmt, int(tags[b, j])) != TERNARY:
            flags |= PROMOTE_NOT_STALE
            continue
        t, a = int(bt[b, j]), int(anchor_slot[i])
        if not (0 <= t < n_tern and 0 <= a < n_anchor):
            flags |= PROMOTE_SLOT
            continue
        for which in ("k", "v"):
            page = dequantize_ternary(getattr(c, which + "_tern")[t:t + 1],
                                      getattr(c, which + "_gamma")[t:t + 1])        # [1][Hkv][P][D]
            if anchor_fmt == BF16:
                getattr(c, which + "_bf16")[a] = page[0]
            else:
                e, sc = quantize_fp8_pages(page)
                getattr(c, which + "_fp8")[a] = e[0]
                getattr(c, which + "_fp8_scale")[a] = sc[0]
        bt[b, j] = a
        tags[b, j] = anchor_fmt
        freed[i] = t
    return c, bt, tags, freed, flags


# ---------------------------------------------------------------------------
# Storage accounting  [Vantage, "Core architecture"; Minima, "Why the KV cache
# becomes a bottleneck" and "What the memory measurements showed"]
# ---------------------------------------------------------------------------

def ternary_group_bytes(page_size: int, head_dim: int) -> int:
    """Bytes of one packed (page, KV head) group: P*D/4 codes + a 4-byte gamma."""
    return page_size * head_dim // 4 + 4


def ternary_bits_per_element(page_size: int, head_dim: int) -> float:
    return 8.0 * ternary_group_bytes(page_size, head_dim) / (page_size * head_dim)


def fp8_page_bytes(page_size: int, n_kv_heads: int, head_dim: int) -> int:
    """Bytes of one FP8 page of K (or V): P*Hkv*D codes + a 4-byte scale."""
    return page_size * n_kv_heads * head_dim + 4


def kv_bytes_per_token(n_layers: int, n_kv_heads: int, head_dim: int, bytes_per_elem: float) -> float:
    """K + V bytes per live token over all attention layers."""
    return 2.0 * n_layers * n_kv_heads * head_dim * bytes_per_elem
