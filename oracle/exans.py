"""Oracle for the lossless exponent-split codec of high-precision (BF16) pages.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: nothing in the product
package imports it; it shares no code with the CUDA path.

Source: "ExANS komprimerer KV-cache og goer AI-svar hurtigere paa H100 GPU"
(ainews.dk), summarising "ExANS - Lossless KV cache compression at 622 GB/s on
H100": a lossless GPU codec for BF16 KV caches. Each BF16 value is split into
two streams, the exponent and the sign + mantissa; exponents repeat in a KV
cache, so that stream compresses. Each physical block is processed on its own,
with one K group and one V group per layer; a centre of the exponents is taken
per group and the exponent stream is coded with a modified asymmetric numeral
system (ANS). Reported: 1.51x, decoding at 622 GB/s on an H100.

The page gives no further detail. The readings taken here (also listed in the
design notes):

* group = one page of one pool (K or V) of one layer: the page's Hkv x 16 x D
  bf16 values in their [head][token][dim] order, N values.
* centre = the most frequent exponent of the group (ties: the smallest).
* symbol = exponent - centre + 8 when that lies in 0..14, else 15, an escape
  whose exponent byte goes to an escape stream in element order.
* sign + mantissa byte = sign bit << 7 | the 7 mantissa bits, kept raw.
* coder: byte-wise rANS (Duda's asymmetric numeral systems, range variant)
  with a 32-bit state kept in [2^23, 2^31), 12-bit probabilities and a static
  table per group; 32 interleaved states share one byte stream so that a GPU
  warp decodes a group with one state per lane.  Lane i codes elements
  128c + 4i + r (chunk c, r = 0..3) in that order.  After every symbol the
  lanes whose state fell below 2^23 read one byte each in lane order, and
  then, if still below, a second byte in lane order.
* frequencies: f_s = max(1, floor(n_s * 4096 / N)) for every present symbol;
  the remainder to 4096 goes to the symbol with the largest f (smallest
  index among ties).
* a group whose coded form would be larger than its raw bytes is stored raw.

Blob of one group (little-endian, 16-byte multiple):

  0  u32 total bytes      4  u32 mode (0 raw, 1 coded)   8  u32 N
  12 u32 centre          16  u32 escapes               20  u32 rANS stream bytes
  24 8 bytes zero        32  u16 f[16]
  64 coded: N sign+mantissa bytes, the escape bytes zero-padded to 16, the
     rANS stream (32 initial states as u32, then the renormalisation bytes)
     zero-padded to 16.   raw: the N bf16 values (2N bytes).
"""

from __future__ import annotations

import numpy as np

LANES = 32
SCALE_BITS = 12
M = 1 << SCALE_BITS                 # probability scale
RANS_L = 1 << 23                    # lower bound of the state
N_SYMBOLS = 16
ESCAPE = 15
BIAS = 8                            # symbol = exponent - centre + BIAS
HEADER = 64
CHUNK = 4 * LANES                   # elements per chunk (4 per lane)


def _round16(x: int) -> int:
    return (x + 15) // 16 * 16


def split_streams(bits: np.ndarray):
    """bf16 bit patterns -> (exponent bytes, sign+mantissa bytes)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32)
    exp = ((b >> 7) & 0xFF).astype(np.uint8)
    sm = (((b >> 8) & 0x80) | (b & 0x7F)).astype(np.uint8)
    return exp, sm


def join_streams(exp: np.ndarray, sm: np.ndarray) -> np.ndarray:
    e = np.asarray(exp, dtype=np.uint32)
    s = np.asarray(sm, dtype=np.uint32)
    return (((s & 0x80) << 8) | (e << 7) | (s & 0x7F)).astype(np.uint16)


def centre(exp: np.ndarray) -> int:
    """Most frequent exponent (smallest among ties)."""
    counts = np.bincount(np.asarray(exp, dtype=np.int64), minlength=256)
    return int(np.argmax(counts))          # argmax returns the first maximum


def symbols(exp: np.ndarray, c: int) -> np.ndarray:
    d = np.asarray(exp, dtype=np.int64) - c + BIAS
    return np.where((d >= 0) & (d < ESCAPE), d, ESCAPE).astype(np.int64)


def normalise(counts: np.ndarray, n: int) -> np.ndarray:
    """Integer frequencies summing to M; every present symbol gets >= 1."""
    counts = np.asarray(counts, dtype=np.int64)
    f = np.where(counts > 0, np.maximum(1, counts * M // n), 0)
    rem = M - int(f.sum())
    s = int(np.argmax(f))
    f[s] += rem
    assert f[s] >= 1 and int(f.sum()) == M
    return f


def element_of(step: int) -> np.ndarray:
    """Element index coded by each lane at a step (k = 4c + r)."""
    c, r = divmod(step, 4)
    return c * CHUNK + 4 * np.arange(LANES) + r


def rans_encode(sym: np.ndarray, f: np.ndarray) -> bytes:
    """Interleaved rANS stream of a group's symbols (element order)."""
    n = len(sym)
    steps = n // LANES
    cum = np.concatenate([[0], np.cumsum(f)[:-1]]).astype(np.int64)
    x = np.full(LANES, RANS_L, dtype=np.int64)
    per_step = []
    for k in range(steps - 1, -1, -1):
        s = sym[element_of(k)]
        fs, cs = f[s], cum[s]
        x_max = (RANS_L >> SCALE_BITS << 8) * fs
        first = np.zeros(LANES, dtype=np.int64)     # byte the decoder reads in round 0
        second = np.zeros(LANES, dtype=np.int64)    # byte read in round 1
        nb = np.zeros(LANES, dtype=np.int64)
        # emitted low byte first; the decoder reads them in reverse
        e1 = x >= x_max
        low = x & 0xFF
        x = np.where(e1, x >> 8, x)
        nb += e1
        e2 = x >= x_max
        second = np.where(e2, low, second)
        first = np.where(e2, x & 0xFF, np.where(e1, low, first))
        x = np.where(e2, x >> 8, x)
        nb += e2
        assert not (x >= x_max).any()
        x = (x // fs << SCALE_BITS) + (x % fs) + cs
        round0 = [int(first[i]) for i in range(LANES) if nb[i] >= 1]
        round1 = [int(second[i]) for i in range(LANES) if nb[i] == 2]
        per_step.append(bytes(round0 + round1))
    head = b"".join(int(v).to_bytes(4, "little") for v in x)
    return head + b"".join(reversed(per_step))


def rans_decode(stream: bytes, f: np.ndarray, n: int) -> np.ndarray:
    """Symbols (element order) of an interleaved rANS stream."""
    cum = np.concatenate([[0], np.cumsum(f)[:-1]]).astype(np.int64)
    sym_of_slot = np.repeat(np.arange(N_SYMBOLS), f)
    x = np.array([int.from_bytes(stream[4 * i:4 * i + 4], "little") for i in range(LANES)], dtype=np.int64)
    pos = 4 * LANES
    out = np.zeros(n, dtype=np.int64)
    for k in range(n // LANES):
        slot = x & (M - 1)
        s = sym_of_slot[slot]
        out[element_of(k)] = s
        x = f[s] * (x >> SCALE_BITS) + slot - cum[s]
        for _ in range(2):
            need = x < RANS_L
            for i in np.nonzero(need)[0]:
                x[i] = (x[i] << 8) | stream[pos]
                pos += 1
    if pos != len(stream):
        raise ValueError("rANS stream not consumed exactly")
    return out


def encode_group(bits: np.ndarray) -> bytes:
    """Blob of one group of N bf16 values (N a multiple of 128)."""
    bits = np.asarray(bits, dtype=np.uint16).reshape(-1)
    n = len(bits)
    assert n % CHUNK == 0 and n > 0
    exp, sm = split_streams(bits)
    c = centre(exp)
    sym = symbols(exp, c)
    f = normalise(np.bincount(sym, minlength=N_SYMBOLS), n)
    esc = exp[sym == ESCAPE]
    stream = rans_encode(sym, f)
    esc_pad = _round16(len(esc))
    total = HEADER + n + esc_pad + _round16(len(stream))
    if total > HEADER + 2 * n:
        return _header(HEADER + 2 * n, 0, n, 0, 0, 0, np.zeros(N_SYMBOLS, np.int64)) + bits.astype("<u2").tobytes()
    body = (sm.tobytes() + esc.tobytes() + bytes(esc_pad - len(esc)) + stream
            + bytes(_round16(len(stream)) - len(stream)))
    return _header(total, 1, n, c, len(esc), len(stream), f) + body


def _header(total, mode, n, c, n_esc, n_stream, f) -> bytes:
    h = b"".join(int(v).to_bytes(4, "little") for v in (total, mode, n, c, n_esc, n_stream))
    h += bytes(8) + b"".join(int(v).to_bytes(2, "little") for v in f)
    assert len(h) == HEADER
    return h


def parse_header(blob: bytes) -> dict:
    u32 = [int.from_bytes(blob[4 * i:4 * i + 4], "little") for i in range(6)]
    f = np.array([int.from_bytes(blob[32 + 2 * i:34 + 2 * i], "little") for i in range(N_SYMBOLS)], np.int64)
    return dict(total=u32[0], mode=u32[1], n=u32[2], centre=u32[3], escapes=u32[4], stream=u32[5], f=f)


def decode_group(blob: bytes) -> np.ndarray:
    h = parse_header(blob)
    n = h["n"]
    if h["mode"] == 0:
        return np.frombuffer(blob[HEADER:HEADER + 2 * n], dtype="<u2").astype(np.uint16)
    sm = np.frombuffer(blob[HEADER:HEADER + n], dtype=np.uint8)
    e0 = HEADER + n
    esc = np.frombuffer(blob[e0:e0 + h["escapes"]], dtype=np.uint8)
    s0 = e0 + _round16(h["escapes"])
    sym = rans_decode(blob[s0:s0 + h["stream"]], h["f"], n)
    exp = (sym - BIAS + h["centre"]).astype(np.int64)
    is_esc = sym == ESCAPE
    if int(is_esc.sum()) != len(esc):
        raise ValueError("escape count mismatch")
    exp[is_esc] = esc
    return join_streams(exp.astype(np.uint8), sm)


def encode_pages(pages_bits: np.ndarray, page_ids=None):
    """Pages [n_src][Hkv][16][D] bf16 bits -> (pool bytes, offsets int64 [n+1]):
    the blobs of the selected pages back to back, offsets[i] where page i's
    blob starts (offsets[n] = total)."""
    src = np.asarray(pages_bits, dtype=np.uint16)
    ids = np.arange(src.shape[0]) if page_ids is None else np.asarray(page_ids)
    blobs = [encode_group(src[i].reshape(-1)) for i in ids]
    offsets = np.zeros(len(blobs) + 1, dtype=np.int64)
    offsets[1:] = np.cumsum([len(b) for b in blobs])
    return b"".join(blobs), offsets


def decode_pages(pool: bytes, offsets: np.ndarray, shape) -> np.ndarray:
    """Inverse of encode_pages: bf16 bits [n][Hkv][16][D]."""
    n = len(offsets) - 1
    out = np.zeros((n,) + tuple(shape), dtype=np.uint16)
    for i in range(n):
        out[i] = decode_group(pool[offsets[i]:offsets[i + 1]]).reshape(shape)
    return out
