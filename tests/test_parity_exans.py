"""The exponent-split lossless codec of BF16 pages (kvc_exans_encode /
kvc_exans_decode) against the oracle, through the C ABI.

Bar: the coded pool and its offsets bit-exact against the oracle's blobs
(both sides take the same integer steps); decoding gives back the input
bits exactly (lossless), from the GPU's blobs and from the oracle's."""

import numpy as np
import pytest
import torch

import oracle.exans as X
import compressed_decode_attention_kvc_b200 as K
from kvc_testlib import bits, from_bits

pytestmark = pytest.mark.gpu


def _pages(kind, n, hkv, d, seed):
    rng = np.random.default_rng(seed)
    shape = (n, hkv, 16, d)
    if kind == "normal":
        x = rng.standard_normal(shape)
    elif kind == "outlier_channels":
        x = rng.standard_normal(shape)
        x[..., rng.random(d) < 0.02] *= 10.0
    elif kind == "channel_offset":
        x = rng.standard_normal(shape) + rng.normal(0, np.sqrt(2), (1, hkv, 1, d))
    elif kind == "laplace":
        x = rng.laplace(size=shape)
    elif kind == "mixed":
        x = rng.standard_normal(shape) * (10.0 ** rng.integers(-30, 30, size=(n, 1, 1, 1)))
        x[0] = 0.0
    b = torch.tensor(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    if kind == "mixed":
        b[1] = rng.integers(0, 65536, size=shape[1:], dtype=np.uint32).astype(np.uint16)   # any pattern
        b[2] = 0x3F80
    return b


def _encode_gpu(pages_bits, ids, hkv, d, dev):
    n = len(ids) if ids is not None else pages_bits.shape[0]
    src = from_bits(pages_bits, dev)
    ws_bytes = K.kvc_exans_workspace_size(n, 16, hkv, d)
    ws = torch.full((ws_bytes,), 0xA5, dtype=torch.uint8, device=dev)
    N = hkv * 16 * d
    dst_bytes = n * (64 + 2 * N)
    dst = torch.full((dst_bytes,), 0x5A, dtype=torch.uint8, device=dev)
    off = torch.full((n + 1,), -7, dtype=torch.int64, device=dev)
    ids_d = None if ids is None else torch.tensor(ids, dtype=torch.int32, device=dev)
    K.kvc_exans_encode(src, ids_d, n, 16, hkv, d, ws, ws_bytes, dst, dst_bytes, off)
    torch.cuda.synchronize()
    return dst, off


@pytest.mark.parametrize("kind,n,hkv,d", [("normal", 6, 8, 128), ("outlier_channels", 5, 2, 128),
                                          ("channel_offset", 4, 8, 128), ("laplace", 3, 4, 256),
                                          ("mixed", 7, 1, 64), ("normal", 9, 4, 64)])
def test_encode_matches_oracle_and_round_trips(cuda_device, kind, n, hkv, d):
    pages = _pages(kind, n, hkv, d, seed=n * 100 + d)
    ids = list(np.random.default_rng(1).permutation(n))[: n - 1] + [0]       # a subset, one page twice
    pool_ref, off_ref = X.encode_pages(pages, ids)
    dst, off = _encode_gpu(pages, ids, hkv, d, cuda_device)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    got = dst[: int(off_ref[-1])].cpu().numpy().tobytes()
    if got != pool_ref:
        for i in range(len(ids)):
            a, b = got[off_ref[i]:off_ref[i + 1]], pool_ref[off_ref[i]:off_ref[i + 1]]
            if a != b:
                k = next(j for j in range(len(a)) if a[j] != b[j])
                raise AssertionError(f"blob {i}: first differing byte {k} of {len(a)} "
                                     f"(header {X.parse_header(b)})")
    # decode the GPU's pool on the GPU: the input pages exactly
    out = torch.full((len(ids), hkv, 16, d), 0x7FC0, dtype=torch.int16, device=cuda_device).view(torch.bfloat16)
    flags = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    K.kvc_exans_decode(dst, dst.numel(), off, len(ids), None, len(ids), 16, hkv, d, out, flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    assert np.array_equal(bits(out.cpu()), pages[ids])


def test_decode_oracle_pool_with_blob_ids(cuda_device):
    hkv, d, n = 8, 128, 8
    pages = _pages("channel_offset", n, hkv, d, seed=3)
    pool, off = X.encode_pages(pages)
    assert len({X.parse_header(pool[off[i]:off[i + 1]])["mode"] for i in range(n)}) == 1
    src = torch.from_numpy(np.frombuffer(pool, np.uint8).copy()).to(cuda_device)
    off_d = torch.from_numpy(off).to(cuda_device)
    want = [5, 0, 7, 7, 2]
    out = torch.zeros((len(want), hkv, 16, d), dtype=torch.bfloat16, device=cuda_device)
    flags = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    K.kvc_exans_decode(src, src.numel(), off_d, n, torch.tensor(want, dtype=torch.int32, device=cuda_device),
                       len(want), 16, hkv, d, out, flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    assert np.array_equal(bits(out.cpu()), pages[want])


def test_decode_flags_bad_ids_and_headers(cuda_device):
    hkv, d, n = 2, 64, 3
    pages = _pages("normal", n, hkv, d, seed=4)
    pool, off = X.encode_pages(pages)
    raw = bytearray(pool)
    # blob 1: a header total that disagrees with the offsets
    raw[off[1]:off[1] + 4] = (int(off[2] - off[1]) + 16).to_bytes(4, "little")
    src = torch.from_numpy(np.frombuffer(bytes(raw), np.uint8).copy()).to(cuda_device)
    off_d = torch.from_numpy(off).to(cuda_device)
    sentinel = 0x1234
    out = torch.full((4, hkv, 16, d), sentinel, dtype=torch.int16, device=cuda_device).view(torch.bfloat16)
    flags = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    ids = torch.tensor([0, 1, 9, 2], dtype=torch.int32, device=cuda_device)   # 1: bad header, 9: no such blob
    K.kvc_exans_decode(src, src.numel(), off_d, n, ids, 4, 16, hkv, d, out, flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 1
    o = bits(out.cpu())
    assert np.array_equal(o[0], pages[0]) and np.array_equal(o[3], pages[2])
    assert (o[1] == sentinel).all() and (o[2] == sentinel).all()
