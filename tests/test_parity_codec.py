"""GPU parity of the page codecs (kvc_quantize_pack_pages,
kvc_dequantize_pages) against the oracle, through the C ABI."""

import numpy as np
import pytest
import torch

import oracle as O
import synth
import compressed_decode_attention_kvc_b200 as K
from kvc_testlib import bits, check_ternary, from_bits

pytestmark = pytest.mark.gpu


def _rand_pages(n, hkv, d, seed, dev, dist="normal"):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn((n, hkv, 16, d), generator=g)
    if dist == "outlier":
        x[..., :3] *= 10
    if dist == "laplace":
        u = torch.rand((n, hkv, 16, d), generator=g, dtype=torch.float64) - 0.5
        x = (-torch.sign(u) * torch.log1p(-2 * u.abs())).float()
    return x.to(torch.bfloat16).to(dev)


def _quant(src, mode, n=None, page_ids=None):
    nsrc, hkv, p, d = src.shape
    n = nsrc if n is None else n
    dev = src.device
    if mode == K.KVC_FMT_TERNARY2:
        dst = torch.full((n, hkv, 16, d // 4), 0xAA, dtype=torch.uint8, device=dev)
        sc = torch.full((n, hkv), float("nan"), device=dev)
    elif mode == K.KVC_FMT_FP8_E4M3:
        dst = torch.full((n, hkv, 16, d), 0x7F, dtype=torch.uint8, device=dev)
        sc = torch.full((n,), float("nan"), device=dev)
    else:
        dst = torch.empty((n, hkv, 16, d), dtype=torch.bfloat16, device=dev)
        sc = None
    K.kvc_quantize_pack_pages(src, page_ids, n, 16, hkv, d, mode, dst, sc)
    torch.cuda.synchronize()
    return dst, sc


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("hkv", [1, 3, 8])
@pytest.mark.parametrize("dist", ["normal", "outlier", "laplace"])
def test_ternary_quantize_matches_oracle(cuda_device, d, hkv, dist):
    src = _rand_pages(37, hkv, d, seed=d * 10 + hkv, dev=cuda_device, dist=dist)
    codes, gamma = _quant(src, K.KVC_FMT_TERNARY2)
    check_ternary(codes.cpu().numpy(), gamma.cpu().numpy(), bits(src))


def test_ternary_special_groups(cuda_device):
    x = torch.zeros((4, 2, 16, 128))
    x[1] = 0.375 * torch.sign(torch.randn((2, 16, 128)))        # all |x| equal: gamma = 0.375
    x[2, :, :, :64] = 1.5
    x[2, :, :, 64:] = 0.5                                         # gamma 1, exact ties at 0.5 -> 0
    x[3] = torch.randn((2, 16, 128)) * 1e-3
    src = x.to(torch.bfloat16).to(cuda_device)
    codes, gamma = _quant(src, K.KVC_FMT_TERNARY2)
    g = gamma.cpu().numpy()
    assert (g[0] == 0).all() and (codes[0] == 0).all()
    assert (g[1] == np.float32(0.375)).all() and (g[2] == 1.0).all()
    c2 = O.unpack_ternary(codes[2].cpu().numpy())
    assert (c2[..., :64] == 1).all() and (c2[..., 64:] == 0).all()
    check_ternary(codes.cpu().numpy(), g, bits(src))


def test_page_ids_gather_and_order(cuda_device):
    src = _rand_pages(20, 2, 128, seed=5, dev=cuda_device)
    ids = torch.tensor([19, 0, 7, 7, 3], dtype=torch.int32, device=cuda_device)
    for mode in (K.KVC_FMT_TERNARY2, K.KVC_FMT_FP8_E4M3, K.KVC_FMT_BF16):
        full, full_s = _quant(src, mode)
        sub, sub_s = _quant(src, mode, n=5, page_ids=ids)
        idx = ids.long().cpu()
        assert torch.equal(sub.cpu(), full.cpu()[idx])
        if full_s is not None:
            assert torch.equal(sub_s.cpu(), full_s.cpu()[idx])


@pytest.mark.parametrize("d,hkv", [(64, 4), (128, 2), (128, 4), (128, 8), (256, 4), (256, 8), (64, 3), (64, 1)])
def test_fp8_quantize_bit_exact(cuda_device, d, hkv):
    src = _rand_pages(29, hkv, d, seed=d + hkv, dev=cuda_device, dist="outlier")
    src[3].zero_()
    src[4, 0, 0, 0] = -0.0
    q, s = _quant(src, K.KVC_FMT_FP8_E4M3)
    q_o, s_o = O.quantize_fp8_pages(bits(src))
    assert np.array_equal(s.cpu().numpy(), s_o)
    assert np.array_equal(q.cpu().numpy(), q_o)


def test_fp8_every_bf16_value(cuda_device):
    # all finite bf16 bit patterns, in pages whose amax is 448 (scale 1, inv 1)
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        v = O.bf16_to_f64(b)
    b = b[np.isfinite(v) & (np.abs(v) <= 448.0)]
    per = 16 * 64
    n = -(-len(b) // (per - 1))
    pages = np.zeros((n, 1, 16, 64), np.uint16)
    flat = pages.reshape(n, per)
    flat[:, 0] = 0x43E0                                   # 448.0 in every page
    vals = np.concatenate([b, np.zeros(n * (per - 1) - len(b), np.uint16)])
    flat[:, 1:] = vals.reshape(n, per - 1)
    src = from_bits(pages, cuda_device)
    q, s = _quant(src, K.KVC_FMT_FP8_E4M3)
    q_o, s_o = O.quantize_fp8_pages(pages)
    assert (s_o == 1.0).all() and np.array_equal(s.cpu().numpy(), s_o)
    assert np.array_equal(q.cpu().numpy(), q_o)


def test_bf16_copy(cuda_device):
    src = _rand_pages(9, 3, 64, seed=9, dev=cuda_device)
    out, _ = _quant(src, K.KVC_FMT_BF16)
    assert torch.equal(out, src)


@pytest.mark.parametrize("d,hkv", [(64, 2), (128, 8), (256, 4)])
def test_dequantize_bit_exact(cuda_device, d, hkv):
    src = _rand_pages(23, hkv, d, seed=3 * d + hkv, dev=cuda_device, dist="laplace")
    n = 23
    # ternary, from the oracle's own packed pages
    codes_o, gamma_o = O.quantize_pack_ternary(bits(src))
    out = torch.empty((n, hkv, 16, d), dtype=torch.bfloat16, device=cuda_device)
    K.kvc_dequantize_pages(torch.from_numpy(codes_o).to(cuda_device), torch.from_numpy(gamma_o).to(cuda_device),
                           None, n, 16, hkv, d, K.KVC_FMT_TERNARY2, out)
    torch.cuda.synchronize()
    assert np.array_equal(bits(out), O.dequantize_ternary(codes_o, gamma_o))
    # fp8
    q_o, s_o = O.quantize_fp8_pages(bits(src))
    K.kvc_dequantize_pages(torch.from_numpy(q_o).to(cuda_device), torch.from_numpy(s_o).to(cuda_device),
                           None, n, 16, hkv, d, K.KVC_FMT_FP8_E4M3, out)
    torch.cuda.synchronize()
    assert np.array_equal(bits(out), O.dequantize_fp8(q_o, s_o))
    # gather order
    ids = torch.tensor([5, 1], dtype=torch.int32, device=cuda_device)
    out2 = torch.empty((2, hkv, 16, d), dtype=torch.bfloat16, device=cuda_device)
    K.kvc_dequantize_pages(torch.from_numpy(q_o).to(cuda_device), torch.from_numpy(s_o).to(cuda_device),
                           ids, 2, 16, hkv, d, K.KVC_FMT_FP8_E4M3, out2)
    torch.cuda.synchronize()
    assert np.array_equal(bits(out2), O.dequantize_fp8(q_o[[5, 1]], s_o[[5, 1]]))


def test_bulk_workload_full_size_sampled(cuda_device):
    """The bulk-compression workload at full size (1 GiB bf16), in the
    launch configuration the benchmark times; pages compared with the
    oracle on a sample."""
    pages = synth.make_bulk_pages(seed=0, device=cuda_device)        # [32768][8][16][128]
    n, hkv, _, d = pages.shape
    codes, gamma = _quant(pages, K.KVC_FMT_TERNARY2)
    rt = torch.empty_like(pages)
    K.kvc_dequantize_pages(codes, gamma, None, n, 16, hkv, d, K.KVC_FMT_TERNARY2, rt)
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    sample = np.unique(np.concatenate([[0, n - 1], rng.integers(0, n, 48)]))
    idx = torch.from_numpy(sample).to(cuda_device)
    check_ternary(codes[idx].cpu().numpy(), gamma[idx].cpu().numpy(), bits(pages[idx]))
    assert np.array_equal(bits(rt[idx]), O.dequantize_ternary(codes[idx].cpu().numpy(), gamma[idx].cpu().numpy()))
    # properties that hold everywhere: gamma > 0, no field 10 anywhere
    assert bool((gamma > 0).all())
    c = codes.view(torch.uint8)
    for sh in (0, 2, 4, 6):
        assert not bool((((c >> sh) & 3) == 2).any())
    del rt, codes, gamma
    q, s = _quant(pages, K.KVC_FMT_FP8_E4M3)
    q_o, s_o = O.quantize_fp8_pages(bits(pages[idx]))
    assert np.array_equal(q[idx].cpu().numpy(), q_o) and np.array_equal(s[idx].cpu().numpy(), s_o)


@pytest.mark.parametrize("mode", [K.KVC_FMT_TERNARY2, K.KVC_FMT_FP8_E4M3, K.KVC_FMT_BF16])
@pytest.mark.parametrize("d", [64, 256])
def test_bad_page_ids_are_skipped_and_flagged(cuda_device, mode, d):
    # host-built ids with two entries outside the 9 source pages: those
    # output pages keep their sentinel bytes, the rest match the oracle's
    # codec on the pages named, and bit 1 of the flag word is set
    hkv, n_src = 2, 9
    src = _rand_pages(n_src, hkv, d, seed=77 + d, dev=cuda_device)
    ids_h = np.array([3, -1, 0, 8, n_src + 4, 5], dtype=np.int32)
    ids = torch.from_numpy(ids_h).to(cuda_device)
    n = len(ids_h)
    flags = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    if mode == K.KVC_FMT_TERNARY2:
        dst = torch.full((n, hkv, 16, d // 4), 0xAA, dtype=torch.uint8, device=cuda_device)
        sc = torch.full((n, hkv), -7.0, device=cuda_device)
    elif mode == K.KVC_FMT_FP8_E4M3:
        dst = torch.full((n, hkv, 16, d), 0x7F, dtype=torch.uint8, device=cuda_device)
        sc = torch.full((n,), -7.0, device=cuda_device)
    else:
        dst = torch.full((n, hkv, 16, d), 5.0, dtype=torch.bfloat16, device=cuda_device)
        sc = None
    K.kvc_quantize_pack_pages(src, ids, n, 16, hkv, d, mode, dst, sc, n_src_pages=n_src, device_flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 1
    good = np.array([0 <= i < n_src for i in ids_h])
    out = dst.cpu()
    src_b = bits(src)
    if mode == K.KVC_FMT_TERNARY2:
        assert (out[~good] == 0xAA).all() and (sc.cpu()[~good] == -7.0).all()
        check_ternary(out[good].numpy(), sc.cpu()[good].numpy(), src_b[ids_h[good]])
    elif mode == K.KVC_FMT_FP8_E4M3:
        assert (out[~good] == 0x7F).all() and (sc.cpu()[~good] == -7.0).all()
        q_o, s_o = O.quantize_fp8_pages(src_b[ids_h[good]])
        assert np.array_equal(out[good].numpy(), q_o) and np.array_equal(sc.cpu()[good].numpy(), s_o)
    else:
        assert (out[~good].float() == 5.0).all()
        assert np.array_equal(bits(out[good]), src_b[ids_h[good]])
    # dequantise from the n compressed pages just made, two ids outside them
    if mode != K.KVC_FMT_BF16:
        ids2 = torch.tensor([0, 2, n + 3, -5], dtype=torch.int32, device=cuda_device)
        rt = torch.full((4, hkv, 16, d), 3.0, dtype=torch.bfloat16, device=cuda_device)
        flags.zero_()
        K.kvc_dequantize_pages(dst, sc, ids2, 4, 16, hkv, d, mode, rt, n_src_pages=n, device_flags=flags)
        torch.cuda.synchronize()
        assert int(flags.item()) == 1
        assert (rt.cpu()[2:].float() == 3.0).all()
        if mode == K.KVC_FMT_TERNARY2:
            ref = O.dequantize_ternary(out[[0, 2]].numpy(), sc.cpu()[[0, 2]].numpy())
        else:
            ref = O.dequantize_fp8(out[[0, 2]].numpy(), sc.cpu()[[0, 2]].numpy())
        assert np.array_equal(bits(rt[:2]), ref)
