"""Decode parity where the kernel's own number formats are stressed.

The decode kernel never sees Q in its given bf16 form on ternary pages: it
re-expresses each query head in fixed point (int8 digits of one scale per
head) to use integer tensor-core products with the 2-bit codes.  The error of
that step grows with the dynamic range of Q, not with any one value, so
these cases give Q outlier channels (decoder queries have them; the ternary
codec of "Show HN: Vantage-V-AI", section "Core architecture", quantises K
and V only, Q stays full precision).  The same holds for the f16 operands of
the high-precision pages: a BF16 value beyond the f16 range must not turn
into a silent inf.

Every case is compared with the fp64 oracle over the same packed pages, at
the attention bar (max-abs 2e-3, rel-L2 1e-3)."""

import numpy as np
import pytest
import torch

import oracle as O
import synth
import compressed_decode_attention_kvc_b200 as K
from kvc_testlib import (HP, assert_attention_close, bits, lib_older_fmt, oracle_build_from_inputs,
                         run_decode, upload_oracle_cache)

pytestmark = pytest.mark.gpu

SHAPES = [(64, 8, 4), (128, 16, 4), (128, 16, 2), (256, 12, 2)]   # (head_dim, Hq, Hkv): GQA 2, 4, 8, 6


def _q_outliers(q: torch.Tensor, pattern: str, seed: int) -> torch.Tensor:
    """Scale channels of Q (input construction, float32 then back to bf16)."""
    g = torch.Generator().manual_seed(seed)
    x = q.float().clone()
    B, hq, d = x.shape
    if pattern == "channels_x100":          # 1% of the (head, dim) channels x100, same for every sequence
        n = max(1, round(0.01 * hq * d))
        idx = torch.randperm(hq * d, generator=g)[:n]
        x.view(B, hq * d)[:, idx] *= 100.0
    elif pattern == "one_channel_x1000":    # a single dim of every query head x1000
        dim = int(torch.randint(0, d, (1,), generator=g))
        x[:, :, dim] *= 1000.0
    elif pattern == "head_range_1e3":       # one query head with max|q| = 1e3 x its median
        h = int(torch.randint(0, hq, (1,), generator=g))
        med = x[:, h].abs().median(dim=-1, keepdim=True).values
        dim = int(torch.randint(0, d, (1,), generator=g))
        x[:, h, dim] = torch.sign(x[:, h, dim] + 0.5) * 1000.0 * med[:, 0]
    return x.to(torch.bfloat16)


def _run(inp, dev, hp="bf16"):
    cfg = inp["cfg"]
    cache, bt, fmt, older = oracle_build_from_inputs(inp, HP[hp])
    _, struct = upload_oracle_cache(cache, dev)
    B, max_pages = bt.shape
    out, ws = run_decode(inp["q"].to(dev), struct, torch.from_numpy(bt).to(dev), lib_older_fmt(older, dev),
                         inp["context_lens"].to(dev), cfg["n_kv_heads"], max_pages, cfg["sink"], cfg["window"],
                         HP[hp])
    torch.cuda.synchronize()
    flags = K.kvc_decode_read_error(ws, B, cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"], max_pages)
    ref = O.decode_attention(bits(inp["q"]), cache, bt, fmt, inp["context_lens"].numpy(), cfg["n_kv_heads"])
    return out.cpu().numpy(), ref, flags


@pytest.mark.parametrize("pattern", ["channels_x100", "one_channel_x1000", "head_range_1e3"])
@pytest.mark.parametrize("d,hq,hkv", SHAPES)
def test_q_outliers_match_oracle(cuda_device, d, hq, hkv, pattern):
    inp = synth.make_decode_inputs("tiny", seed=11 + d + hq, batch=2, n_q_heads=hq, n_kv_heads=hkv,
                                   head_dim=d, context=16 * 21 + 3, window=40, sink=4, hp="bf16")
    inp["q"] = _q_outliers(inp["q"], pattern, seed=d * 7 + hq)
    out, ref, flags = _run(inp, cuda_device)
    assert flags == 0
    assert_attention_close(out, ref, f"{pattern} D={d} G={hq // hkv}")


@pytest.mark.parametrize("d", [64, 128, 256])
def test_bf16_page_beyond_f16_range(cuda_device, d):
    # a sink/window (BF16) page holding values beyond +-65504: BF16 pages are
    # multiplied in bf16 as stored, so they decode like any other page
    inp = synth.make_decode_inputs("tiny", seed=5 + d, batch=2, n_q_heads=8, n_kv_heads=4, head_dim=d,
                                   context=16 * 9 + 5, window=40, sink=4, hp="bf16")
    k = inp["k_pages"].float()
    v = inp["v_pages"].float()
    k[0, 0, 1, 3, 5] = 1.2e5                 # page 0 (sink, BF16) of sequence 0
    v[0, 0, 2, 7, 9] = -9.0e4
    v[1, 9, 0, 2, 4] = 2.0e5                 # the last (window) page of sequence 1
    inp["k_pages"] = k.to(torch.bfloat16)
    inp["v_pages"] = v.to(torch.bfloat16)
    out, ref, flags = _run(inp, cuda_device)
    assert flags == 0 and np.isfinite(out).all()
    # values of 1e5 make output rows of ~1e4, where the fp32 spacing alone is
    # ~1e-3: the absolute bar scales with the largest output magnitude, the
    # relative one stands as is
    scale = max(1.0, float(np.abs(ref).max()))
    diff = np.abs(out.astype(np.float64) - ref)
    assert float(diff.max()) <= 2e-3 * scale, float(diff.max())
    rel = float(np.linalg.norm(diff)) / float(np.linalg.norm(ref))
    assert rel <= 1e-3, rel


@pytest.mark.parametrize("ramp", ["rising", "sawtooth"])
@pytest.mark.parametrize("d,hq,hkv", [(64, 8, 4), (128, 16, 4), (256, 8, 4), (128, 16, 2)])
def test_moving_maximum_matches_oracle(cuda_device, d, hq, hkv, ramp):
    # keys built so that the scores keep rising along the sequence (or rise
    # and fall back every few pages): the running maximum moves on almost
    # every page, so the kernel rescales its partial sums many times after
    # they have accumulated (the digit sums of the int8 P.V path by exact
    # shifts, the fp32 sums by powers of two)
    inp = synth.make_decode_inputs("tiny", seed=3 + d + hq, batch=2, n_q_heads=hq, n_kv_heads=hkv,
                                   head_dim=d, context=16 * 40 + 7, window=20, sink=4, hp="bf16")
    q = inp["q"].float()
    k = inp["k_pages"].float()
    B, max_pages, _, P, _ = k.shape
    g = hq // hkv
    # the mean query direction of each KV head's group
    u = q.view(B, hkv, g, d).mean(dim=2)
    u = u / u.norm(dim=-1, keepdim=True)
    pos = torch.arange(max_pages * P, dtype=torch.float32).view(max_pages, P) / (max_pages * P)
    if ramp == "sawtooth":
        pos = torch.remainder(pos * 7.0, 1.0)
    amp = 6.0 * d ** 0.5                      # ~+6 score units per unit of pos per |q| along u
    k += amp * pos.view(1, max_pages, 1, P, 1) * u.view(B, 1, hkv, 1, d)
    inp["k_pages"] = k.to(torch.bfloat16)
    out, ref, flags = _run(inp, cuda_device)
    assert flags == 0
    assert_attention_close(out, ref, f"{ramp} D={d} G={g}")
