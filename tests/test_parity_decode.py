"""GPU parity of kvc_decode_attention_paged against the fp64 oracle.

Small cases: the GPU reads the oracle's packed pages (uploaded) and every
output is compared.  Full-size cases: the cache is built by the library
itself (planner + pack kernels, the benchmark's launch configuration); the
sampled sequences' pages are checked against the oracle's and then replaced
by the oracle's bytes, so that their attention rows can be compared with the
oracle's fp64 attention; every row is checked against properties that hold
at any size."""

import numpy as np
import pytest
import torch

import oracle as O
import synth
import compressed_decode_attention_kvc_b200 as K
from compressed_decode_attention_kvc_b200 import paged_cache as PC
from kvc_testlib import (HP, assert_attention_close, bits, check_ternary, lib_older_fmt,
                         oracle_build_from_inputs, run_decode, upload_oracle_cache)

pytestmark = pytest.mark.gpu


def _decode_vs_oracle(inp, dev, softmax_scale=0.0):
    cfg = inp["cfg"]
    hp = HP[cfg["hp"]]
    cache, bt, fmt, older = oracle_build_from_inputs(inp, hp)
    t, struct = upload_oracle_cache(cache, dev)
    q = inp["q"].to(dev)
    B, max_pages = bt.shape
    out, ws = run_decode(q, struct, torch.from_numpy(bt).to(dev), lib_older_fmt(older, dev),
                         inp["context_lens"].to(dev), cfg["n_kv_heads"], max_pages, cfg["sink"],
                         cfg["window"], hp, softmax_scale)
    torch.cuda.synchronize()
    flags = K.kvc_decode_read_error(ws, B, cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"], max_pages)
    assert flags == 0
    ref = O.decode_attention(bits(inp["q"]), cache, bt, fmt, inp["context_lens"].numpy(),
                             cfg["n_kv_heads"], softmax_scale)
    return out.cpu().numpy(), ref, fmt


def test_tiny_workload_full(cuda_device):
    inp = synth.make_decode_inputs("tiny", seed=0)
    out, ref, fmt = _decode_vs_oracle(inp, cuda_device)
    assert (fmt[0, :32] == O.BF16).sum() == 5 and (fmt[0, :32] == O.TERNARY).sum() == 27
    assert_attention_close(out, ref, "tiny")


@pytest.mark.parametrize("name,over", [
    ("qwen3b", dict(batch=3, context=1024 + 7)),                       # FP8 window, outlier channels
    ("llama8b", dict(batch=2, context=2048, window=256)),              # BF16 window, permuted slots
    ("longctx", dict(batch=3, context=(200, 3000), window=300)),       # D=256, G=6, anchors, ragged
])
def test_workloads_reduced_full_compare(cuda_device, name, over):
    inp = synth.make_decode_inputs(name, seed=1, **over)
    out, ref, fmt = _decode_vs_oracle(inp, cuda_device)
    assert_attention_close(out, ref, name)


@pytest.mark.parametrize("d,hq,hkv", [(64, 4, 4), (128, 8, 1), (256, 16, 2), (128, 6, 2)])
@pytest.mark.parametrize("hp", ["bf16", "fp8"])
def test_shapes_and_formats(cuda_device, d, hq, hkv, hp):
    inp = synth.make_decode_inputs("tiny", seed=d + hq, batch=3, n_q_heads=hq, n_kv_heads=hkv,
                                   head_dim=d, context=16 * 13 + 5, window=40, sink=4, hp=hp)
    g = torch.Generator().manual_seed(7)
    inp["anchor"] = torch.rand(inp["anchor"].shape, generator=g) < 0.2
    inp["context_lens"] = torch.tensor([16 * 13 + 5, 1, 17], dtype=torch.int32)
    out, ref, _ = _decode_vs_oracle(inp, cuda_device, softmax_scale=0.05 if d == 64 else 0.0)
    assert_attention_close(out, ref, f"{d},{hq},{hkv},{hp}")


def test_edge_lengths_and_windows(cuda_device):
    # L = 0 (zero row), L = 1, exact page multiples, no sink, no window (a
    # partial ternary last page), and a window longer than the context
    for sink, window in ((0, 0), (0, 1), (17, 0), (4, 10**6)):
        inp = synth.make_decode_inputs("tiny", seed=3, batch=6, context=16 * 8, sink=sink, window=window)
        inp["context_lens"] = torch.tensor([0, 1, 16, 16 * 8, 16 * 5 + 3, 33], dtype=torch.int32)
        out, ref, _ = _decode_vs_oracle(inp, cuda_device)
        assert np.all(out[0] == 0.0)
        assert_attention_close(out, ref, f"sink={sink} window={window}")


def test_large_batch_uses_cuda_core_kernel(cuda_device):
    # more sequences than the tensor-core kernel's per-CTA sequence table
    # holds: the CUDA-core kernel serves the call
    inp = synth.make_decode_inputs("tiny", seed=6, batch=1100, context=16 * 3, window=8, n_q_heads=4,
                                   n_kv_heads=2)
    g = torch.Generator().manual_seed(3)
    inp["context_lens"] = torch.randint(0, 16 * 3 + 1, (1100,), generator=g, dtype=torch.int32)
    out, ref, _ = _decode_vs_oracle(inp, cuda_device)
    assert_attention_close(out, ref, "batch 1100")


def test_repeated_calls_reuse_workspace(cuda_device):
    inp = synth.make_decode_inputs("qwen3b", seed=4, batch=2, context=700)
    cfg = inp["cfg"]
    cache, bt, fmt, older = oracle_build_from_inputs(inp, HP[cfg["hp"]])
    t, struct = upload_oracle_cache(cache, cuda_device)
    q = inp["q"].to(cuda_device)
    args = (struct, torch.from_numpy(bt).to(cuda_device), None, inp["context_lens"].to(cuda_device),
            cfg["n_kv_heads"], bt.shape[1], cfg["sink"], cfg["window"], HP[cfg["hp"]])
    out1, ws = run_decode(q, *args)
    out2, _ = run_decode(q, *args, workspace=ws)
    out3, _ = run_decode(q, *args, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2) and torch.equal(out2, out3)


def test_device_checks_flag_bad_block_table(cuda_device):
    inp = synth.make_decode_inputs("tiny", seed=5, batch=2)
    cfg = inp["cfg"]
    cache, bt, fmt, older = oracle_build_from_inputs(inp, K.KVC_FMT_BF16)
    t, struct = upload_oracle_cache(cache, cuda_device)
    bad = bt.copy()
    bad[1, 5] = 10**6                                # outside the ternary pool
    bad[0, 3] = -2
    q = inp["q"].to(cuda_device)
    out, ws = run_decode(q, struct, torch.from_numpy(bad).to(cuda_device), None,
                         inp["context_lens"].to(cuda_device), cfg["n_kv_heads"], bt.shape[1],
                         cfg["sink"], cfg["window"], K.KVC_FMT_BF16)
    flags = K.kvc_decode_read_error(ws, 2, cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"], bt.shape[1])
    assert flags & K.ERR_BLOCK_TABLE
    assert torch.isfinite(out).all()
    assert K.kvc_decode_read_error(ws, 2, cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"], bt.shape[1]) == 0
    lens = inp["context_lens"].clone()
    lens[0] = 10**6                                  # longer than max_pages * 16
    out, ws = run_decode(q, struct, torch.from_numpy(bt).to(cuda_device), None, lens.to(cuda_device),
                         cfg["n_kv_heads"], bt.shape[1], cfg["sink"], cfg["window"], K.KVC_FMT_BF16)
    assert K.kvc_decode_read_error(ws, 2, cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"], bt.shape[1]) & K.ERR_CONTEXT


# ----------------------------------------------------------------- full size

def _full_size_check(name, dev, sample_b, seed=0):
    inp = synth.make_decode_inputs(name, seed=seed, device=dev)
    cfg = inp["cfg"]
    hp = HP[cfg["hp"]]
    B, max_pages, hkv, P, D = inp["k_pages"].shape
    hq = cfg["n_q_heads"]
    older = None
    if inp["anchor"].any():
        older = torch.where(inp["anchor"], K.KVC_FMT_BF16, K.KVC_FMT_TERNARY2).to(torch.uint8)
    lens_h = inp["context_lens"].cpu()
    layout = PC.plan_paged_cache(lens_h, max_pages, cfg["sink"], cfg["window"], hp,
                                 older_fmt=None if older is None else older.cpu(),
                                 slot_key=None if inp["slot_key"] is None else inp["slot_key"].cpu())
    cache = PC.allocate_device_cache(layout, hkv, D, dev)
    kf = inp["k_pages"].view(B * max_pages, hkv, P, D)
    vf = inp["v_pages"].view(B * max_pages, hkv, P, D)
    PC.compress_into(cache, kf, vf)
    torch.cuda.synchronize()

    bt = layout.block_table.numpy()
    pf = layout.page_fmt.numpy()
    pools = cache.pools
    refs = {}
    for b in sample_b:
        L = int(lens_h[b])
        sub = {k: (v[b:b + 1] if isinstance(v, torch.Tensor) and v.dim() > 0 and v.shape[0] == B else v)
               for k, v in inp.items()}
        sub["context_lens"] = lens_h[b:b + 1]
        sub["anchor"] = inp["anchor"][b:b + 1].cpu()
        sub["slot_key"] = None
        oc, obt, ofmt, _ = oracle_build_from_inputs(sub, hp)
        npg = O.num_pages(L)
        assert np.array_equal(ofmt[0, :npg], pf[b, :npg])
        # codec parity of the library-built pages of this sequence, then
        # replace them by the oracle's bytes
        for f, (kn, vn, ks, vs) in ((O.BF16, ("k_bf16", "v_bf16", None, None)),
                                    (O.FP8_E4M3, ("k_fp8", "v_fp8", "k_fp8_scale", "v_fp8_scale")),
                                    (O.TERNARY, ("k_tern", "v_tern", "k_gamma", "v_gamma"))):
            js = np.nonzero(pf[b, :npg] == f)[0]
            if len(js) == 0:
                continue
            gslots = torch.from_numpy(bt[b, js].astype(np.int64)).to(dev)
            oslots = obt[0, js]
            for nm, sn, src in ((kn, ks, kf), (vn, vs, vf)):
                o_pool = getattr(oc, nm)[oslots]
                if f == O.TERNARY:
                    src_bits = bits(src[torch.from_numpy((b * max_pages + js).astype(np.int64)).to(dev)])
                    check_ternary(pools[nm][gslots].cpu().numpy(), pools[sn][gslots].cpu().numpy(), src_bits)
                elif f == O.FP8_E4M3:
                    assert np.array_equal(pools[nm][gslots].cpu().numpy(), o_pool)
                    assert np.array_equal(pools[sn][gslots].cpu().numpy(), getattr(oc, sn)[oslots])
                else:
                    assert np.array_equal(bits(pools[nm][gslots]), o_pool)
                if f == O.BF16:
                    pools[nm][gslots] = torch.from_numpy(o_pool.view(np.int16)).view(torch.bfloat16).to(dev)
                else:
                    pools[nm][gslots] = torch.from_numpy(o_pool).to(dev)
                    pools[sn][gslots] = torch.from_numpy(getattr(oc, sn)[oslots]).to(dev)
        refs[b] = O.decode_attention(bits(inp["q"][b:b + 1]), oc, obt, ofmt, [L], hkv)[0]

    ws_bytes = K.kvc_decode_workspace_size(B, hq, hkv, D, max_pages)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    out = torch.full((B, hq, D), float("nan"), device=dev)
    K.kvc_decode_attention_paged(inp["q"], cache.struct, cache.block_table,
                                 None if older is None else older, inp["context_lens"], B, hq, hkv, D,
                                 16, max_pages, cfg["sink"], cfg["window"], hp, 0.0, out, ws, ws_bytes)
    assert K.kvc_decode_read_error(ws, B, hq, hkv, D, max_pages) == 0
    out_h = out.cpu().numpy()
    for b, ref in refs.items():
        assert_attention_close(out_h[b], ref, f"{name} b={b}")
    # every row: finite, and a convex combination of the decoded values
    assert np.isfinite(out_h).all()
    vmax = inp["v_pages"].abs().amax(dim=(1, 3, 4)).float().cpu().numpy()     # [B][Hkv]
    G = hq // hkv
    bound = np.repeat(vmax, G, axis=1)[:, :, None] * (1 + 1e-3) + 1e-6
    assert np.all(np.abs(out_h) <= bound)


def test_llama8b_full_size_sampled(cuda_device):
    _full_size_check("llama8b", cuda_device, sample_b=[0, 31])


def test_qwen3b_full_size_sampled(cuda_device):
    _full_size_check("qwen3b", cuda_device, sample_b=[0, 7])


def test_longctx_full_size_sampled(cuda_device):
    _full_size_check("longctx", cuda_device, sample_b=[3])
