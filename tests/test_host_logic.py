"""Host-side logic that needs no GPU: the stacked-layer pool allocation of
the paged-cache helper, and the bench's bookkeeping (layers per workload,
traffic records keyed by kernel code and workload)."""

import argparse
import os
import sys

import numpy as np
import torch

import compressed_decode_attention_kvc_b200 as K
from compressed_decode_attention_kvc_b200 import paged_cache as PC

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_stacked_layer_pools_and_page_ids():
    lens = torch.tensor([16 * 9 + 3, 16 * 4, 0], dtype=torch.int32)
    max_pages, n_layers, H, D = 10, 3, 2, 64
    lay = PC.plan_paged_cache(lens, max_pages, 4, 20, K.KVC_FMT_FP8_E4M3)
    cache = PC.allocate_device_cache(lay, H, D, "cpu", n_layers=n_layers)
    per = lay.pool_pages
    assert tuple(cache.struct.n_pages) == tuple(per)                     # per-layer counts
    assert cache.pools["k_fp8"].shape[0] == n_layers * per[1]
    assert cache.pools["k_tern"].shape[0] == n_layers * per[2]
    assert cache.pools["k_gamma"].shape == (n_layers * per[2], H)
    # slot s of layer l reads logical page l * B * max_pages + id(s)
    B = lens.numel()
    for f in range(3):
        ids = cache.page_ids[f].numpy()
        base = lay.pool_src_ids[f].numpy()
        assert len(ids) == n_layers * len(base)
        for l in range(n_layers):
            assert np.array_equal(ids[l * len(base):(l + 1) * len(base)], base + l * B * max_pages)


def _bench():
    sys.path.insert(0, ROOT)
    import bench
    return bench


def test_bench_layers_and_config():
    bench = _bench()
    a = argparse.Namespace(workload="qwen3b", layers=None, batch=None, gpus=1, eager=False)
    assert bench.layers_of(a) == 36
    a.workload = "llama8b"
    assert bench.layers_of(a) == 1
    a.layers = 5
    assert bench.layers_of(a) == 5
    a = argparse.Namespace(workload="qwen3b", layers=None, batch=None, gpus=1, eager=False)
    cfg = dict(batch=8, context=4096, n_q_heads=16, n_kv_heads=2, head_dim=128)
    block = bench.config_block(a, cfg)
    assert block["layers"] == 36 and "36 layers" in block["workload"]


def test_bench_traffic_records_follow_the_kernel_code(tmp_path):
    bench = _bench()
    h_dec = bench.kernel_source_hash("decode")
    h_pack = bench.kernel_source_hash("pack_ternary")
    assert h_dec and h_pack and h_dec != h_pack
    assert bench.kernel_source_hash("no_such_kernel") is None
    # the kernel's own text is hashed: code after it in the file does not matter
    src = open(os.path.join(ROOT, "compressed_decode_attention_kvc_b200", "csrc", "quant.cu")).read()
    a = bench._function_text(src, "quant_ternary_kernel", True)
    b = bench._function_text(src, "launch_quant_ternary", False)
    assert a.startswith("//") and "quant_ternary_kernel(" in a and b.startswith("cudaError_t launch_quant_ternary(")
    # a record is used only for its workload at the default size
    rec = bench.ncu_traffic("decode", "llama8b")
    if rec is not None:
        assert rec > 0
    assert bench.ncu_traffic("decode", None) is None
    assert bench.ncu_traffic("decode", "no_such_workload") is None


def test_bench_algorithmic_bytes_match_the_storage_accounting():
    """The roofline numerator: bytes each kernel of a step must move, from
    the oracle's storage accounting (pinned to the pages' figures)."""
    import oracle as O
    bench = _bench()
    lens = torch.tensor([16 * 9 + 3, 16 * 4, 200], dtype=torch.int32)
    max_pages = 16
    cfg = dict(n_kv_heads=4, head_dim=128, n_q_heads=16)
    H, D, hq, P = 4, 128, 16, 16
    lay = PC.plan_paged_cache(lens, max_pages, 4, 40, K.KVC_FMT_FP8_E4M3)
    n_bf, n_f8, n_t = lay.pool_pages
    got = bench.algorithmic_bytes(cfg, lay, 3, max_pages, has_older=False)
    bf16_page = 2 * P * H * D
    tern_page = H * O.ternary_group_bytes(P, D)                 # codes + one gamma per head
    fp8_page = O.fp8_page_bytes(P, H, D)
    assert got["pack_ternary"] == 2 * n_t * (bf16_page + tern_page)
    assert got["pack_fp8"] == 2 * n_f8 * (bf16_page + fp8_page)
    assert got["pack_bf16"] == 2 * n_bf * 2 * bf16_page
    pages = n_bf + n_f8 + n_t
    per_seq = 2 * hq * D + 4 * hq * D + 4                       # Q bf16, out fp32, length
    assert got["decode"] == 2 * (n_bf * bf16_page + n_f8 * fp8_page + n_t * tern_page) + 3 * per_seq + 4 * pages
    tagged = bench.algorithmic_bytes(cfg, lay, 3, max_pages, has_older=True)
    assert tagged["decode"] == got["decode"] + pages               # one tag byte per page
