"""Seeded synthetic inputs for the decode-attention and compression workloads.

This module is shared by the tests, the benchmark and the oracle harness, and
therefore holds none of the method's arithmetic: it only draws random bf16
tensors with the shapes and value distributions of the workloads, ragged
context lengths, anchor tags and a random physical-placement key.  Nothing
here quantises, packs, classifies pages or computes attention.

The same seed gives the same tensors on the same device type (CPU and CUDA
draw from different generator streams).

Workloads (sizes and distributions):

* ``tiny``     - batch 1, 8 Q / 4 KV heads, head_dim 64, context 512, sink 4,
                 window 64 kept BF16; Q, K, V ~ N(0, 1).
* ``qwen3b``   - Qwen2.5-3B-shaped layer: batch 8, 16 Q / 2 KV heads,
                 head_dim 128, context 4096, sink 4, window 256 kept FP8;
                 K, V ~ N(0, 1) with 2% of the (KV head, dim) channels scaled
                 x10 (one channel set per tensor, for every token).
* ``llama8b``  - Llama-3-8B-shaped layer: batch 32, 32 Q / 8 KV heads,
                 head_dim 128, context 32768, sink 4, window 1024 kept BF16;
                 K ~ N(0, 1) plus a per-channel offset ~ N(0, 2) (variance 2,
                 so sigma = sqrt(2)), V ~ N(0, 1); pages placed at a random
                 permutation of physical slots.
* ``longctx``  - long-context ragged layer: batch 16, 24 Q / 4 KV heads,
                 head_dim 256, context lengths uniform in [8192, 131072],
                 sink 4, window 2048 kept FP8, 5% of the older pages tagged as
                 BF16 anchors (Bernoulli per page); Q, K, V ~ Laplace(0, 1).
* ``bulk``     - 1 GiB of bf16 KV as 32768 pages of 8 KV heads x 16 tokens x
                 128 dims (16384 K pages + 16384 V pages); N(0, 1) with 1% of
                 the entries (Bernoulli per element) scaled x20.
"""

from __future__ import annotations

import math

import torch

PAGE_SIZE = 16

WORKLOADS = {
    "tiny": dict(batch=1, n_q_heads=8, n_kv_heads=4, head_dim=64, context=512,
                 sink=4, window=64, hp="bf16", dist="normal"),
    "qwen3b": dict(batch=8, n_q_heads=16, n_kv_heads=2, head_dim=128, context=4096,
                   sink=4, window=256, hp="fp8", dist="outlier_channels"),
    "llama8b": dict(batch=32, n_q_heads=32, n_kv_heads=8, head_dim=128, context=32768,
                    sink=4, window=1024, hp="bf16", dist="channel_offset", permute=True),
    "longctx": dict(batch=16, n_q_heads=24, n_kv_heads=4, head_dim=256,
                    context=(8192, 131072), sink=4, window=2048, hp="fp8",
                    anchors=0.05, dist="laplace"),
}

BULK = dict(n_pages=32768, n_kv_heads=8, head_dim=128, dist="bulk_outliers")


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(shape, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def _laplace(shape, g, device):
    # inverse CDF of Laplace(0, 1): x = -sign(u) * ln(1 - 2|u|), u ~ U(-1/2, 1/2)
    u = torch.rand(shape, generator=g, device=device, dtype=torch.float64) - 0.5
    u = u.clamp(-0.5 + 1e-12, 0.5 - 1e-12)
    return (-torch.sign(u) * torch.log1p(-2.0 * u.abs())).to(torch.float32)


def _outlier_channel_scale(n_kv_heads, head_dim, frac, factor, g, device):
    n_ch = n_kv_heads * head_dim
    k = max(1, int(round(frac * n_ch)))
    idx = torch.randperm(n_ch, generator=g, device=device)[:k]
    s = torch.ones(n_ch, device=device)
    s[idx] = factor
    return s.view(n_kv_heads, 1, head_dim)  # broadcast over [Hkv][P][D]


def decode_shape(name: str, **overrides) -> dict:
    """The workload's shape parameters, with optional overrides (e.g. a
    smaller batch or context for a case the oracle finishes in seconds)."""
    cfg = dict(WORKLOADS[name])
    cfg.update({k: v for k, v in overrides.items() if v is not None})
    return cfg


def make_decode_inputs(name: str, seed: int = 0, device="cpu", **overrides) -> dict:
    """Draw one batch of decode inputs.

    Returns a dict with
      q            bf16 [B][Hq][D]
      k_pages      bf16 [B][max_pages][Hkv][P][D]   (logical pages, HND)
      v_pages      bf16 [B][max_pages][Hkv][P][D]
      context_lens int32 [B]
      anchor       bool [B][max_pages]  (True: an older page kept as a BF16 anchor)
      slot_key     float32 [B][max_pages] or None (random physical placement)
    plus the shape parameters of the workload (``cfg``).  Slots of the last
    page past the context length hold random values too: the method must
    mask them."""
    cfg = decode_shape(name, **overrides)
    g = _gen(seed, device)
    B, hq, hkv, d = cfg["batch"], cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    ctx = cfg["context"]
    if isinstance(ctx, tuple):
        lens = torch.randint(ctx[0], ctx[1] + 1, (B,), generator=g, device=device)
        max_ctx = ctx[1]
    else:
        lens = torch.full((B,), int(ctx), device=device, dtype=torch.int64)
        max_ctx = int(ctx)
    max_pages = math.ceil(max_ctx / PAGE_SIZE)
    shape = (B, max_pages, hkv, PAGE_SIZE, d)
    dist = cfg["dist"]
    draw = _laplace if dist == "laplace" else _normal
    q = draw((B, hq, d), g, device)
    k = draw(shape, g, device)
    v = draw(shape, g, device)
    if dist == "outlier_channels":
        k.mul_(_outlier_channel_scale(hkv, d, 0.02, 10.0, g, device))
        v.mul_(_outlier_channel_scale(hkv, d, 0.02, 10.0, g, device))
    elif dist == "channel_offset":
        offset = _normal((hkv, 1, d), g, device) * math.sqrt(2.0)
        k.add_(offset)
    anchor = torch.zeros((B, max_pages), dtype=torch.bool, device=device)
    if cfg.get("anchors"):
        anchor = torch.rand((B, max_pages), generator=g, device=device) < cfg["anchors"]
    slot_key = None
    if cfg.get("permute"):
        slot_key = torch.rand((B, max_pages), generator=g, device=device)
    return dict(cfg=cfg, q=q.to(torch.bfloat16), k_pages=k.to(torch.bfloat16),
                v_pages=v.to(torch.bfloat16), context_lens=lens.to(torch.int32),
                anchor=anchor, slot_key=slot_key)


def make_bulk_pages(seed: int = 0, device="cpu", n_pages=None, n_kv_heads=None,
                    head_dim=None) -> torch.Tensor:
    """bf16 pages [n][Hkv][P][D] of the bulk-compression workload: N(0, 1),
    1% of the entries (Bernoulli per element) scaled x20."""
    n = n_pages or BULK["n_pages"]
    hkv = n_kv_heads or BULK["n_kv_heads"]
    d = head_dim or BULK["head_dim"]
    g = _gen(seed, device)
    x = _normal((n, hkv, PAGE_SIZE, d), g, device)
    mask = torch.rand((n, hkv, PAGE_SIZE, d), generator=g, device=device) < 0.01
    x = torch.where(mask, x * 20.0, x)
    return x.to(torch.bfloat16)
