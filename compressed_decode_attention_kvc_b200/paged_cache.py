"""Build a mixed-format paged KV cache on the device with libkvc.

This is the user-facing way to go from a layer's freshly written bf16 K/V
pages to the compressed cache that kvc_decode_attention_paged reads:
kvc_plan_paged_cache (host) decides each page's format and slot, then one
kvc_quantize_pack_pages call per pool and per K/V gathers and compresses the
pages into it.  Python only allocates (torch) and sequences the calls.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

from . import kvc as K


@dataclass
class PagedCacheLayout:
    block_table: torch.Tensor      # host int32 [B][max_pages]
    page_fmt: torch.Tensor         # host uint8 [B][max_pages] (255 unused)
    pool_pages: tuple              # pages per format (BF16, FP8, TERNARY2)
    pool_src_ids: list             # host int32 tensors: logical page ids per pool, slot order


def plan_paged_cache(context_lens, max_pages, sink_tokens, window_tokens, hp_mode,
                     older_fmt=None, slot_key=None) -> PagedCacheLayout:
    lens = torch.as_tensor(context_lens).to("cpu", torch.int32).contiguous()
    B = lens.numel()
    bt = torch.zeros((B, max_pages), dtype=torch.int32)
    pf = torch.zeros((B, max_pages), dtype=torch.uint8)
    pp = torch.zeros(3, dtype=torch.int32)
    ids = torch.zeros(max(1, B * max_pages), dtype=torch.int32)
    of = None if older_fmt is None else older_fmt.to("cpu", torch.uint8).contiguous()
    sk = None if slot_key is None else slot_key.to("cpu", torch.float32).contiguous()
    K.kvc_plan_paged_cache(lens, B, max_pages, K.PAGE_SIZE, sink_tokens, window_tokens, hp_mode,
                           of, sk, bt, pf, pp, ids)
    counts = tuple(int(x) for x in pp)
    offs = [0, counts[0], counts[0] + counts[1]]
    per = [ids[offs[f]:offs[f] + counts[f]].clone() for f in range(3)]
    return PagedCacheLayout(bt, pf, counts, per)


@dataclass
class DevicePagedCache:
    layout: PagedCacheLayout
    block_table: torch.Tensor      # device int32
    pools: dict                    # device tensors by name (kvc_paged_cache fields)
    page_ids: list                 # device int32 source ids per pool
    struct: K.kvc_paged_cache
    n_kv_heads: int
    head_dim: int
    n_layers: int = 1              # pools hold n_layers * pool_pages pages, layer-major

    def pool_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.pools.values())


def allocate_device_cache(layout: PagedCacheLayout, n_kv_heads: int, head_dim: int,
                          device, n_layers: int = 1) -> DevicePagedCache:
    """Pools for n_layers attention layers that share the placement: slot s
    of layer l is pool page l * pool_pages[f] + s (the layout of
    kvc_decode_attention_paged_layers); the struct carries the per-layer
    counts.  page_ids address logical pages of a [n_layers * B * max_pages]
    source, layer-major."""
    n_bf, n_f8, n_t = (n * n_layers for n in layout.pool_pages)
    P, H, D = K.PAGE_SIZE, n_kv_heads, head_dim
    pools = {
        "k_bf16": torch.empty((n_bf, H, P, D), dtype=torch.bfloat16, device=device),
        "v_bf16": torch.empty((n_bf, H, P, D), dtype=torch.bfloat16, device=device),
        "k_fp8": torch.empty((n_f8, H, P, D), dtype=torch.uint8, device=device),
        "v_fp8": torch.empty((n_f8, H, P, D), dtype=torch.uint8, device=device),
        "k_fp8_scale": torch.empty((n_f8,), dtype=torch.float32, device=device),
        "v_fp8_scale": torch.empty((n_f8,), dtype=torch.float32, device=device),
        "k_tern": torch.empty((n_t, H, P, D // 4), dtype=torch.uint8, device=device),
        "v_tern": torch.empty((n_t, H, P, D // 4), dtype=torch.uint8, device=device),
        "k_gamma": torch.empty((n_t, H), dtype=torch.float32, device=device),
        "v_gamma": torch.empty((n_t, H), dtype=torch.float32, device=device),
    }
    struct = K.make_paged_cache(n_pages=layout.pool_pages,
                                **{k: (v if v.numel() else None) for k, v in pools.items()})
    per_layer = layout.block_table.numel()
    ids = [torch.cat([ids + l * per_layer for l in range(n_layers)]) for ids in layout.pool_src_ids]
    return DevicePagedCache(layout=layout, block_table=layout.block_table.to(device),
                            pools=pools, page_ids=[i.to(device) for i in ids],
                            struct=struct, n_kv_heads=n_kv_heads, head_dim=head_dim, n_layers=n_layers)


def compress_into(cache: DevicePagedCache, k_pages: torch.Tensor, v_pages: torch.Tensor,
                  stream=None) -> int:
    """Fill every pool of `cache` from logical bf16 pages [B*max_pages][Hkv][16][D]
    (k_pages / v_pages, contiguous, on the device).  Returns the number of
    kernel launches issued."""
    H, D = cache.n_kv_heads, cache.head_dim
    launches = 0
    for fmt, (kname, vname, ks, vs) in (
            (K.KVC_FMT_BF16, ("k_bf16", "v_bf16", None, None)),
            (K.KVC_FMT_FP8_E4M3, ("k_fp8", "v_fp8", "k_fp8_scale", "v_fp8_scale")),
            (K.KVC_FMT_TERNARY2, ("k_tern", "v_tern", "k_gamma", "v_gamma"))):
        n = cache.layout.pool_pages[fmt] * cache.n_layers
        if n == 0:
            continue
        ids = cache.page_ids[fmt]
        P = cache.pools
        K.kvc_quantize_pack_pages(k_pages, ids, n, K.PAGE_SIZE, H, D, fmt, P[kname],
                                  P[ks] if ks else None, stream)
        K.kvc_quantize_pack_pages(v_pages, ids, n, K.PAGE_SIZE, H, D, fmt, P[vname],
                                  P[vs] if vs else None, stream)
        launches += 2
    return launches
