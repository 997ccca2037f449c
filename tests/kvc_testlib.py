"""Helpers shared by the parity tests: moving oracle (numpy) data to the
device, running the library on it, and the comparison rules.

Comparison rules (the parity bar):
* packed ternary bytes bit-exact, except elements whose |x| lies within
  1e-6 (relative) of the oracle's gamma/2 threshold; gamma within 1e-6
  relative;
* FP8 bytes and scales, BF16 copies and all dequantised bf16 bit-exact;
* attention output within max-abs 2e-3 and relative-L2 1e-3 of the fp64
  oracle, both sides reading the same (oracle-built) packed pages.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle as O
import compressed_decode_attention_kvc_b200 as K

GAMMA_RTOL = 1e-6
ATTN_MAX_ABS = 2e-3
ATTN_REL_L2 = 1e-3

ORACLE_FMT = {K.KVC_FMT_BF16: O.BF16, K.KVC_FMT_FP8_E4M3: O.FP8_E4M3, K.KVC_FMT_TERNARY2: O.TERNARY}


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 bit patterns (numpy, host)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def from_bits(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def check_ternary(codes_gpu, gamma_gpu, src_bits):
    """Compare GPU ternary output with the oracle's on the same source pages.
    Returns the number of exempted (threshold) elements."""
    codes_o, gamma_o = O.quantize_pack_ternary(src_bits)
    g_o = gamma_o.astype(np.float64)
    g_g = np.asarray(gamma_gpu, np.float64)
    assert np.all(np.abs(g_g - g_o) <= GAMMA_RTOL * g_o), "gamma outside 1e-6 relative"
    assert np.array_equal(g_g == 0, g_o == 0)
    c_o = O.unpack_ternary(codes_o)                       # [n][H][P][D]
    c_g = O.unpack_ternary(np.asarray(codes_gpu))
    x = O.bf16_to_f64(src_bits)
    half = 0.5 * g_o[:, :, None, None]
    exempt = np.abs(np.abs(x) - half) <= GAMMA_RTOL * half
    bad = (c_o != c_g) & ~exempt
    assert not bad.any(), f"{int(bad.sum())} codes differ outside the threshold band"
    # bytes whose four elements are all outside the band are bit-exact
    ex_b = exempt.reshape(exempt.shape[:-1] + (exempt.shape[-1] // 4, 4)).any(-1)
    assert np.array_equal(np.asarray(codes_gpu)[~ex_b], codes_o[~ex_b])
    return int(exempt.sum())


def attn_errors(out_gpu: np.ndarray, out_ref: np.ndarray):
    diff = out_gpu.astype(np.float64) - out_ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    denom = float(np.linalg.norm(out_ref))
    rel = float(np.linalg.norm(diff)) / denom if denom > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_attention_close(out_gpu, out_ref, what=""):
    max_abs, rel = attn_errors(out_gpu, out_ref)
    assert max_abs <= ATTN_MAX_ABS and rel <= ATTN_REL_L2, f"{what}: max_abs={max_abs:.3g} rel_l2={rel:.3g}"
    return max_abs, rel


def upload_oracle_cache(cache: "O.PagedCache", device):
    """Oracle pools (numpy) -> device tensors + the kvc_paged_cache struct."""
    t = {}
    t["k_bf16"] = from_bits(cache.k_bf16, device)
    t["v_bf16"] = from_bits(cache.v_bf16, device)
    for name in ("k_fp8", "v_fp8", "k_tern", "v_tern"):
        t[name] = torch.from_numpy(np.ascontiguousarray(getattr(cache, name))).to(device)
    for name in ("k_fp8_scale", "v_fp8_scale", "k_gamma", "v_gamma"):
        t[name] = torch.from_numpy(np.ascontiguousarray(getattr(cache, name), np.float32)).to(device)
    n_pages = (cache.k_bf16.shape[0], cache.k_fp8.shape[0], cache.k_tern.shape[0])
    struct = K.make_paged_cache(n_pages=n_pages, **{k: (v if v.numel() else None) for k, v in t.items()})
    return t, struct


def run_decode(q_bf16, struct, block_table, older_fmt, context_lens, n_kv_heads, max_pages,
               sink, window, hp_mode, softmax_scale=0.0, workspace=None):
    """Call kvc_decode_attention_paged on device tensors; returns out (device)."""
    B, hq, d = q_bf16.shape
    dev = q_bf16.device
    ws_bytes = K.kvc_decode_workspace_size(B, hq, n_kv_heads, d, max_pages)
    if workspace is None:
        workspace = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    out = torch.full((B, hq, d), float("nan"), dtype=torch.float32, device=dev)
    K.kvc_decode_attention_paged(q_bf16, struct, block_table, older_fmt, context_lens, B, hq,
                                 n_kv_heads, d, K.PAGE_SIZE, max_pages, sink, window, hp_mode,
                                 softmax_scale, out, workspace, ws_bytes)
    return out, workspace


def oracle_build_from_inputs(inp, hp_fmt_lib):
    """Run the oracle's cache builder on the generator's logical pages."""
    k = bits(inp["k_pages"])
    v = bits(inp["v_pages"])
    lens = inp["context_lens"].cpu().numpy()
    older = None
    if inp["anchor"].any():
        older = np.where(inp["anchor"].cpu().numpy(), O.BF16, O.TERNARY).astype(np.uint8)
    key = None if inp["slot_key"] is None else inp["slot_key"].cpu().numpy()
    cfg = inp["cfg"]
    cache, bt, fmt = O.build_paged_cache(k, v, lens, cfg["sink"], cfg["window"],
                                         ORACLE_FMT[hp_fmt_lib], older_fmt=older, slot_key=key)
    return cache, bt, fmt, older


def lib_older_fmt(older_oracle, device):
    """Oracle format tags -> library kvc_format tags (device uint8) or None."""
    if older_oracle is None:
        return None
    inv = {v: k for k, v in ORACLE_FMT.items()}
    out = np.vectorize(lambda f: inv[int(f)])(older_oracle).astype(np.uint8)
    return torch.from_numpy(out).to(device)


HP = {"bf16": K.KVC_FMT_BF16, "fp8": K.KVC_FMT_FP8_E4M3}
