"""ctypes binding of libkvc (include/kvc.h).

Argument marshalling only: every function here has the name of the C entry
point it calls, turns torch tensors into raw device or host pointers and the
current CUDA stream into a cudaStream_t, and raises KvcError on a non-zero
status.  All computation happens in the library's CUDA kernels; there is no
Python or CPU fallback, and importing this module fails loudly when the
library has not been built.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkvc.so")

KVC_OK = 0
KVC_ERR_INVALID_ARG = 1
KVC_ERR_UNSUPPORTED = 2
KVC_ERR_WORKSPACE = 3
KVC_ERR_CUDA = 4
KVC_ERR_DEVICE_CHECK = 5
KVC_ERR_TIMEOUT = 6

KVC_FMT_BF16 = 0
KVC_FMT_FP8_E4M3 = 1
KVC_FMT_TERNARY2 = 2

PAGE_SIZE = 16
LAYOUT_VERSION = 1             # KVC_LAYOUT_VERSION of include/kvc.h

# device error flags returned by kvc_decode_read_error
ERR_BLOCK_TABLE = 1
ERR_FORMAT = 2
ERR_CONTEXT = 4
ERR_TIMEOUT = 8
ERR_RANGE = 16

EXPORTS = (
    "kvc_status_string", "kvc_quantize_pack_pages", "kvc_dequantize_pages",
    "kvc_plan_paged_cache", "kvc_decode_workspace_size", "kvc_decode_attention_paged",
    "kvc_decode_read_error", "kvc_decode_attention_paged_noalloc", "kvc_append_retier",
    "kvc_decode_attention_paged_layers", "kvc_promote_pages", "kvc_exans_workspace_size",
    "kvc_exans_encode", "kvc_exans_decode", "kvc_layout_version", "kvc_decode_plan_info",
)

# decode kernels (KVC_DECODE_KERNEL_* of include/kvc.h)
KVC_DECODE_KERNEL_CUDA_CORE = 0
KVC_DECODE_KERNEL_MMA = 1
KVC_DECODE_KERNEL_TCGEN05 = 2

NOALLOC_SCRATCH_BYTES = 16 << 20


class KvcError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {_lib.kvc_status_string(status).decode()} (status {status})")
        self.status = status


class kvc_paged_cache(ctypes.Structure):
    _fields_ = [
        ("k_bf16", ctypes.c_void_p), ("v_bf16", ctypes.c_void_p),
        ("k_fp8", ctypes.c_void_p), ("v_fp8", ctypes.c_void_p),
        ("k_fp8_scale", ctypes.c_void_p), ("v_fp8_scale", ctypes.c_void_p),
        ("k_tern", ctypes.c_void_p), ("v_tern", ctypes.c_void_p),
        ("k_gamma", ctypes.c_void_p), ("v_gamma", ctypes.c_void_p),
        ("n_pages", ctypes.c_int64 * 3),
    ]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python compressed_decode_attention_kvc_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, f32, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_int
    lib.kvc_status_string.restype = ctypes.c_char_p
    lib.kvc_status_string.argtypes = [st]
    lib.kvc_layout_version.restype = ctypes.c_int
    lib.kvc_layout_version.argtypes = []
    lib.kvc_quantize_pack_pages.restype = st
    lib.kvc_quantize_pack_pages.argtypes = [vp, vp, i32, i32, i32, i32, st, vp, vp, ctypes.c_int64, vp, vp]
    lib.kvc_dequantize_pages.restype = st
    lib.kvc_dequantize_pages.argtypes = [vp, vp, vp, i32, i32, i32, i32, st, vp, ctypes.c_int64, vp, vp]
    lib.kvc_append_retier.restype = st
    lib.kvc_append_retier.argtypes = [vp, vp, ctypes.POINTER(kvc_paged_cache), vp, vp, vp, vp, vp, vp,
                                      i32, i32, i32, i32, i32, i32, i32, st, vp]
    lib.kvc_promote_pages.restype = st
    lib.kvc_promote_pages.argtypes = [ctypes.POINTER(kvc_paged_cache), vp, vp, vp, vp, vp, vp, i32, vp, vp,
                                      i32, i32, i32, i32, i32, i32, i32, st, st, vp]
    lib.kvc_exans_workspace_size.restype = st
    lib.kvc_exans_workspace_size.argtypes = [i32, i32, i32, i32, ctypes.POINTER(ctypes.c_size_t)]
    lib.kvc_exans_encode.restype = st
    lib.kvc_exans_encode.argtypes = [vp, vp, i32, i32, i32, i32, vp, ctypes.c_size_t, vp, ctypes.c_size_t, vp,
                                     ctypes.c_int64, vp, vp]
    lib.kvc_exans_decode.restype = st
    lib.kvc_exans_decode.argtypes = [vp, ctypes.c_size_t, vp, i32, vp, i32, i32, i32, i32, vp, vp, vp]
    lib.kvc_plan_paged_cache.restype = st
    lib.kvc_plan_paged_cache.argtypes = [vp, i32, i32, i32, i32, i32, st, vp, vp, vp, vp, vp, vp]
    lib.kvc_decode_workspace_size.restype = st
    lib.kvc_decode_workspace_size.argtypes = [i32, i32, i32, i32, i32, ctypes.POINTER(ctypes.c_size_t)]
    lib.kvc_decode_plan_info.restype = st
    lib.kvc_decode_plan_info.argtypes = [i32, i32, i32, i32, i32, ctypes.POINTER(ctypes.c_int32),
                                         ctypes.POINTER(ctypes.c_int32)]
    lib.kvc_decode_attention_paged.restype = st
    lib.kvc_decode_attention_paged.argtypes = [
        vp, ctypes.POINTER(kvc_paged_cache), vp, vp, vp, i32, i32, i32, i32, i32, i32,
        i32, i32, st, f32, vp, vp, ctypes.c_size_t, vp]
    lib.kvc_decode_attention_paged_layers.restype = st
    lib.kvc_decode_attention_paged_layers.argtypes = [
        vp, ctypes.POINTER(kvc_paged_cache), vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
        i32, i32, st, f32, vp, vp, ctypes.c_size_t, vp]
    lib.kvc_decode_attention_paged_noalloc.restype = st
    lib.kvc_decode_attention_paged_noalloc.argtypes = [
        vp, ctypes.POINTER(kvc_paged_cache), vp, vp, vp, i32, i32, i32, i32, i32, i32,
        i32, i32, st, f32, vp, vp]
    lib.kvc_decode_read_error.restype = st
    lib.kvc_decode_read_error.argtypes = [vp, i32, i32, i32, i32, i32, ctypes.POINTER(ctypes.c_uint32), vp]
    return lib


_lib = _load()


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        if torch.cuda.is_available() and torch.cuda.is_initialized():
            return torch.cuda.current_stream().cuda_stream
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != KVC_OK:
        raise KvcError(status, where)


def kvc_status_string(status: int) -> str:
    return _lib.kvc_status_string(status).decode()


def _src_pages(src, n_src_pages, page_bytes: int, n: int) -> int:
    """Pages in a source buffer: the caller's count, else the tensor's size
    divided by the bytes of one page (a raw pointer without a count is taken
    to hold n pages)."""
    if n_src_pages is not None:
        return int(n_src_pages)
    if isinstance(src, torch.Tensor):
        return src.numel() * src.element_size() // page_bytes
    return max(1, int(n))


def kvc_quantize_pack_pages(src_bf16, page_ids, n, page_size, n_kv_heads, head_dim, mode,
                            dst, dst_scale, stream=None, n_src_pages=None, device_flags=None) -> None:
    ns = _src_pages(src_bf16, n_src_pages, 2 * page_size * n_kv_heads * head_dim, n) if n else 0
    _check(_lib.kvc_quantize_pack_pages(_ptr(src_bf16), _ptr(page_ids), n, page_size, n_kv_heads,
                                        head_dim, mode, _ptr(dst), _ptr(dst_scale), ns, _ptr(device_flags),
                                        _stream(stream)),
           "kvc_quantize_pack_pages")


def kvc_dequantize_pages(src, src_scale, page_ids, n, page_size, n_kv_heads, head_dim, mode,
                         dst_bf16, stream=None, n_src_pages=None, device_flags=None) -> None:
    per = {KVC_FMT_BF16: 2, KVC_FMT_FP8_E4M3: 1}.get(mode, 0.25)
    ns = _src_pages(src, n_src_pages, int(per * page_size * n_kv_heads * head_dim), n) if n else 0
    _check(_lib.kvc_dequantize_pages(_ptr(src), _ptr(src_scale), _ptr(page_ids), n, page_size,
                                     n_kv_heads, head_dim, mode, _ptr(dst_bf16), ns, _ptr(device_flags),
                                     _stream(stream)),
           "kvc_dequantize_pages")


def kvc_append_retier(k_new_bf16, v_new_bf16, cache: kvc_paged_cache, block_table, older_fmt,
                      context_lens, ternary_slot, freed_hp_slot, device_flags, batch, n_kv_heads,
                      head_dim, page_size, max_pages, sink_tokens, window_tokens, hp_mode,
                      stream=None) -> None:
    """Append one token per sequence and move the page that leaves the
    high-precision window to the ternary pool (see include/kvc.h)."""
    _check(_lib.kvc_append_retier(_ptr(k_new_bf16), _ptr(v_new_bf16), ctypes.byref(cache),
                                  _ptr(block_table), _ptr(older_fmt), _ptr(context_lens),
                                  _ptr(ternary_slot), _ptr(freed_hp_slot), _ptr(device_flags), batch,
                                  n_kv_heads, head_dim, page_size, max_pages, sink_tokens,
                                  window_tokens, hp_mode, _stream(stream)),
           "kvc_append_retier")


def kvc_promote_pages(cache: kvc_paged_cache, block_table, older_fmt, context_lens, req_seq, req_page,
                      anchor_slot, n_requests, freed_ternary_slot, device_flags, batch, n_kv_heads,
                      head_dim, page_size, max_pages, sink_tokens, window_tokens, hp_mode, anchor_fmt,
                      stream=None) -> None:
    """Re-expand stale (ternary) pages into BF16 / FP8 anchors (see include/kvc.h)."""
    _check(_lib.kvc_promote_pages(ctypes.byref(cache), _ptr(block_table), _ptr(older_fmt),
                                  _ptr(context_lens), _ptr(req_seq), _ptr(req_page), _ptr(anchor_slot),
                                  n_requests, _ptr(freed_ternary_slot), _ptr(device_flags), batch,
                                  n_kv_heads, head_dim, page_size, max_pages, sink_tokens, window_tokens,
                                  hp_mode, anchor_fmt, _stream(stream)),
           "kvc_promote_pages")


def kvc_layout_version() -> int:
    """Byte-layout version of the loaded library (include/kvc.h, KVC_LAYOUT_VERSION)."""
    return int(_lib.kvc_layout_version())


def kvc_exans_workspace_size(n, page_size, n_kv_heads, head_dim) -> int:
    out = ctypes.c_size_t(0)
    _check(_lib.kvc_exans_workspace_size(n, page_size, n_kv_heads, head_dim, ctypes.byref(out)),
           "kvc_exans_workspace_size")
    return out.value


def kvc_exans_encode(src_bf16, page_ids, n, page_size, n_kv_heads, head_dim, workspace, workspace_bytes, dst,
                     dst_bytes, offsets, stream=None, n_src_pages=None, device_flags=None) -> None:
    """Lossless exponent-split coding of n BF16 pages (see include/kvc.h)."""
    ns = _src_pages(src_bf16, n_src_pages, 2 * page_size * n_kv_heads * head_dim, n) if n else 0
    _check(_lib.kvc_exans_encode(_ptr(src_bf16), _ptr(page_ids), n, page_size, n_kv_heads, head_dim,
                                 _ptr(workspace), int(workspace_bytes), _ptr(dst), int(dst_bytes), _ptr(offsets),
                                 ns, _ptr(device_flags), _stream(stream)),
           "kvc_exans_encode")


def kvc_exans_decode(src, src_bytes, offsets, n_blobs, blob_ids, n, page_size, n_kv_heads, head_dim, dst_bf16,
                     device_flags, stream=None) -> None:
    _check(_lib.kvc_exans_decode(_ptr(src), int(src_bytes), _ptr(offsets), n_blobs, _ptr(blob_ids), n, page_size,
                                 n_kv_heads, head_dim, _ptr(dst_bf16), _ptr(device_flags), _stream(stream)),
           "kvc_exans_decode")


def kvc_plan_paged_cache(context_lens, batch, max_pages, page_size, sink_tokens, window_tokens,
                         hp_mode, older_fmt, slot_key, block_table, page_fmt, pool_pages,
                         pool_src_ids) -> None:
    """All tensors are host (CPU) tensors: int32 / uint8 / float32 as in kvc.h."""
    _check(_lib.kvc_plan_paged_cache(_ptr(context_lens), batch, max_pages, page_size, sink_tokens,
                                     window_tokens, hp_mode, _ptr(older_fmt), _ptr(slot_key),
                                     _ptr(block_table), _ptr(page_fmt), _ptr(pool_pages),
                                     _ptr(pool_src_ids)),
           "kvc_plan_paged_cache")


def kvc_decode_workspace_size(batch, n_q_heads, n_kv_heads, head_dim, max_pages) -> int:
    out = ctypes.c_size_t(0)
    _check(_lib.kvc_decode_workspace_size(batch, n_q_heads, n_kv_heads, head_dim, max_pages,
                                          ctypes.byref(out)),
           "kvc_decode_workspace_size")
    return out.value


def kvc_decode_plan_info(batch, n_q_heads, n_kv_heads, head_dim, max_pages) -> tuple:
    """(kernel, launches): the KVC_DECODE_KERNEL_* a decode call of these
    shapes runs on the current device, and its launches per call."""
    kern, launches = ctypes.c_int32(-1), ctypes.c_int32(-1)
    _check(_lib.kvc_decode_plan_info(batch, n_q_heads, n_kv_heads, head_dim, max_pages,
                                     ctypes.byref(kern), ctypes.byref(launches)),
           "kvc_decode_plan_info")
    return kern.value, launches.value


def make_paged_cache(k_bf16=None, v_bf16=None, k_fp8=None, v_fp8=None, k_fp8_scale=None,
                     v_fp8_scale=None, k_tern=None, v_tern=None, k_gamma=None, v_gamma=None,
                     n_pages=(0, 0, 0)) -> kvc_paged_cache:
    c = kvc_paged_cache()
    for name, t in (("k_bf16", k_bf16), ("v_bf16", v_bf16), ("k_fp8", k_fp8), ("v_fp8", v_fp8),
                    ("k_fp8_scale", k_fp8_scale), ("v_fp8_scale", v_fp8_scale),
                    ("k_tern", k_tern), ("v_tern", v_tern), ("k_gamma", k_gamma),
                    ("v_gamma", v_gamma)):
        setattr(c, name, _ptr(t))
    for f in range(3):
        c.n_pages[f] = int(n_pages[f])
    return c


def kvc_decode_attention_paged(q_bf16, cache: kvc_paged_cache, block_table, older_fmt,
                               context_lens, batch, n_q_heads, n_kv_heads, head_dim, page_size,
                               max_pages, sink_tokens, window_tokens, hp_mode, softmax_scale,
                               out, workspace, workspace_bytes, stream=None) -> None:
    _check(_lib.kvc_decode_attention_paged(
        _ptr(q_bf16), ctypes.byref(cache), _ptr(block_table), _ptr(older_fmt), _ptr(context_lens),
        batch, n_q_heads, n_kv_heads, head_dim, page_size, max_pages, sink_tokens, window_tokens,
        hp_mode, float(softmax_scale), _ptr(out), _ptr(workspace), int(workspace_bytes),
        _stream(stream)),
        "kvc_decode_attention_paged")


def kvc_decode_attention_paged_layers(q_bf16, cache: kvc_paged_cache, block_table, older_fmt,
                                      context_lens, n_layers, batch, n_q_heads, n_kv_heads, head_dim,
                                      page_size, max_pages, sink_tokens, window_tokens, hp_mode,
                                      softmax_scale, out, workspace, workspace_bytes, stream=None) -> None:
    """All layers of one decode step in one launch (see include/kvc.h)."""
    _check(_lib.kvc_decode_attention_paged_layers(
        _ptr(q_bf16), ctypes.byref(cache), _ptr(block_table), _ptr(older_fmt), _ptr(context_lens),
        n_layers, batch, n_q_heads, n_kv_heads, head_dim, page_size, max_pages, sink_tokens,
        window_tokens, hp_mode, float(softmax_scale), _ptr(out), _ptr(workspace), int(workspace_bytes),
        _stream(stream)),
        "kvc_decode_attention_paged_layers")


def kvc_decode_read_error(workspace, batch, n_q_heads, n_kv_heads, head_dim, max_pages,
                          stream=None) -> int:
    flags = ctypes.c_uint32(0)
    _check(_lib.kvc_decode_read_error(_ptr(workspace), batch, n_q_heads, n_kv_heads, head_dim,
                                      max_pages, ctypes.byref(flags), _stream(stream)),
           "kvc_decode_read_error")
    return flags.value


def kvc_decode_attention_paged_noalloc(q_bf16, cache: kvc_paged_cache, block_table, older_fmt,
                                       context_lens, batch, n_q_heads, n_kv_heads, head_dim,
                                       page_size, max_pages, sink_tokens, window_tokens, hp_mode,
                                       softmax_scale, out, stream=None) -> None:
    """kvc_decode_attention_paged without a caller-provided workspace: for
    callers that cannot allocate device memory.  The library uses a fixed
    device array of NOALLOC_SCRATCH_BYTES shared by every call on a device,
    so calls that overlap on the GPU race; make the first call on each
    device outside any stream capture."""
    _check(_lib.kvc_decode_attention_paged_noalloc(
        _ptr(q_bf16), ctypes.byref(cache), _ptr(block_table), _ptr(older_fmt), _ptr(context_lens),
        batch, n_q_heads, n_kv_heads, head_dim, page_size, max_pages, sink_tokens, window_tokens,
        hp_mode, float(softmax_scale), _ptr(out), _stream(stream)),
        "kvc_decode_attention_paged_noalloc")
