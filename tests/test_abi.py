"""The C-ABI library without a GPU: it loads, exports every entry point that
include/kvc.h declares, rejects bad arguments before touching the device,
and its host page planner agrees with the oracle's page classification."""

import os
import re
import subprocess

import numpy as np
import pytest
import torch

import oracle as O
import compressed_decode_attention_kvc_b200 as K

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "kvc.h")).read()
    return sorted(set(re.findall(r"KVC_API\s+[\w\s\*]*?\b(kvc_\w+)\s*\(", src)))


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    assert set(K.EXPORTS) == set(syms), syms
    for name in ("kvc_quantize_pack_pages", "kvc_dequantize_pages", "kvc_decode_attention_paged"):
        assert name in syms


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", K.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s+(kvc_\w+)", out))
    assert set(declared_symbols()) <= exported
    # nothing but the C ABI is exported
    assert exported == set(declared_symbols())


def test_status_strings():
    for s in range(7):
        assert K.kvc_status_string(s)
    assert K.kvc_status_string(99) == "unknown status"


def _expect(status, fn, *args, **kw):
    with pytest.raises(K.KvcError) as e:
        fn(*args, **kw)
    assert e.value.status == status


def test_codec_argument_errors_without_gpu():
    fake = 0x1000  # never dereferenced: validation fails first
    q = K.kvc_quantize_pack_pages
    _expect(K.KVC_ERR_UNSUPPORTED, q, fake, None, 4, 15, 2, 128, K.KVC_FMT_TERNARY2, fake, fake)
    _expect(K.KVC_ERR_UNSUPPORTED, q, fake, None, 4, 16, 2, 96, K.KVC_FMT_TERNARY2, fake, fake)
    _expect(K.KVC_ERR_INVALID_ARG, q, None, None, 4, 16, 2, 128, K.KVC_FMT_TERNARY2, fake, fake)
    _expect(K.KVC_ERR_INVALID_ARG, q, fake, None, 4, 16, 2, 128, K.KVC_FMT_TERNARY2, fake, None)
    _expect(K.KVC_ERR_INVALID_ARG, q, fake + 8, None, 4, 16, 2, 128, K.KVC_FMT_FP8_E4M3, fake, fake)
    _expect(K.KVC_ERR_INVALID_ARG, q, fake, None, -1, 16, 2, 128, K.KVC_FMT_FP8_E4M3, fake, fake)
    _expect(K.KVC_ERR_INVALID_ARG, q, fake, None, 4, 16, 0, 128, K.KVC_FMT_FP8_E4M3, fake, fake)
    _expect(K.KVC_ERR_INVALID_ARG, q, fake, None, 4, 16, 2, 128, 7, fake, fake)
    K.kvc_quantize_pack_pages(None, None, 0, 16, 2, 128, K.KVC_FMT_TERNARY2, None, None)  # n = 0: no-op
    # the source pool must hold the pages named (ids 0..n-1 when page_ids is NULL)
    _expect(K.KVC_ERR_INVALID_ARG, q, fake, None, 4, 16, 2, 128, K.KVC_FMT_TERNARY2, fake, fake, n_src_pages=3)
    _expect(K.KVC_ERR_INVALID_ARG, q, fake, fake, 4, 16, 2, 128, K.KVC_FMT_TERNARY2, fake, fake, n_src_pages=0)
    d = K.kvc_dequantize_pages
    _expect(K.KVC_ERR_UNSUPPORTED, d, fake, fake, None, 4, 16, 2, 32, K.KVC_FMT_TERNARY2, fake)
    _expect(K.KVC_ERR_INVALID_ARG, d, fake, None, None, 4, 16, 2, 64, K.KVC_FMT_FP8_E4M3, fake)
    _expect(K.KVC_ERR_INVALID_ARG, d, fake, fake, None, 4, 16, 2, 64, K.KVC_FMT_BF16, None)


def test_decode_argument_errors_without_gpu():
    fake = 0x1000
    c = K.make_paged_cache(k_tern=fake, v_tern=fake, k_gamma=fake, v_gamma=fake, n_pages=(0, 0, 10))
    dec = K.kvc_decode_attention_paged

    def call(**kw):
        a = dict(q=fake, cache=c, bt=fake, older=None, lens=fake, B=2, hq=8, hkv=2, d=128, p=16,
                 mp=8, sink=4, win=16, hp=K.KVC_FMT_BF16, scale=0.0, out=fake, ws=fake, wsb=1 << 20)
        a.update(kw)
        dec(a["q"], a["cache"], a["bt"], a["older"], a["lens"], a["B"], a["hq"], a["hkv"], a["d"],
            a["p"], a["mp"], a["sink"], a["win"], a["hp"], a["scale"], a["out"], a["ws"], a["wsb"])

    for kw, st in ((dict(hq=6, hkv=4), K.KVC_ERR_INVALID_ARG), (dict(hq=18, hkv=2), K.KVC_ERR_UNSUPPORTED),
                   (dict(d=80), K.KVC_ERR_UNSUPPORTED), (dict(p=32), K.KVC_ERR_UNSUPPORTED),
                   (dict(hp=K.KVC_FMT_TERNARY2), K.KVC_ERR_INVALID_ARG), (dict(q=None), K.KVC_ERR_INVALID_ARG),
                   (dict(bt=None), K.KVC_ERR_INVALID_ARG), (dict(sink=-1), K.KVC_ERR_INVALID_ARG),
                   (dict(out=fake + 4), K.KVC_ERR_INVALID_ARG)):
        with pytest.raises(K.KvcError) as e:
            call(**kw)
        assert e.value.status == st, kw
    bad = K.make_paged_cache(k_tern=fake, v_tern=None, k_gamma=fake, v_gamma=fake, n_pages=(0, 0, 10))
    with pytest.raises(K.KvcError) as e:
        call(cache=bad)
    assert e.value.status == K.KVC_ERR_INVALID_ARG
    call(B=0)  # empty batch: no-op
    with pytest.raises(K.KvcError):
        K.kvc_decode_workspace_size(2, 8, 3, 128, 10)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_planner_matches_oracle_classification(seed):
    rng = np.random.default_rng(seed)
    B, mp = 5, 40
    lens = rng.integers(0, mp * 16 + 1, B).astype(np.int32)
    lens[0], lens[1] = 0, mp * 16
    sink, window = int(rng.integers(0, 40)), int(rng.integers(0, 200))
    older = np.where(rng.random((B, mp)) < 0.2, O.BF16, O.TERNARY).astype(np.uint8)
    key = rng.random((B, mp)).astype(np.float32)
    for hp in (K.KVC_FMT_BF16, K.KVC_FMT_FP8_E4M3):
        lay = K.paged_cache.plan_paged_cache(torch.from_numpy(lens), mp, sink, window, hp,
                                             older_fmt=torch.from_numpy(older), slot_key=torch.from_numpy(key))
        k = np.zeros((B, mp, 1, 16, 64), np.uint16)
        _, bt_o, fmt_o = O.build_paged_cache(k, k, lens, sink, window, hp, older_fmt=older, slot_key=key)
        assert np.array_equal(lay.page_fmt.numpy(), fmt_o)
        assert np.array_equal(lay.block_table.numpy(), bt_o)
        for f in range(3):
            ids = lay.pool_src_ids[f].numpy()
            assert len(ids) == (fmt_o == f).sum()
            for slot, pid in enumerate(ids):
                assert bt_o.reshape(-1)[pid] == slot and fmt_o.reshape(-1)[pid] == f


def test_planner_argument_errors():
    lens = torch.tensor([10, 500], dtype=torch.int32)
    with pytest.raises(K.KvcError):
        K.paged_cache.plan_paged_cache(lens, 4, 4, 16, K.KVC_FMT_BF16)      # 500 > 4 pages
    with pytest.raises(K.KvcError):
        K.paged_cache.plan_paged_cache(lens[:1], 4, 4, 16, K.KVC_FMT_TERNARY2)
    with pytest.raises(K.KvcError):
        K.paged_cache.plan_paged_cache(lens[:1], 4, 4, 16, K.KVC_FMT_BF16,
                                       older_fmt=torch.full((1, 4), 9, dtype=torch.uint8))


def test_append_retier_argument_errors():
    """Host-side validation of kvc_append_retier (no GPU work is launched)."""
    import ctypes
    lib = ctypes.CDLL(K.LIB_PATH)
    lib.kvc_append_retier.restype = ctypes.c_int
    cache = K.kvc_paged_cache()
    vp = ctypes.c_void_p
    def call(batch=1, hkv=2, d=128, page=16, max_pages=4, sink=4, window=16, hp=K.KVC_FMT_BF16,
             ptr=1 << 20, cache_p=True):
        p = vp(ptr) if ptr else None
        return lib.kvc_append_retier(p, p, ctypes.byref(cache) if cache_p else None, p, None, p, p, p,
                                     None, batch, hkv, d, page, max_pages, sink, window, hp, None)
    assert call(window=0) == K.KVC_ERR_INVALID_ARG          # the newest page must be high precision
    assert call(page=8) == K.KVC_ERR_UNSUPPORTED
    assert call(d=96) == K.KVC_ERR_UNSUPPORTED
    assert call(hp=K.KVC_FMT_TERNARY2) == K.KVC_ERR_INVALID_ARG
    assert call(cache_p=False) == K.KVC_ERR_INVALID_ARG
    assert call(batch=0) == K.KVC_OK                        # nothing to do, nothing launched
    assert call(ptr=0) == K.KVC_ERR_INVALID_ARG
    assert call(ptr=(1 << 20) + 8) == K.KVC_ERR_INVALID_ARG  # misaligned new-token rows
    assert call() == K.KVC_ERR_INVALID_ARG                  # no BF16 pools in the cache


def test_promote_argument_errors():
    """Host-side validation of kvc_promote_pages (no GPU work is launched)."""
    import ctypes
    lib = ctypes.CDLL(K.LIB_PATH)
    lib.kvc_promote_pages.restype = ctypes.c_int
    cache = K.kvc_paged_cache()
    vp = ctypes.c_void_p
    def call(n=1, batch=1, hkv=2, d=128, page=16, max_pages=4, sink=4, window=16, hp=K.KVC_FMT_BF16,
             anchor=K.KVC_FMT_BF16, ptr=1 << 20, tags=True, cache_p=True):
        p = vp(ptr) if ptr else None
        return lib.kvc_promote_pages(ctypes.byref(cache) if cache_p else None, p, p if tags else None, p, p, p,
                                     p, n, p, None, batch, hkv, d, page, max_pages, sink, window, hp, anchor,
                                     None)
    assert call(page=8) == K.KVC_ERR_UNSUPPORTED
    assert call(d=96) == K.KVC_ERR_UNSUPPORTED
    assert call(hp=K.KVC_FMT_TERNARY2) == K.KVC_ERR_INVALID_ARG
    assert call(anchor=K.KVC_FMT_TERNARY2) == K.KVC_ERR_INVALID_ARG
    assert call(n=-1) == K.KVC_ERR_INVALID_ARG
    assert call(cache_p=False) == K.KVC_ERR_INVALID_ARG
    assert call(n=0) == K.KVC_OK                            # nothing to do, nothing launched
    assert call(tags=False) == K.KVC_ERR_INVALID_ARG        # the tag makes a page an anchor
    assert call(ptr=0) == K.KVC_ERR_INVALID_ARG
    assert call(batch=1 << 20, max_pages=1 << 12) == K.KVC_ERR_UNSUPPORTED


def test_exans_argument_errors():
    """Host-side validation of the exponent-split codec entry points (nothing launched)."""
    import ctypes
    lib = ctypes.CDLL(K.LIB_PATH)
    lib.kvc_exans_encode.restype = ctypes.c_int
    lib.kvc_exans_decode.restype = ctypes.c_int
    vp = ctypes.c_void_p
    assert K.kvc_exans_workspace_size(10, 16, 8, 128) == 10 * (4 * 8 * 16 * 128 + 192)
    with pytest.raises(K.KvcError):
        K.kvc_exans_workspace_size(1, 8, 8, 128)                  # page size 16 only
    with pytest.raises(K.KvcError):
        K.kvc_exans_workspace_size(1, 16, 8, 96)                  # head_dim 64/128/256
    with pytest.raises(K.KvcError):
        K.kvc_exans_workspace_size(1, 16, 1 << 12, 256)           # N > 2^22
    p = vp(1 << 20)
    N = 8 * 16 * 128
    ws = 4 * N + 192

    def enc(n=2, ptr=p, ws_bytes=2 * ws, dst_bytes=2 * (64 + 2 * N), d=128, n_src=2):
        return lib.kvc_exans_encode(ptr, None, n, 16, 8, d, ptr, ctypes.c_size_t(ws_bytes), ptr,
                                    ctypes.c_size_t(dst_bytes), ptr, ctypes.c_int64(n_src), None, None)
    assert enc(n=-1) == K.KVC_ERR_INVALID_ARG
    assert enc(d=80) == K.KVC_ERR_UNSUPPORTED
    assert enc(ptr=None) == K.KVC_ERR_INVALID_ARG
    assert enc(ptr=vp((1 << 20) + 8)) == K.KVC_ERR_INVALID_ARG   # misaligned
    assert enc(ws_bytes=2 * ws - 1) == K.KVC_ERR_WORKSPACE
    assert enc(dst_bytes=2 * (64 + 2 * N) - 16) == K.KVC_ERR_INVALID_ARG
    assert enc(n_src=0) == K.KVC_ERR_INVALID_ARG                  # no source pages
    assert enc(n_src=1) == K.KVC_ERR_INVALID_ARG                  # ids 0..n-1 need n source pages
    def dec(n=2, ptr=p, d=128):
        return lib.kvc_exans_decode(ptr, ctypes.c_size_t(1 << 20), ptr, 2, None, n, 16, 8, d, ptr, None, None)
    assert dec(n=0) == K.KVC_OK
    assert dec(n=-3) == K.KVC_ERR_INVALID_ARG
    assert dec(d=32) == K.KVC_ERR_UNSUPPORTED
    assert dec(ptr=None) == K.KVC_ERR_INVALID_ARG


def test_layout_version_matches_the_header():
    src = open(os.path.join(ROOT, "include", "kvc.h")).read()
    v = int(re.search(r"#define KVC_LAYOUT_VERSION (\d+)", src).group(1))
    assert K.kvc_layout_version() == v == K.LAYOUT_VERSION


def test_noalloc_scratch_size_matches_header():
    # the binding's copy of KVC_NOALLOC_SCRATCH_BYTES is the header's value
    import re
    hdr = open(os.path.join(ROOT, "include", "kvc.h")).read()
    m = re.search(r"#define\s+KVC_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", hdr)
    assert m, "KVC_NOALLOC_SCRATCH_BYTES not found in kvc.h"
    assert int(m.group(1)) << int(m.group(2)) == K.NOALLOC_SCRATCH_BYTES


def test_decode_plan_info_argument_errors_and_constants():
    lib = K.kvc._lib
    import ctypes
    one = ctypes.c_int32(0)
    assert lib.kvc_decode_plan_info(2, 8, 2, 128, 10, None, ctypes.byref(one)) == K.KVC_ERR_INVALID_ARG
    assert lib.kvc_decode_plan_info(2, 8, 2, 128, 10, ctypes.byref(one), None) == K.KVC_ERR_INVALID_ARG
    _expect(K.KVC_ERR_INVALID_ARG, K.kvc_decode_plan_info, 2, 8, 3, 128, 10)
    _expect(K.KVC_ERR_INVALID_ARG, K.kvc_decode_plan_info, -1, 8, 2, 128, 10)
    _expect(K.KVC_ERR_UNSUPPORTED, K.kvc_decode_plan_info, 2, 18, 2, 128, 10)
    _expect(K.KVC_ERR_UNSUPPORTED, K.kvc_decode_plan_info, 2, 8, 2, 96, 10)
    # the binding's kernel ids are the header's
    hdr = open(os.path.join(ROOT, "include", "kvc.h")).read()
    ids = dict((m.group(1), int(m.group(2)))
               for m in re.finditer(r"#define\s+(KVC_DECODE_KERNEL_\w+)\s+(\d+)", hdr))
    assert ids == {n: getattr(K, n) for n in ("KVC_DECODE_KERNEL_CUDA_CORE", "KVC_DECODE_KERNEL_MMA",
                                                "KVC_DECODE_KERNEL_TCGEN05")}
