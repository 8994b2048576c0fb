"""The C ABI without a GPU: the library loads, exports every declared entry
point, and rejects invalid arguments before touching the device."""
import ctypes
import os
import re

import pytest

from exact_tiled_attention_36_b200 import binding as fb
from exact_tiled_attention_36_b200 import build as fbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    fbuild.build()
    return fb.lib()


def declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(fa_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"fa_fwd", "fa_varlen_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_status_string",
            "fa_get_last_device_error"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for s in range(6):
        assert fb.fa_status_string(s).startswith("FA_")
    assert "unknown" in fb.fa_status_string(77)
    assert re.match(r"\d+\.\d+\.\d+", fb.fa_version())


FAKE = 1 << 20  # a 16-byte aligned non-null address; never dereferenced on these paths


def fwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=2, Hkv=1, Nq=8, Nk=8, d=64, scale=0.125,
             causal=0, dtype=fb.FA_BF16, stream=None)
    a.update(kw)
    return fb.fa_fwd(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), fb.FA_ERR_INVALID_ARG),
    (dict(lse=None), fb.FA_ERR_INVALID_ARG),
    (dict(B=0), fb.FA_ERR_INVALID_ARG),
    (dict(Nq=-1), fb.FA_ERR_INVALID_ARG),
    (dict(Hq=3, Hkv=2), fb.FA_ERR_INVALID_ARG),
    (dict(Hkv=0), fb.FA_ERR_INVALID_ARG),
    (dict(scale=0.0), fb.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), fb.FA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), fb.FA_ERR_INVALID_ARG),
    (dict(causal=2), fb.FA_ERR_INVALID_ARG),
    (dict(d=96), fb.FA_ERR_UNSUPPORTED),
    (dict(d=256), fb.FA_ERR_UNSUPPORTED),
    (dict(dtype=7), fb.FA_ERR_UNSUPPORTED),
    (dict(k=FAKE + 8), fb.FA_ERR_MISALIGNED),
    (dict(lse=FAKE + 4), fb.FA_ERR_MISALIGNED),
    (dict(Nq=0), fb.FA_OK),  # no work: nothing is launched
    # past the grid's per-dimension limit (65535): refused, not truncated
    (dict(Hq=65536, Hkv=1), fb.FA_ERR_UNSUPPORTED),
    (dict(B=65536), fb.FA_ERR_UNSUPPORTED),
])
def test_fwd_rejects_before_launch(lib, kw, code):
    assert fwd(**kw) == code


def varlen(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, cu_q=FAKE, cu_k=FAKE, num_seqs=2, total_q=10, total_k=10,
             max_q=5, max_k=5, Hq=2, Hkv=2, d=128, scale=0.1, causal=0, dtype=fb.FA_FP16, stream=None)
    a.update(kw)
    return fb.fa_varlen_fwd(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(cu_q=None), fb.FA_ERR_INVALID_ARG),
    (dict(num_seqs=0), fb.FA_ERR_INVALID_ARG),
    (dict(total_k=-1), fb.FA_ERR_INVALID_ARG),
    (dict(max_q=-3), fb.FA_ERR_INVALID_ARG),
    (dict(d=32), fb.FA_ERR_UNSUPPORTED),
    (dict(cu_k=FAKE + 2), fb.FA_ERR_MISALIGNED),
    (dict(o=FAKE + 2), fb.FA_ERR_MISALIGNED),
    (dict(max_q=0), fb.FA_OK),
    (dict(total_q=0), fb.FA_OK),
])
def test_varlen_rejects_before_launch(lib, kw, code):
    assert varlen(**kw) == code


def bwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, do=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, ws=FAKE, B=1, Hq=4,
             Hkv=2, Nq=8, Nk=8, d=128, scale=0.1, causal=1, dtype=fb.FA_BF16, stream=None)
    a.update(kw)
    return fb.fa_bwd(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(ws=None), fb.FA_ERR_INVALID_ARG),
    (dict(dq=None), fb.FA_ERR_INVALID_ARG),
    (dict(Hq=5), fb.FA_ERR_INVALID_ARG),
    (dict(d=80), fb.FA_ERR_UNSUPPORTED),
    (dict(ws=FAKE + 8), fb.FA_ERR_MISALIGNED),
    (dict(dv=FAKE + 1), fb.FA_ERR_MISALIGNED),
    (dict(B=65536), fb.FA_ERR_UNSUPPORTED),
    (dict(Hq=65536, Hkv=65536), fb.FA_ERR_UNSUPPORTED),
])
def test_bwd_rejects_before_launch(lib, kw, code):
    assert bwd(**kw) == code


def test_workspace_size(lib):
    B, Hq, Nq, d = 2, 32, 8192, 128
    rows = B * Hq * Nq
    r256 = lambda x: (x + 255) // 256 * 256
    assert fb.fa_bwd_workspace_size(B, Hq, Nq, d) == r256(rows * 4) + r256(rows * d * 4)
    assert fb.fa_bwd_workspace_size(1, 1, 3, 64) == 256 + r256(3 * 64 * 4)
    # d = 128 pads the queries of each (b, h) to a multiple of four
    assert fb.fa_bwd_workspace_size(2, 3, 5, 128) == r256(2 * 3 * 5 * 4) + r256(2 * 3 * 8 * 128 * 4)
    assert fb.fa_bwd_workspace_size(0, 1, 1, 64) == 0
    assert fb.fa_bwd_workspace_size(1, 1, 1, 96) == 0


def varlen_bwd(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, do=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, ws=FAKE, cu_q=FAKE,
             cu_k=FAKE, num_seqs=2, total_q=10, total_k=10, max_q=5, max_k=5, Hq=4, Hkv=2, d=128, scale=0.1,
             causal=1, dtype=fb.FA_BF16, stream=None)
    a.update(kw)
    return fb.fa_varlen_bwd(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(ws=None), fb.FA_ERR_INVALID_ARG),
    (dict(cu_k=None), fb.FA_ERR_INVALID_ARG),
    (dict(dk=None), fb.FA_ERR_INVALID_ARG),
    (dict(num_seqs=0), fb.FA_ERR_INVALID_ARG),
    (dict(max_k=-1), fb.FA_ERR_INVALID_ARG),
    (dict(Hq=3), fb.FA_ERR_INVALID_ARG),
    (dict(d=96), fb.FA_ERR_UNSUPPORTED),
    (dict(cu_q=FAKE + 2), fb.FA_ERR_MISALIGNED),
    (dict(do=FAKE + 8), fb.FA_ERR_MISALIGNED),
])
def test_varlen_bwd_rejects_before_launch(lib, kw, code):
    assert varlen_bwd(**kw) == code


def test_varlen_workspace_size(lib):
    r256 = lambda x: (x + 255) // 256 * 256
    # D [Hq, total_q] and a dQ accumulator padded per sequence to max_seqlen_q (groups of four)
    assert fb.fa_varlen_bwd_workspace_size(3, 100, 41, 2, 128) == r256(100 * 2 * 4) + r256(3 * 2 * 11 * 512 * 4)
    # d = 64: [sequences, max_seqlen_q, Hq, 64]
    assert fb.fa_varlen_bwd_workspace_size(3, 100, 41, 2, 64) == r256(100 * 2 * 4) + r256(3 * 41 * 2 * 64 * 4)
    assert fb.fa_varlen_bwd_workspace_size(3, 100, 41, 2, 96) == 0
    assert fb.fa_varlen_bwd_workspace_size(0, 100, 41, 2, 128) == 0


def fwd_strided(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, sq=(3 * 8 * 64 * 8, 3 * 8 * 64, 64), sk=(3 * 8 * 64 * 8, 3 * 8 * 64, 64),
             sv=(3 * 8 * 64 * 8, 3 * 8 * 64, 64), so=(8 * 8 * 64, 8 * 64, 64), B=1, Hq=8, Hkv=8, Nq=8, Nk=8, d=64,
             scale=0.125, causal=0, dtype=fb.FA_BF16, stream=None)
    a.update(kw)
    return fb.fa_fwd_strided(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(sq=None), fb.FA_ERR_INVALID_ARG),
    (dict(so=(512, 0, 64)), fb.FA_ERR_INVALID_ARG),
    (dict(sk=(-8, 64, 64)), fb.FA_ERR_INVALID_ARG),
    (dict(sv=(4096, 1540, 64)), fb.FA_ERR_MISALIGNED),  # token stride not a multiple of 8 elements
    (dict(sq=(4096, 512, 68)), fb.FA_ERR_MISALIGNED),
    (dict(d=96), fb.FA_ERR_UNSUPPORTED),
    (dict(Nq=0), fb.FA_OK),
])
def test_fwd_strided_rejects_before_launch(lib, kw, code):
    assert fwd_strided(**kw) == code


def test_varlen_fwd_strided_rejects_before_launch(lib):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, sq=(3 * 2 * 128, 128), sk=(3 * 2 * 128, 128),
             sv=(3 * 2 * 128, 128), so=(2 * 128, 128), cu_q=FAKE, cu_k=FAKE, num_seqs=2, total_q=10, total_k=10,
             max_q=5, max_k=5, Hq=2, Hkv=2, d=128, scale=0.1, causal=0, dtype=fb.FA_FP16, stream=None)
    assert fb.fa_varlen_fwd_strided(*{**a, "so": None}.values()) == fb.FA_ERR_INVALID_ARG
    assert fb.fa_varlen_fwd_strided(*{**a, "sk": (770, 128)}.values()) == fb.FA_ERR_MISALIGNED
    assert fb.fa_varlen_fwd_strided(*{**a, "total_q": 0}.values()) == fb.FA_OK


@pytest.mark.parametrize("eps,code", [(-1.0, fb.FA_ERR_INVALID_ARG), (float("nan"), fb.FA_ERR_INVALID_ARG),
                                      (float("inf"), fb.FA_ERR_INVALID_ARG)])
def test_qk_rmsnorm_rejects_bad_eps(lib, eps, code):
    assert fb.fa_fwd_qk_rmsnorm(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 1, 8, 8, 64, 0.1, 0, eps, fb.FA_BF16,
                                None) == code
    assert fb.fa_fwd_qk_rmsnorm(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 1, 8, 8, 96, 0.1, 0, 1e-6, fb.FA_BF16,
                                None) == fb.FA_ERR_UNSUPPORTED
    assert fb.fa_fwd_qk_rmsnorm(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 1, 1, 8, 8, 64, 0.1, 0, 1e-6, fb.FA_BF16,
                                None) == fb.FA_ERR_INVALID_ARG
    assert fb.fa_fwd_qk_rmsnorm(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 8, 1, 1, 1, 8, 8, 64, 0.1, 0, 1e-6,
                                fb.FA_BF16, None) == fb.FA_ERR_MISALIGNED
    assert fb.fa_fwd_qk_rmsnorm_workspace_size(2, 100, 3, 128) == (2 * 100 * 3 * 128 * 2 + 255) // 256 * 256


def dec(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, sl=None, ws=FAKE, B=2, Hq=8, Hkv=2, Nq=1, Nk=64, d=128,
             scale=0.1, causal=0, dtype=fb.FA_BF16, stream=None)
    a.update(kw)
    return fb.fa_decode(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(ws=None), fb.FA_ERR_INVALID_ARG),
    (dict(Hq=5), fb.FA_ERR_INVALID_ARG),
    (dict(causal=2), fb.FA_ERR_INVALID_ARG),
    (dict(Nk=-1), fb.FA_ERR_INVALID_ARG),
    (dict(d=96), fb.FA_ERR_UNSUPPORTED),
    (dict(Nq=64), fb.FA_ERR_UNSUPPORTED),  # 4 heads x 64 tokens > one 128-row tile
    (dict(o=FAKE + 8), fb.FA_ERR_MISALIGNED),
    (dict(sl=FAKE + 2), fb.FA_ERR_MISALIGNED),
    (dict(Nq=0), fb.FA_OK),
])
def test_decode_rejects_before_launch(lib, kw, code):
    assert dec(**kw) == code


def dec_paged(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, sl=FAKE, bt=FAKE, ws=FAKE, B=2, Hq=8, Hkv=2, Nq=1,
             num_pages=10, page_size=64, max_pages=4, d=128, scale=0.1, causal=1, dtype=fb.FA_BF16, stream=None)
    a.update(kw)
    return fb.fa_decode_paged(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(sl=None), fb.FA_ERR_INVALID_ARG),
    (dict(bt=None), fb.FA_ERR_INVALID_ARG),
    (dict(num_pages=0), fb.FA_ERR_INVALID_ARG),
    (dict(page_size=8), fb.FA_ERR_INVALID_ARG),
    (dict(page_size=48), fb.FA_ERR_UNSUPPORTED),
    (dict(bt=FAKE + 1), fb.FA_ERR_MISALIGNED),
    (dict(Nq=0), fb.FA_OK),
    (dict(Nq=0, page_size=16), fb.FA_OK),
    (dict(Nq=0, page_size=192), fb.FA_OK),
])
def test_decode_paged_rejects_before_launch(lib, kw, code):
    assert dec_paged(**kw) == code


def test_decode_workspace_size_invalid(lib):
    for args in ((2, 8, 2, 1, 96), (2, 5, 2, 1, 128), (2, 8, 2, 33, 128), (0, 8, 2, 1, 128)):
        assert fb.fa_decode_workspace_size(*args) == 0


def fp8(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, qs=FAKE, ks=FAKE, vs=FAKE, o=FAKE, lse=FAKE, B=1, Hq=4, Hkv=2, Nq=8, Nk=8,
             d=128, scale=0.1, causal=1, stream=None)
    a.update(kw)
    return fb.fa_fwd_fp8(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(qs=None), fb.FA_ERR_INVALID_ARG),
    (dict(vs=None), fb.FA_ERR_INVALID_ARG),
    (dict(Hq=3), fb.FA_ERR_INVALID_ARG),
    (dict(d=64), fb.FA_ERR_UNSUPPORTED),
    (dict(ks=FAKE + 2), fb.FA_ERR_MISALIGNED),
    (dict(q=FAKE + 8), fb.FA_ERR_MISALIGNED),
    (dict(Nq=0), fb.FA_OK),
])
def test_fp8_rejects_before_launch(lib, kw, code):
    assert fp8(**kw) == code


def test_bwd_strided_rejects_before_launch(lib):
    st = (3 * 8 * 64 * 8, 3 * 8 * 64, 64)
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, do=FAKE, dq=FAKE, dk=FAKE, dv=FAKE, ws=FAKE, sq=st, sk=st,
             sv=st, so=st, sdo=st, sdq=st, sdk=st, sdv=st, B=1, Hq=8, Hkv=8, Nq=8, Nk=8, d=64, scale=0.125, causal=0,
             dtype=fb.FA_BF16, stream=None)
    assert fb.fa_bwd_strided(*{**a, "sdq": None}.values()) == fb.FA_ERR_INVALID_ARG
    assert fb.fa_bwd_strided(*{**a, "sdk": (4096, 1540, 64)}.values()) == fb.FA_ERR_MISALIGNED
    assert fb.fa_bwd_strided(*{**a, "ws": None}.values()) == fb.FA_ERR_INVALID_ARG
    assert fb.fa_bwd_strided(*{**a, "d": 96}.values()) == fb.FA_ERR_UNSUPPORTED


def test_keymask_rejects_before_launch(lib):
    assert fb.fa_fwd_keymask(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 2, 2, 8, 8, 128, 0.1, 0, fb.FA_BF16,
                             None) == fb.FA_ERR_INVALID_ARG
    assert fb.fa_fwd_keymask(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 2, 1, 2, 2, 8, 8, 128, 0.1, 0, fb.FA_BF16,
                             None) == fb.FA_ERR_MISALIGNED
    assert fb.fa_bwd_keymask(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 2, 2, 8, 8, 128,
                             0.1, 0, fb.FA_BF16, None) == fb.FA_ERR_INVALID_ARG
    assert fb.fa_pack_key_mask(None, FAKE, 1, 8, None) == fb.FA_ERR_INVALID_ARG
    assert fb.fa_pack_key_mask(FAKE, FAKE + 1, 1, 8, None) == fb.FA_ERR_MISALIGNED
    assert fb.fa_pack_key_mask(FAKE, FAKE, 1, 0, None) == fb.FA_OK


def test_varlen_window_anchor_rejects_before_launch(lib):
    base = [FAKE] * 5 + [FAKE, FAKE, 2, 256, 256, 128, 128, 4, 2, 128, 0.1, 64, 0]
    assert fb.fa_varlen_fwd_window_anchor(*base, -1, fb.FA_BF16, None) == fb.FA_ERR_INVALID_ARG
    no_cu = [FAKE] * 5 + [None, FAKE] + base[7:]
    assert fb.fa_varlen_fwd_window_anchor(*no_cu, 4, fb.FA_BF16, None) == fb.FA_ERR_INVALID_ARG
    bwd = [FAKE] * 12 + [2, 256, 256, 128, 128, 4, 2, 128, 0.1, 64, 0]
    assert fb.fa_varlen_bwd_window_anchor(*bwd, -1, fb.FA_BF16, None) == fb.FA_ERR_INVALID_ARG
    d96 = bwd[:19] + [96] + bwd[20:]
    assert fb.fa_varlen_bwd_window_anchor(*d96, 4, fb.FA_BF16, None) == fb.FA_ERR_UNSUPPORTED
    assert fb.fa_varlen_bwd_window_anchor(*bwd, 4, fb.FA_BF16 + 7, None) == fb.FA_ERR_UNSUPPORTED


def test_varlen_bwd_strided_rejects_before_launch(lib):
    st = (3 * 4 * 128, 128)
    ptrs = [FAKE] * 10
    strides = [st] * 8
    tail = [FAKE, FAKE, 2, 256, 256, 128, 128, 4, 4, 128, 0.1, 0, fb.FA_BF16, None]
    assert fb.fa_varlen_bwd_strided(*ptrs, *strides[:5], None, *strides[6:], *tail) == fb.FA_ERR_INVALID_ARG
    assert fb.fa_varlen_bwd_strided(*ptrs, *strides[:6], (1540, 64), st, *tail) == fb.FA_ERR_MISALIGNED
    assert fb.fa_varlen_bwd_strided(*ptrs, *strides[:7], (0, 128), *tail) == fb.FA_ERR_INVALID_ARG
    d96 = tail[:9] + [96] + tail[10:]
    assert fb.fa_varlen_bwd_strided(*ptrs, *strides, *d96) == fb.FA_ERR_UNSUPPORTED
    no_ws = [FAKE] * 9 + [None]
    assert fb.fa_varlen_bwd_strided(*no_ws, *strides, *tail) == fb.FA_ERR_INVALID_ARG
