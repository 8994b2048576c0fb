"""Thin ctypes binding of libfa.so.

The functions ``fa_fwd``, ``fa_varlen_fwd``, ``fa_fwd_strided``, ``fa_varlen_fwd_strided``, ``fa_fwd_qk_rmsnorm``,
``fa_fwd_window``, ``fa_bwd_window``, ``fa_varlen_fwd_window``, ``fa_varlen_bwd_window``, ``fa_fwd_window_anchor``,
``fa_bwd_window_anchor``, ``fa_varlen_fwd_window_anchor``, ``fa_varlen_bwd_window_anchor``, ``fa_bwd_strided``,
``fa_varlen_bwd_strided``,
``fa_pack_key_mask``,
``fa_fwd_keymask``, ``fa_bwd_keymask``, ``fa_fwd_fp8``, ``fa_decode``, ``fa_decode_paged``, ``fa_decode_workspace_size``,
``fa_bwd_workspace_size``, ``fa_varlen_bwd``,
``fa_bwd``, ``fa_status_string`` and ``fa_get_last_device_error`` have the
names, argument order and meaning of the C ABI in ``include/fa.h``: pointers
are passed as integers (device addresses), streams as integers (0 = default
stream), and the return value is the ``fa_status`` code. They only marshal
arguments; every step of the computation runs in the library's kernels.

``attention_fwd``, ``attention_varlen_fwd`` and ``attention_bwd`` are the
same calls on torch CUDA tensors: torch allocates the outputs and workspace,
the library fills them. There is no fallback: if ``libfa.so`` is missing or
a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfa.so")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_MISALIGNED, FA_ERR_CUDA, FA_ERR_TIMEOUT = range(6)
FA_BF16, FA_FP16 = 0, 1

_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float

_SIGS = {
    "fa_fwd": ([_P, _P, _P, _P, _P] + [_I] * 6 + [_F, _I, _I, _P], _I),
    "fa_varlen_fwd": ([_P, _P, _P, _P, _P, _P, _P] + [_I] * 8 + [_F, _I, _I, _P], _I),
    "fa_bwd_workspace_size": ([_I] * 4, ctypes.c_size_t),
    "fa_bwd": ([_P] * 10 + [_I] * 6 + [_F, _I, _I, _P], _I),
    "fa_status_string": ([_I], ctypes.c_char_p),
    "fa_get_last_device_error": ([_P], _I),
    "fa_get_last_device_error_site": ([], _I),
    "fa_version": ([], ctypes.c_char_p),
    "fa_bwd_set_timing_events": ([_P, _P], None),
    "fa_bwd_noalloc": ([_P] * 9 + [_I] * 6 + [_F, _I, _I, _P], _I),
    "fa_varlen_bwd_workspace_size": ([_I] * 5, ctypes.c_size_t),
    "fa_fwd_strided": ([_P] * 9 + [_I] * 6 + [_F, _I, _I, _P], _I),
    "fa_fwd_window": ([_P] * 5 + [_I] * 6 + [_F, _I, _I, _I, _P], _I),
    "fa_bwd_window": ([_P] * 10 + [_I] * 6 + [_F, _I, _I, _I, _P], _I),
    "fa_fwd_qk_rmsnorm": ([_P] * 6 + [_I] * 6 + [_F, _I, _F, _I, _P], _I),
    "fa_fwd_qk_rmsnorm_workspace_size": ([_I] * 4, ctypes.c_size_t),
    "fa_varlen_fwd_strided": ([_P] * 11 + [_I] * 8 + [_F, _I, _I, _P], _I),
    "fa_varlen_bwd": ([_P] * 12 + [_I] * 8 + [_F, _I, _I, _P], _I),
    "fa_selftest_bounded_wait": ([_P], _I),
    "fa_decode_workspace_size": ([_I] * 5, ctypes.c_size_t),
    "fa_fwd_fp8": ([_P] * 8 + [_I] * 6 + [_F, _I, _P], _I),
    "fa_pack_key_mask": ([_P, _P, _I, _I, _P], _I),
    "fa_fwd_keymask": ([_P] * 6 + [_I] * 6 + [_F, _I, _I, _P], _I),
    "fa_bwd_keymask": ([_P] * 11 + [_I] * 6 + [_F, _I, _I, _P], _I),
    "fa_bwd_strided": ([_P] * 18 + [_I] * 6 + [_F, _I, _I, _P], _I),
    "fa_varlen_bwd_strided": ([_P] * 20 + [_I] * 8 + [_F, _I, _I, _P], _I),
    "fa_fwd_window_anchor": ([_P] * 5 + [_I] * 6 + [_F, _I, _I, _I, _I, _P], _I),
    "fa_bwd_window_anchor": ([_P] * 10 + [_I] * 6 + [_F, _I, _I, _I, _I, _P], _I),
    "fa_varlen_fwd_window": ([_P] * 7 + [_I] * 8 + [_F, _I, _I, _I, _P], _I),
    "fa_varlen_bwd_window": ([_P] * 12 + [_I] * 8 + [_F, _I, _I, _I, _P], _I),
    "fa_varlen_fwd_window_anchor": ([_P] * 7 + [_I] * 8 + [_F, _I, _I, _I, _I, _P], _I),
    "fa_varlen_bwd_window_anchor": ([_P] * 12 + [_I] * 8 + [_F, _I, _I, _I, _I, _P], _I),
    "fa_decode": ([_P] * 7 + [_I] * 6 + [_F, _I, _I, _P], _I),
    "fa_decode_paged": ([_P] * 8 + [_I] * 8 + [_F, _I, _I, _P], _I),
}


class FAError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {fa_status_string(status)} ({status})")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m exact_tiled_attention_36_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            f = getattr(l, name)
            f.argtypes = args
            f.restype = res
        _lib = l
    return _lib


def fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype, stream) -> int:
    return lib().fa_fwd(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype, stream)


def fa_varlen_fwd(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, num_seqs, total_q, total_k, max_seqlen_q,
                  max_seqlen_k, Hq, Hkv, d, scale, causal, dtype, stream) -> int:
    return lib().fa_varlen_fwd(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, num_seqs, total_q, total_k,
                               max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, causal, dtype, stream)


def fa_bwd_workspace_size(B, Hq, Nq, d) -> int:
    return int(lib().fa_bwd_workspace_size(B, Hq, Nq, d))


def fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype,
           stream) -> int:
    return lib().fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                        dtype, stream)


def fa_fwd_window(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, window_left, window_right, dtype, stream) -> int:
    return lib().fa_fwd_window(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, window_left, window_right, dtype,
                               stream)


def fa_bwd_window(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, scale, window_left,
                  window_right, dtype, stream) -> int:
    return lib().fa_bwd_window(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, scale,
                               window_left, window_right, dtype, stream)


def fa_fwd_qk_rmsnorm_workspace_size(B, Nk, Hkv, d) -> int:
    return int(lib().fa_fwd_qk_rmsnorm_workspace_size(B, Nk, Hkv, d))


def fa_fwd_qk_rmsnorm(q, k, v, o, lse, workspace, B, Hq, Hkv, Nq, Nk, d, scale, causal, eps, dtype,
                      stream) -> int:
    return lib().fa_fwd_qk_rmsnorm(q, k, v, o, lse, workspace, B, Hq, Hkv, Nq, Nk, d, scale, causal, eps, dtype,
                                   stream)


def _strides(st):
    """A host int64 array of element strides (kept alive by the caller's reference)."""
    return (ctypes.c_longlong * len(st))(*[int(x) for x in st]) if st is not None else None


def fa_fwd_strided(q, k, v, o, lse, q_strides, k_strides, v_strides, o_strides, B, Hq, Hkv, Nq, Nk, d, scale,
                   causal, dtype, stream) -> int:
    """Strides are sequences of ints ({batch, token, head} in elements)."""
    arrs = [_strides(x) for x in (q_strides, k_strides, v_strides, o_strides)]
    return lib().fa_fwd_strided(q, k, v, o, lse, *[ctypes.cast(a, _P) if a is not None else None for a in arrs], B,
                                Hq, Hkv, Nq, Nk, d, scale, causal, dtype, stream)


def fa_varlen_fwd_strided(q, k, v, o, lse, q_strides, k_strides, v_strides, o_strides, cu_seqlens_q, cu_seqlens_k,
                          num_seqs, total_q, total_k, max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, causal, dtype,
                          stream) -> int:
    """Strides are sequences of ints ({token, head} in elements)."""
    arrs = [_strides(x) for x in (q_strides, k_strides, v_strides, o_strides)]
    return lib().fa_varlen_fwd_strided(q, k, v, o, lse, *[ctypes.cast(a, _P) if a is not None else None for a in arrs],
                                       cu_seqlens_q, cu_seqlens_k, num_seqs, total_q, total_k, max_seqlen_q,
                                       max_seqlen_k, Hq, Hkv, d, scale, causal, dtype, stream)


def fa_varlen_bwd_workspace_size(num_seqs, total_q, max_seqlen_q, Hq, d) -> int:
    return int(lib().fa_varlen_bwd_workspace_size(num_seqs, total_q, max_seqlen_q, Hq, d))


def fa_varlen_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, cu_seqlens_q, cu_seqlens_k, num_seqs, total_q,
                  total_k, max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, causal, dtype, stream) -> int:
    return lib().fa_varlen_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, cu_seqlens_q, cu_seqlens_k, num_seqs,
                               total_q, total_k, max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, causal, dtype,
                               stream)


def fa_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype, stream) -> int:
    """fa_bwd with the library's own fixed-size workspace (for callers that cannot allocate)."""
    return lib().fa_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype,
                                stream)


def fa_pack_key_mask(keep, key_bits, B, Nk, stream) -> int:
    return lib().fa_pack_key_mask(keep, key_bits, B, Nk, stream)


def fa_fwd_keymask(q, k, v, o, lse, key_bits, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype, stream) -> int:
    return lib().fa_fwd_keymask(q, k, v, o, lse, key_bits, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype, stream)


def fa_bwd_keymask(q, k, v, o, lse, dout, dq, dk, dv, workspace, key_bits, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                   dtype, stream) -> int:
    return lib().fa_bwd_keymask(q, k, v, o, lse, dout, dq, dk, dv, workspace, key_bits, B, Hq, Hkv, Nq, Nk, d, scale,
                                causal, dtype, stream)


def fa_bwd_strided(q, k, v, o, lse, dout, dq, dk, dv, workspace, q_strides, k_strides, v_strides, o_strides,
                   do_strides, dq_strides, dk_strides, dv_strides, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype,
                   stream) -> int:
    """*_strides: (batch, token, head) element strides (host), as fa_fwd_strided."""
    return lib().fa_bwd_strided(q, k, v, o, lse, dout, dq, dk, dv, workspace, _strides(q_strides),
                                _strides(k_strides), _strides(v_strides), _strides(o_strides), _strides(do_strides),
                                _strides(dq_strides), _strides(dk_strides), _strides(dv_strides), B, Hq, Hkv, Nq, Nk,
                                d, scale, causal, dtype, stream)


def fa_varlen_bwd_strided(q, k, v, o, lse, dout, dq, dk, dv, workspace, q_strides, k_strides, v_strides, o_strides,
                          do_strides, dq_strides, dk_strides, dv_strides, cu_seqlens_q, cu_seqlens_k, num_seqs,
                          total_q, total_k, max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, causal, dtype,
                          stream) -> int:
    """*_strides: (token, head) element strides (host), as fa_varlen_fwd_strided."""
    return lib().fa_varlen_bwd_strided(q, k, v, o, lse, dout, dq, dk, dv, workspace, _strides(q_strides),
                                       _strides(k_strides), _strides(v_strides), _strides(o_strides),
                                       _strides(do_strides), _strides(dq_strides), _strides(dk_strides),
                                       _strides(dv_strides), cu_seqlens_q, cu_seqlens_k, num_seqs, total_q, total_k,
                                       max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, causal, dtype, stream)


def fa_fwd_window_anchor(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, window_left, window_right, n_anchor, dtype,
                         stream) -> int:
    return lib().fa_fwd_window_anchor(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, window_left, window_right,
                                      n_anchor, dtype, stream)


def fa_bwd_window_anchor(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, scale, window_left,
                         window_right, n_anchor, dtype, stream) -> int:
    return lib().fa_bwd_window_anchor(q, k, v, o, lse, dout, dq, dk, dv, workspace, B, Hq, Hkv, Nq, Nk, d, scale,
                                      window_left, window_right, n_anchor, dtype, stream)


def fa_varlen_fwd_window(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, num_seqs, total_q, total_k, max_seqlen_q,
                         max_seqlen_k, Hq, Hkv, d, scale, window_left, window_right, dtype, stream) -> int:
    return lib().fa_varlen_fwd_window(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, num_seqs, total_q, total_k,
                                      max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, window_left, window_right, dtype,
                                      stream)


def fa_varlen_bwd_window(q, k, v, o, lse, dout, dq, dk, dv, workspace, cu_seqlens_q, cu_seqlens_k, num_seqs,
                         total_q, total_k, max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, window_left, window_right,
                         dtype, stream) -> int:
    return lib().fa_varlen_bwd_window(q, k, v, o, lse, dout, dq, dk, dv, workspace, cu_seqlens_q, cu_seqlens_k,
                                      num_seqs, total_q, total_k, max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale,
                                      window_left, window_right, dtype, stream)


def fa_varlen_fwd_window_anchor(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, num_seqs, total_q, total_k, max_seqlen_q,
                                max_seqlen_k, Hq, Hkv, d, scale, window_left, window_right, n_anchor, dtype,
                                stream) -> int:
    return lib().fa_varlen_fwd_window_anchor(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, num_seqs, total_q, total_k,
                                             max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, window_left, window_right,
                                             n_anchor, dtype, stream)


def fa_varlen_bwd_window_anchor(q, k, v, o, lse, dout, dq, dk, dv, workspace, cu_seqlens_q, cu_seqlens_k, num_seqs,
                                total_q, total_k, max_seqlen_q, max_seqlen_k, Hq, Hkv, d, scale, window_left,
                                window_right, n_anchor, dtype, stream) -> int:
    return lib().fa_varlen_bwd_window_anchor(q, k, v, o, lse, dout, dq, dk, dv, workspace, cu_seqlens_q,
                                             cu_seqlens_k, num_seqs, total_q, total_k, max_seqlen_q, max_seqlen_k, Hq,
                                             Hkv, d, scale, window_left, window_right, n_anchor, dtype, stream)


def fa_fwd_fp8(q, k, v, q_scale, k_scale, v_scale, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, stream) -> int:
    return lib().fa_fwd_fp8(q, k, v, q_scale, k_scale, v_scale, o, lse, B, Hq, Hkv, Nq, Nk, d, scale, causal, stream)


def fa_decode_workspace_size(B, Hq, Hkv, Nq, d) -> int:
    return int(lib().fa_decode_workspace_size(B, Hq, Hkv, Nq, d))


def fa_decode(q, k, v, o, lse, cache_seqlens, workspace, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype, stream) -> int:
    return lib().fa_decode(q, k, v, o, lse, cache_seqlens, workspace, B, Hq, Hkv, Nq, Nk, d, scale, causal, dtype,
                           stream)


def fa_decode_paged(q, k_pages, v_pages, o, lse, cache_seqlens, block_table, workspace, B, Hq, Hkv, Nq, num_pages,
                    page_size, max_pages, d, scale, causal, dtype, stream) -> int:
    return lib().fa_decode_paged(q, k_pages, v_pages, o, lse, cache_seqlens, block_table, workspace, B, Hq, Hkv, Nq,
                                 num_pages, page_size, max_pages, d, scale, causal, dtype, stream)


def fa_status_string(s: int) -> str:
    return lib().fa_status_string(s).decode()


def fa_get_last_device_error(stream) -> int:
    return lib().fa_get_last_device_error(stream)


def fa_get_last_device_error_site() -> int:
    return lib().fa_get_last_device_error_site()


def fa_bwd_set_timing_events(before, after) -> None:
    lib().fa_bwd_set_timing_events(before, after)


def fa_selftest_bounded_wait(stream) -> int:
    return lib().fa_selftest_bounded_wait(stream)


def fa_version() -> str:
    return lib().fa_version().decode()


# ----------------------------------------------------------------------------- torch tensors
def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return FA_BF16
    if t.dtype == torch.float16:
        return FA_FP16
    raise TypeError(f"q/k/v must be bfloat16 or float16, got {t.dtype}")


def _dev(t):
    if not t.is_cuda:
        raise ValueError("tensors must be on a CUDA device")
    return t if t.is_contiguous() else t.contiguous()


def _stream(stream):
    """The raw CUDA stream handle: `stream` (a torch stream or a handle), or the current
    stream of the current device."""
    import torch
    if stream is None:
        raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)  # the handle without a Stream object
        if raw is not None:
            return raw(torch.cuda.current_device())
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(status: int, what: str):
    if status != FA_OK:
        raise FAError(status, what)


def attention_fwd(q, k, v, scale: float | None = None, causal: bool = False, out=None, lse=None, stream=None):
    """O, L = attention(q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d]); L is float32 [B,Hq,Nq]."""
    import torch
    q, k, v = _dev(q), _dev(k), _dev(v)
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    if scale is None:
        scale = d ** -0.5
    o = torch.empty_like(q) if out is None else out
    L = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), L.data_ptr(), B, Hq, Hkv, Nq, Nk, d,
                  float(scale), int(bool(causal)), _dtype_code(q), _stream(stream)), "fa_fwd")
    return o, L


def attention_varlen_fwd(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                         scale: float | None = None, causal: bool = False, out=None, lse=None, stream=None):
    """Packed varlen forward: q [total_q,Hq,d], k/v [total_k,Hkv,d]; L is float32 [Hq,total_q]."""
    import torch
    q, k, v = _dev(q), _dev(k), _dev(v)
    cu_q = _dev(cu_seqlens_q).to(torch.int32)
    cu_k = _dev(cu_seqlens_k).to(torch.int32)
    Tq, Hq, d = q.shape
    Tk, Hkv, _ = k.shape
    if scale is None:
        scale = d ** -0.5
    o = torch.empty_like(q) if out is None else out
    L = torch.empty((Hq, Tq), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(fa_varlen_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), L.data_ptr(), cu_q.data_ptr(),
                         cu_k.data_ptr(), cu_q.numel() - 1, Tq, Tk, int(max_seqlen_q), int(max_seqlen_k), Hq, Hkv,
                         d, float(scale), int(bool(causal)), _dtype_code(q), _stream(stream)), "fa_varlen_fwd")
    return o, L


def attention_bwd(q, k, v, o, lse, dout, scale: float | None = None, causal: bool = False, workspace=None,
                  stream=None):
    """dQ, dK, dV of the fixed-length forward (same layouts as q, k, v)."""
    import torch
    q, k, v, o, dout = _dev(q), _dev(k), _dev(v), _dev(o), _dev(dout)
    lse = _dev(lse)
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    if scale is None:
        scale = d ** -0.5
    ws_bytes = fa_bwd_workspace_size(B, Hq, Nq, d)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device) if workspace is None else workspace
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    _check(fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), dout.data_ptr(),
                  dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), B, Hq, Hkv, Nq, Nk, d, float(scale),
                  int(bool(causal)), _dtype_code(q), _stream(stream)), "fa_bwd")
    return dq, dk, dv


def attention_varlen_bwd(q, k, v, o, lse, dout, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                         scale: float | None = None, causal: bool = False, workspace=None, stream=None):
    """dQ, dK, dV of the packed varlen forward (same layouts as q, k, v; d = 64 or 128)."""
    import torch
    q, k, v, o, dout = _dev(q), _dev(k), _dev(v), _dev(o), _dev(dout)
    lse = _dev(lse)
    cu_q = _dev(cu_seqlens_q).to(torch.int32)
    cu_k = _dev(cu_seqlens_k).to(torch.int32)
    Tq, Hq, d = q.shape
    Tk, Hkv, _ = k.shape
    n = cu_q.numel() - 1
    if scale is None:
        scale = d ** -0.5
    ws_bytes = fa_varlen_bwd_workspace_size(n, Tq, int(max_seqlen_q), Hq, d)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device) if workspace is None else workspace
    dq, dk, dv = torch.zeros_like(q), torch.zeros_like(k), torch.zeros_like(v)
    _check(fa_varlen_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), dout.data_ptr(),
                         dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), cu_q.data_ptr(), cu_k.data_ptr(),
                         n, Tq, Tk, int(max_seqlen_q), int(max_seqlen_k), Hq, Hkv, d, float(scale),
                         int(bool(causal)), _dtype_code(q), _stream(stream)), "fa_varlen_bwd")
    return dq, dk, dv


def attention_decode(q, k_cache, v_cache, cache_seqlens=None, scale: float | None = None, causal: bool = False,
                     block_table=None, workspace=None, out=None, lse=None, stream=None):
    """Split-KV decode: q [B,Nq,Hq,d] (the newest Nq tokens) against a cache.

    Contiguous cache: k/v [B,Nk,Hkv,d], sequence b using its first cache_seqlens[b]
    keys (all Nk when None). Paged cache (block_table int32 [B,max_pages]): k/v
    [num_pages,page_size,Hkv,d] and cache_seqlens required. Returns O [B,Nq,Hq,d]
    and L float32 [B,Hq,Nq]."""
    import torch
    q, k, v = _dev(q), _dev(k_cache), _dev(v_cache)
    B, Nq, Hq, d = q.shape
    Hkv = k.shape[2]
    if scale is None:
        scale = d ** -0.5
    sl = None if cache_seqlens is None else _dev(cache_seqlens).to(torch.int32)
    ws_bytes = fa_decode_workspace_size(B, Hq, Hkv, Nq, d)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=q.device) if workspace is None else workspace
    o = torch.empty_like(q) if out is None else out
    L = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    if block_table is None:
        st = fa_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), L.data_ptr(),
                       0 if sl is None else sl.data_ptr(), ws.data_ptr(), B, Hq, Hkv, Nq, k.shape[1], d, float(scale),
                       int(bool(causal)), _dtype_code(q), _stream(stream))
        _check(st, "fa_decode")
    else:
        if sl is None:
            raise ValueError("a paged cache needs cache_seqlens")
        bt = _dev(block_table).to(torch.int32)
        st = fa_decode_paged(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), L.data_ptr(), sl.data_ptr(),
                             bt.data_ptr(), ws.data_ptr(), B, Hq, Hkv, Nq, k.shape[0], k.shape[1], bt.shape[1], d,
                             float(scale), int(bool(causal)), _dtype_code(q), _stream(stream))
        _check(st, "fa_decode_paged")
    return o, L


def attention_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, scale: float | None = None, causal: bool = False,
                      out=None, lse=None, stream=None):
    """FP8 forward: q8 [B,Nq,Hq,d], k8/v8 [B,Nk,Hkv,d] uint8 E4M3 codes with float32 block
    factors [B,H,ceil(N/128)]; returns O bf16 [B,Nq,Hq,d] and L float32 [B,Hq,Nq]."""
    import torch
    q8, k8, v8 = _dev(q8), _dev(k8), _dev(v8)
    qs, ks, vs = (_dev(t).to(torch.float32) for t in (q_scale, k_scale, v_scale))
    B, Nq, Hq, d = q8.shape
    _, Nk, Hkv, _ = k8.shape
    if scale is None:
        scale = d ** -0.5
    o = torch.empty((B, Nq, Hq, d), dtype=torch.bfloat16, device=q8.device) if out is None else out
    L = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q8.device) if lse is None else lse
    _check(fa_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), qs.data_ptr(), ks.data_ptr(), vs.data_ptr(),
                      o.data_ptr(), L.data_ptr(), B, Hq, Hkv, Nq, Nk, d, float(scale), int(bool(causal)),
                      _stream(stream)), "fa_fwd_fp8")
    return o, L
