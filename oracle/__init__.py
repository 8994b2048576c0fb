"""fp64 CPU oracle for exact attention: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product library never loads it and
shares no code with it: the only thing both sides share are the seeded
input generators, which hold no attention arithmetic.

Contents
--------
``attn_oracle.c``  the plain definition in C (fp64, OpenMP): one full row of
                   scores per query, two-pass safe softmax, P.V, L = m + ln l,
                   and the exact analytic backward. Built by :func:`build`.
``numpy_ref.py``   an independent whole-matrix numpy version for tiny shapes.
``online.py``      the tiled online-softmax forward written from the pages'
                   step list, used only to pin "online == two-pass".

Every function here works on float64 numpy arrays in the layouts documented
in ``attn_oracle.c`` (q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d], lse [B,Hq,Nq]).
Parity of every function is pinned by ``tests/test_oracle.py`` against
closed forms, invariants, brute force and finite differences.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import time

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "liboracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)
_up = ctypes.POINTER(ctypes.c_ubyte)


def build(force: bool = False) -> str:
    """Compile the C oracle (plain gcc, -O2, OpenMP) into oracle/_build."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", _SRC,
                               "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.ora_attn_fwd.restype = ctypes.c_int
        lib.ora_attn_fwd.argtypes = [_dp, _dp, _dp] + [ctypes.c_int] * 6 + [ctypes.c_double, ctypes.c_int,
                                                                            ctypes.c_int, ctypes.c_int, _up, _ip,
                                                                            ctypes.c_int, _dp, _dp]
        lib.ora_attn_probs.restype = ctypes.c_int
        lib.ora_attn_probs.argtypes = [_dp, _dp] + [ctypes.c_int] * 6 + [ctypes.c_double, ctypes.c_int,
                                                                         ctypes.c_int, ctypes.c_int, _up,
                                                                         ctypes.c_int, ctypes.c_int, _dp]
        lib.ora_attn_bwd.restype = ctypes.c_int
        lib.ora_attn_bwd.argtypes = [_dp, _dp, _dp, _dp] + [ctypes.c_int] * 6 + [ctypes.c_double, ctypes.c_int,
                                                                                 ctypes.c_int, ctypes.c_int, _up,
                                                                                 _dp, _dp, _dp]
        lib.ora_attn_bwd_sampled.restype = ctypes.c_int
        lib.ora_attn_bwd_sampled.argtypes = ([_dp, _dp, _dp, _dp] + [ctypes.c_int] * 6 +
                                             [ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int, _up,
                                              ctypes.c_int,
                                              ctypes.c_int,
                                              _ip, ctypes.c_int, _ip, ctypes.c_int, _dp, _dp, _dp])
        lib.ora_num_threads.restype = ctypes.c_int
        lib.ora_set_num_threads.restype = None
        lib.ora_set_num_threads.argtypes = [ctypes.c_int]
        _lib = lib
    return _lib


def _window(causal, window):
    """(wl, wr, na) of the C oracle: keys visible to query i are those within wl
    before and wr after its bottom-right-aligned key (a negative side is
    unbounded), and below the window also the global anchor keys 0 .. na - 1
    (``window`` = (wl, wr) or (wl, wr, n_anchor))."""
    if window is not None:
        w = [int(x) for x in window]
        wl, wr = w[0], w[1]
        na = w[2] if len(w) > 2 else 0
        return (wl if wl >= 0 else -1), (wr if wr >= 0 else -1), max(na, 0)
    return (-1, 0, 0) if causal else (-1, -1, 0)


def num_threads() -> int:
    return int(_load().ora_num_threads())


def set_num_threads(n: int) -> None:
    """Threads the oracle's parallel loops use from now on."""
    _load().ora_set_num_threads(int(n))


def _f64(x) -> np.ndarray:
    """Exact upcast of a bf16/fp16/fp32 tensor or array to contiguous float64."""
    if hasattr(x, "detach"):
        import torch
        x = x.detach().to("cpu").to(torch.float64).numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a: np.ndarray, t=_dp):
    return a.ctypes.data_as(t)


def _mask_ptr(key_keep, B, Nk):
    if key_keep is None:
        return None, None
    kk = np.ascontiguousarray(np.asarray(key_keep, dtype=np.uint8).reshape(B, Nk))
    return kk, _ptr(kk, _up)


def attn_fwd(q, k, v, scale: float, causal: bool = False, key_keep=None, rows=None, window=None):
    """O [B,Nq,Hq,d] and L [B,Hq,Nq] in fp64 by the plain definition.

    ``window`` = (wl, wr) replaces ``causal`` with a sliding window (see _window).

    ``rows`` (sequence of query indices) restricts the work to those rows;
    the other entries of the returned arrays are NaN.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    o = np.full((B, Nq, Hq, d), np.nan)
    lse = np.full((B, Hq, Nq), np.nan)
    kk, kp = _mask_ptr(key_keep, B, Nk)
    if rows is not None:
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
        assert r.size == 0 or (r.min() >= 0 and r.max() < Nq)
        rp, nr = _ptr(r, _ip), int(r.size)
    else:
        r, rp, nr = None, None, 0
    if B * Hq * (nr if rows is not None else Nq) > 0:
        err = _load().ora_attn_fwd(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Nq, Nk, d, float(scale),
                                   *_window(causal, window), kp, rp, nr, _ptr(o), _ptr(lse))
        if err:
            raise RuntimeError(f"ora_attn_fwd failed with code {err}")
    return o, lse


def rms_normalise(x, eps: float, out_dtype=None):
    """Per-row RMS normalisation over the last axis, unit gain, in fp64:
    x / sqrt(mean(x^2) + eps). This is the Q/K normalisation the InternViT
    attention applies before FlashAttention. With ``out_dtype`` (a torch dtype)
    the result is rounded once to that type, as the tensor core consumes it
    (the reading this build takes for the fused normalisation)."""
    xf = _f64(x)
    y = xf / np.sqrt((xf * xf).mean(axis=-1, keepdims=True) + eps)
    if out_dtype is None:
        return y
    import torch
    return torch.from_numpy(y).to(out_dtype)


def attn_probs(q, k, scale: float, b: int, h: int, causal: bool = False, key_keep=None, window=None):
    """The Nq x Nk probability matrix of one (batch, query head)."""
    q, k = _f64(q), _f64(k)
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    P = np.zeros((Nq, Nk))
    kk, kp = _mask_ptr(key_keep, B, Nk)
    err = _load().ora_attn_probs(_ptr(q), _ptr(k), B, Hq, Hkv, Nq, Nk, d, float(scale),
                                 *_window(causal, window), kp, b, h, _ptr(P))
    if err:
        raise RuntimeError(f"ora_attn_probs failed with code {err}")
    return P


def attn_bwd(q, k, v, do, scale: float, causal: bool = False, key_keep=None, window=None):
    """dQ, dK, dV in fp64 by the exact gradient of the definition."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    kk, kp = _mask_ptr(key_keep, B, Nk)
    err = _load().ora_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(do), B, Hq, Hkv, Nq, Nk, d,
                               float(scale), *_window(causal, window), kp, _ptr(dq), _ptr(dk), _ptr(dv))
    if err:
        raise RuntimeError(f"ora_attn_bwd failed with code {err}")
    return dq, dk, dv


def attn_bwd_sampled(q, k, v, do, scale: float, b: int, hk: int, qrows, krows,
                     causal: bool = False, key_keep=None, window=None):
    """Gradients of sampled rows of one (batch, KV head) group.

    Returns (dq_rows [len(qrows), group, d], dk_rows [len(krows), d],
    dv_rows [len(krows), d]) where group = Hq/Hkv query heads hk*group...
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    group = Hq // Hkv
    qr = np.ascontiguousarray(np.asarray(qrows, dtype=np.int32))
    kr = np.ascontiguousarray(np.asarray(krows, dtype=np.int32))
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    kk, kp = _mask_ptr(key_keep, B, Nk)
    err = _load().ora_attn_bwd_sampled(_ptr(q), _ptr(k), _ptr(v), _ptr(do), B, Hq, Hkv, Nq, Nk, d,
                                       float(scale), *_window(causal, window), kp, b, hk, _ptr(qr, _ip),
                                       int(qr.size), _ptr(kr, _ip), int(kr.size), _ptr(dq), _ptr(dk),
                                       _ptr(dv))
    if err:
        raise RuntimeError(f"ora_attn_bwd_sampled failed with code {err}")
    return (dq[b][qr][:, hk * group:(hk + 1) * group, :], dk[b, kr, hk, :], dv[b, kr, hk, :])


def varlen_fwd(q, k, v, cu_q, cu_k, scale: float, causal: bool = False, window=None):
    """Packed variable-length forward: each sequence is an independent B=1 problem.

    q [total_q,Hq,d], k/v [total_k,Hkv,d]; returns O [total_q,Hq,d] and
    L [Hq,total_q]. This follows the cu_seqlens addressing of the packed path
    on the InternViT page: sequence s owns rows cu[s] .. cu[s+1]-1. ``window``
    applies attn_fwd's window within every sequence.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    cu_q = [int(x) for x in np.asarray(cu_q)]
    cu_k = [int(x) for x in np.asarray(cu_k)]
    T, Hq, d = q.shape
    o = np.zeros((T, Hq, d))
    lse = np.zeros((Hq, T))
    for s in range(len(cu_q) - 1):
        a, e = cu_q[s], cu_q[s + 1]
        ka, ke = cu_k[s], cu_k[s + 1]
        if e == a:
            continue
        os_, ls = attn_fwd(q[None, a:e], k[None, ka:ke], v[None, ka:ke], scale, causal, window=window)
        o[a:e] = os_[0]
        lse[:, a:e] = ls[0]
    return o, lse


def lse_merge(o_parts, l_parts):
    """Merge of partial results over disjoint key sets, in fp64.

    ``o_parts[s]`` is the attention output over key set s alone (normalised by
    its own sum) and ``l_parts[s]`` its log-sum-exp. Over the union,
    L = log sum_s exp(L_s) and O = sum_s exp(L_s - L) O_s: the rescaling step of
    the online softmax ("FlashAttention/zh", section "online softmax trick")
    applied to whole partial results. Parts with L_s = -inf (no key) weigh 0; if
    every part is empty, O = 0 and L = -inf. Shapes: o_parts [S, ..., d],
    l_parts [S, ...]."""
    o = np.asarray(o_parts, dtype=np.float64)
    l = np.asarray(l_parts, dtype=np.float64)
    lm = l.max(axis=0)
    empty = ~np.isfinite(lm)
    lm_safe = np.where(empty, 0.0, lm)
    w = np.where(np.isfinite(l), np.exp(l - lm_safe[None]), 0.0)
    ws = w.sum(axis=0)
    O = (w[..., None] * np.where(np.isfinite(l)[..., None], o, 0.0)).sum(axis=0)
    O = np.where(empty[..., None], 0.0, O / np.where(empty, 1.0, ws)[..., None])
    L = np.where(empty, -np.inf, lm_safe + np.log(np.where(empty, 1.0, ws)))
    return O, L


def paged_gather(pool, table_row, length: int, page_size: int):
    """Keys 0 .. length-1 of one sequence of a paged cache: key p is row
    p % page_size of page table_row[p // page_size] of ``pool``
    [num_pages, page_size, H, d]. Returns [length, H, d]."""
    pos = np.arange(int(length))
    tr = np.asarray(table_row, dtype=np.int64)
    return np.asarray(pool)[tr[pos // page_size], pos % page_size]


def attn_decode(q, k, v, scale: float, seqlens=None, causal: bool = False):
    """Attention of the Nq newest query tokens of each sequence against its
    cache: sequence b attends to its first seqlens[b] keys (all Nk when
    ``seqlens`` is None), as an independent problem of the plain definition
    (attn_fwd; causal is bottom-right aligned within the sequence's keys).
    q [B,Nq,Hq,d], k/v [B,Nk,Hkv,d]; returns O [B,Nq,Hq,d], L [B,Hq,Nq]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, Hq, d = q.shape
    Nk = k.shape[1]
    o = np.zeros((B, Nq, Hq, d))
    lse = np.full((B, Hq, Nq), -np.inf)
    for b in range(B):
        n = Nk if seqlens is None else min(max(int(seqlens[b]), 0), Nk)
        if n == 0 or Nq == 0:
            continue
        ob, lb = attn_fwd(q[b:b + 1], k[b:b + 1, :n], v[b:b + 1, :n], scale, causal)
        o[b], lse[b] = ob[0], lb[0]
    return o, lse


def e4m3_decode(codes):
    """Values of E4M3 bytes in fp64, from the format's definition: 1 sign bit, 4
    exponent bits with bias 7, 3 mantissa bits; exponent field 0 is subnormal
    (m / 8 * 2^-6); the all-ones pattern S.1111.111 is NaN; there is no infinity.
    The largest finite value is 1.75 * 2^8 = 448."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7))
    val = np.where((e == 0xF) & (m == 0x7), np.nan, val)
    return sign * val


def fp8_dequantise(codes, scales, block: int = 128):
    """Real values of a block-scaled E4M3 tensor: codes [B, N, H, d], scales
    [B, H, ceil(N / block)]; element (b, i, h, c) = scales[b, h, i // block] *
    e4m3(codes[b, i, h, c])."""
    x = e4m3_decode(codes)
    sc = np.asarray(scales, dtype=np.float64)
    N = x.shape[1]
    blk = np.arange(N) // block
    return x * np.transpose(sc[:, :, blk], (0, 2, 1))[..., None]


def attn_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, scale: float, causal: bool = False):
    """The FP8 forward's exact result: the plain definition (attn_fwd) on the
    dequantised block-scaled E4M3 inputs."""
    return attn_fwd(fp8_dequantise(q8, q_scale), fp8_dequantise(k8, k_scale), fp8_dequantise(v8, v_scale),
                    scale, causal)


def timed(fn, *args, **kw):
    """(result, seconds) of one call."""
    t0 = time.perf_counter()
    r = fn(*args, **kw)
    return r, time.perf_counter() - t0
