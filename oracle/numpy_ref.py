"""Independent whole-matrix fp64 attention in numpy (TEST INFRASTRUCTURE ONLY).

A second, separately written statement of the same definition as
``attn_oracle.c``, used only on tiny shapes to cross-check it: S = scale Q K^T
as a full matrix, masked entries -inf, softmax by subtracting the row max,
O = P V and L = m + ln(l) ("FlashAttention/zh", sections "why standard
attention is slow" and "FlashAttention algorithm"); the backward is the exact
gradient of that definition, with KV-head gradients summed over the query
heads of a group.
"""
from __future__ import annotations

import numpy as np


def _mask(Nq, Nk, causal, keep_row, window=None):
    """Allowed (query, key) pairs. A window (wl, wr) allows the keys from wl
    before to wr after the bottom-right-aligned diagonal (a negative side is
    unbounded); it replaces `causal`, which is the window (-1, 0). A third entry
    n_anchor also allows keys 0 .. n_anchor - 1 below the window (global anchors)."""
    allowed = np.ones((Nq, Nk), dtype=bool)
    diag = np.arange(Nk)[None, :] - np.arange(Nq)[:, None] - (Nk - Nq)  # key offset from the aligned diagonal
    if window is not None:
        wl, wr = window[0], window[1]
        anchor = np.arange(Nk)[None, :] < (window[2] if len(window) > 2 else 0)  # global anchor keys
        if wl >= 0:
            allowed &= (diag >= -wl) | anchor
        if wr >= 0:
            allowed &= diag <= wr
    elif causal:
        allowed &= diag <= 0
    if keep_row is not None:
        allowed &= np.asarray(keep_row, dtype=bool)[None, :]
    return allowed


def fwd(q, k, v, scale, causal=False, key_keep=None, window=None):
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, Nq))
    for b in range(B):
        allowed = _mask(Nq, Nk, causal, None if key_keep is None else key_keep[b], window)
        for h in range(Hq):
            S = scale * q[b, :, h, :] @ k[b, :, h // g, :].T
            S = np.where(allowed, S, -np.inf)
            m = S.max(axis=1, keepdims=True)
            empty = ~np.isfinite(m[:, 0])
            m_safe = np.where(np.isfinite(m), m, 0.0)
            E = np.where(allowed, np.exp(S - m_safe), 0.0)
            l = E.sum(axis=1, keepdims=True)
            P = E / np.where(l > 0, l, 1.0)
            o[b, :, h, :] = P @ v[b, :, h // g, :]
            lse[b, h] = np.where(empty, -np.inf, m[:, 0] + np.log(np.where(l[:, 0] > 0, l[:, 0], 1.0)))
    return o, lse


def bwd(q, k, v, do, scale, causal=False, key_keep=None, window=None):
    q, k, v, do = (np.asarray(t, dtype=np.float64) for t in (q, k, v, do))
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        allowed = _mask(Nq, Nk, causal, None if key_keep is None else key_keep[b], window)
        for h in range(Hq):
            K = k[b, :, h // g, :]
            V = v[b, :, h // g, :]
            Q = q[b, :, h, :]
            dO = do[b, :, h, :]
            S = np.where(allowed, scale * Q @ K.T, -np.inf)
            m = S.max(axis=1, keepdims=True)
            m = np.where(np.isfinite(m), m, 0.0)
            E = np.where(allowed, np.exp(S - m), 0.0)
            l = E.sum(axis=1, keepdims=True)
            P = E / np.where(l > 0, l, 1.0)
            dP = dO @ V.T
            D = (P * dP).sum(axis=1, keepdims=True)
            dS = P * (dP - D)
            dq[b, :, h, :] = scale * dS @ K
            dk[b, :, h // g, :] += scale * dS.T @ Q
            dv[b, :, h // g, :] += P.T @ dO
    return dq, dk, dv
