"""Tiled online-softmax forward in plain numpy fp64 (TEST INFRASTRUCTURE ONLY).

Written from the step list of the forward algorithm on "FlashAttention/zh"
(section "FlashAttention algorithm"), in its notation: Q is split into blocks
of B_r rows and K, V into blocks of B_c rows; for each query block
O_i = 0, m_i = -inf, l_i = 0; for each key/value block the score block
S_ij, its row max m_ij and the local exponentials P~_ij = exp(S_ij - m_ij) are
formed, then m_new = max(m_i, m_ij), O_i and l_i are rescaled by
exp(m_i - m_new) and the block adds P~_ij V_j exp(m_ij - m_new) to O_i and
rowsum(P~_ij) exp(m_ij - m_new) to l_i. At the end O_i / l_i is the output and
L_i = m_i + log l_i. With B_c = 1 this is the scalar recurrence of the
"online softmax" section (Milakov and Gimelshein).

It exists only so the tests can pin the two-pass oracle to the tiled method
by brute force on tiny shapes. Masking follows the oracle's conventions
(causal is bottom-right aligned, fully masked rows give O = 0, L = -inf).
"""
from __future__ import annotations

import numpy as np


def fwd_head(Q, K, V, scale, Br, Bc, causal=False, keep=None):
    Q, K, V = (np.asarray(t, dtype=np.float64) for t in (Q, K, V))
    Nq, d = Q.shape
    Nk = K.shape[0]
    O = np.zeros((Nq, V.shape[1]))
    L = np.zeros(Nq)
    for r0 in range(0, Nq, Br):
        rows = np.arange(r0, min(r0 + Br, Nq))
        Oi = np.zeros((len(rows), V.shape[1]))
        mi = np.full(len(rows), -np.inf)
        li = np.zeros(len(rows))
        for c0 in range(0, Nk, Bc):
            cols = np.arange(c0, min(c0 + Bc, Nk))
            Sij = scale * Q[rows] @ K[cols].T
            allowed = np.ones_like(Sij, dtype=bool)
            if causal:
                allowed &= cols[None, :] <= rows[:, None] + (Nk - Nq)
            if keep is not None:
                allowed &= np.asarray(keep, dtype=bool)[cols][None, :]
            Sij = np.where(allowed, Sij, -np.inf)
            mij = Sij.max(axis=1)
            live = np.isfinite(mij)  # rows of this block with at least one visible key
            mij_safe = np.where(live, mij, 0.0)
            Pij = np.where(allowed, np.exp(Sij - mij_safe[:, None]), 0.0)
            m_new = np.maximum(mi, mij)
            m_new_safe = np.where(np.isfinite(m_new), m_new, 0.0)
            alpha = np.where(np.isfinite(mi), np.exp(mi - m_new_safe), 0.0)
            beta = np.where(live, np.exp(mij_safe - m_new_safe), 0.0)
            Oi = Oi * alpha[:, None] + (Pij @ V[cols]) * beta[:, None]
            li = li * alpha + Pij.sum(axis=1) * beta
            mi = m_new
        nz = li > 0
        O[rows] = np.where(nz[:, None], Oi / np.where(nz, li, 1.0)[:, None], 0.0)
        L[rows] = np.where(nz, mi + np.log(np.where(nz, li, 1.0)), -np.inf)
    return O, L
