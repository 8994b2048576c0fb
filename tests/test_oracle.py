"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these compares the oracle with itself: each check is a closed form,
an invariant, a hand-worked example, brute force through a separately
written implementation, or finite differences. CPU only.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import numpy_ref, online
from exact_tiled_attention_36_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _num(x):
    if isinstance(x, str):
        import re
        return eval(re.sub(r"ln(\d+)", r"math.log(\1)", x), {"math": math, "inf": math.inf})  # "ln3", "-inf"
    return float(x)


def _grid(a):
    return np.array([[_num(x) for x in row] for row in a])


# ---------------------------------------------------------------- golden example
def test_golden_two_key_example():
    """Hand-worked example: tests/golden/two_key_example.json."""
    g = json.load(open(os.path.join(GOLDEN, "two_key_example.json")))
    q = _grid(g["q"])[None, :, None, :]
    k = _grid(g["k"])[None, :, None, :]
    v = _grid(g["v"])[None, :, None, :]
    do = _grid(g["do"])[None, :, None, :]
    o, lse = oracle.attn_fwd(q, k, v, g["scale"])
    np.testing.assert_allclose(o[0, :, 0, :], _grid(g["o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], [_num(x) for x in g["lse"]], rtol=0, atol=1e-14)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, g["scale"])
    np.testing.assert_allclose(dq[0, :, 0, :], _grid(g["dq"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(dk[0, :, 0, :], _grid(g["dk"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(dv[0, :, 0, :], _grid(g["dv"]), rtol=0, atol=1e-14)


def _mask_cases():
    g = json.load(open(os.path.join(GOLDEN, "mask_alignment_examples.json")))
    return g["cases"]


@pytest.mark.parametrize("case", _mask_cases(), ids=lambda c: c["name"])
def test_golden_mask_alignment_examples(case):
    """Hand-worked causal (bottom-right, Nq != Nk), window and anchor examples:
    tests/golden/mask_alignment_examples.json. The forward, the decode wrapper
    (the keys as a sequence's cache, NaN past its length), the packed varlen
    wrapper and the tiled online recurrence all give the worked values."""
    q = _grid(case["q"])[None, :, None, :]
    k = _grid(case["k"])[None, :, None, :]
    v = _grid(case["v"])[None, :, None, :]
    o_ref = _grid(case["o"])
    l_ref = np.array([_num(x) for x in case["lse"]])
    causal, window = case["causal"], case["window"]
    o, lse = oracle.attn_fwd(q, k, v, 1.0, causal, window=window)
    np.testing.assert_allclose(o[0, :, 0, :], o_ref, rtol=0, atol=1e-14)
    np.testing.assert_array_equal(np.isneginf(lse[0, 0]), np.isneginf(l_ref))
    live = np.isfinite(l_ref)
    np.testing.assert_allclose(lse[0, 0][live], l_ref[live], rtol=0, atol=1e-14)
    Nq, Nk = q.shape[1], k.shape[1]
    if window is None:
        # the same keys as the first Nk rows of a 3-row-longer cache, the rest NaN
        kc = np.concatenate([k, np.full((1, 3, 1, 1), np.nan)], axis=1)
        vc = np.concatenate([v, np.full((1, 3, 1, 1), np.nan)], axis=1)
        od, ld = oracle.attn_decode(q, kc, vc, 1.0, [Nk], causal)
        np.testing.assert_allclose(od[0, :, 0, :], o_ref, rtol=0, atol=1e-14)
        np.testing.assert_allclose(ld[0, 0][live], l_ref[live], rtol=0, atol=1e-14)
        assert np.isneginf(ld[0, 0][~live]).all()
        for Br, Bc in ((1, 1), (2, 2), (4, 1)):
            O2, L2 = online.fwd_head(q[0, :, 0], k[0, :, 0], v[0, :, 0], 1.0, Br, Bc, causal=causal)
            np.testing.assert_allclose(O2, o_ref, rtol=0, atol=1e-14)
            np.testing.assert_allclose(L2[live], l_ref[live], rtol=0, atol=1e-14)
    # packed after a 2-row sequence of its own: the example's rows are unchanged
    rng = np.random.default_rng(5)
    q0, k0, v0 = rng.standard_normal((2, 1, 1)), rng.standard_normal((2, 1, 1)), rng.standard_normal((2, 1, 1))
    ov, lv = oracle.varlen_fwd(np.concatenate([q0, q[0]]), np.concatenate([k0, k[0]]), np.concatenate([v0, v[0]]),
                               [0, 2, 2 + Nq], [0, 2, 2 + Nk], 1.0, causal, window=window)
    np.testing.assert_allclose(ov[2:, 0, :], o_ref, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lv[0, 2:][live], l_ref[live], rtol=0, atol=1e-14)


# ---------------------------------------------------------------- softmax pins
@pytest.mark.parametrize("causal", [False, True])
def test_rows_of_p_sum_to_one(causal):
    rng = np.random.default_rng(1)
    q, k = _rand(rng, 2, 19, 4, 8), _rand(rng, 2, 23, 2, 8)
    for b in range(2):
        for h in range(4):
            P = oracle.attn_probs(q, k, 0.7, b, h, causal=causal)
            assert (P >= 0).all()
            np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-14)
            if causal:  # bottom-right alignment: key j visible to row i iff j <= i + Nk - Nq
                i, j = np.nonzero(P)
                assert (j <= i + (23 - 19)).all()


def test_lse_is_logsumexp_of_scores():
    """L_i = log sum_j exp(S_ij), computed independently with math.fsum."""
    rng = np.random.default_rng(2)
    B, Nq, Nk, H, d, scale = 1, 7, 11, 2, 5, 0.9
    q, k, v = _rand(rng, B, Nq, H, d), _rand(rng, B, Nk, H, d), _rand(rng, B, Nk, H, d)
    _, lse = oracle.attn_fwd(q, k, v, scale)
    for h in range(H):
        for i in range(Nq):
            s = [scale * math.fsum(q[0, i, h, c] * k[0, j, h, c] for c in range(d)) for j in range(Nk)]
            mx = max(s)
            ref = mx + math.log(math.fsum(math.exp(x - mx) for x in s))
            assert abs(lse[0, h, i] - ref) < 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_zero_queries_give_column_mean(causal):
    """Q = 0 makes every score 0: O_i is the mean of the visible V rows, L_i = ln(#visible)."""
    rng = np.random.default_rng(3)
    N, d = 13, 6
    q = np.zeros((1, N, 2, d))
    k, v = _rand(rng, 1, N, 2, d), _rand(rng, 1, N, 2, d)
    o, lse = oracle.attn_fwd(q, k, v, 0.5, causal=causal)
    for h in range(2):
        for i in range(N):
            n = i + 1 if causal else N
            np.testing.assert_allclose(o[0, i, h], v[0, :n, h].mean(axis=0), rtol=0, atol=1e-14)
            assert abs(lse[0, h, i] - math.log(n)) < 1e-14


def test_dominant_logit_selects_its_value_row():
    d, N = 8, 8
    keys = np.eye(N, d)  # orthonormal keys
    rng = np.random.default_rng(4)
    v = _rand(rng, 1, N, 1, d)
    for jstar in range(N):
        t = 60.0
        q = (t * keys[jstar])[None, None, None, :]
        o, lse = oracle.attn_fwd(q, keys[None, :, None, :], v, 1.0)
        # other logits are 0: weight of the rest is (N-1) e^-t
        np.testing.assert_allclose(o[0, 0, 0], v[0, jstar, 0], atol=1e-20 + 8 * (N - 1) * math.exp(-t))
        assert abs(lse[0, 0, 0] - (t + math.log1p((N - 1) * math.exp(-t)))) < 1e-12


def test_single_key():
    rng = np.random.default_rng(5)
    q, k, v = _rand(rng, 2, 9, 3, 4), _rand(rng, 2, 1, 3, 4), _rand(rng, 2, 1, 3, 4)
    o, lse = oracle.attn_fwd(q, k, v, 0.3)
    np.testing.assert_allclose(o, np.broadcast_to(v, o.shape), rtol=0, atol=0)
    s = 0.3 * np.einsum("bihc,bjhc->bhi", q, k)
    np.testing.assert_allclose(lse, s, rtol=0, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_fully_masked_rows_are_zero_and_minus_inf(causal):
    rng = np.random.default_rng(6)
    q, k, v = _rand(rng, 1, 9, 1, 4), _rand(rng, 1, 5, 1, 4), _rand(rng, 1, 5, 1, 4)
    keep = np.ones((1, 5), dtype=np.uint8)
    if not causal:
        keep[:] = 0  # every key masked
    o, lse = oracle.attn_fwd(q, k, v, 1.0, causal=causal, key_keep=keep)
    empty = range(4) if causal else range(9)  # causal: rows i < Nq - Nk see no key
    for i in empty:
        assert (o[0, i] == 0).all() and lse[0, 0, i] == -np.inf
    if causal:
        assert np.isfinite(lse[0, 0, 4:]).all()


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("N", [1, 2, 5, 17, 33])
@pytest.mark.parametrize("d", [1, 4, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_online_softmax_equals_two_pass(N, d, causal):
    """The tiled online recurrence (any B_r, B_c; B_c = 1 is the scalar recurrence) equals the two-pass oracle."""
    rng = np.random.default_rng(100 + N * 10 + d)
    Nk = N + (3 if causal else 0)
    q, k, v = 2 * _rand(rng, 1, N, 1, d), 2 * _rand(rng, 1, Nk, 1, d), _rand(rng, 1, Nk, 1, d)
    o, lse = oracle.attn_fwd(q, k, v, 0.8, causal=causal)
    for Br in (1, 4, N):
        for Bc in (1, 2, 3, 8, Nk):
            O2, L2 = online.fwd_head(q[0, :, 0], k[0, :, 0], v[0, :, 0], 0.8, Br, Bc, causal=causal)
            np.testing.assert_allclose(O2, o[0, :, 0], rtol=0, atol=1e-12)
            np.testing.assert_allclose(L2, lse[0, 0], rtol=0, atol=1e-12)


def test_online_with_key_mask_equals_two_pass():
    rng = np.random.default_rng(7)
    q, k, v = _rand(rng, 1, 12, 1, 4), _rand(rng, 1, 14, 1, 4), _rand(rng, 1, 14, 1, 4)
    keep = (rng.random((1, 14)) > 0.4).astype(np.uint8)
    o, lse = oracle.attn_fwd(q, k, v, 1.1, key_keep=keep)
    O2, L2 = online.fwd_head(q[0, :, 0], k[0, :, 0], v[0, :, 0], 1.1, 5, 3, keep=keep[0])
    np.testing.assert_allclose(O2, o[0, :, 0], atol=1e-12)
    np.testing.assert_allclose(L2, lse[0, 0], atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2), (3, 1)])
def test_numpy_crosscheck(causal, Hq, Hkv):
    rng = np.random.default_rng(8)
    B, Nq, Nk, d = 2, 11, 13, 8
    q, k, v, do = (_rand(rng, B, Nq, Hq, d), _rand(rng, B, Nk, Hkv, d), _rand(rng, B, Nk, Hkv, d),
                   _rand(rng, B, Nq, Hq, d))
    keep = (rng.random((B, Nk)) > 0.2).astype(np.uint8)
    for kk in (None, keep):
        o, lse = oracle.attn_fwd(q, k, v, 0.35, causal, kk)
        o2, lse2 = numpy_ref.fwd(q, k, v, 0.35, causal, kk)
        np.testing.assert_allclose(o, o2, atol=1e-12)
        np.testing.assert_array_equal(np.isinf(lse), np.isinf(lse2))
        fin = np.isfinite(lse)
        np.testing.assert_allclose(lse[fin], lse2[fin], atol=1e-12)
        g1 = oracle.attn_bwd(q, k, v, do, 0.35, causal, kk)
        g2 = numpy_ref.bwd(q, k, v, do, 0.35, causal, kk)
        for a, b in zip(g1, g2):
            np.testing.assert_allclose(a, b, atol=1e-11)


# ---------------------------------------------------------------- invariants
def test_permutation_invariance_non_causal():
    rng = np.random.default_rng(9)
    q, k, v = _rand(rng, 1, 10, 2, 6), _rand(rng, 1, 15, 2, 6), _rand(rng, 1, 15, 2, 6)
    o, lse = oracle.attn_fwd(q, k, v, 0.4)
    perm = rng.permutation(15)
    o2, lse2 = oracle.attn_fwd(q, k[:, perm], v[:, perm], 0.4)
    np.testing.assert_allclose(o2, o, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, atol=1e-13)


def test_linear_in_v_and_constant_v():
    rng = np.random.default_rng(10)
    q, k = _rand(rng, 1, 10, 2, 6), _rand(rng, 1, 12, 2, 6)
    v1, v2 = _rand(rng, 1, 12, 2, 6), _rand(rng, 1, 12, 2, 6)
    o1, _ = oracle.attn_fwd(q, k, v1, 0.4, causal=True)
    o2, _ = oracle.attn_fwd(q, k, v2, 0.4, causal=True)
    o3, _ = oracle.attn_fwd(q, k, 2.0 * v1 - 3.0 * v2, 0.4, causal=True)
    np.testing.assert_allclose(o3, 2.0 * o1 - 3.0 * o2, atol=1e-12)
    c = np.full((1, 12, 2, 6), 1.25)
    oc, _ = oracle.attn_fwd(q, k, c, 0.4, causal=True)
    np.testing.assert_allclose(oc, 1.25, atol=1e-14)


# ---------------------------------------------------------------- backward
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (2, 1)])
def test_backward_matches_finite_differences(causal, Hq, Hkv):
    """phi = sum(dO * O); central differences with h = 1e-6, relative error <= 1e-6."""
    rng = np.random.default_rng(11)
    B, Nq, Nk, d, scale = 1, 5, 7, 4, 0.6
    q, k, v, do = (_rand(rng, B, Nq, Hq, d), _rand(rng, B, Nk, Hkv, d), _rand(rng, B, Nk, Hkv, d),
                   _rand(rng, B, Nq, Hq, d))
    grads = oracle.attn_bwd(q, k, v, do, scale, causal)

    def phi(qq, kk, vv):
        o, _ = oracle.attn_fwd(qq, kk, vv, scale, causal)
        return float((o * do).sum())

    h = 1e-6
    for which, g in zip(range(3), grads):
        base = [q, k, v]
        fd = np.zeros_like(base[which])
        it = np.nditer(base[which], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = [t.copy() for t in base]
            minus = [t.copy() for t in base]
            plus[which][idx] += h
            minus[which][idx] -= h
            fd[idx] = (phi(*plus) - phi(*minus)) / (2 * h)
        rel = np.linalg.norm(fd - g) / np.linalg.norm(g)
        assert rel <= 1e-6, (which, rel)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_invariants(causal):
    """Rows of dS sum to 0 so sum_j dK_j = 0; rows of P sum to 1 so sum_j dV_j = sum_i dO_i (per KV group)."""
    rng = np.random.default_rng(12)
    B, N, Hq, Hkv, d = 2, 16, 4, 2, 8
    q, k, v, do = (_rand(rng, B, N, Hq, d), _rand(rng, B, N, Hkv, d), _rand(rng, B, N, Hkv, d),
                   _rand(rng, B, N, Hq, d))
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, 0.5, causal)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)
    g = Hq // Hkv
    for hk in range(Hkv):
        np.testing.assert_allclose(dv[:, :, hk].sum(axis=1), do[:, :, hk * g:(hk + 1) * g].sum(axis=(1, 2)),
                                   atol=1e-12)


def test_sampled_rows_match_full():
    rng = np.random.default_rng(13)
    B, N, Hq, Hkv, d = 2, 40, 4, 2, 8
    q, k, v, do = (_rand(rng, B, N, Hq, d), _rand(rng, B, N, Hkv, d), _rand(rng, B, N, Hkv, d),
                   _rand(rng, B, N, Hq, d))
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, 0.5, causal)
        rows = [0, 7, 39, 21]
        o2, lse2 = oracle.attn_fwd(q, k, v, 0.5, causal, rows=rows)
        np.testing.assert_array_equal(o2[:, rows], o[:, rows])
        np.testing.assert_array_equal(lse2[:, :, rows], lse[:, :, rows])
        dq, dk, dv = oracle.attn_bwd(q, k, v, do, 0.5, causal)
        for b in range(B):
            for hk in range(Hkv):
                qr, kr = [3, 39], [0, 38, 39, 12]
                sq, sk, sv = oracle.attn_bwd_sampled(q, k, v, do, 0.5, b, hk, qr, kr, causal)
                np.testing.assert_allclose(sq, dq[b][qr][:, hk * 2:hk * 2 + 2], atol=1e-12)
                np.testing.assert_allclose(sk, dk[b, kr, hk], atol=1e-12)
                np.testing.assert_allclose(sv, dv[b, kr, hk], atol=1e-12)


# ---------------------------------------------------------------- varlen / padding / prep
def test_varlen_equals_each_sequence_alone_and_keypad_equals_truncation():
    cfg = inputs.VARLEN_KEYPAD
    vi = inputs.make_varlen(cfg, lengths=[5, 1, 17, 9], Hq=2, Hkv=1, d=8)
    o, lse = oracle.varlen_fwd(vi.q, vi.k, vi.v, vi.cu_seqlens_q, vi.cu_seqlens_k, 0.3)
    # same result through a tail key mask on the full (padded) K/V of each sequence
    for s, (L, Lk) in enumerate(zip(vi.seqlens_q, vi.seqlens_k)):
        a = int(vi.cu_seqlens_q[s])
        keep = np.zeros((1, L), dtype=np.uint8)
        keep[0, :Lk] = 1
        o2, lse2 = oracle.attn_fwd(vi.q[None, a:a + L], vi.k_padded[None, a:a + L], vi.v_padded[None, a:a + L],
                                   0.3, key_keep=keep)
        np.testing.assert_allclose(o[a:a + L], o2[0], atol=1e-13)
        np.testing.assert_allclose(lse[:, a:a + L], lse2[0], atol=1e-13)
        assert Lk == L - int(0.25 * L)


def test_rmsnorm_prep_closed_form():
    """After prep, each head row has mean(x^2) = ms / (ms + eps) (before the bf16 cast)."""
    import torch
    g = torch.Generator().manual_seed(0)
    x = torch.randn(3, 5, 2, 16, generator=g)
    y = inputs.rms_normalise_rows(x)
    ms = (x.double() ** 2).mean(-1)
    np.testing.assert_allclose((y ** 2).mean(-1).numpy(), (ms / (ms + inputs.RMSNORM_EPS)).numpy(), rtol=1e-13)


def test_inputs_are_seeded_and_shaped():
    a = inputs.make_fixed(inputs.TINY)
    b = inputs.make_fixed(inputs.TINY)
    assert a.q.shape == (1, 256, 2, 64) and str(a.q.dtype) == "torch.bfloat16"
    assert (a.q == b.q).all() and (a.v == b.v).all()
    vi = inputs.make_varlen(inputs.VARLEN, Hq=1, Hkv=1, d=8)
    assert len(vi.seqlens_q) == 32 and min(vi.seqlens_q) >= 64 and max(vi.seqlens_q) <= 4096
    assert int(vi.cu_seqlens_q[-1]) == vi.q.shape[0]


def test_rms_normalise_pins():
    """oracle.rms_normalise against what the definition fixes: the mean square of
    each output row is ms / (ms + eps); a constant row c gives c / sqrt(c^2 + eps);
    eps = 0 makes it invariant to positive scaling and keeps signs; and one
    rounding to bf16 is within half an ulp of the fp64 value."""
    import torch
    rng = np.random.default_rng(7)
    x = rng.standard_normal((5, 3, 16)) * rng.uniform(0.1, 10, (5, 3, 1))
    eps = 1e-3
    y = oracle.rms_normalise(x, eps)
    ms = (x * x).mean(-1)
    np.testing.assert_allclose((y * y).mean(-1), ms / (ms + eps), rtol=1e-12)
    c = np.full((2, 8), -0.25)
    np.testing.assert_allclose(oracle.rms_normalise(c, eps), -0.25 / np.sqrt(0.0625 + eps), rtol=1e-14)
    y0 = oracle.rms_normalise(x, 0.0)
    np.testing.assert_allclose(oracle.rms_normalise(3.5 * x, 0.0), y0, rtol=1e-12)
    assert (np.sign(y0) == np.sign(x)).all()
    yb = oracle.rms_normalise(torch.from_numpy(x).to(torch.bfloat16), eps, torch.bfloat16)
    exact = oracle.rms_normalise(torch.from_numpy(x).to(torch.bfloat16), eps)
    assert yb.dtype == torch.bfloat16
    assert (np.abs(yb.double().numpy() - exact) <= np.abs(exact) * 2.0 ** -8 + 1e-30).all()


WINDOWS = [(2, 1), (0, 3), (5, 0), (-1, 2), (3, -1), (0, 0), (1, 0, 2), (2, 1, 3), (0, -1, 1), (2, 0, 20)]


@pytest.mark.parametrize("window", WINDOWS)
@pytest.mark.parametrize("Nq,Nk,Hq,Hkv", [(9, 9, 2, 1), (6, 11, 2, 2), (12, 7, 4, 2)])
def test_window_numpy_crosscheck(window, Nq, Nk, Hq, Hkv):
    """The C oracle's sliding window (per-element visibility) against the numpy
    version's (a mask matrix built from key offsets), forward and backward."""
    rng = np.random.default_rng(17)
    q, k, v, do = (_rand(rng, 2, Nq, Hq, 4), _rand(rng, 2, Nk, Hkv, 4), _rand(rng, 2, Nk, Hkv, 4),
                   _rand(rng, 2, Nq, Hq, 4))
    o, lse = oracle.attn_fwd(q, k, v, 0.7, window=window)
    o2, lse2 = numpy_ref.fwd(q, k, v, 0.7, window=window)
    np.testing.assert_allclose(o, o2, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(lse2))
    fin = np.isfinite(lse)
    np.testing.assert_allclose(lse[fin], lse2[fin], atol=1e-12)
    g = oracle.attn_bwd(q, k, v, do, 0.7, window=window)
    g2 = numpy_ref.bwd(q, k, v, do, 0.7, window=window)
    for a, b in zip(g, g2):
        np.testing.assert_allclose(a, b, atol=1e-11)


def test_window_special_cases():
    """(-1, 0) is the causal mask; a window covering every key is no mask; the
    window (0, 0) leaves each query its aligned key only, so O_i = V_a and L_i = S_ia,
    and a row whose aligned key lies outside the keys sees nothing."""
    rng = np.random.default_rng(19)
    Nq, Nk = 7, 5
    q, k, v = _rand(rng, 1, Nq, 2, 3), _rand(rng, 1, Nk, 2, 3), _rand(rng, 1, Nk, 2, 3)
    for a, b in zip(oracle.attn_fwd(q, k, v, 0.5, window=(-1, 0)), oracle.attn_fwd(q, k, v, 0.5, causal=True)):
        np.testing.assert_array_equal(a, b)
    for a, b in zip(oracle.attn_fwd(q, k, v, 0.5, window=(Nk + Nq, Nk + Nq)), oracle.attn_fwd(q, k, v, 0.5)):
        np.testing.assert_array_equal(a, b)
    o, lse = oracle.attn_fwd(q, k, v, 0.5, window=(0, 0))
    for i in range(Nq):
        a = i + Nk - Nq
        for h in range(2):
            if 0 <= a < Nk:
                np.testing.assert_allclose(o[0, i, h], v[0, a, h], atol=1e-15)
                assert abs(lse[0, h, i] - 0.5 * float(q[0, i, h] @ k[0, a, h])) <= 1e-14
            else:
                assert (o[0, i, h] == 0).all() and np.isneginf(lse[0, h, i])


@pytest.mark.parametrize("window", [(2, 1), (1, 0, 3)])
def test_window_backward_matches_finite_differences(window):
    rng = np.random.default_rng(23)
    q, k, v, do = _rand(rng, 1, 6, 2, 3), _rand(rng, 1, 8, 1, 3), _rand(rng, 1, 8, 1, 3), _rand(rng, 1, 6, 2, 3)
    scale = 0.6
    grads = oracle.attn_bwd(q, k, v, do, scale, window=window)

    def phi(qq, kk, vv):
        o, _ = oracle.attn_fwd(qq, kk, vv, scale, window=window)
        return float((o * do).sum())

    h = 1e-6
    for which, g in zip(range(3), grads):
        base = [q, k, v]
        fd = np.zeros_like(base[which])
        it = np.nditer(base[which], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = [t.copy() for t in base]
            minus = [t.copy() for t in base]
            plus[which][idx] += h
            minus[which][idx] -= h
            fd[idx] = (phi(*plus) - phi(*minus)) / (2 * h)
        assert np.linalg.norm(fd - g) / np.linalg.norm(g) <= 1e-6, which


# ---------------------------------------------------------------- decode: merge, paged cache, cache lengths
@pytest.mark.parametrize("causal", [False, True])
def test_lse_merge_of_key_chunks_equals_whole(causal):
    """Attention over disjoint key chunks, merged by the log-sum-exp rule, equals
    attention over all keys (the whole-problem oracle, and the numpy version)."""
    rng = np.random.default_rng(51)
    B, Nq, Nk, Hq, Hkv, d = 2, 3, 23, 4, 2, 8
    q, k, v = _rand(rng, B, Nq, Hq, d), _rand(rng, B, Nk, Hkv, d), _rand(rng, B, Nk, Hkv, d)
    o_all, l_all = oracle.attn_fwd(q, k, v, 0.7, causal)
    cuts = [0, 5, 5, 16, Nk]  # one empty chunk
    parts_o, parts_l = [], []
    for a, e in zip(cuts[:-1], cuts[1:]):
        keep = np.zeros((B, Nk), dtype=np.uint8)
        keep[:, a:e] = 1
        o_s, l_s = oracle.attn_fwd(q, k, v, 0.7, causal, key_keep=keep)
        parts_o.append(o_s)
        parts_l.append(np.moveaxis(l_s, 1, 2))  # [B, Nq, Hq] like o's leading axes
    O, L = oracle.lse_merge(parts_o, parts_l)
    np.testing.assert_allclose(O, o_all, atol=1e-12)
    np.testing.assert_allclose(np.moveaxis(L, 2, 1), l_all, atol=1e-12)
    o_np, l_np = numpy_ref.fwd(q, k, v, 0.7, causal)
    np.testing.assert_allclose(O, o_np, atol=1e-12)


def test_lse_merge_special_cases():
    rng = np.random.default_rng(52)
    o1, l1 = _rand(rng, 4, 3), _rand(rng, 4)
    O, L = oracle.lse_merge([o1], [l1])  # one part: unchanged
    np.testing.assert_allclose(O, o1, atol=1e-15)
    np.testing.assert_allclose(L, l1, atol=1e-15)
    O, L = oracle.lse_merge([o1, np.full_like(o1, np.nan)], [l1, np.full_like(l1, -np.inf)])  # empty part ignored
    np.testing.assert_allclose(O, o1, atol=1e-15)
    np.testing.assert_allclose(L, l1, atol=1e-15)
    O, L = oracle.lse_merge([o1, o1], [l1, l1])  # two equal halves: O unchanged, L + ln 2
    np.testing.assert_allclose(O, o1, atol=1e-14)
    np.testing.assert_allclose(L, l1 + math.log(2), atol=1e-14)
    O, L = oracle.lse_merge([o1], [np.full_like(l1, -np.inf)])  # nothing: O = 0, L = -inf
    assert (O == 0).all() and np.isneginf(L).all()


def test_paged_gather_inverts_a_scatter():
    rng = np.random.default_rng(53)
    n, page, H, d = 150, 16, 2, 4
    k = _rand(rng, n, H, d)
    n_pages = (n + page - 1) // page
    table = rng.permutation(20)[:n_pages]  # pages drawn from a pool of 20 in random order
    pool = np.full((20, page, H, d), np.nan)
    for p in range(n):
        pool[table[p // page], p % page] = k[p]
    np.testing.assert_array_equal(oracle.paged_gather(pool, table, n, page), k)
    assert oracle.paged_gather(pool, table, 0, page).shape == (0, H, d)


@pytest.mark.parametrize("causal", [False, True])
def test_attn_decode_pins(causal):
    rng = np.random.default_rng(54)
    B, Nq, Nk, Hq, Hkv, d = 4, 3, 40, 4, 2, 8
    q, k, v = _rand(rng, B, Nq, Hq, d), _rand(rng, B, Nk, Hkv, d), _rand(rng, B, Nk, Hkv, d)
    # every sequence full: the plain forward
    o, l = oracle.attn_decode(q, k, v, 0.5, None, causal)
    o2, l2 = oracle.attn_fwd(q, k, v, 0.5, causal)
    np.testing.assert_allclose(o, o2, atol=1e-13)
    np.testing.assert_allclose(l, l2, atol=1e-13)
    # own lengths: keys past the length never matter (NaN there), and each sequence is
    # the numpy whole-matrix version on its prefix; length 0 gives O = 0, L = -inf
    lens = [40, 17, 0, 2]
    kn, vn = k.copy(), v.copy()
    for b, n in enumerate(lens):
        kn[b, n:] = np.nan
        vn[b, n:] = np.nan
    o, l = oracle.attn_decode(q, kn, vn, 0.5, lens, causal)
    for b, n in enumerate(lens):
        if n == 0:
            assert (o[b] == 0).all() and np.isneginf(l[b]).all()
            continue
        ob, lb = numpy_ref.fwd(q[b:b + 1], k[b:b + 1, :n], v[b:b + 1, :n], 0.5, causal)
        np.testing.assert_allclose(o[b], ob[0], atol=1e-12)
        np.testing.assert_allclose(l[b], lb[0], atol=1e-12)
    if not causal:  # a tail key mask on the full cache is the same thing
        keep = np.zeros((B, Nk), dtype=np.uint8)
        for b, n in enumerate(lens):
            keep[b, :n] = 1
        o3, l3 = oracle.attn_fwd(q, k, v, 0.5, False, key_keep=keep)
        np.testing.assert_allclose(o, o3, atol=1e-13)
        np.testing.assert_allclose(l, l3, atol=1e-13)


# ---------------------------------------------------------------- FP8 (E4M3) inputs
def test_e4m3_decode_matches_torch_and_closed_forms():
    import torch
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(lib))
    ok = ~np.isnan(lib)
    np.testing.assert_array_equal(ours[ok], lib[ok])
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF]) and np.isnan(ours).sum() == 2
    assert ours[0x38] == 1.0 and ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6
    assert ours[0xB8] == -1.0 and ours[0x00] == 0.0 and ours[0x80] == 0.0


def test_fp8_dequantise_blocks_and_attention():
    rng = np.random.default_rng(71)
    B, N, H, d = 2, 300, 3, 4
    codes = rng.integers(0, 256, size=(B, N, H, d), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38  # no NaN codes
    scales = rng.uniform(0.5, 2.0, size=(B, H, 3))
    x = oracle.fp8_dequantise(codes, scales)
    for b, i, h in [(0, 0, 0), (1, 127, 2), (1, 128, 1), (0, 299, 2), (1, 256, 0)]:
        np.testing.assert_array_equal(x[b, i, h], scales[b, h, i // 128] * oracle.e4m3_decode(codes[b, i, h]))
    # with unit scales and codes of exactly representable values the FP8 forward is the plain forward
    q = rng.standard_normal((1, 5, 2, 8))
    k = rng.standard_normal((1, 7, 1, 8))
    v = rng.standard_normal((1, 7, 1, 8))
    import torch
    enc = lambda t: torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    q8, k8, v8 = enc(q), enc(k), enc(v)
    o, l = oracle.attn_fwd_fp8(q8, k8, v8, np.ones((1, 2, 1)), np.ones((1, 1, 1)), np.ones((1, 1, 1)), 0.3, True)
    o2, l2 = numpy_ref.fwd(oracle.e4m3_decode(q8), oracle.e4m3_decode(k8), oracle.e4m3_decode(v8), 0.3, True)
    np.testing.assert_allclose(o, o2, atol=1e-12)
    np.testing.assert_allclose(l, l2, atol=1e-12)


def test_varlen_window_equals_numpy_per_sequence():
    """The varlen forward with a window (and anchors): every sequence is the numpy
    whole-matrix version with the same window on that sequence alone."""
    vi = inputs.make_varlen(inputs.VARLEN, lengths=[9, 1, 30, 0, 17], Hq=4, Hkv=2, d=8)
    # (wl, wr) windows, and (wl, wr, n_anchor) with the first keys of every sequence as anchors
    for window in ((3, 0), (5, 2), (-1, 4), (0, 0), (3, 0, 2), (2, 1, 5), (0, -1, 1)):
        o, lse = oracle.varlen_fwd(vi.q, vi.k, vi.v, vi.cu_seqlens_q, vi.cu_seqlens_k, 0.4, window=window)
        for s, n in enumerate(vi.seqlens_q):
            a = int(vi.cu_seqlens_q[s])
            if n == 0:
                continue
            f = lambda t: t[None, a:a + n].double().numpy()
            o2, l2 = numpy_ref.fwd(f(vi.q), f(vi.k), f(vi.v), 0.4, window=window)
            np.testing.assert_allclose(o[a:a + n], o2[0], atol=1e-12)
            np.testing.assert_allclose(lse[:, a:a + n], l2[0], atol=1e-12)


def test_anchor_special_cases():
    """Global anchors: n_anchor = 0 is the plain window; with an unbounded left side
    anchors add nothing; anchors covering every key with an unbounded right side give
    full attention; with the causal right bound (wr = 0) and a zero-width window, row i
    sees exactly keys {0 .. n_anchor - 1} u {a} below its aligned key a, checked against
    a direct softmax over those keys."""
    rng = np.random.default_rng(29)
    Nq, Nk = 9, 9
    q, k, v = _rand(rng, 1, Nq, 2, 3), _rand(rng, 1, Nk, 1, 3), _rand(rng, 1, Nk, 1, 3)
    for a, b in zip(oracle.attn_fwd(q, k, v, 0.5, window=(2, 1, 0)), oracle.attn_fwd(q, k, v, 0.5, window=(2, 1))):
        np.testing.assert_array_equal(a, b)
    for a, b in zip(oracle.attn_fwd(q, k, v, 0.5, window=(-1, 0, 4)), oracle.attn_fwd(q, k, v, 0.5, causal=True)):
        np.testing.assert_array_equal(a, b)
    for a, b in zip(oracle.attn_fwd(q, k, v, 0.5, window=(0, -1, Nk)), oracle.attn_fwd(q, k, v, 0.5)):
        np.testing.assert_array_equal(a, b)
    o, lse = oracle.attn_fwd(q, k, v, 0.5, window=(0, 0, 3))
    for i in range(Nq):
        keys = sorted(set(range(min(3, i + 1))) | {i})
        for h in range(2):
            s_ = np.array([0.5 * float(q[0, i, h] @ k[0, j, 0]) for j in keys])
            w = np.exp(s_ - s_.max())
            np.testing.assert_allclose(o[0, i, h], (w / w.sum()) @ v[0, keys, 0], atol=1e-14)
            assert abs(lse[0, h, i] - (s_.max() + math.log(w.sum()))) <= 1e-13
