"""Helpers shared by the GPU parity tests (comparison only, no attention math).

Every check records, per test, its worst error and its worst excess over the
bound (error minus bound: <= 0 passes); tests/conftest.py prints them at the
end of the run, so each parity test reports how close it came to its bound.
"""
import os

import numpy as np
import torch

ATOL_O = 1e-2  # max |O - O_ref| for unit-variance 16-bit inputs (see o_bound)
ATOL_L = 1e-3  # max |L - L_ref|
RTOL_GRAD = 2e-2  # ||dX - dX_ref||_2 / ||dX_ref||_2
# Where the 16-bit output's own rounding can exceed ATOL_O (half a unit in the last
# place above 1e-2: bf16 |O_ref| >= 4, fp16 |O_ref| >= 32), the bound is that half
# unit plus this much for the computation before the rounding. Such rows are
# dominated by one or two keys (a causal row's first keys); their computed value
# differs from O_ref only by the 16-bit rounding of the smaller weights (relative
# 2^-9 each) times the spread of V between the keys.
O_COMPUTE_MARGIN = 4e-3

SENTINEL = 12345.0

# test id -> {check: [worst error, worst excess over the bound]}
WORST = {}


def _record(check, err, excess):
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" (")[0]
    slot = WORST.setdefault(test, {}).setdefault(check, [-np.inf, -np.inf])
    slot[0] = max(slot[0], float(err))
    slot[1] = max(slot[1], float(excess))


def guarded(shape, dtype, guard=4096):
    """A CUDA tensor of `shape` sitting inside a sentinel-filled buffer, and a checker of the guards."""
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * guard,), SENTINEL, dtype=dtype, device="cuda")
    view = buf[guard:guard + n].view(*shape)

    def intact():
        return bool((buf[:guard] == SENTINEL).all()) and bool((buf[guard + n:] == SENTINEL).all())

    return view, intact


def f64(t):
    return t.detach().float().cpu().double().numpy()


def compare_rows(o, lse, o_ref, lse_ref, what=""):
    """Max errors over the rows present in the reference (NaN rows skipped). Fully
    masked rows (L_ref = -inf) must be exactly O = 0 and L = -inf."""
    o, lse = np.asarray(o), np.asarray(lse)
    have = ~np.isnan(lse_ref)
    empty = have & np.isneginf(lse_ref)
    live = have & np.isfinite(lse_ref)
    assert np.array_equal(np.isneginf(lse[empty]), np.ones(int(empty.sum()), bool)), f"{what}: -inf rows"
    err_l = float(np.abs(lse[live] - lse_ref[live]).max()) if live.any() else 0.0
    return err_l, empty, live


def ulp(x, dtype):
    """Spacing of the 16-bit output format at |x| (bf16: 8 significant bits, fp16: 11)."""
    bits = 8 if "bfloat16" in str(dtype) else 11
    ax = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -14)
    return 2.0 ** (np.floor(np.log2(ax)) - (bits - 1))


def o_bound(o_ref, dtype):
    """Per-element bound on |O - O_ref|: ATOL_O wherever the output format can hold
    O_ref that closely (half a unit in the last place below ATOL_O: bf16 |O_ref| < 4,
    fp16 |O_ref| < 32); above that, half a unit in the last place at |O_ref| (the
    correctly rounded exact value can already be that far away: bf16 values are 2^-5
    apart in [4, 8)) plus O_COMPUTE_MARGIN."""
    half = 0.5 * ulp(o_ref, dtype)
    return np.where(half < ATOL_O, ATOL_O, half + O_COMPUTE_MARGIN)


def check_o(o, o_ref, dtype, what="O"):
    """Assert |O - O_ref| <= o_bound element-wise and record the worst error and excess;
    also record the worst error of the computation alone (beyond half a unit in the
    last place) on the rows the output rounding decides."""
    o, o_ref = np.asarray(o, dtype=np.float64), np.asarray(o_ref, dtype=np.float64)
    if o_ref.size == 0:
        return
    err = np.abs(o - o_ref)
    excess = float((err - o_bound(o_ref, dtype)).max())
    _record(what, err.max(), excess)
    half = 0.5 * ulp(o_ref, dtype)
    wide = half >= ATOL_O
    if wide.any():
        _record(what + " rounding rows: error beyond half ulp", (err - half)[wide].max(),
                ((err - half)[wide] - O_COMPUTE_MARGIN).max())
    assert excess <= 0, (what, float(err.max()), excess)


def check_l(lse, l_ref, what="L"):
    """Assert max |L - L_ref| <= ATOL_L over finite reference rows, and record it."""
    lse, l_ref = np.asarray(lse, dtype=np.float64), np.asarray(l_ref, dtype=np.float64)
    live = np.isfinite(l_ref)
    if not live.any():
        return
    err = float(np.abs(lse[live] - l_ref[live]).max())
    _record(what, err, err - ATOL_L)
    assert err <= ATOL_L, (what, err)


def rel_l2(a, b):
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / (nb if nb > 0 else 1.0))


def check_rel(err, what="dX rel L2"):
    """Assert a relative L2 error <= RTOL_GRAD, and record it."""
    _record(what, err, err - RTOL_GRAD)
    assert err <= RTOL_GRAD, (what, err)


def check_grads(errs, what="dQ/dK/dV rel L2"):
    for name, e in zip(("dQ", "dK", "dV"), errs):
        _record(f"{name} rel L2", e, e - RTOL_GRAD)
    assert max(errs) <= RTOL_GRAD, (what, errs)
