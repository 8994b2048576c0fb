"""Helpers shared by the GPU parity tests (comparison only, no attention math)."""
import numpy as np
import torch

ATOL_O = 1e-2  # max |O - O_ref| for unit-variance 16-bit inputs (see o_bound)
ATOL_L = 1e-3  # max |L - L_ref|
RTOL_GRAD = 2e-2  # ||dX - dX_ref||_2 / ||dX_ref||_2

SENTINEL = 12345.0


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
    """Per-element bound on |O - O_ref|: ATOL_O, or one unit in the last place of the
    16-bit output at |O_ref| where that is larger. A bf16 output cannot hold O_ref
    within 1e-2 once |O_ref| >= 4 (spacing 2^-5): even the correctly rounded exact
    value can be 0.0156 away."""
    return np.maximum(ATOL_O, ulp(o_ref, dtype))
