"""FP8 forward parity: fa_fwd_fp8 (through the C ABI) against the fp64 oracle on the
dequantised E4M3 inputs.

The kernel rounds the probabilities to E4M3 before the P V product, so the O bound is
derived from that rounding rather than taken from the 16-bit forward's 1e-2. With
P*_j = exp(s_j - max_j s_j) the probabilities relative to the row max (what the kernel
holds, up to a power of two <= 1 from its lazy reference max and V's block factors),
E4M3 round-to-nearest moves each weight by at most e_j = max(2^-4 P*_j, 2^-10 v_max /
v_j) (half a step: 3 mantissa bits for normal values, 2^-9 steps below 2^-6; v_j is the
V block factor of key j, v_max the largest one), masked keys stay exactly 0, and O is
normalised by the exact sum, so
    |O_c - O_ref,c| <= sum_j e_j |V_jc| / sum_j P*_j
plus the bf16 rounding of O (2^-8 |O_ref| covers half a unit in the last place) and
1e-3 for the fp32 arithmetic. L comes from the exact scores and keeps max|L - L_ref|
<= 1e-3."""
import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_36_b200 import binding as fb
from exact_tiled_attention_36_b200 import inputs
from tests.gpu_util import _record as record, check_l, f64, guarded

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    fb.lib()
    yield
    assert fb.fa_get_last_device_error(None) == fb.FA_OK


def run(fi, causal):
    q, k, v = fi.q.cuda(), fi.k.cuda(), fi.v.cuda()
    qs, ks, vs = fi.q_scale.cuda(), fi.k_scale.cuda(), fi.v_scale.cuda()
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    o, o_ok = guarded((B, Nq, Hq, d), torch.bfloat16)
    lse, l_ok = guarded((B, Hq, Nq), torch.float32)
    st = fb.fa_fwd_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), qs.data_ptr(), ks.data_ptr(), vs.data_ptr(),
                       o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Nq, Nk, d, d ** -0.5, int(causal), 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    torch.cuda.synchronize()
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
    assert o_ok() and l_ok(), "write outside O / L"
    return f64(o), f64(lse)


def o_bound_fp8(fi, causal, b, h, o_ref_bh):
    """Per-element bound on |O - O_ref| for (batch b, query head h), [Nq, d]."""
    Hq, Hkv = fi.q.shape[2], fi.k.shape[2]
    hk = h // (Hq // Hkv)
    d = fi.q.shape[3]
    qd = oracle.fp8_dequantise(fi.q.numpy(), fi.q_scale.numpy())
    kd = oracle.fp8_dequantise(fi.k.numpy(), fi.k_scale.numpy())
    vd = oracle.fp8_dequantise(fi.v.numpy(), fi.v_scale.numpy())
    P = oracle.attn_probs(qd, kd, d ** -0.5, b, h, causal)  # rows sum to 1 (0 if no key)
    pmax = P.max(axis=1, keepdims=True)
    Pstar = np.divide(P, pmax, out=np.zeros_like(P), where=pmax > 0)
    vs = fi.v_scale.numpy()[b, hk].astype(np.float64)
    ratio = vs.max() / vs[np.arange(P.shape[1]) // 128]
    e = np.where(P > 0, np.maximum(2.0 ** -4 * Pstar, 2.0 ** -10 * ratio[None, :]), 0.0)
    srow = Pstar.sum(axis=1, keepdims=True)
    E = np.divide(e, srow, out=np.zeros_like(e), where=srow > 0)
    return E @ np.abs(vd[b, :, hk, :]) + 2.0 ** -8 * np.abs(o_ref_bh) + 1e-3


def check(fi, o, lse, causal, heads=None):
    o_ref, l_ref = oracle.attn_fwd_fp8(fi.q.numpy(), fi.k.numpy(), fi.v.numpy(), fi.q_scale.numpy(),
                                       fi.k_scale.numpy(), fi.v_scale.numpy(), fi.cfg.scale, causal)
    empty = np.isneginf(l_ref)
    assert np.isneginf(lse[empty]).all()
    live = ~empty
    assert np.isfinite(lse[live]).all() and np.isfinite(o).all()
    check_l(lse[live], l_ref[live])
    B, Hq = o.shape[0], o.shape[2]
    worst = 0.0
    for b in range(B):
        for h in (range(Hq) if heads is None else heads):
            bound = o_bound_fp8(fi, causal, b, h, o_ref[b, :, h])
            err = np.abs(o[b, :, h] - o_ref[b, :, h])
            record("O (FP8 bound)", err.max(), (err - bound).max())
            assert (err <= bound).all(), (b, h, float((err - bound).max()))
            worst = max(worst, float(err.max()))
    return worst


CASES = [
    # B, Hq, Hkv, Nq, Nk, causal
    (2, 4, 2, 300, 300, False),
    (2, 4, 2, 300, 300, True),
    (1, 2, 1, 129, 1000, False),
    (1, 6, 2, 1000, 1000, True),
    (1, 2, 2, 1, 257, False),
    (1, 2, 2, 200, 77, True),  # Nq > Nk: the first rows see no key
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b{}-hq{}-hkv{}-nq{}-nk{}-c{}".format(*c[:5], int(c[5])))
def test_fp8_fwd_small(case):
    B, Hq, Hkv, Nq, Nk, causal = case
    fi = inputs.make_fp8(inputs.CAUSAL_GQA_FP8, B=B, Hq=Hq, Hkv=Hkv, Nq=Nq, Nk=Nk, causal=causal, seed=81)
    o, lse = run(fi, causal)
    check(fi, o, lse, causal)


def test_fp8_fwd_full_size_two_heads():
    """The benchmark workload at full size: every L, and every O row of two heads
    (first and last batch) against the oracle with the derived bound."""
    cfg = inputs.CAUSAL_GQA_FP8
    fi = inputs.make_fp8(cfg)
    o, lse = run(fi, True)
    for b, h in ((0, 0), (cfg.B - 1, cfg.Hq - 1)):
        sub = inputs.Fp8Inputs(cfg, fi.q[b:b + 1, :, h:h + 1], fi.k[b:b + 1, :, h // 4:h // 4 + 1],
                               fi.v[b:b + 1, :, h // 4:h // 4 + 1], fi.q_scale[b:b + 1, h:h + 1],
                               fi.k_scale[b:b + 1, h // 4:h // 4 + 1], fi.v_scale[b:b + 1, h // 4:h // 4 + 1])
        check(sub, o[b:b + 1, :, h:h + 1], lse[b:b + 1, h:h + 1], True)
    rows = [0, 1, 127, 128, 4095, 8190, 8191]
    for b in range(cfg.B):
        qd = oracle.fp8_dequantise(fi.q[b:b + 1].numpy(), fi.q_scale[b:b + 1].numpy())
        kd = oracle.fp8_dequantise(fi.k[b:b + 1].numpy(), fi.k_scale[b:b + 1].numpy())
        vd = oracle.fp8_dequantise(fi.v[b:b + 1].numpy(), fi.v_scale[b:b + 1].numpy())
        _, l_ref = oracle.attn_fwd(qd, kd, vd, cfg.scale, True, rows=rows)
        check_l(lse[b][:, rows], l_ref[0][:, rows])


def test_fp8_close_to_bf16_path_on_the_same_values():
    """The dequantised inputs through the bf16 forward give nearly the same O: the
    difference is the E4M3 rounding of P (and bf16 rounding of the inputs)."""
    fi = inputs.make_fp8(inputs.CAUSAL_GQA_FP8, B=1, Hq=4, Hkv=2, Nq=512, Nk=512, seed=82)
    o8, l8 = run(fi, True)
    deq = lambda c, s: torch.from_numpy(oracle.fp8_dequantise(c.numpy(), s.numpy())).to(torch.bfloat16).cuda()
    o16, l16 = fb.attention_fwd(deq(fi.q, fi.q_scale), deq(fi.k, fi.k_scale), deq(fi.v, fi.v_scale),
                                fi.cfg.scale, True)
    torch.cuda.synchronize()
    assert np.abs(f64(l16) - l8).max() <= 2e-2  # inputs rounded to bf16 in one path only
    assert np.sqrt(np.mean((f64(o16) - o8) ** 2)) <= 1e-2
