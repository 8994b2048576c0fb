"""fa_fwd_qk_rmsnorm (Q/K RMS normalisation fused in front of attention) against the
oracle: RMS-normalise Q and K in fp64, round once to the input type, then the plain
attention definition. The inputs keep their raw values: the call does not modify q or k."""
import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_36_b200 import binding as fb
from exact_tiled_attention_36_b200 import inputs
from tests.gpu_util import check_l, check_o, f64, guarded

pytestmark = pytest.mark.gpu

EPS = 1e-6


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    fb.lib()
    yield
    assert fb.fa_get_last_device_error(None) == fb.FA_OK


def scaled_rows(t, seed):
    """Rows of very different magnitudes (so the normalisation matters), from the
    seeded draw: row (token, head) scaled by a seeded factor in [0.05, 20]."""
    g = torch.Generator().manual_seed(seed)
    f = torch.exp(torch.empty(t.shape[:-1] + (1,)).uniform_(np.log(0.05), np.log(20.0), generator=g))
    return (t.float() * f).to(t.dtype)


def run_fused(q, k, v, causal, eps=EPS):
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o, o_ok = guarded((B, Nq, Hq, d), q.dtype)
    lse, l_ok = guarded((B, Hq, Nq), torch.float32)
    code = fb.FA_BF16 if q.dtype == torch.bfloat16 else fb.FA_FP16
    ws = torch.empty(fb.fa_fwd_qk_rmsnorm_workspace_size(B, Nk, Hkv, d), dtype=torch.uint8, device="cuda")
    st = fb.fa_fwd_qk_rmsnorm(qc.data_ptr(), kc.data_ptr(), vc.data_ptr(), o.data_ptr(), lse.data_ptr(),
                              ws.data_ptr(), B, Hq, Hkv, Nq, Nk, d, d ** -0.5, int(causal), eps, code, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    torch.cuda.synchronize()
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
    assert o_ok() and l_ok(), "write outside O / L"
    return f64(o), f64(lse)


def check(q, k, v, o, lse, causal, rows=None):
    d = q.shape[-1]
    qn = oracle.rms_normalise(q, EPS, q.dtype)
    kn = oracle.rms_normalise(k, EPS, k.dtype)
    o_ref, l_ref = oracle.attn_fwd(qn, kn, v, d ** -0.5, causal, rows=rows)
    sel = slice(None) if rows is None else rows
    check_o(o[:, sel], o_ref[:, sel], q.dtype)
    check_l(lse[:, :, sel], l_ref[:, :, sel])


@pytest.mark.parametrize("B,N,Hq,Hkv,d,causal,dt", [
    (2, 257, 5, 5, 128, False, "bf16"),
    (1, 300, 4, 2, 64, True, "fp16"),
    (1, 640, 2, 1, 128, True, "bf16"),
])
def test_fused_qk_rmsnorm_small(B, N, Hq, Hkv, d, causal, dt):
    fi = inputs.make_fixed(inputs.VIT_RMSNORM, B=B, Nq=N, Nk=N, Hq=Hq, Hkv=Hkv, d=d, dtype=dt, causal=causal,
                           rmsnorm=False, seed=67)
    q, k = scaled_rows(fi.q, 1), scaled_rows(fi.k, 2)
    o, lse = run_fused(q, k, fi.v, causal)
    check(q, k, fi.v, o, lse, causal)


def test_fused_qk_rmsnorm_vit_workload_sampled_rows():
    """The ViT workload's shape (B=8, H=25, N=1025, d=128) with raw Q and K."""
    cfg = inputs.VIT_RMSNORM
    fi = inputs.make_fixed(cfg, rmsnorm=False)
    q, k = scaled_rows(fi.q, 3), scaled_rows(fi.k, 4)
    o, lse = run_fused(q, k, fi.v, cfg.causal)
    check(q, k, fi.v, o, lse, cfg.causal, rows=[0, 1, 511, 1023, 1024])


def test_fused_matches_prenormalised_inputs():
    """Up to the fp32-vs-fp64 rounding of the normalisation, the fused path gives
    fa_fwd on inputs normalised beforehand."""
    fi = inputs.make_fixed(inputs.VIT_RMSNORM, B=1, Nq=200, Nk=200, Hq=3, Hkv=3, rmsnorm=False, seed=71)
    q, k = scaled_rows(fi.q, 5), scaled_rows(fi.k, 6)
    o, lse = run_fused(q, k, fi.v, False)
    qn = oracle.rms_normalise(q, EPS, q.dtype).cuda()
    kn = oracle.rms_normalise(k, EPS, k.dtype).cuda()
    o2, l2 = fb.attention_fwd(qn, kn, fi.v.cuda(), 128 ** -0.5, False)
    torch.cuda.synchronize()
    assert np.abs(o - f64(o2)).max() <= 2e-2
    assert np.abs(lse - f64(l2)).max() <= 2e-3
