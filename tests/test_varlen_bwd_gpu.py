"""Varlen backward parity: fa_varlen_bwd (through the C ABI) against the fp64 oracle's
exact gradients of every sequence on its own."""
import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_36_b200 import binding as fb
from exact_tiled_attention_36_b200 import inputs
from tests.gpu_util import SENTINEL, check_grads, check_rel, f64, guarded, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    fb.lib()
    yield
    assert fb.fa_get_last_device_error(None) == fb.FA_OK


def run_varlen_fwd_bwd(vi, causal, extra_rows=0):
    """Forward then backward through the C ABI. `extra_rows` rows that belong to no
    sequence are appended to every packed buffer; the backward must leave them alone."""
    def pad(t):
        if extra_rows == 0:
            return t.cuda()
        tail = torch.full((extra_rows,) + tuple(t.shape[1:]), 0.5, dtype=t.dtype)
        return torch.cat([t, tail]).cuda()

    q, k, v, do = pad(vi.q), pad(vi.k), pad(vi.v), pad(vi.do)
    cu_q, cu_k = vi.cu_seqlens_q.cuda(), vi.cu_seqlens_k.cuda()
    Tq, Hq, d = q.shape
    Tk, Hkv, _ = k.shape
    n = len(vi.seqlens_q)
    dt = fb.FA_BF16 if q.dtype == torch.bfloat16 else fb.FA_FP16
    scale = d ** -0.5
    o = torch.zeros_like(q)
    lse = torch.zeros((Hq, Tq), dtype=torch.float32, device="cuda")
    st = fb.fa_varlen_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), cu_q.data_ptr(),
                          cu_k.data_ptr(), n, Tq, Tk, vi.max_seqlen_q, vi.max_seqlen_k, Hq, Hkv, d, scale,
                          int(causal), dt, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    ws = torch.full((fb.fa_varlen_bwd_workspace_size(n, Tq, vi.max_seqlen_q, Hq, d),), 255, dtype=torch.uint8,
                    device="cuda")
    dq, dq_ok = guarded((Tq, Hq, d), q.dtype)
    dk, dk_ok = guarded((Tk, Hkv, d), q.dtype)
    dv, dv_ok = guarded((Tk, Hkv, d), q.dtype)
    st = fb.fa_varlen_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                          dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), cu_q.data_ptr(),
                          cu_k.data_ptr(), n, Tq, Tk, vi.max_seqlen_q, vi.max_seqlen_k, Hq, Hkv, d, scale,
                          int(causal), dt, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    torch.cuda.synchronize()
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
    assert dq_ok() and dk_ok() and dv_ok(), "write outside dQ / dK / dV"
    return f64(dq), f64(dk), f64(dv)


def check_sequences(vi, dq, dk, dv, causal):
    """Every sequence against the oracle on that sequence alone: relative L2 error of
    dQ, dK and dV over all sequences' rows, and per sequence wherever its reference
    gradient is not negligible (a gradient that cancels to zero in exact arithmetic,
    like dK of a sequence with a single key, is only zero up to rounding here)."""
    scale = vi.q.shape[-1] ** -0.5
    refs = [np.zeros_like(dq), np.zeros_like(dk), np.zeros_like(dv)]
    spans = []
    for s, (Lq, Lk) in enumerate(zip(vi.seqlens_q, vi.seqlens_k)):
        a, ka = int(vi.cu_seqlens_q[s]), int(vi.cu_seqlens_k[s])
        if Lq == 0 and Lk == 0:
            continue
        rq, rk, rv = oracle.attn_bwd(vi.q[None, a:a + Lq], vi.k[None, ka:ka + Lk], vi.v[None, ka:ka + Lk],
                                     vi.do[None, a:a + Lq], scale, causal)
        refs[0][a:a + Lq], refs[1][ka:ka + Lk], refs[2][ka:ka + Lk] = rq[0], rk[0], rv[0]
        spans.append(((a, a + Lq), (ka, ka + Lk)))
    n_q, n_k = sum(vi.seqlens_q), sum(vi.seqlens_k)
    got = (dq[:n_q], dk[:n_k], dv[:n_k])
    ref = (refs[0][:n_q], refs[1][:n_k], refs[2][:n_k])
    errs = [rel_l2(g, r) for g, r in zip(got, ref)]
    check_grads(errs)
    for (qa, qb), (ka, kb) in spans:
        for g, r, (x, y) in ((dq, refs[0], (qa, qb)), (dk, refs[1], (ka, kb)), (dv, refs[2], (ka, kb))):
            nr = np.linalg.norm(r[x:y])
            if nr > 1e-3 * np.linalg.norm(r):
                check_rel(rel_l2(g[x:y], r[x:y]), "per-sequence rel L2")


CASES = [
    # lengths, Hq, Hkv, dtype, causal, key_pad_frac, d
    ([5, 0, 130, 257, 1, 64], 4, 2, "bf16", False, 0.0, 128),
    ([5, 0, 130, 257, 1, 64], 4, 2, "bf16", True, 0.0, 128),
    ([300, 129, 128, 0, 0, 77], 2, 2, "fp16", False, 0.25, 128),
    ([1000, 3, 513], 6, 3, "bf16", True, 0.25, 128),
    ([700, 411, 129, 256], 8, 2, "fp16", True, 0.0, 128),
    ([5, 0, 130, 257, 1, 64], 4, 2, "bf16", True, 0.0, 64),
    ([300, 129, 128, 0, 0, 77], 2, 2, "fp16", False, 0.25, 64),
    ([1000, 3, 513], 6, 3, "bf16", True, 0.25, 64),
    ([700, 411, 129, 256], 8, 2, "bf16", False, 0.0, 64),
]


@pytest.mark.parametrize("case", CASES,
                         ids=lambda c: f"{len(c[0])}seq-h{c[1]}-{c[2]}-{c[3]}-c{int(c[4])}-p{c[5]}-d{c[6]}")
def test_varlen_bwd_small(case):
    lengths, Hq, Hkv, dt, causal, pad, d = case
    vi = inputs.make_varlen(inputs.VARLEN, lengths=lengths, Hq=Hq, Hkv=Hkv, d=d, dtype=dt, causal=causal,
                            key_pad_frac=pad, seed=37, with_do=True)
    dq, dk, dv = run_varlen_fwd_bwd(vi, causal)
    check_sequences(vi, dq, dk, dv, causal)


@pytest.mark.parametrize("d", [64, 128])
def test_varlen_bwd_leaves_rows_outside_sequences(d):
    """Rows past the last sequence (total > cu[-1]) keep what they held."""
    vi = inputs.make_varlen(inputs.VARLEN, lengths=[200, 77], Hq=4, Hkv=2, d=d, dtype="bf16", seed=41,
                            with_do=True)
    extra = 96
    dq, dk, dv = run_varlen_fwd_bwd(vi, True, extra_rows=extra)
    n_q, n_k = sum(vi.seqlens_q), sum(vi.seqlens_k)
    sentinel = float(torch.tensor(SENTINEL, dtype=torch.bfloat16))  # as the bf16 buffers hold it
    for t, n in ((dq, n_q), (dk, n_k), (dv, n_k)):
        assert (t[n:] == sentinel).all()
    check_sequences(vi, dq[:n_q], dk[:n_k], dv[:n_k], True)


@pytest.mark.parametrize("d", [64, 128])
def test_varlen_bwd_matches_fixed_length_path(d):
    """Equal lengths through the varlen path give the fixed-length path's gradients:
    dK and dV bit for bit (same products in the same order), dQ up to the order of
    its fp32 reductions."""
    B, N, Hq, Hkv = 3, 200, 4, 2
    fi = inputs.make_fixed(inputs.CAUSAL_GQA, B=B, Nq=N, Nk=N, Hq=Hq, Hkv=Hkv, d=d, seed=43)
    q, k, v, do = (t.cuda() for t in (fi.q, fi.k, fi.v, fi.do))
    o, lse = fb.attention_fwd(q, k, v, d ** -0.5, causal=True)
    dq_f, dk_f, dv_f = fb.attention_bwd(q, k, v, o, lse, do, d ** -0.5, causal=True)
    cu = torch.arange(0, (B + 1) * N, N, dtype=torch.int32, device="cuda")
    flat = lambda t: t.reshape(B * N, t.shape[2], d)
    o_v, l_v = fb.attention_varlen_fwd(flat(q), flat(k), flat(v), cu, cu, N, N, d ** -0.5, causal=True)
    dq_v, dk_v, dv_v = fb.attention_varlen_bwd(flat(q), flat(k), flat(v), o_v, l_v, flat(do), cu, cu, N, N,
                                               d ** -0.5, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(dk_v.reshape(B, N, Hkv, d), dk_f)
    assert torch.equal(dv_v.reshape(B, N, Hkv, d), dv_f)
    assert rel_l2(f64(dq_v.reshape(B, N, Hq, d)), f64(dq_f)) <= 1e-2


def test_varlen_bwd_reports_a_sequence_past_max_seqlen():
    """The backward with a max_seqlen_q below a sequence's length returns FA_OK and
    reports FA_ERR_INVALID_ARG through the device error word; nothing is written
    outside the gradient buffers."""
    lengths = [64, 260, 10]
    vi = inputs.make_varlen(inputs.VARLEN, lengths=lengths, Hq=2, Hkv=1, d=128, dtype="bf16", seed=38,
                            with_do=True)
    q, k, v, do = vi.q.cuda(), vi.k.cuda(), vi.v.cuda(), vi.do.cuda()
    cu_q, cu_k = vi.cu_seqlens_q.cuda(), vi.cu_seqlens_k.cuda()
    Tq, Hq, d = q.shape
    Tk, Hkv, _ = k.shape
    n, scale = len(lengths), d ** -0.5
    o = torch.zeros_like(q)
    lse = torch.zeros((Hq, Tq), dtype=torch.float32, device="cuda")
    assert fb.fa_varlen_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), cu_q.data_ptr(),
                            cu_k.data_ptr(), n, Tq, Tk, 260, 260, Hq, Hkv, d, scale, 1, fb.FA_BF16, 0) == fb.FA_OK
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
    bound = 128
    ws = torch.full((fb.fa_varlen_bwd_workspace_size(n, Tq, bound, Hq, d),), 255, dtype=torch.uint8, device="cuda")
    dq, dq_ok = guarded((Tq, Hq, d), q.dtype)
    dk, dk_ok = guarded((Tk, Hkv, d), q.dtype)
    dv, dv_ok = guarded((Tk, Hkv, d), q.dtype)
    st = fb.fa_varlen_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                          dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), cu_q.data_ptr(),
                          cu_k.data_ptr(), n, Tq, Tk, bound, bound, Hq, Hkv, d, scale, 1, fb.FA_BF16, 0)
    assert st == fb.FA_OK
    assert fb.fa_get_last_device_error(None) == fb.FA_ERR_INVALID_ARG
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
    assert dq_ok() and dk_ok() and dv_ok(), "write outside dQ / dK / dV"


def test_varlen_bwd_workload_sampled_rows():
    """The varlen workload at full size (32 sequences of U[64, 4096] tokens, Hq = Hkv = 32,
    d = 128, fp16, no mask), in the configuration the benchmark times. Each sequence is an
    attention problem of its own, so the oracle takes it alone: for the longest, the shortest
    and a middle sequence, in three heads each, dQ, dK and dV of sampled rows element-wise.
    Over every sequence and head, the two identities: the keys' dK sum to zero and their dV
    to the sum of dO over the sequence's queries."""
    cfg = inputs.VARLEN
    vi = inputs.make_varlen(cfg, with_do=True)
    dq, dk, dv = run_varlen_fwd_bwd(vi, cfg.causal)
    scale = cfg.d ** -0.5
    lens = list(vi.seqlens_q)
    order = sorted(range(len(lens)), key=lambda s: lens[s])
    for s in (order[-1], order[0], order[len(order) // 2]):
        a, ka = int(vi.cu_seqlens_q[s]), int(vi.cu_seqlens_k[s])
        L, Lk = vi.seqlens_q[s], vi.seqlens_k[s]
        q1, k1, v1, do1 = (oracle._f64(t) for t in (vi.q[None, a:a + L], vi.k[None, ka:ka + Lk],
                                                      vi.v[None, ka:ka + Lk], vi.do[None, a:a + L]))
        qrows = sorted({0, L - 1} | set(range(0, L, max(1, L // 24))))
        krows = sorted({0, Lk - 1, Lk // 2, min(127, Lk - 1), min(128, Lk - 1)})
        for h in (0, 13, cfg.Hq - 1):
            sq, sk, sv = oracle.attn_bwd_sampled(q1, k1, v1, do1, scale, 0, h, qrows, krows, cfg.causal)
            gq = dq[a + np.asarray(qrows)][:, h:h + 1]
            for t in range(len(qrows)):
                check_rel(rel_l2(gq[t], sq[t]), "varlen dQ per sampled row rel L2")
            for name, got, ref in (("dk", dk[ka + np.asarray(krows), h], sk), ("dv", dv[ka + np.asarray(krows), h], sv)):
                for t in range(len(krows)):
                    check_rel(rel_l2(got[t], ref[t]), f"varlen {name} per sampled row rel L2")
    do = f64(vi.do)
    for s, (L, Lk) in enumerate(zip(vi.seqlens_q, vi.seqlens_k)):
        a, ka = int(vi.cu_seqlens_q[s]), int(vi.cu_seqlens_k[s])
        sdk = dk[ka:ka + Lk].sum(0)
        assert np.abs(sdk).max() <= 2e-2 * np.abs(dk[ka:ka + Lk]).sum(0).max() + 1e-3
        check_rel(rel_l2(dv[ka:ka + Lk].sum(0), do[a:a + L].sum(0)), "varlen sum of dV over keys rel L2")

