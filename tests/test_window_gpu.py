"""Sliding-window (local) attention: fa_fwd_window / fa_bwd_window through the C ABI
against the fp64 oracle with the same window."""
import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_36_b200 import binding as fb
from exact_tiled_attention_36_b200 import inputs
from tests.gpu_util import check_grads, check_l, check_o, check_rel, f64, guarded, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    fb.lib()
    yield
    assert fb.fa_get_last_device_error(None) == fb.FA_OK


def run(fi, window, backward=True):
    q, k, v = fi.q.cuda(), fi.k.cuda(), fi.v.cuda()
    B, Nq, Hq, d = q.shape
    _, Nk, Hkv, _ = k.shape
    dt = fb.FA_BF16 if q.dtype == torch.bfloat16 else fb.FA_FP16
    o, o_ok = guarded((B, Nq, Hq, d), q.dtype)
    lse, l_ok = guarded((B, Hq, Nq), torch.float32)
    wl, wr = window
    st = fb.fa_fwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Nq, Nk,
                          d, d ** -0.5, wl, wr, dt, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    grads = None
    if backward:
        do = fi.do.cuda()
        ws = torch.empty(fb.fa_bwd_workspace_size(B, Hq, Nq, d), dtype=torch.uint8, device="cuda")
        dq, dq_ok = guarded((B, Nq, Hq, d), q.dtype)
        dk, dk_ok = guarded((B, Nk, Hkv, d), q.dtype)
        dv, dv_ok = guarded((B, Nk, Hkv, d), q.dtype)
        st = fb.fa_bwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                              dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), B, Hq, Hkv, Nq, Nk, d,
                              d ** -0.5, wl, wr, dt, 0)
        assert st == fb.FA_OK, fb.fa_status_string(st)
    torch.cuda.synchronize()
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
    assert o_ok() and l_ok(), "write outside O / L"
    if backward:
        assert dq_ok() and dk_ok() and dv_ok(), "write outside dQ / dK / dV"
        grads = (f64(dq), f64(dk), f64(dv))
    return f64(o), f64(lse), grads


CASES = [
    # B, Nq, Nk, Hq, Hkv, d, window, dtype
    (1, 700, 700, 2, 1, 128, (128, 0), "bf16"),
    (2, 513, 513, 4, 2, 128, (200, 300), "fp16"),
    (1, 400, 650, 2, 2, 64, (64, 64), "bf16"),
    (1, 640, 300, 2, 1, 128, (-1, 100), "bf16"),
    (1, 333, 333, 2, 2, 64, (0, 0), "fp16"),
    (2, 300, 300, 4, 4, 128, (1000, -1), "bf16"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"b{c[0]}-{c[1]}x{c[2]}-h{c[3]}-{c[4]}-d{c[5]}-w{c[6][0]}_{c[6][1]}-{c[7]}")
def test_window_fwd_bwd(case):
    B, Nq, Nk, Hq, Hkv, d, window, dt = case
    fi = inputs.make_fixed(inputs.CAUSAL_GQA, B=B, Nq=Nq, Nk=Nk, Hq=Hq, Hkv=Hkv, d=d, dtype=dt, seed=73)
    o, lse, (dq, dk, dv) = run(fi, window)
    o_ref, l_ref = oracle.attn_fwd(fi.q, fi.k, fi.v, d ** -0.5, window=window)
    empty = np.isneginf(l_ref)
    assert np.isneginf(lse[empty]).all()
    assert (o.transpose(0, 2, 1, 3)[empty] == 0).all()
    live = ~empty
    check_l(lse[live], l_ref[live])
    check_o(o, o_ref, fi.q.dtype)
    rq, rk, rv = oracle.attn_bwd(fi.q, fi.k, fi.v, fi.do, d ** -0.5, window=window)
    errs = [rel_l2(g, r) for g, r in ((dq, rq), (dk, rk), (dv, rv))]
    check_grads(errs)


def test_causal_window_is_the_causal_path():
    """(-1, 0) through the window entry points gives fa_fwd / fa_bwd with causal = 1
    bit for bit."""
    B, N, Hq, Hkv, d = 1, 520, 4, 2, 128
    fi = inputs.make_fixed(inputs.CAUSAL_GQA, B=B, Nq=N, Nk=N, Hq=Hq, Hkv=Hkv, d=d, seed=79)
    o, lse, (dq, dk, dv) = run(fi, (-1, 0))
    q, k, v, do = (t.cuda() for t in (fi.q, fi.k, fi.v, fi.do))
    o2, l2 = fb.attention_fwd(q, k, v, d ** -0.5, True)
    dq2, dk2, dv2 = fb.attention_bwd(q, k, v, o2, l2, do, d ** -0.5, True)
    torch.cuda.synchronize()
    assert np.array_equal(o, f64(o2)) and np.array_equal(lse, f64(l2))
    assert np.array_equal(dk, f64(dk2)) and np.array_equal(dv, f64(dv2))
    assert rel_l2(dq, f64(dq2)) <= 1e-2  # dQ differs only in the order of its fp32 reductions


def test_window_long_sequence_sampled_rows():
    """A causal sliding window of 1024 keys over 8192 tokens: sampled rows of O and L,
    and the dV identity sum_j dV_j = sum_i dO_i (rows of P sum to 1)."""
    B, N, Hq, Hkv, d, window = 1, 8192, 4, 1, 128, (1024, 0)
    fi = inputs.make_fixed(inputs.CAUSAL_GQA, B=B, Nq=N, Nk=N, Hq=Hq, Hkv=Hkv, d=d, seed=83)
    o, lse, (dq, dk, dv) = run(fi, window)
    rows = [0, 1, 1023, 1024, 1025, 4000, 8191]
    o_ref, l_ref = oracle.attn_fwd(fi.q, fi.k, fi.v, d ** -0.5, window=window, rows=rows)
    check_o(o[:, rows], o_ref[:, rows], fi.q.dtype)
    check_l(lse[:, :, rows], l_ref[:, :, rows])
    ref = f64(fi.do).sum((0, 1))  # (Hq, d) -> the single KV head sums all query heads
    check_rel(rel_l2(dv.sum((0, 1))[0], ref.sum(0)), "sum of dV rel L2")


VARLEN_CASES = [
    # lengths, Hq, Hkv, d, window, dtype, key_pad_frac
    ([700, 1, 0, 300, 129], 4, 2, 128, (128, 0), "bf16", 0.0),
    ([513, 64, 900], 2, 2, 128, (100, 50), "fp16", 0.25),
    ([257, 1000, 5], 4, 1, 64, (-1, 40), "bf16", 0.0),
    # with global anchors (wl, wr, n_anchor): the first n_anchor keys of every sequence
    ([700, 1, 0, 300, 129], 4, 2, 128, (128, 0, 4), "bf16", 0.0),
    ([513, 64, 900], 2, 2, 128, (100, 50, 130), "fp16", 0.25),
    ([1100, 257, 640], 2, 1, 128, (200, -1, 300), "bf16", 0.0),
    ([257, 1000, 5], 4, 1, 64, (60, 0, 200), "bf16", 0.0),
]


@pytest.mark.parametrize("case", VARLEN_CASES,
                         ids=lambda c: f"{len(c[0])}seq-h{c[1]}-{c[2]}-d{c[3]}-w" + "_".join(map(str, c[4])))
def test_varlen_window(case):
    """fa_varlen_fwd_window and fa_varlen_bwd_window, or with anchors
    fa_varlen_fwd_window_anchor / fa_varlen_bwd_window_anchor: every sequence against
    the oracle with the window (and anchors) applied within that sequence."""
    lengths, Hq, Hkv, d, window, dt, pad = case
    vi = inputs.make_varlen(inputs.VARLEN, lengths=lengths, Hq=Hq, Hkv=Hkv, d=d, dtype=dt, key_pad_frac=pad,
                            seed=87, with_do=True)
    q, k, v, do = vi.q.cuda(), vi.k.cuda(), vi.v.cuda(), vi.do.cuda()
    cu_q, cu_k = vi.cu_seqlens_q.cuda(), vi.cu_seqlens_k.cuda()
    Tq, Tk, n = q.shape[0], k.shape[0], len(lengths)
    code = fb.FA_BF16 if q.dtype == torch.bfloat16 else fb.FA_FP16
    o, o_ok = guarded((Tq, Hq, d), q.dtype)
    lse, l_ok = guarded((Hq, Tq), torch.float32)
    wl, wr = window[:2]
    anchors = tuple(window[2:])  # (n_anchor,) or ()
    fwd = fb.fa_varlen_fwd_window_anchor if anchors else fb.fa_varlen_fwd_window
    st = fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), cu_q.data_ptr(),
             cu_k.data_ptr(), n, Tq, Tk, vi.max_seqlen_q, vi.max_seqlen_k, Hq, Hkv, d, d ** -0.5, wl, wr, *anchors,
             code, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    torch.cuda.synchronize()
    assert fb.fa_get_last_device_error(None) == fb.FA_OK and o_ok() and l_ok()
    o_ref, l_ref = oracle.varlen_fwd(vi.q, vi.k, vi.v, vi.cu_seqlens_q, vi.cu_seqlens_k, d ** -0.5, window=window)
    o64, l64 = f64(o), f64(lse)
    empty = np.isneginf(l_ref)
    assert np.isneginf(l64[empty]).all() and (o64.transpose(1, 0, 2)[empty] == 0).all()
    live = ~empty
    check_l(l64[live], l_ref[live])
    check_o(o64, o_ref, q.dtype)
    ws = torch.empty(fb.fa_varlen_bwd_workspace_size(n, Tq, vi.max_seqlen_q, Hq, d), dtype=torch.uint8, device="cuda")
    dq, dk, dv = torch.zeros_like(q), torch.zeros_like(k), torch.zeros_like(v)
    bwd = fb.fa_varlen_bwd_window_anchor if anchors else fb.fa_varlen_bwd_window
    st = bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(), dq.data_ptr(),
             dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), cu_q.data_ptr(), cu_k.data_ptr(), n, Tq, Tk,
             vi.max_seqlen_q, vi.max_seqlen_k, Hq, Hkv, d, d ** -0.5, wl, wr, *anchors, code, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    torch.cuda.synchronize()
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
    refs = [np.zeros(tuple(t.shape)) for t in (vi.q, vi.k, vi.v)]
    for s, (Lq, Lk) in enumerate(zip(vi.seqlens_q, vi.seqlens_k)):
        a, ka = int(vi.cu_seqlens_q[s]), int(vi.cu_seqlens_k[s])
        if Lq == 0 and Lk == 0:
            continue
        rq, rk, rv = oracle.attn_bwd(vi.q[None, a:a + Lq], vi.k[None, ka:ka + Lk], vi.v[None, ka:ka + Lk],
                                     vi.do[None, a:a + Lq], d ** -0.5, window=window)
        refs[0][a:a + Lq], refs[1][ka:ka + Lk], refs[2][ka:ka + Lk] = rq[0], rk[0], rv[0]
    errs = [rel_l2(f64(g), r) for g, r in zip((dq, dk, dv), refs)]
    check_grads(errs)


ANCHOR_CASES = [
    # B, Nq, Nk, Hq, Hkv, d, (wl, wr, n_anchor), dtype
    (1, 700, 700, 2, 1, 128, (128, 0, 4), "bf16"),      # causal window + 4 anchors (one partial tile)
    (2, 1100, 1100, 4, 2, 128, (200, 0, 130), "fp16"),  # anchors past the first tile, gap before the windows
    (1, 900, 900, 2, 2, 64, (64, 64, 300), "bf16"),     # two-sided window, anchors over 3 tiles
    (1, 640, 1000, 2, 1, 128, (100, -1, 50), "bf16"),   # unbounded right side: anchors seen by every row
    (1, 300, 300, 2, 1, 128, (0, 0, 1), "bf16"),        # each row: key 0 and its own key
]


@pytest.mark.parametrize("case", ANCHOR_CASES, ids=lambda c: f"b{c[0]}-{c[1]}x{c[2]}-d{c[5]}-w{c[6][0]}_{c[6][1]}_a{c[6][2]}")
def test_window_anchor_fwd_bwd(case):
    B, Nq, Nk, Hq, Hkv, d, window, dt = case
    fi = inputs.make_fixed(inputs.CAUSAL_GQA, B=B, Nq=Nq, Nk=Nk, Hq=Hq, Hkv=Hkv, d=d, dtype=dt, seed=89)
    q, k, v, do = (t.cuda() for t in (fi.q, fi.k, fi.v, fi.do))
    code = fb.FA_BF16 if q.dtype == torch.bfloat16 else fb.FA_FP16
    wl, wr, na = window
    o, o_ok = guarded((B, Nq, Hq, d), q.dtype)
    lse, l_ok = guarded((B, Hq, Nq), torch.float32)
    st = fb.fa_fwd_window_anchor(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv,
                                 Nq, Nk, d, d ** -0.5, wl, wr, na, code, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    ws = torch.empty(fb.fa_bwd_workspace_size(B, Hq, Nq, d), dtype=torch.uint8, device="cuda")
    dq, dq_ok = guarded((B, Nq, Hq, d), q.dtype)
    dk, dk_ok = guarded((B, Nk, Hkv, d), q.dtype)
    dv, dv_ok = guarded((B, Nk, Hkv, d), q.dtype)
    st = fb.fa_bwd_window_anchor(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                 do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), B, Hq, Hkv,
                                 Nq, Nk, d, d ** -0.5, wl, wr, na, code, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    torch.cuda.synchronize()
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
    assert o_ok() and l_ok() and dq_ok() and dk_ok() and dv_ok(), "write outside an output"
    o64, l64 = f64(o), f64(lse)
    o_ref, l_ref = oracle.attn_fwd(fi.q, fi.k, fi.v, d ** -0.5, window=window)
    empty = np.isneginf(l_ref)
    assert np.isneginf(l64[empty]).all()
    live = ~empty
    check_l(l64[live], l_ref[live])
    check_o(o64, o_ref, q.dtype)
    rq, rk, rv = oracle.attn_bwd(fi.q, fi.k, fi.v, fi.do, d ** -0.5, window=window)
    errs = [rel_l2(f64(g), r) for g, r in ((dq, rq), (dk, rk), (dv, rv))]
    check_grads(errs)


def test_window_anchor_zero_is_the_window_path():
    B, N, Hq, Hkv, d = 1, 400, 2, 1, 128
    fi = inputs.make_fixed(inputs.CAUSAL_GQA, B=B, Nq=N, Nk=N, Hq=Hq, Hkv=Hkv, d=d, seed=91)
    o, lse, _ = run(fi, (64, 0), backward=False)
    q, k, v = (t.cuda() for t in (fi.q, fi.k, fi.v))
    o2 = torch.empty_like(q)
    l2 = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
    st = fb.fa_fwd_window_anchor(q.data_ptr(), k.data_ptr(), v.data_ptr(), o2.data_ptr(), l2.data_ptr(), B, Hq, Hkv,
                                 N, N, d, d ** -0.5, 64, 0, 0, fb.FA_BF16, 0)
    assert st == fb.FA_OK
    torch.cuda.synchronize()
    assert np.array_equal(o, f64(o2)) and np.array_equal(lse, f64(l2))
