"""Forward on strided views (packed QKV, BHSD output) through the C ABI: the same
result, bit for bit, as the contiguous path on copies of the same values, and
within the oracle's tolerance."""
import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_36_b200 import binding as fb
from exact_tiled_attention_36_b200 import inputs
from tests.gpu_util import check_l, check_o, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    fb.lib()
    yield
    assert fb.fa_get_last_device_error(None) == fb.FA_OK


def el_strides(t, batch=True):
    st = t.stride()
    return (st[0], st[1], st[2]) if batch else (st[0], st[1])


@pytest.mark.parametrize("B,N,H,d,causal,dt", [
    (2, 300, 4, 64, False, "bf16"),
    (1, 513, 2, 128, True, "fp16"),
    (3, 129, 3, 128, False, "bf16"),
])
def test_packed_qkv_matches_contiguous(B, N, H, d, causal, dt):
    fi = inputs.make_fixed(inputs.TINY, B=B, Nq=N, Nk=N, Hq=H, Hkv=H, d=d, dtype=dt, seed=53, with_do=False)
    qkv = torch.stack([fi.q, fi.k, fi.v], dim=2).cuda()  # (B, S, 3, H, d)
    q, k, v = qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2]
    o_bhsd = torch.full((B, H, N, d), 7.0, dtype=q.dtype, device="cuda")
    o = o_bhsd.permute(0, 2, 1, 3)  # a (B, S, H, d) view of a (B, H, S, d) buffer
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    code = fb.FA_BF16 if dt == "bf16" else fb.FA_FP16
    st = fb.fa_fwd_strided(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), el_strides(q),
                           el_strides(k), el_strides(v), el_strides(o), B, H, H, N, N, d, d ** -0.5, int(causal),
                           code, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    o_ref, l_ref = fb.attention_fwd(q.contiguous(), k.contiguous(), v.contiguous(), d ** -0.5, causal)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref)
    assert torch.equal(lse, l_ref)
    rows = [0, 1, N // 2, N - 1]
    o_or, l_or = oracle.attn_fwd(fi.q, fi.k, fi.v, d ** -0.5, causal, rows=rows)
    got = f64(o)[:, rows]
    check_o(got, o_or[:, rows], q.dtype)
    check_l(f64(lse)[:, :, rows], l_or[:, :, rows])


def test_packed_kv_with_grouped_heads():
    """q contiguous, k and v views of a packed (B, S, 2, Hkv, d) buffer, Hq = 4 Hkv."""
    B, N, Hq, Hkv, d = 2, 260, 8, 2, 128
    fi = inputs.make_fixed(inputs.CAUSAL_GQA, B=B, Nq=N, Nk=N, Hq=Hq, Hkv=Hkv, d=d, seed=59, with_do=False)
    q = fi.q.cuda()
    kv = torch.stack([fi.k, fi.v], dim=2).cuda()
    k, v = kv[:, :, 0], kv[:, :, 1]
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
    st = fb.fa_fwd_strided(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), el_strides(q),
                           el_strides(k), el_strides(v), el_strides(o), B, Hq, Hkv, N, N, d, d ** -0.5, 1,
                           fb.FA_BF16, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    o_ref, l_ref = fb.attention_fwd(q, k.contiguous(), v.contiguous(), d ** -0.5, True)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)


def test_varlen_packed_qkv_matches_contiguous():
    vi = inputs.make_varlen(inputs.VARLEN, lengths=[300, 0, 77, 513], Hq=4, Hkv=4, d=128, dtype="fp16", seed=61)
    qkv = torch.stack([vi.q, vi.k, vi.v], dim=1).cuda()  # (total, 3, H, d)
    q, k, v = qkv[:, 0], qkv[:, 1], qkv[:, 2]
    cu = vi.cu_seqlens_q.cuda()
    T, H, d = q.shape
    o = torch.empty((T, H, d), dtype=q.dtype, device="cuda")
    lse = torch.empty((H, T), dtype=torch.float32, device="cuda")
    st = fb.fa_varlen_fwd_strided(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                  el_strides(q, False), el_strides(k, False), el_strides(v, False),
                                  el_strides(o, False), cu.data_ptr(), cu.data_ptr(), 4, T, T, vi.max_seqlen_q,
                                  vi.max_seqlen_k, H, H, d, d ** -0.5, 1, fb.FA_FP16, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    o_ref, l_ref = fb.attention_varlen_fwd(q.contiguous(), k.contiguous(), v.contiguous(), cu, cu, vi.max_seqlen_q,
                                           vi.max_seqlen_k, d ** -0.5, True)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)


def rel_l2(a, b):
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


@pytest.mark.parametrize("B,N,H,d,causal,dt", [
    (2, 300, 4, 64, False, "bf16"),
    (1, 513, 2, 128, True, "fp16"),
    (2, 257, 4, 128, False, "bf16"),
])
def test_packed_qkv_backward(B, N, H, d, causal, dt):
    """fa_bwd_strided on the packed layout: q, k, v views of qkv (B, S, 3, H, d), O in a
    (B, H, S, d) buffer, dO a (B, H, S, d) view, and the gradients written into one
    dqkv (B, S, 3, H, d) buffer. dK and dV equal the contiguous path's bit for bit,
    dQ up to the order of its fp32 reductions, and all three the oracle's."""
    fi = inputs.make_fixed(inputs.TINY, B=B, Nq=N, Nk=N, Hq=H, Hkv=H, d=d, dtype=dt, seed=57, with_do=True)
    qkv = torch.stack([fi.q, fi.k, fi.v], dim=2).cuda()
    q, k, v = qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2]
    o_bhsd = torch.empty((B, H, N, d), dtype=q.dtype, device="cuda")
    o = o_bhsd.permute(0, 2, 1, 3)
    do = fi.do.cuda().permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)  # (B, S, H, d) view of BHSD
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    code = fb.FA_BF16 if dt == "bf16" else fb.FA_FP16
    st = fb.fa_fwd_strided(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), el_strides(q),
                           el_strides(k), el_strides(v), el_strides(o), B, H, H, N, N, d, d ** -0.5, int(causal),
                           code, 0)
    assert st == fb.FA_OK
    dqkv = torch.full_like(qkv, 3.0)
    dq, dk, dv = dqkv[:, :, 0], dqkv[:, :, 1], dqkv[:, :, 2]
    ws = torch.empty(fb.fa_bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
    st = fb.fa_bwd_strided(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                           dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), el_strides(q), el_strides(k),
                           el_strides(v), el_strides(o), el_strides(do), el_strides(dq), el_strides(dk),
                           el_strides(dv), B, H, H, N, N, d, d ** -0.5, int(causal), code, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    torch.cuda.synchronize()
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
    dq_c, dk_c, dv_c = fb.attention_bwd(q.contiguous(), k.contiguous(), v.contiguous(), o.contiguous(), lse,
                                        do.contiguous(), d ** -0.5, causal)
    torch.cuda.synchronize()
    assert torch.equal(dk, dk_c) and torch.equal(dv, dv_c)
    assert rel_l2(f64(dq), f64(dq_c)) <= 1e-2
    rq, rk, rv = oracle.attn_bwd(fi.q, fi.k, fi.v, fi.do, d ** -0.5, causal)
    errs = [rel_l2(f64(g), r) for g, r in ((dq, rq), (dk, rk), (dv, rv))]
    assert max(errs) <= 2e-2, errs


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_packed_qkv_backward(causal):
    """fa_varlen_bwd_strided on a packed (total, 3, H, d) QKV buffer: O in an (H, total,
    d) buffer, dO an (H, total, d) view, the gradients into one dqkv (total, 3, H, d).
    dK and dV equal the contiguous varlen backward's bit for bit, dQ up to the order of
    its fp32 reductions, and all three the oracle's, sequence by sequence."""
    lengths = [300, 0, 77, 513, 129]
    vi = inputs.make_varlen(inputs.VARLEN, lengths=lengths, Hq=4, Hkv=4, d=128, dtype="bf16", seed=63, with_do=True)
    qkv = torch.stack([vi.q, vi.k, vi.v], dim=1).cuda()  # (total, 3, H, d)
    q, k, v = qkv[:, 0], qkv[:, 1], qkv[:, 2]
    cu = vi.cu_seqlens_q.cuda()
    T, H, d = q.shape
    n = len(lengths)
    o = torch.empty((H, T, d), dtype=q.dtype, device="cuda").permute(1, 0, 2)
    do = vi.do.cuda().permute(1, 0, 2).contiguous().permute(1, 0, 2)
    lse = torch.empty((H, T), dtype=torch.float32, device="cuda")
    st = fb.fa_varlen_fwd_strided(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                  el_strides(q, False), el_strides(k, False), el_strides(v, False),
                                  el_strides(o, False), cu.data_ptr(), cu.data_ptr(), n, T, T, vi.max_seqlen_q,
                                  vi.max_seqlen_k, H, H, d, d ** -0.5, int(causal), fb.FA_BF16, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    dqkv = torch.full_like(qkv, 3.0)
    dq, dk, dv = dqkv[:, 0], dqkv[:, 1], dqkv[:, 2]
    ws = torch.empty(fb.fa_varlen_bwd_workspace_size(n, T, vi.max_seqlen_q, H, d), dtype=torch.uint8, device="cuda")
    st = fb.fa_varlen_bwd_strided(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                  do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(),
                                  *[el_strides(t, False) for t in (q, k, v, o, do, dq, dk, dv)], cu.data_ptr(),
                                  cu.data_ptr(), n, T, T, vi.max_seqlen_q, vi.max_seqlen_k, H, H, d, d ** -0.5,
                                  int(causal), fb.FA_BF16, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    torch.cuda.synchronize()
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
    dq_c, dk_c, dv_c = fb.attention_varlen_bwd(q.contiguous(), k.contiguous(), v.contiguous(), o.contiguous(), lse,
                                               do.contiguous(), cu, cu, vi.max_seqlen_q, vi.max_seqlen_k,
                                               d ** -0.5, causal)
    torch.cuda.synchronize()
    assert torch.equal(dk, dk_c) and torch.equal(dv, dv_c)
    assert rel_l2(f64(dq), f64(dq_c)) <= 1e-2
    refs = [np.zeros(tuple(t.shape)) for t in (vi.q, vi.k, vi.v)]
    for s, L in enumerate(lengths):
        a = int(vi.cu_seqlens_q[s])
        if L == 0:
            continue
        rq, rk, rv = oracle.attn_bwd(vi.q[None, a:a + L], vi.k[None, a:a + L], vi.v[None, a:a + L],
                                     vi.do[None, a:a + L], d ** -0.5, causal)
        refs[0][a:a + L], refs[1][a:a + L], refs[2][a:a + L] = rq[0], rk[0], rv[0]
    errs = [rel_l2(f64(g), r) for g, r in zip((dq, dk, dv), refs)]
    assert max(errs) <= 2e-2, errs
