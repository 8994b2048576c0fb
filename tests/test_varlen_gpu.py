"""Varlen forward parity (packed sequences addressed by cu_seqlens) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_36_b200 import binding as fb
from exact_tiled_attention_36_b200 import inputs
from tests.gpu_util import check_l, check_o, f64, guarded

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    fb.lib()
    yield
    assert fb.fa_get_last_device_error(None) == fb.FA_OK


def run_varlen(vi, causal, max_q=None, max_k=None):
    q, k, v = vi.q.cuda(), vi.k.cuda(), vi.v.cuda()
    cu_q, cu_k = vi.cu_seqlens_q.cuda(), vi.cu_seqlens_k.cuda()
    Tq, Hq, d = q.shape
    Tk, Hkv, _ = k.shape
    o, o_ok = guarded((Tq, Hq, d), q.dtype)
    lse, l_ok = guarded((Hq, Tq), torch.float32)
    dt = fb.FA_BF16 if q.dtype == torch.bfloat16 else fb.FA_FP16
    st = fb.fa_varlen_fwd(q.data_ptr(), k.data_ptr() if Tk else None, v.data_ptr() if Tk else None, o.data_ptr(),
                          lse.data_ptr(), cu_q.data_ptr(), cu_k.data_ptr(), len(vi.seqlens_q), Tq, Tk,
                          max_q if max_q is not None else vi.max_seqlen_q,
                          max_k if max_k is not None else vi.max_seqlen_k, Hq, Hkv, d, d ** -0.5, int(causal), dt, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    torch.cuda.synchronize()
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
    assert o_ok() and l_ok(), "write outside O / L"
    return f64(o), f64(lse)


def check_sequences(vi, o, lse, causal, rows_per_seq=None, seed=0):
    """Per sequence, the oracle on that sequence alone (sampled rows if asked)."""
    rng = np.random.default_rng(seed)
    scale = vi.q.shape[-1] ** -0.5
    for s, (Lq, Lk) in enumerate(zip(vi.seqlens_q, vi.seqlens_k)):
        if Lq == 0:
            continue
        a, ka = int(vi.cu_seqlens_q[s]), int(vi.cu_seqlens_k[s])
        if rows_per_seq is None:
            rows = list(range(Lq))
        else:
            rows = sorted(set(rng.choice(Lq, size=min(rows_per_seq, Lq), replace=False).tolist()) | {0, Lq - 1})
        o_ref, l_ref = oracle.attn_fwd(vi.q[None, a:a + Lq], vi.k[None, ka:ka + Lk], vi.v[None, ka:ka + Lk], scale,
                                       causal, rows=rows)
        og = o[a:a + Lq][rows]
        lg = lse[:, a:a + Lq][:, rows]
        orf = o_ref[0][rows]
        lrf = l_ref[0][:, rows]
        empty = np.isneginf(lrf)
        assert np.isneginf(lg[empty]).all()
        assert (og.transpose(1, 0, 2)[empty] == 0).all()
        live = ~empty
        if live.any():
            check_l(lg[live], lrf[live])
        check_o(og, orf, vi.q.dtype)


SMALL = [
    # lengths, Hq, Hkv, d, dtype, causal, key_pad_frac
    ([5, 0, 130, 257, 1, 64], 4, 2, 64, "fp16", False, 0.0),
    ([5, 0, 130, 257, 1, 64], 4, 2, 128, "bf16", True, 0.0),
    ([300, 129, 128, 0, 0, 77], 2, 2, 128, "fp16", False, 0.25),
    ([1000, 3, 513], 6, 3, 64, "bf16", True, 0.25),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"{len(c[0])}seq-h{c[1]}-{c[2]}-d{c[3]}-{c[4]}-c{int(c[5])}-p{c[6]}")
def test_varlen_small(case):
    lengths, Hq, Hkv, d, dt, causal, pad = case
    vi = inputs.make_varlen(inputs.VARLEN, lengths=lengths, Hq=Hq, Hkv=Hkv, d=d, dtype=dt, causal=causal,
                            key_pad_frac=pad, seed=31)
    o, lse = run_varlen(vi, causal)
    check_sequences(vi, o, lse, causal)


@pytest.mark.parametrize("cfg", [inputs.VARLEN, inputs.VARLEN_KEYPAD], ids=lambda c: c.name)
def test_varlen_workload_sampled_rows(cfg):
    vi = inputs.make_varlen(cfg)
    assert len(vi.seqlens_q) == 32
    o, lse = run_varlen(vi, cfg.causal)
    check_sequences(vi, o, lse, cfg.causal, rows_per_seq=6, seed=cfg.seed)


def test_varlen_matches_fixed_length_path():
    """Equal lengths through the varlen path give the fixed-length path's result."""
    B, N, H, d = 3, 200, 4, 128
    fi = inputs.make_fixed(inputs.TINY, B=B, Nq=N, Nk=N, Hq=H, Hkv=H, d=d, seed=5)
    q, k, v = (t.cuda() for t in (fi.q, fi.k, fi.v))
    o_f, l_f = fb.attention_fwd(q, k, v, d ** -0.5, causal=True)
    cu = torch.arange(0, (B + 1) * N, N, dtype=torch.int32, device="cuda")
    o_v, l_v = fb.attention_varlen_fwd(q.reshape(B * N, H, d), k.reshape(B * N, H, d), v.reshape(B * N, H, d), cu, cu,
                                       N, N, d ** -0.5, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o_v.reshape(B, N, H, d), o_f)
    assert torch.equal(l_v.reshape(H, B, N).permute(1, 0, 2), l_f)


@pytest.mark.parametrize("too_small", ["q", "k"])
def test_varlen_reports_a_sequence_past_max_seqlen(too_small):
    """A max_seqlen bound below a sequence's length cannot be caught before the launch
    (cu_seqlens live on the device): the call returns FA_OK, processes that sequence only
    up to the bound, and the next fa_get_last_device_error reports FA_ERR_INVALID_ARG
    (then the word is clear again). Sequences within the bound are still exact."""
    lengths = [100, 300, 50]
    vi = inputs.make_varlen(inputs.VARLEN, lengths=lengths, Hq=2, Hkv=2, d=128, dtype="bf16", seed=37)
    q, k, v = vi.q.cuda(), vi.k.cuda(), vi.v.cuda()
    cu_q, cu_k = vi.cu_seqlens_q.cuda(), vi.cu_seqlens_k.cuda()
    Tq, Hq, d = q.shape
    o, o_ok = guarded((Tq, Hq, d), q.dtype)
    lse, l_ok = guarded((Hq, Tq), torch.float32)
    max_q, max_k = (200, 300) if too_small == "q" else (300, 200)
    st = fb.fa_varlen_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), cu_q.data_ptr(),
                          cu_k.data_ptr(), len(lengths), Tq, k.shape[0], max_q, max_k, Hq, 2, d, d ** -0.5, 0,
                          fb.FA_BF16, 0)
    assert st == fb.FA_OK
    assert fb.fa_get_last_device_error(None) == fb.FA_ERR_INVALID_ARG
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
    assert o_ok() and l_ok(), "write outside O / L"
    # the sequences inside the bounds (0 and 2) are untouched by the clipping
    o64, l64 = f64(o), f64(lse)
    for s in (0, 2):
        a, L = int(vi.cu_seqlens_q[s]), lengths[s]
        o_ref, l_ref = oracle.attn_fwd(vi.q[None, a:a + L], vi.k[None, a:a + L], vi.v[None, a:a + L], d ** -0.5)
        check_o(o64[a:a + L], o_ref[0], q.dtype)
        check_l(l64[:, a:a + L], l_ref[0])
    # within the bounds the word stays clear
    run_varlen(vi, False)
