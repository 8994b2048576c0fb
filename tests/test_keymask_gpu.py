"""General key-padding masks (fa_pack_key_mask, fa_fwd_keymask, fa_bwd_keymask) through
the C ABI against the fp64 oracle with the same boolean key mask."""
import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_36_b200 import binding as fb
from exact_tiled_attention_36_b200 import inputs
from tests.gpu_util import check_grads, check_l, check_o, f64, guarded, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    fb.lib()
    yield
    assert fb.fa_get_last_device_error(None) == fb.FA_OK


def make_keep(kind, B, Nk, rng):
    keep = np.ones((B, Nk), dtype=np.uint8)
    if kind == "left":  # left padding: the first keys of each sequence are padding
        for b in range(B):
            keep[b, :rng.integers(0, Nk // 2)] = 0
    elif kind == "random":  # about a quarter of the keys anywhere
        keep = (rng.random((B, Nk)) >= 0.25).astype(np.uint8)
    elif kind == "blocks":  # whole key tiles masked, one sequence fully masked
        keep[:, 128:256] = 0
        keep[-1, :] = 0
    return keep


CASES = [
    # B, Nq, Nk, Hq, Hkv, d, causal, kind, dtype
    (2, 300, 300, 4, 2, 128, False, "left", "bf16"),
    (2, 513, 513, 2, 1, 128, True, "random", "fp16"),
    (3, 200, 700, 2, 2, 64, False, "random", "bf16"),
    (3, 400, 400, 4, 2, 128, True, "blocks", "bf16"),
    (1, 129, 129, 2, 2, 64, True, "left", "fp16"),
    (2, 160, 288, 2, 1, 128, False, "random", "bf16"),  # last key tile of 32 keys (the narrow tail)
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"b{c[0]}-{c[1]}x{c[2]}-d{c[5]}-c{int(c[6])}-{c[7]}")
def test_keymask_fwd_bwd(case):
    B, Nq, Nk, Hq, Hkv, d, causal, kind, dt = case
    fi = inputs.make_fixed(inputs.CAUSAL_GQA, B=B, Nq=Nq, Nk=Nk, Hq=Hq, Hkv=Hkv, d=d, dtype=dt, seed=101)
    keep = make_keep(kind, B, Nk, np.random.default_rng(7))
    q, k, v, do = (t.cuda() for t in (fi.q, fi.k, fi.v, fi.do))
    keep_d = torch.from_numpy(keep).cuda()
    words = (Nk + 31) // 32
    bits = torch.full((B, words), 0x7, dtype=torch.int32, device="cuda")
    assert fb.fa_pack_key_mask(keep_d.data_ptr(), bits.data_ptr(), B, Nk, 0) == fb.FA_OK
    code = fb.FA_BF16 if q.dtype == torch.bfloat16 else fb.FA_FP16
    scale = d ** -0.5
    o, o_ok = guarded((B, Nq, Hq, d), q.dtype)
    lse, l_ok = guarded((B, Hq, Nq), torch.float32)
    st = fb.fa_fwd_keymask(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), bits.data_ptr(),
                           B, Hq, Hkv, Nq, Nk, d, scale, int(causal), code, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    ws = torch.empty(fb.fa_bwd_workspace_size(B, Hq, Nq, d), dtype=torch.uint8, device="cuda")
    dq, dq_ok = guarded((B, Nq, Hq, d), q.dtype)
    dk, dk_ok = guarded((B, Nk, Hkv, d), q.dtype)
    dv, dv_ok = guarded((B, Nk, Hkv, d), q.dtype)
    st = fb.fa_bwd_keymask(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                           dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), bits.data_ptr(), B, Hq, Hkv,
                           Nq, Nk, d, scale, int(causal), code, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    torch.cuda.synchronize()
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
    assert o_ok() and l_ok() and dq_ok() and dk_ok() and dv_ok(), "write outside an output"
    # the packed bits against the byte mask
    b64 = bits.cpu().numpy().astype(np.uint32)
    for b in range(B):
        got = [(int(b64[b, j // 32]) >> (j % 32)) & 1 for j in range(Nk)]
        assert got == keep[b].tolist()
    o64, l64 = f64(o), f64(lse)
    o_ref, l_ref = oracle.attn_fwd(fi.q, fi.k, fi.v, scale, causal, key_keep=keep)
    empty = np.isneginf(l_ref)
    assert np.isneginf(l64[empty]).all() and (o64.transpose(0, 2, 1, 3)[empty] == 0).all()
    live = ~empty
    check_l(l64[live], l_ref[live])
    check_o(o64, o_ref, q.dtype)
    rq, rk, rv = oracle.attn_bwd(fi.q, fi.k, fi.v, fi.do, scale, causal, key_keep=keep)
    errs = [rel_l2(f64(g), r) for g, r in ((dq, rq), (dk, rk), (dv, rv))]
    check_grads(errs)
    # masked keys get exactly zero gradients
    masked = keep == 0
    assert (f64(dk)[masked] == 0).all() and (f64(dv)[masked] == 0).all()


def test_all_ones_mask_is_the_plain_path():
    B, N, Hq, Hkv, d = 1, 300, 2, 1, 128
    fi = inputs.make_fixed(inputs.CAUSAL_GQA, B=B, Nq=N, Nk=N, Hq=Hq, Hkv=Hkv, d=d, seed=103)
    q, k, v = (t.cuda() for t in (fi.q, fi.k, fi.v))
    bits = torch.full((B, (N + 31) // 32), -1, dtype=torch.int32, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
    st = fb.fa_fwd_keymask(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), bits.data_ptr(),
                           B, Hq, Hkv, N, N, d, d ** -0.5, 1, fb.FA_BF16, 0)
    assert st == fb.FA_OK
    o2, l2 = fb.attention_fwd(q, k, v, d ** -0.5, True)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, l2)
