"""Backward parity: fa_bwd (through the C ABI) against the fp64 oracle's exact gradients."""
import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_36_b200 import binding as fb
from exact_tiled_attention_36_b200 import inputs
from tests.gpu_util import check_grads, check_rel, f64, guarded, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    fb.lib()
    yield
    assert fb.fa_get_last_device_error(None) == fb.FA_OK


def run_fwd_bwd(fi, causal, scale):
    q, k, v, do = fi.q.cuda(), fi.k.cuda(), fi.v.cuda(), fi.do.cuda()
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    dt = fb.FA_BF16 if q.dtype == torch.bfloat16 else fb.FA_FP16
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device="cuda")
    assert fb.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Nq, Nk, d,
                     scale, int(causal), dt, 0) == fb.FA_OK
    ws = torch.full((fb.fa_bwd_workspace_size(B, Hq, Nq, d),), 255, dtype=torch.uint8, device="cuda")
    dq, dq_ok = guarded((B, Nq, Hq, d), q.dtype)
    dk, dk_ok = guarded((B, Nk, Hkv, d), q.dtype)
    dv, dv_ok = guarded((B, Nk, Hkv, d), q.dtype)
    st = fb.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                   dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), B, Hq, Hkv, Nq, Nk, d, scale,
                   int(causal), dt, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    torch.cuda.synchronize()
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
    assert dq_ok() and dk_ok() and dv_ok(), "write outside dQ / dK / dV"
    return dq, dk, dv


SMALL = [
    # B, Hq, Hkv, Nq, Nk, d, causal, dtype
    (1, 2, 2, 128, 128, 64, False, "bf16"),
    (1, 2, 2, 256, 256, 128, False, "bf16"),
    (2, 4, 2, 129, 129, 128, True, "bf16"),
    (1, 2, 1, 300, 200, 64, True, "fp16"),
    (1, 2, 2, 200, 333, 128, True, "bf16"),
    (2, 3, 1, 97, 250, 64, False, "fp16"),
    (1, 4, 4, 1, 5, 128, False, "bf16"),
    (1, 8, 2, 520, 520, 128, True, "bf16"),
    (1, 4, 2, 300, 390, 128, False, "bf16"),
    (2, 2, 1, 1000, 700, 128, False, "fp16"),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "-".join(map(str, c)))
def test_bwd_small_shapes(case):
    B, Hq, Hkv, Nq, Nk, d, causal, dt = case
    fi = inputs.make_fixed(inputs.CAUSAL_GQA, B=B, Hq=Hq, Hkv=Hkv, Nq=Nq, Nk=Nk, d=d, dtype=dt, causal=causal,
                           seed=23)
    scale = d ** -0.5
    dq, dk, dv = run_fwd_bwd(fi, causal, scale)
    rq, rk, rv = oracle.attn_bwd(fi.q, fi.k, fi.v, fi.do, scale, causal)
    errs = [rel_l2(f64(x), r) for x, r in ((dq, rq), (dk, rk), (dv, rv))]
    check_grads(errs)


def test_bwd_causal_gqa_full_size():
    """The causal GQA prefill workload at full size, in the launch configuration the
    benchmark times. Element-wise against the oracle: dK and dV of keys on the longest
    and shortest walks (key tiles 0, 1, 16, 31, 46 and 63: each of their CTAs walks
    every query tile after it, for all 4 query heads of the group, so key tile 0 takes
    64 x 4 = 256 iterations of TMEM accumulation), and dQ of one row in each of the 64
    query tiles (each the sum of the reductions of every key tile before it), in four
    (batch, KV head) groups. On every row of dK and dV, two identities that hold at any
    size."""
    cfg = inputs.CAUSAL_GQA
    fi = inputs.make_fixed(cfg)
    dq, dk, dv = run_fwd_bwd(fi, cfg.causal, cfg.scale)
    dq, dk, dv = f64(dq), f64(dk), f64(dv)
    g = cfg.Hq // cfg.Hkv
    N = cfg.Nq
    qrows = sorted({0, N - 1} | {t * 128 + (37 * t) % 128 for t in range(N // 128)})
    krows = [0, 1, 127, 128, 2048, 4095, 6000, 8191]
    q64, k64, v64, do64 = (oracle._f64(t) for t in (fi.q, fi.k, fi.v, fi.do))
    for (b, hk) in [(0, 0), (0, 3), (1, 4), (1, 7)]:
        sq, sk, sv = oracle.attn_bwd_sampled(q64, k64, v64, do64, cfg.scale, b, hk, qrows, krows, True)
        gq = dq[b][qrows][:, hk * g:(hk + 1) * g]
        check_rel(rel_l2(gq, sq), "dQ sampled rows rel L2")
        # each sampled row on its own, not only their sum
        for name, got, ref in (("dk", dk[b, krows, hk], sk), ("dv", dv[b, krows, hk], sv)):
            check_rel(rel_l2(got, ref), f"{name} sampled rows rel L2")
            for t, key in enumerate(krows):
                check_rel(rel_l2(got[t], ref[t]), f"{name} per sampled row rel L2")
        for t, row in enumerate(qrows):
            check_rel(rel_l2(gq[t], sq[t]), "dQ per sampled row rel L2")
    # sum over keys of dK is 0 (rows of dS sum to 0); sum over keys of dV equals the
    # sum of dO over the group's query rows (rows of P sum to 1).
    do = f64(fi.do)
    for b in range(cfg.B):
        for hk in range(cfg.Hkv):
            sdk = dk[b, :, hk].sum(0)
            assert np.abs(sdk).max() <= 2e-2 * np.abs(dk[b, :, hk]).sum(0).max() + 1e-3
            sdv = dv[b, :, hk].sum(0)
            ref = do[b, :, hk * g:(hk + 1) * g].sum((0, 1))
            check_rel(rel_l2(sdv, ref), "sum of dV over keys rel L2")


@pytest.mark.parametrize("hkv,causal", [(32, True), (8, False)], ids=["causal-hq32-hkv32", "noncausal-hq32-hkv8"])
def test_bwd_full_size_other_grids(hkv, causal):
    """The prefill shape in the two other backward grids, element-wise against the oracle:
    - one query head per KV head, causal (Hq = Hkv = 32): the key tiles of a (batch, head)
      run next to each other (key tile fastest) instead of heaviest first, 4096 CTAs;
    - without the mask (Hq = 32, Hkv = 8): every key tile walks all 64 query tiles of its
      4 heads, starting at a query tile rotated by its key tile.
    dK and dV of keys on the first, middle and last key tiles and dQ of one row in each
    query tile, in four (batch, KV head) groups; on every row of dK and dV the two
    identities that hold at any size."""
    cfg = inputs.CAUSAL_GQA
    fi = inputs.make_fixed(cfg, Hkv=hkv, causal=causal)
    dq, dk, dv = run_fwd_bwd(fi, causal, cfg.scale)
    dq, dk, dv = f64(dq), f64(dk), f64(dv)
    g = cfg.Hq // hkv
    N = cfg.Nq
    qrows = sorted({0, N - 1} | {t * 128 + (53 * t) % 128 for t in range(N // 128)})
    krows = [0, 1, 127, 128, 2048, 4095, 6000, 8191]
    q64, k64, v64, do64 = (oracle._f64(t) for t in (fi.q, fi.k, fi.v, fi.do))
    for (b, hk) in [(0, 0), (0, hkv // 2 + 1), (1, hkv // 4 + 1), (1, hkv - 1)]:
        sq, sk, sv = oracle.attn_bwd_sampled(q64, k64, v64, do64, cfg.scale, b, hk, qrows, krows, causal)
        gq = dq[b][qrows][:, hk * g:(hk + 1) * g]
        check_rel(rel_l2(gq, sq), "dQ sampled rows rel L2 (other grids)")
        for name, got, ref in (("dk", dk[b, krows, hk], sk), ("dv", dv[b, krows, hk], sv)):
            for t in range(len(krows)):
                check_rel(rel_l2(got[t], ref[t]), f"{name} per sampled row rel L2 (other grids)")
        for t in range(len(qrows)):
            check_rel(rel_l2(gq[t], sq[t]), "dQ per sampled row rel L2 (other grids)")
    do = f64(fi.do)
    for b in range(cfg.B):
        for hk in range(hkv):
            sdk = dk[b, :, hk].sum(0)
            assert np.abs(sdk).max() <= 2e-2 * np.abs(dk[b, :, hk]).sum(0).max() + 1e-3
            ref = do[b, :, hk * g:(hk + 1) * g].sum((0, 1))
            check_rel(rel_l2(dv[b, :, hk].sum(0), ref), "sum of dV over keys rel L2 (other grids)")
