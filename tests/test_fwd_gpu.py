"""Forward parity: the CUDA path (through the C ABI) against the fp64 oracle."""
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


def run_fwd(fi, causal, scale=None, guard=True):
    q, k, v = fi.q.cuda(), fi.k.cuda(), fi.v.cuda()
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    scale = d ** -0.5 if scale is None else scale
    o, o_ok = guarded((B, Nq, Hq, d), q.dtype)
    lse, l_ok = guarded((B, Hq, Nq), torch.float32)
    st = fb.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, Nq, Nk, d,
                   scale, int(causal), fb.FA_BF16 if q.dtype == torch.bfloat16 else fb.FA_FP16, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    torch.cuda.synchronize()
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
    assert o_ok() and l_ok(), "write outside O / L"
    return o, lse


def check(o, lse, o_ref, lse_ref, rows=None):
    dtype = o.dtype
    o, lse = f64(o), f64(lse)
    if rows is not None:
        o, lse, o_ref, lse_ref = o[:, rows], lse[:, :, rows], o_ref[:, rows], lse_ref[:, :, rows]
    empty = np.isneginf(lse_ref)
    assert np.isneginf(lse[empty]).all() and (o.transpose(0, 2, 1, 3)[empty] == 0).all()
    live = ~empty
    check_l(lse[live], lse_ref[live])
    check_o(o, o_ref, dtype)


SMALL = [
    # B, Hq, Hkv, Nq, Nk, d, causal, dtype
    (1, 2, 2, 256, 256, 64, False, "bf16"),
    (2, 4, 2, 129, 129, 128, False, "bf16"),
    (1, 2, 1, 1, 1, 64, False, "bf16"),
    (1, 1, 1, 127, 300, 128, False, "fp16"),
    (2, 2, 2, 300, 127, 64, True, "bf16"),
    (1, 4, 1, 257, 257, 128, True, "bf16"),
    (1, 2, 2, 200, 520, 128, True, "fp16"),
    (3, 3, 3, 384, 384, 64, True, "fp16"),
    (1, 6, 2, 640, 700, 64, False, "bf16"),
    (2, 2, 1, 1000, 1000, 128, True, "bf16"),
    # last key tile of exactly 32 keys, a single tile of 32, and one of 33 (the narrow tail's edges)
    (1, 2, 2, 300, 160, 64, False, "fp16"),
    (1, 2, 2, 129, 32, 128, False, "bf16"),
    (2, 2, 1, 200, 33, 128, False, "bf16"),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "-".join(map(str, c)))
def test_fwd_small_shapes(case):
    B, Hq, Hkv, Nq, Nk, d, causal, dt = case
    fi = inputs.make_fixed(inputs.TINY, B=B, Hq=Hq, Hkv=Hkv, Nq=Nq, Nk=Nk, d=d, dtype=dt, causal=causal, seed=17)
    o, lse = run_fwd(fi, causal)
    o_ref, lse_ref = oracle.attn_fwd(fi.q, fi.k, fi.v, d ** -0.5, causal)
    check(o, lse, o_ref, lse_ref)


def test_fwd_no_keys_gives_zero_and_minus_inf():
    fi = inputs.make_fixed(inputs.TINY, Nk=0)
    o, lse = run_fwd(fi, False)
    assert (f64(o) == 0).all() and torch.isneginf(lse).all()


def test_fwd_tiny_workload_exact_config():
    cfg = inputs.TINY
    fi = inputs.make_fixed(cfg)
    o, lse = run_fwd(fi, cfg.causal, cfg.scale)
    o_ref, lse_ref = oracle.attn_fwd(fi.q, fi.k, fi.v, cfg.scale, cfg.causal)
    check(o, lse, o_ref, lse_ref)


def sample_rows(N, n, seed):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(N, size=min(n, N), replace=False).tolist()) | {0, N - 1, (N // 128) * 128 - 1}
    return sorted(r for r in rows if 0 <= r < N)


# The prefill shape's other variants the benchmark times: without the mask (the persistent
# grid keeps a (batch, head)'s units together instead of heaviest first) and with one query
# head per KV head.
_PREFILL_NONCAUSAL = inputs.FixedConfig(**{**inputs.CAUSAL_GQA.__dict__, "causal": False,
                                           "name": inputs.CAUSAL_GQA.name + "_noncausal"})
_PREFILL_MHA = inputs.FixedConfig(**{**inputs.CAUSAL_GQA.__dict__, "Hkv": inputs.CAUSAL_GQA.Hq,
                                     "name": inputs.CAUSAL_GQA.name + "_hkv32"})


@pytest.mark.parametrize("cfg", [inputs.VISION, inputs.VIT_RMSNORM, inputs.CAUSAL_GQA, _PREFILL_NONCAUSAL, _PREFILL_MHA],
                         ids=lambda c: c.name)
def test_fwd_full_size_sampled_rows(cfg):
    fi = inputs.make_fixed(cfg, with_do=False)
    o, lse = run_fwd(fi, cfg.causal, cfg.scale)
    rows = sample_rows(cfg.Nq, 24, cfg.seed)
    if cfg.causal:  # the first rows see few keys: the largest |O| and the hardest rows for 16-bit P and O
        rows = sorted(set(rows) | set(range(256)))
    o_ref, lse_ref = oracle.attn_fwd(fi.q, fi.k, fi.v, cfg.scale, cfg.causal, rows=rows)
    check(o, lse, o_ref, lse_ref, rows)
