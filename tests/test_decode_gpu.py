"""Split-KV decode parity: fa_decode / fa_decode_paged (through the C ABI) against the
fp64 oracle's attention of each sequence over its own cached keys."""
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


def run(di, causal, paged=False, ws=None):
    """One call through the C ABI; O and L come back as fp64 arrays."""
    q = di.q.cuda()
    B, Nq, Hq, d = q.shape
    Hkv = di.k.shape[2]
    dt = fb.FA_BF16 if q.dtype == torch.bfloat16 else fb.FA_FP16
    o, o_ok = guarded((B, Nq, Hq, d), q.dtype)
    lse, l_ok = guarded((B, Hq, Nq), torch.float32)
    if ws is None:
        ws = torch.full((fb.fa_decode_workspace_size(B, Hq, Hkv, Nq, d),), 255, dtype=torch.uint8, device="cuda")
    sl = None if di.seqlens is None else torch.tensor(di.seqlens, dtype=torch.int32, device="cuda")
    if paged:
        kp, vp, bt = di.k_pages.cuda(), di.v_pages.cuda(), di.block_table.cuda()
        st = fb.fa_decode_paged(q.data_ptr(), kp.data_ptr(), vp.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                sl.data_ptr(), bt.data_ptr(), ws.data_ptr(), B, Hq, Hkv, Nq, kp.shape[0],
                                di.page_size, bt.shape[1], d, d ** -0.5, int(causal), dt, 0)
    else:
        k, v = di.k.cuda(), di.v.cuda()
        st = fb.fa_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                          0 if sl is None else sl.data_ptr(), ws.data_ptr(), B, Hq, Hkv, Nq, k.shape[1], d,
                          d ** -0.5, int(causal), dt, 0)
    assert st == fb.FA_OK, fb.fa_status_string(st)
    torch.cuda.synchronize()
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
    assert o_ok() and l_ok(), "write outside O / L"
    return f64(o), f64(lse)


def check(di, o, lse, causal):
    o_ref, l_ref = oracle.attn_decode(di.q, di.k, di.v, di.cfg.scale, di.seqlens, causal)
    empty = np.isneginf(l_ref)
    assert np.isneginf(lse[empty]).all() and (o[np.moveaxis(empty, 1, 2)] == 0).all(), "rows without keys"
    live = ~empty
    assert np.isfinite(lse[live]).all() and np.isfinite(o).all()
    if live.any():
        check_l(lse[live], l_ref[live])
    check_o(o, o_ref, di.q.dtype)


def small(**kw):
    base = dict(B=3, Hq=8, Hkv=2, Nq=1, Nk=1000, d=128, dtype="bf16", causal=False, seed=61)
    base.update(kw)
    return base


CASES = [
    # (config overrides, lengths, causal)
    (small(), None, False),                                     # full caches, ragged last tile (1000 keys)
    (small(Nq=2, B=5, Nk=2048), [0, 1, 129, 1000, 2047], True),  # own lengths, causal, an empty sequence
    (small(Hq=4, Hkv=4, d=64, dtype="fp16", Nk=777), [777, 5, 640], False),  # MHA (one row per item), d = 64
    (small(Hq=32, Hkv=4, Nq=4, Nk=1500), [1500, 3, 1024], True),  # speculative: 4 tokens x 8 heads
    (small(Hq=6, Hkv=2, Nq=20, Nk=300), [300, 260, 17], True),   # 60 rows in lanes 0..59 (no head split)
    (small(Hq=16, Hkv=1, Nq=8, Nk=900, d=64), None, True),       # 128 rows, the whole tile
    (small(B=40, Hkv=8, Hq=32, Nk=700, len_seed=9, min_len=0), None, False),  # many short items
    (small(Hq=8, Hkv=4, Nq=3, Nk=1000, d=64), [1000, 2, 513], True),   # d = 64, paired KV heads, 6 rows each
    (small(Hq=16, Hkv=2, Nq=2, Nk=600, d=64, dtype="fp16"), None, True),  # paired heads, 16 rows each
    (small(Hq=6, Hkv=3, Nq=1, Nk=900, d=64), [900, 1, 128], False),   # d = 64, odd Hkv: no pairing
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(f"{k}{v}" for k, v in c[0].items()
                                                                 if k in ("B", "Hq", "Hkv", "Nq", "Nk", "d"))
                         + f"-c{int(c[2])}")
def test_decode_contiguous(case):
    kw, lengths, causal = case
    cfg = inputs.DecodeConfig(name="t", **kw)
    di = inputs.make_decode(cfg, lengths=lengths)
    o, lse = run(di, causal)
    check(di, o, lse, causal)


@pytest.mark.parametrize("page_size", [16, 32, 64, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_decode_paged(page_size, causal):
    cfg = inputs.DecodeConfig(name="t", **small(B=4, Nq=2, Nk=1100, len_seed=11 + page_size, min_len=0))
    di = inputs.make_decode(cfg, page_size=page_size)
    o, lse = run(di, causal, paged=True)
    check(di, o, lse, causal)
    # the same caches contiguous give the same result up to the order of the merge
    o2, lse2 = run(di, causal)
    assert np.abs(o - o2).max() <= 2 * 2.0 ** -8 and np.abs(np.nan_to_num(lse - lse2)).max() <= 1e-4


@pytest.mark.parametrize("page_size", [16, 32])
def test_decode_paged_small_pages_paired_heads(page_size):
    """16/32-row pages with d = 64 paired KV heads (rows of two heads' 128 values)."""
    cfg = inputs.DecodeConfig(name="t", **small(B=5, Hq=8, Hkv=4, Nq=2, Nk=1300, d=64, len_seed=21, min_len=0))
    di = inputs.make_decode(cfg, page_size=page_size, spare_pages=7)
    o, lse = run(di, True, paged=True)
    check(di, o, lse, True)


@pytest.mark.parametrize("page_size", [16, 64])
def test_decode_paged_out_of_pool_pages(page_size):
    """Block-table entries outside [0, num_pages) inside a sequence's length read zero rows."""
    cfg = inputs.DecodeConfig(name="t", **small(B=3, Nq=2, Nk=700))
    di = inputs.make_decode(cfg, lengths=[700, 300, 650], page_size=page_size)
    n_pages = di.k_pages.shape[0]
    for b, i, page in ((0, 1, -1), (0, 5, n_pages), (1, 0, n_pages + 1000), (2, 650 // page_size, -7)):
        di.block_table[b, i] = page
        di.k[b, i * page_size:(i + 1) * page_size] = 0
        di.v[b, i * page_size:(i + 1) * page_size] = 0
    for b, n in enumerate(di.seqlens):  # rows past the length stay NaN
        di.k[b, n:] = float("nan")
        di.v[b, n:] = float("nan")
    o, lse = run(di, True, paged=True)
    check(di, o, lse, True)


def test_decode_paged_fp16_d64_more_pages_than_used():
    cfg = inputs.DecodeConfig(name="t", **small(B=6, Hq=16, Hkv=4, Nq=1, Nk=900, d=64, dtype="fp16", len_seed=5))
    di = inputs.make_decode(cfg, page_size=128, spare_pages=40)
    o, lse = run(di, False, paged=True)
    check(di, o, lse, False)


def test_decode_workspace_reused_across_layouts():
    """A workspace holding another call's partial results gives the right answer (no
    stale slot is merged)."""
    ws = torch.empty(fb.fa_decode_workspace_size(16, 8, 2, 1, 128), dtype=torch.uint8, device="cuda")
    a = inputs.make_decode(inputs.DecodeConfig(name="t", **small(B=16, Nk=3000, len_seed=3, min_len=0)))
    b = inputs.make_decode(inputs.DecodeConfig(name="t", **small(B=16, Nk=3000, seed=62)),
                           lengths=[0] * 8 + [3000] * 8)
    for di in (a, b, a):
        o, lse = run(di, False, ws=ws)
        check(di, o, lse, False)


def test_decode_no_keys_and_no_queries():
    di = inputs.make_decode(inputs.DecodeConfig(name="t", **small(Nk=0)))
    o, lse = run(di, False)
    assert (o == 0).all() and np.isneginf(lse).all()
    di = inputs.make_decode(inputs.DecodeConfig(name="t", **small()), lengths=[0, 0, 0])
    o, lse = run(di, True)
    assert (o == 0).all() and np.isneginf(lse).all()
    q = torch.empty((2, 0, 8, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((2, 64, 2, 128), dtype=torch.bfloat16, device="cuda")
    st = fb.fa_decode(q.data_ptr(), kv.data_ptr(), kv.data_ptr(), q.data_ptr(), q.data_ptr(), 0, kv.data_ptr(),
                      2, 8, 2, 0, 64, 128, 0.1, 0, fb.FA_BF16, 0)
    assert st == fb.FA_OK


@pytest.mark.parametrize("cfg", [inputs.DECODE, inputs.DECODE_RAGGED], ids=lambda c: c.name)
def test_decode_full_size(cfg):
    """The benchmark workloads at full size, every output row against the oracle."""
    di = inputs.make_decode(cfg)
    o, lse = run(di, cfg.causal)
    check(di, o, lse, cfg.causal)
    if cfg.len_seed >= 0:  # the paged layouts of the benchmark: 64-row pages (TMA) and 16-row pages (cp.async)
        for page_size in (64, 16):
            o_p, lse_p = run(inputs.make_decode(cfg, page_size=page_size), cfg.causal, paged=True)
            check(di, o_p, lse_p, cfg.causal)


def test_attention_decode_wrapper():
    di = inputs.make_decode(inputs.DecodeConfig(name="t", **small(Nq=2)), lengths=[1000, 31, 512], page_size=32)
    sl = torch.tensor(di.seqlens, dtype=torch.int32, device="cuda")
    o, L = fb.attention_decode(di.q.cuda(), di.k.cuda(), di.v.cuda(), sl, causal=True)
    check(di, f64(o), f64(L), True)
    o, L = fb.attention_decode(di.q.cuda(), di.k_pages.cuda(), di.v_pages.cuda(), sl, causal=True,
                               block_table=di.block_table.cuda())
    check(di, f64(o), f64(L), True)
