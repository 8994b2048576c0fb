"""The entry points inside CUDA graphs: a forward + backward, and a decode call (split
kernel with its programmatically dependent merge), captured on a stream and replayed,
give the eager results. Nothing in these calls synchronises or allocates, so a whole
step can be captured once and replayed."""
import pytest
import torch

from exact_tiled_attention_36_b200 import binding as fb
from exact_tiled_attention_36_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    fb.lib()
    yield
    assert fb.fa_get_last_device_error(None) == fb.FA_OK


def test_forward_backward_graph_replay():
    B, N, Hq, Hkv, d = 1, 700, 4, 2, 128
    fi = inputs.make_fixed(inputs.CAUSAL_GQA, B=B, Nq=N, Nk=N, Hq=Hq, Hkv=Hkv, d=d, seed=95)
    q, k, v, do = (t.cuda() for t in (fi.q, fi.k, fi.v, fi.do))
    scale = d ** -0.5
    o, lse = torch.empty_like(q), torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fb.fa_bwd_workspace_size(B, Hq, N, d), dtype=torch.uint8, device="cuda")

    def step(stream):
        st = fb.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N, N, d,
                       scale, 1, fb.FA_BF16, stream)
        assert st == fb.FA_OK
        st = fb.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                       dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), B, Hq, Hkv, N, N, d, scale, 1,
                       fb.FA_BF16, stream)
        assert st == fb.FA_OK

    step(torch.cuda.current_stream().cuda_stream)  # eager (also the one-time set-up of every kernel)
    torch.cuda.synchronize()
    ref = [t.clone() for t in (o, lse, dq, dk, dv)]
    for t in (o, lse, dq, dk, dv):
        t.fill_(0)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=s):
        step(s.cuda_stream)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
    assert torch.equal(o, ref[0]) and torch.equal(lse, ref[1])
    assert torch.equal(dk, ref[3]) and torch.equal(dv, ref[4])
    # dQ: the same fp32 sums, in an order the reductions' arrival decides
    err = (dq.float() - ref[2].float()).norm() / ref[2].float().norm()
    assert float(err) <= 1e-2


@pytest.mark.parametrize("lengths", [None, [8192, 5, 3000, 129]])
def test_decode_graph_replay(lengths):
    cfg = inputs.DecodeConfig(name="t", B=4, Hq=32, Hkv=8, Nq=1, Nk=8192, d=128, dtype="bf16", causal=False,
                              seed=97)
    di = inputs.make_decode(cfg, lengths=lengths)
    q, k, v = di.q.cuda(), di.k.cuda(), di.v.cuda()
    B, Nq, Hq, d = q.shape
    sl = None if lengths is None else torch.tensor(lengths, dtype=torch.int32, device="cuda")
    ws = torch.empty(fb.fa_decode_workspace_size(B, Hq, 8, Nq, d), dtype=torch.uint8, device="cuda")
    o, lse = torch.empty_like(q), torch.empty((B, Hq, Nq), dtype=torch.float32, device="cuda")

    def call(stream):
        st = fb.fa_decode(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                          0 if sl is None else sl.data_ptr(), ws.data_ptr(), B, Hq, 8, Nq, cfg.Nk, d, cfg.scale, 0,
                          fb.FA_BF16, stream)
        assert st == fb.FA_OK

    call(torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    ref_o, ref_l = o.clone(), lse.clone()
    o.fill_(0)
    lse.fill_(0)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=s):
        call(s.cuda_stream)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
    assert torch.equal(o, ref_o) and torch.equal(lse, ref_l)
