"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory.

Such callers (a host framework that owns every device allocation, a loop that
must not pay for cudaMalloc's synchronisation, a plugin with a fixed budget)
cannot hand fa_bwd a workspace, so fa_bwd_noalloc uses a fixed array inside
the library instead. These tests check that it gives fa_bwd's results, call
after call on the same array, and that it refuses sizes its array cannot hold.
This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from exact_tiled_attention_36_b200 import binding as fb
from exact_tiled_attention_36_b200 import build as fbuild
from exact_tiled_attention_36_b200 import inputs
from tests.gpu_util import RTOL_GRAD, f64

MAX_BYTES = 64 << 20  # FA_BWD_NOALLOC_MAX_BYTES in include/fa.h


def test_noalloc_rejects_sizes_beyond_its_array():
    """Refused before any device work, so this runs without a GPU."""
    fbuild.build()
    fake = 1 << 20
    B, Hq, Hkv, N, d = 1, 64, 8, 8192, 128
    assert fb.fa_bwd_workspace_size(B, Hq, N, d) > MAX_BYTES
    st = fb.fa_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake, B, Hq, Hkv, N, N, d, 0.088, 1,
                           fb.FA_BF16, None)
    assert st == fb.FA_ERR_UNSUPPORTED
    assert fb.fa_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake, 0, 1, 1, 8, 8, 64, 0.1, 0,
                             fb.FA_BF16, None) == fb.FA_ERR_INVALID_ARG
    assert fb.fa_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake, 1, 1, 1, 8, 8, 96, 0.1, 0,
                             fb.FA_BF16, None) == fb.FA_ERR_UNSUPPORTED


def _rel_l2(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)


@pytest.mark.gpu
def test_noalloc_matches_fa_bwd_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    fb.lib()
    B, Hq, Hkv, N, d, causal = 1, 8, 2, 1000, 128, True
    assert fb.fa_bwd_workspace_size(B, Hq, N, d) <= MAX_BYTES
    fi = inputs.make_fixed(inputs.CAUSAL_GQA, B=B, Hq=Hq, Hkv=Hkv, Nq=N, Nk=N, d=d, seed=41)
    q, k, v, do = (t.cuda() for t in (fi.q, fi.k, fi.v, fi.do))
    scale = d ** -0.5
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
    assert fb.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq, Hkv, N, N, d,
                     scale, int(causal), fb.FA_BF16, 0) == fb.FA_OK

    # the existing entry point, with a workspace the caller allocated
    ws = torch.empty(fb.fa_bwd_workspace_size(B, Hq, N, d), dtype=torch.uint8, device="cuda")
    ref = [torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)]
    assert fb.fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                     *(t.data_ptr() for t in ref), ws.data_ptr(), B, Hq, Hkv, N, N, d, scale, int(causal),
                     fb.FA_BF16, 0) == fb.FA_OK
    torch.cuda.synchronize()
    ref = [f64(t) for t in ref]

    # two calls in a row on the library's own array: the second must not see
    # what the first left behind
    for call in range(2):
        out = [torch.full_like(q, 7.0), torch.full_like(k, 7.0), torch.full_like(v, 7.0)]
        st = fb.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                               do.data_ptr(), *(t.data_ptr() for t in out), B, Hq, Hkv, N, N, d, scale, int(causal),
                               fb.FA_BF16, 0)
        assert st == fb.FA_OK, fb.fa_status_string(st)
        torch.cuda.synchronize()
        assert fb.fa_get_last_device_error(None) == fb.FA_OK
        for name, got, want in zip(("dq", "dk", "dv"), out, ref):
            err = _rel_l2(f64(got), want)
            assert err <= RTOL_GRAD, (call, name, err)
