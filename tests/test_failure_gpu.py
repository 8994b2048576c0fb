"""Failure detection without a GPU fault: a bounded device wait that runs out
is reported as FA_ERR_TIMEOUT, and the context stays usable afterwards."""
import pytest
import torch

import oracle
from exact_tiled_attention_36_b200 import binding as fb
from exact_tiled_attention_36_b200 import inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    assert fb.fa_get_last_device_error(None) == fb.FA_OK  # clean start
    assert fb.fa_selftest_bounded_wait(None) == fb.FA_OK
    assert fb.fa_get_last_device_error(None) == fb.FA_ERR_TIMEOUT
    assert fb.fa_get_last_device_error_site() == 0x1000 + 99
    assert fb.fa_get_last_device_error(None) == fb.FA_OK  # the word was cleared
    # the context is still usable: a normal call computes the right result
    fi = inputs.make_fixed(inputs.TINY, Nq=64, Nk=64)
    o, lse = fb.attention_fwd(fi.q.cuda(), fi.k.cuda(), fi.v.cuda(), inputs.TINY.scale)
    torch.cuda.synchronize()
    o_ref, _ = oracle.attn_fwd(fi.q, fi.k, fi.v, inputs.TINY.scale)
    assert float((o.float().cpu().double() - torch.from_numpy(o_ref)).abs().max()) <= 1e-2
    assert fb.fa_get_last_device_error(None) == fb.FA_OK
