"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory.

Such callers (a host framework that owns every device allocation, a loop that
must not pay for cudaMalloc's synchronisation, a plugin with a fixed budget)
cannot hand fa_bwd a workspace, so fa_bwd_noalloc uses a fixed array inside
the library instead. These tests check that it gives fa_bwd's results, call
after call on the same array (also when a smaller call follows a larger one,
and for both accumulator layouts, d = 128 and d = 64), and that it refuses
sizes its array cannot hold.

The tests do not depend on what ran before them: each passes alone in a fresh
process and after the rest of the suite. The file name only puts them last in
collection order, so that a run which stops at the first failure has already
run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_36_b200 import binding as fb
from exact_tiled_attention_36_b200 import build as fbuild
from exact_tiled_attention_36_b200 import inputs
from tests.gpu_util import check_rel, f64, rel_l2

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


class _Case:
    """Inputs, forward outputs and fa_bwd's gradients (with a caller workspace)."""

    def __init__(self, B, Hq, Hkv, N, d, causal, seed):
        self.B, self.Hq, self.Hkv, self.N, self.d, self.causal = B, Hq, Hkv, N, d, causal
        assert fb.fa_bwd_workspace_size(B, Hq, N, d) <= MAX_BYTES
        self.fi = inputs.make_fixed(inputs.CAUSAL_GQA, B=B, Hq=Hq, Hkv=Hkv, Nq=N, Nk=N, d=d, seed=seed)
        self.q, self.k, self.v, self.do = (t.cuda() for t in (self.fi.q, self.fi.k, self.fi.v, self.fi.do))
        self.scale = d ** -0.5
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
        assert fb.fa_fwd(*self._ptrs(self.q, self.k, self.v, self.o), self.lse.data_ptr(), B, Hq, Hkv, N, N, d,
                         self.scale, int(causal), fb.FA_BF16, 0) == fb.FA_OK
        ws = torch.empty(fb.fa_bwd_workspace_size(B, Hq, N, d), dtype=torch.uint8, device="cuda")
        ref = self._outputs()
        assert fb.fa_bwd(*self._ptrs(self.q, self.k, self.v, self.o), self.lse.data_ptr(), self.do.data_ptr(),
                         *self._ptrs(*ref), ws.data_ptr(), B, Hq, Hkv, N, N, d, self.scale, int(causal),
                         fb.FA_BF16, 0) == fb.FA_OK
        torch.cuda.synchronize()
        assert fb.fa_get_last_device_error(None) == fb.FA_OK
        self.ref = [t.cpu() for t in ref]

    @staticmethod
    def _ptrs(*ts):
        return [t.data_ptr() for t in ts]

    def _outputs(self):
        return [torch.full_like(self.q, 7.0), torch.full_like(self.k, 7.0), torch.full_like(self.v, 7.0)]

    def noalloc(self):
        out = self._outputs()
        st = fb.fa_bwd_noalloc(*self._ptrs(self.q, self.k, self.v, self.o), self.lse.data_ptr(), self.do.data_ptr(),
                               *self._ptrs(*out), self.B, self.Hq, self.Hkv, self.N, self.N, self.d, self.scale,
                               int(self.causal), fb.FA_BF16, 0)
        assert st == fb.FA_OK, fb.fa_status_string(st)
        torch.cuda.synchronize()
        assert fb.fa_get_last_device_error(None) == fb.FA_OK
        return [t.cpu() for t in out]

    def check(self, out, call):
        dq, dk, dv = out
        # dK and dV come from the same deterministic kernels as fa_bwd's: bit-equal
        assert torch.equal(dk, self.ref[1]), (call, "dk")
        assert torch.equal(dv, self.ref[2]), (call, "dv")
        # dQ sums fp32 reductions in whatever order they land: within the tolerance of
        # fa_bwd's dQ and of the oracle's exact gradient
        check_rel(rel_l2(f64(dq), f64(self.ref[0])), "noalloc dQ vs fa_bwd rel L2")
        rq, _, _ = oracle.attn_bwd(self.fi.q, self.fi.k, self.fi.v, self.fi.do, self.scale, self.causal)
        check_rel(rel_l2(f64(dq), rq), "noalloc dQ vs oracle rel L2")


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    fb.lib()


@pytest.mark.gpu
def test_noalloc_matches_fa_bwd_on_two_calls_in_a_row():
    _need_gpu()
    c = _Case(1, 8, 2, 1000, 128, True, seed=41)
    # two calls in a row on the library's own array: the second must not see
    # what the first left behind
    for call in range(2):
        c.check(c.noalloc(), call)


@pytest.mark.gpu
def test_noalloc_d64_and_a_smaller_call_after_a_larger_one():
    """The d = 64 accumulator layout ([B, Nq, Hq, 64], its own convert kernel), and a
    smaller d = 128 call right after a larger one on the shared array (the smaller call
    must not pick up the rest of the larger call's accumulator)."""
    _need_gpu()
    small64 = _Case(2, 4, 2, 333, 64, False, seed=42)
    big = _Case(2, 8, 4, 1500, 128, False, seed=43)
    small = _Case(1, 2, 1, 130, 128, True, seed=44)
    small64.check(small64.noalloc(), "d64 first")
    big.check(big.noalloc(), "large")
    small.check(small.noalloc(), "small after large")
    small64.check(small64.noalloc(), "d64 after large")
