"""The allocation-free quantise entry point.

Some callers cannot allocate device memory (their host framework owns all of
it, or they run after the device has already run out of memory), so the
library offers qlora_nf4_quantize_noalloc, which keeps its scratch in a
static device array instead of a caller workspace.  These tests call it
through the C ABI and check that it writes exactly what qlora_nf4_quantize
writes, on two calls in a row with different weights (the second call must
not see anything left over by the first).  This file is collected last on
purpose: it runs after every other test, and also passes on its own in a
fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import synthetic

pytestmark = pytest.mark.gpu

q4 = pytest.importorskip("parameter_efficient_fine_nf4_b200")


def _outputs(qw):
    return [qw.codes.cpu().numpy(), qw.absmax_q.cpu().numpy(),
            qw.scale2.cpu().numpy().view(np.uint32), qw.mean.cpu().numpy().view(np.uint32)]


def _noalloc_via_cabi(W0: torch.Tensor) -> "q4.NF4Weight":
    d, k = W0.shape
    out = q4.NF4Weight(d, k, W0.device)
    stream = ctypes.c_void_p(int(torch.cuda.current_stream().cuda_stream))
    st = q4.lib().qlora_nf4_quantize_noalloc(W0.data_ptr(), d, k, 64, ctypes.byref(out.cstruct), stream)
    assert st == 0, q4.strerror(st)
    return out


def test_noalloc_matches_workspace_quantize_two_calls():
    torch.cuda.set_device(0)
    weights = [
        torch.from_numpy(synthetic.make_layer(synthetic.config(3), with_acts=False).W0).cuda(),
        torch.from_numpy(synthetic.custom_layer(seed=77, d=300, k=192, r=4, T=1, alpha=8.0).W0).cuda(),
    ]
    for W0 in weights:                                # two calls in a row, different sizes
        got = _noalloc_via_cabi(W0)
        ref = q4.qlora_nf4_quantize(W0)              # existing entry point, own workspace
        torch.cuda.synchronize()
        assert q4.qlora_get_device_status() == 0
        for a, b in zip(_outputs(got), _outputs(ref)):
            assert np.array_equal(a, b)              # bit-exact, as for every quantise test


def test_noalloc_rejects_sizes_beyond_its_scratch():
    d, k = 1 << 15, (1 << 13) + 64                   # d*k just above 2^28
    dummy = q4.NF4Weight(64, 64)
    stream = ctypes.c_void_p(int(torch.cuda.current_stream().cuda_stream))
    st = q4.lib().qlora_nf4_quantize_noalloc(16, d, k, 64, ctypes.byref(dummy.cstruct), stream)
    assert st == 8
    assert "static scratch" in q4.strerror(st)
