"""The allocation-free Swish backward with d alpha (mea_act_bwd_dparam_noalloc).

Some callers cannot allocate device memory for the reduction scratch: code
whose device memory belongs entirely to another allocator (a framework's
caching allocator or a fixed memory plan), and latency-sensitive paths that
cannot take the synchronisation cudaFree brings.  This entry point serves them
from a fixed array inside the library.  The test calls it through the C ABI,
twice in a row on the same stream (the second call must find the array's
completion counter clear again), and checks dx and d alpha against the
regular entry point (mea_act_bwd with a caller-allocated workspace) under the
same tolerances as the other tests: dx per element (1 bf16 ulp, or 1e-5
relative for fp32) and d alpha within 1e-5 relative.  Both run the
same kernel on the same fixed grid, so the results are expected to be
bitwise equal as well.

This file is collected last on purpose: a failure here leaves every other
test already run when pytest stops at the first failure.
"""
import numpy as np
import pytest
import torch

import memory_efficient_activation_b200 as mea
from _compare import TINY, check, to_f64
from memory_efficient_activation_b200 import _capi, synthetic

pytestmark = pytest.mark.gpu

DT = {"bf16": _capi.MEA_BF16, "f32": _capi.MEA_F32}


def _regular(x, dy, alpha):
    d = torch.empty(1, dtype=torch.float32, device="cuda")
    nbytes = mea.act_bwd_workspace_bytes("swish", x.numel(), True)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    dx = torch.empty_like(x)
    st = _capi.lib().mea_act_bwd(_capi.MEA_SWISH, DT["bf16" if x.dtype == torch.bfloat16 else "f32"],
                                 x.data_ptr(), dy.data_ptr(), dx.data_ptr(), x.numel(), alpha, None,
                                 d.data_ptr(), ws.data_ptr(), nbytes, torch.cuda.current_stream().cuda_stream)
    _capi.check("mea_act_bwd", st)
    return dx, d


def _no_alloc(x, dy, alpha):
    d = torch.empty(1, dtype=torch.float32, device="cuda")
    dx = torch.empty_like(x)
    st = _capi.lib().mea_act_bwd_dparam_noalloc(
        _capi.MEA_SWISH, DT["bf16" if x.dtype == torch.bfloat16 else "f32"], x.data_ptr(), dy.data_ptr(),
        dx.data_ptr(), x.numel(), alpha, None, d.data_ptr(), torch.cuda.current_stream().cuda_stream)
    _capi.check("mea_act_bwd_dparam_noalloc", st)
    return dx, d


@pytest.mark.parametrize("dtype,n,alpha", [
    ("f32", 12042240, 1.37),          # EfficientNet-B0-like [64, 240, 28, 28]
    ("bf16", 1000003, 0.8),           # ragged size, bf16 storage
    ("f32", 4099, 2.0),               # a single reduction block
])
def test_no_alloc_matches_regular_entry_point(dtype, n, alpha):
    x = synthetic.normal(n, 1.5, 401, synthetic.STREAM_X, dtype).cuda()
    dy = synthetic.normal(n, 1.0, 401, synthetic.STREAM_DY, dtype).cuda()
    ref_dx, ref_d = _regular(x, dy, alpha)
    first = _no_alloc(x, dy, alpha)
    second = _no_alloc(x, dy, alpha)
    torch.cuda.synchronize()
    gd = to_f64(dy)
    r = to_f64(ref_dx)
    for dx, d in (first, second):
        check(dtype, dx.cpu(), r, what="no-alloc dx vs regular", floor=TINY * np.maximum(1, np.abs(gd)))
        got, ref = float(d.item()), float(ref_d.item())
        assert abs(got - ref) <= 1e-5 * abs(ref), (got, ref)
        assert torch.equal(dx, ref_dx) and torch.equal(d, ref_d)


def test_no_alloc_without_dparam_is_plain_backward():
    x = synthetic.normal(70001, 2.0, 402, synthetic.STREAM_X, "bf16").cuda()
    dy = synthetic.normal(70001, 1.0, 402, synthetic.STREAM_DY, "bf16").cuda()
    dx = torch.empty_like(x)
    st = _capi.lib().mea_act_bwd_dparam_noalloc(_capi.MEA_SWISH, _capi.MEA_BF16, x.data_ptr(), dy.data_ptr(),
                                                dx.data_ptr(), x.numel(), 1.0, None, None,
                                                torch.cuda.current_stream().cuda_stream)
    _capi.check("mea_act_bwd_dparam_noalloc", st)
    torch.cuda.synchronize()
    assert torch.equal(dx, mea.act_bwd("swish", x, dy))


def test_no_alloc_refuses_what_the_regular_entry_point_refuses():
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    d = torch.empty(1, dtype=torch.float32, device="cuda")
    lib = _capi.lib()
    s = torch.cuda.current_stream().cuda_stream
    assert lib.mea_act_bwd_dparam_noalloc(_capi.MEA_RELU, _capi.MEA_BF16, x.data_ptr(), x.data_ptr(),
                                          x.data_ptr(), 16, 1.0, None, d.data_ptr(), s) == _capi.MEA_ERR_UNSUPPORTED
    assert lib.mea_act_bwd_dparam_noalloc(_capi.MEA_SWISH, _capi.MEA_BF16, x.data_ptr(), x.data_ptr(),
                                          x.data_ptr(), -1, 1.0, None, d.data_ptr(), s) == _capi.MEA_ERR_INVALID_ARG
