"""Failure detection without a GPU fault: the bounded waits of the pipelined
per-channel backward are made to run out and must report it.

mea_affine_bwd_wait_selftest runs the pipelined NHWC backward of the fused
affine + Swish with the producer's copies withheld, so no stage barrier ever
completes (a flag that nothing sets).  Every wait gives up after a few
milliseconds and records the workspace's error word; the kernel returns.
The test checks that the word was set, that the context is still usable
afterwards (the regular backward on the same workspace gives the oracle's
results with the word back at zero), and that a shape off the pipelined
path is refused.
"""
import numpy as np
import pytest
import torch

import memory_efficient_activation_b200 as mea
import oracle
from _compare import TINY, check, to_f64
from memory_efficient_activation_b200 import synthetic

pytestmark = pytest.mark.gpu


def _problem(shape, dtype, seed):
    n = int(np.prod(shape))
    C = shape[3]
    x = synthetic.normal(n, 1.0, seed, synthetic.STREAM_X, dtype).view(shape)
    dy = synthetic.normal(n, 1.0, seed, synthetic.STREAM_DY, dtype).view(shape)
    g = torch.from_numpy(synthetic.uniform_f64(C, 0.5, 1.5, seed, synthetic.STREAM_GAMMA)).float()
    b = torch.from_numpy(synthetic.normal_f64(C, 0.1, seed, synthetic.STREAM_BETA)).float()
    return x, dy, g, b


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_bounded_waits_expire_and_report(dtype):
    shape = (16, 14, 14, 144)
    x, dy, g, b = _problem(shape, dtype, 601)
    xc, dyc, gc, bc = x.cuda(), dy.cuda(), g.cuda(), b.cuda()
    need = mea.affine_swish_bwd_workspace_bytes(xc.dtype, "nhwc", (16, 144, 14, 14))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    assert mea.affine_bwd_wait_selftest(xc, dyc, gc, bc, workspace=ws) == 1
    assert int(ws[4:8].view(torch.int32).item()) == 0          # read and cleared by the call
    # the context is still usable: the regular backward on the same workspace
    dx, dg, db = mea.affine_swish_bwd(xc, dyc, gc, bc, "nhwc", workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[4:8].view(torch.int32).item()) == 0
    xd, gd = to_f64(x), to_f64(dy)
    rdx, rdg, rdb, scale = oracle.affine_swish_bwd("nhwc", (16, 144, 14, 14), xd, gd, g.double().numpy(),
                                                   b.double().numpy(), with_scale=True)
    ey, edx = oracle.affine_act_zround("swish", "nhwc", (16, 144, 14, 14), xd, gd, g.double().numpy(),
                                       b.double().numpy(), 1.0)
    check(dtype, dx.cpu(), rdx, scale=scale, floor=TINY * np.maximum(1, np.abs(gd)), what="dx after self-test",
          zround=edx)


def test_selftest_refuses_shapes_off_the_pipelined_path():
    x, dy, g, b = _problem((2, 3, 5, 6), "bf16", 602)        # C = 6: not the NHWC fast path
    with pytest.raises(mea.MeaError):
        mea.affine_bwd_wait_selftest(x.cuda(), dy.cuda(), g.cuda(), b.cuda())
