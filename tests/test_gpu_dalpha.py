"""GPU parity of the Swish backward with a learnable alpha (d alpha reduction).

EfficientNet-B0-like NCHW fp32 feature maps at batch 64, x ~ N(0, 1.5^2),
dy ~ N(0, 1), alpha ~ U(0.5, 2): dx element by element and d alpha against
the oracle's serial long-double sum (|g - r| <= 1e-5 |r|), bitwise
run-to-run determinism, small and ragged sizes, and the workspace contract
(the completion counter is back at zero after every call).
"""
import numpy as np
import pytest
import torch

import memory_efficient_activation_b200 as mea
import oracle
from _compare import TINY, check, to_f64
from memory_efficient_activation_b200 import synthetic

pytestmark = pytest.mark.gpu


def _dalpha_gpu(x, dy, alpha, ws=None):
    d = torch.empty(1, dtype=torch.float32, device="cuda")
    dx = mea.act_bwd("swish", x, dy, alpha, dparam=d, workspace=ws)
    return dx, d


@pytest.mark.parametrize("shape_index", range(6))
def test_effnet_shapes_full_size(shape_index):
    w = synthetic.effnet_swish_f32(shape_index)
    x, dy = w.x.cuda(), w.dy.cuda()
    dx, d = _dalpha_gpu(x, dy, w.param)
    torch.cuda.synchronize()
    xd, gd = to_f64(w.x), to_f64(w.dy)
    ref = oracle.swish_dalpha(xd, gd, w.param)
    got = float(d.item())
    assert abs(got - ref) <= 1e-5 * abs(ref), (got, ref)
    # dx on a sample of elements
    idx = np.random.Generator(np.random.Philox(key=[201, shape_index])).integers(0, w.n, size=1 << 18)
    rdx = oracle.act_bwd("swish", xd[idx], gd[idx], w.param)
    scale = oracle.act_bwd_scale("swish", xd[idx], gd[idx], w.param)
    check("f32", dx.view(-1)[torch.from_numpy(idx).cuda()].cpu(), rdx, scale=scale, what="effnet dx")


def test_dalpha_bitwise_deterministic():
    w = synthetic.effnet_swish_f32(2)
    x, dy = w.x.cuda(), w.dy.cuda()
    vals = []
    for _ in range(10):
        _, d = _dalpha_gpu(x, dy, w.param)
        vals.append(d.clone())
    torch.cuda.synchronize()
    bits = {int(v.view(torch.int32).item()) for v in vals}
    assert len(bits) == 1, bits


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("n", [0, 1, 5, 8, 4097, 8192 * 3 + 5, 1 << 20])
def test_dalpha_small_and_ragged(dtype, n):
    alpha = 1.3
    xs = synthetic.normal(n, 1.5, 202, synthetic.STREAM_X, dtype)
    gs = synthetic.normal(n, 1.0, 202, synthetic.STREAM_DY, dtype)
    x, dy = xs.cuda(), gs.cuda()
    dx, d = _dalpha_gpu(x, dy, alpha)
    torch.cuda.synchronize()
    xd, gd = to_f64(xs), to_f64(gs)
    ref = oracle.swish_dalpha(xd, gd, alpha)
    got = float(d.item())
    # Relative bound as in the large cases, plus an absolute allowance tied to
    # the size of the terms for tiny sums that may cancel to nearly nothing.
    abs_terms = float(np.sum(np.abs(gd * xd * xd)) * 0.25)
    assert abs(got - ref) <= 1e-5 * abs(ref) + 1e-7 * abs_terms, (got, ref)
    if n:
        check(dtype, dx.cpu(), oracle.act_bwd("swish", xd, gd, alpha),
              scale=oracle.act_bwd_scale("swish", xd, gd, alpha),
              floor=TINY * np.maximum(1, np.abs(gd)), what="dx with dalpha")


def test_dalpha_misaligned_scalar_path():
    n = 70001
    base_x = synthetic.normal(n + 1, 1.5, 203, synthetic.STREAM_X, "bf16").cuda()
    base_g = synthetic.normal(n + 1, 1.0, 203, synthetic.STREAM_DY, "bf16").cuda()
    x, dy = base_x[1:], base_g[1:]             # 2-byte offset: not 16-byte aligned
    dx, d = _dalpha_gpu(x, dy, 0.9)
    torch.cuda.synchronize()
    xd, gd = to_f64(x), to_f64(dy)
    ref = oracle.swish_dalpha(xd, gd, 0.9)
    assert abs(float(d.item()) - ref) <= 1e-5 * abs(ref)


def test_workspace_counter_returns_to_zero_and_alpha_on_device():
    w = synthetic.effnet_swish_f32(4)
    x, dy = w.x.cuda(), w.dy.cuda()
    nbytes = mea.act_bwd_workspace_bytes("swish", w.n, True)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    a = torch.tensor([w.param], dtype=torch.float32, device="cuda")
    d1 = torch.empty(1, dtype=torch.float32, device="cuda")
    d2 = torch.empty(1, dtype=torch.float32, device="cuda")
    mea.act_bwd("swish", x, dy, 0.0, param_dev=a, dparam=d1, workspace=ws)
    assert int(ws[:4].view(torch.int32).item()) == 0
    mea.act_bwd("swish", x, dy, 0.0, param_dev=a, dparam=d2, workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    assert torch.equal(d1, d2)
    ref = oracle.swish_dalpha(to_f64(w.x), to_f64(w.dy), w.param)
    assert abs(float(d1.item()) - ref) <= 1e-5 * abs(ref)


def test_autograd_learnable_alpha():
    torch.manual_seed(0)
    w = synthetic.effnet_swish_f32(5)
    m = mea.MemoryEfficientSwish(alpha=w.param, learnable=True).cuda()
    x = w.x.cuda().requires_grad_(True)
    y = m(x)
    y.backward(w.dy.cuda())
    torch.cuda.synchronize()
    xd, gd = to_f64(w.x), to_f64(w.dy)
    check("f32", y.detach().cpu(), oracle.act_fwd("swish", xd, w.param), what="module fwd")
    check("f32", x.grad.cpu(), oracle.act_bwd("swish", xd, gd, w.param),
          scale=oracle.act_bwd_scale("swish", xd, gd, w.param), what="module dx")
    ref = oracle.swish_dalpha(xd, gd, w.param)
    assert abs(float(m.alpha.grad.item()) - ref) <= 1e-5 * abs(ref)
