"""GPU parity of the fused per-channel affine + Swish (mea_affine_swish_fwd /
mea_affine_swish_bwd) against the oracle, through the C ABI.

NHWC [128, 56, 56, 144] bf16 (the full workload: dgamma / dbeta on every
channel, dx on sampled elements), small NHWC and NCHW shapes in both dtypes
(element by element), channel counts that leave the NHWC fast path, NCHW
planes that are not 16-byte multiples, empty batches, bitwise determinism and
the autograd module.
"""
import numpy as np
import pytest
import torch

import memory_efficient_activation_b200 as mea
import oracle
from _compare import TINY, check, check_channel_sums, to_f64
from memory_efficient_activation_b200 import synthetic

pytestmark = pytest.mark.gpu


def _inputs(shape_mem, layout, dtype, seed):
    n = int(np.prod(shape_mem))
    C = shape_mem[3] if layout == "nhwc" else shape_mem[1]
    x = synthetic.normal(n, 1.0, seed, synthetic.STREAM_X, dtype).view(shape_mem)
    dy = synthetic.normal(n, 1.0, seed, synthetic.STREAM_DY, dtype).view(shape_mem)
    g = torch.from_numpy(synthetic.uniform_f64(C, 0.5, 1.5, seed, synthetic.STREAM_GAMMA)).float()
    b = torch.from_numpy(synthetic.normal_f64(C, 0.1, seed, synthetic.STREAM_BETA)).float()
    return x, dy, g, b


def _nchw(shape_mem, layout):
    if layout == "nhwc":
        N, H, W, C = shape_mem
        return (N, C, H, W)
    return tuple(shape_mem)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("layout,shape", [
    ("nhwc", (2, 5, 7, 144)), ("nhwc", (3, 4, 4, 16)), ("nhwc", (1, 3, 3, 8)),
    ("nhwc", (2, 3, 5, 12)), ("nhwc", (2, 2, 3, 5)), ("nhwc", (4, 9, 9, 1152)),
    # pipelined backward: more tiles than its 296 blocks, not a multiple of
    # them, and a partial tile (a remainder of 441 rows of 288 units)
    ("nhwc", (4, 57, 57, 144)),
    ("nchw", (2, 16, 7, 7)), ("nchw", (2, 8, 4, 8)), ("nchw", (3, 5, 3, 3)),
    ("nchw", (4, 32, 28, 28)), ("nchw", (2, 1152, 7, 7)),
])
def test_affine_small_shapes(dtype, layout, shape):
    x, dy, g, b = _inputs(shape, layout, dtype, 301)
    nchw = _nchw(shape, layout)
    y = mea.affine_swish_fwd(x.cuda(), g.cuda(), b.cuda(), layout)
    dx, dg, db = mea.affine_swish_bwd(x.cuda(), dy.cuda(), g.cuda(), b.cuda(), layout)
    torch.cuda.synchronize()
    xd, gd = to_f64(x), to_f64(dy)
    ry = oracle.affine_swish_fwd(layout, nchw, xd, g.double().numpy(), b.double().numpy())
    rdx, rdg, rdb, scale = oracle.affine_swish_bwd(layout, nchw, xd, gd, g.double().numpy(),
                                                   b.double().numpy(), with_scale=True)
    ey, edx = oracle.affine_act_zround("swish", layout, nchw, xd, gd, g.double().numpy(), b.double().numpy(), 1.0)
    check(dtype, y.cpu(), ry, what="affine fwd", zround=ey)
    check(dtype, dx.cpu(), rdx, scale=scale, floor=TINY * np.maximum(1, np.abs(gd)), what="affine dx", zround=edx)
    N, C, H, W = nchw
    ch = np.arange(xd.size)
    ch = ch % C if layout == "nhwc" else (ch // (H * W)) % C
    dz = rdx / g.double().numpy()[ch]
    tg = np.bincount(ch, np.abs(dz * xd), minlength=C)
    tb = np.bincount(ch, np.abs(dz), minlength=C)
    check_channel_sums(dg, rdg, tg, N * H * W, "dgamma")
    check_channel_sums(db, rdb, tb, N * H * W, "dbeta")


def test_affine_nhwc_full_workload():
    w = synthetic.affine_swish_nhwc()
    x, dy = w.x.cuda(), w.dy.cuda()
    g, b = w.extra["gamma"].cuda(), w.extra["beta"].cuda()
    y = mea.affine_swish_fwd(x, g, b, "nhwc")
    dx, dg, db = mea.affine_swish_bwd(x, dy, g, b, "nhwc")
    torch.cuda.synchronize()
    nchw = w.extra["nchw_shape"]
    xd, gd = to_f64(w.x), to_f64(w.dy)
    gg, bb = w.extra["gamma"].double().numpy(), w.extra["beta"].double().numpy()
    rdx, rdg, rdb, scale = oracle.affine_swish_bwd("nhwc", nchw, xd, gd, gg, bb, with_scale=True)
    # 1e-5 relative per channel, plus 1e-8 of the channel's sum of |terms|
    # for a channel whose 401,408 terms happen to cancel to a small total.
    C = nchw[1]
    ch = np.arange(xd.size) % C
    dz = rdx / gg[ch]
    tg = np.bincount(ch, np.abs(dz * xd), minlength=C)
    tb = np.bincount(ch, np.abs(dz), minlength=C)
    rg = check_channel_sums(dg, rdg, tg, xd.size // C, "dgamma")
    rb = check_channel_sums(db, rdb, tb, xd.size // C, "dbeta")
    print(f"dgamma {rg}, dbeta {rb}")
    idx = np.random.Generator(np.random.Philox(key=[302, 0])).integers(0, w.n, size=1 << 20)
    idx_t = torch.from_numpy(idx).cuda()
    ry = oracle.affine_swish_fwd("nhwc", nchw, xd, gg, bb)
    check("bf16", y.view(-1)[idx_t].cpu(), ry[idx], what="nhwc fwd sampled")
    check("bf16", dx.view(-1)[idx_t].cpu(), rdx[idx], scale=scale[idx], what="nhwc dx sampled")


def test_affine_deterministic_and_counter_reset():
    x, dy, g, b = _inputs((16, 14, 14, 144), "nhwc", "bf16", 303)
    x, dy, g, b = x.cuda(), dy.cuda(), g.cuda(), b.cuda()
    need = mea.affine_swish_bwd_workspace_bytes(torch.bfloat16, "nhwc", (16, 144, 14, 14))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    outs = [mea.affine_swish_bwd(x, dy, g, b, "nhwc", workspace=ws) for _ in range(5)]
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    for o in outs[1:]:
        for a, c in zip(outs[0], o):
            assert torch.equal(a, c)


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_affine_empty_batch(layout):
    shape = (0, 4, 4, 16) if layout == "nhwc" else (0, 16, 4, 4)
    x = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    g = torch.ones(16, device="cuda")
    b = torch.zeros(16, device="cuda")
    y = mea.affine_swish_fwd(x, g, b, layout)
    dx, dg, db = mea.affine_swish_bwd(x, x, g, b, layout,
                                      dgamma=torch.full((16,), 7.0, device="cuda"),
                                      dbeta=torch.full((16,), 7.0, device="cuda"))
    torch.cuda.synchronize()
    assert y.numel() == 0 and dx.numel() == 0
    assert torch.all(dg == 0) and torch.all(db == 0)


def test_affine_module_autograd():
    x, dy, g, b = _inputs((4, 8, 8, 144), "nhwc", "bf16", 304)
    m = mea.MemoryEfficientAffineSwish(144, "nhwc").cuda()
    with torch.no_grad():
        m.gamma.copy_(g)
        m.beta.copy_(b)
    xc = x.cuda().requires_grad_(True)
    y = m(xc)
    y.backward(dy.cuda())
    torch.cuda.synchronize()
    xd, gd = to_f64(x), to_f64(dy)
    rdx, rdg, rdb, scale = oracle.affine_swish_bwd("nhwc", (4, 144, 8, 8), xd, gd, g.double().numpy(),
                                                   b.double().numpy(), with_scale=True)
    check("bf16", xc.grad.cpu(), rdx, scale=scale, what="module dx")
    ch = np.arange(xd.size) % 144
    dz = rdx / g.double().numpy()[ch]
    tg = np.bincount(ch, np.abs(dz * xd), minlength=144)
    tb = np.bincount(ch, np.abs(dz), minlength=144)
    check_channel_sums(m.gamma.grad, rdg, tg, 4 * 8 * 8, "dgamma")
    check_channel_sums(m.beta.grad, rdb, tb, 4 * 8 * 8, "dbeta")
