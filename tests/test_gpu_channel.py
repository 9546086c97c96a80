"""GPU parity of the per-channel operations against the oracle, through the
C ABI: the fused per-channel affine followed by every activation of the
family (mea_affine_act_fwd / mea_affine_act_bwd) and Swish with one learnable
alpha per channel (mea_swish_channel_fwd / mea_swish_channel_bwd).

Small NHWC and NCHW shapes in both dtypes are compared element by element
(shapes that take the NHWC fast path, shapes that leave it, NCHW planes that
are and are not multiples of the vector width); per-channel sums are
compared on every channel (_compare.check_channel_sums).  The full-size
workloads ([128, 56, 56, 144] NHWC bf16 for the affine family, [64, 144, 56,
56] NCHW fp32 for the channel Swish) are compared on every output.  bf16
outputs are held to one ulp of the oracle; fp32 affine outputs to 1e-5 of
their condition scale plus the change that rounding z = gamma x + beta to
fp32 makes to the exact result (oracle.affine_act_zround).  Also: deep tails, alpha of zero and of
either sign, empty batches, bitwise determinism with the workspace counter
returned to zero, agreement of the Swish member with the affine + Swish
entry point, and the autograd modules.
"""
import numpy as np
import pytest
import torch

import memory_efficient_activation_b200 as mea
import oracle
from _compare import TINY, check, check_channel_sums, sum_weights_f32, to_f64
from memory_efficient_activation_b200 import synthetic

pytestmark = pytest.mark.gpu

ACTS = ["relu", "leaky_relu", "sigmoid", "tanh", "gelu_erf", "gelu_tanh", "swish"]
SHAPES = [
    ("nhwc", (2, 5, 7, 144)), ("nhwc", (2, 3, 5, 12)), ("nhwc", (2, 2, 3, 5)), ("nhwc", (2, 3, 3, 1152)),
    # pipelined backward: tiles beyond whole rounds of its grid plus a partial tile
    ("nhwc", (4, 57, 57, 144)),
    ("nchw", (2, 16, 7, 7)), ("nchw", (2, 8, 4, 8)), ("nchw", (3, 5, 3, 3)), ("nchw", (2, 96, 14, 14)),
    # row path: several planes per vector (1 x 1, 1 x 3), a ragged last block
    ("nchw", (5, 37, 1, 1)), ("nchw", (3, 7, 1, 3)), ("nchw", (3, 201, 7, 7)),
    # plane path (planes above the row path's size): scalar and vector loads
    ("nchw", (2, 3, 33, 33)), ("nchw", (2, 4, 40, 40)),
    # the boundary between them: 1024 elements (row path), 1025 (plane path)
    ("nchw", (2, 5, 32, 32)), ("nchw", (2, 3, 41, 25)),
]


def _param(act):
    return 0.01 if act == "leaky_relu" else (1.25 if act == "swish" else 1.0)


def _nchw(shape_mem, layout):
    if layout == "nhwc":
        N, H, W, C = shape_mem
        return (N, C, H, W)
    return tuple(shape_mem)


def _channels(n, layout, nchw):
    N, C, H, W = nchw
    i = np.arange(n)
    return i % C if layout == "nhwc" else (i // (H * W)) % C


def _inputs(shape_mem, layout, dtype, seed, sigma=1.0):
    n = int(np.prod(shape_mem))
    C = shape_mem[3] if layout == "nhwc" else shape_mem[1]
    x = synthetic.normal(n, sigma, seed, synthetic.STREAM_X, dtype).view(shape_mem)
    dy = synthetic.normal(n, 1.0, seed, synthetic.STREAM_DY, dtype).view(shape_mem)
    g = torch.from_numpy(synthetic.uniform_f64(C, 0.5, 1.5, seed, synthetic.STREAM_GAMMA)).float()
    b = torch.from_numpy(synthetic.normal_f64(C, 0.1, seed, synthetic.STREAM_BETA)).float()
    a = torch.from_numpy(synthetic.uniform_f64(C, 0.5, 2.0, seed, synthetic.STREAM_PARAM)).float()
    return x, dy, g, b, a


def _check_sums_against_dx(dx, x, g, dg, db, ch, C):
    """fp32 only: the channel sums agree with the kernel's own dx (dz = dx /
    gamma_c, each dx one fp32 rounding of gamma_c dz), which checks the
    reduction machinery (every element counted once, in its channel) far
    more tightly than the oracle comparison of the values can.  The kernels
    add at most 16 terms in fp32 before moving to fp64; a sequential fp32 sum
    of k terms errs by at most (k - 1) 2^-24 of the sum of |terms|, so with
    the rounding of each dx the bound is 1.1e-6 of that sum."""
    gg = g.double().numpy()
    dz = to_f64(dx) / gg[ch]
    xd = to_f64(x)
    sb = np.bincount(ch, dz, minlength=C)
    sg = np.bincount(ch, dz * xd, minlength=C)
    tb = np.bincount(ch, np.abs(dz), minlength=C)
    tg = np.bincount(ch, np.abs(dz * xd), minlength=C)
    eb = np.abs(db.cpu().double().numpy() - sb)
    eg = np.abs(dg.cpu().double().numpy() - sg)
    assert np.all(eb <= 1.1e-6 * tb + 1e-30), eb.max()
    assert np.all(eg <= 1.1e-6 * tg + 1e-30), eg.max()


def _affine_compare(act, dtype, layout, shape, x, dy, g, b, y, dx, dg, db):
    nchw = _nchw(shape, layout)
    p = _param(act)
    xd, gd = to_f64(x), to_f64(dy)
    gg, bb = g.double().numpy(), b.double().numpy()
    ry = oracle.affine_act_fwd(act, layout, nchw, xd, gg, bb, p)
    rdx, rdg, rdb, scale = oracle.affine_act_bwd(act, layout, nchw, xd, gd, gg, bb, p)
    # fp32: plus the change of the exact result when z = gamma x + beta is
    # rounded once to fp32 (the configurations compute z in fp32); bf16: the
    # plain ulp rule
    ey, edx = oracle.affine_act_zround(act, layout, nchw, xd, gd, gg, bb, p)
    ch = _channels(xd.size, layout, nchw)
    C = nchw[1]
    check(dtype, y.cpu(), ry, what=f"affine {act} fwd", zround=ey)
    check(dtype, dx.cpu(), rdx, scale=scale, floor=TINY * np.maximum(1, np.abs(gd)), what=f"affine {act} dx",
          zround=edx)
    dz = rdx / gg[ch]
    n_c = xd.size // C if C else 0
    if dtype == "f32":
        # terms with fp32 storage: weights by their condition scale, plus the
        # exact change of z's fp32 rounding (the per-element fp32 rule)
        mz = np.asarray(scale, dtype=np.float64).ravel() / np.abs(gg[ch])
        ez = np.asarray(edx, dtype=np.float64).ravel() / np.abs(gg[ch])
        wg, ag = sum_weights_f32(dz * xd, mz * np.abs(xd), ez * xd)
        wb, ab = sum_weights_f32(dz, mz, ez)
        ag, ab = np.bincount(ch, ag, minlength=C), np.bincount(ch, ab, minlength=C)
    else:
        wg, wb, ag, ab = np.abs(dz * xd), np.abs(dz), None, None
    check_channel_sums(dg, rdg, np.bincount(ch, wg, minlength=C), n_c, f"affine {act} dgamma", extra=ag)
    check_channel_sums(db, rdb, np.bincount(ch, wb, minlength=C), n_c, f"affine {act} dbeta", extra=ab)
    if dtype == "f32":
        _check_sums_against_dx(dx, x, g, dg, db, ch, C)


# ------------------------------------------------------------ affine family

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("layout,shape", SHAPES)
@pytest.mark.parametrize("act", ACTS)
def test_affine_act_small(act, dtype, layout, shape):
    x, dy, g, b, _ = _inputs(shape, layout, dtype, 401)
    p = _param(act)
    y = mea.affine_act_fwd(act, x.cuda(), g.cuda(), b.cuda(), p, layout)
    dx, dg, db = mea.affine_act_bwd(act, x.cuda(), dy.cuda(), g.cuda(), b.cuda(), p, layout)
    torch.cuda.synchronize()
    _affine_compare(act, dtype, layout, shape, x, dy, g, b, y, dx, dg, db)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("act", ACTS)
def test_affine_act_deep_tails(act, dtype):
    # x ~ N(0, 60^2): z reaches the saturated tails and the recompute
    # branches of every activation; beta shifts some channels across zero.
    for layout, shape in [("nhwc", (2, 6, 6, 16)), ("nchw", (2, 16, 6, 6))]:
        x, dy, g, b, _ = _inputs(shape, layout, dtype, 402, sigma=60.0)
        p = _param(act)
        y = mea.affine_act_fwd(act, x.cuda(), g.cuda(), b.cuda(), p, layout)
        dx, dg, db = mea.affine_act_bwd(act, x.cuda(), dy.cuda(), g.cuda(), b.cuda(), p, layout)
        torch.cuda.synchronize()
        _affine_compare(act, dtype, layout, shape, x, dy, g, b, y, dx, dg, db)


@pytest.mark.parametrize("act", ["gelu_erf", "tanh", "leaky_relu"])
def test_affine_act_full_workload(act):
    w = synthetic.affine_act_nhwc(act)
    x, dy = w.x.cuda(), w.dy.cuda()
    g, b = w.extra["gamma"].cuda(), w.extra["beta"].cuda()
    y = mea.affine_act_fwd(act, x, g, b, w.param, "nhwc")
    dx, dg, db = mea.affine_act_bwd(act, x, dy, g, b, w.param, "nhwc")
    torch.cuda.synchronize()
    del x, dy
    _affine_compare(act, "bf16", "nhwc", tuple(w.x.shape), w.x, w.dy, w.extra["gamma"], w.extra["beta"],
                    y, dx, dg, db)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("act", ["gelu_erf", "swish", "relu"])
@pytest.mark.parametrize("shape", [(4, 7, 9, 144), (2, 5, 5, 32), (3, 3, 7, 1152)])
def test_affine_act_nhwc_unaligned(act, dtype, shape):
    # tensors that start 8 bytes past a 16-byte boundary: the NHWC backward
    # then streams with plain loads instead of bulk copies into shared memory
    # (and for fp32, whose 16-byte units need 16-byte alignment, the forward
    # and backward take the plane path); same values either way
    x, dy, g, b, _ = _inputs(shape, "nhwc", dtype, 406)
    n = x.numel()
    off = 4 if dtype == "bf16" else 2
    xb = torch.empty(n + off, dtype=x.dtype, device="cuda")
    gb = torch.empty(n + off, dtype=x.dtype, device="cuda")
    xs, gs = xb[off:].view(shape), gb[off:].view(shape)
    xs.copy_(x.cuda())
    gs.copy_(dy.cuda())
    assert xs.data_ptr() % 16 == 8 and gs.data_ptr() % 16 == 8
    p = _param(act)
    y = mea.affine_act_fwd(act, xs, g.cuda(), b.cuda(), p, "nhwc")
    dx, dg, db = mea.affine_act_bwd(act, xs, gs, g.cuda(), b.cuda(), p, "nhwc")
    torch.cuda.synchronize()
    _affine_compare(act, dtype, "nhwc", shape, x, dy, g, b, y, dx, dg, db)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("layout,shape", [("nhwc", (3, 7, 7, 144)), ("nchw", (3, 40, 7, 7))])
def test_affine_act_swish_matches_affine_swish(dtype, layout, shape):
    # affine + Swish is the Swish member of the family with alpha = 1: the
    # same kernels, so the same bits.
    x, dy, g, b, _ = _inputs(shape, layout, dtype, 403)
    x, dy, g, b = x.cuda(), dy.cuda(), g.cuda(), b.cuda()
    y1 = mea.affine_act_fwd("swish", x, g, b, 1.0, layout)
    y2 = mea.affine_swish_fwd(x, g, b, layout)
    o1 = mea.affine_act_bwd("swish", x, dy, g, b, 1.0, layout)
    o2 = mea.affine_swish_bwd(x, dy, g, b, layout)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    for a, c in zip(o1, o2):
        assert torch.equal(a, c)


@pytest.mark.parametrize("act", ["sigmoid", "gelu_tanh"])
@pytest.mark.parametrize("layout,shape", [("nhwc", (16, 14, 14, 144)), ("nchw", (16, 40, 14, 14)),
                                          # remainder rows after whole rounds of the pipelined grid
                                          ("nhwc", (4, 57, 57, 144))])
def test_affine_act_deterministic_and_counter_reset(act, layout, shape):
    x, dy, g, b, _ = _inputs(shape, layout, "bf16", 404)
    x, dy, g, b = x.cuda(), dy.cuda(), g.cuda(), b.cuda()
    need = mea.affine_act_bwd_workspace_bytes(torch.bfloat16, layout, _nchw(shape, layout))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    outs = [mea.affine_act_bwd(act, x, dy, g, b, 1.0, layout, workspace=ws) for _ in range(4)]
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    assert int(ws[4:8].view(torch.int32).item()) == 0     # no bounded wait expired
    for o in outs[1:]:
        for a, c in zip(outs[0], o):
            assert torch.equal(a, c)


def test_affine_act_module_autograd():
    shape = (4, 8, 8, 144)
    x, dy, g, b, _ = _inputs(shape, "nhwc", "bf16", 405)
    m = mea.MemoryEfficientAffineActivation(144, "gelu_tanh", layout="nhwc").cuda()
    with torch.no_grad():
        m.gamma.copy_(g)
        m.beta.copy_(b)
    xc = x.cuda().requires_grad_(True)
    y = m(xc)
    y.backward(dy.cuda())
    torch.cuda.synchronize()
    _affine_compare("gelu_tanh", "bf16", "nhwc", shape, x, dy, g, b, y.detach(), xc.grad, m.gamma.grad,
                    m.beta.grad)


# ------------------------------------------------------------ channel Swish

def _channel_compare(dtype, layout, shape, x, dy, a, y, dx, da):
    nchw = _nchw(shape, layout)
    xd, gd = to_f64(x), to_f64(dy)
    aa = a.double().numpy()
    ry = oracle.swish_channel_fwd(layout, nchw, xd, aa)
    rdx, rda, scale = oracle.swish_channel_bwd(layout, nchw, xd, gd, aa)
    check(dtype, y.cpu(), ry, what="channel swish fwd")
    check(dtype, dx.cpu(), rdx, scale=scale, floor=TINY * np.maximum(1, np.abs(gd)), what="channel swish dx")
    # |terms| of each channel's sum: dy x^2 s (1 - s) = dy x^2 s Sigmoid(-alpha x)
    ch = _channels(xd.size, layout, nchw)
    t = aa[ch] * xd
    with np.errstate(over="ignore"):
        terms = np.abs(gd * xd * xd) / ((1.0 + np.exp(-t)) * (1.0 + np.exp(t)))
    C = nchw[1]
    check_channel_sums(da, rda, np.bincount(ch, terms, minlength=C), xd.size // C if C else 0, "dalpha")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("layout,shape", SHAPES)
def test_swish_channel_small(dtype, layout, shape):
    x, dy, _, _, a = _inputs(shape, layout, dtype, 411, sigma=1.5)
    y = mea.swish_channel_fwd(x.cuda(), a.cuda(), layout)
    dx, da = mea.swish_channel_bwd(x.cuda(), dy.cuda(), a.cuda(), layout)
    torch.cuda.synchronize()
    _channel_compare(dtype, layout, shape, x, dy, a, y, dx, da)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("layout,shape", [("nhwc", (2, 6, 6, 16)), ("nchw", (2, 16, 6, 6))])
def test_swish_channel_special_alphas_and_tails(dtype, layout, shape):
    # alpha = 0 (Swish is x / 2, d alpha = sum dy x^2 / 4), negative, tiny
    # and large alphas; x ~ N(0, 60^2) reaches the recompute branches.
    x, dy, _, _, _ = _inputs(shape, layout, dtype, 412, sigma=60.0)
    a = torch.tensor([0.0, -1.5, 1e-3, 8.0, 1.0, -0.25, 2.0, 0.5,
                      -8.0, 3.0, 0.125, -1e-3, 1.7, 0.9, -3.0, 4.0], dtype=torch.float32)
    y = mea.swish_channel_fwd(x.cuda(), a.cuda(), layout)
    dx, da = mea.swish_channel_bwd(x.cuda(), dy.cuda(), a.cuda(), layout)
    torch.cuda.synchronize()
    _channel_compare(dtype, layout, shape, x, dy, a, y, dx, da)


def test_swish_channel_full_workload():
    w = synthetic.swish_channel_nchw()
    x, dy, a = w.x.cuda(), w.dy.cuda(), w.extra["alpha"].cuda()
    y = mea.swish_channel_fwd(x, a, "nchw")
    dx, da = mea.swish_channel_bwd(x, dy, a, "nchw")
    torch.cuda.synchronize()
    del x, dy
    _channel_compare("f32", "nchw", tuple(w.x.shape), w.x, w.dy, w.extra["alpha"], y, dx, da)


@pytest.mark.parametrize("shape", [(64, 480, 14, 14), (64, 1152, 7, 7), (64, 240, 28, 28)])
def test_swish_channel_effnet_small_planes(shape):
    # EfficientNet-B0's 28 x 28, 14 x 14 and 7 x 7 stages at batch 64 (the
    # row path: hundreds of blocks of whole planes), every output
    x, dy, _, _, a = _inputs(shape, "nchw", "f32", 416, sigma=1.5)
    y = mea.swish_channel_fwd(x.cuda(), a.cuda(), "nchw")
    dx, da = mea.swish_channel_bwd(x.cuda(), dy.cuda(), a.cuda(), "nchw")
    torch.cuda.synchronize()
    _channel_compare("f32", "nchw", shape, x, dy, a, y, dx, da)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [(3, 40, 7, 7), (2, 24, 14, 14)])
def test_channel_ops_nchw_unaligned(dtype, shape):
    # tensors starting one element past a 16-byte boundary leave the row path
    # for the plane path; both must match the oracle
    x, dy, g, b, a = _inputs(shape, "nchw", dtype, 417, sigma=1.5)
    n = x.numel()
    xb = torch.empty(n + 1, dtype=x.dtype, device="cuda")
    gb = torch.empty(n + 1, dtype=x.dtype, device="cuda")
    xs, gs = xb[1:].view(shape), gb[1:].view(shape)
    xs.copy_(x.cuda())
    gs.copy_(dy.cuda())
    assert xs.data_ptr() % 16 != 0 and gs.data_ptr() % 16 != 0
    y = mea.swish_channel_fwd(xs, a.cuda(), "nchw")
    dx, da = mea.swish_channel_bwd(xs, gs, a.cuda(), "nchw")
    ya = mea.affine_act_fwd("gelu_erf", xs, g.cuda(), b.cuda(), 1.0, "nchw")
    dxa, dg, db = mea.affine_act_bwd("gelu_erf", xs, gs, g.cuda(), b.cuda(), 1.0, "nchw")
    torch.cuda.synchronize()
    _channel_compare(dtype, "nchw", shape, x, dy, a, y, dx, da)
    _affine_compare("gelu_erf", dtype, "nchw", shape, x, dy, g, b, ya, dxa, dg, db)


@pytest.mark.parametrize("layout,shape", [("nhwc", (16, 14, 14, 144)), ("nchw", (16, 40, 14, 14)),
                                          ("nchw", (16, 40, 33, 33))])
def test_swish_channel_deterministic_and_counter_reset(layout, shape):
    x, dy, _, _, a = _inputs(shape, layout, "f32", 413, sigma=1.5)
    x, dy, a = x.cuda(), dy.cuda(), a.cuda()
    need = mea.swish_channel_bwd_workspace_bytes(torch.float32, layout, _nchw(shape, layout))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    outs = [mea.swish_channel_bwd(x, dy, a, layout, workspace=ws) for _ in range(4)]
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    assert int(ws[4:8].view(torch.int32).item()) == 0
    for o in outs[1:]:
        for p, q in zip(outs[0], o):
            assert torch.equal(p, q)


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_channel_ops_empty_batch(layout):
    shape = (0, 4, 4, 16) if layout == "nhwc" else (0, 16, 4, 4)
    x = torch.empty(shape, dtype=torch.float32, device="cuda")
    a = torch.ones(16, device="cuda")
    y = mea.swish_channel_fwd(x, a, layout)
    dx, da = mea.swish_channel_bwd(x, x, a, layout, dalpha=torch.full((16,), 7.0, device="cuda"))
    dx2, dg, db = mea.affine_act_bwd("tanh", x, x, a, a, 1.0, layout,
                                     dgamma=torch.full((16,), 7.0, device="cuda"),
                                     dbeta=torch.full((16,), 7.0, device="cuda"))
    torch.cuda.synchronize()
    assert y.numel() == 0 and dx.numel() == 0 and dx2.numel() == 0
    assert torch.all(da == 0) and torch.all(dg == 0) and torch.all(db == 0)


def test_channel_swish_module_autograd():
    shape = (4, 24, 9, 9)
    x, dy, _, _, a = _inputs(shape, "nchw", "bf16", 414, sigma=1.5)
    m = mea.MemoryEfficientChannelSwish(24, layout="nchw").cuda()
    with torch.no_grad():
        m.alpha.copy_(a)
    xc = x.cuda().requires_grad_(True)
    y = m(xc)
    y.backward(dy.cuda())
    torch.cuda.synchronize()
    _channel_compare("bf16", "nchw", shape, x, dy, a, y.detach(), xc.grad, m.alpha.grad)


# Zeros of f' (v = alpha z for Swish), to double precision.
ROOTS = {"swish": -1.2784645427610737951, "gelu_erf": -0.75179152469356445746, "gelu_tanh": -0.75246142207101625849}


def _near_root_inputs(act, layout, shape, dtype, seed, p):
    """Per channel c: a bf16 value x0_c and beta_c such that z = gamma_c x0_c +
    beta_c lies at a chosen offset, anywhere within 2^-8, of the zero of f'
    (in v = alpha z for Swish): inside and outside the kernels' recompute
    windows (2^-10; 2^-9 for GELU-erf); half the positions of every channel
    hold x0_c, the rest N(0, 1) values."""
    n = int(np.prod(shape))
    C = shape[3] if layout == "nhwc" else shape[1]
    x, dy, g, b, _ = _inputs(shape, layout, dtype, seed)
    x0 = synthetic.to_storage(synthetic.uniform_f64(C, -2.0, 2.0, seed, synthetic.STREAM_PARAM), dtype)
    off = synthetic.uniform_f64(C, -2.0 ** -8, 2.0 ** -8, seed + 1, synthetic.STREAM_PARAM)
    off[: C // 4] = 0.0                      # a quarter of the channels at the zero itself
    z0 = ROOTS[act] / p
    gd = g.double().numpy()
    b = torch.from_numpy(z0 + off / p - gd * x0.double().numpy()).float()
    ch = _channels(n, layout, _nchw(shape, layout))
    flat = x.reshape(-1).clone()
    pos = np.arange(n)
    sel = torch.from_numpy((pos // C if layout == "nhwc" else pos) % 2 == 0)
    flat[sel] = x0[torch.from_numpy(ch)][sel]
    return flat.view(shape), dy, g, b


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("layout,shape", [("nhwc", (4, 6, 6, 144)), ("nhwc", (2, 3, 5, 12)), ("nchw", (4, 16, 9, 9)),
                                          ("nhwc", (3, 5, 5, 20)), ("nhwc", (2, 5, 5, 1152))])
@pytest.mark.parametrize("act", ["swish", "gelu_erf", "gelu_tanh"])
def test_affine_act_near_zero_of_derivative(act, dtype, layout, shape):
    # z lands within 2^-8 of the zero of f' for half the elements: bf16 dx
    # stays within one ulp of the exact result (the kernels recompute those
    # inside their window from a compensated z), fp32 within its rule
    p = _param(act)
    x, dy, g, b = _near_root_inputs(act, layout, shape, dtype, 407, p)
    y = mea.affine_act_fwd(act, x.cuda(), g.cuda(), b.cuda(), p, layout)
    dx, dg, db = mea.affine_act_bwd(act, x.cuda(), dy.cuda(), g.cuda(), b.cuda(), p, layout)
    torch.cuda.synchronize()
    _affine_compare(act, dtype, layout, shape, x, dy, g, b, y, dx, dg, db)


@pytest.mark.parametrize("layout,shape", [("nhwc", (4, 6, 6, 16)), ("nchw", (4, 16, 9, 9))])
def test_swish_channel_bf16_near_zero_of_derivative(layout, shape):
    # alpha_c = fp32(v0 / x0_c) for a bf16 x0_c held by half the positions
    x, dy, _, _, _ = _inputs(shape, layout, "bf16", 415, sigma=1.5)
    C = shape[3] if layout == "nhwc" else shape[1]
    n = x.numel()
    x0 = synthetic.to_storage(synthetic.uniform_f64(C, 0.3, 3.0, 415, synthetic.STREAM_PARAM), "bf16")
    x0 = x0 * torch.where(torch.arange(C) % 2 == 0, -1.0, 1.0).to(x0.dtype)
    a = torch.from_numpy(np.float32(ROOTS["swish"] / x0.double().numpy()).astype(np.float32))
    ch = torch.from_numpy(_channels(n, layout, _nchw(shape, layout)))
    flat = x.reshape(-1).clone()
    pos = np.arange(n)
    sel = torch.from_numpy((pos // C if layout == "nhwc" else pos) % 2 == 0)
    flat[sel] = x0[ch][sel]
    x = flat.view(shape)
    y = mea.swish_channel_fwd(x.cuda(), a.cuda(), layout)
    dx, da = mea.swish_channel_bwd(x.cuda(), dy.cuda(), a.cuda(), layout)
    torch.cuda.synchronize()
    _channel_compare("bf16", layout, shape, x, dy, a, y, dx, da)
