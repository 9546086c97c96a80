"""GPU parity of mea_act_fwd / mea_act_bwd against the oracle, through the C ABI.

Covers every activation in both storage dtypes: the exhaustive bf16 sweep
(every finite bf16 x, dy in {1, -0.75, 3.5}), dense and random fp32 inputs,
extreme finite values and deep tails, ragged and misaligned sizes with guard
bands around every buffer, exact aliasing, the device-side parameter, and the
full-size transformer-scale workload on sampled outputs.
"""
import numpy as np
import pytest
import torch

import memory_efficient_activation_b200 as mea
import oracle
from _compare import TINY, assert_bf16, assert_f32, check, to_f64
from memory_efficient_activation_b200 import synthetic

pytestmark = pytest.mark.gpu

ACTS = list(synthetic.ACTIVATIONS)
DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def _param(act, alpha=1.0):
    if act == "leaky_relu":
        return float(np.float32(0.01))
    if act == "swish":
        return float(np.float32(alpha))
    return 1.0


def _run(act, x_cpu, dy_cpu, param):
    x = x_cpu.cuda()
    dy = dy_cpu.cuda()
    y = mea.act_fwd(act, x, param)
    dx = mea.act_bwd(act, x, dy, param)
    torch.cuda.synchronize()
    return y.cpu(), dx.cpu()


def _oracle(act, x_cpu, dy_cpu, param):
    xd = to_f64(x_cpu)
    gd = to_f64(dy_cpu)
    return (oracle.act_fwd(act, xd, param), oracle.act_bwd(act, xd, gd, param),
            oracle.act_bwd_scale(act, xd, gd, param), gd)


def _check_pair(act, dtype, x_cpu, dy_cpu, param, what):
    y, dx = _run(act, x_cpu, dy_cpu, param)
    ry, rdx, scale, gd = _oracle(act, x_cpu, dy_cpu, param)
    floor = TINY * np.maximum(1.0, np.abs(gd))
    a = check(dtype, y, ry, what=f"{what} fwd")
    b = check(dtype, dx, rdx, scale=scale, floor=floor, what=f"{what} bwd")
    return a, b


@pytest.mark.parametrize("act", ACTS)
@pytest.mark.parametrize("g", [1.0, -0.75, 3.5])
def test_bf16_exhaustive(act, g):
    x = synthetic.all_finite_bf16()
    dy = torch.full_like(x, g)
    _check_pair(act, "bf16", x, dy, _param(act), f"{act} bf16 all x, dy={g}")


@pytest.mark.parametrize("alpha", [0.5, 2.0, 1.7])
def test_bf16_exhaustive_swish_alpha(alpha):
    x = synthetic.all_finite_bf16()
    dy = torch.full_like(x, -0.75)
    _check_pair("swish", "bf16", x, dy, _param("swish", alpha), f"swish alpha={alpha}")


@pytest.mark.parametrize("act", ACTS)
def test_f32_dense_grid(act):
    x = synthetic.f32_grid(1 << 22, -30.0, 30.0)
    dy = synthetic.normal(x.numel(), 1.0, 101, synthetic.STREAM_DY, "f32")
    _check_pair(act, "f32", x, dy, _param(act), f"{act} f32 grid")


@pytest.mark.parametrize("act", ACTS)
def test_f32_random(act):
    x = synthetic.normal(1 << 21, 4.0, 102, synthetic.STREAM_X, "f32")
    dy = synthetic.normal(x.numel(), 1.0, 102, synthetic.STREAM_DY, "f32")
    _check_pair(act, "f32", x, dy, _param(act), f"{act} f32 random")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("act", ACTS)
def test_tails_and_extremes(act, dtype):
    # (the largest finite value used is bf16's, so that it stays finite in
    # both storage dtypes)
    parts = [np.linspace(-110.0, -80.0, 20001), np.linspace(-16.0, -8.0, 20001),
             np.linspace(80.0, 110.0, 20001),
             np.linspace(40.0, 46.0, 2001), -np.linspace(40.0, 46.0, 2001),
             np.array([3.3895313892515355e38, -3.3895313892515355e38, 1e30, -1e30, 1e10, -1e10,
                       1.1754943508222875e-38, -1.1754943508222875e-38, 1e-40, -1e-40, 0.0, -0.0])]
    x = synthetic.to_storage(np.concatenate(parts), dtype)
    dy = synthetic.to_storage(np.resize(np.array([1.0, -0.75, 3.5, -2.0]), x.numel()), dtype)
    _check_pair(act, dtype, x, dy, _param(act), f"{act} {dtype} tails")


@pytest.mark.parametrize("alpha", [0.5, 2.0, 1.3])
def test_swish_alpha_f32(alpha):
    x = synthetic.normal(1 << 20, 3.0, 103, synthetic.STREAM_X, "f32")
    dy = synthetic.normal(x.numel(), 1.0, 103, synthetic.STREAM_DY, "f32")
    _check_pair("swish", "f32", x, dy, _param("swish", alpha), f"swish f32 alpha={alpha}")


def test_swish_f32_1m_workload():
    w = synthetic.swish_f32_1m()
    a, b = _check_pair("swish", "f32", w.x, w.dy, 1.0, "swish f32 1M")
    # pure relative error stays small for the forward
    assert a["max_pure_rel"] < 1e-5


def _guarded(n, dtype, offset_bytes, fill):
    """A tensor view of n elements starting offset_bytes into a buffer that has
    256 guard bytes on either side, filled with a canary pattern."""
    es = torch.tensor([], dtype=DT[dtype]).element_size()
    raw = torch.full((n * es + 512 + offset_bytes,), fill, dtype=torch.uint8, device="cuda")
    start = 256 + offset_bytes
    view = raw[start:start + n * es].view(DT[dtype])
    return raw, view, start, start + n * es


def _guards_intact(raw, start, end, fill):
    r = raw.cpu().numpy()
    return bool(np.all(r[:start] == fill) and np.all(r[end:] == fill))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("n", [0, 1, 7, 8, 9, 31, 4095, 4097, (1 << 20) + 3])
@pytest.mark.parametrize("offset", [0, 2, 4, 16])
def test_ragged_misaligned_guarded(dtype, n, offset):
    if dtype == "f32" and offset == 2:
        pytest.skip("fp32 elements are 4-byte aligned")
    act = "swish"
    xs = synthetic.normal(n, 3.0, 104, synthetic.STREAM_X, dtype)
    gs = synthetic.normal(n, 1.0, 104, synthetic.STREAM_DY, dtype)
    bx, x, sx, ex = _guarded(n, dtype, offset, 0xA5)
    bg, dy, sg, eg = _guarded(n, dtype, offset, 0x5A)
    by, y, sy, ey = _guarded(n, dtype, offset, 0xC3)
    bd, dx, sd, ed = _guarded(n, dtype, offset, 0x3C)
    x.copy_(xs)
    dy.copy_(gs)
    mea.act_fwd(act, x, 1.0, out=y)
    mea.act_bwd(act, x, dy, 1.0, out=dx)
    torch.cuda.synchronize()
    for raw, s, e, f in ((bx, sx, ex, 0xA5), (bg, sg, eg, 0x5A), (by, sy, ey, 0xC3), (bd, sd, ed, 0x3C)):
        assert _guards_intact(raw, s, e, f), "a kernel wrote outside its buffer"
    if n:
        ry, rdx, scale, gd = _oracle(act, xs, gs, 1.0)
        check(dtype, y.cpu(), ry, what="ragged fwd")
        check(dtype, dx.cpu(), rdx, scale=scale, floor=TINY * np.maximum(1, np.abs(gd)), what="ragged bwd")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_in_place_backward(dtype):
    xs = synthetic.normal(100003, 2.0, 105, synthetic.STREAM_X, dtype)
    gs = synthetic.normal(100003, 1.0, 105, synthetic.STREAM_DY, dtype)
    x, dy = xs.cuda(), gs.cuda()
    mea.act_bwd("gelu_tanh", x, dy, out=dy)       # dx aliases dy
    torch.cuda.synchronize()
    ry, rdx, scale, gd = _oracle("gelu_tanh", xs, gs, 1.0)
    check(dtype, dy.cpu(), rdx, scale=scale, floor=TINY * np.maximum(1, np.abs(gd)), what="in place")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_param_on_device(dtype):
    xs = synthetic.normal(50000, 2.0, 106, synthetic.STREAM_X, dtype)
    gs = synthetic.normal(50000, 1.0, 106, synthetic.STREAM_DY, dtype)
    x, dy = xs.cuda(), gs.cuda()
    a = torch.tensor([1.75], dtype=torch.float32, device="cuda")
    y = mea.act_fwd("swish", x, 123.0, param_dev=a)      # the device value wins
    dx = mea.act_bwd("swish", x, dy, 123.0, param_dev=a)
    torch.cuda.synchronize()
    ry, rdx, scale, gd = _oracle("swish", xs, gs, 1.75)
    check(dtype, y.cpu(), ry, what="param_dev fwd")
    check(dtype, dx.cpu(), rdx, scale=scale, floor=TINY * np.maximum(1, np.abs(gd)), what="param_dev bwd")


def test_transformer_scale_bf16_sampled():
    # The full [8, 2048, 4096] bf16 workload in the launch configuration the
    # benchmark times, checked on 2^21 sampled outputs.
    w = synthetic.swish_bf16_transformer()
    x, dy = w.x.cuda(), w.dy.cuda()
    y = mea.act_fwd("swish", x)
    dx = mea.act_bwd("swish", x, dy)
    torch.cuda.synchronize()
    idx = torch.from_numpy(np.random.Generator(np.random.Philox(key=[107, 0]))
                           .integers(0, w.n, size=1 << 21))
    idx = torch.cat([idx, torch.arange(w.n - 64, w.n), torch.arange(0, 64)])
    xs, gs = w.x.view(-1)[idx], w.dy.view(-1)[idx]
    ry, rdx, _, _ = _oracle("swish", xs, gs, 1.0)
    assert_bf16(y.view(-1)[idx.cuda()].cpu(), ry, what="67M fwd sampled")
    assert_bf16(dx.view(-1)[idx.cuda()].cpu(), rdx, what="67M bwd sampled")


@pytest.mark.parametrize("act", ACTS)
def test_family_full_size_sampled(act):
    w = synthetic.family_bf16(act)
    x, dy = w.x.cuda(), w.dy.cuda()
    y = mea.act_fwd(act, x, _param(act))
    dx = mea.act_bwd(act, x, dy, _param(act))
    torch.cuda.synchronize()
    idx = torch.from_numpy(np.random.Generator(np.random.Philox(key=[108, 0]))
                           .integers(0, w.n, size=1 << 19))
    xs, gs = w.x.view(-1)[idx], w.dy.view(-1)[idx]
    ry, rdx, _, _ = _oracle(act, xs, gs, _param(act))
    assert_bf16(y.view(-1)[idx.cuda()].cpu(), ry, what=f"{act} 67M fwd sampled")
    assert_bf16(dx.view(-1)[idx.cuda()].cpu(), rdx, floor=TINY * np.maximum(1, np.abs(to_f64(gs))),
                what=f"{act} 67M bwd sampled")


def test_outputs_deterministic():
    w = synthetic.swish_f32_1m(seed=9)
    x, dy = w.x.cuda(), w.dy.cuda()
    a = [mea.act_bwd("gelu_erf", x, dy).cpu() for _ in range(3)]
    assert all(torch.equal(a[0], t) for t in a[1:])


@pytest.mark.parametrize("n,chunks", [(1 << 20, 8), (1000003, 5), (300, 8)])
def test_host_pipelined_matches_device_calls(n, chunks):
    # act_fwd_bwd_host splits the tensor over streams; every element goes
    # through the same kernels, so the results equal the device calls bitwise
    x = synthetic.normal(n, 2.0, 91, synthetic.STREAM_X, "bf16")
    dy = synthetic.normal(n, 1.0, 91, synthetic.STREAM_DY, "bf16")
    hy, hdx = mea.act_fwd_bwd_host("gelu_tanh", x.pin_memory(), dy.pin_memory(), 1.0, chunks=chunks)
    torch.cuda.synchronize()
    y = mea.act_fwd("gelu_tanh", x.cuda())
    dx = mea.act_bwd("gelu_tanh", x.cuda(), dy.cuda())
    torch.cuda.synchronize()
    assert torch.equal(hy, y.cpu()) and torch.equal(hdx, dx.cpu())


# The zero of Swish'(v), v = alpha x: v0 = -(1 + W(1/e)).
SWISH_V0 = -1.2784645427610737951


@pytest.mark.parametrize("x0", [-1.0, -1.5, -0.75, -2.5, -0.3125])
def test_bf16_swish_alpha_at_zero_of_derivative(x0):
    # alpha = fp32(v0 / x0) puts alpha x0 within an fp32 rounding of the zero
    # of f' (|f'| ~ 1e-8 there), and every other bf16 x is swept as well: the
    # backward must still be within one bf16 ulp of the exact dy f'(x)
    alpha = float(np.float32(SWISH_V0 / x0))
    x = synthetic.all_finite_bf16()
    for g in (1.0, -0.75):
        dy = torch.full_like(x, g)
        _check_pair("swish", "bf16", x, dy, alpha, f"swish alpha={alpha} (zero of f' at x={x0}), dy={g}")
    # the same inputs through the d alpha variant of the backward
    xs = x.cuda()
    dy = torch.full_like(xs, -0.75)
    da = torch.empty(1, dtype=torch.float32, device="cuda")
    dx = mea.act_bwd("swish", xs, dy, alpha, dparam=da)
    torch.cuda.synchronize()
    xd = to_f64(x)
    gd = np.full(xd.size, -0.75)
    check("bf16", dx.cpu(), oracle.act_bwd("swish", xd, gd, alpha), what="swish d alpha variant dx")


@pytest.mark.parametrize("alpha", [1.0, 0.5, -2.0])
def test_bf16_swish_exact_scale_forms_agree(alpha):
    # With alpha = 0 or +-2^k and bf16 x the kernels skip the near-zero test
    # (alpha x is exact there); a device-side alpha always takes the general
    # form.  Both must give the same bits on every finite bf16 x, with and
    # without d alpha.
    x = synthetic.all_finite_bf16().cuda()
    dy = torch.full_like(x, -0.75)
    a_dev = torch.tensor([alpha], dtype=torch.float32, device="cuda")
    dx_host = mea.act_bwd("swish", x, dy, alpha)
    dx_dev = mea.act_bwd("swish", x, dy, 0.0, param_dev=a_dev)
    da_h = torch.empty(1, dtype=torch.float32, device="cuda")
    da_d = torch.empty(1, dtype=torch.float32, device="cuda")
    fin = torch.isfinite(x.float()) & (x.float().abs() < 1e4)
    xs, gs = x[fin].contiguous(), dy[fin].contiguous()
    dxa_h = mea.act_bwd("swish", xs, gs, alpha, dparam=da_h)
    dxa_d = mea.act_bwd("swish", xs, gs, 0.0, param_dev=a_dev, dparam=da_d)
    torch.cuda.synchronize()
    assert torch.equal(dx_host.view(torch.int16), dx_dev.view(torch.int16))
    assert torch.equal(dxa_h.view(torch.int16), dxa_d.view(torch.int16))
    assert torch.equal(da_h, da_d)


@pytest.mark.parametrize("alpha", [1.0, 1.3])
def test_f32_swish_dense_grid_2_26(alpha):
    # 2^26 evenly spaced fp32 values in [-30, 30] (the sweep the survey plans
    # for the fp32 path), dy ~ N(0, 1), checked against the oracle in four
    # chunks of 2^24; the largest errors seen are printed (run with -s)
    n = 1 << 26
    x = synthetic.f32_grid(n, -30.0, 30.0)
    dy = synthetic.normal(n, 1.0, 105, synthetic.STREAM_DY, "f32")
    xc, dyc = x.cuda(), dy.cuda()
    y = mea.act_fwd("swish", xc, alpha).cpu()
    dx = mea.act_bwd("swish", xc, dyc, alpha).cpu()
    del xc, dyc
    worst_fwd = worst_bwd = 0.0
    chunk = 1 << 24
    for c0 in range(0, n, chunk):
        sl = slice(c0, c0 + chunk)
        xd, gd = to_f64(x[sl]), to_f64(dy[sl])
        a = check("f32", y[sl], oracle.act_fwd("swish", xd, alpha), what=f"fwd chunk {c0}")
        b = check("f32", dx[sl], oracle.act_bwd("swish", xd, gd, alpha),
                  scale=oracle.act_bwd_scale("swish", xd, gd, alpha), floor=TINY * np.maximum(1.0, np.abs(gd)),
                  what=f"bwd chunk {c0}")
        worst_fwd = max(worst_fwd, a["max_rel"])
        worst_bwd = max(worst_bwd, b["max_rel"])
    print(f"swish fp32 alpha={alpha}, 2^26 points in [-30, 30]: forward max relative error {worst_fwd:.3e}, "
          f"backward max error / condition scale {worst_bwd:.3e}")
