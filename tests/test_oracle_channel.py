"""Pins for the oracle's per-channel family: affine + any activation, and Swish
with a per-channel alpha.

Checked against PyTorch CPU float64 autograd with the channel broadcast written
in torch's own indexing (independent of the oracle's flat-index arithmetic), the
affine + Swish oracle (the act = Swish, param = 1 case), the plain activation
oracle (gamma = 1, beta = 0, or all alpha_c equal), and finite differences in
alpha_c.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from memory_efficient_activation_b200 import synthetic

ACTS = list(synthetic.ACTIVATIONS)


def _torch_act(act, t, p):
    return {
        "relu": lambda: torch.relu(t),
        "leaky_relu": lambda: F.leaky_relu(t, negative_slope=p),
        "sigmoid": lambda: torch.sigmoid(t),
        "tanh": lambda: torch.tanh(t),
        "gelu_erf": lambda: F.gelu(t, approximate="none"),
        "gelu_tanh": lambda: F.gelu(t, approximate="tanh"),
        "swish": lambda: t * torch.sigmoid(p * t),
    }[act]()


def _inputs(shape, seed):
    N, C, H, W = shape
    n = N * C * H * W
    return (synthetic.normal_f64(n, 1.5, seed, 0), synthetic.normal_f64(n, 1.0, seed, 1),
            synthetic.uniform_f64(C, 0.5, 1.5, seed, 3), synthetic.normal_f64(C, 0.1, seed, 4))


def _bshape(layout, C):
    return (1, 1, 1, C) if layout == "nhwc" else (1, C, 1, 1)


def _mem(shape, layout):
    N, C, H, W = shape
    return (N, H, W, C) if layout == "nhwc" else shape


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
@pytest.mark.parametrize("act", ACTS)
def test_affine_act_matches_torch(act, layout):
    shape = (2, 6, 3, 5)
    x, dy, g, b = _inputs(shape, 701)
    p = 0.01 if act == "leaky_relu" else (1.3 if act == "swish" else 1.0)
    tx = torch.from_numpy(x.reshape(_mem(shape, layout)).copy()).requires_grad_(True)
    tg = torch.from_numpy(g.copy()).requires_grad_(True)
    tb = torch.from_numpy(b.copy()).requires_grad_(True)
    z = tg.view(_bshape(layout, 6)) * tx + tb.view(_bshape(layout, 6))
    y = _torch_act(act, z, p)
    y.backward(torch.from_numpy(dy.reshape(_mem(shape, layout))))
    ry = oracle.affine_act_fwd(act, layout, shape, x, g, b, p)
    dx, dg, db, scale = oracle.affine_act_bwd(act, layout, shape, x, dy, g, b, p)
    atol = 1e-15 if act.startswith("gelu") else 1e-300
    np.testing.assert_allclose(ry, y.detach().numpy().ravel(), rtol=2e-14, atol=atol)
    np.testing.assert_allclose(dx, tx.grad.numpy().ravel(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dg, tg.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(db, tb.grad.numpy(), rtol=1e-11, atol=1e-12)
    assert np.all(scale >= np.abs(dx) * (1 - 1e-14))


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_affine_act_swish_is_affine_swish(layout):
    shape = (2, 8, 3, 3)
    x, dy, g, b = _inputs(shape, 702)
    np.testing.assert_array_equal(oracle.affine_act_fwd("swish", layout, shape, x, g, b, 1.0),
                                  oracle.affine_swish_fwd(layout, shape, x, g, b))
    a = oracle.affine_act_bwd("swish", layout, shape, x, dy, g, b, 1.0)
    r = oracle.affine_swish_bwd(layout, shape, x, dy, g, b, with_scale=True)
    for u, v in zip(a, r):
        np.testing.assert_array_equal(u, v)


@pytest.mark.parametrize("act", ACTS)
def test_affine_act_identity_is_plain_activation(act):
    shape = (2, 4, 3, 3)
    x, dy, _, _ = _inputs(shape, 703)
    p = 0.01 if act == "leaky_relu" else 1.0
    one, zero = np.ones(4), np.zeros(4)
    np.testing.assert_array_equal(oracle.affine_act_fwd(act, "nchw", shape, x, one, zero, p),
                                  oracle.act_fwd(act, x, p))
    dx, _, _, _ = oracle.affine_act_bwd(act, "nchw", shape, x, dy, one, zero, p)
    np.testing.assert_array_equal(dx, oracle.act_bwd(act, x, dy, p))


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_swish_channel_matches_torch(layout):
    shape = (3, 5, 4, 2)
    x, dy, _, _ = _inputs(shape, 704)
    a = synthetic.uniform_f64(5, 0.5, 2.0, 704, 2)
    tx = torch.from_numpy(x.reshape(_mem(shape, layout)).copy()).requires_grad_(True)
    ta = torch.from_numpy(a.copy()).requires_grad_(True)
    y = tx * torch.sigmoid(ta.view(_bshape(layout, 5)) * tx)
    y.backward(torch.from_numpy(dy.reshape(_mem(shape, layout))))
    np.testing.assert_allclose(oracle.swish_channel_fwd(layout, shape, x, a), y.detach().numpy().ravel(),
                               rtol=2e-14, atol=1e-300)
    dx, da, scale = oracle.swish_channel_bwd(layout, shape, x, dy, a)
    np.testing.assert_allclose(dx, tx.grad.numpy().ravel(), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(da, ta.grad.numpy(), rtol=1e-11, atol=1e-12)
    assert np.all(scale >= np.abs(dx) * (1 - 1e-14))


def test_swish_channel_equal_alphas_reduce_to_scalar_alpha():
    shape = (2, 6, 3, 3)
    x, dy, _, _ = _inputs(shape, 705)
    a = np.full(6, 1.7)
    np.testing.assert_array_equal(oracle.swish_channel_fwd("nchw", shape, x, a), oracle.act_fwd("swish", x, 1.7))
    dx, da, _ = oracle.swish_channel_bwd("nchw", shape, x, dy, a)
    np.testing.assert_array_equal(dx, oracle.act_bwd("swish", x, dy, 1.7))
    assert np.sum(da) == pytest.approx(oracle.swish_dalpha(x, dy, 1.7), rel=1e-12)


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_swish_channel_dalpha_finite_differences(layout):
    shape = (2, 3, 4, 4)
    x, dy, _, _ = _inputs(shape, 706)
    a = synthetic.uniform_f64(3, 0.5, 2.0, 706, 2)
    _, da, _ = oracle.swish_channel_bwd(layout, shape, x, dy, a)
    h = 1e-6
    for c in range(3):
        ap, am = a.copy(), a.copy()
        ap[c] += h
        am[c] -= h
        fd = (np.sum(dy * oracle.swish_channel_fwd(layout, shape, x, ap))
              - np.sum(dy * oracle.swish_channel_fwd(layout, shape, x, am))) / (2 * h)
        assert da[c] == pytest.approx(fd, rel=1e-6, abs=1e-8)


# ------------------------------------------------- z-rounding sensitivity

U = 2.0 ** -24


def _zround_case(act, seed, n=2000, sigma=3.0):
    shape = (1, 4, 1, n // 4)
    x = synthetic.normal_f64(n, sigma, seed, 0)
    dy = synthetic.normal_f64(n, 1.0, seed, 1)
    g = synthetic.uniform_f64(4, 0.5, 1.5, seed, 3)
    b = synthetic.normal_f64(4, 0.1, seed, 4)
    p = 0.01 if act == "leaky_relu" else (1.25 if act == "swish" else 1.0)
    ey, edx = oracle.affine_act_zround(act, "nchw", shape, x, dy, g, b, p)
    ch = np.arange(n) // (n // 4)
    z = g[ch] * x + b[ch]
    return z, dy, g[ch], p, ey, edx


def test_zround_relu_exact_first_order():
    # ReLU is linear on either side of 0: moving z by u|z| moves y by exactly
    # u|z| for z > 0 and not at all for z < 0; f' does not move at all.
    # (the double evaluation of z (1 + u) - z rounds at 2^-53 |z|: 2^-29
    # relative to u |z|)
    z, _, _, _, ey, edx = _zround_case("relu", 901)
    pos, neg = z > 1e-3, z < -1e-3
    assert np.allclose(ey[pos], U * z[pos], rtol=4e-9, atol=0)
    assert np.all(ey[neg] == 0.0)
    assert np.all(edx[np.abs(z) > 1e-3] == 0.0)


def _swish_d2(v, a):
    # second derivative of x Sigmoid(a x): a s (1 - s) (2 + a x (1 - 2 s))
    s = 1.0 / (1.0 + np.exp(-a * v))
    return a * s * (1.0 - s) * (2.0 + a * v * (1.0 - 2.0 * s))


@pytest.mark.parametrize("act", ["swish", "gelu_erf", "tanh", "sigmoid"])
def test_zround_forward_first_order(act):
    # ey = u |z f'(z)| to first order, f' from the oracle's (pinned)
    # derivative; compared where the double differences' own rounding (about
    # 2^-53 |f|) is below 1e-5 of the value
    z, _, _, p, ey, _ = _zround_case(act, 902)
    d1 = oracle.act_deriv(act, z, p)
    f = oracle.act_fwd(act, z, p)
    keep = U * np.abs(d1 * z) > 1e-11 * np.maximum(np.abs(f), 1e-300)
    assert keep.sum() > 1000
    assert np.allclose(ey[keep], U * np.abs(z[keep] * d1[keep]), rtol=1e-4, atol=0)


def test_zround_swish_backward_closed_form():
    z, dy, g, p, _, edx = _zround_case("swish", 903)
    d2 = _swish_d2(z, p)
    ref = U * np.abs(z * g * dy * d2)
    keep = ref > 1e-12
    assert keep.sum() > 1000
    assert np.allclose(edx[keep], ref[keep], rtol=1e-4, atol=0)


def test_zround_gelu_tanh_backward_against_torch_double_backward():
    # f'' of GELU-tanh from torch float64 autograd (grad of grad), independent
    # of the oracle's derivative code
    z, dy, g, p, ey, edx = _zround_case("gelu_tanh", 904, sigma=4.0)
    t = torch.from_numpy(z.copy()).requires_grad_(True)
    y = F.gelu(t, approximate="tanh")
    (d1,) = torch.autograd.grad(y.sum(), t, create_graph=True)
    (d2,) = torch.autograd.grad(d1.sum(), t)
    d2 = d2.detach().numpy()
    ref_dx = U * np.abs(z * g * dy * d2)
    ref_y = U * np.abs(z * d1.detach().numpy())
    # first order holds away from the zeros of f'' and above the double
    # rounding of f' (about 2^-53); torch forms 1 + tanh(u), which cancels
    # below z ~ -5, so it is trusted above that only
    ok_torch = z > -5.0
    keep = (ref_dx > 1e-11 * np.abs(g * dy)) & (np.abs(d2) > 1e-2) & ok_torch
    assert keep.sum() > 1000
    assert np.allclose(edx[keep], ref_dx[keep], rtol=1e-4, atol=0)
    fy = oracle.act_fwd("gelu_tanh", z)
    keep = (ref_y > 1e-11 * np.abs(fy)) & ok_torch
    assert np.allclose(ey[keep], ref_y[keep], rtol=1e-4, atol=0)
    # in the deep tail the relative sensitivity |z f' / f| u exceeds 1e-5: the
    # reason the fp32 tolerance of the affine outputs carries this term
    deep = z < -7.0
    assert deep.sum() > 0
    assert np.max(ey[deep] / np.abs(fy[deep])) > 1e-5


def test_zround_gelu_tanh_deep_tail_against_mpmath():
    # deep negative tail, where torch's 1 + tanh(u) form cancels: ey against
    # the change of x Sigmoid(2u) evaluated with 40 significant digits
    mp = pytest.importorskip("mpmath")
    mp.mp.dps = 40
    z = np.array([-5.5, -7.25, -9.0, -11.5, -13.0])
    n = z.size
    ey, _ = oracle.affine_act_zround("gelu_tanh", "nchw", (1, 1, 1, n), z, np.ones(n), np.ones(1), np.zeros(1))

    def f(v):
        v = mp.mpf(v)
        u = mp.sqrt(2 / mp.pi) * (v + mp.mpf("0.044715") * v ** 3)
        return v / (1 + mp.exp(-2 * u))

    for i, zi in enumerate(z):
        f0 = f(zi)
        ref = max(abs(f(zi * (1 - U)) - f0), abs(f(zi * (1 + U)) - f0))
        assert abs(ey[i] - float(ref)) <= 1e-6 * float(ref), (zi, ey[i], float(ref))
