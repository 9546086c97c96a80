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
