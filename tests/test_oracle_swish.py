"""Pins for the oracle's Swish forward, backward and d alpha.

Each check ties the oracle to something other than itself: closed forms and
identities of x * Sigmoid(alpha x), the backward expression printed in
"Memory efficient Swish" (section "How is the memory efficient version Swish
implemented?"), PyTorch's own CPU float64 silu / sigmoid and autograd, and
central finite differences of the oracle's forward.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from memory_efficient_activation_b200 import synthetic

ALPHAS = [1.0, 0.5, 2.0, 1.7, -0.8]


def _x(n=2001, lim=12.0):
    return np.linspace(-lim, lim, n)


def test_swish_zero():
    for a in ALPHAS:
        assert oracle.act_fwd("swish", [0.0], a)[0] == 0.0


@pytest.mark.parametrize("alpha", ALPHAS)
def test_swish_odd_part_identity(alpha):
    # x s(ax) - (-x) s(-ax) = x (s(ax) + s(-ax)) = x for every alpha.
    x = _x()
    d = oracle.act_fwd("swish", x, alpha) - oracle.act_fwd("swish", -x, alpha)
    np.testing.assert_allclose(d, x, rtol=1e-14, atol=1e-300)


@pytest.mark.parametrize("alpha", ALPHAS)
def test_swish_scaling(alpha):
    # Swish_a(x) = Swish_1(a x) / a.
    x = _x()
    lhs = oracle.act_fwd("swish", x, alpha)
    rhs = oracle.act_fwd("swish", alpha * x, 1.0) / alpha
    np.testing.assert_allclose(lhs, rhs, rtol=1e-13, atol=1e-300)


def test_swish_alpha_zero_is_half_x():
    x = _x()
    np.testing.assert_array_equal(oracle.act_fwd("swish", x, 0.0), x / 2)


def test_swish_large_alpha_tends_to_relu():
    x = np.array([-3.0, -0.5, 0.25, 2.0])
    y = oracle.act_fwd("swish", x, 1e6)
    np.testing.assert_allclose(y, np.maximum(x, 0.0), atol=1e-300, rtol=1e-14)


def test_swish_limits():
    big = np.array([10.0, 30.0, 3.4028234663852886e38, 1e300])
    y = oracle.act_fwd("swish", big)
    assert abs(y[0] - 10.0) < 10 * 5e-5          # 10 (1 - ~4.5e-5)
    assert y[1] == pytest.approx(30.0, rel=1e-12)
    assert y[2] == 3.4028234663852886e38
    assert y[3] == 1e300
    y = oracle.act_fwd("swish", -big)
    assert -1e-3 < y[0] < 0.0
    assert -1e-11 < y[1] < 0.0
    assert y[2] == 0.0 and y[3] == 0.0
    assert not np.isnan(oracle.act_bwd("swish", -big, np.ones(4))).any()
    assert not np.isnan(oracle.act_bwd("swish", big, np.ones(4))).any()


def _lambert_w(z, w0=0.5):
    # Principal branch by Newton's method on w e^w - z.
    w = w0
    for _ in range(100):
        f = w * math.exp(w) - z
        w_new = w - f / (math.exp(w) * (w + 1))
        if abs(w_new - w) < 1e-17:
            break
        w = w_new
    return w


@pytest.mark.parametrize("alpha", [1.0, 0.5, 2.0])
def test_swish_minimum_lambert(alpha):
    # The minimum of x s(ax) is at x* = -(1 + W(1/e)) / a with value -W(1/e) / a.
    w = _lambert_w(1.0 / math.e)
    assert w == pytest.approx(0.2784645427610738, rel=1e-15)
    xs = -(1.0 + w) / alpha
    assert oracle.act_fwd("swish", [xs], alpha)[0] == pytest.approx(-w / alpha, rel=1e-14)
    assert abs(oracle.act_deriv("swish", [xs], alpha)[0]) < 1e-15
    # and it is a minimum
    h = 1e-3 / alpha
    y = oracle.act_fwd("swish", [xs - h, xs, xs + h], alpha)
    assert y[1] < y[0] and y[1] < y[2]


@pytest.mark.parametrize("alpha", ALPHAS)
def test_swish_derivative_at_zero(alpha):
    # f'(0) = 1/2 for every alpha; f''(0) = alpha / 2.
    assert oracle.act_deriv("swish", [0.0], alpha)[0] == 0.5
    h = 1e-5
    d2 = (oracle.act_deriv("swish", [h], alpha)[0]
          - oracle.act_deriv("swish", [-h], alpha)[0]) / (2 * h)
    assert d2 == pytest.approx(alpha / 2, rel=1e-8, abs=1e-10)


@pytest.mark.parametrize("alpha", ALPHAS)
def test_swish_derivative_symmetry(alpha):
    # d/dx of the odd-part identity: f'(x) + f'(-x) = 1.
    x = _x()
    s = oracle.act_deriv("swish", x, alpha) + oracle.act_deriv("swish", -x, alpha)
    np.testing.assert_allclose(s, 1.0, rtol=0, atol=2e-15)


@pytest.mark.parametrize("alpha", ALPHAS)
def test_swish_derivative_matches_finite_differences(alpha):
    x = synthetic.normal_f64(400, 3.0, 11, 0)
    h = 1e-5 * np.maximum(1.0, np.abs(x))
    fd = (oracle.act_fwd("swish", x + h, alpha) - oracle.act_fwd("swish", x - h, alpha)) / (2 * h)
    d = oracle.act_deriv("swish", x, alpha)
    np.testing.assert_allclose(d, fd, rtol=1e-7, atol=1e-9)


def test_swish_backward_matches_page_expression():
    # The page's backward at alpha = 1: grad * s * (1 + x * (1 - s)).
    x = _x(4001, 20.0)
    dy = synthetic.normal_f64(x.size, 1.0, 12, 1)
    s = 1.0 / (1.0 + np.exp(-x))
    page = dy * (s * (1.0 + x * (1.0 - s)))
    np.testing.assert_allclose(oracle.act_bwd("swish", x, dy, 1.0), page, rtol=1e-10, atol=1e-14)


def test_swish_matches_torch_silu_float64():
    x = synthetic.normal_f64(5000, 4.0, 13, 0)
    t = torch.from_numpy(x.copy()).requires_grad_(True)
    y = torch.nn.functional.silu(t)
    dy = synthetic.normal_f64(x.size, 1.0, 13, 1)
    y.backward(torch.from_numpy(dy))
    np.testing.assert_allclose(oracle.act_fwd("swish", x), y.detach().numpy(), rtol=1e-14, atol=1e-300)
    np.testing.assert_allclose(oracle.act_bwd("swish", x, dy), t.grad.numpy(), rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("alpha", [0.5, 1.3, 2.0])
def test_swish_alpha_against_torch_autograd(alpha):
    # x * sigmoid(alpha x) through torch float64 autograd: dx and d alpha.
    x = synthetic.normal_f64(3000, 1.5, 14, 0)
    dy = synthetic.normal_f64(3000, 1.0, 14, 1)
    tx = torch.from_numpy(x.copy()).requires_grad_(True)
    ta = torch.tensor(alpha, dtype=torch.float64, requires_grad=True)
    y = tx * torch.sigmoid(ta * tx)
    y.backward(torch.from_numpy(dy))
    np.testing.assert_allclose(oracle.act_fwd("swish", x, alpha), y.detach().numpy(), rtol=1e-14)
    np.testing.assert_allclose(oracle.act_bwd("swish", x, dy, alpha), tx.grad.numpy(),
                               rtol=1e-12, atol=1e-15)
    da = oracle.swish_dalpha(x, dy, alpha)
    assert da == pytest.approx(float(ta.grad), rel=1e-11, abs=1e-12)


@pytest.mark.parametrize("alpha", [0.5, 1.0, 1.9])
def test_swish_dalpha_matches_finite_difference_in_alpha(alpha):
    # d/d alpha of L(alpha) = sum dy * Swish_alpha(x).
    x = synthetic.normal_f64(2000, 1.5, 15, 0)
    dy = synthetic.normal_f64(2000, 1.0, 15, 1)
    h = 1e-6

    def L(a):
        return float(np.sum(dy * oracle.act_fwd("swish", x, a)))

    fd = (L(alpha + h) - L(alpha - h)) / (2 * h)
    assert oracle.swish_dalpha(x, dy, alpha) == pytest.approx(fd, rel=1e-6, abs=1e-8)


def test_swish_dalpha_brute_force_small():
    # Element-by-element sum with Python floats (no vectorisation).
    x = synthetic.normal_f64(300, 1.5, 16, 0)
    dy = synthetic.normal_f64(300, 1.0, 16, 1)
    a = 1.25
    tot = 0.0
    for xi, gi in zip(x.tolist(), dy.tolist()):
        s = 1.0 / (1.0 + math.exp(-a * xi))
        tot += gi * xi * xi * s * (1.0 - s)
    assert oracle.swish_dalpha(x, dy, a) == pytest.approx(tot, rel=1e-12, abs=1e-14)


def test_swish_dalpha_empty_and_zero():
    assert oracle.swish_dalpha(np.zeros(0), np.zeros(0), 1.0) == 0.0
    # x = 0 contributes nothing.
    assert oracle.swish_dalpha(np.zeros(10), np.ones(10), 1.0) == 0.0


def test_swish_nan_propagates():
    x = np.array([np.nan, 1.0])
    y = oracle.act_fwd("swish", x)
    assert np.isnan(y[0]) and not np.isnan(y[1])
    dx = oracle.act_bwd("swish", x, np.ones(2))
    assert np.isnan(dx[0]) and not np.isnan(dx[1])


@pytest.mark.parametrize("act", ["swish", "gelu_erf", "gelu_tanh", "sigmoid", "tanh", "relu", "leaky_relu"])
def test_bwd_scale_bounds_and_equalities(act):
    # The condition scale is |dy| times the sum of |terms| of f': never below
    # |dx|, equal to it wherever the terms share a sign (x >= 0 here for all
    # members), and strictly above it where they cancel.
    x = np.linspace(-8.0, 8.0, 3201)
    dy = synthetic.normal_f64(x.size, 1.0, 17, 1)
    p = 0.01 if act == "leaky_relu" else 1.0
    m = oracle.act_bwd_scale(act, x, dy, p)
    dx = np.abs(oracle.act_bwd(act, x, dy, p))
    assert np.all(m >= dx * (1 - 1e-15))
    pos = x >= 0
    np.testing.assert_allclose(m[pos], dx[pos], rtol=1e-14, atol=0)
    if act in ("swish", "gelu_erf", "gelu_tanh"):
        # at the zero of f' the scale stays finite and positive
        assert np.all(m[(x < -0.5) & (x > -2.0)] > 0.1 * np.abs(dy[(x < -0.5) & (x > -2.0)]))
