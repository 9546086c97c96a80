"""Pins for the oracle's activation family (ReLU, LeakyReLU, sigmoid, tanh,
GELU-erf, GELU-tanh): library routines (numpy, scipy.special, PyTorch CPU
float64 and its autograd), textbook values, identities that tie members to
one another, and finite differences of each forward.

The family is named, with its per-element cost, in "What activations cost,
in memory and in arithmetic" (problem B07, GIVEN); the definitions are the
standard ones.
"""
import math

import numpy as np
import pytest
import scipy.special as sp
import torch
import torch.nn.functional as F

import oracle
from memory_efficient_activation_b200 import synthetic

SMOOTH = ["sigmoid", "tanh", "gelu_erf", "gelu_tanh", "swish"]
ALL = ["relu", "leaky_relu"] + SMOOTH


def _torch_fn(act, param):
    return {
        "relu": lambda t: torch.relu(t),
        "leaky_relu": lambda t: F.leaky_relu(t, negative_slope=param),
        "sigmoid": torch.sigmoid,
        "tanh": torch.tanh,
        "gelu_erf": lambda t: F.gelu(t, approximate="none"),
        "gelu_tanh": lambda t: F.gelu(t, approximate="tanh"),
        "swish": lambda t: t * torch.sigmoid(param * t),
    }[act]


def _param(act):
    return 0.01 if act == "leaky_relu" else 1.0


@pytest.mark.parametrize("act", ALL)
def test_family_matches_torch_float64_forward_and_autograd(act):
    x = synthetic.normal_f64(20000, 3.0, 21, 0)
    x[:4] = [0.0, -0.0, 1e-30, -1e-30]
    dy = synthetic.normal_f64(x.size, 1.0, 21, 1)
    p = _param(act)
    t = torch.from_numpy(x.copy()).requires_grad_(True)
    y = _torch_fn(act, p)(t)
    y.backward(torch.from_numpy(dy))
    # torch evaluates both GELUs as x (1 + erf(.)) / 2 and x (1 + tanh(u)) / 2,
    # which cancel for x << 0; those tails are pinned against scipy's ndtr and
    # (through the shared sigmoid) scipy's expit instead.
    atol = 1e-15 if act in ("gelu_erf", "gelu_tanh") else 1e-300
    np.testing.assert_allclose(oracle.act_fwd(act, x, p), y.detach().numpy(), rtol=2e-14, atol=atol)
    # torch evaluates 1 - s, 1 - tanh^2 and 1 + tanh(u) directly (they cancel
    # where the oracle's forms do not), so the backward comparison carries an
    # absolute floor; for GELU-tanh that cancellation is scaled by x u'(x),
    # up to ~10 on x in [-8, -4].
    atol = 1e-14 if act == "gelu_tanh" else 1e-15
    np.testing.assert_allclose(oracle.act_bwd(act, x, dy, p), t.grad.numpy(), rtol=1e-12, atol=atol)


def test_relu_and_leaky_are_exact_and_kinks():
    x = np.array([-2.5, -0.0, 0.0, 1e-300, 3.75, -1e-300])
    np.testing.assert_array_equal(oracle.act_fwd("relu", x), [0.0, 0.0, 0.0, 1e-300, 3.75, 0.0])
    np.testing.assert_array_equal(oracle.act_fwd("leaky_relu", x, 0.01),
                                  [-2.5 * 0.01, -0.0, 0.0, 1e-300, 3.75, -1e-300 * 0.01])
    # derivative is the predicate x > 0: 0 resp. slope at the kink
    np.testing.assert_array_equal(oracle.act_deriv("relu", x), [0, 0, 0, 1, 1, 0])
    np.testing.assert_array_equal(oracle.act_deriv("leaky_relu", x, 0.01),
                                  [0.01, 0.01, 0.01, 1, 1, 0.01])


def test_sigmoid_against_scipy_expit():
    x = np.linspace(-700.0, 700.0, 30001)   # scipy flushes to 0 below ~-709
    np.testing.assert_allclose(oracle.act_fwd("sigmoid", x), sp.expit(x), rtol=1e-14, atol=0)


def test_tanh_against_numpy_and_sigmoid_identity():
    x = np.linspace(-25.0, 25.0, 20001)
    t = oracle.act_fwd("tanh", x)
    np.testing.assert_allclose(t, np.tanh(x), rtol=1e-15, atol=0)
    # tanh(x) = 2 Sigmoid(2x) - 1 ties the tanh and sigmoid oracles together
    np.testing.assert_allclose(t, 2.0 * oracle.act_fwd("sigmoid", 2.0 * x) - 1.0, rtol=0, atol=4e-16)
    # tanh' = 1 - tanh^2 where that does not cancel
    m = np.abs(x) < 2.0
    np.testing.assert_allclose(oracle.act_deriv("tanh", x)[m], 1.0 - np.tanh(x[m]) ** 2, rtol=1e-13)


def test_gelu_erf_against_scipy_ndtr_and_textbook():
    x = np.linspace(-30.0, 30.0, 24001)
    # The deep tail is ill-conditioned (d log Phi / d log x ~ x^2), so the
    # rounding of x / sqrt 2 alone moves the result by ~x^2 * 1e-16.
    np.testing.assert_allclose(oracle.act_fwd("gelu_erf", x), x * sp.ndtr(x), rtol=1e-12, atol=1e-300)
    # Phi(1) = 0.8413447460685429 (standard normal table)
    assert oracle.act_fwd("gelu_erf", [1.0])[0] == pytest.approx(0.8413447460685429, rel=1e-15)
    assert oracle.act_fwd("gelu_erf", [0.0])[0] == 0.0
    assert oracle.act_deriv("gelu_erf", [0.0])[0] == 0.5
    # erf form: x (1 + erf(x / sqrt 2)) / 2 where that does not cancel
    m = x > -3
    np.testing.assert_allclose(oracle.act_fwd("gelu_erf", x[m]),
                               0.5 * x[m] * (1.0 + sp.erf(x[m] / math.sqrt(2.0))), rtol=1e-12, atol=1e-15)


def test_gelu_tanh_against_tanh_form():
    # The published tanh approximation: x (1 + tanh(sqrt(2/pi)(x + 0.044715 x^3))) / 2.
    x = np.linspace(-6.0, 30.0, 20001)
    u = math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)
    ref = 0.5 * x * (1.0 + np.tanh(u))
    np.testing.assert_allclose(oracle.act_fwd("gelu_tanh", x), ref, rtol=1e-12, atol=1e-15)
    assert oracle.act_fwd("gelu_tanh", [0.0])[0] == 0.0
    assert oracle.act_deriv("gelu_tanh", [0.0])[0] == 0.5


def test_gelu_forms_are_close():
    # The two GELU forms differ by a few 1e-4 at most on the real line.
    x = np.linspace(-10, 10, 200001)
    d = np.max(np.abs(oracle.act_fwd("gelu_erf", x) - oracle.act_fwd("gelu_tanh", x)))
    assert 1e-4 < d < 1e-3


@pytest.mark.parametrize("act", ALL)
def test_odd_part_identities(act):
    x = np.linspace(-9.0, 9.0, 1801)
    p = _param(act)
    d = oracle.act_fwd(act, x, p) - oracle.act_fwd(act, -x, p)
    expect = {
        "relu": x, "gelu_erf": x, "gelu_tanh": x, "swish": x,
        "leaky_relu": (1.0 + p) * x,
        "sigmoid": None, "tanh": 2.0 * np.tanh(x),
    }[act]
    if act == "sigmoid":
        s = oracle.act_fwd(act, x) + oracle.act_fwd(act, -x)
        np.testing.assert_allclose(s, 1.0, rtol=0, atol=3e-16)
    else:
        np.testing.assert_allclose(d, expect, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("act", SMOOTH + ["relu", "leaky_relu"])
def test_derivatives_match_finite_differences(act):
    x = synthetic.normal_f64(600, 2.5, 22, 0)
    x = x[np.abs(x) > 1e-3]                     # away from the ReLU kinks
    p = _param(act)
    h = 1e-5 * np.maximum(1.0, np.abs(x))
    fd = (oracle.act_fwd(act, x + h, p) - oracle.act_fwd(act, x - h, p)) / (2 * h)
    np.testing.assert_allclose(oracle.act_deriv(act, x, p), fd, rtol=1e-7, atol=1e-9)


@pytest.mark.parametrize("act", ALL)
def test_extremes_give_no_nan(act):
    x = np.array([3.3895313892515355e38, -3.3895313892515355e38, 1e30, -1e30, 88.7, -88.7, -104.0])
    p = _param(act)
    assert not np.isnan(oracle.act_fwd(act, x, p)).any()
    assert not np.isnan(oracle.act_bwd(act, x, np.ones_like(x), p)).any()


@pytest.mark.parametrize("act", ALL)
def test_nan_forward_propagates(act):
    y = oracle.act_fwd(act, [np.nan], _param(act))
    assert np.isnan(y[0])


def test_unknown_activation_rejected():
    with pytest.raises(KeyError):
        oracle.act_fwd("softplus", [1.0])
