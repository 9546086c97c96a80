"""Pins for the oracle's concatenation + batch normalization + ReLU ("A
memory-efficient implementation of DenseNets", section "Motivation").

Checked against PyTorch CPU float64 (torch.cat, F.batch_norm in training mode
and torch.relu, with autograd for the backward), a small example worked by
hand, and the invariants of batch normalization: with every output above the
ReLU threshold, each channel of the output has mean beta and variance
gamma^2 var / (var + eps), each channel of dx sums to zero, and the sum of
dx xhat is gamma dgamma eps / (var + eps)^(3/2) (zero as eps -> 0).
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from memory_efficient_activation_b200 import synthetic


def _pieces(N, ks, HW, seed, mean=0.0, sigma=1.0):
    out = []
    for i, k in enumerate(ks):
        a = synthetic.normal_f64(N * k * HW, sigma, seed * 16 + i, 0, mean=mean)
        out.append(a.reshape(N, k, HW))
    return out


def _params(C, seed):
    return synthetic.uniform_f64(C, 0.5, 1.5, seed, 3), synthetic.normal_f64(C, 0.2, seed, 4)


@pytest.mark.parametrize("N,ks,HW", [(4, [3, 5, 2], 7), (2, [8], 16), (5, [1, 1, 1], 1), (3, [4, 6], 9)])
def test_matches_torch_autograd(N, ks, HW):
    eps = 1e-5
    pieces = _pieces(N, ks, HW, 51)
    C = sum(ks)
    g, b = _params(C, 52)
    dy = synthetic.normal_f64(N * C * HW, 1.0, 53, 1).reshape(N, C, HW)
    y, mean, var, _ = oracle.concat_bn_relu_fwd(pieces, g, b, eps)
    tp = [torch.from_numpy(p.copy()).requires_grad_(True) for p in pieces]
    tg = torch.from_numpy(g.copy()).requires_grad_(True)
    tb = torch.from_numpy(b.copy()).requires_grad_(True)
    x = torch.cat(tp, dim=1)
    ty = torch.relu(F.batch_norm(x, None, None, tg, tb, training=True, eps=eps))
    assert np.allclose(y, ty.detach().numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(mean, x.detach().mean(dim=(0, 2)).numpy(), rtol=1e-12, atol=1e-14)
    assert np.allclose(var, x.detach().var(dim=(0, 2), unbiased=False).numpy(), rtol=1e-12, atol=1e-14)
    ty.backward(torch.from_numpy(dy))
    dps, dg, db, _ = oracle.concat_bn_relu_bwd(pieces, dy, g, b, mean, var, eps)
    for dp, t in zip(dps, tp):
        assert np.allclose(dp, t.grad.numpy(), rtol=1e-9, atol=1e-12)
    assert np.allclose(dg, tg.grad.numpy(), rtol=1e-10, atol=1e-12)
    assert np.allclose(db, tb.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_hand_example():
    # one channel, x = [0, 1, 5]: mean 2, var 14/3; eps 0, gamma 1, beta 0:
    # xhat = [-2, -1, 3] / sqrt(14/3); relu keeps the last element only
    x = [np.array([[[0.0, 1.0, 5.0]]])]
    y, mean, var, _ = oracle.concat_bn_relu_fwd(x, [1.0], [0.0], eps=0.0)
    s = np.sqrt(14.0 / 3.0)
    assert mean[0] == 2.0 and np.isclose(var[0], 14.0 / 3.0, rtol=1e-15)
    assert np.allclose(y.ravel(), [0.0, 0.0, 3.0 / s], rtol=1e-15)
    # dy = [1, 1, 1]: dz = [0, 0, 1], dbeta = 1, dgamma = 3 / s,
    # dx = (1 / s) (dz - 1/3 - xhat dgamma / 3) = (1 / s) (dz - 1/3 - xhat / s)
    dps, dg, db, _ = oracle.concat_bn_relu_bwd(x, np.ones((1, 1, 3)), [1.0], [0.0], mean, var, eps=0.0)
    xh = np.array([-2.0, -1.0, 3.0]) / s
    ref = (np.array([0.0, 0.0, 1.0]) - 1.0 / 3.0 - xh * (3.0 / s) / 3.0) / s
    assert np.isclose(db[0], 1.0) and np.isclose(dg[0], 3.0 / s, rtol=1e-15)
    assert np.allclose(dps[0].ravel(), ref, rtol=1e-14, atol=1e-15)


def test_invariants_above_threshold():
    # beta = 50 puts every output above zero: y = gamma xhat + beta exactly
    eps = 1e-3
    pieces = _pieces(6, [4, 3], 10, 54, mean=3.0, sigma=2.0)
    C = 7
    g = synthetic.uniform_f64(C, 0.5, 1.5, 55, 3)
    b = np.full(C, 50.0)
    y, mean, var, _ = oracle.concat_bn_relu_fwd(pieces, g, b, eps)
    assert np.all(y > 0)
    assert np.allclose(y.mean(axis=(0, 2)), b, rtol=1e-13)
    assert np.allclose(y.var(axis=(0, 2)), g * g * var / (var + eps), rtol=1e-10)
    dy = synthetic.normal_f64(6 * C * 10, 1.0, 56, 1).reshape(6, C, 10)
    dps, dg, db, _ = oracle.concat_bn_relu_bwd(pieces, dy, g, b, mean, var, eps)
    dx = np.concatenate(dps, axis=1)
    x = np.concatenate(pieces, axis=1)
    xh = (x - mean[None, :, None]) / np.sqrt(var + eps)[None, :, None]
    assert np.allclose(dx.sum(axis=(0, 2)), 0.0, atol=1e-12)
    # sum dx xhat = gamma r dgamma (1 - sum xhat^2 / n) = gamma r dgamma eps / (var + eps)
    r = 1.0 / np.sqrt(var + eps)
    assert np.allclose((dx * xh).sum(axis=(0, 2)), g * r * dg * eps / (var + eps), rtol=1e-9, atol=1e-13)
    assert np.allclose(db, dy.sum(axis=(0, 2)), rtol=1e-12)


@pytest.mark.parametrize("N,C,HW", [(4, 6, 7), (2, 3, 1), (8, 5, 25)])
def test_running_update_matches_torch(N, C, HW):
    # torch's training-mode F.batch_norm updates running_mean / running_var in
    # place with momentum and the unbiased batch variance
    x = synthetic.normal_f64(N * C * HW, 1.3, 54, 0, mean=0.4).reshape(N, C, HW)
    rm0 = synthetic.normal_f64(C, 0.5, 55, 3)
    rv0 = synthetic.uniform_f64(C, 0.5, 2.0, 55, 4)
    g, b = _params(C, 56)
    _, mean, var, _ = oracle.concat_bn_relu_fwd([x], g, b, 1e-5)
    rm, rv = oracle.bn_running_update(rm0, rv0, mean, var, N * HW, 0.1)
    trm, trv = torch.from_numpy(rm0.copy()), torch.from_numpy(rv0.copy())
    F.batch_norm(torch.from_numpy(x.copy()), trm, trv, torch.from_numpy(g), torch.from_numpy(b), training=True,
                 momentum=0.1, eps=1e-5)
    assert np.allclose(rm, trm.numpy(), rtol=1e-13, atol=1e-15)
    assert np.allclose(rv, trv.numpy(), rtol=1e-13, atol=1e-15)


def test_running_update_hand_worked():
    # one channel, values {1, 3}: mean 2, biased variance 1, unbiased 2;
    # momentum 0.25 from (0, 1): mean 0.75 * 0 + 0.25 * 2 = 0.5,
    # var 0.75 * 1 + 0.25 * 2 = 1.25
    rm, rv = oracle.bn_running_update([0.0], [1.0], [2.0], [1.0], 2, 0.25)
    assert rm[0] == 0.5 and rv[0] == 1.25
