"""Pins for the oracle's fused per-channel affine + Swish (NHWC and NCHW).

z = gamma_c x + beta_c, y = z Sigmoid(z); backward dx = gamma_c dz,
dgamma_c = sum dz x, dbeta_c = sum dz, dz = dy Swish'(z).  Checked against
PyTorch CPU float64 autograd with the channel broadcast written in torch's
own indexing (independent of the oracle's flat-index arithmetic), against the
plain Swish oracle (gamma = 1, beta = 0), against finite differences in
gamma_c and beta_c, and by brute force on tiny tensors.
"""
import numpy as np
import pytest
import torch

import oracle
from memory_efficient_activation_b200 import synthetic


def _inputs(shape_nchw, layout, seed):
    N, C, H, W = shape_nchw
    n = N * C * H * W
    x = synthetic.normal_f64(n, 1.0, seed, 0)
    dy = synthetic.normal_f64(n, 1.0, seed, 1)
    g = synthetic.uniform_f64(C, 0.5, 1.5, seed, 3)
    b = synthetic.normal_f64(C, 0.1, seed, 4)
    return x, dy, g, b


def _torch_ref(shape_nchw, layout, x, dy, g, b):
    N, C, H, W = shape_nchw
    mem = (N, H, W, C) if layout == "nhwc" else (N, C, H, W)
    bshape = (1, 1, 1, C) if layout == "nhwc" else (1, C, 1, 1)
    tx = torch.from_numpy(x.reshape(mem).copy()).requires_grad_(True)
    tg = torch.from_numpy(g.copy()).requires_grad_(True)
    tb = torch.from_numpy(b.copy()).requires_grad_(True)
    z = tg.view(bshape) * tx + tb.view(bshape)
    y = torch.nn.functional.silu(z)
    y.backward(torch.from_numpy(dy.reshape(mem)))
    return (y.detach().numpy().ravel(), tx.grad.numpy().ravel(),
            tg.grad.numpy(), tb.grad.numpy())


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
@pytest.mark.parametrize("shape", [(2, 16, 3, 3), (3, 5, 4, 7), (1, 144, 2, 2)])
def test_affine_matches_torch_autograd(layout, shape):
    x, dy, g, b = _inputs(shape, layout, 31)
    y_t, dx_t, dg_t, db_t = _torch_ref(shape, layout, x, dy, g, b)
    y = oracle.affine_swish_fwd(layout, shape, x, g, b)
    dx, dg, db = oracle.affine_swish_bwd(layout, shape, x, dy, g, b)
    np.testing.assert_allclose(y, y_t, rtol=1e-14, atol=1e-300)
    np.testing.assert_allclose(dx, dx_t, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(dg, dg_t, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(db, db_t, rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_affine_identity_reduces_to_swish(layout):
    shape = (2, 8, 3, 5)
    x, dy, _, _ = _inputs(shape, layout, 32)
    C = shape[1]
    one, zero = np.ones(C), np.zeros(C)
    np.testing.assert_array_equal(oracle.affine_swish_fwd(layout, shape, x, one, zero),
                                  oracle.act_fwd("swish", x, 1.0))
    dx, _, _ = oracle.affine_swish_bwd(layout, shape, x, dy, one, zero)
    np.testing.assert_array_equal(dx, oracle.act_bwd("swish", x, dy, 1.0))


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_affine_ones_input_gives_equal_dgamma_dbeta(layout):
    shape = (2, 6, 3, 3)
    _, dy, g, b = _inputs(shape, layout, 33)
    x = np.ones(int(np.prod(shape)))
    _, dg, db = oracle.affine_swish_bwd(layout, shape, x, dy, g, b)
    np.testing.assert_array_equal(dg, db)


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_affine_brute_force_tiny(layout):
    # 2 x 16 x 3 x 3, channel of each element found by walking the memory order.
    N, C, H, W = shape = (2, 16, 3, 3)
    x, dy, g, b = _inputs(shape, layout, 34)
    dx, dg, db = oracle.affine_swish_bwd(layout, shape, x, dy, g, b)
    sg = [0.0] * C
    sb = [0.0] * C
    i = 0
    order = ((n, h, w, c) for n in range(N) for h in range(H) for w in range(W) for c in range(C)) \
        if layout == "nhwc" else \
        ((n, h, w, c) for n in range(N) for c in range(C) for h in range(H) for w in range(W))
    for (_n, _h, _w, c) in order:
        z = g[c] * x[i] + b[c]
        s = 1.0 / (1.0 + np.exp(-z))
        dz = dy[i] * (s + z * s * (1.0 - s))
        assert dx[i] == pytest.approx(g[c] * dz, rel=1e-12, abs=1e-15)
        sg[c] += dz * x[i]
        sb[c] += dz
        i += 1
    np.testing.assert_allclose(dg, sg, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(db, sb, rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
def test_affine_param_grads_match_finite_differences(layout):
    shape = (2, 4, 5, 5)
    x, dy, g, b = _inputs(shape, layout, 35)
    _, dg, db = oracle.affine_swish_bwd(layout, shape, x, dy, g, b)
    h = 1e-6
    for c in range(shape[1]):
        for grads, vec in ((dg, "g"), (db, "b")):
            gp, gm, bp, bm = g.copy(), g.copy(), b.copy(), b.copy()
            if vec == "g":
                gp[c] += h
                gm[c] -= h
            else:
                bp[c] += h
                bm[c] -= h
            Lp = np.sum(dy * oracle.affine_swish_fwd(layout, shape, x, gp, bp))
            Lm = np.sum(dy * oracle.affine_swish_fwd(layout, shape, x, gm, bm))
            assert grads[c] == pytest.approx((Lp - Lm) / (2 * h), rel=1e-6, abs=1e-8)


def test_affine_rejects_bad_layout():
    with pytest.raises(KeyError):
        oracle.affine_swish_fwd("nwhc", (1, 1, 1, 1), [1.0], [1.0], [0.0])
