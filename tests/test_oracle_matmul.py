"""Pins for the oracle's matmul + activation pair (problem B07, SOLUTION
step 4: the activation follows a d x d matrix multiply on the same tensor).

Checked against numpy's float64 matmul (a library routine), hand-computed
small products, a permutation matrix (which catches a transposed operand),
rank-one products (K = 1), and PyTorch CPU float64 autograd of
out = f(Z) W2^T for the backward dZ = (G W2) * f'(Z).
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from memory_efficient_activation_b200 import synthetic

ACTS = list(synthetic.ACTIVATIONS)


def _p(act):
    return 0.1 if act == "leaky_relu" else (1.5 if act == "swish" else 1.0)


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


def _bf16_values(n, sigma, seed, stream):
    """n bf16-representable values (as float64), normal with std sigma."""
    a = synthetic.normal_f64(n, sigma, seed, stream)
    return torch.from_numpy(a).to(torch.bfloat16).double().numpy()


def _xw(M, N, K, seed):
    X = _bf16_values(M * K, 1.0, seed, 0).reshape(M, K)
    W = _bf16_values(N * K, K ** -0.5, seed, 1).reshape(N, K)
    return X, W


def test_hand_example():
    X = np.array([[1.0, 2.0, 3.0], [4.0, 5.0, 6.0]])
    W = np.array([[1.0, 0.0, -1.0], [2.0, 1.0, 0.0]])
    Z, Y, S = oracle.matmul_act_fwd("relu", X, W)
    assert np.array_equal(Z, [[-2.0, 4.0], [-2.0, 13.0]])
    assert np.array_equal(Y, [[0.0, 4.0], [0.0, 13.0]])
    assert np.array_equal(S, [[4.0, 4.0], [10.0, 13.0]])
    _, Y, _ = oracle.matmul_act_fwd("leaky_relu", X, W, 0.25)
    assert np.array_equal(Y, [[-0.5, 4.0], [-0.5, 13.0]])
    # backward: dZ = (G W^T) f'(Z); relu' is the predicate Z > 0
    G = np.array([[1.0, 1.0, 1.0], [0.0, 2.0, -1.0]])
    dZ, D, S = oracle.matmul_act_bwd("relu", G, W, Z)
    assert np.array_equal(D, [[0.0, 3.0], [1.0, 2.0]])
    assert np.array_equal(dZ, [[0.0, 3.0], [0.0, 2.0]])
    assert np.array_equal(S, [[2.0, 3.0], [1.0, 2.0]])


@pytest.mark.parametrize("M,N,K", [(7, 5, 3), (16, 33, 64), (3, 130, 257)])
def test_matches_numpy_matmul(M, N, K):
    X, W = _xw(M, N, K, 11)
    Z, _, S = oracle.matmul_act_fwd("swish", X, W)
    ref = X @ W.T
    assert np.all(np.abs(Z - ref) <= 1e-13 * S + 1e-300)
    G = _bf16_values(M * K, 1.0, 12, 2).reshape(M, K)
    _, D, S2 = oracle.matmul_act_bwd("swish", G, W, Z)
    assert np.all(np.abs(D - G @ W.T) <= 1e-13 * S2 + 1e-300)
    assert np.allclose(S, np.abs(X) @ np.abs(W).T, rtol=1e-13, atol=0)


def test_permutation_catches_transpose():
    # W selects columns of X: W[n, pi(n)] = 1, so Z[:, n] = X[:, pi(n)] exactly;
    # computing X W (not X W^T) would fail the shapes or the values.
    M, N, K = 6, 5, 9
    X, _ = _xw(M, N, K, 13)
    pi = np.array([7, 0, 3, 8, 2])
    W = np.zeros((N, K))
    W[np.arange(N), pi] = 1.0
    Z, _, _ = oracle.matmul_act_fwd("relu", X, W)
    assert np.array_equal(Z, X[:, pi])
    # backward with the same W: D = G W^T picks the same columns of G
    G, _ = _xw(M, N, K, 14)
    _, D, _ = oracle.matmul_act_bwd("relu", G, W, Z)
    assert np.array_equal(D, G[:, pi])


def test_rank_one():
    x = _bf16_values(9, 1.0, 15, 0).reshape(9, 1)
    w = _bf16_values(4, 1.0, 15, 1).reshape(4, 1)
    Z, _, _ = oracle.matmul_act_fwd("tanh", x, w)
    assert np.array_equal(Z, x @ w.T)   # one product each: exact


@pytest.mark.parametrize("act", ACTS)
def test_forward_activation_at_stored_z(act):
    X, W = _xw(12, 20, 96, 16)
    p = _p(act)
    Z, Y, _ = oracle.matmul_act_fwd(act, X, W, p, round_z_bf16=True)
    zr = torch.from_numpy(Z).to(torch.bfloat16).double()
    assert np.array_equal(Y, oracle.act_fwd(act, zr.numpy(), p))
    ref = _torch_act(act, zr, p).numpy()
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-300)
    Z2, Y2, _ = oracle.matmul_act_fwd(act, X, W, p, round_z_bf16=False)
    assert np.array_equal(Z2, Z)
    assert np.allclose(Y2, _torch_act(act, torch.from_numpy(Z), p).numpy(), rtol=1e-12, atol=1e-300)


@pytest.mark.parametrize("act", ACTS)
def test_backward_matches_torch_autograd(act):
    # out = f(Z) W2^T with W2 [K, N]; upstream G [M, K]:
    # dZ = (G W2) * f'(Z), i.e. the oracle's (G W^T) f'(Z) with W = W2^T.
    M, N, K = 10, 24, 40
    p = _p(act)
    Zv = _bf16_values(M * N, 2.0, 17, 0).reshape(M, N)
    W2 = _bf16_values(K * N, N ** -0.5, 17, 1).reshape(K, N)
    G = _bf16_values(M * K, 1.0, 17, 2).reshape(M, K)
    z = torch.from_numpy(Zv.copy()).requires_grad_(True)
    out = _torch_act(act, z, p) @ torch.from_numpy(W2).T
    out.backward(torch.from_numpy(G))
    dZ, D, _ = oracle.matmul_act_bwd(act, G, np.ascontiguousarray(W2.T), Zv, p)
    assert np.allclose(D, G @ W2, rtol=1e-13, atol=1e-300)
    assert np.allclose(dZ, z.grad.numpy(), rtol=1e-9, atol=1e-14)


def test_rejects_bad_shapes():
    with pytest.raises(ValueError):
        oracle.matmul_act_fwd("relu", np.zeros((2, 3)), np.zeros((2, 4)))
    with pytest.raises(ValueError):
        oracle.matmul_act_bwd("relu", np.zeros((2, 3)), np.zeros((4, 3)), np.zeros((2, 5)))
