"""Double-precision CPU oracle for the memory-efficient activation path.

TEST INFRASTRUCTURE ONLY.  The product (the CUDA library under
``memory_efficient_activation_b200/`` and its binding) never imports this
package.  It is used by ``tests/``, by ``__graft_entry__.smoke()`` and by the
CPU-baseline leg of ``bench.py``; nothing else.

The arithmetic lives in ``mea_oracle.c`` (plain C, libm, double precision,
serial long-double reductions).  This module only builds it with gcc when the
shared object is missing or older than the source, and marshals numpy arrays
through ctypes.  Inputs are float64 arrays holding the exact stored values;
outputs are float64 (exact results in double) plus the two rounding helpers
that produce the value a correct bf16 / fp32 kernel output should be near.

Sources (by page and section):

* "Memory efficient Swish" (adeeplearner blog, 2021-05-17): Swish and its
  save-input-only backward ("How is Swish implemented?", "How is the memory
  efficient version Swish implemented?", "What makes this implementation save
  GPU memory?").
* "What activations cost, in memory and in arithmetic" (asifuddin.com,
  problem B07), GIVEN: the activation family; SOLUTION step 4: the matrix
  multiply the activation follows (matmul_act_fwd / matmul_act_bwd).
* "A memory-efficient implementation of DenseNets", "Motivation": the
  concatenation and batch normalization whose outputs are re-populated in
  the backward (concat_bn_relu_fwd / concat_bn_relu_bwd).

Parity pins for every function here live in ``tests/test_oracle_*.py``.
Each function is checked against something other than itself:

* act_fwd, act_bwd, act_deriv: test_oracle_swish.py and test_oracle_family.py.
  Checks: closed forms (Swish(0), f'(0) = 1/2, f''(0) = alpha/2, the
  Lambert-W minimum); odd-part identities; limits; central finite
  differences; torch float64 autograd; scipy expit / ndtr and the textbook
  Phi(1).
* act_bwd_scale: test_oracle_swish.py.  The scale is at least |dx| and equal
  to it away from the zeros of f'.
* swish_dalpha: test_oracle_swish.py (finite differences in alpha, brute-force
  sums) and test_oracle_channel.py (per-channel sums).
* affine_swish_*, affine_act_*, swish_channel_*: test_oracle_affine.py and
  test_oracle_channel.py.  Checks: torch autograd; brute force on tiny
  inputs; finite differences of the parameter gradients; reduction to the
  plain activation at gamma = 1, beta = 0, and to a scalar alpha when all
  alphas are equal.
* matmul_act_*: test_oracle_matmul.py.  Checks: a hand-worked example;
  numpy matmul; a permutation that catches a transposed operand; rank-one
  products; torch autograd for the backward.
* affine_act_zround: test_oracle_channel.py.  Checks: exact first-order
  values for ReLU; u |z f'(z)| against the pinned derivative and u |z f''(z)|
  against Swish's closed-form second derivative and torch float64 double
  backward for GELU-tanh.
* concat_bn_relu_*: test_oracle_bn.py.  Checks: torch.cat + F.batch_norm +
  relu autograd in float64; a hand-worked example; the batch-normalization
  invariants.
* bn_running_update: test_oracle_bn.py.  Checks: torch F.batch_norm's
  running_mean / running_var update (training, momentum 0.1) in float64; a
  hand-worked example.
* round_bf16, round_f32: test_oracle_rounding.py.  Checks: torch's and
  numpy's round-to-nearest-even casts; ties to even and range boundaries;
  identity on every finite bf16 value.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mea_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# gcc command; keep -fno-fast-math / -ffp-contract=off so the double
# arithmetic is the plain IEEE sequence written in the source.
GCC_CMD = [
    "gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC",
    "-shared", "-Wall", "-Wextra", "-o", _LIB, _SRC, "-lm",
]

# The oracle's own activation numbering (mirrors the enum in mea_oracle.c).
ACTS = {
    "relu": 0,
    "leaky_relu": 1,
    "sigmoid": 2,
    "tanh": 3,
    "gelu_erf": 4,
    "gelu_tanh": 5,
    "swish": 6,
}
LAYOUTS = {"nchw": 0, "nhwc": 1}


def build(force: bool = False) -> str:
    """Compile liboracle.so from mea_oracle.c if needed; return its path."""
    stale = (not os.path.exists(_LIB)
             or os.path.getmtime(_LIB) < os.path.getmtime(_SRC))
    if force or stale:
        subprocess.run(GCC_CMD, check=True)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        d = ctypes.POINTER(ctypes.c_double)
        i64 = ctypes.c_int64
        lib.oracle_act_fwd.argtypes = [ctypes.c_int, d, d, i64, ctypes.c_double]
        lib.oracle_act_fwd.restype = ctypes.c_int
        lib.oracle_act_bwd.argtypes = [ctypes.c_int, d, d, d, i64, ctypes.c_double]
        lib.oracle_act_bwd.restype = ctypes.c_int
        lib.oracle_act_deriv.argtypes = [ctypes.c_int, d, d, i64, ctypes.c_double]
        lib.oracle_act_deriv.restype = ctypes.c_int
        lib.oracle_act_bwd_scale.argtypes = [ctypes.c_int, d, d, d, i64, ctypes.c_double]
        lib.oracle_act_bwd_scale.restype = ctypes.c_int
        lib.oracle_swish_dalpha.argtypes = [d, d, i64, ctypes.c_double]
        lib.oracle_swish_dalpha.restype = ctypes.c_double
        shp = ctypes.POINTER(ctypes.c_int64)
        lib.oracle_affine_swish_fwd.argtypes = [ctypes.c_int, shp, d, d, d, d]
        lib.oracle_affine_swish_fwd.restype = ctypes.c_int
        lib.oracle_affine_swish_bwd.argtypes = [ctypes.c_int, shp, d, d, d, d, d, d, d, d]
        lib.oracle_affine_swish_bwd.restype = ctypes.c_int
        lib.oracle_affine_act_fwd.argtypes = [ctypes.c_int, ctypes.c_int, shp, d, d, d, ctypes.c_double, d]
        lib.oracle_affine_act_fwd.restype = ctypes.c_int
        lib.oracle_affine_act_bwd.argtypes = [ctypes.c_int, ctypes.c_int, shp, d, d, d, d, ctypes.c_double,
                                              d, d, d, d]
        lib.oracle_affine_act_bwd.restype = ctypes.c_int
        lib.oracle_affine_act_zround.argtypes = [ctypes.c_int, ctypes.c_int, shp, d, d, d, d, ctypes.c_double,
                                                 d, d]
        lib.oracle_affine_act_zround.restype = ctypes.c_int
        lib.oracle_bn_running_update.argtypes = [i64, i64, d, d, ctypes.c_double, d, d]
        lib.oracle_bn_running_update.restype = ctypes.c_int
        lib.oracle_swish_channel_fwd.argtypes = [ctypes.c_int, shp, d, d, d]
        lib.oracle_swish_channel_fwd.restype = ctypes.c_int
        lib.oracle_swish_channel_bwd.argtypes = [ctypes.c_int, shp, d, d, d, d, d, d]
        lib.oracle_swish_channel_bwd.restype = ctypes.c_int
        lib.oracle_matmul_act_fwd.argtypes = [ctypes.c_int, i64, i64, i64, d, d, ctypes.c_double, ctypes.c_int,
                                              d, d, d]
        lib.oracle_matmul_act_fwd.restype = ctypes.c_int
        lib.oracle_matmul_act_bwd.argtypes = [ctypes.c_int, i64, i64, i64, d, d, d, ctypes.c_double, d, d, d]
        lib.oracle_matmul_act_bwd.restype = ctypes.c_int
        lib.oracle_bn_relu_fwd.argtypes = [i64, i64, i64, d, d, d, ctypes.c_double, d, d, d, d]
        lib.oracle_bn_relu_fwd.restype = ctypes.c_int
        lib.oracle_bn_relu_bwd.argtypes = [i64, i64, i64, d, d, d, d, d, d, ctypes.c_double, d, d, d, d]
        lib.oracle_bn_relu_bwd.restype = ctypes.c_int
        lib.oracle_round_bf16.argtypes = [d, ctypes.POINTER(ctypes.c_uint16), i64]
        lib.oracle_round_bf16.restype = None
        lib.oracle_round_f32.argtypes = [d, ctypes.POINTER(ctypes.c_float), i64]
        lib.oracle_round_f32.restype = None
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_num_threads.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray, ctype=ctypes.c_double):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def num_threads() -> int:
    """OpenMP threads the elementwise loops use."""
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Set the OpenMP threads of the elementwise loops (n >= 1)."""
    _load().oracle_set_num_threads(int(n))


def act_fwd(act: str, x, param: float = 1.0) -> np.ndarray:
    """y = f(x; param) in double.  param: alpha (Swish), slope (LeakyReLU)."""
    x = _f64(x)
    y = np.empty_like(x)
    rc = _load().oracle_act_fwd(ACTS[act], _ptr(x), _ptr(y), x.size, float(param))
    if rc:
        raise ValueError(f"oracle_act_fwd({act}) failed: {rc}")
    return y


def act_bwd(act: str, x, dy, param: float = 1.0) -> np.ndarray:
    """dx = dy * f'(x; param) in double, f' recomputed from x."""
    x = _f64(x)
    dy = _f64(dy)
    if x.shape != dy.shape:
        raise ValueError("x and dy shapes differ")
    dx = np.empty_like(x)
    rc = _load().oracle_act_bwd(ACTS[act], _ptr(x), _ptr(dy), _ptr(dx), x.size, float(param))
    if rc:
        raise ValueError(f"oracle_act_bwd({act}) failed: {rc}")
    return dx


def act_bwd_scale(act: str, x, dy, param: float = 1.0) -> np.ndarray:
    """|dy| times the sum of the absolute terms of f'(x): the scale the error
    of a finite-precision dx is proportional to (equals |dx| where f' has a
    single term)."""
    x = _f64(x)
    dy = _f64(dy)
    m = np.empty_like(x)
    rc = _load().oracle_act_bwd_scale(ACTS[act], _ptr(x), _ptr(dy), _ptr(m), x.size, float(param))
    if rc:
        raise ValueError(f"oracle_act_bwd_scale({act}) failed: {rc}")
    return m


def act_deriv(act: str, x, param: float = 1.0) -> np.ndarray:
    """f'(x; param) in double."""
    x = _f64(x)
    d = np.empty_like(x)
    rc = _load().oracle_act_deriv(ACTS[act], _ptr(x), _ptr(d), x.size, float(param))
    if rc:
        raise ValueError(f"oracle_act_deriv({act}) failed: {rc}")
    return d


def swish_dalpha(x, dy, alpha: float) -> float:
    """d alpha = sum dy x^2 s (1 - s), serial long-double sum."""
    x = _f64(x)
    dy = _f64(dy)
    return float(_load().oracle_swish_dalpha(_ptr(x), _ptr(dy), x.size, float(alpha)))


def _shape4(shape) -> np.ndarray:
    s = np.ascontiguousarray(np.asarray(shape, dtype=np.int64))
    if s.shape != (4,):
        raise ValueError("shape must be (N, C, H, W)")
    return s


def affine_swish_fwd(layout: str, shape, x, gamma, beta) -> np.ndarray:
    """y = z Sigmoid(z), z = gamma_c x + beta_c; shape is (N, C, H, W)."""
    s = _shape4(shape)
    x, gamma, beta = _f64(x), _f64(gamma), _f64(beta)
    y = np.empty_like(x)
    rc = _load().oracle_affine_swish_fwd(LAYOUTS[layout], _ptr(s, ctypes.c_int64),
                                         _ptr(x), _ptr(gamma), _ptr(beta), _ptr(y))
    if rc:
        raise ValueError(f"oracle_affine_swish_fwd failed: {rc}")
    return y


def affine_swish_bwd(layout: str, shape, x, dy, gamma, beta, with_scale: bool = False):
    """Returns (dx, dgamma, dbeta) in double, plus the condition scale of dx
    when with_scale is set."""
    s = _shape4(shape)
    x, dy, gamma, beta = _f64(x), _f64(dy), _f64(gamma), _f64(beta)
    dx = np.empty_like(x)
    C = int(s[1])
    dg = np.empty(C, dtype=np.float64)
    db = np.empty(C, dtype=np.float64)
    scale = np.empty_like(x) if with_scale else None
    rc = _load().oracle_affine_swish_bwd(LAYOUTS[layout], _ptr(s, ctypes.c_int64),
                                         _ptr(x), _ptr(dy), _ptr(gamma), _ptr(beta),
                                         _ptr(dx), _ptr(dg), _ptr(db),
                                         _ptr(scale) if with_scale else None)
    if rc:
        raise ValueError(f"oracle_affine_swish_bwd failed: {rc}")
    return (dx, dg, db, scale) if with_scale else (dx, dg, db)


def affine_act_fwd(act: str, layout: str, shape, x, gamma, beta, param: float = 1.0) -> np.ndarray:
    """y = f(gamma_c x + beta_c; param); shape is (N, C, H, W)."""
    s = _shape4(shape)
    x, gamma, beta = _f64(x), _f64(gamma), _f64(beta)
    y = np.empty_like(x)
    rc = _load().oracle_affine_act_fwd(ACTS[act], LAYOUTS[layout], _ptr(s, ctypes.c_int64), _ptr(x),
                                       _ptr(gamma), _ptr(beta), float(param), _ptr(y))
    if rc:
        raise ValueError(f"oracle_affine_act_fwd failed: {rc}")
    return y


def affine_act_bwd(act: str, layout: str, shape, x, dy, gamma, beta, param: float = 1.0):
    """Returns (dx, dgamma, dbeta, dx condition scale) in double."""
    s = _shape4(shape)
    x, dy, gamma, beta = _f64(x), _f64(dy), _f64(gamma), _f64(beta)
    C = int(s[1])
    dx = np.empty_like(x)
    scale = np.empty_like(x)
    dg = np.empty(C, dtype=np.float64)
    db = np.empty(C, dtype=np.float64)
    rc = _load().oracle_affine_act_bwd(ACTS[act], LAYOUTS[layout], _ptr(s, ctypes.c_int64), _ptr(x), _ptr(dy),
                                       _ptr(gamma), _ptr(beta), float(param), _ptr(dx), _ptr(dg), _ptr(db),
                                       _ptr(scale))
    if rc:
        raise ValueError(f"oracle_affine_act_bwd failed: {rc}")
    return dx, dg, db, scale


def affine_act_zround(act: str, layout: str, shape, x, dy, gamma, beta, param: float = 1.0):
    """Returns (ey, edx): per element, the largest change of y = f(z) and of
    dx = gamma_c dy f'(z) when z = gamma_c x + beta_c moves by one binary32
    rounding (to z (1 -+ 2^-24)).  The part of an fp32 evaluation's error that
    comes from forming z in fp32."""
    s = _shape4(shape)
    x, dy, gamma, beta = _f64(x), _f64(dy), _f64(gamma), _f64(beta)
    ey = np.empty_like(x)
    edx = np.empty_like(x)
    rc = _load().oracle_affine_act_zround(ACTS[act], LAYOUTS[layout], _ptr(s, ctypes.c_int64), _ptr(x), _ptr(dy),
                                          _ptr(gamma), _ptr(beta), float(param), _ptr(ey), _ptr(edx))
    if rc:
        raise ValueError(f"oracle_affine_act_zround failed: {rc}")
    return ey, edx


def swish_channel_fwd(layout: str, shape, x, alpha) -> np.ndarray:
    """y = x Sigmoid(alpha_c x); shape is (N, C, H, W)."""
    s = _shape4(shape)
    x, alpha = _f64(x), _f64(alpha)
    y = np.empty_like(x)
    rc = _load().oracle_swish_channel_fwd(LAYOUTS[layout], _ptr(s, ctypes.c_int64), _ptr(x), _ptr(alpha), _ptr(y))
    if rc:
        raise ValueError(f"oracle_swish_channel_fwd failed: {rc}")
    return y


def swish_channel_bwd(layout: str, shape, x, dy, alpha):
    """Returns (dx, dalpha per channel, dx condition scale) in double."""
    s = _shape4(shape)
    x, dy, alpha = _f64(x), _f64(dy), _f64(alpha)
    dx = np.empty_like(x)
    scale = np.empty_like(x)
    da = np.empty(int(s[1]), dtype=np.float64)
    rc = _load().oracle_swish_channel_bwd(LAYOUTS[layout], _ptr(s, ctypes.c_int64), _ptr(x), _ptr(dy),
                                          _ptr(alpha), _ptr(dx), _ptr(da), _ptr(scale))
    if rc:
        raise ValueError(f"oracle_swish_channel_bwd failed: {rc}")
    return dx, da, scale


def matmul_act_fwd(act: str, X, W, param: float = 1.0, round_z_bf16: bool = True):
    """Z = X W^T (X [M, K], W [N, K]) and Y = f(Z as stored: rounded to bf16
    when round_z_bf16).  Returns (Z, Y, absum) in double, absum = sum_k
    |X[m, k] W[n, k]|."""
    X, W = np.ascontiguousarray(X, dtype=np.float64), np.ascontiguousarray(W, dtype=np.float64)
    M, K = X.shape
    N, K2 = W.shape
    if K != K2:
        raise ValueError("X and W disagree in K")
    Z = np.empty((M, N))
    Y = np.empty((M, N))
    S = np.empty((M, N))
    rc = _load().oracle_matmul_act_fwd(ACTS[act], M, N, K, _ptr(X), _ptr(W), float(param), int(bool(round_z_bf16)),
                                       _ptr(Z), _ptr(Y), _ptr(S))
    if rc:
        raise ValueError(f"oracle_matmul_act_fwd failed: {rc}")
    return Z, Y, S


def matmul_act_bwd(act: str, G, W, Z, param: float = 1.0):
    """dZ = (G W^T) * f'(Z) (G [M, K], W [N, K], Z [M, N] as stored).
    Returns (dZ, D, absum): D = G W^T before the derivative, absum = sum_k
    |G[m, k] W[n, k]|."""
    G, W = np.ascontiguousarray(G, dtype=np.float64), np.ascontiguousarray(W, dtype=np.float64)
    Z = np.ascontiguousarray(Z, dtype=np.float64)
    M, K = G.shape
    N, K2 = W.shape
    if K != K2 or Z.shape != (M, N):
        raise ValueError("shapes disagree")
    dZ = np.empty((M, N))
    D = np.empty((M, N))
    S = np.empty((M, N))
    rc = _load().oracle_matmul_act_bwd(ACTS[act], M, N, K, _ptr(G), _ptr(W), _ptr(Z), float(param), _ptr(dZ),
                                       _ptr(D), _ptr(S))
    if rc:
        raise ValueError(f"oracle_matmul_act_bwd failed: {rc}")
    return dZ, D, S


def concat_bn_relu_fwd(pieces, gamma, beta, eps: float = 1e-5):
    """y = max(BN(concat(pieces, channel axis)), 0) with batch statistics.
    pieces: NCHW arrays [N, k_i, H, W].  Returns (y [N, C, H, W], mean [C],
    biased var [C], y_scale)."""
    x = np.ascontiguousarray(np.concatenate([np.asarray(p, dtype=np.float64) for p in pieces], axis=1))
    N, C = x.shape[0], x.shape[1]
    HW = int(np.prod(x.shape[2:]))
    gamma, beta = _f64(gamma), _f64(beta)
    y = np.empty_like(x)
    ys = np.empty_like(x)
    mean = np.empty(C)
    var = np.empty(C)
    rc = _load().oracle_bn_relu_fwd(N, C, HW, _ptr(x), _ptr(gamma), _ptr(beta), float(eps), _ptr(y), _ptr(mean),
                                    _ptr(var), _ptr(ys))
    if rc:
        raise ValueError(f"oracle_bn_relu_fwd failed: {rc}")
    return y, mean, var, ys


def concat_bn_relu_bwd(pieces, dy, gamma, beta, mean, var, eps: float = 1e-5):
    """Backward of concat_bn_relu_fwd from the pieces, dy [N, C, H, W] and the
    batch statistics.  Returns (list of d piece, dgamma, dbeta, dx_scale as a
    list split like the pieces)."""
    pieces = [np.asarray(p, dtype=np.float64) for p in pieces]
    x = np.ascontiguousarray(np.concatenate(pieces, axis=1))
    dy = np.ascontiguousarray(np.asarray(dy, dtype=np.float64)).reshape(x.shape)
    N, C = x.shape[0], x.shape[1]
    HW = int(np.prod(x.shape[2:]))
    gamma, beta, mean, var = _f64(gamma), _f64(beta), _f64(mean), _f64(var)
    dx = np.empty_like(x)
    sc = np.empty_like(x)
    dg = np.empty(C)
    db = np.empty(C)
    rc = _load().oracle_bn_relu_bwd(N, C, HW, _ptr(x), _ptr(dy), _ptr(gamma), _ptr(beta), _ptr(mean), _ptr(var),
                                    float(eps), _ptr(dx), _ptr(dg), _ptr(db), _ptr(sc))
    if rc:
        raise ValueError(f"oracle_bn_relu_bwd failed: {rc}")
    cuts = np.cumsum([p.shape[1] for p in pieces])[:-1]
    return np.split(dx, cuts, axis=1), dg, db, np.split(sc, cuts, axis=1)


def bn_running_update(running_mean, running_var, mean, var, n: int, momentum: float = 0.1):
    """Running statistics after one training step: returns new (running_mean,
    running_var) from the batch mean and biased variance over n values per
    channel (the unbiased variance var n / (n - 1) enters running_var)."""
    rm, rv = _f64(running_mean).copy(), _f64(running_var).copy()
    mean, var = _f64(mean), _f64(var)
    rc = _load().oracle_bn_running_update(rm.size, int(n), _ptr(mean), _ptr(var), float(momentum), _ptr(rm), _ptr(rv))
    if rc:
        raise ValueError(f"oracle_bn_running_update failed: {rc}")
    return rm, rv


def round_bf16(v) -> np.ndarray:
    """Nearest bf16 (ties to even) of each double, as uint16 bit patterns."""
    v = _f64(v)
    out = np.empty(v.shape, dtype=np.uint16)
    _load().oracle_round_bf16(_ptr(v), _ptr(out, ctypes.c_uint16), v.size)
    return out


def round_f32(v) -> np.ndarray:
    """Nearest binary32 (ties to even) of each double."""
    v = _f64(v)
    out = np.empty(v.shape, dtype=np.float32)
    _load().oracle_round_f32(_ptr(v), _ptr(out, ctypes.c_float), v.size)
    return out
