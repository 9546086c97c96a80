"""Byte, FLOP and saved-memory accounting for the activation path.

Host-side arithmetic only (no kernels).  The benchmark uses it to turn a
measured time into algorithmic GB/s and a roofline fraction; the tests pin it
against the worked example in "What activations cost, in memory and in
arithmetic" (asifuddin.com, problem B07: GIVEN, SOLUTION steps 1-4, Check).

Algorithmic bytes per element (b = bytes of the storage dtype):
  forward  reads x, writes y            -> 2 b
  backward reads x and dy, writes dx    -> 3 b
The save-input-only contract keeps one tensor (x) per layer for the backward;
the plain autograd graph of x * Sigmoid(alpha x) keeps three featuremaps
(x, Sigmoid(alpha x) and the output), as counted in "Memory efficient Swish",
section "Why simple Swish implementation is inefficient?".
"""
from __future__ import annotations

import math

DTYPE_BYTES = {"bf16": 2, "f32": 4}

# Approximate FLOPs per element, from problem B07's GIVEN.  Swish is not on
# that list; x * Sigmoid(alpha x) is read as one sigmoid (4) plus one multiply.
FLOPS_PER_ELEMENT = {
    "relu": 1,
    "leaky_relu": 2,
    "sigmoid": 4,
    "tanh": 6,
    "gelu_erf": 12,
    "gelu_tanh": 8,
    "swish": 5,
}

SAVED_TENSORS_NAIVE_SWISH = 3
SAVED_TENSORS_SAVE_INPUT_ONLY = 1


def elements(shape) -> int:
    return int(math.prod(int(s) for s in shape))


def tensor_bytes(n: int, dtype: str) -> int:
    return int(n) * DTYPE_BYTES[dtype]


def fwd_bytes(n: int, dtype: str) -> int:
    """Algorithmic HBM bytes of one forward: read x, write y."""
    return 2 * tensor_bytes(n, dtype)


def bwd_bytes(n: int, dtype: str) -> int:
    """Algorithmic HBM bytes of one backward: read x and dy, write dx."""
    return 3 * tensor_bytes(n, dtype)


def step_bytes(n: int, dtype: str) -> int:
    """Forward plus backward."""
    return fwd_bytes(n, dtype) + bwd_bytes(n, dtype)


def affine_fwd_bytes(n: int, dtype: str, channels: int) -> int:
    """Fused affine + activation forward: x in, y out, plus gamma and beta (fp32)."""
    return 2 * tensor_bytes(n, dtype) + 2 * 4 * channels


def affine_bwd_bytes(n: int, dtype: str, channels: int) -> int:
    """Fused affine + activation backward: x, dy in, dx out, gamma, beta in,
    dgamma, dbeta out (fp32)."""
    return 3 * tensor_bytes(n, dtype) + 4 * 4 * channels


def channel_swish_fwd_bytes(n: int, dtype: str, channels: int) -> int:
    """Swish with a per-channel alpha, forward: x in, y out, alpha in (fp32)."""
    return 2 * tensor_bytes(n, dtype) + 4 * channels


def channel_swish_bwd_bytes(n: int, dtype: str, channels: int) -> int:
    """Swish with a per-channel alpha, backward: x, dy in, dx out, alpha in,
    dalpha out (fp32)."""
    return 3 * tensor_bytes(n, dtype) + 2 * 4 * channels


def saved_bytes_per_layer(n: int, dtype: str, naive: bool = False) -> int:
    k = SAVED_TENSORS_NAIVE_SWISH if naive else SAVED_TENSORS_SAVE_INPUT_ONLY
    return k * tensor_bytes(n, dtype)


def activation_flops(n: int, act: str) -> int:
    return FLOPS_PER_ELEMENT[act] * int(n)


def matmul_flops(n: int, d: int) -> int:
    """One d x d matrix multiply applied to an (n / d) x d activation: 2 n d."""
    return 2 * int(n) * int(d)


def arithmetic_intensity(act: str, dtype: str) -> float:
    """FLOPs per byte when the activation reads and writes each element once."""
    return FLOPS_PER_ELEMENT[act] / (2 * DTYPE_BYTES[dtype])
