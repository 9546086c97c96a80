"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module holds no arithmetic of the method: it only draws random numbers
and casts them to the storage dtype.  Both the CUDA path and the oracle consume
the tensors it returns, so neither side generates its own inputs.

Generator: numpy's Philox4x32-10 counter-based bit generator (Salmon et al.,
"Parallel random numbers: as easy as 1, 2, 3", SC 2011).  Each logical stream
uses the 128-bit key (seed, stream) with the counter starting at zero, so x
and dy of one workload never share random numbers.  Values are drawn in
float64 (numpy's Generator.normal / Generator.uniform) and cast to the storage
dtype with torch's CPU cast, which rounds to nearest.

The workload recipes below follow the shapes and value distributions of the
configurations the path is measured on (an [8, 2048, 4096] transformer-scale
activation, EfficientNet-B0-like NCHW feature maps at batch 64, and an
NHWC [128, 56, 56, 144] per-channel affine + Swish).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

# Stream ids (second word of the Philox key).
STREAM_X = 0
STREAM_DY = 1
STREAM_PARAM = 2
STREAM_GAMMA = 3
STREAM_BETA = 4

_TORCH_DTYPES = {"bf16": torch.bfloat16, "f32": torch.float32}


def _gen(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=[int(seed), int(stream)]))


def normal_f64(n: int, sigma: float, seed: int, stream: int, mean: float = 0.0) -> np.ndarray:
    """n draws of N(mean, sigma^2) in float64."""
    return _gen(seed, stream).normal(mean, sigma, size=int(n))


def uniform_f64(n: int, lo: float, hi: float, seed: int, stream: int) -> np.ndarray:
    """n draws of U(lo, hi) in float64."""
    return _gen(seed, stream).uniform(lo, hi, size=int(n))


def to_storage(a: np.ndarray, dtype: str) -> torch.Tensor:
    """Cast float64 values to the storage dtype ('bf16' or 'f32') on the CPU."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64)).to(_TORCH_DTYPES[dtype])


def normal(n: int, sigma: float, seed: int, stream: int, dtype: str) -> torch.Tensor:
    return to_storage(normal_f64(n, sigma, seed, stream), dtype)


def all_finite_bf16() -> torch.Tensor:
    """Every finite bf16 value (both zeros included), as a bf16 tensor."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    exp = (bits >> 7) & 0xFF
    bits = bits[exp != 0xFF]
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)


def f32_grid(count: int, lo: float, hi: float) -> torch.Tensor:
    """count evenly spaced float32 values covering [lo, hi] (np.linspace in double, then cast)."""
    return torch.from_numpy(np.linspace(lo, hi, int(count), dtype=np.float64)).to(torch.float32)


# --------------------------------------------------------------------------
# Workload recipes
# --------------------------------------------------------------------------

ACTIVATIONS = ("relu", "leaky_relu", "sigmoid", "tanh", "gelu_erf", "gelu_tanh", "swish")

# EfficientNet-B0-like NCHW feature maps at batch 64.
EFFNET_B0_SHAPES = (
    (64, 32, 112, 112),
    (64, 96, 112, 112),
    (64, 144, 56, 56),
    (64, 240, 28, 28),
    (64, 480, 14, 14),
    (64, 1152, 7, 7),
)

TRANSFORMER_SHAPE = (8, 2048, 4096)
AFFINE_NHWC_SHAPE = (128, 56, 56, 144)   # N, H, W, C in memory order


@dataclass
class Workload:
    """One synthetic workload: its tensors (CPU) and its scalar parameters."""
    name: str
    act: str
    dtype: str
    x: torch.Tensor
    dy: torch.Tensor
    param: float = 1.0
    extra: dict = field(default_factory=dict)

    @property
    def n(self) -> int:
        return self.x.numel()


def swish_f32_1m(seed: int = 0) -> Workload:
    """Swish alpha=1, fp32, 1-D tensor of 1,048,576 elements, x ~ N(0, 3^2), dy ~ N(0, 1)."""
    n = 1 << 20
    return Workload("swish_f32_1m", "swish", "f32",
                    normal(n, 3.0, seed, STREAM_X, "f32"),
                    normal(n, 1.0, seed, STREAM_DY, "f32"), 1.0)


def swish_bf16_transformer(seed: int = 1, shape=TRANSFORMER_SHAPE, act: str = "swish",
                           sigma_x: float = 1.0) -> Workload:
    """Swish alpha=1, bf16 storage, [8, 2048, 4096] (67,108,864 elements), x, dy ~ N(0, 1)."""
    n = int(np.prod(shape))
    return Workload(f"{act}_bf16_{'x'.join(map(str, shape))}", act, "bf16",
                    normal(n, sigma_x, seed, STREAM_X, "bf16").view(shape),
                    normal(n, 1.0, seed, STREAM_DY, "bf16").view(shape),
                    1.0)


def family_bf16(act: str, seed: int = 2, shape=TRANSFORMER_SHAPE) -> Workload:
    """Family sweep member on [8, 2048, 4096] bf16, x ~ N(0, 2^2), dy ~ N(0, 1).
    LeakyReLU uses slope 0.01; Swish uses alpha 1."""
    w = swish_bf16_transformer(seed=seed, shape=shape, act=act, sigma_x=2.0)
    w.param = 0.01 if act == "leaky_relu" else 1.0
    return w


def effnet_swish_f32(shape_index: int, seed: int = 3, shape=None) -> Workload:
    """EfficientNet-B0-like NCHW fp32 feature map, x ~ N(0, 1.5^2), dy ~ N(0, 1),
    learnable scalar alpha ~ U(0.5, 2) (one draw per shape)."""
    if shape is None:
        shape = EFFNET_B0_SHAPES[shape_index]
    n = int(np.prod(shape))
    s = seed * 16 + shape_index
    alpha = float(np.float32(uniform_f64(1, 0.5, 2.0, s, STREAM_PARAM)[0]))
    return Workload(f"swish_f32_nchw_{'x'.join(map(str, shape))}", "swish", "f32",
                    normal(n, 1.5, s, STREAM_X, "f32").view(shape),
                    normal(n, 1.0, s, STREAM_DY, "f32").view(shape),
                    alpha)


def affine_swish_nhwc(seed: int = 4, shape=AFFINE_NHWC_SHAPE, dtype: str = "bf16") -> Workload:
    """Fused per-channel affine + Swish, NHWC, x, dy ~ N(0, 1), gamma ~ U(0.5, 1.5),
    beta ~ N(0, 0.1^2) (fp32 parameters).  shape is (N, H, W, C) in memory order."""
    N, H, W, C = shape
    n = N * H * W * C
    gamma = torch.from_numpy(uniform_f64(C, 0.5, 1.5, seed, STREAM_GAMMA)).to(torch.float32)
    beta = torch.from_numpy(normal_f64(C, 0.1, seed, STREAM_BETA)).to(torch.float32)
    return Workload(f"affine_swish_nhwc_{'x'.join(map(str, shape))}", "affine_swish", dtype,
                    normal(n, 1.0, seed, STREAM_X, dtype).view(shape),
                    normal(n, 1.0, seed, STREAM_DY, dtype).view(shape),
                    1.0, {"gamma": gamma, "beta": beta, "layout": "nhwc",
                          "nchw_shape": (N, C, H, W)})


def affine_swish_nchw(seed: int = 5, shape=(64, 144, 56, 56), dtype: str = "bf16") -> Workload:
    """Fused per-channel affine + Swish, NCHW, same distributions as the NHWC recipe.
    shape is (N, C, H, W) in memory order."""
    N, C, H, W = shape
    n = N * C * H * W
    gamma = torch.from_numpy(uniform_f64(C, 0.5, 1.5, seed, STREAM_GAMMA)).to(torch.float32)
    beta = torch.from_numpy(normal_f64(C, 0.1, seed, STREAM_BETA)).to(torch.float32)
    return Workload(f"affine_swish_nchw_{'x'.join(map(str, shape))}", "affine_swish", dtype,
                    normal(n, 1.0, seed, STREAM_X, dtype).view(shape),
                    normal(n, 1.0, seed, STREAM_DY, dtype).view(shape),
                    1.0, {"gamma": gamma, "beta": beta, "layout": "nchw",
                          "nchw_shape": (N, C, H, W)})


def affine_act_nhwc(act: str, seed: int = 6, shape=AFFINE_NHWC_SHAPE, dtype: str = "bf16") -> Workload:
    """Fused per-channel affine + any activation of the family, NHWC, with the
    distributions of the affine + Swish recipe (LeakyReLU slope 0.01, Swish
    alpha 1)."""
    w = affine_swish_nhwc(seed=seed, shape=shape, dtype=dtype)
    w.name = w.name.replace("affine_swish", f"affine_{act}")
    w.act = act
    w.param = 0.01 if act == "leaky_relu" else 1.0
    return w


def swish_channel_nchw(seed: int = 7, shape=(64, 144, 56, 56), dtype: str = "f32") -> Workload:
    """Swish with a learnable alpha per channel, NCHW (N, C, H, W), x ~ N(0, 1.5^2),
    dy ~ N(0, 1), alpha_c ~ U(0.5, 2) (fp32, one draw per channel)."""
    N, C, H, W = shape
    n = N * C * H * W
    alpha = torch.from_numpy(uniform_f64(C, 0.5, 2.0, seed, STREAM_PARAM)).to(torch.float32)
    return Workload(f"swish_channel_nchw_{'x'.join(map(str, shape))}", "swish_channel", dtype,
                    normal(n, 1.5, seed, STREAM_X, dtype).view(shape),
                    normal(n, 1.0, seed, STREAM_DY, dtype).view(shape),
                    1.0, {"alpha": alpha, "layout": "nchw", "nchw_shape": (N, C, H, W)})
