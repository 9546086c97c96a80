"""Pins for the oracle's storage rounding (double -> bf16 / fp32, ties to even).

bf16 is pinned against PyTorch's float32 -> bfloat16 cast (round to nearest
even) on every double that is exactly a float32, against hand-built ties and
boundary values from the format's definition (8 exponent bits, bias 127,
7 stored mantissa bits), and on doubles that are not float32 values, where a
two-step double -> float -> bf16 rounding would go wrong.  fp32 is pinned
against numpy's cast.
"""
import numpy as np
import torch

import oracle
from memory_efficient_activation_b200 import synthetic


def _bits_of_torch_bf16(f32: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(f32.astype(np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_bf16_matches_torch_on_float32_values():
    rng = np.random.Generator(np.random.Philox(key=[41, 0]))
    # random float32 bit patterns across the whole finite range, subnormals included
    bits = rng.integers(0, 1 << 32, size=400000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    np.testing.assert_array_equal(oracle.round_bf16(f.astype(np.float64)), _bits_of_torch_bf16(f))


def test_bf16_ties_to_even_and_boundaries():
    cases = [
        (1.0 + 2.0 ** -8, 0x3F80),               # tie between 1 and 1+2^-7 -> even (1)
        (1.0 + 3 * 2.0 ** -8, 0x3F82),           # tie between 1+2^-7 and 1+2^-6 -> even (1+2^-6)
        (-1.0 - 2.0 ** -8, 0xBF80),
        (2.0 ** -126, 0x0080),                   # smallest normal
        (2.0 ** -133, 0x0001),                   # smallest subnormal
        (2.0 ** -134, 0x0000),                   # tie between 0 and 2^-133 -> even (0)
        (3 * 2.0 ** -134, 0x0002),               # tie between 2^-133 and 2^-132 -> even
        (255.0 * 2.0 ** 120, 0x7F7F),            # largest finite
        ((2.0 - 2.0 ** -8) * 2.0 ** 127, 0x7F80),  # tie above the largest -> even -> inf
        (1e39, 0x7F80),
        (-1e39, 0xFF80),
        (0.0, 0x0000),
        (-0.0, 0x8000),
        (float("inf"), 0x7F80),
    ]
    v = np.array([c[0] for c in cases])
    np.testing.assert_array_equal(oracle.round_bf16(v), np.array([c[1] for c in cases], dtype=np.uint16))
    assert oracle.round_bf16([np.nan])[0] & 0x7FFF > 0x7F80


def test_bf16_rounds_doubles_directly():
    # 1 + 2^-8 + 2^-30 lies just above the tie, so it rounds up to 1 + 2^-7.
    # A detour through float32 would land exactly on the tie and go to 1.
    v = np.array([1.0 + 2.0 ** -8 + 2.0 ** -30, -(1.0 + 2.0 ** -8 + 2.0 ** -30),
                  1.0 + 2.0 ** -8 - 2.0 ** -30])
    np.testing.assert_array_equal(oracle.round_bf16(v), np.array([0x3F81, 0xBF81, 0x3F80], dtype=np.uint16))


def test_bf16_of_all_finite_bf16_values_is_identity():
    b = synthetic.all_finite_bf16()
    v = b.to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_bf16(v), b.view(torch.int16).numpy().view(np.uint16))


def test_f32_matches_numpy():
    v = synthetic.normal_f64(100000, 10.0, 42, 0) * np.exp(synthetic.normal_f64(100000, 20.0, 42, 1))
    np.testing.assert_array_equal(oracle.round_f32(v), v.astype(np.float32))
