"""Pins the byte/FLOP accounting the benchmark uses against the worked example
in "What activations cost, in memory and in arithmetic" (problem B07), stored
in tests/golden/p3_sizing.txt with its citation."""
import os

import pytest

from memory_efficient_activation_b200 import accounting as acc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "p3_sizing.txt")


def _golden():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split()
            vals[k] = float(v)
    return vals


def test_sizing_matches_worked_example():
    g = _golden()
    shape = (int(g["B"]), int(g["T"]), int(g["d"]))
    n = acc.elements(shape)
    assert n == int(g["elements"])
    assert round(acc.tensor_bytes(n, "bf16") / 1e6, 1) == g["bf16_MB"]
    assert round(acc.tensor_bytes(n, "f32") / 1e6, 1) == g["f32_MB"]
    L = int(g["L"])
    assert round(L * acc.tensor_bytes(n, "bf16") / 1e9, 2) == g["bf16_L_GB"]
    assert round(L * acc.tensor_bytes(n, "f32") / 1e9, 2) == g["f32_L_GB"]
    # bf16 is exactly half of fp32
    assert 2 * acc.tensor_bytes(n, "bf16") == acc.tensor_bytes(n, "f32")


def test_flops_match_worked_example():
    g = _golden()
    n = int(g["elements"])
    d = int(g["d"])
    mm = acc.matmul_flops(n, d)
    assert round(mm / 1e9, 1) == g["matmul_GFLOP"]
    ge = acc.activation_flops(n, "gelu_erf")
    assert round(ge / 1e9, 2) == g["gelu_erf_GFLOP"]
    assert ge == max(acc.activation_flops(n, a) for a in acc.FLOPS_PER_ELEMENT)
    assert round(2 * d / acc.FLOPS_PER_ELEMENT["gelu_erf"]) == g["ratio_exact"]
    assert mm // ge == g["ratio_floor"]
    assert acc.arithmetic_intensity("relu", "bf16") == g["relu_bf16_flop_per_byte"]


def test_path_bytes():
    n = 67108864
    assert acc.fwd_bytes(n, "bf16") == 4 * n
    assert acc.bwd_bytes(n, "bf16") == 6 * n
    assert acc.step_bytes(n, "bf16") == 671088640
    assert acc.step_bytes(n, "f32") == 20 * n
    # one saved tensor instead of three: 134.2 MB kept, 268.4 MB saved per layer
    assert acc.saved_bytes_per_layer(n, "bf16") == 134217728
    assert acc.saved_bytes_per_layer(n, "bf16", naive=True) - acc.saved_bytes_per_layer(n, "bf16") \
        == 268435456


def test_unknown_dtype_rejected():
    with pytest.raises(KeyError):
        acc.tensor_bytes(10, "fp8")
