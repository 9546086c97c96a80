"""Host-side checks of the C ABI (no GPU needed).

The library loads, exports every function include/mea.h declares with the
enumerations the binding uses, and rejects invalid calls synchronously with
the documented status codes before any CUDA call.  Pointer arguments here
are fake addresses: every call below is refused during validation.
"""
import os
import re

import pytest

from memory_efficient_activation_b200 import _capi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mea.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _capi.lib()


def _header_functions():
    src = open(HEADER).read()
    return re.findall(r"MEA_API\s+[\w\s\*]+?\b(mea_\w+)\s*\(", src)


def _header_enum(name):
    src = open(HEADER).read()
    return {k: int(v) for k, v in re.findall(r"\b(" + name + r"\w*)\s*=\s*(\d+)", src)}


def test_every_declared_symbol_is_exported(lib):
    declared = _header_functions()
    assert len(declared) == 30, declared
    for fn in declared:
        assert hasattr(lib, fn), fn
        assert fn in _capi.SIGNATURES, fn
    assert set(_capi.SIGNATURES) == set(declared)


def test_enums_match_header():
    acts = _header_enum("MEA_")
    for name, val in [("MEA_RELU", _capi.MEA_RELU), ("MEA_LEAKY_RELU", _capi.MEA_LEAKY_RELU),
                      ("MEA_SIGMOID", _capi.MEA_SIGMOID), ("MEA_TANH", _capi.MEA_TANH),
                      ("MEA_GELU_ERF", _capi.MEA_GELU_ERF), ("MEA_GELU_TANH", _capi.MEA_GELU_TANH),
                      ("MEA_SWISH", _capi.MEA_SWISH), ("MEA_F32", _capi.MEA_F32), ("MEA_BF16", _capi.MEA_BF16),
                      ("MEA_NCHW", _capi.MEA_NCHW), ("MEA_NHWC", _capi.MEA_NHWC), ("MEA_OK", _capi.MEA_OK),
                      ("MEA_ERR_INVALID_ARG", _capi.MEA_ERR_INVALID_ARG),
                      ("MEA_ERR_UNSUPPORTED", _capi.MEA_ERR_UNSUPPORTED),
                      ("MEA_ERR_WORKSPACE", _capi.MEA_ERR_WORKSPACE), ("MEA_ERR_CUDA", _capi.MEA_ERR_CUDA)]:
        assert acts[name] == val, name


def test_version_and_status_strings(lib):
    assert lib.mea_version() == 10300
    for st in range(5):
        assert lib.mea_status_string(st)
    assert lib.mea_status_string(99) == b"unknown status"


X, Y, G, D = 0x100000, 0x200000, 0x300000, 0x400000


def test_fwd_validation(lib):
    f = lib.mea_act_fwd
    assert f(7, 1, X, Y, 10, 1.0, None, None) == _capi.MEA_ERR_INVALID_ARG
    assert b"act" in lib.mea_last_error()
    assert f(-1, 1, X, Y, 10, 1.0, None, None) == _capi.MEA_ERR_INVALID_ARG
    assert f(6, 2, X, Y, 10, 1.0, None, None) == _capi.MEA_ERR_INVALID_ARG
    assert f(6, 1, X, Y, -1, 1.0, None, None) == _capi.MEA_ERR_INVALID_ARG
    assert f(6, 1, None, Y, 10, 1.0, None, None) == _capi.MEA_ERR_INVALID_ARG
    assert f(6, 1, X, None, 10, 1.0, None, None) == _capi.MEA_ERR_INVALID_ARG
    # y may not overlap x at all (x is the saved tensor)
    assert f(6, 1, X, X, 10, 1.0, None, None) == _capi.MEA_ERR_INVALID_ARG
    assert f(6, 1, X, X + 18, 10, 1.0, None, None) == _capi.MEA_ERR_INVALID_ARG
    assert f(6, 0, X, X + 36, 10, 1.0, None, None) == _capi.MEA_ERR_INVALID_ARG
    # n = 0 is a no-op, even with NULL pointers
    assert f(6, 1, None, None, 0, 1.0, None, None) == _capi.MEA_OK
    assert lib.mea_last_error() == b""


def test_bwd_validation(lib):
    b = lib.mea_act_bwd
    ok_ws = lib.mea_act_bwd_workspace_bytes(6, 1000, 1)
    assert b(6, 1, X, G, D, -5, 1.0, None, None, None, 0, None) == _capi.MEA_ERR_INVALID_ARG
    assert b(6, 1, X, None, D, 5, 1.0, None, None, None, 0, None) == _capi.MEA_ERR_INVALID_ARG
    # d alpha only for Swish
    assert b(0, 1, X, G, D, 5, 1.0, None, 0x500000, 0x600000, ok_ws, None) == _capi.MEA_ERR_UNSUPPORTED
    # workspace missing / small / misaligned
    assert b(6, 1, X, G, D, 1000, 1.0, None, 0x500000, None, ok_ws, None) == _capi.MEA_ERR_WORKSPACE
    assert b(6, 1, X, G, D, 1000, 1.0, None, 0x500000, 0x600000, ok_ws - 1, None) == _capi.MEA_ERR_WORKSPACE
    assert b(6, 1, X, G, D, 1000, 1.0, None, 0x500000, 0x600008, ok_ws, None) == _capi.MEA_ERR_WORKSPACE
    # partial overlap of dx with dy or x is refused; exact aliasing is not checked here
    assert b(6, 1, X, G, G + 2, 100, 1.0, None, None, None, 0, None) == _capi.MEA_ERR_INVALID_ARG
    assert b(6, 1, X, G, X + 64, 100, 1.0, None, None, None, 0, None) == _capi.MEA_ERR_INVALID_ARG
    assert b(6, 1, None, None, None, 0, 1.0, None, None, None, 0, None) == _capi.MEA_OK


def test_workspace_sizes(lib):
    w = lib.mea_act_bwd_workspace_bytes
    assert w(6, 1000, 0) == 0
    assert w(6, 0, 1) == 256 + 8
    assert w(6, 8192, 1) == 256 + 8
    assert w(6, 8193, 1) == 256 + 16
    assert w(6, 1 << 40, 1) == 256 + 8 * 444
    aw = lib.mea_affine_swish_bwd_workspace_bytes
    assert aw(1, 1, _capi.shape4((128, 144, 56, 56))) >= 256 + 16 * 144
    assert aw(1, 0, _capi.shape4((64, 32, 112, 112))) >= 256 + 16 * 32
    assert aw(1, 1, _capi.shape4((1, -1, 1, 1))) == 0
    assert aw(1, 5, _capi.shape4((1, 1, 1, 1))) == 0
    assert aw(3, 1, _capi.shape4((1, 1, 1, 1))) == 0


def test_affine_validation(lib):
    s = _capi.shape4((2, 16, 3, 3))
    fw = lib.mea_affine_swish_fwd
    assert fw(1, 2, s, X, G, D, Y, None) == _capi.MEA_ERR_INVALID_ARG
    assert fw(1, 1, None, X, G, D, Y, None) == _capi.MEA_ERR_INVALID_ARG
    assert fw(1, 1, _capi.shape4((2, -16, 3, 3)), X, G, D, Y, None) == _capi.MEA_ERR_INVALID_ARG
    assert fw(1, 1, s, X, None, D, Y, None) == _capi.MEA_ERR_INVALID_ARG
    assert fw(1, 1, s, X, G, D, X + 2, None) == _capi.MEA_ERR_INVALID_ARG
    assert fw(1, 1, _capi.shape4((0, 16, 3, 3)), None, None, None, None, None) == _capi.MEA_OK
    bw = lib.mea_affine_swish_bwd
    need = lib.mea_affine_swish_bwd_workspace_bytes(1, 1, s)
    assert bw(1, 1, s, X, G, 0x700000, 0x710000, D, 0x720000, 0x730000, None, need, None) \
        == _capi.MEA_ERR_WORKSPACE
    assert bw(1, 1, s, X, G, 0x700000, 0x710000, D, 0x720000, 0x730000, 0x800000, need - 8, None) \
        == _capi.MEA_ERR_WORKSPACE
    assert bw(1, 1, s, X, G, 0x700000, 0x710000, D, 0x720000, 0x720010, 0x800000, need, None) \
        == _capi.MEA_ERR_INVALID_ARG
    assert bw(1, 1, s, X, G, None, 0x710000, D, 0x720000, 0x730000, 0x800000, need, None) \
        == _capi.MEA_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors():
    import torch
    import memory_efficient_activation_b200 as mea
    with pytest.raises(ValueError):
        mea.act_fwd("swish", torch.zeros(4))
    with pytest.raises(ValueError):
        mea.act_fwd("softplus", torch.zeros(4))


def test_affine_act_and_channel_validation(lib):
    s = _capi.shape4((2, 16, 3, 3))
    fa = lib.mea_affine_act_fwd
    assert fa(7, 1, 1, s, X, G, D, 1.0, Y, None) == _capi.MEA_ERR_INVALID_ARG
    assert b"act" in lib.mea_last_error()
    assert fa(0, 1, 1, s, X, G, None, 1.0, Y, None) == _capi.MEA_ERR_INVALID_ARG
    assert fa(0, 1, 1, s, X, G, D, 1.0, X + 4, None) == _capi.MEA_ERR_INVALID_ARG
    assert fa(0, 1, 1, _capi.shape4((0, 16, 3, 3)), None, None, None, 1.0, None, None) == _capi.MEA_OK
    ba = lib.mea_affine_act_bwd
    need = lib.mea_affine_act_bwd_workspace_bytes(1, 1, s)
    assert need == lib.mea_affine_swish_bwd_workspace_bytes(1, 1, s)
    assert ba(9, 1, 1, s, X, G, 0x700000, 0x710000, 0.1, D, 0x720000, 0x730000, 0x800000, need, None) \
        == _capi.MEA_ERR_INVALID_ARG
    assert ba(1, 1, 1, s, X, G, 0x700000, 0x710000, 0.1, D, 0x720000, 0x730000, 0x800008, need, None) \
        == _capi.MEA_ERR_WORKSPACE
    assert ba(1, 1, 1, s, X, G, 0x700000, 0x710000, 0.1, D, 0x720000, None, 0x800000, need, None) \
        == _capi.MEA_ERR_INVALID_ARG
    # zero channels: nothing to write, even without buffers
    assert ba(1, 1, 1, _capi.shape4((2, 0, 3, 3)), None, None, None, None, 0.1, None, None, None, None, 0,
              None) == _capi.MEA_OK
    fc = lib.mea_swish_channel_fwd
    assert fc(1, 1, s, X, None, Y, None) == _capi.MEA_ERR_INVALID_ARG
    assert fc(1, 3, s, X, G, Y, None) == _capi.MEA_ERR_INVALID_ARG
    assert fc(1, 1, s, X, G, X, None) == _capi.MEA_ERR_INVALID_ARG
    bc = lib.mea_swish_channel_bwd
    cneed = lib.mea_swish_channel_bwd_workspace_bytes(1, 1, s)
    # one reduction per channel instead of two: a smaller workspace
    assert 256 + 8 * 16 <= cneed < need
    assert bc(1, 1, s, X, G, 0x700000, D, None, 0x800000, cneed, None) == _capi.MEA_ERR_INVALID_ARG
    assert bc(1, 1, s, X, G, 0x700000, D, 0x720000, 0x800000, cneed - 1, None) == _capi.MEA_ERR_WORKSPACE
    assert bc(1, 1, s, X, G, 0x700000, G + 2, 0x720000, 0x800000, cneed, None) == _capi.MEA_ERR_INVALID_ARG
    assert lib.mea_swish_channel_bwd_workspace_bytes(1, 1, _capi.shape4((1, -2, 1, 1))) == 0


def test_matmul_validation(lib):
    f, b = lib.mea_matmul_act_fwd, lib.mea_matmul_act_bwd
    A, Wt, Z, Yo = 0x1000000, 0x2000000, 0x3000000, 0x4000000
    assert f(9, 16, 16, 16, A, Wt, 1.0, Z, Yo, None) == _capi.MEA_ERR_INVALID_ARG
    assert f(0, -1, 16, 16, A, Wt, 1.0, Z, Yo, None) == _capi.MEA_ERR_INVALID_ARG
    assert f(0, 0, 16, 16, None, None, 1.0, None, None, None) == _capi.MEA_OK      # empty: no-op
    assert f(0, 16, 16, 0, A, Wt, 1.0, Z, Yo, None) == _capi.MEA_ERR_UNSUPPORTED  # K = 0
    assert f(0, 16, 12, 16, A, Wt, 1.0, Z, Yo, None) == _capi.MEA_ERR_UNSUPPORTED # N % 8
    assert f(0, 16, 16, 20, A, Wt, 1.0, Z, Yo, None) == _capi.MEA_ERR_UNSUPPORTED # K % 8
    assert f(0, 16, 16, 16, A + 8, Wt, 1.0, Z, Yo, None) == _capi.MEA_ERR_UNSUPPORTED
    assert f(0, 16, 16, 16, A, Wt, 1.0, None, None, None) == _capi.MEA_ERR_INVALID_ARG
    assert f(0, 16, 16, 16, A, Wt, 1.0, A + 256, None, None) == _capi.MEA_ERR_INVALID_ARG  # z overlaps x
    assert f(0, 16, 16, 16, A, Wt, 1.0, Z, Z + 256, None) == _capi.MEA_ERR_INVALID_ARG     # z overlaps y
    assert f(0, 1 << 31, 16, 16, A, Wt, 1.0, Z, Yo, None) == _capi.MEA_ERR_UNSUPPORTED
    assert b(0, 16, 16, 16, A, Wt, Z, 1.0, None, None) == _capi.MEA_ERR_INVALID_ARG
    assert b(0, 16, 16, 16, A, Wt, Z, 1.0, Z + 16, None) == _capi.MEA_ERR_INVALID_ARG      # partial overlap
    assert b(0, 16, 16, 16, A, Wt, Z, 1.0, Wt, None) == _capi.MEA_ERR_INVALID_ARG          # dz overlaps w


def test_concat_bn_validation(lib):
    P = _capi.ptr_array([0x1000000, 0x2000000])
    ch = _capi.int64_array([3, 5])
    f = lib.mea_concat_bn_relu_fwd
    ws = lib.mea_concat_bn_relu_workspace_bytes(4, 8)
    assert ws >= 256 + 16 * 8
    assert lib.mea_concat_bn_relu_workspace_bytes(0, 8) == 0
    G, B, Mu, Is, Yb, Wk = 0x3000000, 0x3100000, 0x3200000, 0x3300000, 0x4000000, 0x5000000
    assert f(1, 0, P, ch, 4, 9, G, B, 1e-5, 0.1, None, None, Mu, Is, Yb, Wk, ws, None) == _capi.MEA_ERR_UNSUPPORTED
    assert f(1, 129, P, ch, 4, 9, G, B, 1e-5, 0.1, None, None, Mu, Is, Yb, Wk, ws, None) == _capi.MEA_ERR_UNSUPPORTED
    assert f(1, 2, P, ch, 0, 9, G, B, 1e-5, 0.1, None, None, Mu, Is, Yb, Wk, ws, None) == _capi.MEA_ERR_INVALID_ARG
    assert f(1, 2, P, _capi.int64_array([3, 0]), 4, 9, G, B, 1e-5, 0.1, None, None, Mu, Is, Yb, Wk, ws, None) \
        == _capi.MEA_ERR_INVALID_ARG
    assert f(1, 2, P, ch, 4, 9, G, B, 1e-5, 0.1, 0x6000000, None, Mu, Is, Yb, Wk, ws, None) == _capi.MEA_ERR_INVALID_ARG
    assert f(1, 2, P, ch, 4, 9, G, B, 1e-5, 0.1, None, None, Mu, Is, Yb, Wk, ws - 1, None) == _capi.MEA_ERR_WORKSPACE
    # y overlapping a piece
    assert f(1, 2, P, ch, 4, 9, G, B, 1e-5, 0.1, None, None, Mu, Is, 0x2000010, Wk, ws, None) \
        == _capi.MEA_ERR_INVALID_ARG
    b = lib.mea_concat_bn_relu_bwd
    D = _capi.ptr_array([0x7000000, 0x7000040])      # dpieces overlapping each other
    assert b(1, 2, P, ch, 4, 9, Yb, G, B, Mu, Is, D, 0, 0x3400000, 0x3500000, Wk, ws, None) \
        == _capi.MEA_ERR_INVALID_ARG
    D = _capi.ptr_array([0x1000000 + 2, 0x8000000])  # partial overlap with its own piece
    assert b(1, 2, P, ch, 4, 9, Yb, G, B, Mu, Is, D, 0, 0x3400000, 0x3500000, Wk, ws, None) \
        == _capi.MEA_ERR_INVALID_ARG


def test_host_pipeline_validates_outputs():
    import torch
    import memory_efficient_activation_b200 as mea
    # results are copied into the flat view of hy / hdx: a tensor whose
    # reshape would be a copy (non-contiguous), or of another size or dtype,
    # is refused before any device work
    x = torch.zeros(64, dtype=torch.bfloat16)
    dy = torch.zeros(64, dtype=torch.bfloat16)
    bad = [torch.zeros(128, dtype=torch.bfloat16)[::2],          # non-contiguous
           torch.zeros(63, dtype=torch.bfloat16),
           torch.zeros(64, dtype=torch.float32)]
    for b in bad:
        with pytest.raises(ValueError):
            mea.act_fwd_bwd_host("swish", x, dy, hy=b)
        with pytest.raises(ValueError):
            mea.act_fwd_bwd_host("swish", x, dy, hdx=b)
    with pytest.raises(ValueError):
        mea.act_fwd_bwd_host("swish", x, dy[:32])


def test_binding_companion_tensor_checks(monkeypatch):
    # the device-independent part of the checks on outputs and companion
    # tensors (device placement itself needs a GPU): dtype, size, contiguity
    import torch
    import memory_efficient_activation_b200 as mea
    monkeypatch.setattr(mea, "_need_cuda", lambda *ts: None)
    ref = torch.zeros(10, dtype=torch.bfloat16)
    assert mea._like(ref, torch.zeros(10, dtype=torch.bfloat16), "out") is not None
    for bad in (torch.zeros(10, dtype=torch.float32), torch.zeros(11, dtype=torch.bfloat16)):
        with pytest.raises(ValueError):
            mea._like(ref, bad, "out")
    mea._on_device(ref, torch.zeros(1), "dparam", torch.float32, 1)
    with pytest.raises(ValueError):
        mea._on_device(ref, torch.zeros(1, dtype=torch.bfloat16), "dparam", torch.float32, 1)
    with pytest.raises(ValueError):
        mea._on_device(ref, torch.zeros(0), "dparam", torch.float32, 1)
    mea._chan_params(4, torch.zeros(4), torch.zeros(4), device=torch.device("cpu"))
    with pytest.raises(ValueError):
        mea._chan_params(4, torch.zeros(5))
    with pytest.raises(ValueError):
        mea._chan_params(4, torch.zeros(4, dtype=torch.float64))


class _FakeLib:
    """Stands in for libmea.so: every entry point returns MEA_OK (0) and
    records its name, so the binding's marshalling runs on the CPU."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append(name)
            return 0
        return fn


def test_binding_call_patterns_with_stand_in_library(monkeypatch):
    # the calling patterns of the modules, tests and benchmark pass the
    # binding's checks and reach the C ABI; mismatched companions do not
    import torch
    import memory_efficient_activation_b200 as mea
    from memory_efficient_activation_b200 import _capi
    fake = _FakeLib()
    monkeypatch.setattr(_capi, "lib", lambda: fake)
    monkeypatch.setattr(mea, "_need_cuda", lambda *ts: None)
    monkeypatch.setattr(mea, "_stream", lambda t: 0)
    bf = torch.bfloat16
    x = torch.zeros(2, 4, 4, 16, dtype=bf)
    dy = torch.zeros_like(x)
    g, b = torch.ones(16), torch.zeros(16)
    a1 = torch.tensor([1.5])
    mea.act_fwd("swish", x, 1.0, out=torch.empty_like(x))
    mea.act_fwd("swish", x, 0.0, param_dev=a1)
    mea.act_bwd("swish", x, dy, 1.0, out=dy)                      # dx over dy
    mea.act_bwd("swish", x, dy, 0.0, param_dev=a1, dparam=torch.empty(1),
                workspace=torch.zeros(4096, dtype=torch.uint8))
    mea.affine_swish_fwd(x, g, b, "nhwc", out=torch.empty_like(x))
    mea.affine_swish_bwd(x, dy, g, b, "nhwc", out=torch.empty_like(x), dgamma=torch.empty(16),
                         dbeta=torch.empty(16), workspace=torch.zeros(1 << 16, dtype=torch.uint8))
    mea.affine_act_fwd("gelu_tanh", x, g, b, 1.0, "nhwc")
    mea.affine_act_bwd("gelu_tanh", x, dy, g, b, 1.0, "nhwc")
    xc = torch.zeros(2, 16, 4, 4)
    mea.swish_channel_fwd(xc, g, "nchw", out=torch.empty_like(xc))
    mea.swish_channel_bwd(xc, torch.zeros_like(xc), g, "nchw", dalpha=torch.empty(16))
    assert fake.calls.count("mea_act_fwd") == 2 and fake.calls.count("mea_act_bwd") == 2
    assert "mea_affine_swish_bwd" in fake.calls and "mea_swish_channel_bwd" in fake.calls
    n = len(fake.calls)
    for call in (
        lambda: mea.act_fwd("swish", x, 1.0, out=torch.empty(2, 4, 4, 16)),            # fp32 out for bf16 x
        lambda: mea.act_bwd("swish", x, dy, 1.0, out=torch.empty(10, dtype=bf)),        # wrong size
        lambda: mea.act_bwd("swish", x, dy, 0.0, dparam=torch.empty(1, dtype=bf)),      # bf16 d alpha
        lambda: mea.act_fwd("swish", x, 0.0, param_dev=torch.empty(0)),                # empty alpha
        lambda: mea.affine_swish_bwd(x, dy, g, b, "nhwc", dgamma=torch.empty(15)),      # dgamma size
        lambda: mea.swish_channel_bwd(xc, torch.zeros_like(xc), g, "nchw",
                                      dalpha=torch.empty(16, dtype=torch.float64)),
    ):
        with pytest.raises(ValueError):
            call()
    assert len(fake.calls) == n                     # nothing reached the library


def test_binding_matmul_and_bn_patterns_with_stand_in_library(monkeypatch):
    import torch
    import memory_efficient_activation_b200 as mea
    from memory_efficient_activation_b200 import _capi
    fake = _FakeLib()
    monkeypatch.setattr(_capi, "lib", lambda: fake)
    monkeypatch.setattr(mea, "_need_cuda", lambda *ts: None)
    monkeypatch.setattr(mea, "_stream", lambda t: 0)
    bf = torch.bfloat16
    x, w = torch.zeros(16, 8, dtype=bf), torch.zeros(24, 8, dtype=bf)
    z, y = mea.matmul_act_fwd("swish", x, w)
    assert z.shape == (16, 24) and y.shape == (16, 24)
    mea.matmul_act_fwd("swish", x, w, z=torch.empty(16, 24, dtype=bf), want_y=False)
    g = torch.zeros(16, 8, dtype=bf)
    mea.matmul_act_bwd("swish", g, w, z, out=z)                     # dz written over z
    pieces = [torch.zeros(2, 3, 4, 4), torch.zeros(2, 5, 4, 4)]
    gam, bet = torch.ones(8), torch.zeros(8)
    yb, mean, invstd = mea.concat_bn_relu_fwd(pieces, gam, bet, 1e-5, 0.1, torch.zeros(8), torch.ones(8),
                                              out=torch.empty(2, 8, 4, 4))
    mea.concat_bn_relu_apply(pieces, gam, bet, mean, invstd, out=yb)
    mea.concat_bn_relu_bwd(pieces, torch.zeros(2, 8, 4, 4), gam, bet, mean, invstd,
                           dpieces=[torch.zeros_like(p) for p in pieces], accumulate=True)
    n = len(fake.calls)
    for call in (
        lambda: mea.matmul_act_fwd("swish", x, w, z=torch.empty(16, 23, dtype=bf)),
        lambda: mea.matmul_act_bwd("swish", g, w, z, out=torch.empty(16, 24)),           # fp32 out
        lambda: mea.concat_bn_relu_fwd(pieces, gam, bet, out=torch.empty(2, 7, 4, 4)),
        lambda: mea.concat_bn_relu_fwd(pieces, gam, bet, 1e-5, 0.1, torch.zeros(7), torch.ones(8)),
        lambda: mea.concat_bn_relu_bwd(pieces, torch.zeros(2, 8, 4, 4, dtype=bf), gam, bet, mean, invstd),
        lambda: mea.concat_bn_relu_bwd(pieces, torch.zeros(2, 8, 4, 4), gam, bet, mean, invstd,
                                       dpieces=[torch.zeros_like(pieces[0])]),
    ):
        with pytest.raises(ValueError):
            call()
    assert len(fake.calls) == n


def _chan_segs(specs):
    segs = (_capi.ChannelSegment * len(specs))()
    for i, (x, dy, out, alpha, dalpha, shape) in enumerate(specs):
        segs[i] = _capi.ChannelSegment(x, dy, out, alpha, dalpha, (_capi.ctypes.c_int64 * 4)(*shape))
    return segs


def test_channel_grouped_validation(lib):
    # grouped Swish with a per-channel alpha: every refusal happens before a
    # launch (fake addresses), and the workspace is the per-segment sizes,
    # each rounded up to 256 bytes
    sh_a, sh_b = (2, 16, 7, 7), (3, 40, 14, 14)
    f = lib.mea_swish_channel_fwd_grouped
    b = lib.mea_swish_channel_bwd_grouped
    ok2 = _chan_segs([(X, None, Y, G, None, sh_a), (0x500000, None, 0x600000, 0x310000, None, sh_b)])
    assert f(1, 0, None, None) == _capi.MEA_OK
    assert f(1, -1, ok2, None) == _capi.MEA_ERR_INVALID_ARG
    assert f(1, 2, None, None) == _capi.MEA_ERR_INVALID_ARG
    assert f(7, 2, ok2, None) == _capi.MEA_ERR_INVALID_ARG
    neg = _chan_segs([(X, None, Y, G, None, sh_a), (X, None, Y, G, None, (1, -4, 2, 2))])
    assert f(1, 2, neg, None) == _capi.MEA_ERR_INVALID_ARG
    assert b"segment 1" in lib.mea_last_error() and b"negative" in lib.mea_last_error()
    assert f(1, 1, _chan_segs([(X, None, Y, None, None, sh_a)]), None) == _capi.MEA_ERR_INVALID_ARG
    assert f(1, 1, _chan_segs([(X, None, X + 64, G, None, sh_a)]), None) == _capi.MEA_ERR_INVALID_ARG
    # segment 1's output lands on segment 0's input
    cross = _chan_segs([(X, None, Y, G, None, sh_a), (0x500000, None, X + 128, 0x310000, None, sh_b)])
    assert f(1, 2, cross, None) == _capi.MEA_ERR_INVALID_ARG
    assert b"overlaps" in lib.mea_last_error()
    wq = lib.mea_swish_channel_bwd_grouped_workspace_bytes
    per = [lib.mea_swish_channel_bwd_workspace_bytes(1, _capi.MEA_NCHW, _capi.shape4(s)) for s in (sh_a, sh_b)]
    need = wq(1, 2, ok2)
    assert need == sum((p + 255) // 256 * 256 for p in per)
    assert wq(1, 0, ok2) == 0 and wq(1, 2, neg) == 0 and wq(9, 2, ok2) == 0
    bsegs = _chan_segs([(X, D, Y, G, 0x700000, sh_a), (0x500000, 0x580000, 0x600000, 0x310000, 0x710000, sh_b)])
    assert b(1, 2, bsegs, 0x800000, need - 1, None) == _capi.MEA_ERR_WORKSPACE
    assert b(1, 2, bsegs, None, need, None) == _capi.MEA_ERR_WORKSPACE
    assert b(1, 2, bsegs, 0x800010, need, None) == _capi.MEA_ERR_WORKSPACE
    assert b"256-byte" in lib.mea_last_error()
    nod = _chan_segs([(X, D, Y, G, None, sh_a)])
    assert b(1, 1, nod, 0x800000, need, None) == _capi.MEA_ERR_INVALID_ARG
    shared_da = _chan_segs([(X, D, Y, G, 0x700000, sh_a), (0x500000, 0x580000, 0x600000, 0x310000, 0x700020, sh_b)])
    assert b(1, 2, shared_da, 0x800000, need, None) == _capi.MEA_ERR_INVALID_ARG
    assert b"dalpha" in lib.mea_last_error()
    part = _chan_segs([(X, D, X + 2, G, 0x700000, sh_a)])
    assert b(1, 1, part, 0x800000, need, None) == _capi.MEA_ERR_INVALID_ARG


class _RecordingLib(_FakeLib):
    """_FakeLib that also keeps each call's arguments."""

    def __init__(self):
        super().__init__()
        self.args = {}

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append(name)
            self.args[name] = args
            return 0
        return fn


def test_binding_channel_grouped_marshalling(monkeypatch):
    # swish_channel_*_grouped build one mea_channel_segment_t per tensor with
    # its pointers and (N, C, H, W); mismatched lists and companions are
    # refused before the library is reached
    import torch
    import memory_efficient_activation_b200 as mea
    from memory_efficient_activation_b200 import _capi
    fake = _RecordingLib()
    monkeypatch.setattr(_capi, "lib", lambda: fake)
    monkeypatch.setattr(mea, "_need_cuda", lambda *ts: None)
    monkeypatch.setattr(mea, "_stream", lambda t: 0)
    shapes = [(2, 16, 7, 7), (3, 40, 14, 14), (1, 8, 1, 1)]
    xs = [torch.randn(s) for s in shapes]
    dys = [torch.randn(s) for s in shapes]
    alphas = [torch.ones(s[1]) for s in shapes]
    ys = mea.swish_channel_fwd_grouped(xs, alphas)
    nseg, segs = fake.args["mea_swish_channel_fwd_grouped"][1:3]
    assert nseg == 3
    for i, (x, y, a, s) in enumerate(zip(xs, ys, alphas, shapes)):
        g = segs[i]
        assert (g.x, g.out, g.alpha) == (x.data_ptr(), y.data_ptr(), a.data_ptr())
        assert not g.dy and not g.dalpha and tuple(g.shape) == s
    dxs, das = mea.swish_channel_bwd_grouped(xs, dys, alphas, workspace=torch.zeros(1 << 16, dtype=torch.uint8))
    nseg, segs = fake.args["mea_swish_channel_bwd_grouped"][1:3]
    assert nseg == 3 and "mea_swish_channel_bwd_grouped_workspace_bytes" in fake.calls
    for i, (x, dy, dx, da, s) in enumerate(zip(xs, dys, dxs, das, shapes)):
        g = segs[i]
        assert (g.x, g.dy, g.out, g.dalpha) == (x.data_ptr(), dy.data_ptr(), dx.data_ptr(), da.data_ptr())
        assert da.numel() == s[1] and da.dtype == torch.float32 and tuple(g.shape) == s
    assert mea.swish_channel_fwd_grouped([], []) == []
    n = len(fake.calls)
    for call in (
        lambda: mea.swish_channel_fwd_grouped(xs, alphas[:2]),                          # list lengths
        lambda: mea.swish_channel_fwd_grouped(xs, [torch.ones(3)] * 3),                  # alpha size
        lambda: mea.swish_channel_fwd_grouped([xs[0], xs[1].double()], alphas[:2]),      # dtype mix
        lambda: mea.swish_channel_bwd_grouped(xs, dys[:2], alphas),                     # dy list
        lambda: mea.swish_channel_bwd_grouped(xs, [torch.randn(2, 16, 7, 8)] + dys[1:], alphas),  # dy shape
        lambda: mea.swish_channel_fwd_grouped([torch.randn(4, 4)], [torch.ones(4)]),      # not 4-D
    ):
        with pytest.raises(ValueError):
            call()
    assert len(fake.calls) == n
