"""ctypes declarations of the C ABI in include/mea.h (libmea.so).

Marshalling only: this module loads the shared library that sits next to it
and declares argument and result types.  There is no fallback: if the library
is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmea.so")

# Enumerations of include/mea.h.
MEA_RELU, MEA_LEAKY_RELU, MEA_SIGMOID, MEA_TANH, MEA_GELU_ERF, MEA_GELU_TANH, MEA_SWISH = range(7)
MEA_F32, MEA_BF16 = 0, 1
MEA_NCHW, MEA_NHWC = 0, 1
MEA_OK, MEA_ERR_INVALID_ARG, MEA_ERR_UNSUPPORTED, MEA_ERR_WORKSPACE, MEA_ERR_CUDA = range(5)

ACT_IDS = {
    "relu": MEA_RELU,
    "leaky_relu": MEA_LEAKY_RELU,
    "sigmoid": MEA_SIGMOID,
    "tanh": MEA_TANH,
    "gelu_erf": MEA_GELU_ERF,
    "gelu_tanh": MEA_GELU_TANH,
    "swish": MEA_SWISH,
}
LAYOUT_IDS = {"nchw": MEA_NCHW, "nhwc": MEA_NHWC}

# Every symbol the header declares, with (restype, argtypes).
_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_f = ctypes.c_float
_i = ctypes.c_int
_sz = ctypes.c_size_t
_shape = ctypes.POINTER(ctypes.c_int64)
_ptrs = ctypes.POINTER(ctypes.c_void_p)


class ActSegment(ctypes.Structure):
    """mea_act_segment_t: one tensor of a grouped call."""
    _fields_ = [("x", _vp), ("dy", _vp), ("out", _vp), ("n", _i64), ("param", _f), ("param_dev", _vp),
                ("dparam_dev", _vp)]


class ChannelSegment(ctypes.Structure):
    """mea_channel_segment_t: one NCHW tensor of a grouped per-channel Swish call."""
    _fields_ = [("x", _vp), ("dy", _vp), ("out", _vp), ("alpha", _vp), ("dalpha", _vp),
                ("shape", ctypes.c_int64 * 4)]


_segs = ctypes.POINTER(ActSegment)
_csegs = ctypes.POINTER(ChannelSegment)
SIGNATURES = {
    "mea_act_fwd": (_i, [_i, _i, _vp, _vp, _i64, _f, _vp, _vp]),
    "mea_act_bwd_workspace_bytes": (_sz, [_i, _i64, _i]),
    "mea_act_bwd": (_i, [_i, _i, _vp, _vp, _vp, _i64, _f, _vp, _vp, _vp, _sz, _vp]),
    "mea_act_fwd_grouped": (_i, [_i, _i, _i, _segs, _vp]),
    "mea_act_bwd_grouped_workspace_bytes": (_sz, [_i, _i, _segs]),
    "mea_act_bwd_grouped": (_i, [_i, _i, _i, _segs, _vp, _sz, _vp]),
    "mea_swish_channel_fwd_grouped": (_i, [_i, _i, _csegs, _vp]),
    "mea_swish_channel_bwd_grouped_workspace_bytes": (_sz, [_i, _i, _csegs]),
    "mea_swish_channel_bwd_grouped": (_i, [_i, _i, _csegs, _vp, _sz, _vp]),
    "mea_affine_swish_bwd_workspace_bytes": (_sz, [_i, _i, _shape]),
    "mea_affine_swish_fwd": (_i, [_i, _i, _shape, _vp, _vp, _vp, _vp, _vp]),
    "mea_affine_swish_bwd": (_i, [_i, _i, _shape, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "mea_affine_act_bwd_workspace_bytes": (_sz, [_i, _i, _shape]),
    "mea_affine_act_fwd": (_i, [_i, _i, _i, _shape, _vp, _vp, _vp, _f, _vp, _vp]),
    "mea_affine_act_bwd": (_i, [_i, _i, _i, _shape, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp, _vp, _sz, _vp]),
    "mea_swish_channel_bwd_workspace_bytes": (_sz, [_i, _i, _shape]),
    "mea_swish_channel_fwd": (_i, [_i, _i, _shape, _vp, _vp, _vp, _vp]),
    "mea_swish_channel_bwd": (_i, [_i, _i, _shape, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "mea_matmul_act_fwd": (_i, [_i, _i64, _i64, _i64, _vp, _vp, _f, _vp, _vp, _vp]),
    "mea_matmul_act_bwd": (_i, [_i, _i64, _i64, _i64, _vp, _vp, _vp, _f, _vp, _vp]),
    "mea_matmul_error_word": (_i, [_i]),
    "mea_concat_bn_relu_workspace_bytes": (_sz, [_i64, _i64]),
    "mea_concat_bn_relu_fwd": (_i, [_i, _i, _ptrs, _shape, _i64, _i64, _vp, _vp, _f, _f, _vp, _vp, _vp, _vp, _vp,
                                    _vp, _sz, _vp]),
    "mea_concat_bn_relu_apply": (_i, [_i, _i, _ptrs, _shape, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "mea_concat_bn_relu_bwd": (_i, [_i, _i, _ptrs, _shape, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _ptrs, _i, _vp,
                                    _vp, _vp, _sz, _vp]),
    "mea_act_bwd_dparam_noalloc": (_i, [_i, _i, _vp, _vp, _vp, _i64, _f, _vp, _vp, _vp]),
    "mea_affine_bwd_wait_selftest": (_i, [_i, _shape, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                          ctypes.POINTER(ctypes.c_int), _vp]),
    "mea_status_string": (ctypes.c_char_p, [_i]),
    "mea_last_error": (ctypes.c_char_p, []),
    "mea_version": (_i, []),
}

_lib = None


class MeaError(RuntimeError):
    """A libmea call returned a status other than MEA_OK."""

    def __init__(self, fn: str, status: int, detail: str):
        self.status = status
        super().__init__(f"{fn} failed: status {status}: {detail}")


def lib() -> ctypes.CDLL:
    """The loaded libmea.so (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing; build it with `python -m memory_efficient_activation_b200.build` "
                "(the activation path runs only in its CUDA kernels)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def check(fn: str, status: int) -> None:
    if status != MEA_OK:
        detail = lib().mea_last_error().decode(errors="replace")
        raise MeaError(fn, status, detail or lib().mea_status_string(status).decode())


def shape4(shape) -> ctypes.Array:
    vals = [int(v) for v in shape]
    if len(vals) != 4:
        raise ValueError("shape must have four entries (N, C, H, W)")
    return (ctypes.c_int64 * 4)(*vals)


def ptr_array(ptrs) -> ctypes.Array:
    """Host array of device pointers (void *const *)."""
    return (ctypes.c_void_p * len(ptrs))(*[int(p) for p in ptrs])


def int64_array(vals) -> ctypes.Array:
    return (ctypes.c_int64 * len(vals))(*[int(v) for v in vals])
