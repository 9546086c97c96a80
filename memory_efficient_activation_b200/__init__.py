"""Memory-efficient elementwise activations for NVIDIA B200 (sm_100a).

The forward of every activation writes y = f(x) and keeps only x; the backward
recomputes what it needs from x in the same pass ("Memory efficient Swish",
sections "How is the memory efficient version Swish implemented?" and "What
makes this implementation save GPU memory?").  All arithmetic runs in the
CUDA kernels of libmea.so, reached through its C ABI (include/mea.h).  This
module only marshals PyTorch CUDA tensors (device memory and the current
stream) into those calls; PyTorch is plumbing here, not the compute path.

Functions (the C ABI's names without the ``mea_`` prefix):
    act_fwd, act_bwd, affine_swish_fwd, affine_swish_bwd,
    affine_act_fwd, affine_act_bwd, swish_channel_fwd, swish_channel_bwd,
    matmul_act_fwd, matmul_act_bwd,
    concat_bn_relu_fwd, concat_bn_relu_apply, concat_bn_relu_bwd,
    act_fwd_bwd_host,
    act_bwd_workspace_bytes, affine_swish_bwd_workspace_bytes,
    affine_act_bwd_workspace_bytes, swish_channel_bwd_workspace_bytes
Autograd / modules:
    ActivationFunction, MemoryEfficientActivation, MemoryEfficientSwish,
    AffineSwishFunction, MemoryEfficientAffineSwish,
    AffineActFunction, MemoryEfficientAffineActivation,
    SwishChannelFunction, MemoryEfficientChannelSwish,
    MLPFunction, MemoryEfficientMLP,
    SharedBuffer, ConcatBNReLUConvFunction, MemoryEfficientDenseBottleneck
"""
from __future__ import annotations

import ctypes
import threading

import torch

from . import _capi
from ._capi import ACT_IDS, LAYOUT_IDS, MeaError

__all__ = [
    "act_fwd", "act_bwd", "act_fwd_grouped", "act_bwd_grouped", "affine_swish_fwd", "affine_swish_bwd",
    "affine_act_fwd", "affine_act_bwd", "swish_channel_fwd", "swish_channel_bwd",
    "swish_channel_fwd_grouped", "swish_channel_bwd_grouped", "swish_channel_bwd_grouped_workspace_bytes",
    "matmul_act_fwd", "matmul_act_bwd",
    "concat_bn_relu_fwd", "concat_bn_relu_apply", "concat_bn_relu_bwd",
    "act_fwd_bwd_host",
    "act_bwd_workspace_bytes", "act_bwd_grouped_workspace_bytes", "affine_swish_bwd_workspace_bytes",
    "affine_act_bwd_workspace_bytes", "swish_channel_bwd_workspace_bytes",
    "ActivationFunction", "MemoryEfficientActivation", "MemoryEfficientSwish",
    "AffineSwishFunction", "MemoryEfficientAffineSwish",
    "AffineActFunction", "MemoryEfficientAffineActivation",
    "SwishChannelFunction", "MemoryEfficientChannelSwish", "MLPFunction", "MemoryEfficientMLP",
    "SharedBuffer", "ConcatBNReLUConvFunction", "MemoryEfficientDenseBottleneck",
    "affine_bwd_wait_selftest", "MeaError", "ACTIVATIONS",
]

ACTIVATIONS = tuple(ACT_IDS)
_DTYPES = {torch.float32: _capi.MEA_F32, torch.bfloat16: _capi.MEA_BF16}


def _dtype_id(t: torch.Tensor) -> int:
    try:
        return _DTYPES[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}; use torch.float32 or torch.bfloat16") from None


def _need_cuda(*ts):
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _like(ref: torch.Tensor, t: torch.Tensor, name: str) -> torch.Tensor:
    """A tensor the kernels read or write with ref's layout: contiguous, on
    ref's device, with ref's dtype and element count (anything else would
    make the kernel run off its end or onto another device)."""
    _need_cuda(t)
    if t.device != ref.device or t.dtype != ref.dtype or t.numel() != ref.numel():
        raise ValueError(f"{name} must be a contiguous tensor on {ref.device} with x's dtype and size")
    return t


def _on_device(ref: torch.Tensor, t: torch.Tensor, name: str, dtype=None, numel=None) -> torch.Tensor:
    """A companion tensor (parameter, gradient, workspace) on ref's device,
    contiguous, optionally of a given dtype and at least `numel` elements."""
    _need_cuda(t)
    if t.device != ref.device:
        raise ValueError(f"{name} must be on {ref.device}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name} needs at least {numel} elements")
    return t


def _shaped(t: torch.Tensor, shape, dtype, device, name: str) -> torch.Tensor:
    """An output of a given shape, dtype and device (contiguous)."""
    _need_cuda(t)
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or t.device != device:
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)} on {device}")
    return t


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _act_id(act: str) -> int:
    try:
        return ACT_IDS[act]
    except KeyError:
        raise ValueError(f"unknown activation {act!r}; one of {ACTIVATIONS}") from None


# ------------------------------------------------------------- workspaces

class _WorkspacePool:
    """Zero-filled reduction workspaces, one per (device, stream).  The
    kernels return the completion counter to zero, so a buffer is zeroed only
    when it is created or grown."""

    def __init__(self):
        self._lock = threading.Lock()
        self._bufs = {}

    def get(self, device: torch.device, stream: int, nbytes: int) -> torch.Tensor:
        key = (device.index, stream)
        with self._lock:
            buf = self._bufs.get(key)
            if buf is None or buf.numel() < nbytes:
                buf = torch.zeros(max(nbytes, 4096), dtype=torch.uint8, device=device)
                self._bufs[key] = buf
            return buf


_pool = _WorkspacePool()


def act_bwd_workspace_bytes(act: str, n: int, want_dparam: bool) -> int:
    return int(_capi.lib().mea_act_bwd_workspace_bytes(_act_id(act), int(n), int(bool(want_dparam))))


def affine_swish_bwd_workspace_bytes(dtype: torch.dtype, layout: str, shape_nchw) -> int:
    return int(_capi.lib().mea_affine_swish_bwd_workspace_bytes(
        _DTYPES[dtype], LAYOUT_IDS[layout], _capi.shape4(shape_nchw)))


def affine_act_bwd_workspace_bytes(dtype: torch.dtype, layout: str, shape_nchw) -> int:
    return int(_capi.lib().mea_affine_act_bwd_workspace_bytes(
        _DTYPES[dtype], LAYOUT_IDS[layout], _capi.shape4(shape_nchw)))


def swish_channel_bwd_workspace_bytes(dtype: torch.dtype, layout: str, shape_nchw) -> int:
    return int(_capi.lib().mea_swish_channel_bwd_workspace_bytes(
        _DTYPES[dtype], LAYOUT_IDS[layout], _capi.shape4(shape_nchw)))


# ------------------------------------------------------------ entry points

def act_fwd(act: str, x: torch.Tensor, param: float = 1.0, param_dev: torch.Tensor | None = None,
            out: torch.Tensor | None = None) -> torch.Tensor:
    """y = f(x).  param: alpha (Swish) or slope (LeakyReLU); param_dev: an
    optional one-element fp32 CUDA tensor read on the device instead."""
    _need_cuda(x)
    y = torch.empty_like(x) if out is None else _like(x, out, "out")
    if param_dev is not None:
        _on_device(x, param_dev, "param_dev", torch.float32, 1)
    st = _capi.lib().mea_act_fwd(_act_id(act), _dtype_id(x), x.data_ptr(), y.data_ptr(), x.numel(),
                                  float(param), _ptr(param_dev), _stream(x))
    _capi.check("mea_act_fwd", st)
    return y


def act_bwd(act: str, x: torch.Tensor, dy: torch.Tensor, param: float = 1.0,
            param_dev: torch.Tensor | None = None, dparam: torch.Tensor | None = None,
            out: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """dx = dy * f'(x), f' recomputed from x.  If dparam (a one-element fp32
    CUDA tensor) is given, it is overwritten with d alpha (Swish only)."""
    _need_cuda(x, dy)
    if dy.dtype != x.dtype or dy.shape != x.shape:
        raise ValueError("dy must match x in dtype and shape")
    _like(x, dy, "dy")
    dx = torch.empty_like(x) if out is None else _like(x, out, "out")
    ws_ptr, ws_bytes = None, 0
    if dparam is not None:
        _on_device(x, dparam, "dparam", torch.float32, 1)
        ws_bytes = act_bwd_workspace_bytes(act, x.numel(), True)
        ws = _on_device(x, workspace, "workspace") if workspace is not None else \
            _pool.get(x.device, _stream(x), ws_bytes)
        ws_ptr, ws_bytes = ws.data_ptr(), ws.numel() * ws.element_size()
    if param_dev is not None:
        _on_device(x, param_dev, "param_dev", torch.float32, 1)
    st = _capi.lib().mea_act_bwd(_act_id(act), _dtype_id(x), x.data_ptr(), dy.data_ptr(), dx.data_ptr(),
                                  x.numel(), float(param), _ptr(param_dev), _ptr(dparam), ws_ptr, ws_bytes,
                                  _stream(x))
    _capi.check("mea_act_bwd", st)
    return dx


def _group_args(xs, name, params, param_devs, dys=None, dparams=None, outs=None):
    """Checks a grouped call's tensor lists (same device and dtype, shapes
    matching x) and builds its mea_act_segment_t array; returns (segments,
    outputs)."""
    xs = list(xs)
    k = len(xs)
    if k == 0:
        return (_capi.ActSegment * 0)(), []
    _need_cuda(*xs)
    ref = xs[0]
    for x in xs:
        if x.device != ref.device or x.dtype != ref.dtype:
            raise ValueError(f"{name}: every tensor must share the first one's device and dtype")
    params = [1.0] * k if params is None else ([float(params)] * k if isinstance(params, (int, float))
                                               else [float(p) for p in params])
    param_devs = [None] * k if param_devs is None else list(param_devs)
    dparams = [None] * k if dparams is None else list(dparams)
    if len(params) != k or len(param_devs) != k or len(dparams) != k or (dys is not None and len(dys) != k):
        raise ValueError(f"{name}: every list must have one entry per tensor")
    if outs is None:
        outs = [torch.empty_like(x) for x in xs]
    else:
        outs = [_like(x, o, "out") for x, o in zip(xs, outs)]
    segs = (_capi.ActSegment * k)()
    for i, x in enumerate(xs):
        if param_devs[i] is not None:
            _on_device(x, param_devs[i], "param_dev", torch.float32, 1)
        if dparams[i] is not None:
            _on_device(x, dparams[i], "dparam", torch.float32, 1)
        dy = None
        if dys is not None:
            dy = _like(x, dys[i], "dy")
        segs[i] = _capi.ActSegment(x.data_ptr(), dy.data_ptr() if dy is not None else None, outs[i].data_ptr(),
                                   x.numel(), params[i], _ptr(param_devs[i]), _ptr(dparams[i]))
    return segs, outs


def act_bwd_grouped_workspace_bytes(act: str, sizes, want_dparam: bool) -> int:
    """Workspace bytes of a grouped backward over tensors of these element
    counts (0 without d alpha)."""
    sizes = [int(n) for n in sizes]
    if not want_dparam or not sizes:
        return 0
    segs = (_capi.ActSegment * len(sizes))()
    for i, n in enumerate(sizes):
        # the size query reads only n and whether d alpha is asked for
        segs[i] = _capi.ActSegment(None, None, None, n, 1.0, None, 1)
    return int(_capi.lib().mea_act_bwd_grouped_workspace_bytes(_act_id(act), len(sizes), segs))


def act_fwd_grouped(act: str, xs, params=None, param_devs=None, outs=None) -> list:
    """y_i = f(x_i) for every tensor of xs in one launch (many small,
    independent tensors: one grid instead of one launch each).  params: one
    float for all or one per tensor; param_devs: optional one-element fp32
    CUDA tensors.  Each y_i is bitwise what act_fwd gives for x_i."""
    segs, outs = _group_args(xs, "act_fwd_grouped", params, param_devs, outs=outs)
    if len(outs) == 0:
        return []
    st = _capi.lib().mea_act_fwd_grouped(_act_id(act), _dtype_id(xs[0]), len(outs), segs, _stream(xs[0]))
    _capi.check("mea_act_fwd_grouped", st)
    return outs


def act_bwd_grouped(act: str, xs, dys, params=None, param_devs=None, dparams=None, outs=None,
                    workspace: torch.Tensor | None = None) -> list:
    """dx_i = dy_i * f'(x_i) for every pair in one launch; with dparams (one
    one-element fp32 CUDA tensor per tensor, Swish) each is overwritten with
    that tensor's d alpha.  Each result is bitwise what act_bwd gives."""
    segs, outs = _group_args(xs, "act_bwd_grouped", params, param_devs, dys=dys, dparams=dparams, outs=outs)
    if len(outs) == 0:
        return []
    ws_ptr, ws_bytes = None, 0
    if dparams is not None:
        need = int(_capi.lib().mea_act_bwd_grouped_workspace_bytes(_act_id(act), len(outs), segs))
        ws = _on_device(xs[0], workspace, "workspace") if workspace is not None else \
            _pool.get(xs[0].device, _stream(xs[0]), need)
        ws_ptr, ws_bytes = ws.data_ptr(), ws.numel() * ws.element_size()
    st = _capi.lib().mea_act_bwd_grouped(_act_id(act), _dtype_id(xs[0]), len(outs), segs, ws_ptr, ws_bytes,
                                         _stream(xs[0]))
    _capi.check("mea_act_bwd_grouped", st)
    return outs


def _affine_shape(x: torch.Tensor, layout: str):
    if x.dim() != 4:
        raise ValueError("per-channel operations take a 4-D tensor")
    if layout == "nhwc":
        N, H, W, C = x.shape
    elif layout == "nchw":
        N, C, H, W = x.shape
    else:
        raise ValueError(f"layout must be 'nchw' or 'nhwc', not {layout!r}")
    return (N, C, H, W)


def _chan_params(C: int, *ps, device=None):
    for p in ps:
        _need_cuda(p)
        if p.dtype != torch.float32 or p.numel() != C:
            raise ValueError(f"per-channel parameters must be fp32 with {C} elements")
        if device is not None and p.device != device:
            raise ValueError(f"per-channel parameters must be on {device}")


def affine_swish_fwd(x: torch.Tensor, gamma: torch.Tensor, beta: torch.Tensor, layout: str = "nhwc",
                     out: torch.Tensor | None = None) -> torch.Tensor:
    """y = z Sigmoid(z), z = gamma_c x + beta_c.  x is (N, H, W, C) for
    'nhwc' or (N, C, H, W) for 'nchw'; gamma and beta are fp32 [C]."""
    _need_cuda(x)
    shape = _affine_shape(x, layout)
    _chan_params(shape[1], gamma, beta, device=x.device)
    y = torch.empty_like(x) if out is None else _like(x, out, "out")
    st = _capi.lib().mea_affine_swish_fwd(_dtype_id(x), LAYOUT_IDS[layout], _capi.shape4(shape), x.data_ptr(),
                                           gamma.data_ptr(), beta.data_ptr(), y.data_ptr(), _stream(x))
    _capi.check("mea_affine_swish_fwd", st)
    return y


def affine_swish_bwd(x: torch.Tensor, dy: torch.Tensor, gamma: torch.Tensor, beta: torch.Tensor,
                     layout: str = "nhwc", out: torch.Tensor | None = None,
                     dgamma: torch.Tensor | None = None, dbeta: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None):
    """Returns (dx, dgamma, dbeta); z and the sigmoid are recomputed from x."""
    _need_cuda(x, dy)
    if dy.dtype != x.dtype or dy.shape != x.shape:
        raise ValueError("dy must match x in dtype and shape")
    shape = _affine_shape(x, layout)
    C = shape[1]
    _chan_params(C, gamma, beta, device=x.device)
    _like(x, dy, "dy")
    dx = torch.empty_like(x) if out is None else _like(x, out, "out")
    dg = torch.empty(C, dtype=torch.float32, device=x.device) if dgamma is None else dgamma
    db = torch.empty(C, dtype=torch.float32, device=x.device) if dbeta is None else dbeta
    _chan_params(C, dg, db, device=x.device)
    need = affine_swish_bwd_workspace_bytes(x.dtype, layout, shape)
    ws = _on_device(x, workspace, "workspace") if workspace is not None else _pool.get(x.device, _stream(x), need)
    st = _capi.lib().mea_affine_swish_bwd(_dtype_id(x), LAYOUT_IDS[layout], _capi.shape4(shape), x.data_ptr(),
                                           dy.data_ptr(), gamma.data_ptr(), beta.data_ptr(), dx.data_ptr(),
                                           dg.data_ptr(), db.data_ptr(), ws.data_ptr(),
                                           ws.numel() * ws.element_size(), _stream(x))
    _capi.check("mea_affine_swish_bwd", st)
    return dx, dg, db


def affine_act_fwd(act: str, x: torch.Tensor, gamma: torch.Tensor, beta: torch.Tensor, param: float = 1.0,
                   layout: str = "nhwc", out: torch.Tensor | None = None) -> torch.Tensor:
    """y = f(z), z = gamma_c x + beta_c, f any activation of the family
    (param: LeakyReLU slope or Swish alpha)."""
    _need_cuda(x)
    shape = _affine_shape(x, layout)
    _chan_params(shape[1], gamma, beta, device=x.device)
    y = torch.empty_like(x) if out is None else _like(x, out, "out")
    st = _capi.lib().mea_affine_act_fwd(_act_id(act), _dtype_id(x), LAYOUT_IDS[layout], _capi.shape4(shape),
                                         x.data_ptr(), gamma.data_ptr(), beta.data_ptr(), float(param),
                                         y.data_ptr(), _stream(x))
    _capi.check("mea_affine_act_fwd", st)
    return y


def affine_act_bwd(act: str, x: torch.Tensor, dy: torch.Tensor, gamma: torch.Tensor, beta: torch.Tensor,
                   param: float = 1.0, layout: str = "nhwc", out: torch.Tensor | None = None,
                   dgamma: torch.Tensor | None = None, dbeta: torch.Tensor | None = None,
                   workspace: torch.Tensor | None = None):
    """Returns (dx, dgamma, dbeta); z and f'(z) are recomputed from x."""
    _need_cuda(x, dy)
    if dy.dtype != x.dtype or dy.shape != x.shape:
        raise ValueError("dy must match x in dtype and shape")
    shape = _affine_shape(x, layout)
    C = shape[1]
    _chan_params(C, gamma, beta, device=x.device)
    _like(x, dy, "dy")
    dx = torch.empty_like(x) if out is None else _like(x, out, "out")
    dg = torch.empty(C, dtype=torch.float32, device=x.device) if dgamma is None else dgamma
    db = torch.empty(C, dtype=torch.float32, device=x.device) if dbeta is None else dbeta
    _chan_params(C, dg, db, device=x.device)
    need = affine_act_bwd_workspace_bytes(x.dtype, layout, shape)
    ws = _on_device(x, workspace, "workspace") if workspace is not None else _pool.get(x.device, _stream(x), need)
    st = _capi.lib().mea_affine_act_bwd(_act_id(act), _dtype_id(x), LAYOUT_IDS[layout], _capi.shape4(shape),
                                         x.data_ptr(), dy.data_ptr(), gamma.data_ptr(), beta.data_ptr(),
                                         float(param), dx.data_ptr(), dg.data_ptr(), db.data_ptr(), ws.data_ptr(),
                                         ws.numel() * ws.element_size(), _stream(x))
    _capi.check("mea_affine_act_bwd", st)
    return dx, dg, db


def swish_channel_fwd(x: torch.Tensor, alpha: torch.Tensor, layout: str = "nchw",
                      out: torch.Tensor | None = None) -> torch.Tensor:
    """y = x Sigmoid(alpha_c x), alpha fp32 [C]."""
    _need_cuda(x)
    shape = _affine_shape(x, layout)
    _chan_params(shape[1], alpha, device=x.device)
    y = torch.empty_like(x) if out is None else _like(x, out, "out")
    st = _capi.lib().mea_swish_channel_fwd(_dtype_id(x), LAYOUT_IDS[layout], _capi.shape4(shape), x.data_ptr(),
                                            alpha.data_ptr(), y.data_ptr(), _stream(x))
    _capi.check("mea_swish_channel_fwd", st)
    return y


def swish_channel_bwd(x: torch.Tensor, dy: torch.Tensor, alpha: torch.Tensor, layout: str = "nchw",
                      out: torch.Tensor | None = None, dalpha: torch.Tensor | None = None,
                      workspace: torch.Tensor | None = None):
    """Returns (dx, dalpha); the sigmoid is recomputed from x."""
    _need_cuda(x, dy)
    if dy.dtype != x.dtype or dy.shape != x.shape:
        raise ValueError("dy must match x in dtype and shape")
    shape = _affine_shape(x, layout)
    C = shape[1]
    _chan_params(C, alpha, device=x.device)
    _like(x, dy, "dy")
    dx = torch.empty_like(x) if out is None else _like(x, out, "out")
    da = torch.empty(C, dtype=torch.float32, device=x.device) if dalpha is None else dalpha
    _chan_params(C, da, device=x.device)
    need = swish_channel_bwd_workspace_bytes(x.dtype, layout, shape)
    ws = _on_device(x, workspace, "workspace") if workspace is not None else _pool.get(x.device, _stream(x), need)
    st = _capi.lib().mea_swish_channel_bwd(_dtype_id(x), LAYOUT_IDS[layout], _capi.shape4(shape), x.data_ptr(),
                                            dy.data_ptr(), alpha.data_ptr(), dx.data_ptr(), da.data_ptr(),
                                            ws.data_ptr(), ws.numel() * ws.element_size(), _stream(x))
    _capi.check("mea_swish_channel_bwd", st)
    return dx, da


def _channel_group_args(xs, alphas, name, dys=None, dalphas=None, outs=None):
    """Checks a grouped per-channel call's lists (NCHW, one device and dtype,
    alpha fp32 [C] per tensor) and builds its mea_channel_segment_t array;
    returns (segments, outputs, d alphas)."""
    xs, alphas = list(xs), list(alphas)
    k = len(xs)
    if len(alphas) != k or (dys is not None and len(dys) != k) or (outs is not None and len(outs) != k) \
            or (dalphas is not None and len(dalphas) != k):
        raise ValueError(f"{name}: every list must have one entry per tensor")
    if k == 0:
        return (_capi.ChannelSegment * 0)(), [], []
    _need_cuda(*xs)
    ref = xs[0]
    for x in xs:
        if x.device != ref.device or x.dtype != ref.dtype:
            raise ValueError(f"{name}: every tensor must share the first one's device and dtype")
    outs = [torch.empty_like(x) for x in xs] if outs is None else [_like(x, o, "out") for x, o in zip(xs, outs)]
    das = []
    segs = (_capi.ChannelSegment * k)()
    for i, x in enumerate(xs):
        shape = _affine_shape(x, "nchw")
        C = shape[1]
        _chan_params(C, alphas[i], device=x.device)
        dy = _like(x, dys[i], "dy") if dys is not None else None
        da = None
        if dys is not None:
            da = torch.empty(C, dtype=torch.float32, device=x.device) if dalphas is None else dalphas[i]
            _chan_params(C, da, device=x.device)
            das.append(da)
        segs[i] = _capi.ChannelSegment(x.data_ptr(), dy.data_ptr() if dy is not None else None, outs[i].data_ptr(),
                                       alphas[i].data_ptr(), da.data_ptr() if da is not None else None,
                                       (ctypes.c_int64 * 4)(*shape))
    return segs, outs, das


def swish_channel_fwd_grouped(xs, alphas, outs=None) -> list:
    """y_i = x_i Sigmoid(alpha_i,c x_i) for every NCHW tensor of xs in one
    launch where the planes allow it (H W <= 1024 and 16-byte aligned); each
    y_i is bitwise what swish_channel_fwd gives for x_i."""
    segs, outs, _ = _channel_group_args(xs, alphas, "swish_channel_fwd_grouped", outs=outs)
    if not outs:
        return []
    st = _capi.lib().mea_swish_channel_fwd_grouped(_dtype_id(outs[0]), len(outs), segs, _stream(outs[0]))
    _capi.check("mea_swish_channel_fwd_grouped", st)
    return outs


def swish_channel_bwd_grouped_workspace_bytes(dtype: torch.dtype, shapes) -> int:
    """Workspace bytes of a grouped per-channel backward over NCHW tensors of
    these (N, C, H, W) shapes."""
    shapes = [tuple(int(v) for v in sh) for sh in shapes]
    if not shapes:
        return 0
    segs = (_capi.ChannelSegment * len(shapes))()
    for i, sh in enumerate(shapes):
        segs[i].shape = (ctypes.c_int64 * 4)(*sh)
    return int(_capi.lib().mea_swish_channel_bwd_grouped_workspace_bytes(_DTYPES[dtype], len(shapes), segs))


def swish_channel_bwd_grouped(xs, dys, alphas, outs=None, dalphas=None,
                              workspace: torch.Tensor | None = None):
    """Returns (dxs, dalphas) for every NCHW tensor of xs in one launch where
    the planes allow it; each pair is bitwise what swish_channel_bwd gives."""
    segs, outs, das = _channel_group_args(xs, alphas, "swish_channel_bwd_grouped", dys=dys, dalphas=dalphas,
                                          outs=outs)
    if not outs:
        return [], []
    x0 = outs[0]
    need = int(_capi.lib().mea_swish_channel_bwd_grouped_workspace_bytes(_dtype_id(x0), len(outs), segs))
    ws = _on_device(x0, workspace, "workspace") if workspace is not None else _pool.get(x0.device, _stream(x0), need)
    st = _capi.lib().mea_swish_channel_bwd_grouped(_dtype_id(x0), len(outs), segs, ws.data_ptr(),
                                                    ws.numel() * ws.element_size(), _stream(x0))
    _capi.check("mea_swish_channel_bwd_grouped", st)
    return outs, das


def _mat2d(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16")
    _need_cuda(t)
    return t


def matmul_act_fwd(act: str, x: torch.Tensor, w: torch.Tensor, param: float = 1.0, want_z: bool = True,
                   want_y: bool = True, z: torch.Tensor | None = None, y: torch.Tensor | None = None):
    """Z = x w^T on the tensor cores (x [M, K], w [N, K], bf16), with the
    activation in the epilogue: returns (z, y), z = Z in bf16 (the tensor to
    keep for the backward) and y = f(z); either may be skipped (None)."""
    _mat2d(x, "x")
    _mat2d(w, "w")
    M, K = x.shape
    N = w.shape[0]
    if w.shape[1] != K:
        raise ValueError("x and w disagree in K")
    if w.device != x.device:
        raise ValueError("x and w must be on the same device")
    if want_z:
        z = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if z is None else \
            _shaped(z, (M, N), torch.bfloat16, x.device, "z")
    if want_y:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device) if y is None else \
            _shaped(y, (M, N), torch.bfloat16, x.device, "y")
    st = _capi.lib().mea_matmul_act_fwd(_act_id(act), M, N, K, x.data_ptr(), w.data_ptr(), float(param),
                                         _ptr(z if want_z else None), _ptr(y if want_y else None), _stream(x))
    _capi.check("mea_matmul_act_fwd", st)
    return (z if want_z else None), (y if want_y else None)


def matmul_act_bwd(act: str, g: torch.Tensor, w: torch.Tensor, z: torch.Tensor, param: float = 1.0,
                   out: torch.Tensor | None = None) -> torch.Tensor:
    """dz = (g w^T) * f'(z) with the product never written: g [M, K] the
    upstream gradient, w [N, K] (the transpose of the next layer's weight),
    z [M, N] the stored pre-activation (bf16)."""
    _mat2d(g, "g")
    _mat2d(w, "w")
    _mat2d(z, "z")
    M, K = g.shape
    N = w.shape[0]
    if w.shape[1] != K or z.shape != (M, N):
        raise ValueError("g, w and z disagree in shape")
    if w.device != g.device or z.device != g.device:
        raise ValueError("g, w and z must be on the same device")
    dz = torch.empty_like(z) if out is None else _shaped(out, (M, N), torch.bfloat16, g.device, "out")
    st = _capi.lib().mea_matmul_act_bwd(_act_id(act), M, N, K, g.data_ptr(), w.data_ptr(), z.data_ptr(),
                                         float(param), dz.data_ptr(), _stream(g))
    _capi.check("mea_matmul_act_bwd", st)
    return dz


def _bn_pieces(pieces):
    if not pieces:
        raise ValueError("at least one piece")
    N, HW = pieces[0].shape[0], int(pieces[0][0, 0].numel())
    dtype = pieces[0].dtype
    for p in pieces:
        _need_cuda(p)
        if p.dim() < 2 or p.shape[0] != N or int(p[0, 0].numel()) != HW or p.dtype != dtype:
            raise ValueError("pieces must share N, the spatial size and the dtype")
        if p.device != pieces[0].device:
            raise ValueError("pieces must be on one device")
    chans = [int(p.shape[1]) for p in pieces]
    return N, HW, chans, _capi.ptr_array([p.data_ptr() for p in pieces]), _capi.int64_array(chans)


def concat_bn_relu_fwd(pieces, gamma, beta, eps: float = 1e-5, momentum: float = 0.1, running_mean=None,
                       running_var=None, out=None, workspace=None):
    """y = max(BN(cat(pieces, dim=1)), 0) with batch statistics, without
    forming the concatenation.  Returns (y, mean, invstd)."""
    N, HW, chans, parr, carr = _bn_pieces(pieces)
    C = sum(chans)
    dev = pieces[0].device
    _chan_params(C, gamma, beta, device=dev)
    for r in (running_mean, running_var):
        if r is not None:
            _chan_params(C, r, device=dev)
    shape = (N, C) + tuple(pieces[0].shape[2:])
    y = torch.empty(shape, dtype=pieces[0].dtype, device=dev) if out is None else \
        _shaped(out, shape, pieces[0].dtype, dev, "out")
    mean = torch.empty(C, dtype=torch.float32, device=dev)
    invstd = torch.empty(C, dtype=torch.float32, device=dev)
    need = int(_capi.lib().mea_concat_bn_relu_workspace_bytes(N, C))
    ws = _on_device(y, workspace, "workspace") if workspace is not None else _pool.get(dev, _stream(y), need)
    st = _capi.lib().mea_concat_bn_relu_fwd(_dtype_id(y), len(pieces), parr, carr, N, HW, gamma.data_ptr(),
                                             beta.data_ptr(), float(eps), float(momentum), _ptr(running_mean),
                                             _ptr(running_var), mean.data_ptr(), invstd.data_ptr(), y.data_ptr(),
                                             ws.data_ptr(), ws.numel() * ws.element_size(), _stream(y))
    _capi.check("mea_concat_bn_relu_fwd", st)
    return y, mean, invstd


def concat_bn_relu_apply(pieces, gamma, beta, mean, invstd, out=None):
    """Re-populates y from the pieces and saved statistics (the forward's
    output, bitwise)."""
    N, HW, chans, parr, carr = _bn_pieces(pieces)
    C = sum(chans)
    dev = pieces[0].device
    _chan_params(C, gamma, beta, mean, invstd, device=dev)
    shape = (N, C) + tuple(pieces[0].shape[2:])
    y = torch.empty(shape, dtype=pieces[0].dtype, device=dev) if out is None else \
        _shaped(out, shape, pieces[0].dtype, dev, "out")
    st = _capi.lib().mea_concat_bn_relu_apply(_dtype_id(y), len(pieces), parr, carr, N, HW, gamma.data_ptr(),
                                               beta.data_ptr(), mean.data_ptr(), invstd.data_ptr(), y.data_ptr(),
                                               _stream(y))
    _capi.check("mea_concat_bn_relu_apply", st)
    return y


def concat_bn_relu_bwd(pieces, dy, gamma, beta, mean, invstd, dpieces=None, accumulate: bool = False,
                       workspace=None):
    """Returns (list of piece gradients, dgamma, dbeta); the ReLU mask and
    xhat are recomputed from the pieces."""
    N, HW, chans, parr, carr = _bn_pieces(pieces)
    C = sum(chans)
    dev = pieces[0].device
    _shaped(dy, (N, C) + tuple(pieces[0].shape[2:]), pieces[0].dtype, dev, "dy")
    _chan_params(C, gamma, beta, mean, invstd, device=dev)
    if dpieces is None:
        dpieces = [torch.zeros_like(p) if accumulate else torch.empty_like(p) for p in pieces]
    if len(dpieces) != len(pieces):
        raise ValueError("one gradient tensor per piece")
    for p, d in zip(pieces, dpieces):
        _shaped(d, p.shape, p.dtype, dev, "dpieces[i]")
    dg = torch.empty(C, dtype=torch.float32, device=dev)
    db = torch.empty(C, dtype=torch.float32, device=dev)
    need = int(_capi.lib().mea_concat_bn_relu_workspace_bytes(N, C))
    ws = _on_device(dy, workspace, "workspace") if workspace is not None else _pool.get(dev, _stream(dy), need)
    st = _capi.lib().mea_concat_bn_relu_bwd(_dtype_id(dy), len(pieces), parr, carr, N, HW, dy.data_ptr(),
                                             gamma.data_ptr(), beta.data_ptr(), mean.data_ptr(), invstd.data_ptr(),
                                             _capi.ptr_array([d.data_ptr() for d in dpieces]), int(bool(accumulate)),
                                             dg.data_ptr(), db.data_ptr(), ws.data_ptr(),
                                             ws.numel() * ws.element_size(), _stream(dy))
    _capi.check("mea_concat_bn_relu_bwd", st)
    return dpieces, dg, db


class _HostPipe:
    """Device buffers and streams reused by act_fwd_bwd_host (per device)."""

    def __init__(self, device, numel, dtype):
        self.key = (device, numel, dtype)
        self.bufs = [torch.empty(numel, dtype=dtype, device=device) for _ in range(4)]   # x, dy, y, dx
        self.streams = [torch.cuda.Stream(device) for _ in range(3)]                     # copy in, compute, copy out


_host_pipes: dict = {}
# One pipeline submission at a time: calls from several threads share a
# device's buffers and streams.
_host_pipe_lock = threading.Lock()


def act_fwd_bwd_host(act: str, hx: torch.Tensor, hdy: torch.Tensor, param: float = 1.0,
                     hy: torch.Tensor | None = None, hdx: torch.Tensor | None = None, chunks: int = 8,
                     device=None):
    """Forward and backward of an activation on data in pinned host memory:
    y = f(x) and dx = dy f'(x) copied back to host.  The tensor is split into
    `chunks` pieces that flow through three streams (host to device, the two
    kernels, device to host), so the copy of one piece overlaps the kernels of
    the previous one and the copy back of the one before (PCIe carries both
    directions at once).  Returns (hy, hdx); the work is queued behind the
    current stream and the current stream waits for its end."""
    if hx.is_cuda or hdy.is_cuda:
        raise ValueError("hx and hdy must be host tensors")
    if hx.shape != hdy.shape or hx.dtype != hdy.dtype:
        raise ValueError("hx and hdy must match")
    for name, out in (("hy", hy), ("hdx", hdx)):
        # results are copied into the flat view of the output, so it must be
        # that tensor's own storage: contiguous, on the host, same size and dtype
        if out is not None and (out.is_cuda or not out.is_contiguous() or out.numel() != hx.numel()
                                or out.dtype != hx.dtype):
            raise ValueError(f"{name} must be a contiguous host tensor with hx's size and dtype")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    n = hx.numel()
    hy = torch.empty_like(hx).pin_memory() if hy is None else hy
    hdx = torch.empty_like(hx).pin_memory() if hdx is None else hdx
    key = (dev, n, hx.dtype)
    with _host_pipe_lock:
        pipe = _host_pipes.get(dev)
        if pipe is None or pipe.key != key:
            if pipe is not None:
                # the old buffers may still be in use by queued work
                torch.cuda.current_stream(dev).wait_stream(pipe.streams[2])
            pipe = _HostPipe(dev, n, hx.dtype)
            _host_pipes[dev] = pipe
        return _host_pipe_run(pipe, dev, act, hx, hdy, hy, hdx, param, chunks)


def _host_pipe_run(pipe, dev, act, hx, hdy, hy, hdx, param, chunks):
    n = hx.numel()
    x, dy, y, dx = pipe.bufs
    s_in, s_run, s_out = pipe.streams
    cur = torch.cuda.current_stream(dev)
    fx, fdy, fy, fdx = hx.reshape(-1), hdy.reshape(-1), hy.reshape(-1), hdx.reshape(-1)
    step = -(-n // max(1, chunks))
    step = -(-step // 256) * 256                 # pieces start 16-byte aligned
    s_in.wait_stream(cur)
    s_in.wait_stream(s_out)                      # a previous call's pieces are out of the buffers
    for lo in range(0, n, step):
        hi = min(n, lo + step)
        with torch.cuda.stream(s_in):
            x[lo:hi].copy_(fx[lo:hi], non_blocking=True)
            dy[lo:hi].copy_(fdy[lo:hi], non_blocking=True)
        s_run.wait_stream(s_in)
        with torch.cuda.stream(s_run):
            act_fwd(act, x[lo:hi], param, out=y[lo:hi])
            act_bwd(act, x[lo:hi], dy[lo:hi], param, out=dx[lo:hi])
        s_out.wait_stream(s_run)
        with torch.cuda.stream(s_out):
            fy[lo:hi].copy_(y[lo:hi], non_blocking=True)
            fdx[lo:hi].copy_(dx[lo:hi], non_blocking=True)
    cur.wait_stream(s_out)
    return hy, hdx


# ---------------------------------------------------------------- autograd

class ActivationFunction(torch.autograd.Function):
    """Save-input-only autograd function: ctx keeps x (and alpha), nothing else."""

    @staticmethod
    def forward(ctx, x, act: str, param: float, alpha: torch.Tensor | None):
        x = x.contiguous()
        y = act_fwd(act, x, param, param_dev=alpha)
        ctx.act, ctx.param = act, param
        if alpha is None:
            ctx.save_for_backward(x)
        else:
            ctx.save_for_backward(x, alpha)
        return y

    @staticmethod
    def backward(ctx, dy):
        saved = ctx.saved_tensors
        x = saved[0]
        alpha = saved[1] if len(saved) > 1 else None
        dy = dy.contiguous()
        want = alpha is not None and ctx.needs_input_grad[3]
        dalpha = torch.empty(1, dtype=torch.float32, device=x.device) if want else None
        dx = act_bwd(ctx.act, x, dy, ctx.param, param_dev=alpha, dparam=dalpha)
        return dx, None, None, (dalpha.view_as(alpha) if want else None)


class MemoryEfficientActivation(torch.nn.Module):
    """An activation of the family whose backward recomputes from x."""

    def __init__(self, act: str = "swish", param: float | None = None):
        super().__init__()
        _act_id(act)
        self.act = act
        self.param = (0.01 if act == "leaky_relu" else 1.0) if param is None else float(param)

    def forward(self, x):
        return ActivationFunction.apply(x, self.act, self.param, None)


class MemoryEfficientSwish(torch.nn.Module):
    """Swish x * Sigmoid(alpha x); alpha fixed (default 1) or learnable."""

    def __init__(self, alpha: float = 1.0, learnable: bool = False):
        super().__init__()
        if learnable:
            self.alpha = torch.nn.Parameter(torch.tensor([float(alpha)], dtype=torch.float32))
        else:
            self.register_buffer("alpha", None)
            self.alpha_value = float(alpha)

    def forward(self, x):
        if self.alpha is not None:
            return ActivationFunction.apply(x, "swish", 1.0, self.alpha)
        return ActivationFunction.apply(x, "swish", self.alpha_value, None)


class AffineSwishFunction(torch.autograd.Function):
    """Fused per-channel affine + Swish that saves only x (and gamma, beta)."""

    @staticmethod
    def forward(ctx, x, gamma, beta, layout: str):
        x = x.contiguous()
        y = affine_swish_fwd(x, gamma, beta, layout)
        ctx.layout = layout
        ctx.save_for_backward(x, gamma, beta)
        return y

    @staticmethod
    def backward(ctx, dy):
        x, gamma, beta = ctx.saved_tensors
        dx, dg, db = affine_swish_bwd(x, dy.contiguous(), gamma, beta, ctx.layout)
        return dx, dg, db, None


class MemoryEfficientAffineSwish(torch.nn.Module):
    """y = z Sigmoid(z), z = gamma_c x + beta_c, with learnable fp32 gamma, beta."""

    def __init__(self, channels: int, layout: str = "nhwc"):
        super().__init__()
        self.layout = layout
        self.gamma = torch.nn.Parameter(torch.ones(channels, dtype=torch.float32))
        self.beta = torch.nn.Parameter(torch.zeros(channels, dtype=torch.float32))

    def forward(self, x):
        return AffineSwishFunction.apply(x, self.gamma, self.beta, self.layout)


class AffineActFunction(torch.autograd.Function):
    """Fused per-channel affine + activation that saves only x (and gamma, beta)."""

    @staticmethod
    def forward(ctx, x, gamma, beta, act: str, param: float, layout: str):
        x = x.contiguous()
        y = affine_act_fwd(act, x, gamma, beta, param, layout)
        ctx.act, ctx.param, ctx.layout = act, param, layout
        ctx.save_for_backward(x, gamma, beta)
        return y

    @staticmethod
    def backward(ctx, dy):
        x, gamma, beta = ctx.saved_tensors
        dx, dg, db = affine_act_bwd(ctx.act, x, dy.contiguous(), gamma, beta, ctx.param, ctx.layout)
        return dx, dg, db, None, None, None


class MemoryEfficientAffineActivation(torch.nn.Module):
    """y = f(gamma_c x + beta_c) for any activation of the family, with
    learnable fp32 gamma, beta (a folded batch norm or a per-channel scale)."""

    def __init__(self, channels: int, act: str = "swish", param: float | None = None, layout: str = "nhwc"):
        super().__init__()
        _act_id(act)
        self.act, self.layout = act, layout
        self.param = (0.01 if act == "leaky_relu" else 1.0) if param is None else float(param)
        self.gamma = torch.nn.Parameter(torch.ones(channels, dtype=torch.float32))
        self.beta = torch.nn.Parameter(torch.zeros(channels, dtype=torch.float32))

    def forward(self, x):
        return AffineActFunction.apply(x, self.gamma, self.beta, self.act, self.param, self.layout)


class SwishChannelFunction(torch.autograd.Function):
    """Swish with one alpha per channel that saves only x (and alpha)."""

    @staticmethod
    def forward(ctx, x, alpha, layout: str):
        x = x.contiguous()
        y = swish_channel_fwd(x, alpha, layout)
        ctx.layout = layout
        ctx.save_for_backward(x, alpha)
        return y

    @staticmethod
    def backward(ctx, dy):
        x, alpha = ctx.saved_tensors
        dx, da = swish_channel_bwd(x, dy.contiguous(), alpha, ctx.layout)
        return dx, (da if ctx.needs_input_grad[1] else None), None


class MemoryEfficientChannelSwish(torch.nn.Module):
    """Swish x Sigmoid(alpha_c x) with a learnable fp32 alpha per channel."""

    def __init__(self, channels: int, alpha: float = 1.0, layout: str = "nchw"):
        super().__init__()
        self.layout = layout
        self.alpha = torch.nn.Parameter(torch.full((channels,), float(alpha), dtype=torch.float32))

    def forward(self, x):
        return SwishChannelFunction.apply(x, self.alpha, self.layout)


class MLPFunction(torch.autograd.Function):
    """out = f(x W1^T) W2^T that keeps x and z = x W1^T (bf16) for the
    backward, not f(z): the first matmul writes z and f(z) from one epilogue,
    and the backward multiplies dout W2 by f'(z) inside the matmul that forms
    it (matmul_act_bwd), recomputing f(z) only for W2's gradient.  The two
    other products (f(z) W2^T forward; dW2, dW1, dx backward) are plain
    matmuls (torch.matmul)."""

    @staticmethod
    def forward(ctx, x, w1, w2, act: str, param: float):
        z, y = matmul_act_fwd(act, x, w1, param)
        out = torch.matmul(y, w2.t())
        ctx.act, ctx.param = act, param
        ctx.save_for_backward(x, w1, w2, z)
        return out

    @staticmethod
    def backward(ctx, dout):
        x, w1, w2, z = ctx.saved_tensors
        dout = dout.contiguous()
        y = act_fwd(ctx.act, z, ctx.param)
        dw2 = torch.matmul(dout.t(), y)
        del y                                  # freed before dz exists: one hidden-sized buffer at a time
        dz = matmul_act_bwd(ctx.act, dout, w2.t().contiguous(), z, ctx.param)
        dw1 = torch.matmul(dz.t(), x)
        dx = torch.matmul(dz, w1)
        return dx, dw1, dw2, None, None


class MemoryEfficientMLP(torch.nn.Module):
    """Linear(d_model -> d_hidden, no bias) -> activation -> Linear(d_hidden
    -> d_model, no bias) in bf16, keeping only the input and the hidden
    pre-activation for the backward.  d_model and d_hidden must be multiples
    of 8; inputs are [..., d_model] bf16 CUDA tensors."""

    def __init__(self, d_model: int, d_hidden: int, act: str = "gelu_tanh", param: float | None = None):
        super().__init__()
        _act_id(act)
        if d_model % 8 or d_hidden % 8:
            raise ValueError("d_model and d_hidden must be multiples of 8")
        self.act = act
        self.param = (0.01 if act == "leaky_relu" else 1.0) if param is None else float(param)
        self.w1 = torch.nn.Parameter(torch.empty(d_hidden, d_model, dtype=torch.bfloat16))
        self.w2 = torch.nn.Parameter(torch.empty(d_model, d_hidden, dtype=torch.bfloat16))
        with torch.no_grad():
            self.w1.normal_(0.0, d_model ** -0.5)
            self.w2.normal_(0.0, d_hidden ** -0.5)

    def forward(self, x):
        shape = x.shape
        out = MLPFunction.apply(x.reshape(-1, shape[-1]).contiguous(), self.w1, self.w2, self.act, self.param)
        return out.view(*shape[:-1], out.shape[-1])


class SharedBuffer:
    """One device buffer reused by every layer for its batch-normalization
    output (grown on demand).  A layer's output lives there only until the
    next layer overwrites it; the backward re-populates it."""

    def __init__(self):
        self._buf = None

    def get(self, shape, dtype, device) -> torch.Tensor:
        n = 1
        for d in shape:
            n *= int(d)
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        if self._buf is None or self._buf.numel() < nbytes or self._buf.device != torch.device(device):
            self._buf = torch.empty(nbytes, dtype=torch.uint8, device=device)
        return self._buf[:nbytes].view(dtype).view(shape)


class ConcatBNReLUConvFunction(torch.autograd.Function):
    """conv1x1(relu(BN(cat(pieces)))) with batch statistics, keeping only the
    pieces (which the network keeps anyway), the weights and 2 C floats of
    statistics: the normalized tensor lives in a shared buffer and the
    backward re-populates it before the weight gradient needs it.  The 1x1
    convolution and its gradients are the library's (cuDNN through
    torch.nn.functional.conv2d and torch.nn.grad), as in a plain layer."""

    @staticmethod
    def forward(ctx, shared, weight, gamma, beta, running_mean, running_var, eps, momentum, *pieces):
        N = pieces[0].shape[0]
        C = sum(int(p.shape[1]) for p in pieces)
        spatial = tuple(pieces[0].shape[2:])
        y = shared.get((N, C) + spatial, pieces[0].dtype, pieces[0].device)
        y, mean, invstd = concat_bn_relu_fwd(list(pieces), gamma, beta, eps, momentum, running_mean, running_var,
                                             out=y)
        out = torch.nn.functional.conv2d(y, weight)
        ctx.shared, ctx.spatial = shared, spatial
        ctx.save_for_backward(weight, gamma, beta, mean, invstd, *pieces)
        return out

    @staticmethod
    def backward(ctx, dout):
        weight, gamma, beta, mean, invstd, *pieces = ctx.saved_tensors
        N = pieces[0].shape[0]
        C = sum(int(p.shape[1]) for p in pieces)
        y = ctx.shared.get((N, C) + ctx.spatial, pieces[0].dtype, pieces[0].device)
        concat_bn_relu_apply(pieces, gamma, beta, mean, invstd, out=y)
        dout = dout.contiguous()
        dw = torch.nn.grad.conv2d_weight(y, weight.shape, dout)
        dy = torch.nn.grad.conv2d_input(y.shape, weight, dout)
        dpieces, dg, db = concat_bn_relu_bwd(pieces, dy, gamma, beta, mean, invstd)
        return (None, dw, dg, db, None, None, None, None, *dpieces)


class MemoryEfficientDenseBottleneck(torch.nn.Module):
    """The bottleneck of a DenseNet layer: concatenation of the previous
    feature maps, batch normalization, ReLU and a 1x1 convolution to
    `out_channels`, with the concatenated and normalized tensors kept only in
    `shared` (one buffer for every layer).  NCHW bf16 or fp32; the gradient
    of the normalized tensor (the 1x1 convolution's input gradient) is a
    transient of the backward."""

    def __init__(self, in_channels: int, out_channels: int, shared: SharedBuffer | None = None,
                 eps: float = 1e-5, momentum: float = 0.1, dtype=torch.bfloat16):
        super().__init__()
        self.shared = shared if shared is not None else SharedBuffer()
        self.eps, self.momentum = eps, momentum
        self.weight = torch.nn.Parameter(torch.empty(out_channels, in_channels, 1, 1, dtype=dtype))
        with torch.no_grad():
            self.weight.normal_(0.0, in_channels ** -0.5)
        self.gamma = torch.nn.Parameter(torch.ones(in_channels, dtype=torch.float32))
        self.beta = torch.nn.Parameter(torch.zeros(in_channels, dtype=torch.float32))
        self.register_buffer("running_mean", torch.zeros(in_channels, dtype=torch.float32))
        self.register_buffer("running_var", torch.ones(in_channels, dtype=torch.float32))

    def forward(self, *pieces):
        return ConcatBNReLUConvFunction.apply(self.shared, self.weight, self.gamma, self.beta, self.running_mean,
                                              self.running_var, self.eps, self.momentum,
                                              *[p.contiguous() for p in pieces])


def affine_bwd_wait_selftest(x: torch.Tensor, dy: torch.Tensor, gamma: torch.Tensor, beta: torch.Tensor,
                             workspace: torch.Tensor | None = None) -> int:
    """Self-test of the bounded waits: runs the pipelined NHWC backward of the
    fused affine + Swish on these tensors (x, dy: (N, H, W, C)) with its
    shared-memory copies withheld, so that every stage wait expires; returns
    the error word the kernel recorded (1 when the waits expired and the
    kernel returned, as designed).  Synchronises the current stream."""
    _need_cuda(x, dy)
    _like(x, dy, "dy")
    shape = _affine_shape(x, "nhwc")
    _chan_params(shape[1], gamma, beta, device=x.device)
    need = affine_swish_bwd_workspace_bytes(x.dtype, "nhwc", shape)
    ws = torch.zeros(need, dtype=torch.uint8, device=x.device) if workspace is None else \
        _on_device(x, workspace, "workspace")
    dx = torch.empty_like(x)
    expired = ctypes.c_int(0)
    st = _capi.lib().mea_affine_bwd_wait_selftest(_dtype_id(x), _capi.shape4(shape), x.data_ptr(), dy.data_ptr(),
                                                  gamma.data_ptr(), beta.data_ptr(), dx.data_ptr(), ws.data_ptr(),
                                                  ws.numel(), ctypes.byref(expired), _stream(x))
    _capi.check("mea_affine_bwd_wait_selftest", st)
    return int(expired.value)
