"""The save-input-only contract, observed through PyTorch's saved-tensor hooks.

The Swish page's point ("What makes this implementation save GPU memory?") is
that only the input is kept for the backward.  Checked here on the autograd
functions of the binding: every activation of the family keeps exactly one
tensor (x), the learnable-alpha Swish keeps x and alpha, and the fused affine
keeps x, gamma and beta; the plain autograd Swish (the pages' first listing)
keeps more.
"""
import pytest
import torch

import memory_efficient_activation_b200 as mea
from memory_efficient_activation_b200 import synthetic

pytestmark = pytest.mark.gpu


def _saved(fn, *args):
    saved = []

    def pack(t):
        saved.append(t)
        return t

    with torch.autograd.graph.saved_tensors_hooks(pack, lambda t: t):
        out = fn(*args)
    return out, saved


@pytest.mark.parametrize("act", synthetic.ACTIVATIONS)
def test_family_saves_only_input(act):
    x = synthetic.normal(4096, 2.0, 601, synthetic.STREAM_X, "bf16").cuda().requires_grad_(True)
    m = mea.MemoryEfficientActivation(act)
    y, saved = _saved(m, x)
    assert len(saved) == 1 and saved[0].data_ptr() == x.data_ptr()
    y.backward(torch.ones_like(y))
    assert x.grad is not None and x.grad.shape == x.shape


def test_learnable_swish_saves_input_and_alpha():
    x = synthetic.normal(4096, 2.0, 602, synthetic.STREAM_X, "f32").cuda().requires_grad_(True)
    m = mea.MemoryEfficientSwish(1.3, learnable=True).cuda()
    _, saved = _saved(m, x)
    assert len(saved) == 2
    assert {t.numel() for t in saved} == {4096, 1}


def test_affine_saves_input_gamma_beta():
    x = synthetic.normal(2 * 4 * 4 * 16, 1.0, 603, synthetic.STREAM_X, "bf16").view(2, 4, 4, 16).cuda()
    m = mea.MemoryEfficientAffineSwish(16, "nhwc").cuda()
    _, saved = _saved(m, x.requires_grad_(True))
    assert len(saved) == 3
    assert sorted(t.numel() for t in saved) == [16, 16, x.numel()]


def test_plain_autograd_swish_keeps_more():
    x = synthetic.normal(4096, 2.0, 604, synthetic.STREAM_X, "bf16").cuda().requires_grad_(True)
    _, saved = _saved(lambda t: t * torch.sigmoid(1.0 * t), x)
    big = [t for t in saved if t.numel() == x.numel()]
    assert len(big) >= 2


def test_stack_peak_memory_is_lower():
    # 8 layers of [8, 512, 1024] bf16: the save-input-only stack keeps one
    # tensor per layer, the plain one at least two.
    shape = (8, 512, 1024)
    layer_bytes = 8 * 512 * 1024 * 2
    x0 = synthetic.normal(8 * 512 * 1024, 1.0, 605, synthetic.STREAM_X, "bf16").view(shape).cuda()
    peaks = {}
    for impl in ("plain", "mea"):
        mods = [mea.MemoryEfficientSwish() if impl == "mea" else None for _ in range(8)]
        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats()
        base = torch.cuda.memory_allocated()
        x = x0.detach().requires_grad_(True)
        y = x
        for m in mods:
            y = m(y) if m is not None else y * torch.sigmoid(1.0 * y)
        peaks[impl] = torch.cuda.max_memory_allocated() - base
        y.backward(torch.ones_like(y))
        del x, y
    assert peaks["mea"] < peaks["plain"] - 6 * layer_bytes, peaks
