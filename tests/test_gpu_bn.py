"""GPU parity of the concatenation + batch normalization + ReLU kernels
(mea_concat_bn_relu_fwd / _apply / _bwd) against the oracle, through the C
ABI, and the memory-efficient DenseNet bottleneck built on them.

Rules (tests/_compare.py, check_bn): y is held to one bf16 ulp or, in fp32,
1e-5 of its condition scale (|gamma| r (|x| + |mean|) + |beta|, the terms any
evaluation of gamma xhat + beta adds); with bf16 storage a y that misses the
ulp rule may meet the fp32 rule against that scale (the batch statistics are
fp32 results: where gamma xhat + beta cancels their rounding alone exceeds a
bf16 ulp), for at most 1e-3 of the elements.  The statistics: see
_check_stats (fp32 sums of at most 8 shifted values, then fp64).  dx is held to the same rules with
the oracle's scale |gamma| r (|dz| + sum|dz| / n + |xhat| sum|dz xhat| / n).
An element whose exact gamma xhat + beta lies within 1e-5 of its scale of
zero may take either side of the ReLU: its dz may differ by dy, which adds
|gamma r dy| to its dx allowance and |dy| (|dy xhat|) to its channel's
dbeta (dgamma) allowance.  dgamma and dbeta: 1e-5 relative plus 1e-8 of the
sum of their terms' magnitudes for channels of at least 2^16 values (1e-6
below that: the worst case of the kernels' short fp32 runs).
"""
import numpy as np
import pytest
import torch

import memory_efficient_activation_b200 as mea
import oracle
from _compare import TINY, check_bn, to_f64
from memory_efficient_activation_b200 import synthetic

pytestmark = pytest.mark.gpu

EPS = 1e-5


def _pieces(N, ks, spatial, dtype, seed, mean=0.3, sigma=1.5):
    HW = int(np.prod(spatial))
    out = []
    for i, k in enumerate(ks):
        a = synthetic.normal(N * k * HW, sigma, seed * 64 + i, synthetic.STREAM_X, dtype)
        out.append((a.double() + mean).to(a.dtype).view((N, k) + tuple(spatial)))
    return out


def _params(C, seed):
    g = torch.from_numpy(synthetic.uniform_f64(C, 0.5, 1.5, seed, synthetic.STREAM_GAMMA)).float()
    b = torch.from_numpy(synthetic.normal_f64(C, 0.3, seed, synthetic.STREAM_BETA)).float()
    return g, b


def _np(ps):
    return [p.double().numpy().reshape(p.shape[0], p.shape[1], -1) for p in ps]


def _check_stats(mean, invstd, rm, rv, pieces):
    # The kernels sum d = x - shift (shift: an element of the channel) in
    # fp32 over at most 8 values, then in fp64: the sum of d errs by at most
    # 8 2^-24 of sum |d|, and sum |d| / n <= mean|x| + max|x|; the fp32
    # results add one rounding.  E[d^2] errs likewise, relative to E[d^2] =
    # var + (mean - shift)^2 <= var + (|mean| + max|x|)^2.
    x = np.concatenate(_np(pieces), axis=1)
    am = np.abs(x).mean(axis=(0, 2))
    mx = np.abs(x).max(axis=(0, 2))
    assert np.all(np.abs(mean.cpu().double().numpy() - rm) <= 1e-6 * np.abs(rm) + 5e-7 * (am + mx))
    ri = 1.0 / np.sqrt(rv + EPS)
    tol = 2e-6 + 5e-7 * (np.abs(rm) + mx) ** 2 / (rv + EPS)
    assert np.all(np.abs(invstd.cpu().double().numpy() - ri) <= tol * ri)


def _ambiguous(pieces, g, b, rm, rv, ys):
    x = np.concatenate(_np(pieces), axis=1)
    r = 1.0 / np.sqrt(rv + EPS)
    z = g.double().numpy()[None, :, None] * (x - rm[None, :, None]) * r[None, :, None] + b.double().numpy()[None, :, None]
    return np.abs(z) <= 1e-5 * ys.reshape(z.shape), x, r


def _run(N, ks, spatial, dtype, seed, accumulate=False, cap=1e-3):
    pieces = _pieces(N, ks, spatial, dtype, seed)
    C = sum(ks)
    g, b = _params(C, seed + 1)
    HW = int(np.prod(spatial))
    dy = synthetic.normal(N * C * HW, 1.0, seed + 2, synthetic.STREAM_DY, dtype).view((N, C) + tuple(spatial))
    pc = [p.cuda() for p in pieces]
    y, mean, invstd = mea.concat_bn_relu_fwd(pc, g.cuda(), b.cuda(), EPS)
    y2 = mea.concat_bn_relu_apply(pc, g.cuda(), b.cuda(), mean, invstd)
    prev = None
    if accumulate:
        prev = [synthetic.normal(p.numel(), 0.5, seed + 3 + i, synthetic.STREAM_PARAM, dtype).view(p.shape)
                for i, p in enumerate(pieces)]
        dps_in = [q.cuda() for q in prev]
        dps, dg, db = mea.concat_bn_relu_bwd(pc, dy.cuda(), g.cuda(), b.cuda(), mean, invstd, dpieces=dps_in,
                                             accumulate=True)
    else:
        dps, dg, db = mea.concat_bn_relu_bwd(pc, dy.cuda(), g.cuda(), b.cuda(), mean, invstd)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)                     # the re-populated output is the forward's, bitwise
    ry, rm, rv, ys = oracle.concat_bn_relu_fwd(_np(pieces), g.double().numpy(), b.double().numpy(), EPS)
    _check_stats(mean, invstd, rm, rv, pieces)
    check_bn(dtype, y.cpu(), ry.ravel(), scale=ys.ravel(), what="y", cap=cap)
    dyn = dy.double().numpy().reshape(N, C, HW)
    rdp, rdg, rdb, rsc = oracle.concat_bn_relu_bwd(_np(pieces), dyn, g.double().numpy(), b.double().numpy(),
                                                   rm, rv, EPS)
    amb, x, r = _ambiguous(pieces, g, b, rm, rv, ys)
    gr = np.abs(g.double().numpy())[None, :, None] * r[None, :, None]
    extra = np.where(amb, gr * np.abs(dyn), 0.0)
    cuts = np.cumsum(ks)[:-1]
    extras = np.split(extra, cuts, axis=1)
    for i, (dp, ref, sc, ex) in enumerate(zip(dps, rdp, rsc, extras)):
        floor = TINY + ex.ravel()
        if accumulate:
            ref = ref + prev[i].double().numpy().reshape(ref.shape)
            sc = sc + np.abs(prev[i].double().numpy().reshape(ref.shape))
        check_bn(dtype, dp.cpu(), ref.ravel(), scale=sc.ravel() + ex.ravel() * 1e5, floor=floor, what=f"dpiece {i}",
                 cap=cap)
    xh = (x - rm[None, :, None]) * r[None, :, None]
    dz = np.where(g.double().numpy()[None, :, None] * xh + b.double().numpy()[None, :, None] > 0, dyn, 0.0)
    # per-channel sums (the rule of _compare.check_channel_sums), plus |dy|
    # (|dy xhat|) for every element whose ReLU side is ambiguous
    c = 1e-8 if N * HW >= (1 << 16) else 1e-6
    tb = np.abs(dz).sum(axis=(0, 2))
    tg = np.abs(dz * xh).sum(axis=(0, 2))
    ab = np.where(amb, np.abs(dyn), 0).sum(axis=(0, 2))
    ag = np.where(amb, np.abs(dyn * xh), 0).sum(axis=(0, 2))
    eb = np.abs(db.cpu().double().numpy() - rdb)
    eg = np.abs(dg.cpu().double().numpy() - rdg)
    assert np.all(eb <= 1e-5 * np.abs(rdb) + c * tb + ab), (eb / (1e-5 * np.abs(rdb) + c * tb + ab)).max()
    assert np.all(eg <= 1e-5 * np.abs(rdg) + c * tg + ag), (eg / (1e-5 * np.abs(rdg) + c * tg + ag)).max()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("N,ks,spatial", [
    (4, [3, 5, 2], (7, 7)),          # planes of 49: scalar path
    (8, [16, 32, 32], (16, 16)),     # planes of 256: 16-byte vectors
    (2, [1] * 7, (3, 5)),            # many one-channel pieces
    (3, [24], (8, 8)),               # a single piece
    (16, [64, 32, 32], (14, 14)),    # 196-element planes: vectors for fp32 only
    # the pipelined path (planes of 16-byte multiples up to 16 KB): one sample
    # and 300 channels (blocks span three channels), 300 samples of two
    # channels (16-byte planes, 300 planes per stage), 16 KB fp32 planes,
    # one-channel pieces, pieces that end inside a block
    (1, [300], (8, 8)),
    (300, [2], (2, 4)),
    (4, [8, 8], (64, 64)),
    (2, [1] * 7, (2, 4)),
    (5, [17, 40], (4, 6)),
])
def test_concat_bn_relu(dtype, N, ks, spatial):
    _run(N, ks, spatial, dtype, 61)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_concat_bn_relu_accumulate(dtype):
    _run(4, [8, 16], (8, 8), dtype, 62, accumulate=True)


def test_concat_bn_relu_densenet_block_size():
    # DenseNet-121, first dense block, sixth layer: 64 + 5 x 32 channels at 56 x 56, batch 64
    _run(64, [64, 32, 32, 32, 32, 32], (56, 56), "bf16", 63)


@pytest.mark.parametrize("spatial", [(9, 9), (8, 8)])   # plane path, pipelined path
def test_concat_bn_relu_running_stats_and_determinism(spatial):
    N, ks = 8, [12, 20]
    pieces = [p.cuda() for p in _pieces(N, ks, spatial, "f32", 64)]
    C = sum(ks)
    g, b = [t.cuda() for t in _params(C, 65)]
    rmean = torch.full((C,), 0.5, device="cuda")
    rvar = torch.full((C,), 2.0, device="cuda")
    y1, m1, i1 = mea.concat_bn_relu_fwd(pieces, g, b, EPS, 0.1, rmean, rvar)
    y2, m2, i2 = mea.concat_bn_relu_fwd(pieces, g, b, EPS)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(m1, m2) and torch.equal(i1, i2)
    _, rm, rv, _ = oracle.concat_bn_relu_fwd(_np([p.cpu() for p in pieces]), g.cpu().double().numpy(),
                                             b.cpu().double().numpy(), EPS)
    em, ev = oracle.bn_running_update(np.full(C, 0.5), np.full(C, 2.0), rm, rv, N * spatial[0] * spatial[1], 0.1)
    # the kernel's statistics are fp32 results (see _check_stats); the update
    # adds one fp64 blend and one rounding to fp32
    assert np.allclose(rmean.cpu().double().numpy(), em, rtol=2e-6, atol=1e-7)
    assert np.allclose(rvar.cpu().double().numpy(), ev, rtol=2e-6, atol=1e-7)


def test_dense_bottleneck_module():
    # normwise agreement of out and every gradient with float64 torch autograd
    # (bf16 storage of y, dy and the outputs: 1e-2), and the saved-tensor
    # contract: neither the concatenation nor the normalized tensor is kept
    import torch.nn.functional as F
    N, ks, spatial = 16, [32, 16, 16, 16], (14, 14)
    C = sum(ks)
    shared = mea.SharedBuffer()
    m = mea.MemoryEfficientDenseBottleneck(C, 64, shared).cuda()
    with torch.no_grad():
        g, b = _params(C, 66)
        m.gamma.copy_(g)
        m.beta.copy_(b)
    pieces = [p.cuda().requires_grad_(True) for p in _pieces(N, ks, spatial, "bf16", 67)]
    dout = synthetic.normal(N * 64 * 196, 1.0, 68, synthetic.STREAM_DY, "bf16").view(N, 64, 14, 14).cuda()
    saved = []

    def pack(t):
        saved.append(tuple(t.shape))
        return t

    with torch.autograd.graph.saved_tensors_hooks(pack, lambda t: t):
        out = m(*pieces)
    out.backward(dout)
    torch.cuda.synchronize()
    assert (N, C) + spatial not in saved
    pd = [p.detach().cpu().double().requires_grad_(True) for p in pieces]
    gd = m.gamma.detach().cpu().double().requires_grad_(True)
    bd = m.beta.detach().cpu().double().requires_grad_(True)
    wd = m.weight.detach().cpu().double().requires_grad_(True)
    ref = F.conv2d(torch.relu(F.batch_norm(torch.cat(pd, 1), None, None, gd, bd, training=True, eps=EPS)), wd)
    ref.backward(dout.cpu().double())

    def rel(a, r):
        return float((a.detach().double().cpu() - r).norm() / r.norm())

    assert rel(out, ref.detach()) < 1e-2
    for p, q in zip(pieces, pd):
        assert rel(p.grad, q.grad) < 1e-2
    assert rel(m.gamma.grad, gd.grad) < 1e-2
    assert rel(m.beta.grad, bd.grad) < 1e-2
    assert rel(m.weight.grad, wd.grad) < 1e-2


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_concat_bn_relu_one_value_per_channel(dtype):
    # N H W = 1: the batch variance is 0 and xhat = 0, so y = max(beta, 0) up
    # to the rounding of the folded gamma' x + beta' (held to the oracle's
    # rules), invstd = eps^-1/2, and dgamma = 0 exactly (x equals its mean).
    # The exact dx is 0 for every element (dz - dbeta / n - xhat dgamma / n
    # cancels completely), so every bf16 dx that is not exactly 0 is held to
    # the scale rule: no cap on their number here.
    _run(1, [5, 3], (1, 1), dtype, 69, cap=1.0)
    pieces = [p.cuda() for p in _pieces(1, [5, 3], (1, 1), dtype, 69)]
    g, b = [t.cuda() for t in _params(8, 70)]
    y, mean, invstd = mea.concat_bn_relu_fwd(pieces, g, b, EPS)
    dps, dg, db = mea.concat_bn_relu_bwd(pieces, torch.ones_like(y), g, b, mean, invstd)
    torch.cuda.synchronize()
    assert torch.allclose(invstd.cpu(), torch.full((8,), EPS ** -0.5), rtol=1e-6)
    assert torch.all(dg == 0)
