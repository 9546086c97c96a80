"""GPU parity of the matmul + activation kernels (mea_matmul_act_fwd /
mea_matmul_act_bwd, tcgen05 tensor cores) against the oracle, through the
C ABI.

Tolerances, from the arithmetic:
  * Z: the tensor cores multiply bf16 exactly and accumulate in fp32, so the
    accumulated sum differs from the exact one by at most K 2^-23 of
    S = sum_k |x_k w_k| (every addition may err by one fp32 ulp of a partial
    sum bounded by S); the stored value then adds the bf16 rounding (half an
    ulp, one ulp when the two roundings meet).  Besides the bound, at least
    99% of the elements must equal the oracle's bf16 rounding or its
    neighbour: a systematic fault (a misplaced K step, a transposed operand)
    breaks every element, not a few.
  * y = f(z as stored): within L (the bound on Z) plus two bf16 ulps of the
    oracle's f at the exact Z, L the largest |f'| of the activation (a
    Lipschitz constant: 1 for ReLU, LeakyReLU and tanh, 1/4 for sigmoid,
    1.129 for both GELUs, 1.0998 for Swish at any alpha); and 99% of the
    elements within one ulp of the oracle's f at its own bf16 rounding of Z.
  * dz = (G W^T) f'(z) for a z given as input (the oracle's rounded Z): one
    bf16 ulp of the exact value plus |f'(z)| times the accumulation bound of
    G W^T, plus 2^-20 relative for the fp32 evaluation of f'; and the same
    99% rule.
Shapes cover one tile, ragged M / N / K (boundary tiles, a partial last K
block), many tiles per CTA (both accumulator buffers in turn) and the
full-size [16384 x 4096] x [4096 x 4096] case on sampled rows.
"""
import numpy as np
import pytest
import torch

import memory_efficient_activation_b200 as mea
import oracle
from _compare import TINY, bf16_bits, bits_to_f64
from memory_efficient_activation_b200 import synthetic

pytestmark = pytest.mark.gpu

ACTS = list(synthetic.ACTIVATIONS)


def _p(act):
    return 0.01 if act == "leaky_relu" else (1.25 if act == "swish" else 1.0)


def _bf16(n, sigma, seed, stream):
    return synthetic.normal(n, sigma, seed, stream, "bf16")


def _inputs(M, N, K, seed):
    x = _bf16(M * K, 1.0, seed, synthetic.STREAM_X).view(M, K)
    w = _bf16(N * K, K ** -0.5, seed, synthetic.STREAM_PARAM).view(N, K)
    g = _bf16(M * K, 1.0, seed, synthetic.STREAM_DY).view(M, K)
    return x, w, g


def _ordered(bits):
    b = bits.astype(np.int64)
    return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)


def _ulp_bf16(v):
    a = np.maximum(np.abs(v), TINY)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def _z_bound(Z, S, K):
    return _ulp_bf16(Z) + K * 2.0 ** -23 * S + TINY


def _check_z(z_gpu, Z, S, K, what):
    zg = bits_to_f64(bf16_bits(z_gpu)).reshape(Z.shape)
    err = np.abs(zg - Z)
    bound = _z_bound(Z, S, K)
    assert np.all(err <= bound), (what, float((err / bound).max()))
    dist = np.abs(_ordered(bf16_bits(z_gpu)) - _ordered(oracle.round_bf16(Z.ravel())))
    assert np.mean(dist <= 1) >= 0.99, (what, np.bincount(np.minimum(dist, 9)))


LIPSCHITZ = {"relu": 1.0, "leaky_relu": 1.0, "sigmoid": 0.25, "tanh": 1.0, "gelu_erf": 1.1290,
             "gelu_tanh": 1.1290, "swish": 1.0999}


def _check_y(act, p, y_gpu, Yexact, Yround, zbound, what):
    yg = bits_to_f64(bf16_bits(y_gpu)).reshape(Yexact.shape)
    err = np.abs(yg - Yexact)
    bound = LIPSCHITZ[act] * zbound + 2 * _ulp_bf16(Yexact) + TINY
    assert np.all(err <= bound), (what, float((err / bound).max()))
    dist = np.abs(_ordered(bf16_bits(y_gpu)) - _ordered(oracle.round_bf16(Yround.ravel())))
    assert np.mean(dist <= 1) >= 0.99, (what, np.bincount(np.minimum(dist, 9)))


def _check_dz(act, p, dz_gpu, dZ, D, S, zst, K, what):
    dg = bits_to_f64(bf16_bits(dz_gpu)).reshape(dZ.shape)
    fp = np.abs(oracle.act_deriv(act, zst.ravel(), p)).reshape(dZ.shape)
    bound = _ulp_bf16(dZ) + fp * K * 2.0 ** -23 * S + 2.0 ** -20 * np.abs(dZ) + TINY
    err = np.abs(dg - dZ)
    assert np.all(err <= bound), (what, float((err / bound).max()))
    dist = np.abs(_ordered(bf16_bits(dz_gpu)) - _ordered(oracle.round_bf16(dZ.ravel())))
    assert np.mean(dist <= 1) >= 0.99, (what, np.bincount(np.minimum(dist, 9)))


def _run(act, M, N, K, seed, rows=None):
    p = _p(act)
    x, w, g = _inputs(M, N, K, seed)
    sel = slice(None) if rows is None else torch.from_numpy(rows)
    xd = x.double().numpy() if rows is None else x[sel].double().numpy()
    wd = w.double().numpy()
    # the backward's stored z: the oracle's own Z rounded to bf16, all rows
    # when every row is checked, else only the sampled rows are meaningful
    if rows is None:
        Zfull, Yround, S = oracle.matmul_act_fwd(act, xd, wd, p, round_z_bf16=True)
        zin = torch.from_numpy(Zfull).to(torch.bfloat16)
    else:
        Zs, Yround, S = oracle.matmul_act_fwd(act, xd, wd, p, round_z_bf16=True)
        zin = torch.zeros(M, N, dtype=torch.bfloat16)
        zin[sel] = torch.from_numpy(Zs).to(torch.bfloat16)
    xc, wc, gc = x.cuda(), w.cuda(), g.cuda()
    z, y = mea.matmul_act_fwd(act, xc, wc, p)
    dz = mea.matmul_act_bwd(act, gc, wc, zin.cuda(), p)
    torch.cuda.synchronize()
    Z = Zfull if rows is None else Zs
    _, Yexact, _ = oracle.matmul_act_fwd(act, xd, wd, p, round_z_bf16=False)
    _check_z(z.cpu()[sel], Z, S, K, f"{act} z {M}x{N}x{K}")
    _check_y(act, p, y.cpu()[sel], Yexact, Yround, _z_bound(Z, S, K), f"{act} y {M}x{N}x{K}")
    zst = zin[sel].double().numpy()
    gd = g.double().numpy() if rows is None else g[sel].double().numpy()
    dZ, D, S2 = oracle.matmul_act_bwd(act, gd, wd, zst, p)
    _check_dz(act, p, dz.cpu()[sel], dZ, D, S2, zst, K, f"{act} dz {M}x{N}x{K}")


@pytest.mark.parametrize("act", ACTS)
@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (300, 264, 200), (1000, 520, 1024)])
def test_matmul_act_small(act, M, N, K):
    _run(act, M, N, K, 31)


@pytest.mark.parametrize("act", ["swish", "gelu_erf"])
def test_matmul_act_many_tiles_per_cta(act):
    # 32 x 8 = 256 tiles over at most 148 CTAs: CTAs take two tiles, using
    # both tensor-memory accumulators; rows sampled across all row tiles
    M, N, K = 4096, 2048, 512
    rows = np.sort(np.random.Generator(np.random.Philox(key=[32, 0])).choice(M, 192, replace=False))
    _run(act, M, N, K, 32, rows)


def test_matmul_act_full_size_sampled():
    # the d x d matmul of problem B07: [8 x 2048, 4096] x [4096, 4096]
    M, N, K = 16384, 4096, 4096
    rows = np.sort(np.random.Generator(np.random.Philox(key=[33, 0])).choice(M, 48, replace=False))
    _run("gelu_erf", M, N, K, 33, rows)


def test_matmul_act_z_only_and_y_only():
    x, w, _ = _inputs(256, 512, 128, 34)
    xc, wc = x.cuda(), w.cuda()
    z1, y1 = mea.matmul_act_fwd("tanh", xc, wc)
    z2, none_y = mea.matmul_act_fwd("tanh", xc, wc, want_y=False)
    none_z, y3 = mea.matmul_act_fwd("tanh", xc, wc, want_z=False)
    torch.cuda.synchronize()
    assert none_y is None and none_z is None
    assert torch.equal(z1, z2) and torch.equal(y1, y3)


def test_matmul_act_deterministic_and_in_place_dz():
    x, w, g = _inputs(640, 768, 320, 35)
    xc, wc, gc = x.cuda(), w.cuda(), g.cuda()
    outs = [mea.matmul_act_fwd("swish", xc, wc, 1.25) for _ in range(3)]
    dzs = [mea.matmul_act_bwd("swish", gc, wc, outs[0][0], 1.25) for _ in range(3)]
    zc = outs[0][0].clone()
    dz_in = mea.matmul_act_bwd("swish", gc, wc, zc, 1.25, out=zc)    # dz written over z
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o[0], outs[0][0]) and torch.equal(o[1], outs[0][1])
    for d in dzs[1:]:
        assert torch.equal(d, dzs[0])
    assert torch.equal(dz_in, dzs[0])


def test_matmul_act_matches_unfused_path():
    # fused epilogue == the same product followed by the streaming activation
    # kernels on the stored z (the kernels' own activation arithmetic)
    x, w, g = _inputs(512, 1024, 256, 36)
    xc, wc, gc = x.cuda(), w.cuda(), g.cuda()
    for act in ACTS:
        p = _p(act)
        z, y = mea.matmul_act_fwd(act, xc, wc, p)
        y2 = mea.act_fwd(act, z, p)
        dz = mea.matmul_act_bwd(act, gc, wc, z, p)
        d = mea.matmul_act_bwd("relu", gc, wc, torch.full_like(z, 1.0))   # relu'(1) = 1: the bare product
        dz2 = mea.act_bwd(act, z, d, p)
        torch.cuda.synchronize()
        dy = np.abs(_ordered(bf16_bits(y)) - _ordered(bf16_bits(y2)))
        assert dy.max() <= 1, (act, dy.max())
        # dz2 saw the product rounded to bf16 first; the fused path did not
        dist = np.abs(_ordered(bf16_bits(dz)) - _ordered(bf16_bits(dz2)))
        assert dist.max() <= 1, (act, dist.max())


def _mlp_ref(act, p, x, w1, w2):
    """float64 torch autograd of the same MLP (a library check of the
    module's plumbing, not of the kernels' rounding)."""
    import torch.nn.functional as F
    fn = {
        "relu": lambda t: torch.relu(t),
        "leaky_relu": lambda t: F.leaky_relu(t, negative_slope=p),
        "sigmoid": torch.sigmoid,
        "tanh": torch.tanh,
        "gelu_erf": lambda t: F.gelu(t, approximate="none"),
        "gelu_tanh": lambda t: F.gelu(t, approximate="tanh"),
        "swish": lambda t: t * torch.sigmoid(p * t),
    }[act]
    xd = x.double().requires_grad_(True)
    w1d = w1.double().requires_grad_(True)
    w2d = w2.double().requires_grad_(True)
    out = fn(xd @ w1d.t()) @ w2d.t()
    return out, xd, w1d, w2d


@pytest.mark.parametrize("act", ["gelu_tanh", "swish", "relu"])
def test_memory_efficient_mlp_module(act):
    # normwise agreement with float64 autograd: every bf16 store (z, f(z),
    # dz, and the outputs) rounds by at most 2^-9 relative, and the two
    # matmul stages compound a few of them: 1e-2 normwise bounds it
    torch.manual_seed(0)
    M, d, h = 512, 256, 1024
    m = mea.MemoryEfficientMLP(d, h, act).cuda()
    x = _bf16(M * d, 1.0, 37, synthetic.STREAM_X).view(4, M // 4, d).cuda().requires_grad_(True)
    dout = _bf16(M * d, 1.0, 37, synthetic.STREAM_DY).view(4, M // 4, d).cuda()
    saved = []

    def pack(t):
        saved.append(t)
        return t

    with torch.autograd.graph.saved_tensors_hooks(pack, lambda t: t):
        out = m(x)
    out.backward(dout)
    torch.cuda.synchronize()
    p = m.param
    ref, xd, w1d, w2d = _mlp_ref(act, p, x.detach().cpu().view(M, d), m.w1.detach().cpu(), m.w2.detach().cpu())
    ref.backward(dout.cpu().view(M, d).double())

    def rel(a, b):
        return float((a.detach().double().cpu() - b.detach()).norm() / b.detach().norm())

    assert rel(out.view(M, d), ref) < 1e-2
    assert rel(x.grad.view(M, d), xd.grad) < 1e-2
    assert rel(m.w1.grad, w1d.grad) < 1e-2
    assert rel(m.w2.grad, w2d.grad) < 1e-2
    # saved for the backward: x, w1, w2 and z = x w1^T, not f(z)
    hidden = [t for t in saved if t.dim() == 2 and t.shape == (M, h)]
    assert len(hidden) == 1


@pytest.mark.parametrize("M,N,K", [(1, 8, 8), (7, 16, 24), (100, 8, 64), (129, 264, 8)])
def test_matmul_act_tiny_and_ragged(M, N, K):
    # single rows, the narrowest N and K the C ABI takes, M that leaves the
    # second CTA of the pair (or most of the first) without rows
    _run("swish", M, N, K, 38)


def test_matmul_error_word_clear():
    # no bounded wait expired in any matmul launched by this test session
    assert mea._capi.lib().mea_matmul_error_word(1) == 0
    assert mea._capi.lib().mea_matmul_error_word(0) == 0
