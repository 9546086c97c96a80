"""GPU tests of the grouped entry points (mea_act_fwd_grouped /
mea_act_bwd_grouped, mea_swish_channel_fwd_grouped /
mea_swish_channel_bwd_grouped) through the C ABI.

Each segment of a grouped launch runs exactly the work of its own single
launch (same block count, element assignment and summation order), so the
grouped outputs and d alpha must equal mea_act_fwd / mea_act_bwd on each
tensor bit for bit: checked for every activation and both dtypes over
segments of ragged sizes (0, 1, 7, 4097, 100003, 2^20 + 3), a view that is
not 16-byte aligned, more than 32 segments (several launches), host and
device alphas.  The EfficientNet-B0 shapes of the fp32 learnable-alpha
workload are also compared with the oracle directly.  The grouped
per-channel calls are held to the same rule against mea_swish_channel_fwd /
mea_swish_channel_bwd (NCHW) on every segment, including the segments they
launch alone (large planes, unaligned tensors), an empty batch, more than
32 segments and a workspace of arbitrary contents; the EfficientNet-B0 small
stages with alpha per channel are compared with the oracle.
"""
import numpy as np
import pytest
import torch

import memory_efficient_activation_b200 as mea
import oracle
from _compare import TINY, check, check_channel_sums, to_f64
from memory_efficient_activation_b200 import synthetic

pytestmark = pytest.mark.gpu

SIZES = [0, 1, 7, 4097, 100003, (1 << 20) + 3]


def _tensors(sizes, dtype, seed, misaligned=True):
    xs, dys = [], []
    for i, n in enumerate(sizes):
        x = synthetic.normal(n, 3.0, seed + i, synthetic.STREAM_X, dtype).cuda()
        dy = synthetic.normal(n, 1.0, seed + i, synthetic.STREAM_DY, dtype).cuda()
        xs.append(x)
        dys.append(dy)
    if misaligned:
        # one more segment whose tensors start 4 bytes past a 16-byte boundary
        n = 5003
        bx = synthetic.normal(n + 1, 3.0, seed + 99, synthetic.STREAM_X, "f32").to(xs[0].dtype).cuda()
        bg = synthetic.normal(n + 1, 1.0, seed + 99, synthetic.STREAM_DY, "f32").to(xs[0].dtype).cuda()
        xs.append(bx[1:] if dtype == "f32" else bx[2:])
        dys.append(bg[1:] if dtype == "f32" else bg[2:])
    return xs, dys


def _bits(t):
    return t.view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("act", list(synthetic.ACTIVATIONS))
def test_grouped_equals_single_launches(act, dtype):
    xs, dys = _tensors(SIZES, dtype, 501)
    p = 0.01 if act == "leaky_relu" else (1.3 if act == "swish" else 1.0)
    ys = mea.act_fwd_grouped(act, xs, p)
    dxs = mea.act_bwd_grouped(act, xs, dys, p)
    ref_y = [mea.act_fwd(act, x, p) for x in xs]
    ref_dx = [mea.act_bwd(act, x, g, p) for x, g in zip(xs, dys)]
    torch.cuda.synchronize()
    for a, b in zip(ys, ref_y):
        assert torch.equal(_bits(a), _bits(b))
    for a, b in zip(dxs, ref_dx):
        assert torch.equal(_bits(a), _bits(b))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_grouped_dalpha_equals_single_launches(dtype):
    xs, dys = _tensors(SIZES, dtype, 502)
    k = len(xs)
    alphas = [0.5 + 0.25 * i for i in range(k)]
    a_dev = torch.tensor([1.75], dtype=torch.float32, device="cuda")
    param_devs = [a_dev if i % 3 == 2 else None for i in range(k)]
    das = [torch.full((1,), 7.0, device="cuda") for _ in range(k)]
    dxs = mea.act_bwd_grouped("swish", xs, dys, alphas, param_devs=param_devs, dparams=das)
    for _ in range(2):      # the counters return to zero: the same workspace again
        dxs2 = mea.act_bwd_grouped("swish", xs, dys, alphas, param_devs=param_devs,
                                   dparams=[torch.empty(1, device="cuda") for _ in range(k)])
    ref_da = [torch.empty(1, device="cuda") for _ in range(k)]
    ref_dx = [mea.act_bwd("swish", x, g, a, param_dev=pd, dparam=d)
              for x, g, a, pd, d in zip(xs, dys, alphas, param_devs, ref_da)]
    torch.cuda.synchronize()
    for a, b, c in zip(dxs, ref_dx, dxs2):
        assert torch.equal(_bits(a), _bits(b)) and torch.equal(_bits(a), _bits(c))
    for a, b in zip(das, ref_da):
        assert torch.equal(a, b)
    assert float(das[0].item()) == 0.0          # the empty segment's sum


def test_grouped_many_segments():
    # 40 segments: two launches of at most 32
    sizes = [(i * 7919) % 20011 + 1 for i in range(40)]
    xs, dys = _tensors(sizes, "bf16", 503, misaligned=False)
    das = [torch.empty(1, device="cuda") for _ in xs]
    dxs = mea.act_bwd_grouped("swish", xs, dys, 1.0, dparams=das)
    ys = mea.act_fwd_grouped("gelu_tanh", xs)
    torch.cuda.synchronize()
    for x, g, dx, da, y in zip(xs, dys, dxs, das, ys):
        d1 = torch.empty(1, device="cuda")
        assert torch.equal(_bits(dx), _bits(mea.act_bwd("swish", x, g, 1.0, dparam=d1)))
        assert torch.equal(da, d1)
        assert torch.equal(_bits(y), _bits(mea.act_fwd("gelu_tanh", x)))


def test_grouped_effnet_small_shapes_against_oracle():
    # the three smallest EfficientNet-B0 maps of the fp32 learnable-alpha
    # workload in one grouped forward and one grouped backward with d alpha
    ws = [synthetic.effnet_swish_f32(i) for i in (3, 4, 5)]
    xs = [w.x.cuda() for w in ws]
    dys = [w.dy.cuda() for w in ws]
    alphas = [w.param for w in ws]
    ys = mea.act_fwd_grouped("swish", xs, alphas)
    das = [torch.empty(1, device="cuda") for _ in ws]
    dxs = mea.act_bwd_grouped("swish", xs, dys, alphas, dparams=das)
    torch.cuda.synchronize()
    rng = np.random.Generator(np.random.Philox(key=[504, 0]))
    for w, y, dx, da in zip(ws, ys, dxs, das):
        xd, gd = to_f64(w.x), to_f64(w.dy)
        idx = rng.integers(0, w.n, size=1 << 18)
        ti = torch.from_numpy(idx).cuda()
        check("f32", y.view(-1)[ti].cpu(), oracle.act_fwd("swish", xd[idx], w.param), what="grouped fwd")
        check("f32", dx.view(-1)[ti].cpu(), oracle.act_bwd("swish", xd[idx], gd[idx], w.param),
              scale=oracle.act_bwd_scale("swish", xd[idx], gd[idx], w.param),
              floor=TINY * np.maximum(1, np.abs(gd[idx])), what="grouped dx")
        ref = oracle.swish_dalpha(xd, gd, w.param)
        assert abs(float(da.item()) - ref) <= 1e-5 * abs(ref)


def test_grouped_rejects_overlap_and_partial_dparam():
    x = torch.zeros(1000, device="cuda")
    out = torch.empty(1000, device="cuda")
    with pytest.raises(mea.MeaError):
        mea.act_fwd_grouped("swish", [x, x[:10]], outs=[out, out[5:15]])
    with pytest.raises(mea.MeaError):
        mea.act_bwd_grouped("swish", [x, x.clone()], [x.clone(), x.clone()],
                            dparams=[torch.empty(1, device="cuda"), None])


# ------------------------------------------------- Swish with alpha per channel

# Row-path shapes (several planes per vector, a ragged last block, EfficientNet
# stages, 1024-element planes), an empty batch, and plane-path shapes (40 x 40
# and 41 x 25 planes) that the grouped call launches alone.
CHANNEL_SHAPES = [(2, 16, 7, 7), (3, 201, 7, 7), (5, 37, 1, 1), (3, 7, 1, 3), (0, 16, 7, 7), (2, 4, 40, 40),
                  (4, 96, 14, 14), (2, 24, 28, 28), (2, 5, 32, 32), (2, 3, 41, 25)]


def _channel_tensors(shapes, dtype, seed, misaligned=True):
    xs, dys, alphas = [], [], []
    for i, shape in enumerate(shapes):
        w = synthetic.swish_channel_nchw(seed + i, shape, dtype)
        xs.append(w.x.cuda())
        dys.append(w.dy.cuda())
        alphas.append(w.extra["alpha"].cuda())
    if misaligned:
        # tensors one element past a 16-byte boundary: launched alone on the plane path
        shape = (2, 24, 14, 14)
        w = synthetic.swish_channel_nchw(seed + 99, shape, dtype)
        n = w.x.numel()
        bx = torch.empty(n + 1, dtype=w.x.dtype, device="cuda")
        bg = torch.empty(n + 1, dtype=w.x.dtype, device="cuda")
        bx[1:].copy_(w.x.reshape(-1).cuda())
        bg[1:].copy_(w.dy.reshape(-1).cuda())
        xs.append(bx[1:].view(shape))
        dys.append(bg[1:].view(shape))
        alphas.append(w.extra["alpha"].cuda())
    return xs, dys, alphas


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_channel_grouped_equals_single_launches(dtype):
    xs, dys, alphas = _channel_tensors(CHANNEL_SHAPES, dtype, 511)
    ys = mea.swish_channel_fwd_grouped(xs, alphas)
    dxs, das = mea.swish_channel_bwd_grouped(xs, dys, alphas)
    ref_y = [mea.swish_channel_fwd(x, a, "nchw") for x, a in zip(xs, alphas)]
    ref = [mea.swish_channel_bwd(x, g, a, "nchw") for x, g, a in zip(xs, dys, alphas)]
    torch.cuda.synchronize()
    for a, b in zip(ys, ref_y):
        assert torch.equal(_bits(a), _bits(b))
    for dx, da, (rdx, rda) in zip(dxs, das, ref):
        assert torch.equal(_bits(dx), _bits(rdx))
        assert torch.equal(da.view(torch.int32), rda.view(torch.int32))
    assert torch.all(das[CHANNEL_SHAPES.index((0, 16, 7, 7))] == 0)


def test_channel_grouped_many_segments_and_dirty_workspace():
    # 40 row-path segments (two grids of at most 32), a workspace filled with
    # garbage before each call: the same bits every time
    shapes = [(1 + i % 3, 8 + 4 * (i % 5), 7, 7) if i % 2 else (2, 12 + i, 14, 14) for i in range(40)]
    xs, dys, alphas = _channel_tensors(shapes, "f32", 521, misaligned=False)
    need = mea.swish_channel_bwd_grouped_workspace_bytes(torch.float32, [tuple(x.shape) for x in xs])
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    outs = []
    for fill in (0, 255, 77):
        ws.fill_(fill)
        outs.append(mea.swish_channel_bwd_grouped(xs, dys, alphas, workspace=ws))
    ref = [mea.swish_channel_bwd(x, g, a, "nchw") for x, g, a in zip(xs, dys, alphas)]
    torch.cuda.synchronize()
    for dxs, das in outs:
        for dx, da, (rdx, rda) in zip(dxs, das, ref):
            assert torch.equal(dx.view(torch.int32), rdx.view(torch.int32))
            assert torch.equal(da.view(torch.int32), rda.view(torch.int32))


def test_channel_grouped_effnet_small_planes_against_oracle():
    # EfficientNet-B0's 28 x 28, 14 x 14 and 7 x 7 stages with alpha per
    # channel, batch 64, fp32, in one grouped forward and backward: every
    # output against the oracle
    shapes = [(64, 240, 28, 28), (64, 480, 14, 14), (64, 1152, 7, 7)]
    ws = [synthetic.swish_channel_nchw(531 + i, s) for i, s in enumerate(shapes)]
    xs = [w.x.cuda() for w in ws]
    ys = mea.swish_channel_fwd_grouped(xs, [w.extra["alpha"].cuda() for w in ws])
    dxs, das = mea.swish_channel_bwd_grouped(xs, [w.dy.cuda() for w in ws], [w.extra["alpha"].cuda() for w in ws])
    torch.cuda.synchronize()
    del xs
    for w, y, dx, da in zip(ws, ys, dxs, das):
        xd, gd = to_f64(w.x), to_f64(w.dy)
        aa = w.extra["alpha"].double().numpy()
        N, C, H, W = w.extra["nchw_shape"]
        ry = oracle.swish_channel_fwd("nchw", (N, C, H, W), xd, aa)
        rdx, rda, scale = oracle.swish_channel_bwd("nchw", (N, C, H, W), xd, gd, aa)
        check("f32", y.cpu(), ry, what="grouped channel fwd")
        check("f32", dx.cpu(), rdx, scale=scale, floor=TINY * np.maximum(1, np.abs(gd)), what="grouped channel dx")
        ch = (np.arange(xd.size) // (H * W)) % C
        t = aa[ch] * xd
        terms = np.abs(gd * xd * xd) / ((1.0 + np.exp(-t)) * (1.0 + np.exp(t)))
        check_channel_sums(da, rda, np.bincount(ch, terms, minlength=C), xd.size // C, "grouped dalpha")


def test_channel_grouped_rejects_overlap():
    x = torch.zeros(2, 16, 7, 7, device="cuda")
    a = torch.ones(16, device="cuda")
    out = torch.empty(2 * 16 * 49 + 10, device="cuda")
    with pytest.raises(mea.MeaError):
        mea.swish_channel_fwd_grouped([x, x.clone()], [a, a], outs=[out[:1568].view(2, 16, 7, 7),
                                                                   out[10:1578].view(2, 16, 7, 7)])
    with pytest.raises(mea.MeaError):
        da = torch.empty(16, device="cuda")
        mea.swish_channel_bwd_grouped([x, x.clone()], [x.clone(), x.clone()], [a, a], dalphas=[da, da])
