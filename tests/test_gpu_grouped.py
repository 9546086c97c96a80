"""GPU tests of the grouped entry points (mea_act_fwd_grouped /
mea_act_bwd_grouped) through the C ABI.

Each segment of a grouped launch runs exactly the work of its own single
launch (same block count, element assignment and summation order), so the
grouped outputs and d alpha must equal mea_act_fwd / mea_act_bwd on each
tensor bit for bit: checked for every activation and both dtypes over
segments of ragged sizes (0, 1, 7, 4097, 100003, 2^20 + 3), a view that is
not 16-byte aligned, more than 32 segments (several launches), host and
device alphas.  The EfficientNet-B0 shapes of the fp32 learnable-alpha
workload are also compared with the oracle directly.
"""
import numpy as np
import pytest
import torch

import memory_efficient_activation_b200 as mea
import oracle
from _compare import TINY, check, to_f64
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
