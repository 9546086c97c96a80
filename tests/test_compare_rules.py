"""CPU checks of the comparison rules themselves (tests/_compare.py): each
rule must pass what a correct kernel's rounding produces and catch the
mistakes it is there for.  Mistakes are planted in the expected values'
neighbourhood on the CPU; no GPU and no kernel is involved.

* bf16: one ulp of the oracle rounded to bf16 passes, two fail.
* per-channel sums: a single dropped term of average size fails, also with
  the fp32-storage weighting, where near the zero of f' a term's weight is
  its condition scale rather than |t|.
"""
import numpy as np
import pytest
import torch

from _compare import assert_bf16, check_channel_sums, sum_weights_f32


def _bf16_neighbour(v: np.ndarray, steps: int) -> torch.Tensor:
    """The bf16 value `steps` ulps above the bf16 rounding of v (v > 0)."""
    b = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16)
    bits = b.view(torch.int16).to(torch.int32) + steps
    return bits.to(torch.int16).view(torch.bfloat16)


def test_bf16_rule_one_ulp_passes_two_fail():
    rng = np.random.default_rng(11)
    ref = rng.uniform(0.5, 4.0, 1000)
    assert_bf16(_bf16_neighbour(ref, 1), ref, what="one ulp")
    with pytest.raises(AssertionError):
        assert_bf16(_bf16_neighbour(ref, 2), ref, what="two ulps")


def _channels(n_c: int, C: int, seed: int, near_root: bool):
    """Per-channel terms t = dz x of fp32 magnitude, half of them (when
    near_root) tiny with a condition scale of the size of an ordinary term."""
    rng = np.random.default_rng(seed)
    t = rng.normal(0.0, 1.0, (C, n_c))
    cond = np.abs(t).copy()
    if near_root:
        t[:, ::2] *= 1e-4                     # f' near its zero: small terms
        cond[:, ::2] = 0.45 * np.abs(rng.normal(0.0, 1.0, (C, n_c // 2)))
    return t, cond


@pytest.mark.parametrize("near_root", [False, True])
def test_channel_sums_catch_a_dropped_term(near_root):
    C, n_c = 16, 50
    t, cond = _channels(n_c, C, 21, near_root)
    ref = t.sum(axis=1)
    w, z = sum_weights_f32(t, cond, np.zeros_like(t))
    weights, extra = w.sum(axis=1), z.sum(axis=1)
    # a correct fp32 kernel: the terms rounded to fp32 and summed in fp32
    got_ok = torch.from_numpy(t.astype(np.float32).sum(axis=1, dtype=np.float32))
    check_channel_sums(got_ok, ref, weights, n_c, "rounded sums", extra=extra)
    # one ordinary (non-near-root) term dropped from channel 3
    bad = ref.copy()
    bad[3] -= t[3, 1]
    with pytest.raises(AssertionError):
        check_channel_sums(torch.from_numpy(bad), ref, weights, n_c, "dropped term", extra=extra)


def test_fp32_weighting_changes_nothing_away_from_the_root():
    t, cond = _channels(50, 8, 31, near_root=False)
    w, z = sum_weights_f32(t, cond, np.zeros_like(t))
    assert np.array_equal(w, np.abs(t))
    assert not np.any(z)
