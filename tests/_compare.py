"""Comparison rules between GPU outputs and the oracle (test helpers).

bf16 outputs: the ordered-integer distance between the GPU's bit pattern and
the oracle's double result rounded to nearest-even bf16 is at most 1 (+0 and
-0 count as equal; NaN matches NaN).  No other allowance.

fp32 outputs: |g - r| <= 1e-5 * max(|r|, m) + e, where r is the oracle's
double result, m the condition scale of the output (for a backward product,
|dy| times the sum of the absolute terms of f'; for a forward, |r| itself)
and e, for outputs of the per-channel affine only, the oracle's bound on how
far the exact result moves when z = gamma x + beta is rounded once to fp32
(oracle.affine_act_zround; zero elsewhere).  This is the fp32 bound "max
relative error 1e-5" read per element, with the denominator taken from the
terms where f' cancels near its zero, and with the error that forming the
affine's z in fp32 carries into any fp32 evaluation.

Both: results whose exact value is below the smallest normal, 2^-126, may be
flushed; they pass when |g - r| <= floor (2^-126 unless a caller scales it,
e.g. by |dy| for a backward product).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TINY = 2.0 ** -126
F32_TOL = 1e-5


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16).ravel()


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy().ravel()


def _ordered(bits: np.ndarray) -> np.ndarray:
    b = bits.astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def bf16_report(gpu: torch.Tensor, ref: np.ndarray, floor=None) -> dict:
    g_bits = bf16_bits(gpu)
    ref = np.asarray(ref, dtype=np.float64).ravel()
    r_bits = oracle.round_bf16(ref)
    dist = np.abs(_ordered(g_bits) - _ordered(r_bits))
    g = bits_to_f64(g_bits)
    fl = TINY if floor is None else np.asarray(floor, dtype=np.float64).ravel()
    with np.errstate(invalid="ignore"):
        nan_ok = np.isnan(g) & np.isnan(ref)
        tiny_ok = (np.abs(ref) < TINY) & (np.abs(g - ref) <= fl)
    ok = (dist <= 1) | nan_ok | tiny_ok
    bad = np.flatnonzero(~ok)
    return {
        "n": ref.size,
        "bad": bad.size,
        "ok": ok,
        "max_ulp": int(dist[~(nan_ok | tiny_ok)].max(initial=0)),
        "exact_frac": float(np.mean(dist == 0)) if ref.size else 1.0,
        "first_bad": [(int(i), float(ref[i]), float(g[i]), int(dist[i])) for i in bad[:8]],
    }


def f32_report(gpu: torch.Tensor, ref: np.ndarray, scale=None, floor=None, tol=F32_TOL, zround=None) -> dict:
    g = to_f64(gpu)
    ref = np.asarray(ref, dtype=np.float64).ravel()
    denom = np.abs(ref) if scale is None else np.maximum(np.abs(ref), np.asarray(scale).ravel())
    fl = TINY if floor is None else np.asarray(floor, dtype=np.float64).ravel()
    e = 0.0 if zround is None else np.asarray(zround, dtype=np.float64).ravel()
    with np.errstate(invalid="ignore", divide="ignore"):
        err = np.abs(g - ref)
        nan_ok = np.isnan(g) & np.isnan(ref)
        same = g == ref
        tiny_ok = (np.abs(ref) < TINY) & (err <= fl)
        base_ok = (err <= tol * denom) | nan_ok | same | tiny_ok
        ok = base_ok | (err <= tol * denom + e)
        rel = np.where(denom > 0, err / denom, 0.0)
        pure = np.where(np.abs(ref) >= TINY, err / np.abs(ref), 0.0)
    bad = np.flatnonzero(~ok)
    sel = ~(nan_ok | same | tiny_ok)
    return {
        "n": ref.size,
        "bad": bad.size,
        "ok": ok,
        "zround_only": int(np.sum(ok & ~base_ok)),
        "max_rel": float(np.nanmax(rel[sel], initial=0.0)),
        "max_pure_rel": float(np.nanmax(pure[sel], initial=0.0)),
        "pure_over_tol": int(np.sum(pure[sel] > tol)),
        "first_bad": [(int(i), float(ref[i]), float(g[i])) for i in bad[:8]],
    }


def _shown(r):
    return {k: v for k, v in r.items() if k != "ok"}


def assert_bf16(gpu, ref, floor=None, what=""):
    r = bf16_report(gpu, ref, floor)
    assert r["bad"] == 0, f"{what}: {_shown(r)}"
    return r


def assert_f32(gpu, ref, scale=None, floor=None, what="", tol=F32_TOL, zround=None):
    r = f32_report(gpu, ref, scale, floor, tol, zround)
    assert r["bad"] == 0, f"{what}: {_shown(r)}"
    return r


def check(dtype: str, gpu, ref, scale=None, floor=None, what="", zround=None):
    """bf16: the 1-ulp rule.  fp32: the rule above; zround is the oracle's
    z-rounding bound of each element (per-channel affine outputs only)."""
    if dtype == "bf16":
        return assert_bf16(gpu, ref, floor, what)
    return assert_f32(gpu, ref, scale, floor, what, zround=zround)


def check_bn(dtype: str, gpu, ref, scale, floor=None, what="", cap=1e-3) -> dict:
    """Outputs of batch normalization (y and dx).  They depend on the batch
    statistics, which any kernel holds in fp32 (mean and invstd are each
    rounded, 2^-24 relative), so where gamma xhat + beta, or the terms of dx,
    cancel, that rounding alone moves the exact result by more than a bf16
    ulp.  A bf16 element that misses the 1-ulp rule therefore passes when it
    meets the fp32 rule against the oracle's scale of its terms:
    |g - r| <= 1e-5 scale.  How many elements pass only that way is returned
    ("scale_only") and must stay below cap of the total.  fp32 outputs use
    the fp32 rule with the same scale."""
    if dtype != "bf16":
        return assert_f32(gpu, ref, scale, floor, what)
    r = bf16_report(gpu, ref, floor)
    g = bits_to_f64(bf16_bits(gpu))
    ref = np.asarray(ref, dtype=np.float64).ravel()
    with np.errstate(invalid="ignore"):
        scale_ok = np.abs(g - ref) <= F32_TOL * np.asarray(scale, dtype=np.float64).ravel()
    ok = r["ok"] | scale_ok
    r["scale_only"] = int(np.sum(scale_ok & ~r["ok"]))
    r["bad"] = int(np.sum(~ok))
    r["first_bad"] = [f for f in r["first_bad"] if not scale_ok[f[0]]]
    assert r["bad"] == 0, f"{what}: {_shown(r)}"
    assert r["scale_only"] <= cap * max(r["n"], 1), f"{what}: {_shown(r)}"
    return r


def check_channel_sums(got, ref, terms_abs, terms_per_channel: int, what="", extra=None):
    """Per-channel fp32 sums (dgamma, dbeta, dalpha):
    |g - r| <= 1e-5 |r| + c sum_i |t_i| (+ extra, a per-channel allowance the
    caller derives from the per-element rule of fp32 storage; see
    sum_weights_f32).  Where every channel sums at least
    2^16 terms, c = 1e-8: the kernels' rounding is then random-signed (dy has
    random sign), about sqrt(n) 2^-24 mean|t| in all, far below 1e-8 n mean|t|,
    while a single dropped or doubled term of average size moves the sum by
    1/n of sum|t|, 1.5e-5 or more.  Smaller channels use c = 1e-6, which covers
    the worst case of the kernels' fp32 runs (at most 16 terms: 15 2^-24 =
    8.9e-7) and is still below 1/n for every n here."""
    c = 1e-8 if terms_per_channel >= (1 << 16) else 1e-6
    g = got.detach().cpu().double().numpy().ravel()
    ref = np.asarray(ref, dtype=np.float64).ravel()
    ta = np.asarray(terms_abs, dtype=np.float64).ravel()
    err = np.abs(g - ref)
    ok = err <= 1e-5 * np.abs(ref) + c * ta + (0.0 if extra is None else np.asarray(extra, dtype=np.float64).ravel())
    assert np.all(ok), (what, [(int(i), float(g[i]), float(ref[i]), float(ta[i])) for i in np.flatnonzero(~ok)[:6]])
    with np.errstate(invalid="ignore", divide="ignore"):
        return {"max_rel": float(np.nanmax(np.where(ref != 0, err / np.abs(ref), 0.0), initial=0.0)),
                "max_err_over_terms": float(np.nanmax(np.where(ta > 0, err / ta, 0.0), initial=0.0))}


def sum_weights_f32(terms, cond, zround):
    """Term weights and the additive allowance of a per-channel sum whose
    terms come from fp32 storage: each term obeys the fp32 rule (error
    relative to the condition scale `cond` of its f', plus the exact change
    `zround` when z is rounded once to fp32), so its weight in the sum rule
    is max(|t|, cond) and the z-rounding changes add up exactly.  Away from
    the zero of f' cond = |t| and nothing changes; near it the fp32 terms
    cancel inside f' (bf16 storage recomputes those elements and keeps
    |t|).  Returns (weights, allowance) per element."""
    t = np.abs(np.asarray(terms, dtype=np.float64))
    return np.maximum(t, np.asarray(cond, dtype=np.float64)), np.abs(np.asarray(zround, dtype=np.float64))
