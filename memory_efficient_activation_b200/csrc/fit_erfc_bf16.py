"""Fits the polynomials of the bf16-storage GELU-erf kernels (mea_math.cuh,
GeluErf).  Both use t = 1 / (1 + a / 2), a = |w|, the variable of Press et
al., "Numerical Recipes in C", 2nd ed., section 6.2:

  forward  (nr5_parts):  log(erfc(a) / t) + a^2 ~ P5(t)   (degree 5; the
           Numerical Recipes form with fewer terms)
  backward (q8, q8_2):   erfcx(a) / t = erfc(a) e^(a^2) / t ~ Q8(t)
           (degree 8), so that erfc(a) = t e^(-a^2) Q8(t) shares its
           exponential with the Gaussian of the derivative.

Each is a least-squares fit in a Chebyshev basis over t in [1 / (1 + 9.6 / 2),
1] (a in [0, 9.6]: x down to -13.6, below which the kernels' tail branch
takes over), reweighted toward the minimax solution (Lawson's iteration;
relative weighting for Q8), then converted to monomials in t and rounded to
fp32.  Prints the coefficients t^0 .. t^n and the maximum error of each.

    python memory_efficient_activation_b200/csrc/fit_erfc_bf16.py
"""
import numpy as np
from scipy.special import erfcx

A_MAX = 9.6


def _to_monomials(c, tmin):
    sp = np.polynomial.Polynomial([-(1.0 + tmin) / (1.0 - tmin), 2.0 / (1.0 - tmin)])
    prev, cur = np.polynomial.Polynomial([1.0]), sp
    poly = c[0] * prev + c[1] * cur
    for k in range(2, len(c)):
        prev, cur = cur, 2.0 * sp * cur - prev
        poly = poly + c[k] * cur
    return poly.coef


def _lawson(t, target, degree, tmin, relative, iterations):
    s = (2.0 * t - (1.0 + tmin)) / (1.0 - tmin)
    v = np.polynomial.chebyshev.chebvander(s, degree)
    scale = target if relative else np.ones_like(target)
    w = np.ones_like(t)
    for _ in range(iterations):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(v * (sw / scale)[:, None], target * sw / scale, rcond=None)
        e = (v @ c - target) / scale
        w = w * np.abs(e)
        w /= w.sum()
    return _to_monomials(c, tmin)


def fit(degree=5, a_max=A_MAX, points=400001, iterations=200):
    """P5 of the forward: log(erfc(a) / t) + a^2 (absolute error of log erfc,
    i.e. relative error of erfc)."""
    tmin = 1.0 / (1.0 + a_max / 2.0)
    t = np.linspace(tmin, 1.0, points)
    a = 2.0 * (1.0 / t - 1.0)
    q = np.log(erfcx(a) / t)                   # log(erfc(a) / t) + a^2
    coef32 = _lawson(t, q, degree, tmin, False, iterations).astype(np.float32)
    err = np.abs(np.polynomial.polynomial.polyval(t, coef32.astype(np.float64)) - q).max()
    return coef32, err


def fit_q(degree=8, a_max=A_MAX, points=200001, iterations=150):
    """Q8 of the backward: erfcx(a) / t (relative error)."""
    tmin = 1.0 / (1.0 + a_max / 2.0)
    t = np.linspace(tmin, 1.0, points)
    a = 2.0 * (1.0 / t - 1.0)
    q = erfcx(a) / t
    coef32 = _lawson(t, q, degree, tmin, True, iterations).astype(np.float32)
    err = np.abs(np.polynomial.polynomial.polyval(t, coef32.astype(np.float64)) / q - 1.0).max()
    return coef32, err


if __name__ == "__main__":
    coef, err = fit()
    print("forward P5: max |error| of log erfc:", err)
    for k, c in enumerate(coef):
        print(f"  t^{k}: {float(c):.9g}")
    coef, err = fit_q()
    print("backward Q8: max relative error:", err)
    for k, c in enumerate(coef):
        print(f"  t^{k}: {float(c):.9g}")
