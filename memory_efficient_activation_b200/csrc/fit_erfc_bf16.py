"""Fits the degree-5 polynomial of the bf16-storage GELU-erf forward
(mea_math.cuh, GeluErf::nr5_parts): log(erfc(a) / t) + a^2 ~ P(t) with
t = 1 / (1 + a / 2), the form of Press et al., "Numerical Recipes in C",
2nd ed., section 6.2, with fewer terms.  Least squares in a Chebyshev basis
over t in [1 / (1 + 9.6 / 2), 1] (a in [0, 9.6]: x down to -13.6, below
which the kernel's tail branch takes over), reweighted toward the minimax
solution (Lawson's iteration), then converted to monomials in t and rounded
to fp32.  Prints the coefficients t^0 .. t^5 and the maximum error of
log erfc (7.6e-6, i.e. relative error of erfc).

    python memory_efficient_activation_b200/csrc/fit_erfc_bf16.py
"""
import numpy as np
from scipy.special import erfcx

DEGREE = 5
A_MAX = 9.6


def fit(degree=DEGREE, a_max=A_MAX, points=400001, iterations=200):
    tmin = 1.0 / (1.0 + a_max / 2.0)
    t = np.linspace(tmin, 1.0, points)
    a = 2.0 * (1.0 / t - 1.0)
    q = np.log(erfcx(a) / t)                   # log(erfc(a) / t) + a^2
    s = (2.0 * t - (1.0 + tmin)) / (1.0 - tmin)
    v = np.polynomial.chebyshev.chebvander(s, degree)
    w = np.ones_like(t)
    for _ in range(iterations):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(v * sw[:, None], q * sw, rcond=None)
        e = v @ c - q
        w = w * np.abs(e)
        w /= w.sum()
    sp = np.polynomial.Polynomial([-(1.0 + tmin) / (1.0 - tmin), 2.0 / (1.0 - tmin)])
    prev, cur = np.polynomial.Polynomial([1.0]), sp
    poly = c[0] * prev + c[1] * cur
    for k in range(2, degree + 1):
        prev, cur = cur, 2.0 * sp * cur - prev
        poly = poly + c[k] * cur
    coef32 = poly.coef.astype(np.float32)
    err = np.abs(np.polynomial.polynomial.polyval(t, coef32.astype(np.float64)) - q).max()
    return coef32, err


if __name__ == "__main__":
    coef, err = fit()
    print("max |error| of log erfc:", err)
    for k, c in enumerate(coef):
        print(f"t^{k}: {float(c):.9g}")
