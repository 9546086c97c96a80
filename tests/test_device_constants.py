"""Host-side checks of the polynomial constants the bf16 GELU-erf kernels use
(mea_math.cuh, GeluErf::nr_parts, nr5_parts and q8), read from the source
text and evaluated in float64 against scipy's scaled complementary error
function.  All are polynomials in t = 1 / (1 + a / 2) (Press et al.,
"Numerical Recipes in C", 2nd ed., section 6.2); the kernels evaluate them in
h = t / 2 with coefficient k times 2^k, which the parser checks and undoes.  nr_parts and nr5_parts
approximate log(erfc(a) / t) + a^2; q8 approximates erfcx(a) / t.  The
claims checked are the fractional error bounds that the kernel comments and
the design notes state, over the range each is used on (a up to 9.6, where
the kernels' tail branch takes over):
  - 1.2e-7 for the degree-9 form (the published bound);
  - 7.7e-6 for the degree-5 refit;
  - 5e-8 for the degree-8 Q.
"""
import os
import re

import numpy as np
import pytest
from scipy.special import erfcx

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "memory_efficient_activation_b200", "csrc", "mea_math.cuh")


# One Horner term of the kernels' h-form (h = t / 2): a coefficient literal,
# optionally times its power of two.
_TERM = r"([-0-9.eE]+)f(?: \* ([0-9.]+)f)?"


def _unscale(terms) -> list[float]:
    """The published coefficients (highest degree first) from the kernel's
    h-form terms: the coefficient of degree k must carry exactly 2^k, so that
    the polynomial in h = t / 2 is the published polynomial in t."""
    deg = len(terms) - 1
    out = []
    for i, (lit, scale) in enumerate(terms):
        assert float(scale or 1) == 2.0 ** (deg - i), (i, lit, scale)
        out.append(float(lit))
    return out


def _horner_coefficients(func: str) -> list[float]:
    """The Horner chain of `func` in GeluErf, highest degree first, in t."""
    text = open(SRC).read()
    start = text.index("struct GeluErf")
    body = text[text.index(f"float {func}(float a, float &h)", start):]
    body = body[:body.index("return")]
    first = re.search(r"float p = " + _TERM + ";", body).groups()
    rest = re.findall(r"p = fmaf\(p, h, " + _TERM + r"\);", body)
    return _unscale([first] + rest)


def _q8_coefficients() -> list[float]:
    """q8's Horner chain, highest degree first, in t."""
    text = open(SRC).read()
    start = text.index("struct GeluErf")
    body = text[text.index("float q8(float h)", start):]
    body = body[:body.index("}")]
    first = re.search(r"float q = " + _TERM + ";", body).groups()
    rest = re.findall(r"fmaf\(q, h, " + _TERM + r"\)", body)
    return _unscale([first] + rest)


def test_h_form_is_the_t_form_bitwise():
    # Horner in h = t / 2 with coefficient k times 2^k: every step is the
    # t-form's step times a power of two, so the float32 results agree bit
    # for bit (checked here with separately rounded multiply and add)
    rng = np.random.default_rng(5)
    t = np.float32(1.0) / (np.float32(1.0) + rng.uniform(0, 4.8, 100001).astype(np.float32))
    h = (t * np.float32(0.5)).astype(np.float32)
    for c in (_horner_coefficients("nr_parts"), _horner_coefficients("nr5_parts"), _q8_coefficients()):
        c32 = np.array(c, dtype=np.float32)
        deg = len(c32) - 1
        pt = np.full_like(t, c32[0])
        ph = np.full_like(t, np.float32(c32[0] * np.float32(2.0 ** deg)))
        for i in range(1, len(c32)):
            pt = (pt * t + c32[i]).astype(np.float32)
            ph = (ph * h + np.float32(c32[i] * np.float32(2.0 ** (deg - i)))).astype(np.float32)
        assert np.array_equal(pt.view(np.int32), ph.view(np.int32))


def _max_fractional_error(coef_high_first, a_max=9.6, points=200001):
    a = np.linspace(0.0, a_max, points)
    t = 1.0 / (1.0 + a / 2.0)
    coef32 = np.array(coef_high_first, dtype=np.float32).astype(np.float64)
    p = np.polyval(coef32, t)
    # erfc(a) = t exp(-a^2 + P(t)) and erfcx(a) = exp(a^2) erfc(a)
    approx_over_exact = t * np.exp(p) / erfcx(a)
    return float(np.max(np.abs(approx_over_exact - 1.0)))


def test_degree9_matches_published_bound():
    c = _horner_coefficients("nr_parts")
    assert len(c) == 10
    assert _max_fractional_error(c) < 1.2e-7


def test_degree5_refit_bound():
    c = _horner_coefficients("nr5_parts")
    assert len(c) == 6
    err = _max_fractional_error(c)
    assert err < 7.7e-6
    # far inside half a bf16 ulp (2^-9 relative), the forward's output precision
    assert err < 2.0 ** -9 / 100


def test_degree5_is_the_fit_script_result():
    import importlib.util
    path = os.path.join(os.path.dirname(SRC), "fit_erfc_bf16.py")
    spec = importlib.util.spec_from_file_location("fit_erfc_bf16", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    coef, err = mod.fit(points=100001, iterations=120)
    kernel = np.array(_horner_coefficients("nr5_parts")[::-1], dtype=np.float32)
    # the refit with fewer points lands on the same fp32 constants to within
    # a few ulps of each (the Lawson iteration converges to the same minimax)
    assert np.allclose(coef, kernel, rtol=1e-4, atol=1e-5), (coef, kernel)
    assert err < 7.7e-6


def test_q8_bound_and_fit():
    c = _q8_coefficients()
    assert len(c) == 9
    a = np.linspace(0.0, 9.6, 200001)
    t = 1.0 / (1.0 + a / 2.0)
    q = np.polyval(np.array(c, dtype=np.float32).astype(np.float64), t)
    # erfc(a) = t e^(-a^2) Q(t)  <=>  Q(t) = erfcx(a) / t
    err = float(np.max(np.abs(q * t / erfcx(a) - 1.0)))
    assert err < 5e-8
    assert abs(q[0] - 1.0) < 1e-7          # a = 0: erfc(0) = 1 = t Q(t) with t = 1
    import importlib.util
    path = os.path.join(os.path.dirname(SRC), "fit_erfc_bf16.py")
    spec = importlib.util.spec_from_file_location("fit_erfc_bf16", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    coef, ferr = mod.fit_q(points=100001, iterations=100)
    assert np.allclose(coef, np.array(c[::-1], dtype=np.float32), rtol=1e-4, atol=1e-6), (coef, c)
    assert ferr < 1e-7                      # a shorter refit, less converged


# ------------------------------------------------ zeros of f' (near-root recompute)

def _root_constants(struct: str) -> dict:
    """kRootD, kRootHi, kRootF2, kRootF3h of `struct` in mea_math.cuh."""
    text = open(SRC).read()
    head = f"struct {struct} {{" if struct != "Swish" else "struct SwishT {"
    body = text[text.index(head):]
    body = body[:body.index("root_scale")]
    out = {}
    for name in ("kRootD", "kRootHi", "kRootF2", "kRootF3h"):
        m = re.search(name + r" = ([-0-9.eE]+)f?;", body)
        out[name] = float(m.group(1))
    return out


@pytest.mark.parametrize("struct,act,alpha", [("Swish", "swish", 1.0), ("GeluErf", "gelu_erf", 1.0),
                                              ("GeluTanh", "gelu_tanh", 1.0)])
def test_root_constants_against_oracle_derivative(struct, act, alpha):
    # The zero of f' and the Taylor coefficients there, checked against the
    # oracle's f' (itself pinned by closed forms, finite differences and
    # torch autograd): f'(v0) vanishes to double rounding, f'' and f'''/2 by
    # central differences of f'.
    import oracle
    c = _root_constants(struct)
    v0 = c["kRootD"]
    assert np.float32(v0) == np.float32(c["kRootHi"])
    d = lambda v: oracle.act_deriv(act, np.asarray(v, dtype=np.float64), alpha)   # noqa: E731
    assert abs(d([v0])[0]) < 1e-15
    h = 1e-4
    fm, f0, fp = d([v0 - h, v0, v0 + h])
    f2 = (fp - fm) / (2 * h)
    f3h = (fp - 2 * f0 + fm) / (h * h) / 2
    assert abs(c["kRootF2"] - f2) <= 1e-6 * abs(f2)
    assert abs(c["kRootF3h"] - f3h) <= 1e-5 * abs(f3h)


def test_swish_root_is_lambert_w():
    # v0 = -(1 + W(1/e)) (the zero of s + v s (1 - s))
    from scipy.special import lambertw
    c = _root_constants("Swish")
    assert abs(c["kRootD"] + 1.0 + float(lambertw(np.exp(-1.0)).real)) < 1e-15
