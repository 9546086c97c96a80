"""Prints the constants of the near-zero recompute of f' in the bf16 backward
kernels (mea_math.cuh, "near the zero of f'").

Swish' (as a function of v = alpha x), GELU-erf' and GELU-tanh' each vanish
at one negative point v0.  Within kRootWin = 2^-10 of it the kernels evaluate
f'(v0 + d) = d (f''(v0) + d f'''(v0) / 2) from d formed in fp64.  For each
activation this script finds v0 to 40 digits (mpmath), prints it to 20
digits (the kernels hold it in fp64) and its fp32 rounding (for the window
test), evaluates f''(v0) and f'''(v0) / 2, and reports the largest relative
error of the two-term polynomial against f' over the window, and |f'| at the
window edge (which bounds the main path's relative error from below).

    python memory_efficient_activation_b200/csrc/near_root_constants.py
"""
import mpmath as mp
import numpy as np

mp.mp.dps = 40
WINDOW = 2.0 ** -10


def _sigmoid(v):
    return 1 / (1 + mp.exp(-v))


FUNCTIONS = {
    # Swish in v = alpha x: x Sigmoid(alpha x) = Swish_1(alpha x) / alpha, whose
    # x-derivative is Swish_1'(alpha x)
    "Swish": lambda v: v * _sigmoid(v),
    "GeluErf": lambda x: x * mp.erfc(-x / mp.sqrt(2)) / 2,
    "GeluTanh": lambda x: x * _sigmoid(2 * mp.sqrt(2 / mp.pi) * (x + mp.mpf("0.044715") * x ** 3)),
}


def constants(name):
    f = FUNCTIONS[name]
    d1 = lambda v: mp.diff(f, v, 1)   # noqa: E731
    v0 = mp.findroot(d1, -1.0)
    hi = np.float32(float(v0))
    f2 = mp.diff(f, v0, 2)
    f3h = mp.diff(f, v0, 3) / 2
    worst = 0.0
    for d in np.linspace(-WINDOW, WINDOW, 201):
        if d == 0.0:
            continue
        exact = d1(v0 + d)
        approx = f2 * d + f3h * d * d
        worst = max(worst, abs(float((approx - exact) / exact)))
    edge = min(abs(float(d1(v0 - WINDOW))), abs(float(d1(v0 + WINDOW))))
    return {"v0": v0, "hi": float(hi), "f2": float(np.float32(float(f2))),
            "f3h": float(np.float32(float(f3h))), "taylor_rel_err": worst, "edge_abs_df": edge}


# The exponent variable t of the kernels' sigmoid (Sigmoid(v) = 1 / (1 + 2^t)):
# t = -v log2 e for Swish (v = alpha x), t = -2u log2 e for GELU-tanh with
# u = sqrt(2/pi) (x + 0.044715 x^3).  The packed bf16 backwards test the
# window on t, which they compute anyway: |t - t0| < kRootWinT, t0 = t(v0),
# kRootWinT = 2^-10 |dt/dv| at v0.
def t_space(name, v0):
    if name == "Swish":
        t0 = -v0 / mp.log(2)
        dt = 1 / mp.log(2)
    elif name == "GeluTanh":
        k1 = 2 * mp.sqrt(2 / mp.pi)
        t0 = -k1 * (v0 + mp.mpf("0.044715") * v0 ** 3) / mp.log(2)
        dt = k1 * (1 + 3 * mp.mpf("0.044715") * v0 ** 2) / mp.log(2)
    else:
        return None
    return float(np.float32(float(t0))), float(np.float32(float(WINDOW * dt)))


def main():
    for name in FUNCTIONS:
        c = constants(name)
        print(f"{name}: v0 = {mp.nstr(c['v0'], 25)}")
        ts = t_space(name, c["v0"])
        if ts:
            print(f"    kRootT = {ts[0]!r}f, kRootWinT = {ts[1]!r}f  (window on t)")
        print(f"    kRootD = {mp.nstr(c['v0'], 20)}, kRootHi = {c['hi']!r}f")
        print(f"    kRootF2 = {c['f2']!r}f, kRootF3h = {c['f3h']!r}f")
        print(f"    two-term relative error over |d| <= 2^-10: {c['taylor_rel_err']:.2e}; "
              f"|f'| at the window edge >= {c['edge_abs_df']:.3e}")


if __name__ == "__main__":
    main()
