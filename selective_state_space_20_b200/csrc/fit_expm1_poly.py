"""Coefficients of the e^x - 1 polynomial (expm1_f in device_math.cuh) that
the fp32-activation paths of every scan kernel, real and complex, use for
their decays.

For x in [-1, 1], e^x - 1 = x + x^2 P(x), P the degree-DEG Chebyshev
interpolant of (e^x - 1 - x) / x^2 on [-1, 1] (a near-minimax fit, computed
in fp64 with numpy).  Writing the result as x plus a correction keeps its
relative error small however close x is to 0, which a value of e^x rounded
near 1 cannot.  The fp32-rounded coefficients are checked by evaluating the
form with fp32 Horner steps against fp64 expm1 on a dense grid.

Run:  python fit_expm1_poly.py [DEG]   (prints the coefficients, highest first)
"""
import sys

import numpy as np


def _g(x):
    x = np.asarray(x, dtype=np.float64)
    small = np.abs(x) < 1e-4
    safe = np.where(small, 1.0, x)
    series = 0.5 + x / 6 + x * x / 24 + x ** 3 / 120
    return np.where(small, series, (np.expm1(safe) - safe) / (safe * safe))


def fit(deg: int):
    k = np.arange(deg + 1)
    nodes = np.cos((2 * k + 1) * np.pi / (2 * (deg + 1)))
    cheb = np.polynomial.chebyshev.Chebyshev.fit(nodes, _g(nodes), deg, domain=[-1.0, 1.0])
    poly = cheb.convert(kind=np.polynomial.Polynomial, domain=[-1.0, 1.0], window=[-1.0, 1.0])
    return poly.coef[::-1].astype(np.float32)  # highest degree first


def check(c32):
    x = np.linspace(-1.0, 1.0, 400001).astype(np.float32)
    x = x[x != 0]
    p = np.full_like(x, c32[0])
    for c in c32[1:]:
        p = (p.astype(np.float64) * x + c).astype(np.float32)  # one rounding per step, like an fma
    x2 = (x.astype(np.float64) * x).astype(np.float32)
    e = (x2.astype(np.float64) * p + x).astype(np.float32)
    exact = np.expm1(x.astype(np.float64))
    return float(np.max(np.abs(e.astype(np.float64) - exact) / np.abs(exact)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 6
    c = fit(deg)
    print(f"degree {deg}: max relative error of x + x^2 P(x) in fp32 = {check(c):.3e}")
    print(", ".join(f"{float(v):.9e}f" for v in c))
