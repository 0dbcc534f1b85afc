"""Coefficients of the 2^f polynomial used by the kernels' FMA-pipe exp2.

2^x = 2^j * 2^f with j = rint(x) and f = x - j in [-1/2, 1/2] (the classic
Cody-Waite split into an exponent-field part and a reduced argument).
2^f is approximated by Q(f), the degree-DEG Chebyshev interpolant of 2^f at
the DEG+1 Chebyshev points of [-1/2, 1/2] (a near-minimax fit), computed in
fp64 with numpy; the fp32-rounded coefficients are checked by evaluating Q
with fp32 Horner steps against fp64 2^f on a dense grid.

Run:  python fit_exp2_poly.py [DEG]   (prints the coefficients, highest first)
"""
import sys

import numpy as np


def fit(deg: int):
    k = np.arange(deg + 1)
    nodes = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * (deg + 1)))
    cheb = np.polynomial.chebyshev.Chebyshev.fit(nodes, np.exp2(nodes), deg, domain=[-0.5, 0.5])
    poly = cheb.convert(kind=np.polynomial.Polynomial, domain=[-1.0, 1.0], window=[-1.0, 1.0])
    return poly.coef[::-1].astype(np.float32)  # highest degree first


def check(c32):
    f = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    p = np.full_like(f, c32[0])
    for c in c32[1:]:
        p = (p.astype(np.float64) * f + c).astype(np.float32)  # one rounding per step, like an fma
    exact = np.exp2(f.astype(np.float64))
    return float(np.max(np.abs(p.astype(np.float64) - exact) / exact))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 5
    c = fit(deg)
    print(f"degree {deg}: max relative error of Q(f) in fp32 = {check(c):.3e}")
    print(", ".join(f"{float(v):.9e}f" for v in c))
