"""Coefficients of the log1p polynomial used by the kernels' softplus.

softplus(x) = max(x, 0) + log1p(w),  w = exp(-|x|) in (0, 1].
log1p(w) = w * P(w) with P a degree-DEG polynomial approximating
g(w) = log1p(w) / w on [0, 1] (g(0) = 1).  P is the Chebyshev interpolant of g
at the DEG+1 Chebyshev points of [0, 1] (a near-minimax fit), computed in fp64
with numpy; the fp32-rounded coefficients are then checked by evaluating
w * P(w) with fp32 Horner steps against fp64 log1p on a dense grid.

Run:  python fit_log1p_poly.py [DEG]   (prints the coefficients, highest first)
"""
import sys

import numpy as np


def fit(deg: int):
    k = np.arange(deg + 1)
    nodes = 0.5 + 0.5 * np.cos((2 * k + 1) * np.pi / (2 * (deg + 1)))
    g = np.log1p(nodes) / nodes
    cheb = np.polynomial.chebyshev.Chebyshev.fit(nodes, g, deg, domain=[0.0, 1.0])
    poly = cheb.convert(kind=np.polynomial.Polynomial, domain=[-1.0, 1.0], window=[-1.0, 1.0])
    return poly.coef[::-1].astype(np.float32)  # highest degree first


def check(c32):
    w = np.concatenate([np.linspace(0.0, 1.0, 200001, dtype=np.float64)[1:],
                        np.logspace(-30, 0, 20001)]).astype(np.float32)
    p = np.full_like(w, c32[0])
    for c in c32[1:]:
        p = (p * w + c).astype(np.float32)  # fp32 fma-like Horner step (one rounding)
    approx = (w * p).astype(np.float32).astype(np.float64)
    exact = np.log1p(w.astype(np.float64))
    return float(np.max(np.abs(approx - exact) / exact))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 8
    c = fit(deg)
    print(f"degree {deg}: max relative error of w*P(w) in fp32 = {check(c):.3e}")
    print(", ".join(f"{float(v):.9e}f" for v in c))
