"""Coefficients of the 2^f polynomial used by the kernels' FMA-pipe exp2.

2^x = 2^j * 2^f with j = rint(x) and f = x - j in [-1/2, 1/2] (the classic
Cody-Waite split into an exponent-field part and a reduced argument).
2^f is approximated by Q(f) = 1 + f P(f), P the degree-DEG Chebyshev
interpolant of (2^f - 1) / f at the DEG+1 Chebyshev points of [-1/2, 1/2]
(a near-minimax fit, computed in fp64 with numpy).  Q(0) = 1 exactly, and
the relative error of Q stays small as f -> 0: a decay exp(delta A) close to
1 (a small step, a slow state) carries no fixed bias that would add up over
the many steps such a state remembers.  The fp32-rounded coefficients are
checked by evaluating Q with fp32 Horner steps against fp64 2^f on a dense
grid.

Run:  python fit_exp2_poly.py [DEG]   (prints P's coefficients, highest first)
"""
import sys

import numpy as np


def _g(f):
    f = np.asarray(f, dtype=np.float64)
    small = np.abs(f) < 1e-6
    safe = np.where(small, 1.0, f)
    ln2 = np.log(2.0)
    return np.where(small, ln2 + f * ln2 ** 2 / 2, np.expm1(safe * ln2) / safe)


def fit(deg: int):
    k = np.arange(deg + 1)
    nodes = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * (deg + 1)))
    cheb = np.polynomial.chebyshev.Chebyshev.fit(nodes, _g(nodes), deg, domain=[-0.5, 0.5])
    poly = cheb.convert(kind=np.polynomial.Polynomial, domain=[-1.0, 1.0], window=[-1.0, 1.0])
    return poly.coef[::-1].astype(np.float32)  # highest degree first


def check(c32):
    f = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    p = np.full_like(f, c32[0])
    for c in c32[1:]:
        p = (p.astype(np.float64) * f + c).astype(np.float32)  # one rounding per step, like an fma
    q = (p.astype(np.float64) * f + 1.0).astype(np.float32)
    exact = np.exp2(f.astype(np.float64))
    return float(np.max(np.abs(q.astype(np.float64) - exact) / exact)), float(q[len(q) // 2])


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    c = fit(deg)
    err, q0 = check(c)
    print(f"degree {deg} (Q = 1 + f P): max relative error of Q(f) in fp32 = {err:.3e}, Q(0) = {q0!r}")
    print(", ".join(f"{float(v):.9e}f" for v in c))
