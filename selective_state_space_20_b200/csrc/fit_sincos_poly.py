"""Coefficients of the sin / cos polynomials used by the complex-mode scan's
FMA-pipe rotation.

After the angle is reduced to r in [-pi/4, pi/4] (a quadrant index q =
rint(2 x / pi) and r = x - q pi / 2), sin r = r * P(r^2) and
cos r - 1 = r^2 * G(r^2), with P and G the degree-DEG Chebyshev interpolants
of sin(sqrt(s)) / sqrt(s) and (cos(sqrt(s)) - 1) / s in s = r^2 on
[0, (pi/4)^2] (near-minimax fits, computed in fp64 with numpy).  Fitting
cos r - 1 itself keeps its relative error small as r -> 0 (a fit of cos r
would spread its error over the r^2 coefficient and bias cos r - 1 there).
The fp32-rounded coefficients are checked by evaluating both with fp32
Horner steps against fp64 sin and cos - 1 on a dense grid of r.

Run:  python fit_sincos_poly.py [DEG]   (prints the coefficients, highest first)
"""
import sys

import numpy as np

HI = (np.pi / 4) ** 2


def _fit(fn, deg: int):
    k = np.arange(deg + 1)
    nodes = 0.5 * HI * (1 + np.cos((2 * k + 1) * np.pi / (2 * (deg + 1))))
    cheb = np.polynomial.chebyshev.Chebyshev.fit(nodes, fn(nodes), deg, domain=[0.0, HI])
    poly = cheb.convert(kind=np.polynomial.Polynomial, domain=[-1.0, 1.0], window=[-1.0, 1.0])
    return poly.coef[::-1].astype(np.float32)  # highest degree first


def _sinc(s):
    r = np.sqrt(np.maximum(s, 1e-300))
    return np.where(s > 1e-12, np.sin(r) / r, 1.0 - s / 6)


def _cosm1_over_s(s):
    r = np.sqrt(np.maximum(s, 1e-300))
    return np.where(s > 1e-12, -2.0 * np.sin(r / 2) ** 2 / np.maximum(s, 1e-300), -0.5 + s / 24)


def fit(deg: int):
    return _fit(_sinc, deg), _fit(_cosm1_over_s, deg)


def _horner(c32, s):
    p = np.full_like(s, c32[0])
    for c in c32[1:]:
        p = (p.astype(np.float64) * s + c).astype(np.float32)  # one rounding per step, like an fma
    return p


def check(P, G):
    r = np.linspace(-np.pi / 4, np.pi / 4, 400001).astype(np.float32)
    r = r[r != 0]
    s = (r.astype(np.float64) * r).astype(np.float32)
    sn = (r.astype(np.float64) * _horner(P, s)).astype(np.float32)
    cm1 = (s.astype(np.float64) * _horner(G, s)).astype(np.float32)
    r64 = r.astype(np.float64)
    e_s = np.max(np.abs(sn.astype(np.float64) - np.sin(r64)) / np.abs(np.sin(r64)))
    exact = -2.0 * np.sin(r64 / 2) ** 2  # cos r - 1 without cancellation
    e_c = np.max(np.abs(cm1.astype(np.float64) - exact) / np.abs(exact))
    return float(e_s), float(e_c)


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    P, G = fit(deg)
    e_s, e_c = check(P, G)
    print(f"degree {deg} in r^2: max relative error sin {e_s:.3e}, cos - 1 {e_c:.3e} (fp32)")
    print("P:", ", ".join(f"{float(v):.9e}f" for v in P))
    print("G:", ", ".join(f"{float(v):.9e}f" for v in G))
