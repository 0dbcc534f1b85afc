"""Write ``oracle_tiny.txt``: a small seeded scan problem and the fp64 oracle's
outputs for it.  Calls only ``oracle`` (and numpy for the inputs).

Run from the repository root:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.txt")


def problem():
    rng = np.random.default_rng(2024)
    Bt, Dm, L, N = 2, 3, 19, 5
    f = lambda *s: rng.normal(size=s).astype(np.float32)  # noqa: E731
    return dict(u=f(Bt, Dm, L), delta=(0.5 * f(Bt, Dm, L)).astype(np.float32),
                A=(-rng.uniform(0.5, 5.0, size=(Dm, N))).astype(np.float32),
                B=f(Bt, N, L), C=f(Bt, N, L),
                D=rng.uniform(0.5, 1.5, size=Dm).astype(np.float32),
                z=f(Bt, Dm, L),
                delta_bias=rng.uniform(-5.0, -1.0, size=Dm).astype(np.float32))


def main():
    p = problem()
    out, last = oracle.scan(**p, delta_softplus=True)
    with open(OUT, "w") as fh:
        fh.write("# fp64 oracle outputs for the seeded tiny problem of make_golden.py\n")
        fh.write("# (numpy default_rng(2024); batch 2, dim 3, L 19, N 5; softplus on, gate on)\n")
        for name, arr in (("out", out), ("last_state", last)):
            fh.write(f"{name} {' '.join(str(s) for s in arr.shape)}\n")
            fh.write(" ".join(repr(float(v)) for v in arr.ravel()) + "\n")


if __name__ == "__main__":
    main()
