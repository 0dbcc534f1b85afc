"""Planted mistakes: each test copies the oracle's C source, plants one
plausible mistake (a dropped term, a wrong sign or index, a swapped operand),
compiles the copy on the CPU and checks that at least one pin rejects it.
This shows the pins are strong enough to catch such a mistake in the real
oracle.  The real oracle source is never modified.
"""
import os

import pytest

import oracle
import oracle_pins
from oracle import build as obuild

SRC = open(obuild.SRC).read()

# (id, text in the oracle, replacement)
MUTANTS = [
    ("input-term-sign", "h[n] = Abar * h[n] + Bbar_u;\n            y += (double)Cb",
     "h[n] = Abar * h[n] - Bbar_u;\n            y += (double)Cb"),
    ("decay-dropped", "h[n] = Abar * h[n] + Bbar_u;\n            y += (double)Cb",
     "h[n] = h[n] + Bbar_u;\n            y += (double)Cb"),
    ("update-decay-dropped", "h[n] = Abar * h[n] + Bbar_u;\n                y += (double)C[",
     "h[n] = h[n] + Bbar_u;\n                y += (double)C["),
    ("decay-exponent-sign", "exp(delta * (double)Ad[n])", "exp(-delta * (double)Ad[n])"),
    ("A-index", "exp(delta * (double)Ad[n])", "exp(delta * (double)Ad[0])"),
    ("D-skip-dropped", "y += Dd * ut;", "y += 0.0 * ut;"),
    ("gate-dropped", "y *= s6_oracle_silu((double)z[t]);", "y *= 1.0;"),
    ("B-C-swapped", "(double)Bb[n * L + t] * ut", "(double)Cb[n * L + t] * ut"),
    ("B-time-lag", "(double)Bb[n * L + t] * ut", "(double)Bb[n * L + (t > 0 ? t - 1 : 0)] * ut"),
    ("C-reads-old-state", "            h[n] = Abar * h[n] + Bbar_u;\n            y += (double)Cb[n * L + t] * h[n];",
     "            y += (double)Cb[n * L + t] * h[n];\n            h[n] = Abar * h[n] + Bbar_u;"),
    ("bias-after-softplus", "double delta = (double)dr[t] + bias;\n        if (j->softplus)\n            delta = s6_oracle_softplus(delta);",
     "double delta = (double)dr[t];\n        if (j->softplus)\n            delta = s6_oracle_softplus(delta);\n        delta += bias;"),
    ("softplus-dropped", "            delta = s6_oracle_softplus(delta);\n        const double ut",
     "            delta = delta;\n        const double ut"),
    ("Bbar-without-delta", "const double Bbar_u = delta * (double)Bb[n * L + t] * ut;",
     "const double Bbar_u = (double)Bb[n * L + t] * ut;"),
    ("B-batch-index", "const float *Bb = j->B + b * N * L;", "const float *Bb = j->B;"),
    ("h0-ignored", "h[n] = j->h0 ? j->h0[row * N + n] : 0.0;", "h[n] = 0.0;"),
    ("softplus-wrong-branch", "return log1p(exp(x));", "return log(exp(x));"),
    ("silu-sigmoid-only", "return z / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(-z));"),
    ("state-update-C-lag", "y += (double)C[b * N + n] * h[n];", "y += (double)C[b * N + n] * (h[n] - Bbar_u);"),
    ("last-state-off-by-one", "j->last_state[row * N + n] = h[n];", "j->last_state[row * N + n] = h[n] * 0.5;"),
    # causal depthwise convolution
    ("conv-kernel-flipped", "v += (double)wr[k] * (double)xr[s];", "v += (double)wr[width - 1 - k] * (double)xr[s];"),
    ("conv-off-by-one", "const int64_t s = t - (width - 1) + k;", "const int64_t s = t - width + k;"),
    ("conv-centred-padding", "const int64_t s = t - (width - 1) + k;\n                    if (s >= 0)",
     "const int64_t s = t - (width - 1) / 2 + k;\n                    if (s >= 0 && s < seqlen)"),
    ("conv-bias-dropped", "double v = bias ? (double)bias[d] : 0.0;\n                for",
     "double v = 0.0;\n                for"),
    ("conv-silu-dropped", "o[t] = silu ? s6_oracle_silu(v) : v;", "o[t] = v;"),
    ("conv-stride-ignored", "const float *xr = x + b * x_batch_stride + d * seqlen;",
     "const float *xr = x + b * dim * seqlen + d * seqlen;"),
    ("conv-update-no-shift", "st[k] = st[k + 1];", "st[k] = st[k];"),
    ("conv-update-newest-first", "v += (double)wr[k] * (k < S ? st[k] : xt);",
     "v += (double)wr[k] * (k == 0 ? xt : st[k - 1]);"),
    # backward
    ("bwd-ddelta-decay-term-dropped", "ddelta += g[n] * (hp[n] * Abar * (double)Aw[n] + (double)Bw[n * L + t] * ut);",
     "ddelta += g[n] * ((double)Bw[n * L + t] * ut);"),
    ("bwd-carry-without-decay", "g[n] *= Abar;", "g[n] *= 1.0;"),
    ("bwd-dC-uses-previous-state", "j->dC[b * N * L + n * L + t] += dy * h[n];",
     "j->dC[b * N * L + n * L + t] += dy * hp[n];"),
    ("bwd-softplus-derivative-dropped", "const double ddraw = j->softplus ? ddelta * s6_oracle_sigmoid(draw) : ddelta;",
     "const double ddraw = ddelta;"),
    ("bwd-silu-derivative-wrong", "s * (1.0 + zt * (1.0 - s))", "s"),
    ("bwd-dlast-ignored", "g[n] = j->dlast ? j->dlast[row * N + n] : 0.0;", "g[n] = 0.0;"),
    ("bwd-dA-without-delta", "j->dA[d * N + n] += g[n] * hp[n] * Abar * delta;",
     "j->dA[d * N + n] += g[n] * hp[n] * Abar;"),
    ("bwd-du-input-term-dropped", "du += g[n] * delta * (double)Bw[n * L + t];", "du += 0.0;"),
    ("bwd-dB-without-u", "j->dB[b * N * L + n * L + t] += g[n] * delta * ut;",
     "j->dB[b * N * L + n * L + t] += g[n] * delta;"),
    ("bwd-dD-without-gate", "j->dD[d] += dy * ut;", "j->dD[d] += dout[t] * ut;"),
    ("bwd-dbias-without-softplus-derivative", "j->dbias[d] += ddraw;", "j->dbias[d] += ddelta;"),
    ("bwd-dh0-missing-first-decay", "                g[n] *= Abar;\n            }\n            const double ddraw",
     "                if (t > 0)\n                    g[n] *= Abar;\n            }\n            const double ddraw"),
    ("bwd-du-skip-term-dropped", "double du = dy * Dd, ddelta = 0.0;", "double du = 0.0, ddelta = 0.0;"),
    ("bwd-dz-without-skip", "double y = Dd * ut;\n            for (int64_t n = 0; n < N; ++n)\n                y += (double)Cw",
     "double y = 0.0;\n            for (int64_t n = 0; n < N; ++n)\n                y += (double)Cw"),
    # one-token state update
    ("update-gate-dropped", "y *= s6_oracle_silu((double)z[row]);", "y *= 1.0;"),
    ("update-skip-dropped", "y += (D ? (double)D[d] : 0.0) * ut;", "y += 0.0 * ut;"),
    ("update-softplus-dropped", "delta_t = s6_oracle_softplus(delta_t);", "delta_t = delta_t;"),
    # complex mode
    ("cplx-readout-conjugated", "y += creal(Cn * h[n]);", "y += creal(conj(Cn) * h[n]);"),
    ("cplx-readout-magnitude", "y += creal(Cn * h[n]);", "y += cabs(Cn * h[n]);"),
    ("cplx-rotation-reversed", "cexp(delta * An)", "cexp(delta * conj(An))"),
    ("cplx-rotation-dropped", "cexp(delta * An)", "exp(delta * creal(An))"),
    ("cplx-B-imag-dropped", "(double)Bb[(n * L + t) * 2] + I * (double)Bb[(n * L + t) * 2 + 1]",
     "(double)Bb[(n * L + t) * 2]"),
    ("cplx-B-parts-swapped", "(double)Bb[(n * L + t) * 2] + I * (double)Bb[(n * L + t) * 2 + 1]",
     "(double)Bb[(n * L + t) * 2 + 1] + I * (double)Bb[(n * L + t) * 2]"),
    ("cplx-C-time-lag", "(double)Cb[(n * L + t) * 2] + I * (double)Cb[(n * L + t) * 2 + 1]",
     "(double)Cb[(n * L + (t > 0 ? t - 1 : 0)) * 2] + I * (double)Cb[(n * L + (t > 0 ? t - 1 : 0)) * 2 + 1]"),
    ("cplx-h0-imag-dropped", "h[n] = j->h0 ? j->h0[(row * N + n) * 2] + I * j->h0[(row * N + n) * 2 + 1] : 0.0;",
     "h[n] = j->h0 ? j->h0[(row * N + n) * 2] : 0.0;"),
    ("cplx-last-state-conjugated", "j->last_state[(row * N + n) * 2 + 1] = cimag(h[n]);",
     "j->last_state[(row * N + n) * 2 + 1] = -cimag(h[n]);"),
    ("cplx-D-dropped", "y += Dd * (double)u[t];", "y += 0.0 * (double)u[t];"),
    ("cplx-gate-dropped", "y = y * s6_oracle_silu((double)z[t]);", "y = y * 1.0;"),
    ("cplx-A-index", "const double complex An = (double)Ad[2 * n] + I * (double)Ad[2 * n + 1];",
     "const double complex An = (double)Ad[0] + I * (double)Ad[1];"),
]


def test_mutation_patterns_exist():
    for mid, old, _ in MUTANTS:
        assert SRC.count(old) == 1, f"mutant {mid}: pattern must occur exactly once"


# a planted mistake may drive values to inf or nan; numpy's warnings about
# that are part of the expected failure, not a problem of the test
@pytest.mark.filterwarnings("ignore::RuntimeWarning")
@pytest.mark.parametrize("mid,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(mid, old, new, tmp_path):
    src = tmp_path / f"mutant_{mid}.c"
    src.write_text(SRC.replace(old, new, 1))
    so = str(tmp_path / f"libmutant_{mid}.so")
    obuild.compile_source(str(src), so)
    lib = oracle.load_library(so)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, RuntimeError, FloatingPointError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"planted mistake {mid!r} passed every pin"
