"""Pins for the fp64 oracle: checks against facts fixed by the mathematics,
not by the oracle's own code.

Each ``pin_*`` function takes an oracle library handle (the real one, or a
copy of the oracle compiled with a planted mistake) and raises
``AssertionError`` if the oracle disagrees with the independent fact.  The
expected values are computed here by other means -- a closed form, a
convolution, a library routine, an explicit product formula -- never by the
oracle's recurrence.

Sources of the facts (titles of the pages the method is described on):
* recurrence, ZOH exponent, dB_u = delta*B*u, y + u*D and the swish gate:
  "Mamba SSM concept and implementation in Keras and TensorFlow", sections
  "Going from continuous to discrete spaces", the selective_scan listing and
  MambaBlock.call/ssm;
* convolutional (LTI) form with kernel K_k = C Abar^k Bbar: same page, the
  convolutional-kernel discussion (derived from a zero initial state);
* the cumulative-sum (log-space) form: same page, selective_scan listing.
"""
from __future__ import annotations

import math

import numpy as np
from scipy import signal, special

import oracle

RTOL = 1e-11


def _close(a, b, rtol=RTOL, scale=None, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    s = scale if scale is not None else max(1e-300, float(np.max(np.abs(b))))
    err = float(np.max(np.abs(a - b))) / s if a.size else 0.0
    assert err <= rtol, f"{what}: normwise error {err:.3e} > {rtol:.1e}"


def _f32(x):
    return np.asarray(x, dtype=np.float32)


# ---------------------------------------------------------------- pointwise
def pin_softplus_silu(lib):
    """softplus against numpy's logaddexp(0, x) = ln(e^0 + e^x) and the
    identity softplus(x) - softplus(-x) = x; silu against x * expit(x)."""
    xs = [-40.0, -20.0, -9.21, -3.0, -0.5, 0.0, 1e-8, 0.3, 2.0, 15.0, 40.0]
    for x in xs:
        sp = oracle.softplus(x, lib=lib)
        ref = float(np.logaddexp(0.0, x))
        assert abs(sp - ref) <= 1e-15 * abs(ref), ("softplus", x, sp, ref)
        assert abs((sp - oracle.softplus(-x, lib=lib)) - x) <= 1e-14 * max(1.0, abs(x))
        si = oracle.silu(x, lib=lib)
        ref = x * float(special.expit(x))
        assert abs(si - ref) <= 1e-15 * max(1e-300, abs(ref)) + 1e-300, ("silu", x, si, ref)
    assert abs(oracle.softplus(0.0, lib=lib) - math.log(2.0)) < 1e-16


# ---------------------------------------------------------------- closed forms
def _const_problem(L, N, softplus, raw, bias, u, Bv, Cv, Av, Dv, zv=None):
    shape = (1, 1, L)
    ins = dict(
        u=np.full(shape, u, np.float32),
        delta=np.full(shape, raw, np.float32),
        A=_f32(np.asarray(Av).reshape(1, N)),
        B=np.repeat(_f32(np.asarray(Bv).reshape(1, N, 1)), L, axis=2),
        C=np.repeat(_f32(np.asarray(Cv).reshape(1, N, 1)), L, axis=2),
        D=np.full((1,), Dv, np.float32),
        z=None if zv is None else np.full(shape, zv, np.float32),
        delta_bias=np.full((1,), bias, np.float32),
        delta_softplus=softplus,
    )
    return ins


def pin_geometric_series(lib):
    """Constant inputs: h_t = b (1 - a^{t+1}) / (1 - a), a = e^{delta A},
    b = delta B u; y_t = sum_n C_n h_t[n] + D u, times silu(z)."""
    L, N = 300, 5
    raw, bias = np.float32(-0.75), np.float32(-2.5)
    delta = float(np.logaddexp(0.0, float(raw) + float(bias)))
    u = np.float32(0.8125)
    Av = _f32([-1.0, -2.0, -0.37, -5.5, -0.01])
    Bv = _f32([0.5, -1.25, 2.0, 0.75, 1.5])
    Cv = _f32([1.5, 0.25, -0.75, 1.0, -2.0])
    Dv = np.float32(0.625)
    zv = np.float32(-0.4375)
    ins = _const_problem(L, N, True, raw, bias, u, Bv, Cv, Av, Dv, zv)
    out, last = oracle.scan(**ins, lib=lib)
    t = np.arange(L, dtype=np.float64)[:, None]
    a = np.exp(delta * Av.astype(np.float64))[None, :]
    b = (delta * Bv.astype(np.float64) * float(u))[None, :]
    h = b * (1.0 - a ** (t + 1.0)) / (1.0 - a)
    y = h @ Cv.astype(np.float64) + float(Dv) * float(u)
    gate = float(zv) * float(special.expit(float(zv)))
    _close(out[0, 0], y * gate, what="geometric series out")
    _close(last[0, 0], h[-1], what="geometric series last_state")


def pin_lti_convolution(lib):
    """delta, B, C constant in time, u random: y = K * u + D u with
    K_k = sum_n C_n Abar_n^k Bbar_n (Bbar_n = delta B_n), as an explicit
    causal convolution (numpy.convolve); no gate."""
    rng = np.random.default_rng(7)
    L, N = 257, 6
    raw, bias = np.float32(0.3), np.float32(-3.0)
    delta = float(np.logaddexp(0.0, float(raw) + float(bias)))
    Av = _f32(-rng.uniform(0.2, 6.0, N))
    Bv = _f32(rng.normal(size=N))
    Cv = _f32(rng.normal(size=N))
    Dv = np.float32(1.375)
    u = _f32(rng.normal(size=L))
    ins = _const_problem(L, N, True, raw, bias, 0.0, Bv, Cv, Av, Dv)
    ins["u"] = u.reshape(1, 1, L)
    out, _ = oracle.scan(**ins, lib=lib)
    k = np.arange(L, dtype=np.float64)[:, None]
    Abar = np.exp(delta * Av.astype(np.float64))[None, :]
    K = (Abar ** k) @ (Cv.astype(np.float64) * delta * Bv.astype(np.float64))
    y = np.convolve(K, u.astype(np.float64))[:L] + float(Dv) * u.astype(np.float64)
    _close(out[0, 0], y, rtol=1e-10, what="LTI convolution")


def pin_first_order_iir(lib):
    """N = 1 with constant delta and B: h is a first-order recursive filter,
    h_t = a h_{t-1} + delta B u_t, which scipy.signal.lfilter computes."""
    rng = np.random.default_rng(11)
    L = 500
    raw, bias = np.float32(0.0), np.float32(-1.0)
    delta = float(np.logaddexp(0.0, -1.0))
    Av, Bv, Cv, Dv = _f32([-0.7]), _f32([1.75]), _f32([-0.5]), np.float32(0.25)
    u = _f32(rng.normal(size=L))
    ins = _const_problem(L, 1, True, raw, bias, 0.0, Bv, Cv, Av, Dv)
    ins["u"] = u.reshape(1, 1, L)
    out, last = oracle.scan(**ins, lib=lib)
    a = math.exp(delta * float(Av[0]))
    h = signal.lfilter([delta * float(Bv[0])], [1.0, -a], u.astype(np.float64))
    _close(out[0, 0], float(Cv[0]) * h + float(Dv) * u, rtol=1e-10, what="lfilter")
    _close(last[0, 0, 0], h[-1], rtol=1e-10, what="lfilter last_state")


def pin_zero_step_keeps_state(lib):
    """delta = 0 (softplus off, zero raw delta and bias): Abar = 1 and
    Bbar = 0, so the state never moves from h0 and y_t = C_t . h0 + D u_t."""
    rng = np.random.default_rng(3)
    Bt, Dm, L, N = 2, 3, 40, 4
    u = _f32(rng.normal(size=(Bt, Dm, L)))
    B = _f32(rng.normal(size=(Bt, N, L)))
    C = _f32(rng.normal(size=(Bt, N, L)))
    A = _f32(-rng.uniform(0.5, 3, size=(Dm, N)))
    D = _f32(rng.normal(size=Dm))
    h0 = rng.normal(size=(Bt, Dm, N))
    out, last = oracle.scan(u, np.zeros_like(u), A, B, C, D=D, z=None,
                            delta_bias=np.zeros(Dm, np.float32),
                            delta_softplus=False, h0=h0, lib=lib)
    y = np.einsum("bdn,bnl->bdl", h0, C.astype(np.float64)) + D[None, :, None].astype(np.float64) * u
    _close(out, y, what="delta=0 readout")
    assert np.array_equal(last, h0), "delta=0 must leave the state unchanged"


def pin_memoryless_limit(lib):
    """Large delta with A < 0: Abar underflows (e^{-60}), so h_t = delta B_t u_t
    and y_t = delta u_t (B_t . C_t) + D u_t."""
    rng = np.random.default_rng(5)
    L, N = 64, 3
    u = _f32(rng.normal(size=(1, 1, L)))
    B = _f32(rng.normal(size=(1, N, L)))
    C = _f32(rng.normal(size=(1, N, L)))
    A = _f32([[-2.0, -3.0, -4.0]])
    raw = np.full((1, 1, L), 30.0, np.float32)
    out, _ = oracle.scan(u, raw, A, B, C, D=_f32([0.5]), z=None,
                         delta_bias=_f32([0.0]), delta_softplus=True, lib=lib)
    delta = float(np.logaddexp(0.0, 30.0))
    u64 = u[0, 0].astype(np.float64)
    y = delta * u64 * np.sum(B[0].astype(np.float64) * C[0], axis=0) + 0.5 * u64
    _close(out[0, 0], y, rtol=1e-12, what="memoryless limit")


# ---------------------------------------------------------------- brute force
def _rand_problem(rng, Bt, Dm, L, N, gate=True, small_delta=False):
    u = _f32(rng.normal(size=(Bt, Dm, L)))
    delta = _f32(0.5 * rng.normal(size=(Bt, Dm, L)))
    A = _f32(-rng.uniform(0.3, 4.0, size=(Dm, N)))
    B = _f32(rng.normal(size=(Bt, N, L)))
    C = _f32(rng.normal(size=(Bt, N, L)))
    D = _f32(rng.uniform(0.5, 1.5, size=Dm))
    z = _f32(rng.normal(size=(Bt, Dm, L))) if gate else None
    lo, hi = (-6.0, -4.0) if small_delta else (-4.0, 0.0)
    bias = _f32(rng.uniform(lo, hi, size=Dm))
    return dict(u=u, delta=delta, A=A, B=B, C=C, D=D, z=z, delta_bias=bias)


def pin_brute_force_products(lib):
    """Tiny shapes, everything time-varying: the state written as the sum of
    past inputs weighted by explicit products of the discretised decays,
    h_t = sum_{s<=t} (prod_{k=s+1..t} Abar_k) Bbar_s u_s, in pure Python."""
    rng = np.random.default_rng(1234)
    Bt, Dm, L, N = 2, 3, 13, 4
    p = _rand_problem(rng, Bt, Dm, L, N)
    out, last = oracle.scan(**p, delta_softplus=True, lib=lib)
    for b in range(Bt):
        for d in range(Dm):
            dl = [float(np.logaddexp(0.0, float(p["delta"][b, d, t]) + float(p["delta_bias"][d])))
                  for t in range(L)]
            for t in range(L):
                y = 0.0
                hT = []
                for n in range(N):
                    acc = 0.0
                    for s in range(t + 1):
                        w = 1.0
                        for k in range(s + 1, t + 1):
                            w *= math.exp(dl[k] * float(p["A"][d, n]))
                        acc += w * dl[s] * float(p["B"][b, n, s]) * float(p["u"][b, d, s])
                    hT.append(acc)
                    y += float(p["C"][b, n, t]) * acc
                y += float(p["D"][d]) * float(p["u"][b, d, t])
                zt = float(p["z"][b, d, t])
                y *= zt * float(special.expit(zt))
                assert abs(out[b, d, t] - y) <= 1e-11 * max(1.0, abs(y)), (b, d, t, out[b, d, t], y)
                if t == L - 1:
                    _close(last[b, d], hT, rtol=1e-11, what="brute-force last_state")


def pin_cumsum_form(lib):
    """The cumulative-sum form of the scan: with P_t = sum_{k<=t} delta_k A,
    h_t = e^{P_t} sum_{s<=t} e^{-P_s} Bbar_s u_s (vectorised with numpy
    cumsum/einsum; valid while e^{-P} stays finite, so short L, small delta)."""
    rng = np.random.default_rng(99)
    Bt, Dm, L, N = 2, 4, 48, 5
    p = _rand_problem(rng, Bt, Dm, L, N, small_delta=True)
    out, last = oracle.scan(**p, delta_softplus=True, lib=lib)
    dl = np.logaddexp(0.0, p["delta"].astype(np.float64) + p["delta_bias"][None, :, None])
    dA = np.einsum("bdl,dn->bdln", dl, p["A"].astype(np.float64))
    P = np.cumsum(dA, axis=2)
    dBu = np.einsum("bdl,bnl,bdl->bdln", dl, p["B"].astype(np.float64), p["u"].astype(np.float64))
    h = np.exp(P) * np.cumsum(np.exp(-P) * dBu, axis=2)
    y = np.einsum("bdln,bnl->bdl", h, p["C"].astype(np.float64))
    y = y + p["D"][None, :, None].astype(np.float64) * p["u"]
    z = p["z"].astype(np.float64)
    y = y * z * special.expit(z)
    _close(out, y, rtol=1e-10, what="cumsum form")
    _close(last, h[:, :, -1, :], rtol=1e-10, what="cumsum form last_state")


# ---------------------------------------------------------------- invariants
def pin_chunk_split(lib):
    """Scanning [0, L1) then [L1, L) from the carried last_state equals one
    scan over [0, L), bit for bit."""
    rng = np.random.default_rng(21)
    Bt, Dm, L, N = 2, 5, 97, 16
    p = _rand_problem(rng, Bt, Dm, L, N)
    full, last = oracle.scan(**p, delta_softplus=True, lib=lib)
    for L1 in (1, 31, 64, 96):
        def part(sl):
            q = dict(p)
            for k in ("u", "delta", "z", "B", "C"):
                q[k] = np.ascontiguousarray(p[k][:, :, sl])
            return q
        o1, s1 = oracle.scan(**part(slice(0, L1)), delta_softplus=True, lib=lib)
        o2, s2 = oracle.scan(**part(slice(L1, L)), delta_softplus=True, h0=s1, lib=lib)
        assert np.array_equal(np.concatenate([o1, o2], axis=2), full), f"split at {L1}"
        assert np.array_equal(s2, last), f"split at {L1}: last_state"


def pin_steps_equal_scan(lib):
    """L calls of the one-token state update reproduce the scan exactly."""
    rng = np.random.default_rng(22)
    Bt, Dm, L, N = 3, 4, 20, 16
    p = _rand_problem(rng, Bt, Dm, L, N)
    full, last = oracle.scan(**p, delta_softplus=True, lib=lib)
    state = np.zeros((Bt, Dm, N))
    for t in range(L):
        o, state = oracle.state_update(state, p["u"][:, :, t], p["delta"][:, :, t],
                                       p["A"], p["B"][:, :, t], p["C"][:, :, t],
                                       D=p["D"], z=p["z"][:, :, t],
                                       delta_bias=p["delta_bias"], delta_softplus=True,
                                       lib=lib)
        assert np.array_equal(o, full[:, :, t]), f"step {t}"
    assert np.array_equal(state, last)


def pin_causality(lib):
    """Changing u at time t0 leaves every output before t0 bit-identical and
    changes the output at t0."""
    rng = np.random.default_rng(23)
    p = _rand_problem(rng, 1, 2, 50, 8)
    o1, _ = oracle.scan(**p, delta_softplus=True, lib=lib)
    q = dict(p)
    q["u"] = p["u"].copy()
    q["u"][:, :, 30] += 1.0
    o2, _ = oracle.scan(**q, delta_softplus=True, lib=lib)
    assert np.array_equal(o1[:, :, :30], o2[:, :, :30])
    assert np.all(o1[:, :, 30] != o2[:, :, 30])


def pin_linearity(lib):
    """With delta fixed and no gate, y is linear in u (and affine in B with
    the D u term counted once): y(u1 + u2) = y(u1) + y(u2)."""
    rng = np.random.default_rng(24)
    p = _rand_problem(rng, 2, 3, 40, 6, gate=False)
    u1 = _f32(rng.normal(size=p["u"].shape))
    u2 = _f32(rng.normal(size=p["u"].shape))
    y = {}
    for name, uu in (("1", u1), ("2", u2), ("12", _f32(u1.astype(np.float64) + u2))):
        q = dict(p)
        q["u"] = uu
        y[name], _ = oracle.scan(**q, delta_softplus=True, lib=lib)
    # u1 + u2 is exactly representable only approximately in fp32: compare
    # against the fp32-rounded sum's own linear combination bound.
    _close(y["12"], y["1"] + y["2"], rtol=1e-6, what="linearity in u")
    B1 = _f32(rng.normal(size=p["B"].shape))
    q1, q2 = dict(p), dict(p)
    q1["B"], q2["B"] = B1, _f32(-B1)
    ya, _ = oracle.scan(**q1, delta_softplus=True, lib=lib)
    yb, _ = oracle.scan(**q2, delta_softplus=True, lib=lib)
    Du = p["D"][None, :, None].astype(np.float64) * p["u"]
    _close(ya + yb, 2 * Du, rtol=1e-12, scale=float(np.max(np.abs(ya))), what="odd in B")


def pin_shared_bc_and_independence(lib):
    """B and C belong to a batch row and are shared by its channels; rows are
    independent.  Changing B of batch 1 leaves batch 0 bit-identical, and
    permuting channels (with A, D, bias) permutes the outputs."""
    rng = np.random.default_rng(25)
    p = _rand_problem(rng, 2, 5, 30, 4)
    o, s = oracle.scan(**p, delta_softplus=True, lib=lib)
    q = dict(p)
    q["B"] = p["B"].copy()
    q["B"][1] *= -2.0
    o2, _ = oracle.scan(**q, delta_softplus=True, lib=lib)
    assert np.array_equal(o[0], o2[0]) and not np.array_equal(o[1], o2[1])
    perm = np.array([3, 0, 4, 1, 2])
    r = dict(p)
    for k in ("u", "delta", "z"):
        r[k] = np.ascontiguousarray(p[k][:, perm])
    r["A"] = np.ascontiguousarray(p["A"][perm])
    r["D"] = np.ascontiguousarray(p["D"][perm])
    r["delta_bias"] = np.ascontiguousarray(p["delta_bias"][perm])
    o3, s3 = oracle.scan(**r, delta_softplus=True, lib=lib)
    assert np.array_equal(o3, o[:, perm]) and np.array_equal(s3, s[:, perm])


def pin_zero_b_or_c(lib):
    """B = 0 or C = 0 removes the state's contribution: y = D u silu(z)."""
    rng = np.random.default_rng(26)
    p = _rand_problem(rng, 1, 3, 25, 4)
    z = p["z"].astype(np.float64)
    y = p["D"][None, :, None] * p["u"].astype(np.float64) * z * special.expit(z)
    for key in ("B", "C"):
        q = dict(p)
        q[key] = np.zeros_like(p[key])
        o, _ = oracle.scan(**q, delta_softplus=True, lib=lib)
        _close(o, y, rtol=1e-15, what=f"{key} = 0")


def pin_gate_and_softplus_flags(lib):
    """z = None means no gate; softplus off means delta = raw + bias is used
    as is (checked on one step against the closed form of a single update)."""
    rng = np.random.default_rng(27)
    p = _rand_problem(rng, 1, 2, 1, 3)
    q = dict(p)
    q["z"] = None
    o_nogate, _ = oracle.scan(**q, delta_softplus=True, lib=lib)
    o_gate, _ = oracle.scan(**p, delta_softplus=True, lib=lib)
    z = p["z"].astype(np.float64)
    _close(o_gate, o_nogate * z * special.expit(z), rtol=1e-15, what="gate")
    # softplus off, one step from h = 0: h = (raw + bias) B u, y = C.h + D u
    raw = np.abs(p["delta"]).astype(np.float32)
    q["delta"] = raw
    o, s = oracle.scan(**q, delta_softplus=False, lib=lib)
    dl = raw[0, :, 0].astype(np.float64) + p["delta_bias"]
    h = dl[:, None] * p["B"][0, :, 0].astype(np.float64)[None, :] * p["u"][0, :, 0].astype(np.float64)[:, None]
    y = h @ p["C"][0, :, 0].astype(np.float64) + p["D"].astype(np.float64) * p["u"][0, :, 0]
    _close(s[0], h, rtol=1e-15, what="softplus off state")
    _close(o[0, :, 0], y, rtol=1e-14, what="softplus off out")


# ------------------------------------------------------------ convolution
# The causal depthwise Conv1D (+ bias, + swish) of MambaBlock on the same
# page: channels-first, one group per channel, causal padding.

def _conv_inputs(rng, batch, dim, L, K):
    x = rng.standard_normal((batch, dim, L)).astype(np.float32)
    w = rng.standard_normal((dim, K)).astype(np.float32)
    bias = rng.standard_normal(dim).astype(np.float32)
    return x, w, bias


def pin_conv_numpy(lib):
    """silu off: every row is numpy.convolve of the row with the reversed
    kernel (causal padding = the first L terms of the full convolution) plus
    the bias."""
    rng = np.random.default_rng(101)
    for K in (1, 2, 3, 4):
        x, w, bias = _conv_inputs(rng, 2, 5, 37, K)
        got = oracle.conv1d(x, w, bias, silu=False, lib=lib)
        exp = np.empty_like(got)
        for b in range(2):
            for d in range(5):
                full = np.convolve(x[b, d].astype(np.float64), w[d, ::-1].astype(np.float64))
                exp[b, d] = full[:37] + float(bias[d])
        _close(got, exp, rtol=1e-14, what=f"conv vs numpy K={K}")


def pin_conv_impulse(lib):
    """A unit impulse at t0 gives back the kernel, newest tap first, on top of
    the bias, and only the bias elsewhere."""
    K, L, t0 = 4, 12, 5
    x = np.zeros((1, 3, L), dtype=np.float32)
    x[:, :, t0] = 1.0
    w = (np.arange(12, dtype=np.float32).reshape(3, 4) + 1.0) * 0.25
    bias = np.array([0.5, -1.0, 2.0], dtype=np.float32)
    got = oracle.conv1d(x, w, bias, silu=False, lib=lib)
    exp = np.repeat(bias.astype(np.float64)[:, None], L, axis=1)[None]
    for d in range(3):
        for j in range(K):
            exp[0, d, t0 + j] += w[d, K - 1 - j]
    assert np.array_equal(got, exp), "impulse response"


def pin_conv_silu(lib):
    """silu on: z * expit(z) of the silu-off result (scipy)."""
    rng = np.random.default_rng(102)
    x, w, bias = _conv_inputs(rng, 2, 4, 29, 4)
    v = oracle.conv1d(x, w, bias, silu=False, lib=lib)
    got = oracle.conv1d(x, w, bias, silu=True, lib=lib)
    _close(got, v * special.expit(v), rtol=1e-14, what="conv silu")


def pin_conv_wide_input(lib):
    """x as the first dim channel rows of a (batch, 2 dim, L) tensor (the x
    half of the input projection) gives the same as a contiguous x."""
    rng = np.random.default_rng(103)
    xz, w, bias = _conv_inputs(rng, 3, 8, 21, 3)
    w, bias = w[:4], bias[:4]
    got = oracle.conv1d(xz, w, bias, silu=True, dim=4, lib=lib)
    ref = oracle.conv1d(np.ascontiguousarray(xz[:, :4]), w, bias, silu=True, lib=lib)
    assert np.array_equal(got, ref), "wide input"
    # and the other rows do matter when they are the ones selected
    other = oracle.conv1d(np.ascontiguousarray(xz[:, 4:]), w, bias, silu=True, lib=lib)
    assert not np.allclose(got, other)


def pin_conv_update_stream(lib):
    """One-token updates from a zero state reproduce the whole-sequence
    convolution bit for bit (same summation order)."""
    rng = np.random.default_rng(104)
    for K in (1, 2, 4):
        x, w, bias = _conv_inputs(rng, 2, 3, 15, K)
        ref = oracle.conv1d(x, w, bias, silu=True, lib=lib)
        st = np.zeros((2, 3, K - 1))
        for t in range(15):
            o, st = oracle.conv1d_update(st, x[:, :, t], w, bias, silu=True, lib=lib)
            assert np.array_equal(o, ref[:, :, t]), f"step {t}, K={K}"
        if K > 1:
            assert np.array_equal(st, x[:, :, 15 - (K - 1):].astype(np.float64)), "final state"


def pin_conv_causality(lib):
    """Changing x at t* changes no output before t* and the output at t*."""
    rng = np.random.default_rng(105)
    x, w, bias = _conv_inputs(rng, 1, 4, 20, 4)
    a = oracle.conv1d(x, w, bias, silu=True, lib=lib)
    x2 = x.copy()
    x2[:, :, 11] += 3.0
    b = oracle.conv1d(x2, w, bias, silu=True, lib=lib)
    assert np.array_equal(a[:, :, :11], b[:, :, :11])
    assert np.all(a[:, :, 11] != b[:, :, 11])


# ------------------------------------------------------------ backward
# Gradients of the scan: against torch.autograd on an fp64 forward written
# here with torch tensor ops (a different program from the oracle's loop),
# and against central finite differences of the oracle's own (pinned)
# forward.

def _bwd_problem(seed, batch=2, dim=3, L=9, N=4, gate=True):
    rng = np.random.default_rng(seed)
    f = lambda *s, scale=1.0: (rng.standard_normal(s) * scale).astype(np.float32)  # noqa: E731
    p = dict(u=f(batch, dim, L), delta=f(batch, dim, L, scale=0.5),
             A=-np.abs(f(dim, N)) - 0.2, B=f(batch, N, L), C=f(batch, N, L),
             D=f(dim), z=f(batch, dim, L) if gate else None, delta_bias=f(dim, scale=0.3))
    h0 = f(batch, dim, N).astype(np.float64)
    dout = f(batch, dim, L).astype(np.float64)
    dlast = f(batch, dim, N).astype(np.float64)
    return p, h0, dout, dlast


def _torch_scan(u, delta, A, B, C, D, z, bias, h0, softplus=True):
    import torch
    dl = delta + bias[None, :, None]
    if softplus:
        dl = torch.logaddexp(dl, torch.zeros_like(dl))
    h, ys = h0, []
    for t in range(u.shape[-1]):
        h = torch.exp(dl[..., t, None] * A) * h + dl[..., t, None] * B[:, None, :, t] * u[..., t, None]
        y = (h * C[:, None, :, t]).sum(-1) + D * u[..., t]
        if z is not None:
            y = y * z[..., t] * torch.sigmoid(z[..., t])
        ys.append(y)
    return torch.stack(ys, -1), h


def pin_bwd_autograd(lib):
    """Every gradient equals torch.autograd's through an fp64 forward written
    with torch ops, with and without the gate and softplus."""
    import torch
    for seed, gate, sp in ((301, True, True), (302, False, True), (303, True, False)):
        p, h0, dout, dlast = _bwd_problem(seed, gate=gate)
        if not sp:
            p["delta"] = np.abs(p["delta"])
            p["delta_bias"] = np.abs(p["delta_bias"])
        names = ["u", "delta", "A", "B", "C", "D", "z", "delta_bias"]
        t = {k: (None if p[k] is None else torch.tensor(p[k], dtype=torch.float64, requires_grad=True))
             for k in names}
        th0 = torch.tensor(h0, requires_grad=True)
        out, last = _torch_scan(t["u"], t["delta"], t["A"], t["B"], t["C"], t["D"], t["z"],
                                t["delta_bias"], th0, softplus=sp)
        loss = (out * torch.tensor(dout)).sum() + (last * torch.tensor(dlast)).sum()
        wrt = [t[k] for k in names if t[k] is not None] + [th0]
        grads = dict(zip([k for k in names if t[k] is not None] + ["h0"], torch.autograd.grad(loss, wrt)))
        r = oracle.scan_bwd(dout, **p, delta_softplus=sp, h0=h0, dlast=dlast, lib=lib)
        pairs = [("du", "u"), ("ddelta", "delta"), ("dA", "A"), ("dB", "B"), ("dC", "C"),
                 ("dD", "D"), ("ddelta_bias", "delta_bias"), ("dh0", "h0")] + ([("dz", "z")] if gate else [])
        for mine, theirs in pairs:
            _close(r[mine], grads[theirs].numpy(), rtol=1e-11, what=f"{mine} vs autograd (seed {seed})")


def pin_bwd_finite_differences(lib):
    """Central differences of the oracle's forward loss at a few entries of
    every input; the perturbed values are fp32 numbers, and the divisor is
    their exact difference."""
    p, h0, dout, dlast = _bwd_problem(304, L=6, N=3)
    r = oracle.scan_bwd(dout, **p, h0=h0, dlast=dlast, lib=lib)

    def loss(q, hh):
        o, s = oracle.scan(**q, h0=hh, lib=lib)
        return float(np.sum(o * dout) + np.sum(s * dlast))
    rng = np.random.default_rng(305)
    for name, gname in (("u", "du"), ("delta", "ddelta"), ("A", "dA"), ("B", "dB"), ("C", "dC"),
                        ("D", "dD"), ("z", "dz"), ("delta_bias", "ddelta_bias"), ("h0", "dh0")):
        base = h0 if name == "h0" else p[name]
        for _ in range(3):
            idx = tuple(int(rng.integers(0, n)) for n in base.shape)
            x = float(base[idx])
            step = 1e-3 * max(abs(x), 1.0)
            vals = []
            for sgn in (1, -1):
                q = {k: (None if v is None else v.copy()) for k, v in p.items()}
                hh = h0.copy()
                tgt = hh if name == "h0" else q[name]
                tgt[idx] = np.float32(x + sgn * step)
                vals.append((loss(q, hh), float(np.float32(x + sgn * step))))
            fd = (vals[0][0] - vals[1][0]) / (vals[0][1] - vals[1][1])
            g = float(r[gname][idx])
            assert abs(fd - g) <= 2e-5 * max(1.0, abs(g)), f"{gname}{idx}: fd {fd} vs {g}"


# ---------------------------------------------------------------- complex mode
def _cplx32(rng, shape, scale=1.0):
    """Complex values whose real and imaginary parts are fp32-exact."""
    re = _f32(rng.normal(size=shape) * scale).astype(np.float64)
    im = _f32(rng.normal(size=shape) * scale).astype(np.float64)
    return re + 1j * im


def _cplx_problem(rng, Bt, Dm, L, N, gate=True):
    A = (-_f32(rng.uniform(0.1, 2.0, (Dm, N))).astype(np.float64)
         + 1j * _f32(rng.uniform(-6.0, 6.0, (Dm, N))).astype(np.float64))
    return dict(u=_f32(rng.normal(size=(Bt, Dm, L))), delta=_f32(0.5 * rng.normal(size=(Bt, Dm, L))),
                A=A, B=_cplx32(rng, (Bt, N, L)), C=_cplx32(rng, (Bt, N, L)),
                D=_f32(rng.uniform(0.5, 1.5, Dm)), z=_f32(rng.normal(size=(Bt, Dm, L))) if gate else None,
                delta_bias=_f32(rng.uniform(-3.0, -1.0, Dm)))


def pin_complex_real_case(lib):
    """Imaginary parts zero: the complex mode is the real scan (the real
    oracle is pinned on its own), outputs and states bit for bit."""
    rng = np.random.default_rng(41)
    p = _rand_problem(rng, 2, 3, 37, 5)
    pc = dict(p, A=p["A"].astype(np.complex128), B=p["B"].astype(np.complex128),
              C=p["C"].astype(np.complex128))
    o_r, s_r = oracle.scan(**p, lib=lib)
    o_c, s_c = oracle.scan_complex(**pc, lib=lib)
    assert np.array_equal(o_r, o_c), "complex mode with real inputs differs from the real scan"
    assert np.array_equal(s_r, s_c.real) and not np.any(s_c.imag)


def pin_complex_geometric_series(lib):
    """Constant inputs: h_t = b (1 - a^{t+1}) / (1 - a) over the complex
    numbers, a = e^{delta A}, b = delta B u; y_t = Re(sum_n C_n h_t[n]) + D u,
    times silu(z)."""
    rng = np.random.default_rng(42)
    L, N = 200, 4
    raw, bias = np.float32(-0.5), np.float32(-2.0)
    delta = float(np.logaddexp(0.0, float(raw) + float(bias)))
    A = -_f32([0.5, 0.05, 1.3, 0.2]).astype(np.float64) + 1j * _f32([3.0, -1.5, 0.25, 9.0]).astype(np.float64)
    Bv, Cv = _cplx32(rng, N), _cplx32(rng, N)
    u, Dv, zv = np.float32(0.75), np.float32(0.5), np.float32(0.8125)
    ins = dict(u=np.full((1, 1, L), u, np.float32), delta=np.full((1, 1, L), raw, np.float32),
               A=A.reshape(1, N), B=np.repeat(Bv.reshape(1, N, 1), L, axis=2),
               C=np.repeat(Cv.reshape(1, N, 1), L, axis=2), D=np.full((1,), Dv, np.float32),
               z=np.full((1, 1, L), zv, np.float32), delta_bias=np.full((1,), bias, np.float32))
    out, last = oracle.scan_complex(**ins, lib=lib)
    t = np.arange(L, dtype=np.float64)[:, None]
    a = np.exp(delta * A)[None, :]
    b = (delta * Bv * float(u))[None, :]
    h = b * (1.0 - a ** (t + 1.0)) / (1.0 - a)
    y = (h @ Cv).real + float(Dv) * float(u)
    gate = float(zv) * float(special.expit(float(zv)))
    _close(out[0, 0], y * gate, what="complex geometric series out")
    _close(np.abs(last[0, 0] - h[-1]), np.zeros(N), scale=float(np.max(np.abs(h[-1]))),
           what="complex geometric series last_state")


def pin_complex_lti_convolution(lib):
    """delta, B, C constant in time: y = K * u + D u with the real kernel
    K_k = Re(sum_n C_n Abar_n^k delta B_n) (numpy.convolve)."""
    rng = np.random.default_rng(43)
    L, N = 181, 5
    raw, bias = np.float32(0.2), np.float32(-2.5)
    delta = float(np.logaddexp(0.0, float(raw) + float(bias)))
    A = (-_f32(rng.uniform(0.2, 3.0, N)).astype(np.float64)
         + 1j * _f32(rng.uniform(-8.0, 8.0, N)).astype(np.float64))
    Bv, Cv = _cplx32(rng, N), _cplx32(rng, N)
    u = _f32(rng.normal(size=L))
    Dv = np.float32(1.25)
    ins = dict(u=u.reshape(1, 1, L), delta=np.full((1, 1, L), raw, np.float32), A=A.reshape(1, N),
               B=np.repeat(Bv.reshape(1, N, 1), L, axis=2), C=np.repeat(Cv.reshape(1, N, 1), L, axis=2),
               D=np.full((1,), Dv, np.float32), z=None, delta_bias=np.full((1,), bias, np.float32))
    out, _ = oracle.scan_complex(**ins, lib=lib)
    k = np.arange(L, dtype=np.float64)[:, None]
    K = ((np.exp(delta * A)[None, :] ** k) @ (Cv * delta * Bv)).real
    y = np.convolve(K, u.astype(np.float64))[:L] + float(Dv) * u.astype(np.float64)
    _close(out[0, 0], y, rtol=1e-10, what="complex LTI convolution")


def pin_complex_iir(lib):
    """One state, delta constant, B and u varying: the state is the output
    of the complex first-order filter h_t = a h_{t-1} + x_t
    (scipy.signal.lfilter with a complex pole), started from h0."""
    rng = np.random.default_rng(44)
    L = 150
    raw, bias = np.float32(-1.0), np.float32(0.25)
    delta = float(np.logaddexp(0.0, float(raw) + float(bias)))
    A = complex(-_f32(0.3), _f32(2.5))
    Bs = _cplx32(rng, L)
    u = _f32(rng.normal(size=L))
    h0 = complex(0.75, -1.5)
    ins = dict(u=u.reshape(1, 1, L), delta=np.full((1, 1, L), raw, np.float32), A=np.array([[A]]),
               B=Bs.reshape(1, 1, L), C=np.ones((1, 1, L), np.complex128), D=None, z=None,
               delta_bias=np.full((1,), bias, np.float32), h0=np.array([[[h0]]]))
    out, last = oracle.scan_complex(**ins, lib=lib)
    a = np.exp(delta * A)
    x = delta * Bs * u.astype(np.float64)
    h, _ = signal.lfilter([1.0], [1.0, -a], x, zi=[a * h0])
    _close(out[0, 0], h.real, what="complex IIR (real part readout)")
    assert abs(last[0, 0, 0] - h[-1]) <= 1e-11 * abs(h[-1])


def pin_complex_brute_force(lib):
    """Tiny shapes: h_t = sum_{s<=t} (prod_{r=s+1..t} Abar_r) Bbar_s u_s
    with Python complex arithmetic (cmath), no recurrence; y as defined."""
    import cmath
    rng = np.random.default_rng(45)
    Bt, Dm, L, N = 2, 2, 9, 3
    p = _cplx_problem(rng, Bt, Dm, L, N)
    out, last = oracle.scan_complex(**p, lib=lib)
    for b in range(Bt):
        for d in range(Dm):
            dl = [float(np.logaddexp(0.0, float(p["delta"][b, d, t]) + float(p["delta_bias"][d]))) for t in range(L)]
            for t in range(L):
                y = 0.0
                for n in range(N):
                    hs = 0j
                    for s_ in range(t + 1):
                        prod = 1 + 0j
                        for r in range(s_ + 1, t + 1):
                            prod *= cmath.exp(dl[r] * complex(p["A"][d, n]))
                        hs += prod * dl[s_] * complex(p["B"][b, n, s_]) * float(p["u"][b, d, s_])
                    y += (complex(p["C"][b, n, t]) * hs).real
                    if t == L - 1:
                        assert abs(last[b, d, n] - hs) <= 1e-12 * max(1.0, abs(hs))
                y += float(p["D"][d]) * float(p["u"][b, d, t])
                zt = float(p["z"][b, d, t])
                y *= zt / (1.0 + math.exp(-zt))
                assert abs(out[b, d, t] - y) <= 1e-12 * max(1.0, abs(y)), (b, d, t, out[b, d, t], y)


def pin_complex_phase_invariance(lib):
    """Rotating state n by e^{i phi_n} -- B times e^{i phi_n}, C times
    e^{-i phi_n}, h0 times e^{i phi_n} -- leaves every output unchanged and
    rotates the final state; conjugating A, B, C and h0 leaves the outputs
    unchanged and conjugates the state."""
    rng = np.random.default_rng(46)
    Bt, Dm, L, N = 2, 3, 64, 4
    p = _cplx_problem(rng, Bt, Dm, L, N)
    h0 = _cplx32(rng, (Bt, Dm, N), 0.3)
    o1, s1 = oracle.scan_complex(**p, h0=h0, lib=lib)
    rot = np.exp(1j * rng.uniform(0, 2 * np.pi, N))
    q = dict(p, B=p["B"] * rot[None, :, None], C=p["C"] * np.conj(rot)[None, :, None])
    # the rotated inputs are rounded to fp32 on the way in: compare at that level
    o2, s2 = oracle.scan_complex(**q, h0=h0 * rot[None, None, :], lib=lib)
    _close(o2, o1, rtol=2e-6, what="phase rotation: outputs")
    _close(np.abs(s2 - s1 * rot[None, None, :]), np.zeros(s1.shape), scale=float(np.max(np.abs(s1))),
           rtol=2e-6, what="phase rotation: state")
    c = dict(p, A=np.conj(p["A"]), B=np.conj(p["B"]), C=np.conj(p["C"]))
    o3, s3 = oracle.scan_complex(**c, h0=np.conj(h0), lib=lib)
    _close(o3, o1, rtol=1e-13, what="conjugation: outputs")
    _close(np.abs(s3 - np.conj(s1)), np.zeros(s1.shape), scale=float(np.max(np.abs(s1))), rtol=1e-13,
           what="conjugation: state")


ALL_PINS = [pin_softplus_silu, pin_geometric_series, pin_lti_convolution,
            pin_first_order_iir, pin_zero_step_keeps_state, pin_memoryless_limit,
            pin_brute_force_products, pin_cumsum_form, pin_chunk_split,
            pin_steps_equal_scan, pin_causality, pin_linearity,
            pin_shared_bc_and_independence, pin_zero_b_or_c,
            pin_gate_and_softplus_flags,
            pin_conv_numpy, pin_conv_impulse, pin_conv_silu, pin_conv_wide_input,
            pin_conv_update_stream, pin_conv_causality,
            pin_bwd_autograd, pin_bwd_finite_differences,
            pin_complex_real_case, pin_complex_geometric_series, pin_complex_lti_convolution,
            pin_complex_iir, pin_complex_brute_force, pin_complex_phase_invariance]
