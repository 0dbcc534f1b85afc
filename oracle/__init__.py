"""fp64 CPU oracle for the selective scan (S6) forward pass and state update.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  It shares
no code with the CUDA library in ``selective_state_space_20_b200``; neither
imports the other.

The arithmetic lives in ``s6_oracle.c`` (a plain sequential fp64 loop, see
its header for the equations and where each comes from).  This module only
marshals numpy/torch CPU arrays into it:

* :func:`scan` -- the whole forward scan (optionally from an initial state).
* :func:`scan_complex` -- the forward scan with complex A, B, C.
* :func:`scan_bwd` -- gradients of the forward scan (reverse mode).
* :func:`state_update` -- one recurrent step for every (batch, channel).
* :func:`conv1d`, :func:`conv1d_update` -- the causal depthwise convolution
  (+ bias, + silu) that feeds the scan, whole-sequence and one token.
* :func:`softplus`, :func:`silu` -- the pointwise functions the oracle uses.

Inputs may be numpy arrays or CPU torch tensors of any float dtype; they are
widened to fp32 (exact for bf16 and fp32 values) before the call, and all
arithmetic happens in fp64 inside the C code.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import numpy as np

from . import build as _build

_lib = None


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load (building first if needed) an oracle shared library."""
    lib = ctypes.CDLL(path or _build.build())
    f32p = ctypes.POINTER(ctypes.c_float)
    f64p = ctypes.POINTER(ctypes.c_double)
    i64 = ctypes.c_int64
    lib.s6_oracle_scan.restype = ctypes.c_int
    lib.s6_oracle_scan.argtypes = [f32p, f32p, f32p, f32p, f32p, f32p, f32p,
                                   f32p, ctypes.c_int, f64p, f64p, f64p,
                                   i64, i64, i64, i64, ctypes.c_int]
    lib.s6_oracle_state_update.restype = ctypes.c_int
    lib.s6_oracle_state_update.argtypes = [f64p, f32p, f32p, f32p, f32p, f32p,
                                           f32p, f32p, f32p, ctypes.c_int, f64p,
                                           i64, i64, i64]
    lib.s6_oracle_conv1d.restype = ctypes.c_int
    lib.s6_oracle_conv1d.argtypes = [f32p, f32p, f32p, ctypes.c_int, f64p, i64, i64, i64, i64, i64]
    lib.s6_oracle_conv1d_update.restype = ctypes.c_int
    lib.s6_oracle_conv1d_update.argtypes = [f64p, f32p, f32p, f32p, ctypes.c_int, f64p, i64, i64, i64]
    lib.s6_oracle_scan_bwd.restype = ctypes.c_int
    lib.s6_oracle_scan_bwd.argtypes = [f32p, f32p, f32p, f32p, f32p, f32p, f32p, f32p, ctypes.c_int,
                                       f64p, f64p, f64p, f64p, f64p, f64p, f64p, f64p, f64p, f64p,
                                       f64p, f64p, i64, i64, i64, i64, ctypes.c_int]
    lib.s6_oracle_scan_complex.restype = ctypes.c_int
    lib.s6_oracle_scan_complex.argtypes = lib.s6_oracle_scan.argtypes
    lib.s6_oracle_softplus.restype = ctypes.c_double
    lib.s6_oracle_softplus.argtypes = [ctypes.c_double]
    lib.s6_oracle_silu.restype = ctypes.c_double
    lib.s6_oracle_silu.argtypes = [ctypes.c_double]
    return lib


def _get():
    global _lib
    if _lib is None:
        _lib = load_library()
    return _lib


def _f32(x):
    """Exact fp32 numpy copy of an array/tensor (None passes through)."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float32).contiguous().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        import torch
        x = x.detach().to("cpu").to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p32(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def _p64(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def scan(u, delta, A, B, C, D=None, z=None, delta_bias=None,
         delta_softplus: bool = True, h0=None, nthreads: int = 0,
         lib: Optional[ctypes.CDLL] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Selective scan forward in fp64.

    Shapes: u, delta, z (batch, dim, L); B, C (batch, N, L); A (dim, N);
    D, delta_bias (dim,); h0 (batch, dim, N).  Returns ``(out, last_state)``
    as fp64 arrays of shapes (batch, dim, L) and (batch, dim, N).
    """
    lib = lib or _get()
    u, delta, A, B, C = (_f32(t) for t in (u, delta, A, B, C))
    D, z, delta_bias = _f32(D), _f32(z), _f32(delta_bias)
    h0 = _f64(h0)
    batch, dim, L = u.shape
    N = A.shape[1]
    assert delta.shape == u.shape and (z is None or z.shape == u.shape)
    assert A.shape == (dim, N) and B.shape == (batch, N, L) and C.shape == B.shape
    assert D is None or D.shape == (dim,)
    assert delta_bias is None or delta_bias.shape == (dim,)
    assert h0 is None or h0.shape == (batch, dim, N)
    out = np.empty((batch, dim, L), dtype=np.float64)
    last = np.empty((batch, dim, N), dtype=np.float64)
    rc = lib.s6_oracle_scan(_p32(u), _p32(delta), _p32(A), _p32(B), _p32(C),
                            _p32(D), _p32(z), _p32(delta_bias),
                            int(bool(delta_softplus)), _p64(h0), _p64(out),
                            _p64(last), batch, dim, L, N, int(nthreads))
    if rc != 0:
        raise RuntimeError(f"s6_oracle_scan failed with code {rc}")
    return out, last


def _pairs(x):
    """A complex array, or a real one whose last axis holds (re, im), as an
    fp32 (..., 2) array (exact for bf16 / fp32 parts)."""
    if x is None:
        return None
    if hasattr(x, "detach") and x.is_complex():
        x = x.detach().to("cpu").numpy()
    if isinstance(x, np.ndarray) and np.iscomplexobj(x):
        return np.ascontiguousarray(np.stack([x.real, x.imag], axis=-1).astype(np.float32))
    return _f32(x)


def scan_complex(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                 delta_softplus: bool = True, h0=None, nthreads: int = 0,
                 lib: Optional[ctypes.CDLL] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Complex-mode selective scan in fp64.

    u, delta, z (batch, dim, L) real; A (dim, N), B, C (batch, N, L) and
    h0 (batch, dim, N) complex -- complex arrays, or real ones with a
    trailing (re, im) axis.  Returns ``(out, last_state)``: out (batch, dim,
    L) fp64 and last_state (batch, dim, N) complex128.
    """
    lib = lib or _get()
    u, delta, D, z, delta_bias = _f32(u), _f32(delta), _f32(D), _f32(z), _f32(delta_bias)
    A, B, C = _pairs(A), _pairs(B), _pairs(C)
    if h0 is not None:
        h0 = np.asarray(h0.detach().cpu().numpy() if hasattr(h0, "detach") else h0)
        if np.iscomplexobj(h0):
            h0 = np.stack([h0.real, h0.imag], axis=-1)
        h0 = np.ascontiguousarray(h0, dtype=np.float64)
    batch, dim, L = u.shape
    N = A.shape[1]
    assert delta.shape == u.shape and (z is None or z.shape == u.shape)
    assert A.shape == (dim, N, 2) and B.shape == (batch, N, L, 2) and C.shape == B.shape
    assert D is None or D.shape == (dim,)
    assert delta_bias is None or delta_bias.shape == (dim,)
    assert h0 is None or h0.shape == (batch, dim, N, 2)
    out = np.empty((batch, dim, L), dtype=np.float64)
    last = np.empty((batch, dim, N, 2), dtype=np.float64)
    rc = lib.s6_oracle_scan_complex(_p32(u), _p32(delta), _p32(A), _p32(B), _p32(C),
                                    _p32(D), _p32(z), _p32(delta_bias),
                                    int(bool(delta_softplus)), _p64(h0), _p64(out),
                                    _p64(last), batch, dim, L, N, int(nthreads))
    if rc != 0:
        raise RuntimeError(f"s6_oracle_scan_complex failed with code {rc}")
    return out, last[..., 0] + 1j * last[..., 1]


def scan_bwd(dout, u, delta, A, B, C, D=None, z=None, delta_bias=None,
             delta_softplus: bool = True, h0=None, dlast=None, nthreads: int = 0,
             lib: Optional[ctypes.CDLL] = None) -> dict:
    """Gradients of :func:`scan` in fp64 for dL/dout = ``dout`` (batch, dim,
    L) and optionally dL/dlast_state = ``dlast`` (batch, dim, N).

    Returns a dict with du, ddelta, dz (batch, dim, L; dz None without z),
    dA (dim, N), dB, dC (batch, N, L), dD, ddelta_bias (dim,) and dh0
    (batch, dim, N)."""
    lib = lib or _get()
    u, delta, A, B, C = (_f32(t) for t in (u, delta, A, B, C))
    D, z, delta_bias = _f32(D), _f32(z), _f32(delta_bias)
    h0, dout, dlast = _f64(h0), _f64(dout), _f64(dlast)
    batch, dim, L = u.shape
    N = A.shape[1]
    assert dout.shape == u.shape and (dlast is None or dlast.shape == (batch, dim, N))
    r = {k: np.empty(s, dtype=np.float64) for k, s in (
        ("du", (batch, dim, L)), ("ddelta", (batch, dim, L)), ("dA", (dim, N)),
        ("dB", (batch, N, L)), ("dC", (batch, N, L)), ("dD", (dim,)),
        ("ddelta_bias", (dim,)), ("dh0", (batch, dim, N)))}
    r["dz"] = np.empty((batch, dim, L), dtype=np.float64) if z is not None else None
    rc = lib.s6_oracle_scan_bwd(_p32(u), _p32(delta), _p32(A), _p32(B), _p32(C), _p32(D), _p32(z),
                                _p32(delta_bias), int(bool(delta_softplus)), _p64(h0), _p64(dout),
                                _p64(dlast), _p64(r["du"]), _p64(r["ddelta"]), _p64(r["dA"]),
                                _p64(r["dB"]), _p64(r["dC"]), _p64(r["dD"]), _p64(r["dz"]),
                                _p64(r["ddelta_bias"]), _p64(r["dh0"]), batch, dim, L, N, int(nthreads))
    if rc != 0:
        raise RuntimeError(f"s6_oracle_scan_bwd failed with code {rc}")
    return r


def state_update(state, u, delta, A, B, C, D=None, z=None, delta_bias=None,
                 delta_softplus: bool = True,
                 lib: Optional[ctypes.CDLL] = None) -> Tuple[np.ndarray, np.ndarray]:
    """One recurrent step.  Returns ``(out, new_state)`` in fp64.

    Shapes: state (batch, dim, N); u, delta, z (batch, dim); B, C (batch, N);
    A (dim, N); D, delta_bias (dim,).  ``state`` is not modified.
    """
    lib = lib or _get()
    st = _f64(state).copy()
    u, delta, A, B, C = (_f32(t) for t in (u, delta, A, B, C))
    D, z, delta_bias = _f32(D), _f32(z), _f32(delta_bias)
    batch, dim = u.shape
    N = A.shape[1]
    assert st.shape == (batch, dim, N) and B.shape == (batch, N) and C.shape == B.shape
    out = np.empty((batch, dim), dtype=np.float64)
    rc = lib.s6_oracle_state_update(_p64(st), _p32(u), _p32(delta), _p32(A),
                                    _p32(B), _p32(C), _p32(D), _p32(z),
                                    _p32(delta_bias), int(bool(delta_softplus)),
                                    _p64(out), batch, dim, N)
    if rc != 0:
        raise RuntimeError(f"s6_oracle_state_update failed with code {rc}")
    return out, st


def conv1d(x, weight, bias=None, silu: bool = True, dim: Optional[int] = None,
           lib: Optional[ctypes.CDLL] = None) -> np.ndarray:
    """Causal depthwise convolution + bias (+ silu) in fp64.

    x: (batch, C, L) with C >= dim (the first ``dim`` channel rows are used,
    as when x is the x half of a (batch, 2 * dim, L) projection output);
    weight (dim, K); bias (dim,).  Returns (batch, dim, L) fp64.
    """
    lib = lib or _get()
    x, weight, bias = _f32(x), _f32(weight), _f32(bias)
    batch, C, L = x.shape
    dim = dim or C
    K = weight.shape[1]
    assert weight.shape == (dim, K) and C >= dim and (bias is None or bias.shape == (dim,))
    out = np.empty((batch, dim, L), dtype=np.float64)
    rc = lib.s6_oracle_conv1d(_p32(x), _p32(weight), _p32(bias), int(bool(silu)), _p64(out),
                              batch, dim, L, K, C * L)
    if rc != 0:
        raise RuntimeError(f"s6_oracle_conv1d failed with code {rc}")
    return out


def conv1d_update(state, x, weight, bias=None, silu: bool = True,
                  lib: Optional[ctypes.CDLL] = None) -> Tuple[np.ndarray, np.ndarray]:
    """One token of :func:`conv1d`.  state (batch, dim, K-1), oldest input
    first; x (batch, dim).  Returns ``(out, new_state)`` in fp64; ``state`` is
    not modified."""
    lib = lib or _get()
    st = _f64(state).copy()
    x, weight, bias = _f32(x), _f32(weight), _f32(bias)
    batch, dim = x.shape
    K = weight.shape[1]
    assert st.shape == (batch, dim, K - 1) and weight.shape == (dim, K)
    out = np.empty((batch, dim), dtype=np.float64)
    rc = lib.s6_oracle_conv1d_update(_p64(st), _p32(x), _p32(weight), _p32(bias), int(bool(silu)),
                                     _p64(out), batch, dim, K)
    if rc != 0:
        raise RuntimeError(f"s6_oracle_conv1d_update failed with code {rc}")
    return out, st


def softplus(x: float, lib: Optional[ctypes.CDLL] = None) -> float:
    return (lib or _get()).s6_oracle_softplus(float(x))


def silu(x: float, lib: Optional[ctypes.CDLL] = None) -> float:
    return (lib or _get()).s6_oracle_silu(float(x))


def library_path() -> str:
    return os.path.abspath(_build.LIB)
