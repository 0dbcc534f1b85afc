"""Seeded synthetic inputs for the selective scan and the state update.

This module only draws random numbers and lays them out; it holds none of the
scan's arithmetic.  Both the fp64 oracle and the CUDA library are fed from it,
so the two always see bit-identical input values: everything is drawn in fp32
from a seeded ``torch.Generator`` and cast to the activation dtype *before*
either side reads it.

Recipe (the shapes follow the Mamba layer sizes of the state-spaces model
table, d_inner = 2 * d_model with d_state 16; the distributions follow the
dt initialisation of the mamba-jax ``train.py`` flags and the Keras/TensorFlow
``ModelArgs``):

* ``A[d, n] = -(n + 1)``  (S4D-real: A = -exp(A_log), A_log = log(1..N)).
* ``delta_raw ~ 0.5 * N(0, 1)`` per (b, d, t).
* ``delta_bias[d] = log(expm1(dt_d))`` with ``dt_d`` log-uniform in
  ``[dt_min, dt_max]`` and floored at ``dt_floor`` -- the bias that makes
  softplus(bias) equal dt, which is how the dt projection's bias is
  initialised to target a range of step sizes.
* ``u, B, C, z ~ N(0, 1)``.
* ``D = 1`` or ``D ~ U(0.5, 1.5)`` depending on the workload.

Convolution inputs (the causal depthwise conv1d that produces u): the x half
of the input projection's output ``xz ~ N(0, 1)`` of shape (batch, 2 dim, L)
(x = the first dim channel rows), conv weight and bias ``~ U(-1/sqrt(K),
1/sqrt(K))`` -- the default uniform initialisation bound of a convolution
with fan-in K (one input channel per group, K taps).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch

DTYPES = {"fp32": torch.float32, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class ScanWorkload:
    """One named scan-forward workload."""
    name: str
    batch: int
    dim: int
    seqlen: int
    dstate: int
    dtype: str            # activation dtype of u/delta/z/B/C/out
    dt_min: float
    dt_max: float
    d_mode: str           # "ones" or "uniform" (U(0.5, 1.5))
    seed: int
    dt_floor: float = 1e-4
    gate: bool = True
    softplus: bool = True
    emit_last_state: bool = True

    @property
    def elements(self) -> int:
        return self.batch * self.dim * self.seqlen


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """Recurrent decoding: one token per call for ``steps`` calls."""
    name: str
    batch: int
    dim: int
    dstate: int
    steps: int
    dtype: str
    dt_min: float
    dt_max: float
    d_mode: str
    seed: int
    dt_floor: float = 1e-4
    gate: bool = True
    softplus: bool = True


# The five workloads the path is measured and checked on.
TINY_FP32 = ScanWorkload("tiny-fp32 1x64x256 N16", 1, 64, 256, 16, "fp32",
                         1e-3, 1e-1, "ones", seed=20)
MAMBA_130M = ScanWorkload("mamba-130m layer 8x1536x2048 N16", 8, 1536, 2048, 16,
                          "bf16", 1e-3, 1e-1, "ones", seed=21)
MAMBA_2_8B = ScanWorkload("mamba-2.8b layer 4x5120x4096 N16", 4, 5120, 4096, 16,
                          "bf16", 1e-3, 1e-1, "uniform", seed=22)
LONG_CONTEXT = ScanWorkload("long-context 1x2048x262144 N16", 1, 2048, 262144, 16,
                            "bf16", 1e-4, 1e-2, "uniform", seed=23)
DECODE = DecodeWorkload("decode 256x5120 N16 x1024 steps", 256, 5120, 16, 1024,
                        "bf16", 1e-3, 1e-1, "uniform", seed=24)

SCAN_WORKLOADS = {"tiny": TINY_FP32, "mamba130m": MAMBA_130M,
                  "mamba2.8b": MAMBA_2_8B, "long": LONG_CONTEXT}


def custom(batch: int, dim: int, seqlen: int, dstate: int = 16,
           dtype: str = "fp32", seed: int = 0, dt_min: float = 1e-3,
           dt_max: float = 1e-1, d_mode: str = "uniform", gate: bool = True,
           softplus: bool = True, name: Optional[str] = None) -> ScanWorkload:
    """An ad-hoc workload with the standard distributions (tests use this)."""
    return ScanWorkload(name or f"custom {batch}x{dim}x{seqlen} N{dstate} {dtype}",
                        batch, dim, seqlen, dstate, dtype, dt_min, dt_max, d_mode,
                        seed, gate=gate, softplus=softplus)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _params(dim: int, dstate: int, dt_min: float, dt_max: float,
            dt_floor: float, d_mode: str, g: torch.Generator, device):
    """Per-channel parameters A (dim, N), D (dim,), delta_bias (dim,), fp32."""
    A = -torch.arange(1, dstate + 1, dtype=torch.float32, device=device)
    A = A.unsqueeze(0).expand(dim, dstate).contiguous()
    r = torch.rand(dim, generator=g, device=device, dtype=torch.float64)
    dt = torch.exp(r * (math.log(dt_max) - math.log(dt_min)) + math.log(dt_min))
    dt = dt.clamp(min=dt_floor)
    bias = torch.log(torch.expm1(dt)).to(torch.float32)
    if d_mode == "ones":
        D = torch.ones(dim, dtype=torch.float32, device=device)
    elif d_mode == "uniform":
        D = (torch.rand(dim, generator=g, device=device, dtype=torch.float32) + 0.5)
    else:
        raise ValueError(f"unknown d_mode {d_mode!r}")
    return A, D.contiguous(), bias.contiguous()


def _normal(shape, g, device, dtype, scale: float = 1.0) -> torch.Tensor:
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(dtype).contiguous()


def scan_inputs(w: ScanWorkload, device="cpu") -> Dict[str, torch.Tensor]:
    """All inputs of one scan workload, as contiguous tensors on ``device``.

    Keys: u, delta, z (batch, dim, L) and B, C (batch, N, L) in the
    activation dtype; A (dim, N), D (dim,), delta_bias (dim,) in fp32.
    ``z`` is None when the workload has no gate.
    The values depend only on the workload and the device type's generator
    (CPU draws are identical on every machine).
    """
    dt = DTYPES[w.dtype]
    g = _gen(w.seed, device)
    A, D, bias = _params(w.dim, w.dstate, w.dt_min, w.dt_max, w.dt_floor,
                         w.d_mode, g, device)
    shp = (w.batch, w.dim, w.seqlen)
    u = _normal(shp, g, device, dt)
    delta = _normal(shp, g, device, dt, 0.5)
    z = _normal(shp, g, device, dt) if w.gate else None
    B = _normal((w.batch, w.dstate, w.seqlen), g, device, dt)
    C = _normal((w.batch, w.dstate, w.seqlen), g, device, dt)
    return {"u": u, "delta": delta, "A": A, "B": B, "C": C, "D": D, "z": z,
            "delta_bias": bias}


def decode_inputs(w: DecodeWorkload, device="cpu", steps: Optional[int] = None
                  ) -> Dict[str, torch.Tensor]:
    """Per-step inputs for ``steps`` decoding calls, stacked on a leading axis.

    Keys: u, delta, z (steps, batch, dim) and B, C (steps, batch, N) in the
    activation dtype; A (dim, N), D, delta_bias (dim,) in fp32.
    Step t of the decode sees exactly what time index t of a full scan over
    the same values would see (see :func:`decode_as_scan`).
    """
    steps = w.steps if steps is None else steps
    dt = DTYPES[w.dtype]
    g = _gen(w.seed, device)
    A, D, bias = _params(w.dim, w.dstate, w.dt_min, w.dt_max, w.dt_floor,
                         w.d_mode, g, device)
    shp = (steps, w.batch, w.dim)
    u = _normal(shp, g, device, dt)
    delta = _normal(shp, g, device, dt, 0.5)
    z = _normal(shp, g, device, dt) if w.gate else None
    B = _normal((steps, w.batch, w.dstate), g, device, dt)
    C = _normal((steps, w.batch, w.dstate), g, device, dt)
    return {"u": u, "delta": delta, "A": A, "B": B, "C": C, "D": D, "z": z,
            "delta_bias": bias}


def decode_as_scan(d: Dict[str, torch.Tensor]) -> Dict[str, torch.Tensor]:
    """Re-lay stacked decode inputs as one scan problem (a pure transpose):
    (steps, batch, dim) -> (batch, dim, steps) and (steps, batch, N) ->
    (batch, N, steps)."""
    out = dict(d)
    for k in ("u", "delta", "z"):
        if d.get(k) is not None:
            out[k] = d[k].permute(1, 2, 0).contiguous()
    for k in ("B", "C"):
        out[k] = d[k].permute(1, 2, 0).contiguous()
    return out


def conv_inputs(batch: int, dim: int, seqlen: int, width: int = 4, dtype: str = "bf16",
                seed: int = 40, device="cpu", wide: bool = True) -> Dict[str, torch.Tensor]:
    """Inputs of the causal depthwise conv1d: ``xz`` (batch, 2 dim, L) in the
    activation dtype when ``wide`` (the projection output; x = xz[:, :dim]),
    else ``x`` (batch, dim, L); ``weight`` (dim, width) and ``bias`` (dim,)
    fp32."""
    g = _gen(seed, device)
    bound = 1.0 / math.sqrt(width)
    weight = ((torch.rand(dim, width, generator=g, device=device) * 2 - 1) * bound).contiguous()
    bias = ((torch.rand(dim, generator=g, device=device) * 2 - 1) * bound).contiguous()
    rows = 2 * dim if wide else dim
    x = _normal((batch, rows, seqlen), g, device, DTYPES[dtype])
    return {"xz" if wide else "x": x, "weight": weight, "bias": bias}


def initial_state(batch: int, dim: int, dstate: int, seed: int = 50, device="cpu",
                  scale: float = 0.25) -> torch.Tensor:
    """A seeded fp32 state (batch, dim, dstate) to start a scan from: normal
    values times ``scale``.  The default is about the spread of the states a
    scan of unit-variance inputs leaves behind: h_t = a h_{t-1} + delta B u
    with a = exp(delta A) settles at variance delta^2 / (1 - a^2), close to
    delta / (2 |A|) = 0.05 for delta = 0.1, A = -1."""
    return _normal((batch, dim, dstate), _gen(seed, device), device, torch.float32, scale)


def complex_inputs(batch: int, dim: int, seqlen: int, dstate: int = 16, dtype: str = "bf16",
                   seed: int = 60, device="cpu", dt_min: float = 0.001, dt_max: float = 0.1,
                   gate: bool = True) -> Dict[str, torch.Tensor]:
    """Inputs of one complex-mode scan.  u, delta, z (batch, dim, L) as in
    :func:`scan_inputs`; A (dim, N, 2) fp32 with real part -1/2 and
    imaginary part pi n (the usual complex diagonal initialisation with
    linearly spaced frequencies); B, C (batch, N, L, 2) with N(0, 1/2) real
    and imaginary parts (unit mean square magnitude); D ~ U(0.5, 1.5) and the
    dt bias as in :func:`scan_inputs`."""
    dt = DTYPES[dtype]
    g = _gen(seed, device)
    _, D, bias = _params(dim, dstate, dt_min, dt_max, 1e-4, "uniform", g, device)
    n = torch.arange(dstate, dtype=torch.float32, device=device)
    A = torch.stack([torch.full((dim, dstate), -0.5, device=device),
                     (math.pi * n).expand(dim, dstate)], dim=-1).contiguous()
    shp = (batch, dim, seqlen)
    u = _normal(shp, g, device, dt)
    delta = _normal(shp, g, device, dt, 0.5)
    z = _normal(shp, g, device, dt) if gate else None
    B = _normal((batch, dstate, seqlen, 2), g, device, dt, math.sqrt(0.5))
    C = _normal((batch, dstate, seqlen, 2), g, device, dt, math.sqrt(0.5))
    return {"u": u, "delta": delta, "A": A, "B": B, "C": C, "D": D, "z": z, "delta_bias": bias}
