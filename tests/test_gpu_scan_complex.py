"""Complex-valued mode of the scan through the C ABI against the fp64
oracle's complex mode (GPU)."""
import numpy as np
import pytest
import torch

import oracle
from parity import TOL, record, rel_err, to_np
from selective_state_space_20_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def _oracle(cpu, softplus=True, h0=None):
    return oracle.scan_complex(cpu["u"], cpu["delta"], cpu["A"], cpu["B"], cpu["C"], D=cpu["D"], z=cpu["z"],
                               delta_bias=cpu["delta_bias"], delta_softplus=softplus, h0=h0)


def _run(dev, softplus=True, **kw):
    return binding.mamba_scan_fwd_complex(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"],
                                          z=dev["z"], delta_bias=dev["delta_bias"], delta_softplus=softplus,
                                          return_last_state=True, **kw)


def _check(name, cpu, dtype, softplus=True, h0=None, **kw):
    dev = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    out, last = _run(dev, softplus=softplus, h0=None if h0 is None else h0.cuda(), **kw)
    torch.cuda.synchronize()
    ro, rs = _oracle(cpu, softplus=softplus, h0=h0)
    rs2 = np.stack([rs.real, rs.imag], axis=-1)
    tol = TOL[inputs.DTYPES[dtype]]
    e1, e2 = rel_err(to_np(out), ro), rel_err(to_np(last), rs2)
    record(f"complex {name} {kw}", out=e1, state=e2)
    assert e1 <= tol and e2 <= tol, (name, kw, e1, e2)
    return out, last


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape,dstate", [((2, 64, 256), 16), ((3, 37, 129), 16), ((1, 5, 7), 3),
                                          ((2, 40, 333), 8), ((1, 1, 1), 16), ((2, 33, 100), 1)])
@pytest.mark.parametrize("lanes", [0, 1, 2, 4])
def test_complex_matches_oracle(dtype, shape, dstate, lanes):
    b, d, L = shape
    cpu = inputs.complex_inputs(b, d, L, dstate, dtype, seed=d + L + dstate)
    _check(f"{b}x{d}x{L} N{dstate} {dtype}", cpu, dtype, lanes_per_channel=lanes)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_complex_long_rows_and_large_steps(dtype):
    # dt up to 0.5: rotation angles delta * pi * n well past pi, reduced
    # before sin / cos; 4096 steps carry any phase error far
    cpu = inputs.complex_inputs(2, 32, 4096, 16, dtype, seed=3, dt_min=0.01, dt_max=0.5)
    _check(f"long rows {dtype}", cpu, dtype)


def test_complex_optional_inputs_and_softplus_off():
    cpu = inputs.complex_inputs(2, 48, 200, 16, "fp32", seed=8, gate=False)
    cpu["D"] = None
    cpu["delta_bias"] = None
    _check("no z / D / bias", cpu, "fp32")
    cpu = inputs.complex_inputs(2, 48, 200, 16, "fp32", seed=9)
    cpu["delta"] = cpu["delta"].abs() * 0.1
    cpu["delta_bias"] = cpu["delta_bias"].abs() * 0.01
    _check("softplus off", cpu, "fp32", softplus=False)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_complex_from_a_state_and_chained(dtype):
    b, d, L, N = 2, 40, 512, 16
    cpu = inputs.complex_inputs(b, d, L, N, dtype, seed=14)
    h0 = inputs.initial_state(b, d, N * 2, seed=6).reshape(b, d, N, 2).contiguous()
    _check("from h0", cpu, dtype, h0=h0)
    dev = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    full, last = _run(dev)
    L1 = 200
    seq = ("u", "delta", "z")
    head = {k: (v[:, :, :L1].contiguous() if k in seq else v[:, :, :L1].contiguous() if k in ("B", "C") else v)
            for k, v in dev.items()}
    tail = {k: (v[:, :, L1:].contiguous() if k in seq or k in ("B", "C") else v) for k, v in dev.items()}
    o1, s1 = _run(head)
    o2, s2 = _run(tail, h0=s1)
    tol = TOL[inputs.DTYPES[dtype]]
    assert rel_err(to_np(torch.cat([o1, o2], dim=-1)), to_np(full)) <= tol
    assert rel_err(to_np(s2), to_np(last)) <= 1e-4
    # in place: h0 is last_state
    st = s1.clone()
    o3, s3 = _run(tail, h0=st, last_state=st)
    assert torch.equal(o3, o2) and torch.equal(s3, s2)


def test_complex_with_real_parts_only_matches_the_real_scan():
    w = inputs.custom(2, 64, 256, 16, "fp32", seed=21)
    cpu = inputs.scan_inputs(w)
    dev = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    o_r, s_r = binding.mamba_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                                      delta_bias=dev["delta_bias"], return_last_state=True,
                                      schedule=binding.SCHEDULE_STATIC)
    cplx = dict(dev, A=torch.stack([dev["A"], torch.zeros_like(dev["A"])], -1).contiguous(),
                B=torch.stack([dev["B"], torch.zeros_like(dev["B"])], -1).contiguous(),
                C=torch.stack([dev["C"], torch.zeros_like(dev["C"])], -1).contiguous())
    o_c, s_c = _run(cplx)
    # two fp32 evaluations of one recurrence (different exp forms): each is
    # within the fp32 tolerance of the exact values
    assert rel_err(to_np(o_c), to_np(o_r)) <= 1e-4
    assert rel_err(to_np(s_c[..., 0]), to_np(s_r)) <= 1e-4 and not torch.any(s_c[..., 1])


def test_complex_rejects_bad_arguments():
    cpu = inputs.complex_inputs(1, 8, 64, 16, "bf16", seed=1)
    dev = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    with pytest.raises(ValueError):
        binding.mamba_scan_fwd_complex(dev["u"], dev["delta"], dev["A"][..., 0].contiguous(), dev["B"], dev["C"])
    big = inputs.complex_inputs(1, 8, 64, 17, "bf16", seed=1)
    dev = {k: (None if v is None else v.cuda()) for k, v in big.items()}
    with pytest.raises(binding.MambaError):  # dstate > 16
        _run(dev)


def test_complex_benchmark_shape_sampled():
    """The shape the bench times complex mode on (4 x 5120 x 4096, N = 16,
    bf16), sampled rows against the oracle run on each row alone."""
    b, d, L, N = 4, 5120, 4096, 16
    dev = {k: (None if v is None else v.cuda()) for k, v in inputs.complex_inputs(b, d, L, N, "bf16", device="cuda").items()}
    out, last = _run(dev)
    torch.cuda.synchronize()
    rows = [(0, 0), (0, 5119), (1, 777), (2, 2048), (3, 0), (3, 5119)]
    cpu = lambda t: None if t is None else t.detach().to("cpu")  # noqa: E731
    errs = []
    for bi, di in rows:
        ro, rs = oracle.scan_complex(cpu(dev["u"][bi:bi + 1, di:di + 1]), cpu(dev["delta"][bi:bi + 1, di:di + 1]),
                                     cpu(dev["A"][di:di + 1]), cpu(dev["B"][bi:bi + 1]), cpu(dev["C"][bi:bi + 1]),
                                     D=cpu(dev["D"][di:di + 1]), z=cpu(dev["z"][bi:bi + 1, di:di + 1]),
                                     delta_bias=cpu(dev["delta_bias"][di:di + 1]), nthreads=1)
        errs.append((rel_err(to_np(out[bi, di]), ro[0, 0]),
                     rel_err(to_np(last[bi, di]), np.stack([rs.real, rs.imag], -1)[0, 0])))
    e_out, e_state = max(e[0] for e in errs), max(e[1] for e in errs)
    record("complex 4x5120x4096 N16 bf16 sampled", out=e_out, state=e_state)
    assert e_out <= TOL[torch.bfloat16] and e_state <= TOL[torch.bfloat16], errs
