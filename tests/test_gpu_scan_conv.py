"""The causal conv1d + silu fused into the scan's prologue
(mamba_scan_fwd_conv): bit for bit the same as the conv1d kernel followed by
the scan, and within tolerance of the oracle's conv1d + scan (GPU)."""
import numpy as np
import pytest
import torch

import oracle
from parity import TOL, record, rel_err, to_np
from selective_state_space_20_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def _problem(batch, dim, L, N, dtype, K, seed, wide=True):
    w = inputs.custom(batch, dim, L, N, dtype, seed=seed)
    ins = inputs.scan_inputs(w, device="cuda")
    conv = inputs.conv_inputs(batch, dim, L, width=K, dtype=dtype, seed=seed + 1, device="cuda", wide=wide)
    x = conv["xz"] if wide else conv["x"]
    if wide:  # z as the other half of the same projection output
        x[:, dim:] = ins["z"]
        ins["z"] = x[:, dim:]
    return ins, x, conv["weight"], conv["bias"]


def _two_calls(ins, x, w, cb, dim, lanes, h0=None):
    u = binding.mamba_conv1d_fwd(x, w, cb, dim=dim)
    z = ins["z"].contiguous() if ins["z"] is not None else None
    out, last = binding.mamba_scan_fwd(u, ins["delta"], ins["A"], ins["B"], ins["C"], D=ins["D"], z=z,
                                       delta_bias=ins["delta_bias"], return_last_state=True, h0=h0,
                                       schedule=binding.SCHEDULE_PERSISTENT, lanes_per_channel=lanes)
    return u, out, last


def _plan_lanes(batch, dim, L, N, act):
    lanes, _, sched = binding.mamba_scan_plan(batch, dim, L, N, act)
    return lanes if sched == binding.SCHEDULE_PERSISTENT and lanes in (2, 4) else 2


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 64, 512), (3, 40, 1000), (1, 16, 16384), (4, 96, 2048)])
@pytest.mark.parametrize("K", [4, 2])
def test_fused_equals_two_calls(dtype, shape, K):
    b, d, L = shape
    L = L // 8 * 8
    ins, x, w, cb = _problem(b, d, L, 16, dtype, K, seed=d + L + K)
    out, last, u = binding.mamba_scan_fwd_conv(x, w, cb, ins["delta"], ins["A"], ins["B"], ins["C"], D=ins["D"],
                                               z=ins["z"], delta_bias=ins["delta_bias"], return_last_state=True,
                                               return_u=True)
    lanes = _plan_lanes(b, d, L, 16, inputs.DTYPES[dtype])
    u2, out2, last2 = _two_calls(ins, x, w, cb, d, lanes)
    torch.cuda.synchronize()
    assert torch.equal(u, u2)
    assert torch.equal(out, out2) and torch.equal(last, last2)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_fused_matches_oracle(dtype):
    b, d, L, N, K = 2, 48, 640, 16, 4
    ins, x, w, cb = _problem(b, d, L, N, dtype, K, seed=5)
    h0 = inputs.initial_state(b, d, N, seed=3).cuda()
    out, last = binding.mamba_scan_fwd_conv(x, w, cb, ins["delta"], ins["A"], ins["B"], ins["C"], D=ins["D"],
                                            z=ins["z"], delta_bias=ins["delta_bias"], h0=h0, return_last_state=True)
    torch.cuda.synchronize()
    cpu = lambda t: None if t is None else t.detach().to("cpu")  # noqa: E731
    u_ref = oracle.conv1d(cpu(x), cpu(w), cpu(cb), silu=True, dim=d)
    # u is an activation: the oracle's u rounded to the activation type
    u_act = torch.tensor(u_ref, dtype=torch.float32).to(inputs.DTYPES[dtype])
    ro, rs = oracle.scan(u_act, cpu(ins["delta"]), cpu(ins["A"]), cpu(ins["B"]), cpu(ins["C"]), D=cpu(ins["D"]),
                         z=cpu(ins["z"]), delta_bias=cpu(ins["delta_bias"]), h0=cpu(h0))
    tol = TOL[inputs.DTYPES[dtype]]
    e1, e2 = rel_err(to_np(out), ro), rel_err(to_np(last), rs)
    record(f"fused conv+scan {b}x{d}x{L} {dtype}", out=e1, state=e2)
    assert e1 <= tol and e2 <= tol, (e1, e2)


def test_fused_benchmark_layer():
    """The Mamba-2.8B layer, x and z as halves of one (4, 10240, 4096) bf16
    projection output: bit-equal to the two calls."""
    w = inputs.MAMBA_2_8B
    ins, x, cw, cb = _problem(w.batch, w.dim, w.seqlen, w.dstate, w.dtype, 4, seed=20)
    out, last = binding.mamba_scan_fwd_conv(x, cw, cb, ins["delta"], ins["A"], ins["B"], ins["C"], D=ins["D"],
                                            z=ins["z"], delta_bias=ins["delta_bias"], return_last_state=True)
    lanes = _plan_lanes(w.batch, w.dim, w.seqlen, w.dstate, inputs.DTYPES[w.dtype])
    _, out2, last2 = _two_calls(ins, x, cw, cb, w.dim, lanes)
    torch.cuda.synchronize()
    assert torch.equal(out, out2) and torch.equal(last, last2)


@pytest.mark.parametrize("K", [1, 3])
def test_fused_short_kernels_without_bias(K):
    b, d, L = 2, 64, 512
    ins, x, w, cb = _problem(b, d, L, 16, "bf16", K, seed=40 + K)
    out, last, u = binding.mamba_scan_fwd_conv(x, w, None, ins["delta"], ins["A"], ins["B"], ins["C"], D=ins["D"],
                                               z=ins["z"], delta_bias=ins["delta_bias"], return_last_state=True,
                                               return_u=True)
    lanes = _plan_lanes(b, d, L, 16, torch.bfloat16)
    u2, out2, last2 = _two_calls(ins, x, w, None, d, lanes)
    torch.cuda.synchronize()
    assert torch.equal(u, u2) and torch.equal(out, out2) and torch.equal(last, last2)
