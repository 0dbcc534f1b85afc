"""Parity of the one-token state update with the oracle and with the full
scan (GPU, through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle
from parity import TOL, oracle_rows, record, rel_err, sample_rows, to_np
from selective_state_space_20_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def step_inputs(batch, dim, N, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    dt = inputs.DTYPES[dtype]
    r = lambda *s, scale=1.0: (torch.randn(*s, generator=g) * scale).to(dt)  # noqa: E731
    return dict(state=torch.randn(batch, dim, N, generator=g, dtype=torch.float64).float(),
                u=r(batch, dim), delta=r(batch, dim, scale=0.5),
                A=-(torch.rand(dim, N, generator=g) * 4 + 0.2), B=r(batch, N), C=r(batch, N),
                D=torch.rand(dim, generator=g) + 0.5, z=r(batch, dim),
                delta_bias=torch.log(torch.expm1(torch.rand(dim, generator=g) * 0.1 + 1e-3)).float())


def run_step(ins, softplus=True):
    st = ins["state"].clone()
    out = binding.mamba_state_update(st, ins["u"], ins["delta"], ins["A"], ins["B"], ins["C"],
                                     D=ins["D"], z=ins["z"], delta_bias=ins["delta_bias"],
                                     delta_softplus=softplus)
    return out, st


@pytest.mark.parametrize("dstate", [1, 3, 4, 8, 13, 16, 32, 48, 64])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_one_step_matches_oracle(dstate, dtype):
    cpu = step_inputs(7, 301, dstate, dtype, seed=dstate)
    dev = {k: v.cuda() for k, v in cpu.items()}
    out, st = run_step(dev)
    ro, rs = oracle.state_update(cpu["state"], cpu["u"], cpu["delta"], cpu["A"], cpu["B"], cpu["C"],
                                 D=cpu["D"], z=cpu["z"], delta_bias=cpu["delta_bias"])
    tol = TOL[inputs.DTYPES[dtype]]
    e_out, e_st = rel_err(to_np(out), ro), rel_err(to_np(st), rs)
    record(f"state_update one step N={dstate} {dtype}", out=e_out, state=e_st)
    assert e_out <= tol and e_st <= 1e-4  # the state is fp32 from exact inputs


def test_optional_inputs_and_softplus_off():
    cpu = step_inputs(3, 64, 16, "fp32", seed=5)
    cpu["delta"] = cpu["delta"].abs()
    for drop in ("z", "D", "delta_bias"):
        c = dict(cpu)
        c[drop] = None
        dev = {k: (None if v is None else v.cuda()) for k, v in c.items()}
        out, st = run_step(dev, softplus=False)
        ro, rs = oracle.state_update(c["state"], c["u"], c["delta"], c["A"], c["B"], c["C"],
                                     D=c["D"], z=c["z"], delta_bias=c["delta_bias"],
                                     delta_softplus=False)
        assert rel_err(to_np(out), ro) <= 1e-4 and rel_err(to_np(st), rs) <= 1e-5


def test_misaligned_state_takes_scalar_path():
    cpu = step_inputs(2, 33, 16, "bf16", seed=6)
    dev = {k: v.cuda() for k, v in cpu.items()}
    buf = torch.empty(dev["state"].numel() + 1, device="cuda")
    st = buf[1:].view(dev["state"].shape)
    st.copy_(dev["state"])
    out = binding.mamba_state_update(st, dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"],
                                     D=dev["D"], z=dev["z"], delta_bias=dev["delta_bias"])
    ro, rs = oracle.state_update(cpu["state"], cpu["u"], cpu["delta"], cpu["A"], cpu["B"], cpu["C"],
                                 D=cpu["D"], z=cpu["z"], delta_bias=cpu["delta_bias"])
    assert rel_err(to_np(out), ro) <= 2e-2 and rel_err(to_np(st), rs) <= 1e-5


def test_decode_workload_1024_steps():
    """The decoding workload: 256 x 5120 channels, N = 16, 1024 one-token
    calls on an fp32 state resident in HBM, checked against one full scan of
    the same inputs and, on sampled rows, against the oracle."""
    w = inputs.DECODE
    d = inputs.decode_inputs(w, device="cuda")
    state = torch.zeros(w.batch, w.dim, w.dstate, device="cuda")
    outs = torch.empty(w.steps, w.batch, w.dim, device="cuda", dtype=inputs.DTYPES[w.dtype])
    for t in range(w.steps):
        binding.mamba_state_update(state, d["u"][t], d["delta"][t], d["A"], d["B"][t], d["C"][t],
                                   D=d["D"], z=d["z"][t], delta_bias=d["delta_bias"], out=outs[t])
    s = inputs.decode_as_scan(d)
    del d
    scan_out, scan_last = binding.mamba_scan_fwd(s["u"], s["delta"], s["A"], s["B"], s["C"],
                                                 D=s["D"], z=s["z"], delta_bias=s["delta_bias"],
                                                 return_last_state=True)
    torch.cuda.synchronize()
    dec = outs.permute(1, 2, 0)  # (batch, dim, steps)
    # GPU decode vs GPU scan: same fp32 arithmetic up to summation order
    diff = (dec.float() - scan_out.float()).abs().max().item()
    scale = scan_out.float().abs().max().item()
    assert diff <= 2e-2 * scale
    e_state = rel_err(to_np(state), to_np(scan_last))
    assert e_state <= 1e-4, e_state
    rows = sample_rows(w.batch, w.dim, 16, seed=w.seed)
    ro, rs = oracle_rows(s, rows)
    idx = torch.tensor(rows, device="cuda")
    go = to_np(dec.reshape(w.batch * w.dim, w.steps).index_select(0, idx))
    gs = to_np(state.view(-1, w.dstate).index_select(0, idx))
    e_out, e_st = rel_err(go, ro), rel_err(gs, rs)
    record("decode 1024 steps, sampled rows", out=e_out, state=e_st, scan_vs_decode=diff / scale,
           state_vs_scan=e_state)
    assert e_out <= 2e-2 and e_st <= 2e-2


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_misaligned_b_c_take_row_kernel(dtype):
    # aligned state and A, B / C rows starting off their 16-byte grid
    cpu = step_inputs(3, 40, 16, dtype, seed=8)
    dev = {k: v.cuda() for k, v in cpu.items()}
    for k in ("B", "C"):
        buf = torch.empty(dev[k].numel() + 1, device="cuda", dtype=dev[k].dtype)
        t = buf[1:].view(dev[k].shape)
        t.copy_(dev[k])
        dev[k] = t
    out, st = run_step(dev)
    ro, rs = oracle.state_update(cpu["state"], cpu["u"], cpu["delta"], cpu["A"], cpu["B"], cpu["C"],
                                 D=cpu["D"], z=cpu["z"], delta_bias=cpu["delta_bias"])
    assert rel_err(to_np(out), ro) <= TOL[inputs.DTYPES[dtype]] and rel_err(to_np(st), rs) <= 1e-4
