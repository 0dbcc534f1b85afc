"""The scan on sequences in host memory (mamba_scan_fwd_host): chunks copied
in, scanned and copied back on overlapping streams must give the device
scan's results (GPU)."""
import pytest
import torch

import oracle
from parity import TOL, record, rel_err, to_np
from selective_state_space_20_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def _host(cpu, pinned):
    return {k: (None if v is None else (v.pin_memory() if pinned else v.clone()))
            for k, v in cpu.items() if k in ("u", "delta", "z", "B", "C")}


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape,dstate", [((4, 96, 1024), 16), ((1, 37, 333), 16), ((3, 8, 64), 5),
                                          ((2, 40, 256), 24)])
@pytest.mark.parametrize("pinned", [True, False])
def test_host_scan_matches_oracle(dtype, shape, dstate, pinned):
    b, d, L = shape
    w = inputs.custom(b, d, L, dstate, dtype, seed=b + d + L + dstate)
    cpu = inputs.scan_inputs(w)
    h = _host(cpu, pinned)
    par = {k: (None if cpu[k] is None else cpu[k].cuda()) for k in ("A", "D", "delta_bias")}
    out, last = binding.mamba_scan_fwd_host(h["u"], h["delta"], par["A"], h["B"], h["C"], D=par["D"], z=h["z"],
                                            delta_bias=par["delta_bias"], return_last_state=True)
    torch.cuda.current_stream().synchronize()
    ro, rs = oracle.scan(cpu["u"], cpu["delta"], cpu["A"], cpu["B"], cpu["C"], D=cpu["D"], z=cpu["z"],
                         delta_bias=cpu["delta_bias"])
    tol = TOL[inputs.DTYPES[dtype]]
    e1, e2 = rel_err(to_np(out), ro), rel_err(to_np(last), rs)
    record(f"host-memory scan {w.name} pinned={pinned}", out=e1, state=e2)
    assert e1 <= tol and e2 <= tol, (e1, e2)


def test_host_scan_from_a_state_without_gate():
    w = inputs.custom(2, 64, 512, 16, "bf16", seed=8)
    cpu = inputs.scan_inputs(w)
    cpu["z"] = None
    h = _host(cpu, True)
    h0 = inputs.initial_state(2, 64, 16, seed=2)
    par = {k: cpu[k].cuda() for k in ("A", "D", "delta_bias")}
    out, last = binding.mamba_scan_fwd_host(h["u"], h["delta"], par["A"], h["B"], h["C"], D=par["D"],
                                            delta_bias=par["delta_bias"], h0=h0.cuda(), return_last_state=True)
    torch.cuda.current_stream().synchronize()
    ro, rs = oracle.scan(cpu["u"], cpu["delta"], cpu["A"], cpu["B"], cpu["C"], D=cpu["D"],
                         delta_bias=cpu["delta_bias"], h0=h0)
    assert rel_err(to_np(out), ro) <= 2e-2 and rel_err(to_np(last), rs) <= 2e-2


def test_host_scan_benchmark_layer_matches_device_scan():
    """The Mamba-2.8B layer from pinned host memory against the device scan
    of the whole problem (the chunks run as their own problems, so lane
    splits, and with them summation orders, may differ: compared within the
    bf16 tolerance)."""
    wl = inputs.MAMBA_2_8B
    dev = inputs.scan_inputs(wl, device="cuda")
    h = {k: dev[k].cpu().pin_memory() for k in ("u", "delta", "z", "B", "C")}
    out, last = binding.mamba_scan_fwd_host(h["u"], h["delta"], dev["A"], h["B"], h["C"], D=dev["D"], z=h["z"],
                                            delta_bias=dev["delta_bias"], return_last_state=True)
    o2, s2 = binding.mamba_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                                    delta_bias=dev["delta_bias"], return_last_state=True)
    torch.cuda.current_stream().synchronize()
    e1, e2 = rel_err(to_np(out), to_np(o2)), rel_err(to_np(last), to_np(s2))
    record("host-memory scan mamba-2.8b vs device scan", out=e1, state=e2)
    assert e1 <= 2e-2 and e2 <= 1e-3, (e1, e2)
