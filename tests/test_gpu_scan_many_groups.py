"""Shapes with enough channel groups that no piece of the lane-split kernel
is two-phase (lane pairs: every block at least 5 whole 16-channel groups
for its 8 warps, or 1184 device-wide workers at least 652 groups; four
lanes: 7 whole 8-channel groups for 12 warps, or 1776 workers at least 977
groups): the launch then takes the kernel's unrolled form.  Every output
and final state against the fp64 oracle (GPU)."""
import pytest
import torch

import oracle
from parity import TOL, record, rel_err, to_np
from selective_state_space_20_b200 import binding, inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("form", ["block-local", "device-wide"])
@pytest.mark.parametrize("lanes,L,with_h0,gate", [(2, 96, False, True), (2, 104, True, True), (2, 64, False, False),
                                                  (4, 96, False, True), (4, 104, True, True)])
def test_many_groups_match_oracle(form, lanes, L, with_h0, gate):
    b, N = 4, 16
    d = 2960 if lanes == 2 else 2072  # 740 groups of 16 channels, or 1036 of 8
    w = inputs.custom(b, d, L, N, "bf16", seed=L + d)
    cpu = inputs.scan_inputs(w)
    if not gate:
        cpu["z"] = None
    dev = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    h0 = inputs.initial_state(b, d, N, seed=9, scale=0.25) if with_h0 else None
    kw = {}
    if form == "device-wide":
        kw = dict(workspace=torch.empty(binding.mamba_scan_workspace_size(b, d, L, N, torch.bfloat16), device="cuda",
                                        dtype=torch.uint8), schedule=binding.SCHEDULE_PERSISTENT, lanes_per_channel=lanes)
    else:
        kw = dict(schedule=binding.SCHEDULE_LOCAL, lanes_per_channel=lanes)
    out, last = binding.mamba_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                                       delta_bias=dev["delta_bias"], return_last_state=True,
                                       h0=None if h0 is None else h0.cuda(), **kw)
    torch.cuda.synchronize()
    ro, rs = oracle.scan(cpu["u"], cpu["delta"], cpu["A"], cpu["B"], cpu["C"], D=cpu["D"], z=cpu["z"],
                         delta_bias=cpu["delta_bias"], h0=h0)
    e1, e2 = rel_err(to_np(out), ro), rel_err(to_np(last), rs)
    record(f"many groups {b}x{d}x{L} lanes={lanes} {form} h0={with_h0} gate={gate}", out=e1, state=e2)
    assert e1 <= TOL[torch.bfloat16] and e2 <= TOL[torch.bfloat16], (e1, e2)
