"""Shapes with enough channel groups that no piece of the lane-pair kernel is
two-phase (the block-local form gives every block at least 5 whole
16-channel groups for its 8 warps, the device-wide form gives 1184 workers
at least 652 groups): the launch then takes the kernel's unrolled form.
Every output and final state against the fp64 oracle (GPU)."""
import pytest
import torch

import oracle
from parity import TOL, record, rel_err, to_np
from selective_state_space_20_b200 import binding, inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("form", ["block-local", "device-wide"])
@pytest.mark.parametrize("L,with_h0,gate", [(96, False, True), (104, True, True), (64, False, False)])
def test_many_groups_match_oracle(form, L, with_h0, gate):
    b, d, N = 4, 2960, 16  # 740 groups of 16 channels
    w = inputs.custom(b, d, L, N, "bf16", seed=L + d)
    cpu = inputs.scan_inputs(w)
    if not gate:
        cpu["z"] = None
    dev = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    h0 = inputs.initial_state(b, d, N, seed=9, scale=0.25) if with_h0 else None
    kw = {}
    if form == "device-wide":
        kw = dict(workspace=torch.empty(binding.mamba_scan_workspace_size(b, d, L, N, torch.bfloat16), device="cuda",
                                        dtype=torch.uint8), schedule=binding.SCHEDULE_PERSISTENT, lanes_per_channel=2)
    else:
        kw = dict(schedule=binding.SCHEDULE_LOCAL, lanes_per_channel=2)
    out, last = binding.mamba_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                                       delta_bias=dev["delta_bias"], return_last_state=True,
                                       h0=None if h0 is None else h0.cuda(), **kw)
    torch.cuda.synchronize()
    ro, rs = oracle.scan(cpu["u"], cpu["delta"], cpu["A"], cpu["B"], cpu["C"], D=cpu["D"], z=cpu["z"],
                         delta_bias=cpu["delta_bias"], h0=h0)
    e1, e2 = rel_err(to_np(out), ro), rel_err(to_np(last), rs)
    record(f"many groups {b}x{d}x{L} {form} h0={with_h0} gate={gate}", out=e1, state=e2)
    assert e1 <= TOL[torch.bfloat16] and e2 <= TOL[torch.bfloat16], (e1, e2)
