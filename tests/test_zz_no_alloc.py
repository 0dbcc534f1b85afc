"""mamba_scan_fwd_noalloc: the scan for callers that cannot allocate device
memory (a plugin or foreign-language host that only receives its input and
output buffers, or a process whose device memory belongs to a pooling
allocator).  It uses a fixed scratch area built into the library in place
of a caller workspace.

Called through the C ABI.  The same shape is run twice in a row and both
results must be bit-equal to the workspace entry point (mamba_scan_fwd_ws,
via the binding) on the same inputs -- it is the same kernel with the same
schedule -- and sampled rows must match the fp64 oracle within the parity
tolerance.  A call whose bounded wait ran out (the library's stall hook)
must be reported and must not leave anything behind for the next call, and
a call after the first must not consume device memory.  This file is
collected last so a stop-at-first-failure run has already run every other
test; it also passes on its own in a fresh process (the first call loads
the library's device code, which reserves the area).
"""
import ctypes

import pytest
import torch

from parity import TOL, oracle_rows, rel_err, sample_rows, to_np
from selective_state_space_20_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def call_noalloc(lib, ins, out, last):
    u = ins["u"]
    batch, dim, L = u.shape
    N = ins["A"].shape[1]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.mamba_scan_fwd_noalloc(
        _p(u), _p(ins["delta"]), _p(ins["A"]), _p(ins["B"]), _p(ins["C"]), _p(ins["D"]),
        _p(ins["z"]), _p(ins["delta_bias"]), 1, _p(out), _p(last), batch, dim, L, N,
        binding._ACT[u.dtype], stream)


def workspace_entry(ins):
    """mamba_scan_fwd_ws with a workspace of its own and automatic tuning --
    the call the scratch-area entry point makes with its scratch area."""
    batch, dim, L = ins["u"].shape
    N = ins["A"].shape[1]
    ws = torch.empty(binding.mamba_scan_workspace_size(batch, dim, L, N, ins["u"].dtype), device="cuda",
                     dtype=torch.uint8)
    return binding.mamba_scan_fwd(ins["u"], ins["delta"], ins["A"], ins["B"], ins["C"], D=ins["D"],
                                  z=ins["z"], delta_bias=ins["delta_bias"], return_last_state=True, workspace=ws)


def fresh_outputs(ins):
    batch, dim, _ = ins["u"].shape
    out = torch.full_like(ins["u"], float("nan"))
    last = torch.full((batch, dim, ins["A"].shape[1]), float("nan"), device=ins["u"].device)
    return out, last


@pytest.mark.parametrize("w", [inputs.custom(4, 5120, 512, 16, "bf16", seed=41),
                               inputs.custom(4, 5120, 256, 16, "fp32", seed=42),
                               inputs.custom(1, 2048, 4096, 16, "bf16", seed=43)],
                         ids=["bf16-4x5120x512", "fp32-4x5120x256", "bf16-1x2048x4096-two-phase"])
def test_noalloc_matches_workspace_entry_on_two_calls(w):
    lib = binding.load_library()
    # every shape has enough channel groups for the persistent schedule,
    # i.e. the path that uses the scratch area
    assert binding.mamba_scan_plan(w.batch, w.dim, w.seqlen, w.dstate,
                                   inputs.DTYPES[w.dtype])[2] == binding.SCHEDULE_PERSISTENT
    cpu = inputs.scan_inputs(w)
    ins = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    ref_out, ref_last = workspace_entry(ins)
    for _ in range(2):  # the same shape twice: the second call starts from the first's leftovers
        out, last = fresh_outputs(ins)
        assert call_noalloc(lib, ins, out, last) == 0
        torch.cuda.synchronize()
        assert binding.device_status() == 0
        assert torch.equal(out, ref_out) and torch.equal(last, ref_last)
    rows = sample_rows(w.batch, w.dim, 8, seed=w.seed)
    ro, rs = oracle_rows(cpu, rows)
    idx = torch.tensor(rows, device="cuda")
    tol = TOL[inputs.DTYPES[w.dtype]]
    assert rel_err(to_np(out.view(w.batch * w.dim, -1).index_select(0, idx)), ro) <= tol
    assert rel_err(to_np(last.view(w.batch * w.dim, -1).index_select(0, idx)), rs) <= tol


def test_noalloc_consumes_no_device_memory():
    lib = binding.load_library()
    w = inputs.custom(4, 5120, 512, 16, "bf16", seed=44)
    ins = inputs.scan_inputs(w, device="cuda")
    out, last = fresh_outputs(ins)
    assert call_noalloc(lib, ins, out, last) == 0  # loads the device code on a fresh process
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for _ in range(2):
        assert call_noalloc(lib, ins, out, last) == 0
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after >= free_before, (free_before, free_after)


def test_noalloc_recovers_after_a_timed_out_call():
    """The stall hook keeps channel group 0 from publishing its carried
    state, so the next piece's bounded wait (2 s) runs out: the scratch
    area's error word reports it.  The next call clears what the failed one
    left and is bit-equal to the workspace entry point."""
    lib = binding.load_library()
    w = inputs.custom(1, 2048, 16384, 16, "bf16", seed=45)  # few groups, long rows: split groups
    ins = inputs.scan_inputs(w, device="cuda")
    ref_out, ref_last = workspace_entry(ins)
    out, last = fresh_outputs(ins)
    prev = lib.mamba_debug_stall_group(0)
    try:
        assert call_noalloc(lib, ins, out, last) == 0
        status = binding.device_status()
    finally:
        lib.mamba_debug_stall_group(prev)
    assert status == binding.MAMBA_ERR_TIMEOUT
    out, last = fresh_outputs(ins)
    assert call_noalloc(lib, ins, out, last) == 0
    assert binding.device_status() == 0
    assert torch.equal(out, ref_out) and torch.equal(last, ref_last)


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = binding.load_library()
    # 256 x 5120 channels: 40960 groups of carried states, far beyond 4 MiB
    rc = lib.mamba_scan_fwd_noalloc(None, None, None, None, None, None, None, None, 1, None,
                                    None, 256, 5120, 64, 16, binding.MAMBA_BF16, None)
    assert rc == -8  # MAMBA_ERR_WORKSPACE, nothing enqueued
