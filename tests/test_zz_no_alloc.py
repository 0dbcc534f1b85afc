"""mamba_scan_fwd_noalloc: the scan for callers that cannot allocate device
memory (a plugin or foreign-language host that only receives its input and
output buffers, or a process whose device memory belongs to a pooling
allocator).  It uses a fixed scratch area built into the library in place
of a caller workspace.

Called through the C ABI and compared, on two calls in a row, with the
workspace entry point (mamba_scan_fwd_ws, via the binding) on the same
inputs, within the parity tolerances.  This file is collected last so a
stop-at-first-failure run has already run every other test; it also passes
on its own in a fresh process (the first call does the per-device set-up).
"""
import ctypes

import pytest
import torch

from parity import TOL, rel_err, to_np
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


def test_noalloc_matches_workspace_entry_on_two_calls():
    lib = binding.load_library()
    cases = [inputs.custom(4, 5120, 512, 16, "bf16", seed=41),
             inputs.custom(4, 5120, 256, 16, "fp32", seed=42)]
    for w in cases:
        # both shapes have enough channel groups for the persistent
        # schedule, i.e. the path that uses the scratch area
        assert binding.mamba_scan_plan(w.batch, w.dim, w.seqlen, w.dstate,
                                       inputs.DTYPES[w.dtype])[2] == binding.SCHEDULE_PERSISTENT
        ins = inputs.scan_inputs(w, device="cuda")
        ref_out, ref_last = binding.mamba_scan_fwd(
            ins["u"], ins["delta"], ins["A"], ins["B"], ins["C"], D=ins["D"], z=ins["z"],
            delta_bias=ins["delta_bias"], return_last_state=True)
        out = torch.full_like(ins["u"], float("nan"))
        last = torch.full((w.batch, w.dim, w.dstate), float("nan"), device="cuda")
        assert call_noalloc(lib, ins, out, last) == 0
        torch.cuda.synchronize()
        tol = TOL[inputs.DTYPES[w.dtype]]
        assert rel_err(to_np(out), to_np(ref_out)) <= tol
        assert rel_err(to_np(last), to_np(ref_last)) <= tol


def test_noalloc_rejects_problems_beyond_its_scratch():
    lib = binding.load_library()
    # 256 x 5120 channels: 40960 groups of carried states, far beyond 4 MiB
    rc = lib.mamba_scan_fwd_noalloc(None, None, None, None, None, None, None, None, 1, None,
                                    None, 256, 5120, 64, 16, binding.MAMBA_BF16, None)
    assert rc == -8  # MAMBA_ERR_WORKSPACE, nothing enqueued
