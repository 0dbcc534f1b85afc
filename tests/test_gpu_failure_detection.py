"""Failure detection and out-of-bounds writes without a GPU fault (GPU).

* A bounded wait that runs out: the library's test hook stops one channel
  group's pieces from publishing their carried state; the piece after them
  waits out its 2 s limit, raises the workspace's error word and stops, the
  rest of the launch completes, the host reads MAMBA_ERR_TIMEOUT, and the
  next launch on the same context and workspace is correct.
* Canary-guarded outputs: every output buffer of every entry point sits
  between guard regions filled with a canary value, and the guards must come
  back untouched (compute-sanitizer's out-of-bounds check is not available).
"""
import pytest
import torch

import oracle
from parity import TOL, rel_err, to_np
from selective_state_space_20_b200 import binding, inputs

pytestmark = pytest.mark.gpu

G = 4096  # guard elements on each side
CANARY = 12345.0


def test_stalled_carry_times_out_and_is_reported():
    w = inputs.custom(1, 64, 16384, 16, "bf16", seed=71)
    dev = inputs.scan_inputs(w, device="cuda")
    ws = torch.empty(binding.mamba_scan_workspace_size(w.batch, w.dim, w.seqlen, w.dstate), device="cuda",
                     dtype=torch.uint8)
    lib = binding.load_library()
    run = lambda: binding.mamba_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"],  # noqa: E731
                                         z=dev["z"], delta_bias=dev["delta_bias"], return_last_state=True,
                                         schedule=binding.SCHEDULE_PERSISTENT, lanes_per_channel=2,
                                         workspace=ws)
    prev = lib.mamba_debug_stall_group(0)
    try:
        run()
        status = binding.workspace_status(ws)
        device_status = binding.device_status()
    finally:
        lib.mamba_debug_stall_group(prev)
    assert status == binding.MAMBA_ERR_TIMEOUT and device_status == binding.MAMBA_ERR_TIMEOUT
    # the context and the workspace are fine: the next launch is complete and correct
    out, last = run()
    assert binding.workspace_status(ws) == 0 and binding.device_status() == 0
    rows = [0, 17, 63]
    cpu = {k: v for k, v in dev.items()}
    from parity import oracle_rows
    ro, rs = oracle_rows(cpu, rows)
    idx = torch.tensor(rows, device="cuda")
    assert rel_err(to_np(out.view(64, -1).index_select(0, idx)), ro) <= TOL[torch.bfloat16]


@pytest.mark.parametrize("lanes", [2, 4])
def test_local_schedule_stalled_carry_is_reported(lanes):
    """The local schedule (no workspace) keeps its carries in shared memory;
    when the hook stops group 0 from publishing, the next warp's bounded wait
    runs out, the library's device word reports it (once: reading clears it),
    and the next launch is complete and correct."""
    w = inputs.custom(1, 64, 16384, 16, "bf16", seed=76)  # few groups, long rows: split groups
    dev = inputs.scan_inputs(w, device="cuda")
    lib = binding.load_library()
    run = lambda: binding.mamba_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"],  # noqa: E731
                                         z=dev["z"], delta_bias=dev["delta_bias"], return_last_state=True,
                                         schedule=binding.SCHEDULE_LOCAL, lanes_per_channel=lanes)
    assert binding.device_status() == 0
    prev = lib.mamba_debug_stall_group(0)
    try:
        run()
        status = binding.device_status()
    finally:
        lib.mamba_debug_stall_group(prev)
    assert status == binding.MAMBA_ERR_TIMEOUT
    assert binding.device_status() == 0  # read once, cleared
    out, last = run()
    assert binding.device_status() == 0
    rows = [0, 17, 63]
    from parity import oracle_rows
    ro, rs = oracle_rows({k: v for k, v in dev.items()}, rows)
    idx = torch.tensor(rows, device="cuda")
    assert rel_err(to_np(out.view(64, -1).index_select(0, idx)), ro) <= TOL[torch.bfloat16]


def _guarded(shape, dtype, device="cuda", pinned=False):
    n = 1
    for s in shape:
        n *= s
    buf = torch.full((n + 2 * G,), CANARY, dtype=dtype, device=device)
    if pinned:
        buf = buf.pin_memory()
    return buf, buf[G:G + n].view(*shape)


def _intact(buf):
    head, tail = buf[:G], buf[-G:]
    return bool((head == CANARY).all()) and bool((tail == CANARY).all())


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("mode", ["persistent2", "persistent4", "persistent1", "local2", "local4", "static",
                                  "static_unaligned"])
def test_scan_writes_stay_inside(dtype, mode):
    b, d, L, N = 2, 70, 336, 16
    w = inputs.custom(b, d, L, N, dtype, seed=72)
    dev = inputs.scan_inputs(w, device="cuda")
    act = inputs.DTYPES[dtype]
    ob, out = _guarded((b, d, L), act)
    sb, last = _guarded((b, d, N), torch.float32)
    kw = {"persistent2": dict(schedule=binding.SCHEDULE_PERSISTENT, lanes_per_channel=2),
          "persistent4": dict(schedule=binding.SCHEDULE_PERSISTENT, lanes_per_channel=4),
          "persistent1": dict(schedule=binding.SCHEDULE_PERSISTENT, lanes_per_channel=1),
          "local2": dict(schedule=binding.SCHEDULE_LOCAL, lanes_per_channel=2),
          "local4": dict(schedule=binding.SCHEDULE_LOCAL, lanes_per_channel=4),
          "static": dict(schedule=binding.SCHEDULE_STATIC),
          "static_unaligned": dict(schedule=binding.SCHEDULE_STATIC)}[mode]
    if mode == "static_unaligned":  # out one element off 16 bytes: the element path
        ob = torch.full((b * d * L + 2 * G + 1,), CANARY, dtype=act, device="cuda")
        out = ob[G + 1:G + 1 + b * d * L].view(b, d, L)
        binding.mamba_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                               delta_bias=dev["delta_bias"], out=out, last_state=last, **kw)
        torch.cuda.synchronize()
        assert bool((ob[:G + 1] == CANARY).all()) and bool((ob[G + 1 + b * d * L:] == CANARY).all())
    else:
        binding.mamba_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"], z=dev["z"],
                               delta_bias=dev["delta_bias"], out=out, last_state=last, **kw)
        torch.cuda.synchronize()
        assert _intact(ob)
    assert _intact(sb)


def test_other_entry_points_write_inside():
    b, d, L, N = 2, 48, 256, 16
    w = inputs.custom(b, d, L, N, "bf16", seed=73)
    dev = inputs.scan_inputs(w, device="cuda")
    bf = torch.bfloat16
    # complex mode
    cx = inputs.complex_inputs(b, d, L, N, "bf16", seed=74, device="cuda")
    ob, out = _guarded((b, d, L), bf)
    sb, last = _guarded((b, d, N, 2), torch.float32)
    binding.mamba_scan_fwd_complex(cx["u"], cx["delta"], cx["A"], cx["B"], cx["C"], D=cx["D"], z=cx["z"],
                                   delta_bias=cx["delta_bias"], out=out, last_state=last)
    torch.cuda.synchronize()
    assert _intact(ob) and _intact(sb)
    # channel-contiguous strided output
    cl = {k: (v.transpose(1, 2).contiguous().transpose(1, 2) if k in ("u", "delta", "z", "B", "C") else v)
          for k, v in dev.items()}
    ob, flat = _guarded((b, L, d), bf)
    binding.mamba_scan_fwd_strided(cl["u"], cl["delta"], cl["A"], cl["B"], cl["C"], D=cl["D"], z=cl["z"],
                                   delta_bias=cl["delta_bias"], out=flat.transpose(1, 2))
    torch.cuda.synchronize()
    assert _intact(ob)
    # conv1d, and the conv fused into the scan (out and u)
    conv = inputs.conv_inputs(b, d, L, 4, "bf16", seed=75, device="cuda")
    ob, u = _guarded((b, d, L), bf)
    binding.mamba_conv1d_fwd(conv["xz"], conv["weight"], conv["bias"], dim=d, out=u)
    torch.cuda.synchronize()
    assert _intact(ob)
    ob, out = _guarded((b, d, L), bf)
    o2, u2 = binding.mamba_scan_fwd_conv(conv["xz"], conv["weight"], conv["bias"], dev["delta"], dev["A"], dev["B"],
                                         dev["C"], D=dev["D"], z=conv["xz"][:, d:], delta_bias=dev["delta_bias"],
                                         out=out, return_u=True)
    torch.cuda.synchronize()
    assert _intact(ob)
    # one decode step: the state in place and the output
    sb, state = _guarded((b, d, N), torch.float32)
    state.zero_()
    ob, y = _guarded((b, d), bf)
    binding.mamba_state_update(state, dev["u"][..., 0].contiguous(), dev["delta"][..., 0].contiguous(), dev["A"],
                               dev["B"][..., 0].contiguous(), dev["C"][..., 0].contiguous(), D=dev["D"],
                               z=dev["z"][..., 0].contiguous(), delta_bias=dev["delta_bias"], out=y)
    torch.cuda.synchronize()
    assert _intact(sb) and _intact(ob)
    # the host-memory scan's host output
    h = {k: dev[k].cpu().pin_memory() for k in ("u", "delta", "z", "B", "C")}
    ob, out_h = _guarded((b, d, L), bf, device="cpu", pinned=True)
    binding.mamba_scan_fwd_host(h["u"], h["delta"], dev["A"], h["B"], h["C"], D=dev["D"], z=h["z"],
                                delta_bias=dev["delta_bias"], out=out_h)
    torch.cuda.synchronize()
    assert _intact(ob)
