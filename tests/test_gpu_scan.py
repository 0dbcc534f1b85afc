"""Parity of the CUDA scan with the fp64 oracle, through the C ABI (GPU)."""
import numpy as np
import pytest
import torch

import oracle
from parity import TOL, oracle_rows, record, rel_err, sample_rows, to_np
from selective_state_space_20_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def dev_inputs(ins, device="cuda"):
    return {k: (None if v is None else v.to(device)) for k, v in ins.items()}


def run_scan(ins, softplus=True, **kw):
    return binding.mamba_scan_fwd(ins["u"], ins["delta"], ins["A"], ins["B"], ins["C"],
                                  D=ins["D"], z=ins["z"], delta_bias=ins["delta_bias"],
                                  delta_softplus=softplus, return_last_state=True, **kw)


def oracle_full(ins, softplus=True):
    return oracle.scan(ins["u"], ins["delta"], ins["A"], ins["B"], ins["C"], D=ins["D"],
                       z=ins["z"], delta_bias=ins["delta_bias"], delta_softplus=softplus)


def check_full(w: inputs.ScanWorkload, softplus=True, drop=(), **kw):
    cpu = inputs.scan_inputs(w)
    for k in drop:
        cpu[k] = None
    if not softplus:  # the raw projections are negative; keep delta positive
        cpu["delta"] = cpu["delta"].abs() * 0.1
        if cpu["delta_bias"] is not None:
            cpu["delta_bias"] = cpu["delta_bias"].abs() * 0.01
    ins = dev_inputs(cpu)
    out, last = run_scan(ins, softplus=softplus, **kw)
    torch.cuda.synchronize()
    ro, rs = oracle_full(cpu, softplus=softplus)
    tol = TOL[inputs.DTYPES[w.dtype]]
    go, gs = to_np(out), to_np(last)
    e_out, e_state = rel_err(go, ro), rel_err(gs, rs)
    record(f"{w.name} {kw} drop={drop}", out=e_out, state=e_state,
           out_floor_0_1=rel_err(go, ro, floor=0.1), state_floor_0_1=rel_err(gs, rs, floor=0.1))
    assert e_out <= tol and e_state <= tol, (w.name, kw, e_out, e_state)
    return e_out, e_state


def test_tiny_fp32_workload():
    e = check_full(inputs.TINY_FP32)
    print("tiny fp32", e)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 70, 333), (3, 37, 129), (1, 1, 1), (1, 5, 7), (2, 9, 64),
                                   (1, 3, 1000), (5, 130, 96)])
def test_shapes_span_tiles_and_ragged_tails(dtype, shape):
    b, d, L = shape
    check_full(inputs.custom(b, d, L, 16, dtype, seed=hash(shape) % 1000))


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("L", [1, 3, 7, 9])
@pytest.mark.parametrize("dstate", [1, 2])
def test_tiny_odd_lengths_and_states(dtype, L, dstate):
    # every schedule the planner may pick for these (static, and persistent where L allows)
    check_full(inputs.custom(2, 33, L, dstate, dtype, seed=L * 10 + dstate))


@pytest.mark.parametrize("dstate", [1, 2, 3, 5, 8, 13, 16, 17, 24, 32, 33, 40, 64])
def test_every_dstate(dstate):
    check_full(inputs.custom(2, 19, 100, dstate, "fp32", seed=dstate))
    check_full(inputs.custom(2, 19, 104, dstate, "bf16", seed=dstate + 100))


@pytest.mark.parametrize("dstate", [16, 24, 32, 64])
@pytest.mark.parametrize("seed", [0, 1, 2, 3, 4])
def test_fp32_large_dstate_several_seeds(dstate, seed):
    """fp32 at the 1e-4 bar with the fast-decaying states of A = -(n + 1) up
    to n = 63 (decay exponents down to ~-20 per step), five seeds each, on
    the tiny workload's shape and its distributions."""
    check_full(inputs.custom(1, 64, 256, dstate, "fp32", seed=1000 * dstate + seed, d_mode="ones"))
    check_full(inputs.custom(2, 40, 256, dstate, "fp32", seed=2000 * dstate + seed))


def _lane_configs():
    cfg = []
    for np_, lanes in ((8, (1, 2, 4, 8)), (16, (1, 2, 4, 8, 16)), (32, (2, 4, 8, 16)), (64, (4, 8, 16))):
        for r in lanes:
            for th in (128, 256):
                cfg.append((np_, r, th))
    return cfg


@pytest.mark.parametrize("np_,lanes,threads", _lane_configs())
def test_every_kernel_variant(np_, lanes, threads):
    for dtype in ("fp32", "bf16"):
        check_full(inputs.custom(2, 45, 200, np_, dtype, seed=np_ + lanes), lanes_per_channel=lanes,
                   threads_per_block=threads)


@pytest.mark.parametrize("drop", [("z",), ("D",), ("delta_bias",), ("z", "D", "delta_bias")])
def test_optional_inputs(drop):
    for dtype in ("fp32", "bf16"):
        check_full(inputs.custom(2, 33, 150, 16, dtype, seed=7), drop=drop)


def test_softplus_off():
    w = inputs.custom(2, 33, 150, 16, "fp32", seed=8)
    cpu = inputs.scan_inputs(w)
    cpu["delta"] = cpu["delta"].abs() * 0.1  # keep delta positive without softplus
    cpu["delta_bias"] = torch.zeros_like(cpu["delta_bias"])
    ins = dev_inputs(cpu)
    out, last = run_scan(ins, softplus=False)
    ro, rs = oracle_full(cpu, softplus=False)
    assert rel_err(to_np(out), ro) <= 1e-4 and rel_err(to_np(last), rs) <= 1e-4


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_misaligned_pointers_take_scalar_path(dtype):
    w = inputs.custom(2, 21, 96, 16, dtype, seed=9)
    cpu = inputs.scan_inputs(w)
    ins = {}
    for k, v in cpu.items():
        if v is None:
            ins[k] = None
            continue
        buf = torch.empty(v.numel() + 1, dtype=v.dtype, device="cuda")
        t = buf[1:].view(v.shape)  # storage offset of one element
        t.copy_(v)
        ins[k] = t
    assert ins["u"].data_ptr() % 16 != 0
    out, last = run_scan(ins)
    ro, rs = oracle_full(cpu)
    tol = TOL[inputs.DTYPES[dtype]]
    assert rel_err(to_np(out), ro) <= tol and rel_err(to_np(last), rs) <= tol


@pytest.mark.parametrize("alias", ["u", "delta", "z"])
def test_in_place_output(alias):
    w = inputs.custom(2, 40, 256, 16, "bf16", seed=10)
    cpu = inputs.scan_inputs(w)
    ins = dev_inputs(cpu)
    out, _ = run_scan(ins, out=ins[alias])
    assert out.data_ptr() == ins[alias].data_ptr()
    ro, _ = oracle_full(cpu)
    assert rel_err(to_np(out), ro) <= 2e-2


def test_deterministic():
    w = inputs.custom(4, 300, 512, 16, "bf16", seed=11)
    ins = dev_inputs(inputs.scan_inputs(w))
    o1, s1 = run_scan(ins)
    o2, s2 = run_scan(ins)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_runs_on_a_side_stream():
    w = inputs.custom(2, 64, 512, 16, "bf16", seed=12)
    cpu = inputs.scan_inputs(w)
    ins = dev_inputs(cpu)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        out, last = run_scan(ins)
    s.synchronize()
    ro, rs = oracle_full(cpu)
    assert rel_err(to_np(out), ro) <= 2e-2 and rel_err(to_np(last), rs) <= 2e-2


def test_auto_plan_is_valid():
    for w in (inputs.TINY_FP32, inputs.MAMBA_130M, inputs.MAMBA_2_8B, inputs.LONG_CONTEXT):
        lanes, threads, sched = binding.mamba_scan_plan(w.batch, w.dim, w.seqlen, w.dstate,
                                                        inputs.DTYPES[w.dtype])
        assert lanes in (1, 2, 4, 8, 16) and threads in (128, 256) and sched in (1, 2)
    # the Mamba-2.8B layer has enough channel groups for the persistent schedule
    w = inputs.MAMBA_2_8B
    assert binding.mamba_scan_plan(w.batch, w.dim, w.seqlen, w.dstate)[2] == binding.SCHEDULE_PERSISTENT
    # the long-context layer has few groups but long sequences: two-phase pieces
    w = inputs.LONG_CONTEXT
    assert binding.mamba_scan_plan(w.batch, w.dim, w.seqlen, w.dstate)[:3:2] == (2, binding.SCHEDULE_PERSISTENT)


# ------------------------------------------------------------ persistent schedule
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape", [(1, 32, 64), (2, 70, 336), (3, 33, 1000), (1, 1, 8),
                                   (4, 100, 2048), (2, 64, 4096)])
@pytest.mark.parametrize("dstate", [16, 5])
@pytest.mark.parametrize("lanes", [1, 2, 4])
def test_persistent_schedule(dtype, shape, dstate, lanes):
    b, d, L = shape
    w = inputs.custom(b, d, L, dstate, dtype, seed=b * 1000 + d + L + dstate)
    cpu = inputs.scan_inputs(w)
    ins = dev_inputs(cpu)
    nbytes = binding.mamba_scan_workspace_size(b, d, L, dstate, inputs.DTYPES[dtype])
    assert nbytes > 0
    ws = torch.full((nbytes,), 0x5A, device="cuda", dtype=torch.uint8)  # garbage-filled
    out, last = run_scan(ins, schedule=binding.SCHEDULE_PERSISTENT, lanes_per_channel=lanes, workspace=ws)
    assert binding.workspace_status(ws) == 0
    ro, rs = oracle_full(cpu)
    tol = TOL[inputs.DTYPES[dtype]]
    e1, e2 = rel_err(to_np(out), ro), rel_err(to_np(last), rs)
    record(f"persistent lanes={lanes} {w.name}", out=e1, state=e2)
    assert e1 <= tol and e2 <= tol, (e1, e2)
    # same workspace again (state of the previous launch must not leak in)
    out2, last2 = run_scan(ins, schedule=binding.SCHEDULE_PERSISTENT, lanes_per_channel=lanes, workspace=ws)
    assert torch.equal(out, out2) and torch.equal(last, last2)


@pytest.mark.parametrize("lanes", [1, 2, 4])
def test_persistent_matches_static_schedule(lanes):
    w = inputs.custom(4, 640, 1024, 16, "bf16", seed=31)
    ins = dev_inputs(inputs.scan_inputs(w))
    o1, s1 = run_scan(ins, schedule=binding.SCHEDULE_PERSISTENT, lanes_per_channel=lanes)
    o2, s2 = run_scan(ins, schedule=binding.SCHEDULE_STATIC)
    assert rel_err(to_np(o1), to_np(o2)) <= 2e-2
    # bf16 runs of two schedules (the persistent one may cut rows into pieces
    # combined through exp(A sum(delta))): their fp32 states agree well inside
    # the bf16 bar each one meets against the oracle
    assert rel_err(to_np(s1), to_np(s2)) <= 1e-3


@pytest.mark.parametrize("lanes", [1, 2, 4])
@pytest.mark.parametrize("drop,softplus", [(("z",), True), (("D", "delta_bias"), True), ((), False),
                                           (("z", "D", "delta_bias"), False)])
def test_persistent_optional_inputs(lanes, drop, softplus):
    for dtype in ("fp32", "bf16"):
        check_full(inputs.custom(2, 33, 152, 16, dtype, seed=17), softplus=softplus, drop=drop,
                   schedule=binding.SCHEDULE_PERSISTENT, lanes_per_channel=lanes)


@pytest.mark.parametrize("lanes", [1, 2, 4])
@pytest.mark.parametrize("chunk", [64, 200, 4096])
def test_persistent_short_units(lanes, chunk):
    # few channel groups and many short time chunks: most claimed units are
    # not ready when claimed, so the workers mostly wait on one another
    check_full(inputs.custom(2, 96, 2048, 16, "bf16", seed=chunk + lanes),
               schedule=binding.SCHEDULE_PERSISTENT, lanes_per_channel=lanes, chunk_timesteps=chunk)


@pytest.mark.parametrize("lanes", [2, 4])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape", [(1, 64, 16384), (1, 16, 16384), (2, 40, 6000)])
def test_persistent_few_groups_long_sequences(lanes, dtype, shape):
    # fewer channel groups than workers: every group is cut into many pieces
    # that run at once (each from its own end state, then corrected by the
    # carry of the piece before it)
    b, d, L = shape
    check_full(inputs.custom(b, d, L, 16, dtype, seed=d + L), schedule=binding.SCHEDULE_PERSISTENT,
               lanes_per_channel=lanes)


# ------------------------------------------------------------ local schedule
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape", [(1, 32, 64), (2, 70, 336), (3, 33, 1000), (1, 1, 8),
                                   (4, 100, 2048), (2, 64, 4096), (4, 1030, 256)])
@pytest.mark.parametrize("dstate", [16, 5])
@pytest.mark.parametrize("lanes", [2, 4])
def test_local_schedule(dtype, shape, dstate, lanes):
    """No workspace: one block per SM splits whole channel groups among its
    warps (few groups per block: two-phase pieces; many: chained pieces)."""
    b, d, L = shape
    w = inputs.custom(b, d, L, dstate, dtype, seed=b * 1000 + d + L + dstate + 7)
    cpu = inputs.scan_inputs(w)
    ins = dev_inputs(cpu)
    out, last = run_scan(ins, schedule=binding.SCHEDULE_LOCAL, lanes_per_channel=lanes)
    assert binding.device_status() == 0
    ro, rs = oracle_full(cpu)
    tol = TOL[inputs.DTYPES[dtype]]
    e1, e2 = rel_err(to_np(out), ro), rel_err(to_np(last), rs)
    record(f"local lanes={lanes} {w.name}", out=e1, state=e2)
    assert e1 <= tol and e2 <= tol, (e1, e2)
    out2, last2 = run_scan(ins, schedule=binding.SCHEDULE_LOCAL, lanes_per_channel=lanes)
    assert torch.equal(out, out2) and torch.equal(last, last2)


@pytest.mark.parametrize("lanes", [2, 4])
@pytest.mark.parametrize("drop,softplus", [(("z",), True), (("D", "delta_bias"), True), ((), False)])
def test_local_optional_inputs(lanes, drop, softplus):
    for dtype in ("fp32", "bf16"):
        check_full(inputs.custom(2, 33, 152, 16, dtype, seed=19), softplus=softplus, drop=drop,
                   schedule=binding.SCHEDULE_LOCAL, lanes_per_channel=lanes)


@pytest.mark.parametrize("lanes", [2, 4])
def test_local_from_an_initial_state(lanes):
    for dtype in ("fp32", "bf16"):
        w = inputs.custom(2, 96, 1024, 16, dtype, seed=23)
        cpu = inputs.scan_inputs(w)
        h0 = inputs.initial_state(2, 96, 16, seed=24)
        ins = dev_inputs(cpu)
        out, last = binding.mamba_scan_fwd(ins["u"], ins["delta"], ins["A"], ins["B"], ins["C"], D=ins["D"],
                                           z=ins["z"], delta_bias=ins["delta_bias"], return_last_state=True,
                                           h0=h0.cuda(), schedule=binding.SCHEDULE_LOCAL, lanes_per_channel=lanes)
        ro, rs = oracle.scan(cpu["u"], cpu["delta"], cpu["A"], cpu["B"], cpu["C"], D=cpu["D"], z=cpu["z"],
                             delta_bias=cpu["delta_bias"], h0=h0)
        tol = TOL[inputs.DTYPES[dtype]]
        assert rel_err(to_np(out), ro) <= tol and rel_err(to_np(last), rs) <= tol


def test_local_matches_device_wide_persistent():
    """Where no piece of a group is split in either form (as many groups as
    workers would take, every warp a whole number of groups) the two forms run
    identical arithmetic: 148 SMs x 8 warps = 1184 groups of 16 channels."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    w = inputs.custom(2, 16 * 8 * sms // 2, 512, 16, "bf16", seed=25)
    ins = dev_inputs(inputs.scan_inputs(w))
    o1, s1 = run_scan(ins, schedule=binding.SCHEDULE_LOCAL, lanes_per_channel=2)
    o2, s2 = run_scan(ins, schedule=binding.SCHEDULE_PERSISTENT, lanes_per_channel=2)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_default_call_takes_the_local_schedule():
    """mamba_scan_fwd (no workspace) on the Mamba-2.8B layer runs the local
    schedule; through the C ABI entry point itself, sampled rows vs the oracle."""
    w = inputs.MAMBA_2_8B
    cpu = inputs.scan_inputs(w)
    ins = dev_inputs(cpu)
    out, last = run_scan(ins)
    torch.cuda.synchronize()
    assert binding.device_status() == 0
    rows = sample_rows(w.batch, w.dim, 24, seed=3)
    ro, rs = oracle_rows(cpu, rows)
    idx = torch.tensor(rows, device="cuda")
    assert rel_err(to_np(out.view(-1, w.seqlen).index_select(0, idx)), ro) <= TOL[torch.bfloat16]
    assert rel_err(to_np(last.view(-1, w.dstate).index_select(0, idx)), rs) <= TOL[torch.bfloat16]


def test_persistent_rejects_unsupported():
    w = inputs.custom(1, 32, 64, 32, "bf16", seed=1)  # dstate 32 > 16
    ins = dev_inputs(inputs.scan_inputs(w))
    with pytest.raises(binding.MambaError):
        run_scan(ins, schedule=binding.SCHEDULE_PERSISTENT)
    w = inputs.custom(1, 32, 60, 16, "bf16", seed=1)  # L not a multiple of 8
    ins = dev_inputs(inputs.scan_inputs(w))
    with pytest.raises(binding.MambaError):
        run_scan(ins, schedule=binding.SCHEDULE_PERSISTENT)


# ------------------------------------------------------------ full sizes
def check_sampled(w: inputs.ScanWorkload, k: int):
    """Full-size launch (the one the benchmark times); every output and final
    state of k sampled (batch, channel) rows against the oracle, plus finite
    checks on everything."""
    cpu = inputs.scan_inputs(w)
    ins = dev_inputs(cpu)
    out, last = run_scan(ins)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(last).all()
    rows = sample_rows(w.batch, w.dim, k, seed=w.seed)
    ro, rs = oracle_rows(cpu, rows)
    flat_out = out.view(w.batch * w.dim, w.seqlen)
    flat_st = last.view(w.batch * w.dim, w.dstate)
    idx = torch.tensor(rows, device=out.device)
    go = to_np(flat_out.index_select(0, idx))
    gs = to_np(flat_st.index_select(0, idx))
    tol = TOL[inputs.DTYPES[w.dtype]]
    e_out, e_state = rel_err(go, ro), rel_err(gs, rs)
    record(f"{w.name} sampled {len(rows)} rows", out=e_out, state=e_state)
    assert e_out <= tol and e_state <= tol
    return e_out, e_state


def test_mamba_130m_layer_full_size():
    check_sampled(inputs.MAMBA_130M, 48)


def test_mamba_2_8b_layer_full_size():
    check_sampled(inputs.MAMBA_2_8B, 48)


def test_long_context_full_size():
    check_sampled(inputs.LONG_CONTEXT, 12)


def test_scan_then_steps_continue_the_sequence():
    """Scan over [0, L1), then one state update per remaining token, equals a
    single scan over [0, L) -- the resume path used by generation."""
    w = inputs.custom(3, 50, 300, 16, "bf16", seed=13)
    cpu = inputs.scan_inputs(w)
    ins = dev_inputs(cpu)
    full, last = run_scan(ins)
    L1 = 211
    head = {k: (v[..., :L1].contiguous() if k in ("u", "delta", "z", "B", "C") else v) for k, v in ins.items()}
    o1, state = run_scan(head)
    assert torch.equal(o1, full[..., :L1]) or rel_err(to_np(o1), to_np(full[..., :L1])) <= 2e-2
    outs = []
    for t in range(L1, w.seqlen):
        outs.append(binding.mamba_state_update(state, ins["u"][..., t].contiguous(),
                                               ins["delta"][..., t].contiguous(), ins["A"],
                                               ins["B"][..., t].contiguous(), ins["C"][..., t].contiguous(),
                                               D=ins["D"], z=ins["z"][..., t].contiguous(),
                                               delta_bias=ins["delta_bias"]))
    tail = torch.stack(outs, dim=-1)
    ro, rs = oracle_full(cpu)
    assert rel_err(to_np(tail), ro[..., L1:]) <= 2e-2
    assert rel_err(to_np(state), rs) <= 2e-2
    assert rel_err(to_np(tail), to_np(full[..., L1:])) <= 2e-2


def test_past_32_bit_indexing():
    """4 x 5120 x 131072 bf16: 2.7 G elements per tensor, past 2^31, so every
    row offset of the lane-split kernel needs 64-bit arithmetic; sampled rows
    at both ends of the address range against the oracle."""
    w = inputs.custom(4, 5120, 131072, 16, "bf16", seed=61, name="4x5120x131072 bf16")
    assert w.batch * w.dim * w.seqlen > 2 ** 31
    dev = inputs.scan_inputs(w, device="cuda")
    out, last = run_scan(dev)
    torch.cuda.synchronize()
    rows = [0, 1, 5119, 5120 * 2 + 77, 5120 * 3, 5120 * 4 - 1]
    cpu = {k: (None if v is None else v) for k, v in dev.items()}
    ro, rs = oracle_rows(cpu, rows)
    flat_out = out.view(w.batch * w.dim, w.seqlen)
    flat_st = last.view(w.batch * w.dim, w.dstate)
    idx = torch.tensor(rows, device=out.device)
    e_out = rel_err(to_np(flat_out.index_select(0, idx)), ro)
    e_state = rel_err(to_np(flat_st.index_select(0, idx)), rs)
    record("4x5120x131072 bf16 sampled rows", out=e_out, state=e_state)
    assert e_out <= TOL[torch.bfloat16] and e_state <= TOL[torch.bfloat16]


@pytest.mark.parametrize("sched,lanes", [(binding.SCHEDULE_STATIC, 0), (binding.SCHEDULE_PERSISTENT, 1),
                                         (binding.SCHEDULE_PERSISTENT, 2), (binding.SCHEDULE_PERSISTENT, 4)])
def test_zero_step_keeps_the_state(sched, lanes):
    """delta = 0 (softplus off, no bias): Abar = 1 and no input, so the state
    stays h0 bit for bit and y_t = C_t . h0 + D u_t (the oracle's pin, on
    the GPU)."""
    w = inputs.custom(2, 48, 256, 16, "fp32", seed=62)
    cpu = inputs.scan_inputs(w)
    cpu["delta"] = torch.zeros_like(cpu["delta"])
    cpu["delta_bias"] = None
    cpu["z"] = None
    dev = dev_inputs(cpu)
    h0 = inputs.initial_state(2, 48, 16, seed=5)
    out, last = binding.mamba_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"],
                                       delta_softplus=False, return_last_state=True, h0=h0.cuda(), schedule=sched,
                                       lanes_per_channel=lanes)
    torch.cuda.synchronize()
    assert torch.equal(last.cpu(), h0)
    y = torch.einsum("bdn,bnl->bdl", h0.double(), cpu["C"].double()) + cpu["D"].double()[None, :, None] * cpu["u"].double()
    assert rel_err(to_np(out), y.numpy()) <= 1e-4


def test_memoryless_limit():
    """A very negative: Abar underflows to 0 and h_t = delta_t B_t u_t, so
    y_t = delta_t u_t (C_t . B_t) + D u_t -- a closed form without the
    recurrence."""
    w = inputs.custom(2, 40, 200, 16, "fp32", seed=63)
    cpu = inputs.scan_inputs(w)
    cpu["A"] = torch.full_like(cpu["A"], -1e7)  # delta A log2 e < -126 for every delta
    cpu["z"] = None
    dev = dev_inputs(cpu)
    out, last = binding.mamba_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"],
                                       delta_bias=dev["delta_bias"], return_last_state=True)
    torch.cuda.synchronize()
    dl = torch.nn.functional.softplus(cpu["delta"].double() + cpu["delta_bias"].double()[None, :, None])
    cb = (cpu["C"].double() * cpu["B"].double()).sum(1)  # (batch, L)
    y = dl * cpu["u"].double() * cb[:, None, :] + cpu["D"].double()[None, :, None] * cpu["u"].double()
    assert rel_err(to_np(out), y.numpy()) <= 1e-4
