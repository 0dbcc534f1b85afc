"""The scan started from a given state h0 instead of zeros, through the C ABI,
against the fp64 oracle run from the same state (GPU)."""
import pytest
import torch

import oracle
from parity import TOL, record, rel_err, to_np
from selective_state_space_20_b200 import binding, inputs

pytestmark = pytest.mark.gpu

SEQ = ("u", "delta", "z", "B", "C")


def _dev(ins):
    return {k: (None if v is None else v.cuda()) for k, v in ins.items()}


def _run(ins, h0, **kw):
    return binding.mamba_scan_fwd(ins["u"], ins["delta"], ins["A"], ins["B"], ins["C"],
                                  D=ins["D"], z=ins["z"], delta_bias=ins["delta_bias"],
                                  return_last_state=True, h0=h0, **kw)


def _check(w, seed=7, scale=0.25, **kw):
    cpu = inputs.scan_inputs(w)
    h0 = inputs.initial_state(w.batch, w.dim, w.dstate, seed=seed, scale=scale)
    out, last = _run(_dev(cpu), h0.cuda(), **kw)
    torch.cuda.synchronize()
    ro, rs = oracle.scan(cpu["u"], cpu["delta"], cpu["A"], cpu["B"], cpu["C"], D=cpu["D"],
                         z=cpu["z"], delta_bias=cpu["delta_bias"], h0=h0)
    tol = TOL[inputs.DTYPES[w.dtype]]
    e1, e2 = rel_err(to_np(out), ro), rel_err(to_np(last), rs)
    record(f"h0 {w.name} {kw}", out=e1, state=e2)
    assert e1 <= tol and e2 <= tol, (w.name, kw, e1, e2)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape,dstate", [((2, 70, 333), 16), ((1, 5, 7), 3), ((3, 37, 129), 17),
                                          ((2, 9, 64), 64), ((1, 1, 1), 16)])
def test_static_schedule_from_a_state(dtype, shape, dstate):
    b, d, L = shape
    _check(inputs.custom(b, d, L, dstate, dtype, seed=L + dstate), schedule=binding.SCHEDULE_STATIC)


@pytest.mark.parametrize("lanes", [1, 2, 4])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape,dstate", [((2, 70, 336), 16), ((3, 33, 1000), 5), ((1, 1, 8), 16)])
def test_persistent_schedule_from_a_state(lanes, dtype, shape, dstate):
    b, d, L = shape
    _check(inputs.custom(b, d, L, dstate, dtype, seed=d + L), schedule=binding.SCHEDULE_PERSISTENT,
           lanes_per_channel=lanes)


@pytest.mark.parametrize("lanes", [2, 4])
@pytest.mark.parametrize("shape", [(1, 64, 16384), (1, 16, 16384), (2, 40, 6000)])
def test_split_groups_from_a_state(lanes, shape):
    # groups cut into pieces that run at once: only the first piece of each
    # group starts from h0; the others take it through the carry
    b, d, L = shape
    _check(inputs.custom(b, d, L, 16, "bf16", seed=d + L), schedule=binding.SCHEDULE_PERSISTENT,
           lanes_per_channel=lanes)


@pytest.mark.parametrize("sched,lanes", [(binding.SCHEDULE_STATIC, 0), (binding.SCHEDULE_PERSISTENT, 2)])
def test_large_initial_state(sched, lanes):
    # a state 8x the settled spread: its decay dominates the first outputs
    _check(inputs.custom(2, 64, 1024, 16, "bf16", seed=23), scale=2.0, schedule=sched,
           lanes_per_channel=lanes)


@pytest.mark.parametrize("lanes", [1, 2, 4])
def test_short_units_from_a_state(lanes):
    _check(inputs.custom(2, 96, 2048, 16, "bf16", seed=5), schedule=binding.SCHEDULE_PERSISTENT,
           lanes_per_channel=lanes, chunk_timesteps=200)


def test_zero_state_equals_the_plain_scan():
    w = inputs.custom(2, 64, 512, 16, "bf16", seed=3)
    ins = _dev(inputs.scan_inputs(w))
    zero = torch.zeros(w.batch, w.dim, w.dstate, device="cuda")
    for sched in (binding.SCHEDULE_STATIC, binding.SCHEDULE_PERSISTENT):
        o1, s1 = _run(ins, zero, schedule=sched)
        o2, s2 = _run(ins, None, schedule=sched)
        assert torch.equal(o1, o2) and torch.equal(s1, s2), sched


@pytest.mark.parametrize("sched,lanes", [(binding.SCHEDULE_STATIC, 0), (binding.SCHEDULE_PERSISTENT, 1),
                                         (binding.SCHEDULE_PERSISTENT, 2), (binding.SCHEDULE_PERSISTENT, 4)])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_two_scans_chain_into_one(sched, lanes, dtype):
    """Scanning [0, L1) and then [L1, L) from the first part's last state
    equals one scan over [0, L): outputs and final state."""
    w = inputs.custom(2, 80, 2048, 16, dtype, seed=11)
    ins = _dev(inputs.scan_inputs(w))
    kw = dict(schedule=sched, lanes_per_channel=lanes)
    full, last = _run(ins, None, **kw)
    L1 = 1024 + 8 * 37
    head = {k: (v[..., :L1].contiguous() if k in SEQ else v) for k, v in ins.items()}
    tail = {k: (v[..., L1:].contiguous() if k in SEQ else v) for k, v in ins.items()}
    o1, s1 = _run(head, None, **kw)
    o2, s2 = _run(tail, s1, **kw)
    tol = TOL[inputs.DTYPES[dtype]]
    e_out = rel_err(to_np(torch.cat([o1, o2], dim=-1)), to_np(full))
    e_state = rel_err(to_np(s2), to_np(last))
    record(f"chain {w.name} sched={sched} lanes={lanes}", out=e_out, state=e_state)
    assert e_out <= tol and e_state <= 1e-4, (e_out, e_state)


@pytest.mark.parametrize("sched,lanes", [(binding.SCHEDULE_STATIC, 0), (binding.SCHEDULE_PERSISTENT, 1),
                                         (binding.SCHEDULE_PERSISTENT, 2), (binding.SCHEDULE_PERSISTENT, 4)])
def test_state_advances_in_place(sched, lanes):
    w = inputs.custom(2, 40, 6000, 16, "bf16", seed=19)
    ins = _dev(inputs.scan_inputs(w))
    h0 = inputs.initial_state(w.batch, w.dim, w.dstate, seed=2).cuda()
    o1, s1 = _run(ins, h0, schedule=sched, lanes_per_channel=lanes)
    state = h0.clone()
    o2, s2 = _run(ins, state, last_state=state, schedule=sched, lanes_per_channel=lanes)
    assert s2.data_ptr() == state.data_ptr()
    assert torch.equal(o1, o2) and torch.equal(s1, state)


def test_initial_state_validation():
    w = inputs.custom(1, 8, 64, 16, "bf16", seed=1)
    ins = _dev(inputs.scan_inputs(w))
    with pytest.raises(ValueError):
        _run(ins, torch.zeros(1, 8, 15, device="cuda"))
    with pytest.raises(TypeError):
        _run(ins, torch.zeros(1, 8, 16, device="cuda", dtype=torch.bfloat16))
    out = torch.empty_like(ins["u"])
    h0 = out.view(-1).view(torch.float32)[:128].view(1, 8, 16)  # inside out
    with pytest.raises(binding.MambaError):
        _run(ins, h0, out=out)
