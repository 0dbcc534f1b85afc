"""The scan on strided tensors -- (batch, L, dim) activations, slices of
projection outputs, broadcast B / C -- through the C ABI, against the fp64
oracle on the same values laid out densely (GPU)."""
import pytest
import torch

import oracle
from parity import TOL, oracle_rows, record, rel_err, sample_rows, to_np
from selective_state_space_20_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def _oracle(cpu, softplus=True, h0=None):
    dense = {k: (None if v is None else v.contiguous()) for k, v in cpu.items()}
    return oracle.scan(dense["u"], dense["delta"], dense["A"], dense["B"], dense["C"], D=dense["D"],
                       z=dense["z"], delta_bias=dense["delta_bias"], delta_softplus=softplus, h0=h0)


def _channels_last(t):
    """The same values as a (batch, L, rows) tensor viewed as (batch, rows, L)."""
    return t.transpose(1, 2).contiguous().transpose(1, 2)


def _run(dev, **kw):
    return binding.mamba_scan_fwd_strided(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"],
                                          z=dev["z"], delta_bias=dev["delta_bias"], return_last_state=True,
                                          **kw)


def _check(name, cpu, dev, dtype, h0=None, **kw):
    out, last = _run(dev, h0=None if h0 is None else h0.cuda(), **kw)
    torch.cuda.synchronize()
    ro, rs = _oracle(cpu, h0=h0)
    tol = TOL[inputs.DTYPES[dtype]]
    e1, e2 = rel_err(to_np(out), ro), rel_err(to_np(last), rs)
    record(f"strided {name}", out=e1, state=e2)
    assert e1 <= tol and e2 <= tol, (name, e1, e2)
    return out, last


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape,dstate", [((2, 64, 333), 16), ((3, 40, 129), 16), ((1, 37, 100), 16),
                                          ((2, 96, 64), 8), ((1, 16, 1), 16), ((2, 24, 77), 5)])
@pytest.mark.parametrize("lanes", [0, 1, 4])
def test_channels_last_activations(dtype, shape, dstate, lanes):
    b, d, L = shape
    w = inputs.custom(b, d, L, dstate, dtype, seed=d + L + dstate)
    cpu = inputs.scan_inputs(w)
    cl = {k: (_channels_last(v) if k in ("u", "delta", "z", "B", "C") else v) for k, v in cpu.items()}
    dev = {k: (None if v is None else v.cuda()) for k, v in cl.items()}
    # .cuda() keeps the strides of a non-contiguous view
    assert L == 1 or dev["u"].stride(1) == 1
    out, _ = _check(f"channels-last {w.name} lanes={lanes}", cpu, dev, dtype, lanes_per_channel=lanes)
    assert L == 1 or out.stride(1) == 1  # allocated in u's layout


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 64, 256), (1, 48, 333)])
def test_slices_of_projection_outputs(dtype, shape):
    """x and z as the two halves of one (batch, L, 2 dim) tensor, B and C as
    columns of one (batch, L, R + 2 N) tensor, delta (batch, L, dim)."""
    b, d, L = shape
    N, R = 16, 8
    w = inputs.custom(b, d, L, N, dtype, seed=L + 1)
    cpu = inputs.scan_inputs(w)
    act = inputs.DTYPES[dtype]
    xz = torch.cat([cpu["u"], cpu["z"]], dim=1).transpose(1, 2).contiguous().cuda()      # (b, L, 2d)
    proj = torch.cat([torch.zeros(b, R, L, dtype=act), cpu["B"], cpu["C"]], dim=1)
    proj = proj.transpose(1, 2).contiguous().cuda()                                       # (b, L, R + 2N)
    dev = {"u": xz[..., :d].transpose(1, 2), "z": xz[..., d:].transpose(1, 2),
           "B": proj[..., R:R + N].transpose(1, 2), "C": proj[..., R + N:].transpose(1, 2),
           "delta": _channels_last(cpu["delta"]).cuda(),
           "A": cpu["A"].cuda(), "D": cpu["D"].cuda(), "delta_bias": cpu["delta_bias"].cuda()}
    assert dev["u"].stride() == (L * 2 * d, 1, 2 * d) and dev["B"].stride() == (L * (R + 2 * N), 1, R + 2 * N)
    _check(f"projection slices {w.name}", cpu, dev, dtype)


def test_mixed_layouts_and_broadcast_B():
    """u channel-contiguous, delta and z time-contiguous, B shared by every
    batch row (batch stride 0), C in the state-contiguous layout."""
    b, d, L, N = 3, 40, 200, 16
    w = inputs.custom(b, d, L, N, "bf16", seed=77)
    cpu = inputs.scan_inputs(w)
    cpu["B"] = cpu["B"][:1].expand(b, N, L)
    dev = {"u": _channels_last(cpu["u"]).cuda(), "delta": cpu["delta"].cuda(), "z": cpu["z"].cuda(),
           "B": cpu["B"][:1].cuda().expand(b, N, L), "C": _channels_last(cpu["C"]).cuda(),
           "A": cpu["A"].cuda(), "D": cpu["D"].cuda(), "delta_bias": cpu["delta_bias"].cuda()}
    assert dev["B"].stride(0) == 0
    _check("mixed + broadcast B", cpu, dev, "bf16")


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_dense_strides_match_the_dense_entry_point(dtype):
    w = inputs.custom(2, 64, 512, 16, dtype, seed=5)
    dev = {k: (None if v is None else v.cuda()) for k, v in inputs.scan_inputs(w).items()}
    o1, s1 = _run(dev)
    o2, s2 = binding.mamba_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"],
                                    z=dev["z"], delta_bias=dev["delta_bias"], return_last_state=True,
                                    schedule=binding.SCHEDULE_STATIC)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_channels_last_matches_dense_bitwise(dtype):
    # same kernel arithmetic, other staging: results identical
    w = inputs.custom(2, 64, 320, 16, dtype, seed=9)
    cpu = inputs.scan_inputs(w)
    dense = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    cl = {k: (_channels_last(v).cuda() if k in ("u", "delta", "z", "B", "C") else v.cuda()) for k, v in cpu.items()}
    o1, s1 = _run(dense, lanes_per_channel=2, threads_per_block=128)
    o2, s2 = _run(cl, lanes_per_channel=2, threads_per_block=128)
    assert torch.equal(o1, o2.contiguous()) and torch.equal(s1, s2)


def _page_layout(cpu, keep=()):
    """The pages' layout: (batch, L, dim) activations and (batch, L, N) B / C,
    dense, seen as (batch, dim, L) / (batch, N, L) views."""
    return {k: (None if v is None else (_channels_last(v) if k in ("u", "delta", "z", "B", "C") else v).cuda())
            for k, v in cpu.items()}


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape,dstate", [((2, 96, 336), 16), ((3, 40, 128), 8), ((1, 16, 64), 16),
                                          ((2, 1280, 512), 16), ((1, 64, 8192), 16)],
                         ids=["2x96x336", "3x40x128-N8", "1x16x64", "2x1280x512", "1x64x8192-two-phase"])
@pytest.mark.parametrize("lanes", [0, 2, 4])
def test_page_layout_on_the_local_kernel(dtype, shape, dstate, lanes):
    """The pages' (b, l, d) layout runs the block-local lane-split kernel:
    bit-equal to mamba_scan_fwd on the same values laid out densely with the
    same lanes (the same scan, other staging), and within the tolerance of
    the oracle.  The long row with few channels splits each group's sequence
    among a block's warps (two-phase pieces)."""
    b, d, L = shape
    w = inputs.custom(b, d, L, dstate, dtype, seed=b + d + L + lanes)
    cpu = inputs.scan_inputs(w)
    dense = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    kw = dict(schedule=binding.SCHEDULE_LOCAL, lanes_per_channel=lanes)
    o1, s1 = binding.mamba_scan_fwd(dense["u"], dense["delta"], dense["A"], dense["B"], dense["C"], D=dense["D"],
                                    z=dense["z"], delta_bias=dense["delta_bias"], return_last_state=True, **kw)
    o2, s2 = _check(f"page layout {w.name} lanes={lanes}", cpu, _page_layout(cpu), dtype, **kw)
    assert o2.stride(1) == 1
    assert torch.equal(o1, o2.contiguous()) and torch.equal(s1, s2)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("lanes", [2, 4])
def test_page_layout_ragged_length_and_optional_inputs(dtype, lanes):
    """Lengths that are no whole number of sub-chunks or of 16-byte chunks,
    no gate, no bias, no D (the local kernel takes any length in this
    layout)."""
    for L, drop in ((333, ()), (97, ("z", "delta_bias", "D")), (1000, ("z",))):
        w = inputs.custom(2, 48, L, 16, dtype, seed=L + lanes)
        cpu = inputs.scan_inputs(w)
        for k in drop:
            cpu[k] = None
        _check(f"page layout {w.name} lanes={lanes} drop={drop}", cpu, _page_layout(cpu), dtype,
               schedule=binding.SCHEDULE_LOCAL, lanes_per_channel=lanes)


@pytest.mark.parametrize("lanes", [2, 4])
def test_page_layout_in_place_from_a_state(lanes):
    """The local kernel on the pages' layout writing out over u (same
    pointer and strides) and starting from h0: bit-equal to the same call
    with a separate output."""
    w = inputs.custom(2, 96, 512, 16, "bf16", seed=41 + lanes)
    cpu = inputs.scan_inputs(w)
    h0 = inputs.initial_state(2, 96, 16, seed=5).cuda()
    dev = _page_layout(cpu)
    kw = dict(schedule=binding.SCHEDULE_LOCAL, lanes_per_channel=lanes)
    ref, ref_state = _run(dev, h0=h0, **kw)
    dev["u"] = dev["u"].clone().transpose(1, 2).contiguous().transpose(1, 2)
    out, state = _run(dev, out=dev["u"], h0=h0, **kw)
    assert out.data_ptr() == dev["u"].data_ptr()
    assert torch.equal(out, ref) and torch.equal(state, ref_state)


def test_page_layout_default_call_at_layer_size():
    """Without a schedule the pages' layout of a Mamba-sized layer (1,280
    lane-pair groups) takes the block-local kernel: bit-equal to the dense
    call, sampled rows against the oracle."""
    w = inputs.custom(4, 5120, 512, 16, "bf16", seed=43)
    cpu = inputs.scan_inputs(w)
    dense = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    o1, s1 = binding.mamba_scan_fwd(dense["u"], dense["delta"], dense["A"], dense["B"], dense["C"], D=dense["D"],
                                    z=dense["z"], delta_bias=dense["delta_bias"], return_last_state=True)
    assert binding.mamba_scan_plan(4, 5120, 512, 16, torch.bfloat16, workspace=False)[2] == binding.SCHEDULE_LOCAL
    o2, s2 = _run(_page_layout(cpu))
    assert torch.equal(o1, o2.contiguous()) and torch.equal(s1, s2)
    rows = sample_rows(w.batch, w.dim, 8, seed=w.seed)
    ro, rs = oracle_rows(cpu, rows)
    idx = torch.tensor(rows, device="cuda")
    e1 = rel_err(to_np(o2.contiguous().view(w.batch * w.dim, -1).index_select(0, idx)), ro)
    e2 = rel_err(to_np(s2.view(w.batch * w.dim, -1).index_select(0, idx)), rs)
    record(f"page layout default call {w.name} sampled", out=e1, state=e2)
    assert e1 <= TOL[torch.bfloat16] and e2 <= TOL[torch.bfloat16]


def test_page_layout_local_schedule_needs_the_layout():
    """SCHEDULE_LOCAL on a layout the local kernel cannot stage (dim not a
    multiple of 8 bf16 values) is refused; AUTO runs the static kernel."""
    w = inputs.custom(1, 36, 64, 16, "bf16", seed=6)
    cpu = inputs.scan_inputs(w)
    dev = _page_layout(cpu)
    with pytest.raises(binding.MambaError):
        _run(dev, schedule=binding.SCHEDULE_LOCAL)
    _check("page layout dim 36 (static)", cpu, dev, "bf16")


def test_in_place_and_initial_state():
    w = inputs.custom(2, 32, 256, 16, "bf16", seed=12)
    cpu = inputs.scan_inputs(w)
    h0 = inputs.initial_state(2, 32, 16, seed=4)
    dev = {k: (_channels_last(v).cuda() if k in ("u", "delta", "z", "B", "C") else v.cuda()) for k, v in cpu.items()}
    ref, ref_state = _check("channels-last from h0", cpu, dev, "bf16", h0=h0)
    u = dev["u"].clone().transpose(1, 2).contiguous().transpose(1, 2)
    dev["u"] = u
    out, state = _run(dev, out=u, h0=h0.cuda())
    assert out.data_ptr() == u.data_ptr()
    assert torch.equal(out, ref) and torch.equal(state, ref_state)


def test_rejected_layouts():
    w = inputs.custom(1, 16, 64, 16, "bf16", seed=3)
    dev = {k: (None if v is None else v.cuda()) for k, v in inputs.scan_inputs(w).items()}
    with pytest.raises(binding.MambaError):  # out with a zero stride writes one address twice
        _run(dev, out=torch.empty(1, 16, 1, device="cuda", dtype=torch.bfloat16).expand(1, 16, 64))
    wide = torch.empty(1, 16, 128, device="cuda", dtype=torch.bfloat16)
    dev["u"] = wide[..., :64]
    with pytest.raises(binding.MambaError):  # out interleaved with u inside one buffer
        _run(dev, out=wide[..., 64:])
