"""The bounds-checked build (libmamba_scan_checked.so, MSCAN_BOUNDS_CHECK).

Its instrumented kernels -- the lane-split scan in every form that uses it,
the one-lane scan, the static scan in its staging forms, the complex mode,
the backward, the decode step, the conv1d kernels -- test every global
access against the byte range of its tensor.  On the shapes below (ragged groups and lengths,
N < 16, both lane counts, two-phase pieces, the device-wide and block-local
forms, the (b, l, d) layout, the fused conv1d with u written out,
checkpoints, initial and final states) they must record no access outside a
tensor and give the normal build's results bit for bit.  A test hook then
shortens the output range the launches record: the checks must report the
output site at the first byte past the shortened range, skip that access
(the tail of the output keeps its old contents) and leave everything else
equal to the normal build's.  No access leaves allocated memory in any of
these runs.
"""
import contextlib

import pytest
import torch

from selective_state_space_20_b200 import binding, inputs

pytestmark = pytest.mark.gpu

SITE_OUT = 13


@pytest.fixture(scope="module")
def checked():
    lib = binding.load_checked_library()
    assert lib.mamba_bounds_checked() == 1
    assert binding.load_library().mamba_bounds_checked() == 0
    return lib


@contextlib.contextmanager
def using(lib):
    prev = binding._lib
    binding._lib = lib
    try:
        yield
    finally:
        binding._lib = prev


def both(checked, fn):
    """fn() with the normal library, then with the checked one; the checked
    run must record no violation."""
    ref = fn()
    torch.cuda.synchronize()
    with using(checked):
        got = fn()
        torch.cuda.synchronize()
        assert binding.bounds_status(checked) is None
    return ref, got


def equal(a, b):
    if isinstance(a, (tuple, list)):
        return all(equal(x, y) for x, y in zip(a, b))
    return torch.equal(a, b)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape,dstate,lanes", [((2, 70, 336), 16, 2), ((3, 33, 1000), 5, 4),
                                                ((1, 64, 8192), 16, 2), ((4, 1030, 256), 16, 0),
                                                ((4, 2960, 96), 16, 2)],
                         ids=["2x70x336-R2", "3x33x1000-N5-R4", "1x64x8192-two-phase", "4x1030x256-lanes-auto",
                              "4x2960x96-unrolled"])
def test_block_local_scan(checked, dtype, shape, dstate, lanes):
    b, d, L = shape
    ins = inputs.scan_inputs(inputs.custom(b, d, L, dstate, dtype, seed=b + d + L), device="cuda")
    h0 = inputs.initial_state(b, d, dstate, seed=3, device="cuda")
    # lanes 0: the library's choice within the block-local schedule
    kw = dict(schedule=binding.SCHEDULE_LOCAL, lanes_per_channel=lanes)
    run = lambda: binding.mamba_scan_fwd(ins["u"], ins["delta"], ins["A"], ins["B"], ins["C"], D=ins["D"],  # noqa: E731
                                         z=ins["z"], delta_bias=ins["delta_bias"], h0=h0, return_last_state=True,
                                         **kw)
    ref, got = both(checked, run)
    assert equal(ref, got)


@pytest.mark.parametrize("lanes", [2, 4])
def test_device_wide_scan_and_checkpoints(checked, lanes):
    w = inputs.custom(2, 16 * 30, 512, 16, "bf16", seed=31)
    ins = inputs.scan_inputs(w, device="cuda")
    ws = torch.empty(binding.mamba_scan_workspace_size(w.batch, w.dim, w.seqlen, w.dstate, torch.bfloat16),
                     device="cuda", dtype=torch.uint8)
    run = lambda: binding.mamba_scan_fwd(ins["u"], ins["delta"], ins["A"], ins["B"], ins["C"], D=ins["D"],  # noqa: E731
                                         z=ins["z"], delta_bias=ins["delta_bias"], return_last_state=True,
                                         workspace=ws, schedule=binding.SCHEDULE_PERSISTENT,
                                         lanes_per_channel=lanes)
    ref, got = both(checked, run)
    assert equal(ref, got)
    ck = lambda: binding.mamba_scan_fwd_ckpt(ins["u"], ins["delta"], ins["A"], ins["B"], ins["C"], D=ins["D"],  # noqa: E731
                                             z=ins["z"], delta_bias=ins["delta_bias"])
    ref, got = both(checked, ck)
    assert equal(ref, got)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("with_ws", [False, True])
def test_state_only_scan(checked, dtype, with_ws):
    """The lane-split kernel run for the final state alone: C, z and out are
    not passed, so any access to them would leave its (empty) range."""
    w = inputs.custom(3, 70, 1000, 16, dtype, seed=36)
    ins = inputs.scan_inputs(w, device="cuda")
    h0 = inputs.initial_state(3, 70, 16, seed=8, device="cuda")
    ws = torch.empty(binding.mamba_scan_workspace_size(3, 70, 1000, 16, ins["u"].dtype), device="cuda",
                     dtype=torch.uint8) if with_ws else None
    run = lambda: binding.mamba_scan_state(ins["u"], ins["delta"], ins["A"], ins["B"],  # noqa: E731
                                           delta_bias=ins["delta_bias"], h0=h0, workspace=ws)
    ref, got = both(checked, run)
    assert equal(ref, got)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape,dstate,chunk", [((2, 70, 1000), 16, 64), ((3, 33, 344), 5, 0)],
                         ids=["2x70x1000-chunks64", "3x33x344-N5"])
def test_one_lane_scan(checked, dtype, shape, dstate, chunk):
    """The one-lane kernel (scan warp + helper warp, on request): ragged
    channel groups and lengths, carries between chunks, h0 and last_state."""
    b, d, L = shape
    w = inputs.custom(b, d, L, dstate, dtype, seed=b + d + L + 1)
    ins = inputs.scan_inputs(w, device="cuda")
    h0 = inputs.initial_state(b, d, dstate, seed=4, device="cuda")
    ws = torch.empty(binding.mamba_scan_workspace_size(b, d, L, dstate, ins["u"].dtype), device="cuda",
                     dtype=torch.uint8)
    run = lambda: binding.mamba_scan_fwd(ins["u"], ins["delta"], ins["A"], ins["B"], ins["C"], D=ins["D"],  # noqa: E731
                                         z=ins["z"], delta_bias=ins["delta_bias"], h0=h0, return_last_state=True,
                                         workspace=ws, schedule=binding.SCHEDULE_PERSISTENT, lanes_per_channel=1,
                                         chunk_timesteps=chunk)
    ref, got = both(checked, run)
    assert equal(ref, got)


@pytest.mark.parametrize("lanes", [2, 4])
def test_page_layout_and_fused_conv(checked, lanes):
    w = inputs.custom(2, 96, 336, 16, "bf16", seed=32)
    cpu = inputs.scan_inputs(w)
    cl = {k: (None if v is None else (v.transpose(1, 2).contiguous().transpose(1, 2)
                                      if k in ("u", "delta", "z", "B", "C") else v).cuda())
          for k, v in cpu.items()}
    run = lambda: binding.mamba_scan_fwd_strided(cl["u"], cl["delta"], cl["A"], cl["B"], cl["C"], D=cl["D"],  # noqa: E731
                                                 z=cl["z"], delta_bias=cl["delta_bias"], return_last_state=True,
                                                 schedule=binding.SCHEDULE_LOCAL, lanes_per_channel=lanes)
    ref, got = both(checked, run)
    assert equal(ref, got)
    ci = inputs.conv_inputs(2, 96, 512, 4, "bf16", seed=33, device="cuda")
    ins = inputs.scan_inputs(inputs.custom(2, 96, 512, 16, "bf16", seed=34), device="cuda")
    x, z = ci["xz"][:, :96], ci["xz"][:, 96:]
    fused = lambda: binding.mamba_scan_fwd_conv(x, ci["weight"], ci["bias"], ins["delta"], ins["A"], ins["B"],  # noqa: E731
                                                ins["C"], D=ins["D"], z=z, delta_bias=ins["delta_bias"],
                                                return_last_state=True, return_u=True)
    ref, got = both(checked, fused)
    assert equal(ref, got)


def _channels_last(t):
    return t.transpose(1, 2).contiguous().transpose(1, 2)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("case", ["dense", "dense-N40", "unaligned", "channels-last", "mixed-broadcast-B",
                                  "odd-strides"])
def test_static_scan(checked, dtype, case):
    """The static kernel in its staging forms: 16-byte copies along time or
    along channels, B / C along time or along states, element copies."""
    b, d, L, N = (2, 40, 333, 40) if case == "dense-N40" else (2, 40, 333, 16)
    cpu = inputs.scan_inputs(inputs.custom(b, d, L, N, dtype, seed=L + N))
    dev = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    kw = dict(schedule=binding.SCHEDULE_STATIC)
    if case == "unaligned":  # u one element off its 16-byte grid: element copies
        buf = torch.empty(dev["u"].numel() + 1, device="cuda", dtype=dev["u"].dtype)
        dev["u"] = buf[1:].view(dev["u"].shape)
        dev["u"].copy_(cpu["u"].cuda())
    if case == "channels-last":
        dev = {k: (_channels_last(v) if k in ("u", "delta", "z", "B", "C") else v) for k, v in dev.items()}
    if case == "mixed-broadcast-B":
        dev["u"] = _channels_last(dev["u"])
        dev["B"] = dev["B"][:1].expand(b, N, L)
        dev["C"] = _channels_last(dev["C"])
    if case == "odd-strides":  # every 3rd element of a wider buffer along time
        wide = torch.zeros(b, d, 3 * L, device="cuda", dtype=dev["delta"].dtype)
        wide[..., ::3] = dev["delta"]
        dev["delta"] = wide[..., ::3]
    if case.startswith("dense"):
        run = lambda: binding.mamba_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"],  # noqa: E731
                                             z=dev["z"], delta_bias=dev["delta_bias"], return_last_state=True,
                                             **kw)
    else:
        run = lambda: binding.mamba_scan_fwd_strided(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"],  # noqa: E731
                                                     D=dev["D"], z=dev["z"], delta_bias=dev["delta_bias"],
                                                     return_last_state=True, **kw)
    ref, got = both(checked, run)
    assert equal(ref, got)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("dstate", [16, 13, 8])
def test_decode_step(checked, dtype, dstate):
    d = inputs.decode_inputs(inputs.DecodeWorkload("decode test", 7, 301, dstate, 2, dtype, 1e-3, 1e-1,
                                                   "uniform", seed=35), device="cuda", steps=2)
    state0 = inputs.initial_state(7, 301, dstate, seed=8, device="cuda")

    def run():
        st = state0.clone()
        outs = [binding.mamba_state_update(st, d["u"][t], d["delta"][t], d["A"], d["B"][t], d["C"][t], D=d["D"],
                                           z=d["z"][t], delta_bias=d["delta_bias"]) for t in range(2)]
        return outs + [st]

    ref, got = both(checked, run)
    assert equal(ref, got)


@pytest.mark.parametrize("L", [4096, 333])
def test_conv1d(checked, L):
    ci = inputs.conv_inputs(3, 40, L, 4, "bf16", seed=36, device="cuda")
    run = lambda: binding.mamba_conv1d_fwd(ci["xz"], ci["weight"], ci["bias"], dim=40)  # noqa: E731
    ref, got = both(checked, run)
    assert equal(ref, got)
    state0 = torch.randn(3, 40, 3, device="cuda")

    def step():
        st = state0.clone()
        return binding.mamba_conv1d_update(st, ci["xz"][:, :40, 0].contiguous(), ci["weight"], ci["bias"]), st

    ref, got = both(checked, step)
    assert equal(ref, got)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 70, 336), (1, 100, 1000)])
def test_backward(checked, dtype, shape):
    """Self-contained (its own checkpoint sweep) and from the forward's
    checkpoints, from an initial state, with dL/dlast_state.  dA / dB / dC /
    dD / dbias sum with atomics whose order varies, so those are compared
    within a few ulps; du, ddelta, dz bit for bit."""
    b, d, L = shape
    w = inputs.custom(b, d, L, 16, dtype, seed=b + d + L + 1)
    ins = inputs.scan_inputs(w, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(3)
    dout = torch.randn(b, d, L, generator=g, device="cuda").to(ins["u"].dtype)
    dlast = torch.randn(b, d, 16, generator=g, device="cuda")
    h0 = inputs.initial_state(b, d, 16, seed=4, device="cuda")
    kw = dict(D=ins["D"], z=ins["z"], delta_bias=ins["delta_bias"])
    _, _, ck = binding.mamba_scan_fwd_ckpt(ins["u"], ins["delta"], ins["A"], ins["B"], ins["C"], h0=h0, **kw)
    for ckpt in (None, ck):
        run = lambda: binding.mamba_scan_bwd(dout, ins["u"], ins["delta"], ins["A"], ins["B"], ins["C"],  # noqa: E731
                                             dlast_state=dlast, h0=h0, ckpt=ckpt, **kw)
        ref, got = both(checked, run)
        for k in ref:
            if ref[k] is None:
                continue
            if k in ("du", "ddelta", "dz"):
                assert torch.equal(ref[k], got[k]), k
            else:
                assert torch.allclose(ref[k], got[k], rtol=1e-5, atol=1e-6 * ref[k].abs().max().item()), k


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_complex_mode(checked, dtype):
    d = inputs.complex_inputs(2, 40, 333, 16, dtype, device="cuda")
    h0 = torch.randn(2, 40, 16, 2, device="cuda") * 0.25
    run = lambda: binding.mamba_scan_fwd_complex(d["u"], d["delta"], d["A"], d["B"], d["C"], D=d["D"],  # noqa: E731
                                                 z=d["z"], delta_bias=d["delta_bias"], h0=h0,
                                                 return_last_state=True)
    ref, got = both(checked, run)
    assert equal(ref, got)


def _shrunk(checked, fn, out_of, shrink):
    """fn() with the normal library, then with the checked one and the
    output range `shrink` bytes short; checks the violation recorded (the
    output site, at the first byte past the range) and returns both results."""
    ref = fn()
    torch.cuda.synchronize()
    with using(checked):
        prev = checked.mamba_debug_shrink_output_extent(shrink)
        try:
            got = fn()
            torch.cuda.synchronize()
        finally:
            checked.mamba_debug_shrink_output_extent(prev)
        hit = binding.bounds_status(checked)
    nbytes = out_of(ref).numel() * out_of(ref).element_size()
    assert hit == (SITE_OUT, nbytes - shrink), (hit, nbytes)
    return ref, got


def test_a_short_output_range_is_reported_and_its_store_skipped(checked):
    w = inputs.custom(2, 64, 512, 16, "bf16", seed=37)
    ins = inputs.scan_inputs(w, device="cuda")
    sentinel = torch.full_like(ins["u"], 7.0)

    def scan():
        out = sentinel.clone()
        # the block-local lane-split kernel (a shape this small would otherwise
        # take the static kernel, shortened further below)
        binding.mamba_scan_fwd(ins["u"], ins["delta"], ins["A"], ins["B"], ins["C"], D=ins["D"], z=ins["z"],
                               delta_bias=ins["delta_bias"], out=out, schedule=binding.SCHEDULE_LOCAL)
        return out

    ref, got = _shrunk(checked, scan, lambda o: o, 16)
    flat_r, flat_g = ref.reshape(-1), got.reshape(-1)
    assert torch.equal(flat_g[:-8], flat_r[:-8])  # every 16-byte chunk but the last
    assert torch.all(flat_g[-8:] == 7.0)          # the last was skipped

    d = inputs.decode_inputs(inputs.DecodeWorkload("decode shrink", 4, 96, 16, 1, "bf16", 1e-3, 1e-1,
                                                   "uniform", seed=38), device="cuda", steps=1)
    st0 = inputs.initial_state(4, 96, 16, seed=9, device="cuda")

    def step():
        st = st0.clone()
        out = torch.full((4, 96), 7.0, device="cuda", dtype=torch.bfloat16)
        binding.mamba_state_update(st, d["u"][0], d["delta"][0], d["A"], d["B"][0], d["C"][0], D=d["D"],
                                   z=d["z"][0], delta_bias=d["delta_bias"], out=out)
        return out

    ref, got = _shrunk(checked, step, lambda o: o, 2)
    assert torch.equal(got.reshape(-1)[:-1], ref.reshape(-1)[:-1]) and got.reshape(-1)[-1] == 7.0

    def static_scan():  # the static kernel, its scalar stores (L not a whole number of vectors)
        ins2 = inputs.scan_inputs(inputs.custom(2, 40, 333, 16, "fp32", seed=40), device="cuda")
        out = torch.full_like(ins2["u"], 7.0)
        binding.mamba_scan_fwd(ins2["u"], ins2["delta"], ins2["A"], ins2["B"], ins2["C"], D=ins2["D"],
                               z=ins2["z"], delta_bias=ins2["delta_bias"], out=out,
                               schedule=binding.SCHEDULE_STATIC)
        return out

    ref, got = _shrunk(checked, static_scan, lambda o: o, 4)
    assert torch.equal(got.reshape(-1)[:-1], ref.reshape(-1)[:-1]) and got.reshape(-1)[-1] == 7.0

    ws = torch.empty(binding.mamba_scan_workspace_size(w.batch, w.dim, w.seqlen, w.dstate, torch.bfloat16),
                     device="cuda", dtype=torch.uint8)

    def one_lane():  # the one-lane kernel's 16-byte stores
        out = sentinel.clone()
        binding.mamba_scan_fwd(ins["u"], ins["delta"], ins["A"], ins["B"], ins["C"], D=ins["D"], z=ins["z"],
                               delta_bias=ins["delta_bias"], out=out, workspace=ws,
                               schedule=binding.SCHEDULE_PERSISTENT, lanes_per_channel=1)
        return out

    ref, got = _shrunk(checked, one_lane, lambda o: o, 16)
    assert torch.equal(got.reshape(-1)[:-8], ref.reshape(-1)[:-8]) and torch.all(got.reshape(-1)[-8:] == 7.0)

    ci = inputs.conv_inputs(2, 32, 256, 4, "bf16", seed=39, device="cuda")
    conv = lambda: binding.mamba_conv1d_fwd(ci["xz"], ci["weight"], ci["bias"], dim=32,  # noqa: E731
                                            out=torch.full((2, 32, 256), 7.0, device="cuda", dtype=torch.bfloat16))
    ref, got = _shrunk(checked, conv, lambda o: o, 16)
    assert torch.equal(got.reshape(-1)[:-8], ref.reshape(-1)[:-8]) and torch.all(got.reshape(-1)[-8:] == 7.0)

    # the device status reports it too (and reading clears the record)
    with using(checked):
        prev = checked.mamba_debug_shrink_output_extent(16)
        try:
            scan()
        finally:
            checked.mamba_debug_shrink_output_extent(prev)
        assert binding.device_status() == binding.MAMBA_ERR_BOUNDS
        assert binding.device_status() == 0 and binding.bounds_status(checked) is None
