"""Parity of the scan's backward pass with the fp64 oracle's gradients,
through the C ABI (GPU)."""
import numpy as np
import pytest
import torch

import oracle
from parity import TOL, record, rel_err, to_np
from selective_state_space_20_b200 import binding, inputs

pytestmark = pytest.mark.gpu

# gradients kept in fp32 (sums over channels / time) and those stored in the
# activation dtype
FP32_GRADS = ("dA", "dB", "dC", "dD", "ddelta_bias")
ACT_GRADS = ("du", "ddelta", "dz")


def check_bwd(batch, dim, L, N, dtype, seed, gate=True, softplus=True, dlast=True, drop=(), h0=False):
    w = inputs.custom(batch, dim, L, N, dtype, seed=seed)
    cpu = inputs.scan_inputs(w)
    if not gate:
        cpu["z"] = None
    for k in drop:
        cpu[k] = None
    if not softplus:
        cpu["delta"] = cpu["delta"].abs() * 0.1
        if cpu["delta_bias"] is not None:
            cpu["delta_bias"] = cpu["delta_bias"].abs() * 0.01
    g = torch.Generator().manual_seed(seed + 1)
    dout = torch.randn(batch, dim, L, generator=g).to(inputs.DTYPES[dtype])
    dl = torch.randn(batch, dim, N, generator=g) if dlast else None
    hs = inputs.initial_state(batch, dim, N, seed=seed + 2) if h0 else None
    dev = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    got = binding.mamba_scan_bwd(dout.cuda(), dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"],
                                 D=dev["D"], z=dev["z"], delta_bias=dev["delta_bias"],
                                 delta_softplus=softplus, dlast_state=None if dl is None else dl.cuda(),
                                 h0=None if hs is None else hs.cuda())
    ref = oracle.scan_bwd(dout, cpu["u"], cpu["delta"], cpu["A"], cpu["B"], cpu["C"], D=cpu["D"], z=cpu["z"],
                          delta_bias=cpu["delta_bias"], delta_softplus=softplus, h0=hs,
                          dlast=None if dl is None else dl.double())
    errs = {}
    for k in FP32_GRADS + ACT_GRADS + (("dh0",) if h0 else ()):
        if got.get(k) is None:
            continue
        errs[k] = rel_err(to_np(got[k]), ref[k])
    record(f"scan_bwd {batch}x{dim}x{L} N{N} {dtype} gate={gate} sp={softplus} dlast={dlast} h0={h0}", **errs)
    for k, e in errs.items():
        assert e <= grad_tol(k, dtype), (k, e, errs)
    return errs


def grad_tol(name, dtype):
    """The activation-dtype bar (1e-4 fp32, 2e-2 bf16) for every gradient of
    fp32 inputs; with bf16 inputs the fp32 parameter gradients (sums over
    channels and time) are held to 1e-3, stricter than the bf16 bar."""
    if dtype == "fp32" or name in ACT_GRADS:
        return TOL[inputs.DTYPES[dtype]]
    return 1e-3


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 37, 100, 16), (1, 64, 257, 16), (3, 20, 33, 5), (1, 1, 1, 16),
                                   (2, 96, 512, 16)])
def test_bwd_matches_oracle(dtype, shape):
    check_bwd(*shape, dtype, seed=sum(shape))


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("h0", [False, True])
def test_bwd_six_warp_blocks(dtype, h0):
    """1 x 5120 channels: 48-channel blocks (6 warps) spread more evenly over
    the SMs than 32-channel ones, so the kernel takes them; every gradient
    against the oracle, with a ragged last 32-step piece."""
    check_bwd(1, 5120, 72, 16, dtype, seed=77, h0=h0)


@pytest.mark.parametrize("gate,softplus,dlast", [(False, True, True), (True, False, True), (True, True, False)])
def test_bwd_flags(gate, softplus, dlast):
    for dtype in ("fp32", "bf16"):
        check_bwd(2, 40, 80, 16, dtype, seed=7, gate=gate, softplus=softplus, dlast=dlast)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 37, 100, 16), (3, 20, 33, 5), (1, 64, 257, 16)])
@pytest.mark.parametrize("dlast", [True, False])
def test_bwd_from_an_initial_state(dtype, shape, dlast):
    """The forward started from h0: every gradient, and dh0 = dL/dh_{-1}."""
    check_bwd(*shape, dtype, seed=sum(shape) + 3, dlast=dlast, h0=True)


def test_bwd_without_D_and_bias():
    check_bwd(2, 33, 64, 16, "fp32", seed=8, drop=("D", "delta_bias"))


def test_bwd_rejects_large_dstate():
    w = inputs.custom(1, 32, 64, 32, "bf16", seed=1)
    d = {k: (None if v is None else v.cuda()) for k, v in inputs.scan_inputs(w).items()}
    with pytest.raises(binding.MambaError):
        binding.mamba_scan_bwd(torch.zeros_like(d["u"]), d["u"], d["delta"], d["A"], d["B"], d["C"])


def test_bwd_full_size_layer():
    """The Mamba-130M layer (8 x 1536 x 2048): gradients finite; du, ddelta,
    dz on sampled rows and dA, dD, dbias for the sampled channels against the
    oracle run on those rows (dB / dC sum over all channels: checked whole on
    the smaller shapes above)."""
    w = inputs.MAMBA_130M
    cpu = inputs.scan_inputs(w)
    dev = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    g = torch.Generator().manual_seed(99)
    dout = torch.randn(w.batch, w.dim, w.seqlen, generator=g).to(torch.bfloat16)
    got = binding.mamba_scan_bwd(dout.cuda(), dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"],
                                 D=dev["D"], z=dev["z"], delta_bias=dev["delta_bias"])
    torch.cuda.synchronize()
    for k, v in got.items():
        if v is not None:
            assert torch.isfinite(v.float()).all(), k
    # one batch row, a few channels: the per-row gradients (du, ddelta, dz)
    b, chans = 3, [0, 1, 700, 1535]
    sub = {k: (None if v is None else v) for k, v in cpu.items()}
    r = oracle.scan_bwd(dout[b:b + 1, chans], sub["u"][b:b + 1, chans], sub["delta"][b:b + 1, chans],
                        sub["A"][chans], sub["B"][b:b + 1], sub["C"][b:b + 1], D=sub["D"][chans],
                        z=sub["z"][b:b + 1, chans], delta_bias=sub["delta_bias"][chans])
    for k in ACT_GRADS:
        e = rel_err(to_np(got[k][b:b + 1, chans]), r[k])
        assert e <= 2e-2, (k, e)


def test_bwd_benchmark_layer_sampled():
    """The layer the bench times the backward on (Mamba-2.8B, 4 x 5120 x 4096,
    bf16, with dL/dlast_state): du, ddelta, dz on sampled channels of two batch
    rows, and dA, dD, dbias of sampled channels (sums over all four batch
    rows) against the oracle run on exactly those rows."""
    w = inputs.MAMBA_2_8B
    dev = inputs.scan_inputs(w, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(7)
    dout = torch.randn(w.batch, w.dim, w.seqlen, generator=g, device="cuda").to(torch.bfloat16)
    dlast = torch.randn(w.batch, w.dim, w.dstate, generator=g, device="cuda")
    got = binding.mamba_scan_bwd(dout, dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"],
                                 z=dev["z"], delta_bias=dev["delta_bias"], dlast_state=dlast)
    torch.cuda.synchronize()
    chans = [0, 31, 32, 2047, 4096, 5119]
    cpu = lambda t: t.detach().to("cpu")  # noqa: E731
    r = oracle.scan_bwd(cpu(dout[:, chans]), cpu(dev["u"][:, chans]), cpu(dev["delta"][:, chans]),
                        cpu(dev["A"][chans]), cpu(dev["B"]), cpu(dev["C"]), D=cpu(dev["D"][chans]),
                        z=cpu(dev["z"][:, chans]), delta_bias=cpu(dev["delta_bias"][chans]),
                        dlast=cpu(dlast[:, chans]).double())
    errs = {k: rel_err(to_np(got[k][:, chans]), r[k]) for k in ACT_GRADS}
    errs.update({k: rel_err(to_np(got[k][chans]), r[k]) for k in ("dA", "dD", "ddelta_bias")})
    record("scan_bwd mamba-2.8b layer sampled channels", **errs)
    for k, e in errs.items():
        assert e <= grad_tol(k, "bf16"), (k, e, errs)


# ------------------------------------------------ checkpoints from the forward
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 37, 104, 16), (1, 64, 256, 16), (3, 20, 40, 5), (2, 96, 512, 16),
                                   (1, 33, 8, 16)])
@pytest.mark.parametrize("h0", [False, True])
def test_bwd_from_forward_checkpoints(dtype, shape, h0):
    """mamba_scan_fwd_ckpt keeps the state every 32 steps; mamba_scan_bwd_ckpt
    recomputes from them instead of sweeping the inputs: the forward's outputs
    and every gradient against the oracle."""
    batch, dim, L, N = shape
    w = inputs.custom(batch, dim, L, N, dtype, seed=sum(shape) + 11)
    cpu = inputs.scan_inputs(w)
    g = torch.Generator().manual_seed(sum(shape) + 12)
    dout = torch.randn(batch, dim, L, generator=g).to(inputs.DTYPES[dtype])
    dl = torch.randn(batch, dim, N, generator=g)
    hs = inputs.initial_state(batch, dim, N, seed=sum(shape) + 13) if h0 else None
    dev = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    out, last, ck = binding.mamba_scan_fwd_ckpt(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"],
                                                z=dev["z"], delta_bias=dev["delta_bias"],
                                                h0=None if hs is None else hs.cuda())
    got = binding.mamba_scan_bwd(dout.cuda(), dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"],
                                 z=dev["z"], delta_bias=dev["delta_bias"], dlast_state=dl.cuda(),
                                 h0=None if hs is None else hs.cuda(), ckpt=ck)
    ro, rs = oracle.scan(cpu["u"], cpu["delta"], cpu["A"], cpu["B"], cpu["C"], D=cpu["D"], z=cpu["z"],
                         delta_bias=cpu["delta_bias"], h0=hs)
    tol = TOL[inputs.DTYPES[dtype]]
    assert rel_err(to_np(out), ro) <= tol and rel_err(to_np(last), rs) <= tol
    ref = oracle.scan_bwd(dout, cpu["u"], cpu["delta"], cpu["A"], cpu["B"], cpu["C"], D=cpu["D"], z=cpu["z"],
                          delta_bias=cpu["delta_bias"], h0=hs, dlast=dl.double())
    errs = {k: rel_err(to_np(got[k]), ref[k]) for k in FP32_GRADS + ACT_GRADS + (("dh0",) if h0 else ())}
    record(f"scan_bwd from forward checkpoints {batch}x{dim}x{L} N{N} {dtype} h0={h0}", **errs)
    for k, e in errs.items():
        assert e <= grad_tol(k, dtype), (k, e, errs)


@pytest.mark.parametrize("batch,dim", [(2, 70), (4, 2960)])  # the second: 740 groups, the unrolled form
def test_forward_checkpoints_hold_the_states(batch, dim):
    """Entry s of the checkpoints is the state entering step 32 s: compared
    with the final state of a scan over the first 32 s steps."""
    w = inputs.custom(batch, dim, 160, 16, "bf16", seed=91)
    dev = inputs.scan_inputs(w, device="cuda")
    _, _, ck = binding.mamba_scan_fwd_ckpt(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], D=dev["D"],
                                           z=dev["z"], delta_bias=dev["delta_bias"])
    g32 = (w.dim + 31) // 32
    ck = ck[: w.batch * g32 * 5 * 32 * 16].view(w.batch, g32, 5, 32, 16)
    for s in (1, 3, 4):
        head = {k: (v[..., :32 * s].contiguous() if k in ("u", "delta", "z", "B", "C") else v) for k, v in dev.items()}
        _, st = binding.mamba_scan_fwd(head["u"], head["delta"], head["A"], head["B"], head["C"], D=head["D"],
                                       z=head["z"], delta_bias=head["delta_bias"], return_last_state=True)
        flat = ck[:, :, s].reshape(w.batch, g32 * 32, 16)[:, :w.dim]
        assert rel_err(to_np(flat), to_np(st)) <= 1e-3
    assert torch.all(ck[:, :, 0].reshape(w.batch, g32 * 32, 16)[:, :w.dim] == 0)  # entering step 0: zeros


def test_forward_checkpoints_reject_unsupported_layouts():
    w = inputs.custom(1, 32, 60, 16, "bf16", seed=92)  # L not a multiple of 8
    d = {k: (None if v is None else v.cuda()) for k, v in inputs.scan_inputs(w).items()}
    with pytest.raises(binding.MambaError):
        binding.mamba_scan_fwd_ckpt(d["u"], d["delta"], d["A"], d["B"], d["C"])
