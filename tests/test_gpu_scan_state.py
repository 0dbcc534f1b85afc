"""The final state alone (mamba_scan_state: the lane-split kernel run
state-only, each piece of a group combined with the state before it) through
the C ABI, against the fp64 oracle's final state (GPU)."""
import pytest
import torch

import oracle
from parity import TOL, record, rel_err, to_np
from selective_state_space_20_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def _dev(ins):
    return {k: (None if v is None else v.cuda()) for k, v in ins.items()}


def _oracle_state(cpu, h0=None):
    _, rs = oracle.scan(cpu["u"], cpu["delta"], cpu["A"], cpu["B"], cpu["C"], D=cpu["D"], z=cpu["z"],
                        delta_bias=cpu["delta_bias"], h0=h0)
    return rs


def _workspace(w, dtype):
    return torch.empty(binding.mamba_scan_workspace_size(w.batch, w.dim, w.seqlen, w.dstate, dtype),
                       device="cuda", dtype=torch.uint8)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shape,dstate", [((2, 70, 336), 16), ((3, 33, 1000), 5), ((1, 64, 8192), 16),
                                          ((4, 300, 256), 16), ((1, 1, 8), 16)],
                         ids=["2x70x336", "3x33x1000-N5", "1x64x8192-pieces", "4x300x256", "1x1x8"])
@pytest.mark.parametrize("form", ["block-local", "device-wide"])
@pytest.mark.parametrize("with_h0", [False, True])
def test_state_matches_oracle(dtype, shape, dstate, form, with_h0):
    b, d, L = shape
    w = inputs.custom(b, d, L, dstate, dtype, seed=b + d + L + dstate)
    cpu = inputs.scan_inputs(w)
    dev = _dev(cpu)
    h0 = inputs.initial_state(b, d, dstate, seed=5, scale=0.25) if with_h0 else None
    ws = _workspace(w, dev["u"].dtype) if form == "device-wide" else None
    last = binding.mamba_scan_state(dev["u"], dev["delta"], dev["A"], dev["B"], delta_bias=dev["delta_bias"],
                                    h0=None if h0 is None else h0.cuda(), workspace=ws)
    torch.cuda.synchronize()
    err = rel_err(to_np(last), _oracle_state(cpu, h0))
    record(f"state only {w.name} {form} h0={with_h0}", state=err)
    assert err <= TOL[inputs.DTYPES[dtype]], err


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_state_agrees_with_the_full_scan(dtype):
    """Within the tolerance of the full scan's last_state (not bit for bit:
    the pieces are combined in another order), softplus off as well."""
    w = inputs.custom(2, 96, 4096, 16, dtype, seed=11)
    dev = inputs.scan_inputs(w, device="cuda")
    h0 = inputs.initial_state(2, 96, 16, seed=6, scale=0.25, device="cuda")
    # softplus off: steps that are already positive (the raw draws would let
    # states grow without bound over 4096 steps)
    steps = torch.nn.functional.softplus(dev["delta"].float() + dev["delta_bias"][:, None]).to(dev["delta"].dtype)
    for softplus, delta, bias in ((True, dev["delta"], dev["delta_bias"]), (False, steps, None)):
        _, full = binding.mamba_scan_fwd(dev["u"], delta, dev["A"], dev["B"], dev["C"], D=dev["D"],
                                         z=dev["z"], delta_bias=bias, delta_softplus=softplus,
                                         h0=h0, return_last_state=True)
        only = binding.mamba_scan_state(dev["u"], delta, dev["A"], dev["B"], delta_bias=bias,
                                        delta_softplus=softplus, h0=h0)
        torch.cuda.synchronize()
        assert rel_err(to_np(only), to_np(full)) <= TOL[inputs.DTYPES[dtype]]


def test_state_in_place_and_chained():
    """h0 may be last_state itself; two halves chained in place equal the
    whole sequence within the tolerance."""
    w = inputs.custom(2, 64, 2048, 16, "bf16", seed=12)
    cpu = inputs.scan_inputs(w)
    dev = _dev(cpu)
    st = torch.zeros(2, 64, 16, device="cuda")
    for lo, hi in ((0, 1024), (1024, 2048)):
        part = {k: dev[k][..., lo:hi].contiguous() for k in ("u", "delta", "B")}
        binding.mamba_scan_state(part["u"], part["delta"], dev["A"], part["B"], delta_bias=dev["delta_bias"],
                                 h0=st, last_state=st)
    torch.cuda.synchronize()
    assert rel_err(to_np(st), _oracle_state(cpu)) <= TOL[torch.bfloat16]


def test_state_benchmark_layer_sampled():
    """The Mamba-2.8B layer (4 x 5120 x 4096, bf16): sampled rows of the
    final state against the oracle run on each row alone."""
    w = inputs.MAMBA_2_8B
    dev = inputs.scan_inputs(w, device="cuda")
    last = binding.mamba_scan_state(dev["u"], dev["delta"], dev["A"], dev["B"], delta_bias=dev["delta_bias"])
    torch.cuda.synchronize()
    cpu = lambda t: None if t is None else t.detach().to("cpu")  # noqa: E731
    errs = []
    for bi, di in [(0, 0), (1, 2047), (3, 5119)]:
        _, rs = oracle.scan(cpu(dev["u"][bi:bi + 1, di:di + 1]), cpu(dev["delta"][bi:bi + 1, di:di + 1]),
                            cpu(dev["A"][di:di + 1]), cpu(dev["B"][bi:bi + 1]), cpu(dev["C"][bi:bi + 1]),
                            D=cpu(dev["D"][di:di + 1]), z=cpu(dev["z"][bi:bi + 1, di:di + 1]),
                            delta_bias=cpu(dev["delta_bias"][di:di + 1]), nthreads=1)
        errs.append(rel_err(to_np(last[bi, di]), rs[0, 0]))
    record("state only 4x5120x4096 bf16 sampled", state=max(errs))
    assert max(errs) <= TOL[torch.bfloat16], errs


def test_state_rejects_what_its_kernel_cannot_run():
    w = inputs.custom(1, 8, 64, 17, "bf16", seed=13)  # dstate > 16
    dev = inputs.scan_inputs(w, device="cuda")
    with pytest.raises(binding.MambaError) as e:
        binding.mamba_scan_state(dev["u"], dev["delta"], dev["A"], dev["B"])
    assert e.value.code == binding.MAMBA_ERR_UNSUPPORTED
    w = inputs.custom(1, 8, 61, 16, "bf16", seed=14)  # rows not whole 16-byte vectors
    dev = inputs.scan_inputs(w, device="cuda")
    with pytest.raises(binding.MambaError) as e:
        binding.mamba_scan_state(dev["u"], dev["delta"], dev["A"], dev["B"])
    assert e.value.code == binding.MAMBA_ERR_UNSUPPORTED
