"""The sequence-split kernels on one GPU: the per-row delta sums and the
fold of shard summaries against fp64 numpy, and a whole sequence cut into
shards -- each shard's summary, the fold, and the second scan run one after
another on one device -- against the oracle's scan of the whole sequence."""
import numpy as np
import pytest
import torch

import oracle
from parity import TOL, record, rel_err, to_np
from selective_state_space_20_b200 import binding, inputs, seqpar

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("softplus,bias", [(True, True), (False, True), (True, False)])
def test_delta_sum(dtype, softplus, bias):
    w = inputs.custom(3, 33, 1000, 16, dtype, seed=4)
    cpu = inputs.scan_inputs(w)
    b = cpu["delta_bias"] if bias else None
    got = binding.mamba_delta_sum(cpu["delta"].cuda(), None if b is None else b.cuda(), softplus)
    x = cpu["delta"].double().numpy() + (0.0 if b is None else b.double().numpy()[None, :, None])
    ref = (np.logaddexp(0.0, x) if softplus else x).sum(axis=-1)
    assert got.dtype == torch.float64
    assert np.max(np.abs(got.cpu().numpy() - ref)) <= 1e-6 * np.max(np.abs(ref))


@pytest.mark.parametrize("count", [0, 1, 5])
@pytest.mark.parametrize("with_init", [False, True])
def test_state_fold(count, with_init):
    g = torch.Generator().manual_seed(count + 10 * with_init)
    batch, dim, N = 2, 40, 16
    A = -torch.rand(dim, N, generator=g) * 3 - 0.1
    sums = torch.rand(count, batch, dim, generator=g, dtype=torch.float64) * 5
    hl = torch.randn(count, batch, dim, N, generator=g)
    h0 = torch.randn(batch, dim, N, generator=g) if with_init else None
    got = binding.mamba_state_fold(A.cuda(), sums.cuda(), hl.cuda(), None if h0 is None else h0.cuda())
    h = np.zeros((batch, dim, N)) if h0 is None else h0.double().numpy()
    for k in range(count):
        h = np.exp(A.double().numpy()[None] * sums[k].numpy()[:, :, None]) * h + hl[k].double().numpy()
    assert np.max(np.abs(got.cpu().double().numpy() - h)) <= 1e-6 * max(1.0, np.max(np.abs(h)))
    # in place over the initial state
    if with_init and count:
        st = h0.cuda()
        binding.mamba_state_fold(A.cuda(), sums.cuda(), hl.cuda(), st, out=st)
        assert torch.equal(st, got)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("shards", [2, 4])
def test_sequence_split_one_device(dtype, shards):
    w = inputs.custom(2, 64, 4096, 16, dtype, seed=30 + shards)
    cpu = inputs.scan_inputs(w)
    dev = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    h0 = inputs.initial_state(w.batch, w.dim, w.dstate, seed=9).cuda()
    bounds = [w.seqlen * k // shards for k in range(shards + 1)]
    seq = ("u", "delta", "z", "B", "C")
    parts = [{k: (v[..., bounds[k2]:bounds[k2 + 1]].contiguous() if k in seq else v) for k, v in dev.items()}
             for k2 in range(shards)]
    summ = [seqpar.shard_summary(**pt) for pt in parts]
    all_sums = torch.stack([s for s, _ in summ])
    all_h = torch.stack([h for _, h in summ])
    outs = []
    for r, pt in enumerate(parts):
        h_in = seqpar.shard_initial_state(dev["A"], all_sums, all_h, r, h0)
        o, last = seqpar.shard_outputs(**pt, h_in=h_in)
        outs.append(o)
    torch.cuda.synchronize()
    ro, rs = oracle.scan(cpu["u"], cpu["delta"], cpu["A"], cpu["B"], cpu["C"], D=cpu["D"], z=cpu["z"],
                         delta_bias=cpu["delta_bias"], h0=h0.cpu())
    tol = TOL[inputs.DTYPES[dtype]]
    e_out = rel_err(to_np(torch.cat(outs, dim=-1)), ro)
    e_state = rel_err(to_np(last), rs)
    record(f"sequence split x{shards} {w.name}", out=e_out, state=e_state)
    assert e_out <= tol and e_state <= tol, (e_out, e_state)
