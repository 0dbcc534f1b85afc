"""Parity of the causal depthwise conv1d (+ bias, + silu) and its one-token
update with the fp64 oracle, through the C ABI (GPU)."""
import pytest
import torch

import oracle
from parity import TOL, record, rel_err, sample_rows, to_np
from selective_state_space_20_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def check(batch, dim, L, K, dtype, silu=True, bias=True, wide=True, seed=1):
    cpu = inputs.conv_inputs(batch, dim, L, K, dtype, seed=seed, wide=wide)
    x = cpu["xz"] if wide else cpu["x"]
    b = cpu["bias"] if bias else None
    out = binding.mamba_conv1d_fwd(x.cuda(), cpu["weight"].cuda(), None if b is None else b.cuda(),
                                   apply_silu=silu, dim=dim)
    ref = oracle.conv1d(x, cpu["weight"], b, silu=silu, dim=dim)
    e = rel_err(to_np(out), ref)
    record(f"conv1d {batch}x{dim}x{L} K={K} {dtype} silu={silu} bias={bias} wide={wide}", out=e)
    assert e <= TOL[inputs.DTYPES[dtype]], e


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("K", [1, 2, 3, 4])
@pytest.mark.parametrize("shape", [(2, 37, 333), (3, 64, 1024), (1, 5, 1), (4, 130, 264), (2, 8, 12)])
def test_conv1d_matches_oracle(dtype, K, shape):
    check(*shape, K, dtype, seed=K + sum(shape))


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_conv1d_flags_and_layouts(dtype):
    check(2, 48, 256, 4, dtype, silu=False)
    check(2, 48, 256, 4, dtype, bias=False)
    check(2, 48, 256, 4, dtype, wide=False)


def test_conv1d_unaligned_takes_scalar_path():
    cpu = inputs.conv_inputs(2, 16, 64, 4, "bf16", seed=9, wide=False)
    buf = torch.empty(cpu["x"].numel() + 1, dtype=torch.bfloat16, device="cuda")
    x = buf[1:].view(cpu["x"].shape)
    x.copy_(cpu["x"])
    out = binding.mamba_conv1d_fwd(x, cpu["weight"].cuda(), cpu["bias"].cuda())
    ref = oracle.conv1d(cpu["x"], cpu["weight"], cpu["bias"])
    assert rel_err(to_np(out), ref) <= 2e-2


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("K", [1, 2, 4])
def test_update_stream_equals_sequence(dtype, K):
    """One-token updates from a zero state give the whole-sequence result."""
    batch, dim, L = 3, 40, 24
    cpu = inputs.conv_inputs(batch, dim, L, K, dtype, seed=20 + K, wide=False)
    x, w, b = cpu["x"].cuda(), cpu["weight"].cuda(), cpu["bias"].cuda()
    seq = binding.mamba_conv1d_fwd(x, w, b)
    st = torch.zeros(batch, dim, K - 1, device="cuda") if K > 1 else None
    steps = []
    for t in range(L):
        steps.append(binding.mamba_conv1d_update(st, x[:, :, t].contiguous(), w, b))
    got = torch.stack(steps, dim=2)
    assert torch.equal(got, seq)  # same fp32 operations in the same order
    ref = oracle.conv1d(cpu["x"], cpu["weight"], cpu["bias"])
    assert rel_err(to_np(got), ref) <= TOL[inputs.DTYPES[dtype]]
    if K > 1:  # the state holds the last K-1 inputs, oldest first
        assert torch.equal(st, x[:, :, L - (K - 1):].float())


def test_conv1d_full_size_sampled():
    """The Mamba-2.8B layer shape (x half of a 4 x 10240 x 4096 projection
    output): every output of sampled channel rows against the oracle."""
    batch, dim, L = 4, 5120, 4096
    dev = inputs.conv_inputs(batch, dim, L, 4, "bf16", seed=44, device="cuda")
    out = binding.mamba_conv1d_fwd(dev["xz"], dev["weight"], dev["bias"], dim=dim)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    for r in sample_rows(batch, dim, 24, seed=44):
        b, d = divmod(r, dim)
        x = dev["xz"][b:b + 1, d:d + 1].cpu()
        ref = oracle.conv1d(x, dev["weight"][d:d + 1].cpu(), dev["bias"][d:d + 1].cpu())
        assert rel_err(to_np(out[b:b + 1, d:d + 1]), ref) <= 2e-2, (b, d)
