"""Accuracy of the kernels' softplus and silu, observed through the C ABI.

With A = 0 (Abar = 1), B = C = u = 1, D = 0, zero initial state and no gate,
the first output of the scan is h_0 = delta_0 * B * u = softplus(delta_raw)
exactly in fp32 arithmetic, so it exposes the kernel's softplus alone.  With
softplus off, delta_raw = 1 and a gate, it is 1 * silu(z).  Both are compared
with the oracle's fp64 functions (which are pinned against numpy/scipy).
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_20_b200 import binding

pytestmark = pytest.mark.gpu

SCHEDULES = [dict(schedule=binding.SCHEDULE_PERSISTENT, lanes_per_channel=1),
             dict(schedule=binding.SCHEDULE_PERSISTENT, lanes_per_channel=2),
             dict(schedule=binding.SCHEDULE_PERSISTENT, lanes_per_channel=4),
             dict(schedule=binding.SCHEDULE_STATIC, lanes_per_channel=1),
             dict(schedule=binding.SCHEDULE_STATIC, lanes_per_channel=8),
             dict(schedule=binding.SCHEDULE_STATIC, lanes_per_channel=4, threads_per_block=256)]


def probe(raw, z=None, softplus=True, dtype=torch.float32, L=8, **kw):
    dim = raw.numel()
    dev = "cuda"
    u = torch.ones(1, dim, L, device=dev, dtype=dtype)
    delta = raw.to(dev, dtype).view(1, dim, 1).expand(1, dim, L).contiguous()
    A = torch.zeros(dim, 1, device=dev)
    B = torch.ones(1, 1, L, device=dev, dtype=dtype)
    C = torch.ones(1, 1, L, device=dev, dtype=dtype)
    zz = None if z is None else z.to(dev, dtype).view(1, dim, 1).expand(1, dim, L).contiguous()
    out = binding.mamba_scan_fwd(u, delta, A, B, C, D=None, z=zz, delta_bias=None,
                                 delta_softplus=softplus, **kw)
    return out[0, :, 0].double().cpu().numpy()


@pytest.mark.parametrize("kw", SCHEDULES, ids=lambda k: str(k))
def test_softplus_accuracy(kw):
    raw = torch.cat([torch.linspace(-40, 40, 4001), torch.tensor([-87.0, -20.0, -9.21, 0.0, 20.0, 30.0, 87.0])])
    got = probe(raw, **kw)
    x = raw.double().numpy()
    ref = np.array([oracle.softplus(v) for v in x])
    rel = np.abs(got - ref) / np.maximum(ref, 1e-38)
    # ex2's 2^-22 and the rounding of -|x| log2(e) (relative 2^-24 of |x|)
    bound = 4e-7 + 1.2e-7 * np.abs(x)
    assert np.all(rel <= bound), (x[np.argmax(rel / bound)], rel.max())


@pytest.mark.parametrize("kw", SCHEDULES, ids=lambda k: str(k))
def test_silu_accuracy(kw):
    z = torch.cat([torch.linspace(-30, 30, 3001), torch.tensor([-100.0, -88.0, 0.0, 88.0])])
    got = probe(torch.ones(z.numel()), z=z, softplus=False, **kw)
    ref = np.array([oracle.silu(v) for v in z.double().numpy()])
    err = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)
    small = np.abs(ref) < 1e-30
    assert np.all(err[~small] <= 2e-6), err[~small].max()
    assert np.all(np.abs(got[small]) <= 1e-30)


def test_state_update_pointwise():
    raw = torch.linspace(-30, 30, 2001)
    dim = raw.numel()
    st = torch.zeros(1, dim, 1, device="cuda")
    one = torch.ones(1, dim, device="cuda")
    out = binding.mamba_state_update(st, one, raw.view(1, dim).cuda(), torch.zeros(dim, 1, device="cuda"),
                                     torch.ones(1, 1, device="cuda"), torch.ones(1, 1, device="cuda"))
    got = out[0].double().cpu().numpy()
    ref = np.array([oracle.softplus(v) for v in raw.double().numpy()])
    rel = np.abs(got - ref) / ref
    assert np.all(rel <= 4e-7 + 1.2e-7 * np.abs(raw.double().numpy()))


@pytest.mark.parametrize("kw", SCHEDULES, ids=lambda k: str(k))
@pytest.mark.parametrize("state", [0, 13, 14, 15])
def test_decay_accuracy(kw, state):
    """The decay exp(delta A) of one state, observed through the scan: with
    delta = 1 (softplus off), u = 1, B = 1 at t = 0 and 0 after, C = 1 for the
    probed state at t = 1 and 0 elsewhere, the output at t = 1 is
    exp(A[c, state]) exactly in fp32 arithmetic.  Every state index is probed
    because kernels may compute the decays of different states on different
    units (e.g. a polynomial on the FMA pipe for some of them)."""
    a = torch.cat([torch.linspace(-100, 80, 3601), torch.tensor([-87.0, -86.0, -0.5, 0.0, 1e-6, 0.5])])
    dim, L, N = a.numel(), 8, 16
    dev = "cuda"
    u = torch.ones(1, dim, L, device=dev)
    delta = torch.ones(1, dim, L, device=dev)
    A = torch.zeros(dim, N, device=dev)
    A[:, state] = a.to(dev)
    B = torch.zeros(1, N, L, device=dev)
    B[0, :, 0] = 1.0
    C = torch.zeros(1, N, L, device=dev)
    C[0, state, 1] = 1.0
    out = binding.mamba_scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                                 delta_softplus=False, **kw)
    got = out[0, :, 1].double().cpu().numpy()
    x = a.double().numpy()
    ref = np.exp(x)
    normal = ref >= 2.0 ** -124
    rel = np.abs(got[normal] - ref[normal]) / ref[normal]
    # 2^-22 for the exponential, plus the rounding of A log2(e) (relative 2^-24 of |x|)
    bound = 4e-7 + 1.2e-7 * np.abs(x[normal])
    assert np.all(rel <= bound), (x[normal][np.argmax(rel / bound)], rel.max())
    # beyond fp32's normal range: tiny or zero, never garbage
    assert np.all((got[~normal] >= 0) & (got[~normal] <= 2.0 ** -123))
