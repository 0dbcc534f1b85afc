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
