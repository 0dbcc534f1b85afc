"""Golden fixtures and the seeded input generators (CPU only)."""
import math
import os

import numpy as np
import pytest
import torch

from selective_state_space_20_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_model_table():
    rows = {}
    for line in open(os.path.join(GOLDEN, "model_table.txt")):
        if line.startswith("#") or not line.strip():
            continue
        name, layers, d_model = line.split()
        rows[name] = (int(layers), int(d_model))
    return rows


def read_oracle_tiny():
    data = {}
    lines = [ln for ln in open(os.path.join(GOLDEN, "oracle_tiny.txt")) if not ln.startswith("#")]
    for i in range(0, len(lines), 2):
        name, *shape = lines[i].split()
        vals = np.array([float(v) for v in lines[i + 1].split()])
        data[name] = vals.reshape([int(s) for s in shape])
    return data


def test_workload_shapes_follow_model_table():
    """Channel counts are d_inner = 2 * d_model of the published model sizes."""
    t = read_model_table()
    assert inputs.MAMBA_130M.dim == 2 * t["130M"][1]
    assert inputs.MAMBA_2_8B.dim == 2 * t["2.8B"][1]
    assert inputs.DECODE.dim == 2 * t["2.8B"][1]
    for w in (inputs.TINY_FP32, inputs.MAMBA_130M, inputs.MAMBA_2_8B,
              inputs.LONG_CONTEXT):
        assert w.dstate == 16


def test_oracle_regression_fixture():
    """The oracle still reproduces the outputs stored by make_golden.py."""
    import oracle
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(GOLDEN, "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    g = read_oracle_tiny()
    out, last = oracle.scan(**mg.problem(), delta_softplus=True)
    np.testing.assert_allclose(out, g["out"], rtol=1e-14, atol=1e-300)
    np.testing.assert_allclose(last, g["last_state"], rtol=1e-14, atol=1e-300)


@pytest.mark.parametrize("w", [inputs.TINY_FP32, inputs.custom(2, 40, 77, 16, "bf16", seed=3)])
def test_scan_inputs_recipe(w):
    a = inputs.scan_inputs(w)
    b = inputs.scan_inputs(w)
    for k in a:
        if a[k] is None:
            assert b[k] is None
            continue
        assert torch.equal(a[k], b[k]), f"{k} not deterministic"
        assert a[k].is_contiguous()
    dt = inputs.DTYPES[w.dtype]
    assert a["u"].shape == (w.batch, w.dim, w.seqlen) and a["u"].dtype == dt
    assert a["B"].shape == (w.batch, w.dstate, w.seqlen) and a["B"].dtype == dt
    assert a["A"].dtype == torch.float32 and a["D"].dtype == torch.float32
    # A = -(n + 1) for every channel (S4D-real)
    assert torch.equal(a["A"], -torch.arange(1, w.dstate + 1, dtype=torch.float32).expand(w.dim, -1))
    # softplus(bias) lands in [dt_min, dt_max] (logaddexp(0, x) = ln(1 + e^x))
    sp = np.logaddexp(0.0, a["delta_bias"].double().numpy())
    assert sp.min() >= w.dt_min * (1 - 1e-5) and sp.max() <= w.dt_max * (1 + 1e-5)


def test_d_modes():
    a = inputs.scan_inputs(inputs.custom(1, 1000, 8, d_mode="uniform", seed=1))
    assert 0.5 <= a["D"].min() and a["D"].max() <= 1.5 and abs(a["D"].mean() - 1) < 0.05
    b = inputs.scan_inputs(inputs.custom(1, 10, 8, d_mode="ones", seed=1))
    assert torch.equal(b["D"], torch.ones(10))


def test_decode_inputs_match_scan_layout():
    w = inputs.DecodeWorkload("t", 3, 5, 4, 6, "bf16", 1e-3, 1e-1, "uniform", seed=9)
    d = inputs.decode_inputs(w)
    s = inputs.decode_as_scan(d)
    assert s["u"].shape == (3, 5, 6) and s["B"].shape == (3, 4, 6)
    for t in range(6):
        assert torch.equal(s["u"][:, :, t], d["u"][t])
        assert torch.equal(s["C"][:, :, t], d["C"][t])


def test_distribution_moments():
    w = inputs.custom(2, 64, 4096, seed=5)
    a = inputs.scan_inputs(w)
    assert abs(a["u"].float().std().item() - 1.0) < 0.01
    assert abs(a["delta"].float().std().item() - 0.5) < 0.01
    dt = np.logaddexp(0.0, a["delta_bias"].double().numpy())
    # log-uniform: log(dt) spread over [log 1e-3, log 1e-1]
    assert math.log(1e-3) - 1e-6 <= np.log(dt).min() and np.log(dt).max() <= math.log(1e-1) + 1e-6


def test_complex_conv_and_state_recipes():
    """The generators of the further rows: shapes, dtypes and the stated
    distributions (complex A = -1/2 + i pi n, B and C with unit mean square
    magnitude; conv taps within +-1/sqrt(K); initial states with spread 1/4);
    deterministic under a seed."""
    c = inputs.complex_inputs(2, 8, 512, 16, "bf16", seed=3)
    assert c["A"].shape == (8, 16, 2) and c["A"].dtype == torch.float32
    assert torch.all(c["A"][..., 0] == -0.5)
    assert torch.allclose(c["A"][0, :, 1], math.pi * torch.arange(16, dtype=torch.float32))
    assert c["B"].shape == (2, 16, 512, 2) and c["B"].dtype == torch.bfloat16
    ms = (c["B"].float() ** 2).sum(-1).mean().item()
    assert 0.9 < ms < 1.1
    c2 = inputs.complex_inputs(2, 8, 512, 16, "bf16", seed=3)
    assert all(torch.equal(c[k], c2[k]) for k in ("u", "delta", "B", "C", "A"))
    k = inputs.conv_inputs(2, 8, 64, width=3, dtype="fp32", seed=4)
    assert k["xz"].shape == (2, 16, 64) and k["weight"].shape == (8, 3)
    assert k["weight"].abs().max().item() <= 1 / math.sqrt(3)
    h = inputs.initial_state(4, 256, 16, seed=5)
    assert h.shape == (4, 256, 16) and 0.22 < h.std().item() < 0.28
