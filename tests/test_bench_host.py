"""bench.py's host-side arithmetic (CPU only): the algorithmic bytes behind
the HBM roofline, and the rule that a committed DRAM-traffic record is used
only while the kernel's sources are the ones it was captured on."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from selective_state_space_20_b200 import inputs  # noqa: E402


def test_algorithmic_bytes_mamba_2_8b():
    # bf16 4 x 5120 x 4096, N = 16: u, delta, z read and out written (4 x 167,772,160),
    # B and C once (2 x 524,288), A (5120 x 16) + D + bias fp32 (368,640), last_state fp32 (1,310,720)
    assert bench.algorithmic_bytes(inputs.MAMBA_2_8B) == 4 * 167_772_160 + 2 * 524_288 + 368_640 + 1_310_720
    assert abs(bench.algorithmic_bytes(inputs.MAMBA_2_8B) / inputs.MAMBA_2_8B.elements - 8.03) < 0.005


def test_algorithmic_bytes_fp32_doubles_the_activations():
    w = inputs.TINY_FP32  # 1 x 64 x 256, N = 16, fp32
    assert bench.algorithmic_bytes(w) == 4 * 64 * 256 * 4 + 2 * 16 * 256 * 4 + (64 * 16 + 128) * 4 + 64 * 16 * 4


def test_traffic_record_follows_the_sources(monkeypatch):
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as fh:
        records = json.load(fh)
    assert records, "no committed traffic records"
    key, rec = next(iter(records.items()))
    kernel = key.split(" ")[0]
    assert set(rec["sources"]) == set(bench.KERNEL_SOURCES[kernel])
    monkeypatch.setattr(bench, "source_hash", lambda k="": rec["source_hash"])
    assert bench.measured_traffic(key) == float(rec["dram_bytes_per_launch"])
    monkeypatch.setattr(bench, "source_hash", lambda k="": "0" * 16)  # a source changed since the capture
    assert bench.measured_traffic(key) is None
    assert bench.measured_traffic("no such kernel") is None
