#!/usr/bin/env python3
"""Benchmark of the selective-scan forward pass on B200.

One "step" is one fused scan launch (softplus -> discretisation -> recurrence
-> readout -> D skip -> silu gate -> last state) over the Mamba-2.8B layer
shape: batch 4, 5120 channels (d_model 2560, expand 2), L = 4096, N = 16,
bf16 activations, fp32 state and arithmetic, through the C ABI's
mamba_scan_fwd (no workspace).  Inputs are synthetic and seeded, resident in
HBM, and larger than L2 (504 MB of u/delta/z), so no L2 flush is needed
between steps.  Sections beside the headline time the same call on the
Mamba-130M layer and the long-context shape, the workspace entry point, the
decode step, the conv1d prologue, the backward and the complex mode.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

prints one JSON line (rank 0).  For N > 1 (torchrun, one process per GPU) every
rank runs its own problem of the same shape (weak scaling: the (batch,
channel) recurrences are independent, there is no data-path collective); the
time is the max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from selective_state_space_20_b200 import binding, inputs  # noqa: E402

WORKLOAD = inputs.MAMBA_2_8B
METRIC = "scan fwd Gelem/s (batch·dim·L) and % of HBM/MUFU roofline on 1 B200"
UNIT = "Gelem/s"

# Roofline denominators.  MUFU ex2 throughput is 16 results per clock per SM
# (CUDA arithmetic-throughput table for compute capability 10.0); one ex2 per
# (element, state) is the algorithmic exp count.  HBM peak is the measured copy
# bandwidth of this GPU type.
SM_COUNT = 148
MUFU_PER_CLK_PER_SM = 16
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return {"hbm_gbs": float(p["hbm_gbs"]), "sm_max_mhz": float(p["sm_max_mhz"]), "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS, source="fallback")


def algorithmic_bytes(w) -> int:
    """Bytes the scan must move at least once: u, delta, z read, out written
    (act dtype), B and C read once, A/D/bias read, last_state written."""
    es = 2 if w.dtype == "bf16" else 4
    x = w.batch * w.dim * w.seqlen * es
    bc = 2 * w.batch * w.dstate * w.seqlen * es
    params = (w.dim * w.dstate + 2 * w.dim) * 4
    state = w.batch * w.dim * w.dstate * 4
    return 4 * x + bc + params + state


# The sources each benchmarked kernel is built from (its file, the headers it
# includes and the host code that plans its launch): a committed DRAM-traffic
# record stays valid until one of them changes.
KERNEL_SOURCES = {
    "scan_fwd_pairs_kernel": ("scan_fwd_persistent_pairs.cu", "persistent_common.cuh", "persistent_kernels.h",
                              "persistent_host.cu", "device_math.cuh", "internal.h"),
    "scan_fwd_spec_kernel": ("scan_fwd_persistent_spec.cu", "persistent_common.cuh", "persistent_kernels.h",
                             "persistent_host.cu", "device_math.cuh", "internal.h"),
    "scan_fwd_kernel": ("scan_fwd.cu", "device_math.cuh", "internal.h"),
    "scan_fwd_complex_kernel": ("scan_fwd_complex.cu", "device_math.cuh", "internal.h"),
    "scan_bwd_kernel": ("scan_bwd.cu", "device_math.cuh", "internal.h"),
    "state_update_lanes_kernel": ("state_update.cu", "device_math.cuh", "internal.h"),
    "conv1d_tiles_kernel": ("conv1d.cu", "device_math.cuh", "internal.h"),
}


def source_hash(kernel: str = "scan_fwd_pairs_kernel") -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "selective_state_space_20_b200", "csrc")
    for name in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(csrc, name), "rb") as fh:
            h.update(name.encode() + fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel_key: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as fh:
            rec = json.load(fh)
        e = rec.get(kernel_key)
        if e and e.get("source_hash") == source_hash(kernel_key.split(" ")[0]):
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.marks = {}

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, name):
        self.marks[name] = time.time()

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0=None, t1=None):
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            rows.append((ts, parts))
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"], "samples": 0}
        inside = [r for r in rows if (t0 is None or r[0] >= t0) and (t1 is None or r[0] <= t1)]
        use = inside if inside else rows
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(p[1]) for _, p in use if num(p[1]) is not None]
        mx = [num(p[2]) for _, p in use if num(p[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, p in use for i in range(4) if p[5 + i].lower() == "active"})
        pw = [num(p[3]) for _, p in use if num(p[3]) is not None]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(use),
                "samples_in_timed_region": len(inside),
                "power_w_max": max(pw) if pw else None}


class NvmlSampler:
    """SM clock and clock-event reasons read through NVML every ~1 ms in a
    thread: the timed region of a short run (tens of ms) is far shorter than
    nvidia-smi's sampling period."""
    # NVML clock-event reason bits
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device: torch.device):
        self.samples = []
        self.handle = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self.nvml = pynvml
        except Exception:
            self.handle = None

    def start(self):
        if self.handle is None:
            return
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                except AttributeError:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.handle)
                self.samples.append((time.time(), sm, mx, rs))
            except Exception:
                return
            time.sleep(0.001)

    def stop(self):
        self._stop.set()

    def summary(self, t0, t1):
        inside = [x for x in self.samples if t0 <= x[0] <= t1]
        if not inside:
            return None
        sm = [x[1] for x in inside]
        reasons = sorted({name for x in inside for bit, name in self.REASONS.items() if x[3] & bit})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(x[2] for x in inside),
                "sm_mhz_min": min(sm), "reasons": reasons, "samples": len(inside), "source": "nvml"}


# ------------------------------------------------------------ distributed
def dist_setup():
    # NCCL's own log lines (its version at communicator set-up) go to stderr:
    # stdout carries the one JSON line
    os.environ.setdefault("NCCL_DEBUG_FILE", "/dev/stderr")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------ oracle timing
def _oracle_run(data, cores):
    import oracle
    t0 = time.perf_counter()
    oracle.scan(data["u"], data["delta"], data["A"], data["B"], data["C"], D=data["D"],
                z=data["z"], delta_bias=data["delta_bias"], nthreads=cores)
    return time.perf_counter() - t0


def oracle_sample(w, seconds: float):
    """A sub-problem of the workload sized for about `seconds` of oracle time
    on this host's cores: every batch row, the first k channels, full L (the
    whole workload when it fits).  Returns (inputs, k)."""
    cores = os.cpu_count() or 1
    probe = max(cores * 4, 64)
    cal = inputs.scan_inputs(dataclasses.replace(w, batch=1, dim=min(probe, w.dim)))
    rate = min(probe, w.dim) * w.seqlen / max(_oracle_run(cal, cores), 1e-6)  # elements/s
    k = int(rate * seconds / (w.batch * w.seqlen))
    k = max(1, min(w.dim, k))
    return inputs.scan_inputs(dataclasses.replace(w, dim=k)), k


def oracle_beside(kind: str, w, k: int = 32):
    """The fp64 oracle of one section timed on this host's cores on a fixed
    sample (every batch row, the first k channels, full L), for the section's
    line: Gelem/s as the section counts elements."""
    import oracle
    cores = os.cpu_count() or 1
    sw = dataclasses.replace(w, dim=min(k, w.dim))
    elems = sw.batch * sw.dim * sw.seqlen
    if kind == "scan":
        d = inputs.scan_inputs(sw)
        t0 = time.perf_counter()
        oracle.scan(d["u"], d["delta"], d["A"], d["B"], d["C"], D=d["D"], z=d["z"], delta_bias=d["delta_bias"],
                    nthreads=cores)
    elif kind == "backward":
        d = inputs.scan_inputs(sw)
        g = torch.Generator().manual_seed(7)
        dout = torch.randn(sw.batch, sw.dim, sw.seqlen, generator=g)
        t0 = time.perf_counter()
        oracle.scan_bwd(dout, d["u"], d["delta"], d["A"], d["B"], d["C"], D=d["D"], z=d["z"],
                        delta_bias=d["delta_bias"], nthreads=cores)
    elif kind == "complex":
        d = inputs.complex_inputs(sw.batch, sw.dim, sw.seqlen, sw.dstate, sw.dtype)
        t0 = time.perf_counter()
        oracle.scan_complex(d["u"], d["delta"], d["A"], d["B"], d["C"], D=d["D"], z=d["z"],
                            delta_bias=d["delta_bias"], nthreads=cores)
    else:  # conv1d
        d = inputs.conv_inputs(sw.batch, sw.dim, sw.seqlen, 4, sw.dtype, wide=False)
        t0 = time.perf_counter()
        oracle.conv1d(d["x"], d["weight"], d["bias"])
    dt = time.perf_counter() - t0
    return {"value": elems / dt / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"all {sw.batch} batch rows, first {sw.dim} channels, full L={sw.seqlen}: "
                      f"{elems} elements in {dt:.2f} s"}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(w, seconds=25.0):
    cores = os.cpu_count() or 1
    data, k = oracle_sample(w, seconds)
    dt = _oracle_run(data, cores)
    elems = w.batch * k * w.seqlen
    what = "the whole workload" if k == w.dim else f"all {w.batch} batch rows, first {k} of {w.dim} channels"
    # one thread on a small fixed sample (best of 3), for the per-core rate
    k1 = min(64, w.dim)
    one = inputs.scan_inputs(dataclasses.replace(w, batch=1, dim=k1))
    dt1 = min(_oracle_run(one, 1) for _ in range(3))
    return {"value": elems / dt / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{what}, full L={w.seqlen}, N={w.dstate}: {elems} elements in {dt:.2f} s "
                      f"(fp64 C loop over {cores} threads)",
            "cpu_model": cpu_model(),
            "single_thread": {"value": k1 * w.seqlen / dt1 / 1e9, "unit": UNIT,
                              "sample": f"1 batch row, first {k1} channels, full L={w.seqlen}, "
                                        f"best of 3 runs on 1 thread"}}


def run_reference(args, world, rank):
    """The reference arm: the fp64 oracle, as it stands, on the host cores.
    Each step runs a bounded sample of the workload (every batch row, the
    first k channels, full L) sized so the whole run takes a few minutes."""
    if rank != 0:
        return 0
    w = WORKLOAD
    cores = os.cpu_count() or 1
    per_step = max(0.05, 150.0 / max(1, args.steps + args.warmup))
    data, k = oracle_sample(w, per_step)
    for _ in range(args.warmup):
        _oracle_run(data, cores)
    times = [_oracle_run(data, cores) for _ in range(args.steps)]
    tot = sum(times)
    elems = w.batch * k * w.seqlen * args.steps
    value = elems / tot / 1e9
    sample = f"all {w.batch} batch rows, first {k} of {w.dim} channels, full L={w.seqlen}, N={w.dstate} per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "dim": w.dim, "seqlen": w.seqlen,
                       "dstate": w.dstate, "act_dtype": w.dtype, "sample_per_step": sample},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample, "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------ GPU timing
_WS = {}


def workspace_for(w, device):
    key = (w.batch, w.dim, w.seqlen, w.dstate, w.dtype, str(device))
    if key not in _WS:
        n = binding.mamba_scan_workspace_size(w.batch, w.dim, w.seqlen, w.dstate, inputs.DTYPES[w.dtype])
        _WS[key] = torch.empty(max(n, 16), device=device, dtype=torch.uint8)
    return _WS[key]


def scan_call(ins, out, last, ws=None):
    binding.mamba_scan_fwd(ins["u"], ins["delta"], ins["A"], ins["B"], ins["C"], D=ins["D"],
                           z=ins["z"], delta_bias=ins["delta_bias"], out=out, last_state=last,
                           workspace=ws)


def time_device(w, ins, steps, warmup):
    out = torch.empty_like(ins["u"])
    last = torch.empty(w.batch, w.dim, w.dstate, device=ins["u"].device)
    for _ in range(warmup):
        scan_call(ins, out, last)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    return out, last, starts, ends, stream


def e2e_measure(w, dev_ins, steps):
    """Same metric through the C ABI from pinned HOST buffers
    (mamba_scan_fwd_host): every step copies that step's inputs host->device,
    scans, and copies the output and final state back to the host; the
    library pipelines those copies with the scans chunk by chunk."""
    host = {k: dev_ins[k].to("cpu").pin_memory() for k in ("u", "delta", "z", "B", "C")}
    out_h = torch.empty(dev_ins["u"].shape, dtype=dev_ins["u"].dtype).pin_memory()
    last_h = torch.empty(w.batch, w.dim, w.dstate).pin_memory()
    scratch = torch.empty(binding.load_library().mamba_scan_host_scratch_size(
        w.batch, w.dim, w.seqlen, w.dstate, 1 if w.dtype == "bf16" else 0), device=dev_ins["u"].device,
        dtype=torch.uint8)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_h.numel() * out_h.element_size() + last_h.numel() * 4

    def one():
        binding.mamba_scan_fwd_host(host["u"], host["delta"], dev_ins["A"], host["B"], host["C"], D=dev_ins["D"],
                                    z=host["z"], delta_bias=dev_ins["delta_bias"], out=out_h, last_state=last_h,
                                    scratch=scratch)

    one()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        one()
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    return ms, h2d, d2h


def _median_us(fn, reps, warmup=3):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in ev:
        a.record(st)
        fn()
        b.record(st)
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in ev) * 1e3


def scan_kernel_name(lanes, sched):
    if sched in (binding.SCHEDULE_PERSISTENT, binding.SCHEDULE_LOCAL):
        return "scan_fwd_pairs_kernel" if lanes > 1 else "scan_fwd_spec_kernel"
    return "scan_fwd_kernel"


SCHED_NAMES = {1: "static", 2: "persistent (device-wide, workspace)", 3: "local (block per SM, no workspace)"}


def layer_measure(w, reps, oracle_k, cpu_oracle=True):
    """One more Mamba-layer shape through mamba_scan_fwd (no workspace):
    median CUDA-event time of `reps` launches (inputs larger than L2, or
    re-read from L2 at most once per launch: see `l2`), Gelem/s, algorithmic
    GB/s, the MUFU roofline, and the oracle on a fixed sample of the shape."""
    dev = torch.device("cuda", torch.cuda.current_device())
    ins = inputs.scan_inputs(w, device=dev)
    out = torch.empty_like(ins["u"])
    last = torch.empty(w.batch, w.dim, w.dstate, device=dev)
    us = _median_us(lambda: scan_call(ins, out, last), reps)
    peaks = load_peaks()
    mufu = MUFU_PER_CLK_PER_SM * SM_COUNT * peaks["sm_max_mhz"] * 1e6 / w.dstate / 1e9
    gel = w.elements / (us * 1e-6) / 1e9
    alg = algorithmic_bytes(w)
    lanes, threads, sched = binding.mamba_scan_plan(w.batch, w.dim, w.seqlen, w.dstate, inputs.DTYPES[w.dtype],
                                                    workspace=False)
    kernel = scan_kernel_name(lanes, sched)
    if binding.device_status() != 0:
        raise SystemExit(f"{w.name}: the scan reported a timeout")
    act_bytes = 3 * w.elements * (2 if w.dtype == "bf16" else 4)
    sec = {"workload": w.name, "entry": "mamba_scan_fwd", "us_per_call": us, "value": gel, "unit": UNIT,
           "reps": reps, "gbs": alg / (us * 1e-6) / 1e9,
           "l2": "inputs larger than L2" if act_bytes > 126e6 else
                 f"inputs {act_bytes / 1e6:.0f} MB: may stay partly in L2 between launches",
           "launch": {"schedule": SCHED_NAMES.get(sched, sched), "lanes_per_channel": lanes,
                      "threads_per_block": threads},
           "roofline": {"bound": "alu", "achieved": gel, "peak": mufu, "unit": UNIT, "frac": gel / mufu,
                        "kernel": kernel, "traffic": measured_traffic(f"{kernel} {w.name}"),
                        "hbm": {"algorithmic_bytes_per_launch": alg, "frac": alg / (us * 1e-6) / 1e9 /
                                peaks["hbm_gbs"]}}}
    ws = workspace_for(w, dev)
    us_ws = _median_us(lambda: scan_call(ins, out, last, ws), reps)
    if binding.workspace_status(ws) != 0:
        raise SystemExit(f"{w.name}: the persistent scan reported a timeout")
    lw, tw, sw = binding.mamba_scan_plan(w.batch, w.dim, w.seqlen, w.dstate, inputs.DTYPES[w.dtype])
    gws = w.elements / (us_ws * 1e-6) / 1e9
    sec["with_workspace"] = {"entry": "mamba_scan_fwd_ws", "us_per_call": us_ws, "value": gws, "unit": UNIT,
                             "frac": gws / mufu, "workspace_bytes": ws.numel(),
                             "launch": {"schedule": SCHED_NAMES.get(sw, sw), "lanes_per_channel": lw,
                                        "threads_per_block": tw}}
    del ins, out, last, ws
    torch.cuda.empty_cache()
    if cpu_oracle:
        sec["cpu_oracle"] = oracle_beside("scan", w, k=oracle_k)
    return sec


def page_layout_measure(w, ins, reps, headline_us):
    """The benchmark layer in the pages' own layout -- (batch, L, dim)
    activations, (batch, L, N) B / C -- through mamba_scan_fwd_strided (the
    block-local kernel with channel-last staging), beside the headline's
    dense call."""
    cl = {k: (v.transpose(1, 2).contiguous().transpose(1, 2) if k in ("u", "delta", "z", "B", "C") else v)
          for k, v in ins.items()}
    out = torch.empty((w.batch, w.seqlen, w.dim), device=cl["u"].device, dtype=cl["u"].dtype).transpose(1, 2)
    last = torch.empty(w.batch, w.dim, w.dstate, device=cl["u"].device)
    run = lambda: binding.mamba_scan_fwd_strided(cl["u"], cl["delta"], cl["A"], cl["B"], cl["C"], D=cl["D"],  # noqa: E731
                                                 z=cl["z"], delta_bias=cl["delta_bias"], out=out,
                                                 last_state=last)
    us = _median_us(run, reps)
    if binding.device_status() != 0:
        raise SystemExit("page-layout scan reported a timeout")
    gel = w.elements / (us * 1e-6) / 1e9
    mufu = MUFU_PER_CLK_PER_SM * SM_COUNT * load_peaks()["sm_max_mhz"] * 1e6 / w.dstate / 1e9
    del cl, out, last
    torch.cuda.empty_cache()
    return {"workload": f"{w.name}, (b, l, d) activations and (b, l, n) B / C", "entry": "mamba_scan_fwd_strided",
            "us_per_call": us, "value": gel, "unit": UNIT, "frac": gel / mufu, "reps": reps,
            "vs_dense": us / headline_us, "l2": "inputs larger than L2, no flush"}


def workspace_measure(w, ins, reps):
    """The Mamba-2.8B layer through mamba_scan_fwd_ws (caller workspace,
    device-wide persistent schedule) beside the headline's no-workspace call."""
    out = torch.empty_like(ins["u"])
    last = torch.empty(w.batch, w.dim, w.dstate, device=ins["u"].device)
    ws = workspace_for(w, ins["u"].device)
    us = _median_us(lambda: scan_call(ins, out, last, ws), reps)
    if binding.workspace_status(ws) != 0:
        raise SystemExit("persistent scan reported a timeout")
    lanes, threads, sched = binding.mamba_scan_plan(w.batch, w.dim, w.seqlen, w.dstate, inputs.DTYPES[w.dtype])
    return {"entry": "mamba_scan_fwd_ws", "us_per_call": us, "value": w.elements / (us * 1e-6) / 1e9,
            "unit": UNIT, "reps": reps, "workspace_bytes": ws.numel(),
            "launch": {"schedule": SCHED_NAMES.get(sched, sched), "lanes_per_channel": lanes,
                       "threads_per_block": threads}}


def decode_measure(steps=256):
    """Per-token cost of mamba_state_update on the decoding shape (256 x 5120,
    N = 16, fp32 state in HBM), captured in a CUDA graph of `steps` calls."""
    w = inputs.DECODE
    d = inputs.decode_inputs(w, device="cuda", steps=steps)
    state = torch.zeros(w.batch, w.dim, w.dstate, device="cuda")
    outs = torch.empty(steps, w.batch, w.dim, device="cuda", dtype=inputs.DTYPES[w.dtype])

    def run():
        for t in range(steps):
            binding.mamba_state_update(state, d["u"][t], d["delta"][t], d["A"], d["B"][t], d["C"][t],
                                       D=d["D"], z=d["z"][t], delta_bias=d["delta_bias"], out=outs[t])
    run()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            run()
    torch.cuda.current_stream().wait_stream(s)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 4
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (reps * steps)
    bytes_step = w.batch * w.dim * (2 * w.dstate * 4 + 4 * 2) + 2 * w.batch * w.dstate * 2 + w.dim * (w.dstate + 2) * 4
    del g
    # the same step with L2 flushed before it: a read of twice the L2 size
    # (a read leaves no dirty lines behind for the step to write back), each
    # step timed alone with events around it; the flush is queued ahead, so
    # the events bracket the kernel itself.  The step's own writes partly
    # drain to HBM after it ends, as with any one-kernel timing; the graph
    # above includes them (each step pays for the previous one's).
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    flush = torch.ones(2 * l2 // 4, dtype=torch.float32, device="cuda")
    acc = torch.zeros(1, device="cuda")
    evs = []
    for t in range(32):
        torch.sum(flush, dim=0, keepdim=True, out=acc)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        binding.mamba_state_update(state, d["u"][t], d["delta"][t], d["A"], d["B"][t], d["C"][t],
                                   D=d["D"], z=d["z"][t], delta_bias=d["delta_bias"], out=outs[t])
        b.record()
        evs.append((a, b))
    torch.cuda.synchronize()
    cold = sorted(a.elapsed_time(b) * 1e3 for a, b in evs)
    del flush
    us_cold = cold[len(cold) // 2]
    hbm = load_peaks()["hbm_gbs"]
    return {"workload": w.name, "us_per_step": us, "Gelem_per_s": w.batch * w.dim / us / 1e3,
            "GB_per_s": bytes_step / us / 1e3, "algorithmic_bytes_per_step": bytes_step,
            "hbm_frac": bytes_step / us / 1e3 / hbm, "graph_of_steps": steps,
            "note": "back-to-back steps in a CUDA graph: each step also pays for the write-back of the previous "
                    "one's state; the state (84 MB) can stay partly L2-resident",
            "traffic": measured_traffic(f"state_update_lanes_kernel {w.name}"),
            "l2_flushed": {"us_per_step": us_cold, "GB_per_s": bytes_step / us_cold / 1e3,
                           "hbm_frac": bytes_step / us_cold / 1e3 / hbm,
                           "note": f"median of 32 steps, each after a {2 * l2 >> 20} MB read, the kernel timed "
                                   "alone with events (flush queued ahead)"}}


def conv1d_measure(reps=20):
    """The causal depthwise conv1d (+ bias + silu) that produces u, on the
    benchmark layer's shape: x = the first 5120 channel rows of a
    (4, 10240, 4096) bf16 projection output, width 4.  HBM-bound stream:
    x read once (168 MB) and out written once (168 MB) per call."""
    w = inputs.MAMBA_2_8B
    K = 4
    d = inputs.conv_inputs(w.batch, w.dim, w.seqlen, K, w.dtype, seed=44, device="cuda")
    out = torch.empty(w.batch, w.dim, w.seqlen, device="cuda", dtype=inputs.DTYPES[w.dtype])
    run = lambda: binding.mamba_conv1d_fwd(d["xz"], d["weight"], d["bias"], dim=w.dim, out=out)  # noqa: E731
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        run()
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / reps
    es = 2 if w.dtype == "bf16" else 4
    nbytes = 2 * w.batch * w.dim * w.seqlen * es + w.dim * (K + 1) * 4
    hbm = load_peaks()["hbm_gbs"]

    # the same conv fused into the scan's prologue (x and z read from the
    # projection output), against the conv kernel followed by the scan
    s = inputs.scan_inputs(w, device="cuda")
    xz = d["xz"]
    xz[:, w.dim:] = s["z"]
    z = xz[:, w.dim:]
    ws = torch.empty(binding.mamba_scan_workspace_size(w.batch, w.dim, w.seqlen, w.dstate), device="cuda",
                     dtype=torch.uint8)
    y = torch.empty_like(out)
    last = torch.empty(w.batch, w.dim, w.dstate, device="cuda")

    def fused():
        binding.mamba_scan_fwd_conv(xz, d["weight"], d["bias"], s["delta"], s["A"], s["B"], s["C"], D=s["D"],
                                    z=z, delta_bias=s["delta_bias"], out=y, last_state=last, workspace=ws)

    def separate():
        binding.mamba_conv1d_fwd(xz, d["weight"], d["bias"], dim=w.dim, out=out)
        binding.mamba_scan_fwd(out, s["delta"], s["A"], s["B"], s["C"], D=s["D"], z=s["z"],
                               delta_bias=s["delta_bias"], out=y, last_state=last, workspace=ws)

    def time_us(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, c = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn()
        c.record()
        torch.cuda.synchronize()
        return a.elapsed_time(c) * 1e3 / reps

    us_fused, us_sep = time_us(fused), time_us(separate)
    return {"workload": f"conv1d K={K} {w.batch}x{w.dim}x{w.seqlen} {w.dtype} (x half of a 2x-wide input)",
            "us_per_call": us, "Gelem_per_s": w.elements / us / 1e3,
            "roofline": {"bound": "hbm", "achieved": nbytes / us / 1e3, "peak": hbm, "unit": "GB/s",
                         "frac": nbytes / us / 1e3 / hbm, "algorithmic_bytes": nbytes,
                         "traffic": measured_traffic(f"conv1d_tiles_kernel conv1d K={K} {w.batch}x{w.dim}x{w.seqlen} "
                                                     f"{w.dtype}")},
            "fused_with_scan": {"us_per_call": us_fused, "Gelem_per_s": w.elements / us_fused / 1e3,
                                "separate_conv_then_scan_us": us_sep,
                                "note": "mamba_scan_fwd_conv: u formed in the scan's prologue, never stored"},
            "reps": reps, "l2": "inputs larger than L2, no flush"}


def backward_measure(reps=5):
    """The scan's backward pass on the benchmark layer (Mamba-2.8B shape,
    bf16): every input gradient for a random dL/dout and dL/dlast_state.
    Timed two ways: from the checkpoints the forward keeps (mamba_scan_fwd_ckpt
    then mamba_scan_bwd_ckpt, the training path; the forward's extra cost is
    reported beside) and self-contained (mamba_scan_bwd, which sweeps the
    inputs for its checkpoints first).  The roof counts the decays the
    gradients need at least once (16 per element, N = 16) on the MUFU; the
    kernel evaluates them twice from checkpoints (the 32-step recompute and
    the 4-step window recompute), three times self-contained."""
    w = inputs.MAMBA_2_8B
    d = inputs.scan_inputs(w, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(7)
    dout = torch.randn(w.batch, w.dim, w.seqlen, generator=g, device="cuda").to(inputs.DTYPES[w.dtype])
    dlast = torch.randn(w.batch, w.dim, w.dstate, generator=g, device="cuda")
    ws = torch.empty(binding.load_library().mamba_scan_bwd_workspace_size(w.batch, w.dim, w.seqlen, w.dstate),
                     device="cuda", dtype=torch.uint8)
    kw = dict(D=d["D"], z=d["z"], delta_bias=d["delta_bias"])
    out = torch.empty_like(d["u"])
    last = torch.empty(w.batch, w.dim, w.dstate, device="cuda")
    _, _, ck = binding.mamba_scan_fwd_ckpt(d["u"], d["delta"], d["A"], d["B"], d["C"], out=out, last_state=last, **kw)
    bwd_ck = lambda: binding.mamba_scan_bwd(dout, d["u"], d["delta"], d["A"], d["B"], d["C"],  # noqa: E731
                                            dlast_state=dlast, workspace=ws, ckpt=ck, **kw)
    bwd_self = lambda: binding.mamba_scan_bwd(dout, d["u"], d["delta"], d["A"], d["B"], d["C"],  # noqa: E731
                                              dlast_state=dlast, workspace=ws, **kw)
    fwd = lambda: binding.mamba_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], out=out,  # noqa: E731
                                         last_state=last, **kw)
    fwd_ck = lambda: binding.mamba_scan_fwd_ckpt(d["u"], d["delta"], d["A"], d["B"], d["C"], out=out,  # noqa: E731
                                                 last_state=last, ckpt=ck, **kw)
    us = _median_us(bwd_ck, reps)
    us_self = _median_us(bwd_self, reps)
    us_fwd, us_fwd_ck = _median_us(fwd, 20), _median_us(fwd_ck, 20)
    peak = MUFU_PER_CLK_PER_SM * SM_COUNT * load_peaks()["sm_max_mhz"] * 1e6 / w.dstate / 1e9
    achieved = w.elements / us / 1e3
    return {"workload": w.name, "entry": "mamba_scan_bwd_ckpt (checkpoints from mamba_scan_fwd_ckpt)",
            "us_per_call": us, "Gelem_per_s": achieved,
            "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "Gelem/s",
                         "frac": achieved / peak,
                         "traffic": measured_traffic(f"scan_bwd_kernel {w.name}"),
                         "note": "peak = 16 decays per element once on the MUFU; from checkpoints the kernel "
                                 "evaluates them twice (32-step recompute, 4-step window recompute)"},
            "self_contained": {"entry": "mamba_scan_bwd", "us_per_call": us_self,
                               "Gelem_per_s": w.elements / us_self / 1e3},
            "forward_checkpoint_cost": {"mamba_scan_fwd_us": us_fwd, "mamba_scan_fwd_ckpt_us": us_fwd_ck,
                                        "checkpoint_bytes": ck.numel() * 4},
            "reps": reps, "deterministic": "du, ddelta, dz yes; dA, dB, dC, dD, dbias sum with atomics"}


def complex_measure(reps=10):
    """Complex-valued mode on the benchmark layer's shape (4 x 5120 x 4096,
    N = 16 complex states, bf16 activations; A = -1/2 + i pi n).  Each
    state-step takes three special-function ops (ex2, sin, cos), so the roof
    is the MUFU rate over 3 N ops per element."""
    w = inputs.MAMBA_2_8B
    d = inputs.complex_inputs(w.batch, w.dim, w.seqlen, w.dstate, w.dtype, device="cuda")
    out = torch.empty_like(d["u"])
    last = torch.empty(w.batch, w.dim, w.dstate, 2, device="cuda")
    run = lambda: binding.mamba_scan_fwd_complex(d["u"], d["delta"], d["A"], d["B"], d["C"], D=d["D"],  # noqa: E731
                                                 z=d["z"], delta_bias=d["delta_bias"], out=out,
                                                 last_state=last)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        run()
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / reps
    peak = MUFU_PER_CLK_PER_SM * SM_COUNT * load_peaks()["sm_max_mhz"] * 1e6 / (3 * w.dstate) / 1e9
    achieved = w.elements / us / 1e3
    return {"workload": f"complex mode {w.batch}x{w.dim}x{w.seqlen} N{w.dstate} {w.dtype}",
            "us_per_call": us, "Gelem_per_s": achieved,
            "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "Gelem/s",
                         "frac": achieved / peak,
                         "traffic": measured_traffic(f"scan_fwd_complex_kernel complex mode {w.batch}x{w.dim}x{w.seqlen} "
                                                     f"N{w.dstate} {w.dtype}"),
                         "note": "peak = MUFU ops/s over 3 N (ex2, sin, cos per complex state-step)"},
            "reps": reps, "l2": "inputs larger than L2, no flush"}


def seqpar_shard(w, world, rank, device):
    """This rank's shard of one sequence of workload ``w``: timesteps
    [rank L / world, (rank + 1) L / world), drawn with seed + rank; the
    per-channel parameters (A, D, bias) are the base seed's on every rank."""
    Lr = w.seqlen // world
    shard = inputs.scan_inputs(dataclasses.replace(w, seqlen=Lr, seed=w.seed + rank), device=device)
    params = inputs.scan_inputs(dataclasses.replace(w, batch=1, seqlen=8), device=device)
    for k in ("A", "D", "delta_bias"):
        shard[k] = params[k]
    return shard, Lr


def seqpar_run(w, world, rank, steps, warmup, device, ops=None, group=None):
    """Time `steps` calls of the sequence split (each rank runs its shard
    from zero for its final state alone, the ranks all-gather the shard
    summaries, each folds the shards before it and scans its shard from the
    result) after `warmup` untimed ones; returns
    (max over ranks of the time per step in ms, elements per step of the
    whole sequence).  ``ops`` replaces the per-shard steps (CPU stand-ins in
    the multi-process test)."""
    import torch.distributed as dist
    from selective_state_space_20_b200 import seqpar
    shard, Lr = seqpar_shard(w, world, rank, device)
    run = lambda: seqpar.scan_sequence_parallel(shard["u"], shard["delta"], shard["A"], shard["B"],  # noqa: E731
                                                shard["C"], D=shard["D"], z=shard["z"],
                                                delta_bias=shard["delta_bias"], group=group, _ops=ops)
    for _ in range(warmup):
        run()
    on_gpu = device.type == "cuda"
    if on_gpu:
        torch.cuda.synchronize()
    dist.barrier(group)
    if on_gpu:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
    t0 = time.perf_counter()
    for _ in range(steps):
        run()
    if on_gpu:
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
    else:
        ms = (time.perf_counter() - t0) * 1e3
    dist.barrier(group)
    ms = max_over_ranks(ms, world)
    return ms / steps, w.batch * w.dim * Lr * world


def seqpar_main(args, world, rank, local):
    """--seqpar: the long-context layer as ONE sequence split over the ranks
    (strong scaling: the whole job is one 1 x 2048 x 262144 scan)."""
    if world > 1 and not torch.distributed.is_initialized():
        raise SystemExit("--seqpar with several ranks needs the launcher's process group")
    if world == 1 and not torch.distributed.is_initialized():  # a group of one: the exchange is trivial
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", str(29500 + os.getpid() % 1000))
        dist.init_process_group("nccl", rank=0, world_size=1)
    w = inputs.LONG_CONTEXT
    dev = torch.device("cuda", torch.cuda.current_device())
    binding.load_library()
    ms, elems = seqpar_run(w, world, rank, args.steps, args.warmup, dev)
    if rank == 0:
        line = {"metric": METRIC, "value": elems / (ms * 1e-3) / 1e9, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                "config": {"workload": f"{w.name}, one sequence split over {world} ranks",
                           "batch": w.batch, "dim": w.dim, "seqlen": w.seqlen, "dstate": w.dstate,
                           "act_dtype": w.dtype, "seqlen_per_rank": w.seqlen // world,
                           "exchange": "all-gather of per-shard (delta sums fp64, final states fp32) "
                                       "through torch.distributed, then an fp64 fold",
                           "l2": "inputs larger than L2"},
                "gpu_launches": args.steps * (4 if world > 1 else 3)}
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-conv", action="store_true")
    ap.add_argument("--no-bwd", action="store_true")
    ap.add_argument("--no-complex", action="store_true")
    ap.add_argument("--no-layers", action="store_true", help="skip the Mamba-130M / long-context / workspace sections")
    ap.add_argument("--seqpar", action="store_true",
                    help="time one long-context sequence split over the ranks (seqpar.scan_sequence_parallel)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world, rank, local = dist_setup()
    if args.impl == "reference":
        rc = run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return rc
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    if args.seqpar:
        rc = seqpar_main(args, world, rank, local)
        if torch.distributed.is_initialized():
            torch.distributed.destroy_process_group()
        return rc

    w = WORKLOAD
    dev = torch.device("cuda", torch.cuda.current_device())
    binding.load_library()
    ins = inputs.scan_inputs(dataclasses.replace(w, seed=w.seed + rank), device=dev)
    out, last, starts, ends, stream = time_device(w, ins, args.steps, args.warmup)

    clocks = ClockSampler(local)
    nvml = NvmlSampler(dev)
    if rank == 0:
        clocks.start()
        nvml.start()
        time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    g0 = torch.cuda.Event(enable_timing=True)
    g1 = torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for i in range(args.steps):
        starts[i].record(stream)
        scan_call(ins, out, last)
        ends[i].record(stream)
    g1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    barrier(world)
    total_ms = g0.elapsed_time(g1)
    launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(total_ms, world)
    clk = clocks.summary(t_wall0, t_wall1) if rank == 0 else None
    nvml.stop()
    clocks.stop()
    if rank == 0:
        fast = nvml.summary(t_wall0, t_wall1)
        if fast:  # NVML samples inside the timed region decide; nvidia-smi's kept beside
            clk = dict(fast, nvidia_smi=clk)

    ms_step = total_ms / args.steps
    elems = w.elements
    value = world * elems * args.steps / (total_ms * 1e-3) / 1e9
    peaks = load_peaks()
    avg_launch_ms = sum(launch_ms) / len(launch_ms)
    mufu_peak_gelem = MUFU_PER_CLK_PER_SM * SM_COUNT * peaks["sm_max_mhz"] * 1e6 / w.dstate / 1e9
    achieved = elems / (avg_launch_ms * 1e-3) / 1e9
    alg_bytes = algorithmic_bytes(w)
    lanes, threads, sched = binding.mamba_scan_plan(w.batch, w.dim, w.seqlen, w.dstate, inputs.DTYPES[w.dtype],
                                                    workspace=False)
    if binding.device_status() != 0:
        raise SystemExit("the scan reported a timeout")
    kernel = scan_kernel_name(lanes, sched)
    roof = {"bound": "alu", "achieved": achieved, "peak": mufu_peak_gelem, "unit": UNIT,
            "frac": achieved / mufu_peak_gelem,
            "traffic": measured_traffic(f"{kernel} {w.name}"),
            "peak_source": f"MUFU ex2 16/clk/SM x {SM_COUNT} SMs x {peaks['sm_max_mhz']:.0f} MHz "
                           f"({peaks['source']} sm_max_mhz) / N={w.dstate} exps per element",
            "kernel": kernel, "avg_launch_us": avg_launch_ms * 1e3,
            "hbm": {"algorithmic_bytes_per_launch": alg_bytes,
                    "achieved_gbs": alg_bytes / (avg_launch_ms * 1e-3) / 1e9,
                    "peak_gbs": peaks["hbm_gbs"],
                    "frac": alg_bytes / (avg_launch_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}}
    if clk and clk.get("sm_mhz"):
        roof["frac_at_sampled_clock"] = achieved / (mufu_peak_gelem * clk["sm_mhz"] / peaks["sm_max_mhz"])

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "dim": w.dim, "seqlen": w.seqlen,
                       "dstate": w.dstate, "act_dtype": w.dtype, "state_dtype": "f32",
                       "gate": True, "softplus": True, "emit_last_state": True,
                       "l2": "inputs larger than L2 (3 x 168 MB act tensors), no flush",
                       "entry": "mamba_scan_fwd (C ABI, no workspace)",
                       "launch": {"schedule": SCHED_NAMES.get(sched, sched),
                                  "lanes_per_channel": lanes, "threads_per_block": threads},
                       "per_rank": "independent problem of this shape (seed + rank)"},
            "gpu_launches": args.steps, "roofline": roof, "clocks": clk}

    if rank == 0 and not args.no_e2e:
        e2e_steps = max(3, min(args.steps, 10))
        ms_e2e, h2d, d2h = e2e_measure(w, ins, e2e_steps)
        line["e2e"] = {"value": elems / (ms_e2e * 1e-3) / 1e9, "unit": UNIT,
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "ms_per_step": ms_e2e, "steps": e2e_steps,
                       "path": "mamba_scan_fwd_host: pinned host buffers in and out; copies in, scans and "
                               "copies out pipelined over 16 chunks on three streams"}
    if rank == 0 and not args.no_layers:
        line["with_workspace"] = workspace_measure(w, ins, reps=50)
        line["with_workspace"]["vs_headline"] = line["with_workspace"]["us_per_call"] / (avg_launch_ms * 1e3)
        line["page_layout"] = page_layout_measure(w, ins, reps=30, headline_us=avg_launch_ms * 1e3)
    if rank == 0 and not args.no_decode:
        line["decode"] = decode_measure()
    if rank == 0 and not args.no_conv:
        line["conv1d"] = conv1d_measure()
    if rank == 0 and not args.no_bwd:
        line["backward"] = backward_measure()
    if rank == 0 and not args.no_complex:
        line["complex"] = complex_measure()
    if rank == 0 and not args.no_layers:
        del ins
        torch.cuda.empty_cache()
        with_oracle = world == 1 and not args.no_cpu_baseline
        line["mamba_130m"] = layer_measure(inputs.MAMBA_130M, reps=50, oracle_k=64, cpu_oracle=with_oracle)
        line["long_context"] = layer_measure(inputs.LONG_CONTEXT, reps=5, oracle_k=32, cpu_oracle=with_oracle)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        for key, kind in (("conv1d", "conv1d"), ("backward", "backward"), ("complex", "complex")):
            if key in line:
                line[key]["cpu_oracle"] = oracle_beside(kind, w, k={"conv1d": 1024}.get(kind, 256))
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        barrier(world)
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
