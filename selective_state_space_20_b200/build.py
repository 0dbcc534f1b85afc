"""Build ``libmamba_scan.so`` (the C-ABI library) from ``csrc/`` with nvcc for
sm_100a, and on request the bounds-checked build of the same sources,
``libmamba_scan_checked.so`` (MSCAN_BOUNDS_CHECK: see csrc/bounds.cuh).  Both
are built in-tree, next to this file.

Usage:  python -m selective_state_space_20_b200.build [--force] [--verbose] [--checked]
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import hashlib
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libmamba_scan.so")
STAMP = LIB + ".srchash"
BUILD_DIR = os.path.join(HERE, "_build")
CHECKED_LIB = os.path.join(HERE, "libmamba_scan_checked.so")
CHECKED_FLAGS = ["-DMSCAN_BOUNDS_CHECK"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2",
              "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC] + ARCH


def nvcc() -> str:
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build the library")
    return exe


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")) + [__file__]


def _paths(checked: bool):
    """(library, stamp, object directory) of the normal or the checked build."""
    if checked:
        return CHECKED_LIB, CHECKED_LIB + ".srchash", os.path.join(HERE, "_build_checked")
    return LIB, STAMP, BUILD_DIR


def _flags(checked: bool):
    return NVCC_FLAGS + (CHECKED_FLAGS if checked else [])


def source_digest(checked: bool = False) -> str:
    """Hash of every input of the build (sources, headers, flags)."""
    flags = [f for f in _flags(checked) if not os.path.isabs(f)]  # paths differ per checkout
    h = hashlib.sha256(" ".join(flags).encode())
    for p in sorted(_deps()):
        with open(p, "rb") as fh:
            h.update(os.path.relpath(p, ROOT).encode() + b"\0" + fh.read())
    return h.hexdigest()


def up_to_date(checked: bool = False) -> bool:
    """True if the library exists and was built from the current sources."""
    lib, stamp, _ = _paths(checked)
    if not (os.path.exists(lib) and os.path.exists(stamp)):
        return False
    with open(stamp) as fh:
        return fh.read().strip() == source_digest(checked)


def _compile(src: str, verbose: bool, checked: bool = False) -> str:
    obj = os.path.join(_paths(checked)[2], os.path.basename(src) + ".o")
    cmd = [nvcc()] + _flags(checked) + (["-Xptxas", "-v"] if verbose else []) + ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    if verbose:
        sys.stderr.write(r.stderr)
    return obj


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    """Compile every ``csrc/*.cu`` and link ``libmamba_scan.so`` (or, with
    ``checked``, ``libmamba_scan_checked.so``)."""
    lib, stamp, build_dir = _paths(checked)
    if not force and up_to_date(checked):
        return lib
    os.makedirs(build_dir, exist_ok=True)
    srcs = sources()
    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, checked), srcs))
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc()] + ARCH + ["-shared", "-cudart", "static", "-o", tmp] + objs
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    with open(stamp, "w") as fh:
        fh.write(source_digest(checked))
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, checked="--checked" in sys.argv))
