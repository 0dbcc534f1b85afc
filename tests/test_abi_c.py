"""The C ABI from plain C, without a GPU: tests/abi_from_c.c compiles against
include/mamba_scan.h as strict C99 (all warnings errors), links against the
library and runs its host-side checks."""
import os
import shutil
import subprocess

import pytest

from selective_state_space_20_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc is needed to build the C client")
def test_c_client(tmp_path):
    binding.load_library()  # builds the library if it is out of date
    libdir = os.path.dirname(build.LIB)
    libname = os.path.basename(build.LIB)
    exe = str(tmp_path / "abi_from_c")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Wpedantic", "-Werror",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "abi_from_c.c"),
           "-o", exe, "-L", libdir, f"-l:{libname}", f"-Wl,-rpath,{libdir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
