"""Compile the fp64 CPU oracle (``s6_oracle.c``) into ``libs6_oracle.so``.

Test infrastructure only: the product path never builds against, links or
loads this library.  Compiled with -O2 and without -ffast-math so that the
compiler may not reassociate the fp64 arithmetic.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "s6_oracle.c")
LIB = os.path.join(HERE, "libs6_oracle.so")


def compile_source(src: str, out: str) -> str:
    """Compile one oracle-style C file into a shared library at ``out``."""
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", "-o", out, src, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    return out


def build(force: bool = False) -> str:
    """Build the oracle library if it is missing or older than its source."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    compile_source(SRC, tmp)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
