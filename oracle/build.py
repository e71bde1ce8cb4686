"""Build the oracle's C scan into ``oracle/libgdn_oracle.so``.

TEST INFRASTRUCTURE ONLY: the shared object built here is loaded by tests,
``__graft_entry__.smoke()`` and bench.py's CPU-baseline/reference leg, never by
the product library.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gdn_scan.c")
LIB = os.path.join(HERE, "libgdn_oracle.so")


def build(force: bool = False) -> str:
    """Compile the fp64 scan with gcc -O2 -fopenmp; return the library path."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
