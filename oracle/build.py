"""Build the fp64 CPU oracle (test infrastructure) into oracle/libmamba2_oracle.so.

Plain gcc, no -march flags: the library must run on whatever x86-64 host the
tests land on, and no floating-point contraction or fast-math is enabled, so
every double operation is the one written in mamba2_oracle.c.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "mamba2_oracle.c")
LIB = os.path.join(HERE, "libmamba2_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-ffp-contract=off", "-fPIC",
           "-shared", "-pthread", "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
