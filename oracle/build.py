"""Compile the oracle (plain C, fp64, OpenMP) into ``oracle/_la_oracle.so``.

Test infrastructure: the oracle is the CPU reference the CUDA path is checked
against; it is built with gcc and loaded by ``oracle/__init__.py``.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "la_oracle.c")
LIB = os.path.join(HERE, "_la_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    # -ffp-contract=off: no fused multiply-add contraction, so the fp64 result is
    # the plain sequence of roundings written in the source on every host.
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", SRC, "-o", tmp, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
