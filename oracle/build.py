"""Compile the CPU oracle (plain C99 + OpenMP) into ``oracle/liboracle.so``.

Test infrastructure (see ``oracle/__init__.py``). Built without fast-math and without FMA
contraction so that every f32 operation the FP8 quantizer performs is the IEEE one written.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liboracle.so")
SRC = os.path.join(HERE, "moe_oracle.c")


def build() -> str:
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c99", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(), file=sys.stderr)
