"""Compile the CPU oracle (``oracle.c``) into ``liboracle.so`` beside it.

Test infrastructure: the oracle is a checker, never part of the product path.
Flags keep every fp32 operation a single IEEE round-to-nearest-even step
(no FMA contraction, no fast-math); OpenMP parallelises over rows only.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = [
    "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fexcess-precision=standard",
    "-fopenmp", "-shared", "-fPIC", "-Wall", "-Wextra", "-Wno-unused-parameter",
]


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
