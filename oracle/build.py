"""Compile the CPU oracle (wq_oracle.c) into oracle/liboracle.so.

Test infrastructure only: the product library never loads this file.
Strict IEEE binary64 arithmetic: no fast-math, no floating-point
contraction (so no fused multiply-add changes a rounding).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "wq_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = [
        "gcc", "-std=c11", "-O2", "-fopenmp", "-fno-fast-math", "-ffp-contract=off",
        "-fPIC", "-shared", "-Wall", "-Wextra", "-o", LIB, SRC, "-lm",
    ]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
