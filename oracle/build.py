"""Compile the C oracle into ``oracle/liboracle_if4.so`` (test infrastructure).

Flags keep the arithmetic exactly as written: binary32/binary64 IEEE with
round-to-nearest-even, no contraction into FMA, no fast-math, no
flush-to-zero.  OpenMP parallelises over rows only.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "if4_oracle.c")
LIB = os.path.join(HERE, "liboracle_if4.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
          "-fno-fast-math", "-fno-finite-math-only", "-frounding-math",
          "-fopenmp"]


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    cmd = ["gcc", *CFLAGS, "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
