"""Compile the C oracle into oracle/libkvq_oracle.so.

TEST INFRASTRUCTURE ONLY: the oracle is built so that the test suite, the
smoke check and the benchmark's CPU-baseline leg can load it; the CUDA
library never links or loads it.
"""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kvq_oracle.c")
OUT = os.path.join(HERE, "libkvq_oracle.so")

# Strict IEEE: no contraction into FMA, no fast-math, baseline x86-64 (SSE2)
# so that binary32 arithmetic is evaluated in binary32.
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fno-unsafe-math-optimizations",
          "-fopenmp", "-shared", "-fPIC", "-Wall", "-Wextra", "-Wno-unused-parameter"]


def build(force: bool = False) -> str:
    if not force and os.path.exists(OUT) and os.path.getmtime(OUT) >= os.path.getmtime(SRC):
        return OUT
    cmd = ["gcc", *CFLAGS, "-o", OUT, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
