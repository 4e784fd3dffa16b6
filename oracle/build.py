"""Build the oracle's shared library (plain C, gcc, OpenMP).

TEST INFRASTRUCTURE: the library is only loaded by the test suite, the smoke
check and the bench's CPU-baseline leg.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = [os.path.join(HERE, "ttt_oracle.c")]
DEPS = SRC + [os.path.join(HERE, "ttt_oracle_impl.h")]
LIB = os.path.join(HERE, "libttt_oracle.so")

# IEEE arithmetic only: no fast-math, no FMA contraction, so results do not
# depend on the compiler's choice of instructions.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
          "-fno-fast-math", "-Wall", "-Wno-unknown-pragmas"]


def build(force: bool = False) -> str:
    stale = (not os.path.exists(LIB)) or any(
        os.path.getmtime(p) > os.path.getmtime(LIB) for p in DEPS)
    if force or stale:
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", *CFLAGS, "-o", tmp, *SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
