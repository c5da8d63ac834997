"""Build step of the CPU oracle (test infrastructure): compiles
``prox_oracle.c`` into ``libprox_oracle.so`` next to it with gcc.

Flags: ``-ffp-contract=off -fno-fast-math`` keep every fp32/fp64 operation a
single IEEE-rounded operation, as the oracle's quantiser requires; OpenMP
spreads independent tokens over threads."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "prox_oracle.c")
LIB = os.path.join(HERE, "libprox_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
           "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
