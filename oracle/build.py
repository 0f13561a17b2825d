"""Build the CPU oracle (plain C, gcc) into oracle/libhc_oracle.so.

Test infrastructure: the oracle is built so the tests and the benchmark's CPU
baseline can load it; the product library never links it.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "hc_oracle.c")
LIB = os.path.join(HERE, "libhc_oracle.so")

# -ffp-contract=off: no multiply-add is fused unless the source calls fmaf.
# -fno-fast-math keeps IEEE semantics; -O2 is safe under both.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
          "-fno-fast-math", "-Wall", "-Wextra"]


def needs_build() -> bool:
    return (not os.path.exists(LIB)) or os.path.getmtime(LIB) < os.path.getmtime(SRC)


def build(force: bool = False) -> str:
    if force or needs_build():
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", *CFLAGS, SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
