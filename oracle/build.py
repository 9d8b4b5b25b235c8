"""Compile the CPU oracle (plain C, OpenMP) into oracle/libcosa_oracle.so.

Test infrastructure: the oracle is built here and loaded only by tests/, the
smoke check and the benchmark's CPU-baseline leg.  IEEE fp32/fp64 semantics
are required (no fast-math, no FMA contraction), because the oracle takes the
selection decisions in fp32 exactly as written.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "cosa_oracle.c")
LIB = os.path.join(HERE, "libcosa_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-Wextra", "-o", LIB + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
