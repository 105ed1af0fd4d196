"""Compile the fp64 CPU oracle (test infrastructure) into oracle/libkla_oracle.so.

Only the tests, the package smoke check and the benchmark's CPU-baseline leg load
the result; the CUDA library never links or calls it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "kla_oracle.c")
LIB = os.path.join(HERE, "libkla_oracle.so")


def build(force: bool = False) -> str:
    """Build the oracle shared library if it is missing or older than its source."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    # -ffp-contract=off: plain multiply-then-add, no fused rounding, so results do not
    # depend on the host compiler's contraction choices.
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
