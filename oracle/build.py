"""Compile the CPU oracle (oracle.c) into oracle/liboracle.so.

Test infrastructure only: the oracle is the plain reference that the CUDA path
is compared against; building it does not make the product depend on it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Build liboracle.so if it is missing or older than its sources."""
    deps = [SRC, os.path.join(HERE, "oracle.h"), __file__]
    if not force and os.path.exists(LIB):
        if os.path.getmtime(LIB) >= max(os.path.getmtime(d) for d in deps):
            return LIB
    # -O2 without -ffast-math and without -march: IEEE fp64, no contraction
    # into FMA on x86-64, so the arithmetic is exactly what the source says.
    # a per-process temporary name: processes that build at once (several
    # ranks) never write the same file, and the rename is atomic
    tmp = f"{LIB}.{os.getpid()}.tmp"
    cmd = ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
           "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
