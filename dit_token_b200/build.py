"""Build libdit_token.so (the CUDA kernels + C ABI) in-tree for sm_100a.

    python -m dit_token_b200.build [--force] [--verbose]
    python -m dit_token_b200.build --define DIT_PDL=0 --out PATH.so

nvcc compiles every csrc/*.cu for sm_100a (cross-compiles without a GPU) and
links them into one shared library with the CUDA runtime linked statically,
so loading the library needs no GPU and no libcudart on the search path.
A build with compile-time switches (``--define``, e.g. DIT_PDL=0: launches
without programmatic dependent launch) goes to its own file, never over the
in-tree library; load it by setting DIT_TOKEN_LIB to its path.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libdit_token.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
    "-cudart", "static",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))) + \
        [os.path.join(INCLUDE, "dit_token.h"), os.path.abspath(__file__)]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    return os.path.getmtime(LIB) >= max(os.path.getmtime(d) for d in _deps())


def build(force: bool = False, verbose: bool = False, out: str = None, defines=()) -> str:
    if defines and (out is None or os.path.abspath(out) == LIB):
        raise ValueError("a build with --define needs its own --out path")
    target = LIB if out is None else os.path.abspath(out)
    if target == LIB and not force and up_to_date():
        return LIB
    tmp = f"{target}.{os.getpid()}.tmp"  # per process: concurrent builds never share a file
    # Exported symbols: only the extern "C" entry points (default visibility is
    # hidden for everything else, see -fvisibility=hidden and the header).
    cmd = [NVCC, *NVCC_FLAGS, *[f"-D{d}" for d in defines], "-I", INCLUDE, "-I", CSRC, "-shared", "-o", tmp,
           *sources()]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(tmp, target)
    return target


def _arg(flag: str, argv) -> list:
    return [argv[i + 1] for i, a in enumerate(argv[:-1]) if a == flag]


if __name__ == "__main__":
    outs = _arg("--out", sys.argv)
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, out=outs[-1] if outs else None,
                defines=_arg("--define", sys.argv)))
