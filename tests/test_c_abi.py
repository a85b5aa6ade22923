"""The C ABI from a plain C program (tests/c_abi/abi_demo.c): the header
compiles as C11 and the program links against the library (CPU); on a GPU
the program runs the entry points on raw device pointers and checks closed
forms (GPU)."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def build_demo(tmp_path):
    from dit_token_b200 import build
    lib = build.build()
    exe = str(tmp_path / "abi_demo")
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-O1",
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           os.path.join(ROOT, "tests", "c_abi", "abi_demo.c"), "-o", exe,
           "-L", os.path.dirname(lib), "-ldit_token", "-Wl,-rpath," + os.path.dirname(lib),
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-Wl,-rpath," + os.path.join(CUDA, "lib64")]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_header_and_program_build(tmp_path):
    assert os.path.exists(build_demo(tmp_path))


@pytest.mark.gpu
def test_program_runs_on_the_gpu(tmp_path):
    r = subprocess.run([build_demo(tmp_path)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "abi_demo: ok" in r.stdout
