"""The C ABI from a plain C program (examples/c_api_solve.c): the header
compiles as C99 and links against the library; on a GPU the program solves
and checks itself against the library's sequential kernel."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")
PKG = os.path.join(ROOT, "nonlinear_rnn_newton_b200")


def build(tmp_path):
    from nonlinear_rnn_newton_b200 import build as nb
    nb.build()
    exe = str(tmp_path / "c_api_solve")
    cmd = ["gcc", "-std=c99", "-Wall", "-Werror", os.path.join(ROOT, "examples", "c_api_solve.c"),
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"), "-L", PKG, "-lpararnn",
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-lm", f"-Wl,-rpath,{PKG}",
           f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_c_program_compiles_and_links(tmp_path):
    assert os.path.exists(build(tmp_path))


@pytest.mark.gpu
def test_c_program_solves(cuda, tmp_path):
    exe = build(tmp_path)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "iters" in r.stdout
