"""The C ABI from a plain C program (tests/c/forward_example.c): it compiles and links
against include/moe.h and libmoe.so here; on a GPU it runs the layer through
moe_forward and moe_forward_host and checks both agree and that bad arguments are
reported."""
import os
import shutil
import subprocess

import pytest

from sparse_mixture_experts_09_b200 import build_lib

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _build(tmp_path):
    cc = shutil.which("cc") or shutil.which("gcc")
    if cc is None:
        pytest.skip("no C compiler")
    lib = build_lib.build()
    exe = str(tmp_path / "forward_example")
    cmd = [cc, "-O2", "-std=c11", os.path.join(HERE, "c", "forward_example.c"),
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", lib,
           "-Wl,-rpath," + os.path.dirname(lib), "-Wl,-rpath," + os.path.join(CUDA, "lib64"),
           "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True)
    return exe


def test_c_example_compiles_and_links(tmp_path):
    assert os.path.exists(_build(tmp_path))


@pytest.mark.gpu
def test_c_example_runs(tmp_path):
    exe = _build(tmp_path)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok:")
