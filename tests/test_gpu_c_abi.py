"""GPU: the C ABI called from C, without Python in between.

tests/c/forward_ones.c is compiled with the system C compiler against
include/bsa.h and the in-tree libbsa.so, and run: bsa_forward on a
tensor-core plan (ragged grid, text tokens, two densities) with V = 1 must
give an output of ones (every attention row is a convex combination of value
rows), and a too-small workspace must be refused with BSA_ERR_WORKSPACE.
"""
import os
import shutil
import subprocess

import pytest

import block_sparse_attention_permute_b200 as bsa

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_forward_from_c(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    assert cc, "a C compiler is needed"
    lib = bsa.lib_path()
    assert os.path.exists(lib), "libbsa.so is not built"
    lib_dir = os.path.dirname(lib)
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    exe = tmp_path / "forward_ones"
    subprocess.check_call([cc, "-std=c99", "-O2", "-I", os.path.join(ROOT, "include"),
                           "-I", os.path.join(cuda, "include"),
                           os.path.join(ROOT, "tests", "c", "forward_ones.c"), "-o", str(exe),
                           "-L", lib_dir, "-lbsa", "-L", os.path.join(cuda, "lib64"), "-lcudart",
                           "-lm", f"-Wl,-rpath,{lib_dir}"])
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    print(run.stdout, run.stderr)
    assert run.returncode == 0, run.stdout + run.stderr
