"""Host test of the integer division the attention kernel's copy-issuing
thread uses for block coordinates (FastDiv in csrc/common.cuh): compiled with
g++ from the same header and compared with the plain quotient."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "block_sparse_attention_permute_b200", "csrc")


def _cuda_include():
    for cand in ("/usr/local/cuda/include", os.path.join(os.environ.get("CUDA_HOME", ""), "include")):
        if os.path.exists(os.path.join(cand, "cuda_runtime.h")):
            return cand
    return None


@pytest.mark.skipif(shutil.which("g++") is None or _cuda_include() is None,
                    reason="needs g++ and the CUDA headers")
def test_fastdiv_matches_integer_division(tmp_path):
    exe = tmp_path / "fastdiv_check"
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-I", _cuda_include(), "-I", CSRC,
                           os.path.join(ROOT, "tests", "c", "fastdiv_check.cpp"), "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "0 wrong" in out.stdout
