"""Host-side tests of libbsa (no GPU needed): the C ABI loads, exports every
function include/bsa.h declares, and rejects bad arguments before touching a
device.  The Python binding fails loudly when the library is missing."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_permute_b200 as bsa
from block_sparse_attention_permute_b200 import build as bsa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    bsa_build.build()
    return bsa.load()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "bsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["bsa_plan_create", "bsa_plan_destroy", "bsa_permute", "bsa_unpermute", "bsa_select",
              "bsa_attention", "bsa_forward", "bsa_last_error_string"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_library_is_sm100a_build():
    # the build targets sm_100a only
    assert "arch=compute_100a,code=sm_100a" in " ".join(bsa_build.ARCH)


def test_version(lib):
    assert lib.bsa_version() == 100


def _create(lib, *args):
    h = ctypes.c_void_p()
    st = lib.bsa_plan_create(ctypes.byref(h), *args)
    return st, lib.bsa_last_error_string().decode()


@pytest.mark.parametrize("args,needle", [
    ((1, 4, 8, 8, 2, 4, 4, 2, 96, 0, 0), "head_dim"),
    ((1, 4, 8, 8, 2, 4, 4, 0, 64, 0, 0), "heads"),
    ((0, 4, 8, 8, 2, 4, 4, 2, 64, 0, 0), "batch"),
    ((1, 4, 8, 8, 0, 4, 4, 2, 64, 0, 0), "block"),
    ((1, 4, 8, 8, 4, 8, 16, 2, 64, 0, 0), "exceeds 256"),
    ((1, 4, 8, 8, 2, 4, 4, 2, 64, -1, 0), "n_text"),
    ((1, 4, 8, 8, 2, 4, 4, 2, 64, 0, 7), "dtype"),
])
def test_plan_validation_rejects_bad_arguments(lib, args, needle):
    st, msg = _create(lib, *args)
    assert st == 1 and needle in msg


def test_plan_block_count_limit(lib):
    # the selection kernel holds 8 score rows of nb floats per CTA (8 query
    # rows per CTA once 16 no longer fit twice on an SM) beside 8 query
    # summaries and two 256 x 12-float key chunks: up to 6368 blocks at
    # head_dim 128 in 227 KB; beyond that the plan is refused before any
    # device work
    st, msg = _create(lib, 1, 1, 1, 6369, 1, 1, 1, 1, 128, 0, 1)
    assert st == 2 and "selection kernel" in msg
    # at the limit validation passes; without a GPU the device query then fails
    h = ctypes.c_void_p()
    st = lib.bsa_plan_create(ctypes.byref(h), 1, 1, 1, 6368, 1, 1, 1, 1, 128, 0, 1)
    assert st in (0, 3), lib.bsa_last_error_string().decode()
    if st == 0:
        lib.bsa_plan_destroy(h)


def test_null_arguments_are_rejected(lib):
    assert lib.bsa_plan_create(None, 1, 4, 8, 8, 2, 4, 4, 2, 64, 0, 0) == 1
    k = ctypes.c_int()
    assert lib.bsa_kmax_for(None, 0, None, ctypes.byref(k)) == 1
    assert lib.bsa_plan_get_info(None, None) == 1
    assert lib.bsa_plan_destroy(None) == 0


def test_aggregation_scores_rejects_bad_candidate_lists(lib):
    P = ctypes.c_void_p
    lib.bsa_aggregation_scores.argtypes = [P, ctypes.c_int, P, P, P, P, P]
    lib.bsa_aggregation_scores.restype = ctypes.c_int
    plans = (P * 9)()
    outs = (P * 9)()
    assert lib.bsa_aggregation_scores(None, 1, None, outs, None, None, None) == 1
    assert lib.bsa_aggregation_scores(plans, 1, None, None, None, None, None) == 1
    for n in (0, 9, -1):
        assert lib.bsa_aggregation_scores(plans, n, None, outs, None, None, None) == 1
        assert "n_plans" in lib.bsa_last_error_string().decode()


def test_plan_create_without_device_reports_cuda_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    st, msg = _create(lib, 1, 4, 8, 8, 2, 4, 4, 2, 64, 0, 0)
    assert st == 3, msg


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(bsa, "_LIB_PATH", "/nonexistent/libbsa.so")
    monkeypatch.setattr(bsa, "_lib", None)
    with pytest.raises(bsa.BsaError, match="missing"):
        bsa.load()
    with pytest.raises(bsa.BsaError):
        bsa.Plan(1, 4, 8, 8, 2, 4, 4, 2, 64)


def test_binding_rejects_cpu_device():
    with pytest.raises(bsa.BsaError):
        bsa.Plan(1, 4, 8, 8, 2, 4, 4, 2, 64, device="cpu")
