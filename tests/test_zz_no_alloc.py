"""bsa_select_static: the index search for callers that cannot allocate.

Serving engines and plugin hosts that plan every byte of device memory before
they start, and hot loops that cannot pay cudaMalloc's implicit device-wide
synchronisation, cannot hand bsa_select a workspace.  bsa_select_static keeps
its centroid scratch in a fixed 16 MiB array inside libbsa instead.  These
tests call it through the C ABI twice in a row, on two different problems,
and check each result against bsa_select run with a caller-provided
workspace: index lists and counts must be identical, scores within the
parity tolerance.  A plan whose centroids do not fit the array must be
refused before anything is launched.

The file is named so that pytest collects it last; it builds its own inputs,
so it passes alone in a fresh process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_permute_b200 as bsa
import synthetic

pytestmark = pytest.mark.gpu


def _static_fn():
    fn = bsa.load().bsa_select_static
    P, I = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [P, P, P, I, P, I, P, P, P, P]
    fn.restype = I
    return fn


def _call_static(plan, qb, kb, mode, params, kmax):
    i = plan.info
    idx = torch.full((i.batch, i.heads, i.nb, kmax), -7, dtype=torch.int32, device=plan.device)
    cnt = torch.full((i.batch, i.heads, i.nb), -7, dtype=torch.int32, device=plan.device)
    sc = torch.full((i.batch, i.heads, i.nb, i.nb), float("nan"), dtype=torch.float32,
                    device=plan.device)
    st = _static_fn()(plan._h, bsa._ptr(qb), bsa._ptr(kb), mode, bsa._params(params, i.heads),
                      kmax, bsa._ptr(idx), bsa._ptr(cnt), bsa._ptr(sc), bsa._stream(plan.device))
    assert st == 0, bsa.load().bsa_last_error_string().decode()
    return idx, cnt, sc


def _problem(w, dev):
    q, k, _ = synthetic.make_qkv(w)
    plan = bsa.plan_for(w, dev)
    qb, kb = plan.permute(q.to(dev)), plan.permute(k.to(dev))
    return plan, qb, kb


def test_static_select_matches_workspace_select_twice_in_a_row():
    dev = torch.device("cuda", 0)
    problems = [
        synthetic.workload("wan13"),
        synthetic.Workload("ragged_text_topp", 1, 6, 12, 20, 1, 8, 16, 3, 128, "bf16", 1,
                           [0.9] * 3, n_text=130),
    ]
    for w in problems:
        plan, qb, kb = _problem(w, dev)
        kmax = plan.kmax_for(w.mode, w.params)
        got_idx, got_cnt, got_sc = _call_static(plan, qb, kb, w.mode, w.params, kmax)
        ref_idx, ref_cnt, ref_sc = plan.select(qb, kb, w.mode, w.params, kmax=kmax, scores=True)
        torch.cuda.synchronize()
        assert torch.equal(got_cnt, ref_cnt), w.name
        c = ref_cnt.cpu().numpy()
        gi, ri = got_idx.cpu().numpy(), ref_idx.cpu().numpy()
        for b, h, i in np.ndindex(*c.shape):
            assert np.array_equal(gi[b, h, i, :c[b, h, i]], ri[b, h, i, :c[b, h, i]]), (w.name, b, h, i)
        np.testing.assert_allclose(got_sc.cpu().numpy(), ref_sc.cpu().numpy(), rtol=2e-5, atol=1e-7)


def test_static_select_refuses_plans_beyond_its_array():
    dev = torch.device("cuda", 0)
    # 2 * 1 * 64 heads * 1176 blocks * 128 * 4 bytes = 77 MB > 16 MiB; the call
    # must refuse on the plan's sizes alone, so small dummy buffers suffice
    plan = bsa.Plan(1, 84, 30, 52, 4, 4, 8, 64, 128, 0, torch.bfloat16, dev)
    dummy = torch.zeros(64, dtype=torch.int32, device=dev)
    kmax = plan.kmax_for(0, 0.1)
    st = _static_fn()(plan._h, bsa._ptr(dummy), bsa._ptr(dummy), 0, bsa._params(0.1, 64), kmax,
                      bsa._ptr(dummy), bsa._ptr(dummy), None, bsa._stream(dev))
    assert st == 2
    assert "16 MiB" in bsa.load().bsa_last_error_string().decode()
    torch.cuda.synchronize()
    assert bool(torch.all(dummy == 0))     # nothing was launched
