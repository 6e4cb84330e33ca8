"""bsa_forward_timed: per-phase device times of one forward call (events at
the phase boundaries inside the library).  The output must equal a plain
bsa_forward bit for bit, the phases must be positive where they run and add
up to the total, and a NULL timings pointer is refused before any launch."""
import ctypes

import pytest
import torch

import block_sparse_attention_permute_b200 as bsa
import synthetic
from parity import custom_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bsa.load()
    return torch.device("cuda", 0)


CASES = {
    "hy_ragged_text": custom_workload("hy_ragged_text", 1, 6, 12, 20, 1, 8, 16, 3, 128, 130,
                                      "bf16", 0, 0.3),
    "tiny": synthetic.workload("tiny"),
}


@pytest.mark.parametrize("name", list(CASES))
def test_forward_timed_matches_forward(name, dev):
    w = CASES[name]
    q, k, v = synthetic.make_qkv(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    plan = bsa.plan_for(w, dev)
    ref = plan.forward(qd, kd, vd, w.mode, w.params)
    out, tm = plan.forward_timed(qd, kd, vd, w.mode, w.params)
    plan.check_status()
    assert torch.equal(out, ref)
    parts = ["summaries_ms", "select_ms", "pairing_ms", "attention_ms", "unpermute_ms"]
    assert all(tm[p] >= 0.0 for p in parts)
    assert tm["summaries_ms"] > 0 and tm["select_ms"] > 0 and tm["attention_ms"] > 0
    if plan.info.attn_path == 1:
        assert tm["pairing_ms"] > 0 and tm["unpermute_ms"] == 0.0
    else:
        assert tm["pairing_ms"] == 0.0 and tm["unpermute_ms"] > 0
    total = sum(tm[p] for p in parts)
    assert abs(total - tm["total_ms"]) <= 1e-3 + 0.01 * tm["total_ms"], tm


def test_full_workload_phase_split(dev):
    """HunyuanVideo: the attention dominates the pattern search (summaries,
    selection, pairing) — the split SPADE Fig. 5 reports for one layer."""
    w = synthetic.workload("hunyuan")
    q, k, v = synthetic.make_qkv(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    plan = bsa.plan_for(w, dev)
    plan.forward(qd, kd, vd, w.mode, w.params)          # warm-up
    _, tm = plan.forward_timed(qd, kd, vd, w.mode, w.params)
    plan.check_status()
    search = tm["summaries_ms"] + tm["select_ms"] + tm["pairing_ms"]
    print(f"hunyuan: {tm}")
    assert tm["attention_ms"] > 10 * search


def test_forward_timed_refuses_null_timings(dev):
    w = CASES["hy_ragged_text"]
    plan = bsa.plan_for(w, dev)
    kmax = plan.kmax_for(w.mode, w.params)
    L = bsa.load()
    dummy = torch.zeros(64, dtype=torch.int32, device=dev)
    st = L.bsa_forward_timed(plan._h, bsa._ptr(dummy), bsa._ptr(dummy), bsa._ptr(dummy), w.mode,
                             bsa._params(w.params, w.Hd), kmax, bsa._ptr(dummy), None, None,
                             bsa._ptr(dummy), 0, None, bsa._stream(dev), None)
    assert st == 1
    assert "timings" in L.bsa_last_error_string().decode()
