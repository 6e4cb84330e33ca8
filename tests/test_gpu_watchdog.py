"""Failure detection of the tensor-core attention kernel: bounded in-kernel waits.

Every mbarrier wait of attn_tc_kernel gives up after the plan's wait limit
(bsa_plan_set_watchdog).  These tests make one wait run out the allowed way,
without faulting or hanging the GPU: the plan's test hook makes CTA 0 skip one
K/V copy, so the full-barrier of that ring slot is a flag nothing ever sets.
The MMA issuer's wait then runs out after a short limit; the CTA aborts, waits
for the copies and MMAs it did issue, frees its TMEM and returns, and the
status word reads BSA_ERR_TIMEOUT.  The launch itself completes (the CUDA
context stays usable), every other CTA's rows are unaffected, and the next
call on the same plan, hook off, matches the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_permute_b200 as bsa
import oracle as orc
import synthetic
from parity import check_output, custom_workload, geometry, to_np

pytestmark = pytest.mark.gpu

# about 1 ms at the B200's clocks: far above any wait of these small launches
SHORT_LIMIT = 2_000_000
CASES = {
    "hy_ragged_text": custom_workload("hy_ragged_text", 1, 6, 12, 20, 1, 8, 16, 3, 128, 130,
                                      "bf16", 0, 0.3),
    "d64_text": custom_workload("d64_text", 1, 5, 12, 20, 1, 8, 16, 3, 64, 200, "bf16", 0, 0.35),
}


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bsa.load()
    return torch.device("cuda", 0)


def _oracle_out(w, q, k, v, idx, cnt):
    g = geometry(w)
    return orc.attention(g, to_np(q), to_np(k), to_np(v), idx.cpu().numpy(), cnt.cpu().numpy())


def _timeout_rows_ok(bad, good, max_rows):
    """Rows of `bad` that differ from `good` are all zero, and at most max_rows."""
    b = bad.float().reshape(-1, bad.shape[-1])
    g = good.float().reshape(-1, good.shape[-1])
    diff = (b != g).any(-1)
    assert torch.all(b[diff] == 0), "a timed-out row holds non-zero values"
    assert int(diff.sum()) <= max_rows, int(diff.sum())
    return int(diff.sum())


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("withhold", [1, 3])
def test_forward_wait_runs_out_then_recovers(name, withhold, dev):
    w = CASES[name]
    q, k, v = synthetic.make_qkv(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    plan = bsa.plan_for(w, dev)
    assert plan.info.attn_path == 1
    good, idx, cnt = plan.forward(qd, kd, vd, w.mode, w.params, return_lists=True)
    plan.check_status()

    plan.set_watchdog(SHORT_LIMIT, withhold_copy=withhold)
    bad = plan.forward(qd, kd, vd, w.mode, w.params)
    torch.cuda.synchronize()            # the launch completed: no CUDA error
    with pytest.raises(bsa.BsaError) as e:
        plan.check_status()
    assert e.value.status == 4          # BSA_ERR_TIMEOUT
    plan.check_status()                 # the status word was cleared
    # CTA 0 owns two query tiles: only their token rows (per head) may differ
    n = _timeout_rows_ok(bad, good, 2 * 128)
    assert n > 0

    # hook off, default limit: the same plan computes the right answer again
    plan.set_watchdog(0, 0)
    again, idx2, cnt2 = plan.forward(qd, kd, vd, w.mode, w.params, return_lists=True)
    plan.check_status()
    assert torch.equal(again, good)
    check_output(to_np(again), _oracle_out(w, q, k, v, idx2, cnt2), w.dtype, name)


def test_blocked_attention_wait_runs_out(dev):
    w = CASES["hy_ragged_text"]
    q, k, v = synthetic.make_qkv(w)
    plan = bsa.plan_for(w, dev)
    qb, kb, vb, qc, kc = plan.permute_qkv(q.to(dev), k.to(dev), v.to(dev))
    idx, cnt = plan.select_centroids(qc, kc, w.mode, w.params)
    good = plan.attention(qb, kb, vb, idx, cnt)
    plan.check_status()
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    plan.set_watchdog(SHORT_LIMIT, withhold_copy=2)
    bad = plan.attention(qb, kb, vb, idx, cnt, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 4      # recorded in the caller's word
    plan.check_status()                 # ... not in the plan's
    _timeout_rows_ok(bad, good, 2 * 128)
    plan.set_watchdog(0, 0)
    assert torch.equal(plan.attention(qb, kb, vb, idx, cnt), good)
    plan.check_status()


def test_short_limit_alone_changes_nothing(dev):
    """A tight bound with no copy withheld: no wait runs out, results are
    bit-identical to the default bound's."""
    w = CASES["hy_ragged_text"]
    q, k, v = synthetic.make_qkv(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    plan = bsa.plan_for(w, dev)
    ref = plan.forward(qd, kd, vd, w.mode, w.params)
    plan.check_status()
    plan.set_watchdog(SHORT_LIMIT, 0)
    for _ in range(3):
        out = plan.forward(qd, kd, vd, w.mode, w.params)
        plan.check_status()
        assert torch.equal(out, ref)
    plan.set_watchdog(0, 0)


def test_watchdog_rejects_negative_values(dev):
    w = CASES["hy_ragged_text"]
    plan = bsa.plan_for(w, dev)
    with pytest.raises(bsa.BsaError) as e:
        plan.set_watchdog(-1, 0)
    assert e.value.status == 1
    with pytest.raises(bsa.BsaError) as e:
        plan.set_watchdog(0, -2)
    assert e.value.status == 1
