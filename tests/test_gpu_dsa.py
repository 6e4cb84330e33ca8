"""GPU parity of the box estimators (SPADE §3.1 DSA-SPADE and DSA2-SPADE):
bsa_box_summaries, bsa_select_box and bsa_forward_estimator through the C
ABI against the fp64 oracle on the same seeded inputs.

Box summaries are max / min of exactly widened inputs: bit-exact.  Scores
are compared with the forward error bound of the fp32 estimate; lists bit
for bit (tie rows: a valid selection); outputs against the oracle's
attention over the GPU's own lists.
"""
import zlib

import numpy as np
import pytest
import torch

import block_sparse_attention_permute_b200 as bsa
import oracle as orc
import synthetic
from parity import (bound_ties, check_lists, check_output, check_union_lists, custom_workload,
                    geometry, sample_rows, to_np, union_extras)

pytestmark = pytest.mark.gpu

EST = {"dsa": 1, "dsa2": 2}

SMALL = {
    "hy_ragged_text": custom_workload("hy_ragged_text", 1, 6, 12, 20, 1, 8, 16, 3, 128, 130,
                                      "bf16", 0, 0.3),
    "wan_d64_b2": custom_workload("wan_d64_b2", 2, 9, 10, 20, 4, 4, 8, 2, 64, 0, "bf16", 0, 0.25),
    "wan_topp": custom_workload("wan_topp", 1, 9, 10, 20, 4, 4, 8, 3, 128, 0, "bf16", 1, 0.9),
    "simt_bf16_bs32": custom_workload("simt_bf16_bs32", 1, 5, 9, 12, 2, 4, 4, 2, 128, 40, "bf16",
                                      0, 0.3),
    "f32_bs128": custom_workload("f32_bs128", 1, 6, 12, 20, 1, 8, 16, 2, 64, 0, "f32", 0, 0.3),
}


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bsa.load()
    return torch.device("cuda", 0)


def _score_tol(g, qbox, kbox, variant, p):
    """Bound on |p_gpu - p_ref|: the fp32 estimate is a 2D-term sum of products
    of exact summaries (DSA: plus the rounded centre), so
    |d est| <= (2D + 3) u sum_d |term_d|, and the scale adds 2u|s|, so |d s| <=
    (2D + 5) u sum_d |term_d| / sqrt(D); the
    softmax moves p_ij by at most p_ij (|d s_ij| + max_j |d s_ij|) to first order."""
    u = 2.0 ** -24
    qM, qm, kM, km = qbox[..., 0], qbox[..., 1], kbox[..., 0], kbox[..., 1]
    if variant == 1:
        c = (qM + qm) / 2
        terms = np.maximum(np.abs(c)[:, :, :, None, :] * np.abs(kM)[:, :, None, :, :],
                           np.abs(c)[:, :, :, None, :] * np.abs(km)[:, :, None, :, :])
    else:
        a = np.maximum(np.abs(qM), np.abs(qm))[:, :, :, None, :]
        b = np.maximum(np.abs(kM), np.abs(km))[:, :, None, :, :]
        terms = a * b
    ds = (2 * g.D + 5) * u * terms.sum(-1) / np.sqrt(g.D)
    return p * (ds + ds.max(-1, keepdims=True)) * 1.01 + 1e-12


@pytest.mark.parametrize("name", list(SMALL))
def test_box_summaries_bit_exact(name, dev):
    w = SMALL[name]
    g = geometry(w)
    q, k, _ = synthetic.make_qkv(w)
    plan = bsa.plan_for(w, dev)
    qb, kb = plan.box_summaries(q.to(dev), k.to(dev))
    torch.cuda.synchronize()
    assert np.array_equal(qb.cpu().numpy().astype(np.float64), orc.box_summaries(g, to_np(q)))
    assert np.array_equal(kb.cpu().numpy().astype(np.float64), orc.box_summaries(g, to_np(k)))


@pytest.mark.parametrize("est", list(EST))
@pytest.mark.parametrize("name", list(SMALL))
def test_select_box_lists_and_scores(name, est, dev):
    w = SMALL[name]
    g = geometry(w)
    q, k, _ = synthetic.make_qkv(w)
    plan = bsa.plan_for(w, dev)
    qb, kb = plan.box_summaries(q.to(dev), k.to(dev))
    idx, cnt, sc = plan.select_box(EST[est], qb, kb, w.mode, w.params, scores=True)
    torch.cuda.synchronize()
    oq, ok = orc.box_summaries(g, to_np(q)), orc.box_summaries(g, to_np(k))
    p = orc.scores_box(g, oq, ok, EST[est])
    o_idx, o_cnt, tie = orc.select(g, p, w.mode, w.params)
    tol = _score_tol(g, oq, ok, EST[est], p)
    tie = tie | bound_ties(g, p, tol, w.mode, w.params)
    n_tie = check_lists(g, idx, cnt, o_idx, o_cnt, tie, p, w.mode, w.params, tol=tol)
    err = np.abs(sc.cpu().numpy() - p)
    assert np.all(err <= tol), float((err / tol).max())
    print(f"{name}/{est}: ties {n_tie}, worst score err/bound {float((err / tol).max()):.2e}")


@pytest.mark.parametrize("est", list(EST))
@pytest.mark.parametrize("name", list(SMALL))
def test_forward_estimator(name, est, dev):
    w = SMALL[name]
    g = geometry(w)
    q, k, v = synthetic.make_qkv(w)
    plan = bsa.plan_for(w, dev)
    out, idx, cnt = plan.forward_estimator(q.to(dev), k.to(dev), v.to(dev), EST[est], w.mode,
                                           w.params)
    plan.check_status()
    qn, kn, vn = to_np(q), to_np(k), to_np(v)
    oq, ok = orc.box_summaries(g, qn), orc.box_summaries(g, kn)
    p = orc.scores_box(g, oq, ok, EST[est])
    o_idx, o_cnt, tie = orc.select(g, p, w.mode, w.params)
    tol = _score_tol(g, oq, ok, EST[est], p)
    tie = tie | bound_ties(g, p, tol, w.mode, w.params)
    check_lists(g, idx, cnt, o_idx, o_cnt, tie, p, w.mode, w.params, tol=tol)
    ref = orc.attention(g, qn, kn, vn, idx.cpu().numpy(), cnt.cpu().numpy())
    check_output(to_np(out), ref, w.dtype, f"{name}/{est}")
    # the whole path agrees with the oracle's own forward on the lists too
    o_ref, r_idx, r_cnt, r_tie, _ = orc.forward(g, qn, kn, vn, w.mode, w.params, estimator=EST[est])
    assert np.array_equal(r_cnt, o_cnt)


def test_forward_estimator_with_union_and_mean(dev):
    w = SMALL["hy_ragged_text"]
    g = geometry(w)
    q, k, v = synthetic.make_qkv(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    plan = bsa.plan_for(w, dev)
    u = bsa.mask_union(w.Hd, window=(1, 0), sink_tokens=20)
    out, idx, cnt = plan.forward_estimator(qd, kd, vd, 2, w.mode, w.params, u)
    plan.check_status()
    qn, kn, vn = to_np(q), to_np(k), to_np(v)
    p = orc.scores_box(g, orc.box_summaries(g, qn), orc.box_summaries(g, kn), 2)
    o_idx, o_cnt, tie = orc.select_union(g, p, w.mode, w.params, window=(1, 0), sink_tokens=20)
    extras = union_extras(g, (1, 0), 20, [[set() for _ in range(g.Hd)] for _ in range(g.B)])
    check_union_lists(g, idx, cnt, o_idx, o_cnt, tie, p, w.mode, w.params, extras)
    ref = orc.attention(g, qn, kn, vn, idx.cpu().numpy(), cnt.cpu().numpy())
    check_output(to_np(out), ref, w.dtype, "dsa2 + union")
    # MEAN through the estimator entry point is bsa_forward_union
    o1, i1, c1 = plan.forward_estimator(qd, kd, vd, 0, w.mode, w.params, u)
    o2, i2, c2 = plan.forward_union(qd, kd, vd, w.mode, w.params, u)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(c1, c2)
    with pytest.raises(bsa.BsaError):
        plan.forward_estimator(qd, kd, vd, 3, w.mode, w.params)
    with pytest.raises(bsa.BsaError):
        qb, kb = plan.box_summaries(qd, kd)
        plan.select_box(0, qb, kb, w.mode, w.params)


FULL = {"hunyuan": "dsa", "wan13": "dsa2", "wan14_topp": "dsa"}


@pytest.mark.parametrize("name", list(FULL))
def test_full_workload_forward_estimator(name, dev):
    w = synthetic.workload(name)
    g = geometry(w)
    est = EST[FULL[name]]
    q, k, v = synthetic.make_qkv(w)
    plan = bsa.plan_for(w, dev)
    out, idx, cnt = plan.forward_estimator(q.to(dev), k.to(dev), v.to(dev), est, w.mode, w.params)
    plan.check_status()
    qn, kn, vn = to_np(q), to_np(k), to_np(v)
    oq, ok = orc.box_summaries(g, qn), orc.box_summaries(g, kn)
    p = orc.scores_box(g, oq, ok, est)
    o_idx, o_cnt, tie = orc.select(g, p, w.mode, w.params)
    tol = _score_tol(g, oq, ok, est, p)
    tie = tie | bound_ties(g, p, tol, w.mode, w.params)
    n_tie = check_lists(g, idx, cnt, o_idx, o_cnt, tie, p, w.mode, w.params, tol=tol)
    rows = sample_rows(g, seed=zlib.crc32(name.encode()) % 1000)
    ref = orc.attention(g, qn, kn, vn, idx.cpu().numpy(), cnt.cpu().numpy(), rows=rows)
    got = out[:, torch.from_numpy(rows).to(dev)]
    mx, mean = check_output(to_np(got), ref, w.dtype, name)
    print(f"{name}/{FULL[name]}: ties={n_tie} mean list {float(cnt.float().mean()):.1f} "
          f"max_abs={mx:.3e}")
