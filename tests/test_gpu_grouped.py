"""GPU parity of head grouping with per-head blocking schemes (SPADE §3.3 (2),
§3.2 Selected Blocking Scheme): bsa_forward_grouped through the C ABI.

Each (b, h) is served by the plan the head map names.  Its lists must equal
the oracle's for that plan's geometry, its output the oracle's attention over
those lists, and — since a tile's arithmetic does not depend on which tiles
share its launch — its output rows must be bit-identical to the single-plan
forward of that plan.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_permute_b200 as bsa
import oracle as orc
import synthetic
from parity import check_lists, check_output, sample_rows, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bsa.load()
    return torch.device("cuda", 0)


# name: (B, T, H, W, Hd, D, n_text, shapes, head_plan [B*Hd], mode, param)
CASES = {
    "three_schemes_text": (1, 6, 12, 20, 3, 128, 130, [(1, 8, 16), (2, 4, 16), (4, 4, 8)],
                           [2, 0, 1], 0, 0.3),
    "batch2_mixed_d64": (2, 8, 8, 16, 2, 64, 0, [(1, 8, 16), (4, 4, 8)], [1, 0, 0, 1], 0, 0.25),
    "topp_one_group_empty": (1, 8, 8, 16, 3, 128, 0, [(2, 4, 16), (4, 4, 8), (8, 2, 8)],
                             [0, 0, 2], 1, 0.9),
}


def _geom(B, T, H, W, Hd, D, n_text, shape):
    return orc.Geometry(B, T, H, W, shape[0], shape[1], shape[2], Hd, D, n_text)


@pytest.mark.parametrize("union", [None, dict(window=(1, 0), sink_tokens=20, intra_mode=0,
                                              intra_params=0.2)])
@pytest.mark.parametrize("name", list(CASES))
def test_forward_grouped(name, union, dev):
    B, T, H, W, Hd, D, n_text, shapes, head_plan, mode, param = CASES[name]
    q, k, v = synthetic.make_custom(B, T, H, W, Hd, D, n_text, "bf16")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    plans = [bsa.Plan(B, T, H, W, a, b, c, Hd, D, n_text, torch.bfloat16, dev) for a, b, c in shapes]
    params = [param] * Hd
    u = bsa.mask_union(Hd, **union) if union else None
    out, lists = bsa.forward_grouped(plans, head_plan, qd, kd, vd, mode, params, u)
    plans[0].check_status()
    qn, kn, vn = to_np(q), to_np(k), to_np(v)
    hp = np.array(head_plan).reshape(B, Hd)
    for c, plan in enumerate(plans):
        sel = [(b, h) for b in range(B) for h in range(Hd) if hp[b, h] == c]
        if not sel:
            continue
        g = _geom(B, T, H, W, Hd, D, n_text, shapes[c])
        # single-plan forward of plan c: the grouped rows of its heads are identical
        if u is None:
            ref_out, ridx, rcnt = plan.forward(qd, kd, vd, mode, params, return_lists=True)
        else:
            ref_out, ridx, rcnt = plan.forward_union(qd, kd, vd, mode, params, u)
        torch.cuda.synchronize()
        idx, cnt = lists[c]
        for b, h in sel:
            assert torch.equal(out[b, :, h], ref_out[b, :, h]), (name, c, b, h)
            assert torch.equal(cnt[b, h], rcnt[b, h])
        if u is None:
            p = orc.scores(g, orc.centroids(g, qn), orc.centroids(g, kn))
            o_idx, o_cnt, tie = orc.select(g, p, mode, params)
            mask = np.zeros((B, Hd, g.nb), dtype=bool)
            for b, h in sel:
                mask[b, h] = True
            gi, gc = idx.cpu().numpy().copy(), cnt.cpu().numpy().copy()
            # compare the selected heads only: copy the oracle's rows elsewhere
            gi_full = np.where(mask[..., None], gi[..., :o_idx.shape[-1]], o_idx)
            gc_full = np.where(mask, gc, o_cnt)
            check_lists(g, torch.from_numpy(gi_full), torch.from_numpy(gc_full), o_idx, o_cnt, tie,
                        p, mode, params)
        ref = orc.attention(g, qn, kn, vn, idx.cpu().numpy(), cnt.cpu().numpy())
        for b, h in sel:
            check_output(to_np(out[b:b + 1, :, h:h + 1]), ref[b:b + 1, :, h:h + 1], "bf16",
                         f"{name} plan {c} head {h}")


def test_grouped_rejects_bad_calls(dev):
    B, T, H, W, Hd, D = 1, 8, 8, 16, 2, 128
    q, k, v = (torch.zeros((B, T * H * W, Hd, D), dtype=torch.bfloat16, device=dev) for _ in range(3))
    pa = bsa.Plan(B, T, H, W, 1, 8, 16, Hd, D, 0, torch.bfloat16, dev)
    pb = bsa.Plan(B, T, H, W, 4, 4, 8, Hd, D, 0, torch.bfloat16, dev)
    with pytest.raises(bsa.BsaError):          # plan index out of range
        bsa.forward_grouped([pa, pb], [0, 2], q, k, v, 0, [0.5] * Hd)
    simt = bsa.Plan(B, T, H, W, 2, 4, 4, Hd, D, 0, torch.bfloat16, dev)   # 32-token blocks
    with pytest.raises(bsa.BsaError) as e:
        bsa.forward_grouped([pa, simt], [0, 1], q, k, v, 0, [0.5] * Hd)
    assert e.value.status == 2
    other = bsa.Plan(B, T, H, W + 16, 1, 8, 16, Hd, D, 0, torch.bfloat16, dev)
    with pytest.raises(bsa.BsaError):          # a different problem
        bsa.forward_grouped([pa, other], [0, 1], q, k, v, 0, [0.5] * Hd)
    with pytest.raises(bsa.BsaError):          # list width below the bound
        bsa.forward_grouped([pa, pb], [0, 1], q, k, v, 0, [0.5] * Hd, kmax=[1, 1])


def test_full_hunyuan_scheme_adaptive(dev):
    """Scheme choice by aggregation score, then the grouped forward, on the
    full Hunyuan workload: every head's rows equal its plan's single-plan
    forward; sampled rows of two heads against the oracle."""
    w = synthetic.workload("hunyuan")
    q, k, v = synthetic.make_qkv(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    shapes = [(1, 8, 16), (4, 4, 8), (16, 1, 8)]
    plans = [bsa.Plan(w.B, w.T, w.H, w.W, a, b, c, w.Hd, w.D, w.n_text, torch.bfloat16, dev)
             for a, b, c in shapes]
    _, _, choice = bsa.aggregation_scores(plans, qd)
    head_plan = choice.cpu().flatten().tolist()
    out, lists = bsa.forward_grouped(plans, head_plan, qd, kd, vd, w.mode, w.params)
    plans[0].check_status()
    used = sorted(set(head_plan))
    assert len(used) >= 2, head_plan
    qn, kn, vn = to_np(q), to_np(k), to_np(v)
    for c in used:
        ref_out = plans[c].forward(qd, kd, vd, w.mode, w.params)
        torch.cuda.synchronize()
        heads = [h for h in range(w.Hd) if head_plan[h] == c]
        for h in heads:
            assert torch.equal(out[0, :, h], ref_out[0, :, h]), (c, h)
        g = _geom(w.B, w.T, w.H, w.W, w.Hd, w.D, w.n_text, shapes[c])
        h = heads[0]
        idx, cnt = lists[c]
        rows = sample_rows(g, seed=11 + c)
        gq = orc.Geometry(w.B, w.T, w.H, w.W, *shapes[c], 1, w.D, w.n_text)
        ref = orc.attention(gq, qn[:, :, h:h + 1], kn[:, :, h:h + 1], vn[:, :, h:h + 1],
                            idx[:, h:h + 1].cpu().numpy(), cnt[:, h:h + 1].cpu().numpy(), rows=rows)
        got = out[:, torch.from_numpy(rows).to(dev), h:h + 1]
        check_output(to_np(got), ref, "bf16", f"hunyuan plan {c} head {h}")
    print(f"scheme choice {head_plan}")
