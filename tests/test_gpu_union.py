"""GPU parity of the mask union (SPADE §3.3: inter selection OR intra scores
broadcast over query blocks, united with local-window and attention-sink
blocks): bsa_select_union and bsa_forward_union through the C ABI against the
fp64 oracle on the same seeded inputs.

bsa_select_union gets the same fp32 intra scores on both sides, so its lists
are compared bit for bit (tie rows: a valid selection).  bsa_forward_union
computes the intra scores itself (the SICS of the K blocks, in fp32); a head
whose intra decision could flip within the SICS error bound is checked for
its window and sink blocks only and counted.  Outputs are compared with the
oracle's attention over the GPU's own lists.
"""
import zlib

import numpy as np
import pytest
import torch

import block_sparse_attention_permute_b200 as bsa
import oracle as orc
import synthetic
from parity import (check_output, check_union_lists, custom_workload, geometry, intra_near_tie,
                    sample_rows, sics_tol, to_np, union_extras)

pytestmark = pytest.mark.gpu

SMALL = {
    "hy_ragged_text": custom_workload("hy_ragged_text", 1, 6, 12, 20, 1, 8, 16, 3, 128, 130,
                                      "bf16", 0, 0.3),
    "wan_d64_b2": custom_workload("wan_d64_b2", 2, 9, 10, 20, 4, 4, 8, 2, 64, 0, "bf16", 0, 0.25),
    "wan_topp": custom_workload("wan_topp", 1, 9, 10, 20, 4, 4, 8, 3, 128, 0, "bf16", 1, 0.9),
    "simt_bf16_bs32": custom_workload("simt_bf16_bs32", 1, 5, 9, 12, 2, 4, 4, 2, 128, 40, "bf16",
                                      0, 0.3),
    "f32_bs128": custom_workload("f32_bs128", 1, 6, 12, 20, 1, 8, 16, 2, 64, 0, "f32", 0, 0.3),
}

UNIONS = {
    "window": dict(window=(1, 1)),
    "causal_window": dict(window=(2, 0)),
    "open_right": dict(window=(0, -1)),
    "sink": dict(sink_tokens=40),
    "intra_topk": dict(intra_mode=0, intra_params=0.2),
    "intra_topp": dict(intra_mode=1, intra_params=0.3),
    "all": dict(window=(1, 0), sink_tokens=17, intra_mode=0, intra_params=0.15),
}


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bsa.load()
    return torch.device("cuda", 0)


def _u(plan, kw):
    return bsa.mask_union(plan.info.heads, **kw)


def _intra_sets(g, values, mode, param_list):
    """Intra selection per (b, h) from exact values, by the rule's definition
    (used to validate tie rows only; bit-exact rows come from the oracle)."""
    out = []
    for b in range(g.B):
        row = []
        for h in range(g.Hd):
            if values is None or param_list[h] <= 0:
                row.append(set())
                continue
            v = values[b, h]
            order = sorted(range(g.nb), key=lambda j: (-v[j], j))
            if mode == 0:
                row.append(set(order[:orc.k_for_density(param_list[h], g.nb)]))
            else:
                target, c, s = param_list[h] * v.sum(), 0.0, set()
                for j in order:
                    s.add(j)
                    c += v[j]
                    if c >= target:
                        break
                row.append(s)
        out.append(row)
    return out


@pytest.mark.parametrize("uname", list(UNIONS))
@pytest.mark.parametrize("name", ["hy_ragged_text", "wan_d64_b2", "wan_topp"])
def test_select_union_with_given_intra_scores(name, uname, dev):
    w = SMALL[name]
    g = geometry(w)
    q, k, _ = synthetic.make_qkv(w)
    plan = bsa.plan_for(w, dev)
    kw = UNIONS[uname]
    qc, kc = plan.centroids(q.to(dev), k.to(dev))
    intra = None
    if "intra_params" in kw:
        rng = np.random.default_rng(zlib.crc32(f"{name}{uname}".encode()) % 10000)
        intra = (rng.random((g.B, g.Hd, g.nb)) * 100.0).astype(np.float32)
    u = _u(plan, kw)
    idx, cnt = plan.select_union(qc, kc, w.mode, w.params, u,
                                 intra_scores=None if intra is None else torch.from_numpy(intra).to(dev))
    torch.cuda.synchronize()
    p = orc.scores(g, orc.centroids(g, to_np(q)), orc.centroids(g, to_np(k)))
    ip = None if intra is None else [float(kw["intra_params"])] * g.Hd
    o_idx, o_cnt, tie = orc.select_union(g, p, w.mode, w.params, window=kw.get("window", (-1, -1)),
                                         sink_tokens=kw.get("sink_tokens", 0),
                                         intra=None if intra is None else intra.astype(np.float64),
                                         intra_mode=kw.get("intra_mode", 0), intra_params=ip)
    isets = _intra_sets(g, None if intra is None else intra.astype(np.float64),
                        kw.get("intra_mode", 0), ip or [0.0] * g.Hd)
    extras = union_extras(g, kw.get("window", (-1, -1)), kw.get("sink_tokens", 0), isets)
    n_tie = check_union_lists(g, idx, cnt, o_idx, o_cnt, tie, p, w.mode, w.params, extras)
    assert int(cnt.max()) <= plan.kmax_for_union(w.mode, w.params, u)
    print(f"{name}/{uname}: ties {n_tie}, mean list {float(cnt.float().mean()):.1f}")


@pytest.mark.parametrize("uname", ["all", "intra_topp", "window"])
@pytest.mark.parametrize("name", list(SMALL))
def test_forward_union(name, uname, dev):
    w = SMALL[name]
    g = geometry(w)
    q, k, v = synthetic.make_qkv(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    plan = bsa.plan_for(w, dev)
    kw = UNIONS[uname]
    u = _u(plan, kw)
    out, idx, cnt = plan.forward_union(qd, kd, vd, w.mode, w.params, u)
    plan.check_status()
    qn, kn, vn = to_np(q), to_np(k), to_np(v)
    p = orc.scores(g, orc.centroids(g, qn), orc.centroids(g, kn))
    intra, ip, loose = None, None, set()
    if "intra_params" in kw:
        intra = orc.sics(g, kn)
        ip = [float(kw["intra_params"])] * g.Hd
        tol = sics_tol(g, intra)
        for b in range(g.B):
            for h in range(g.Hd):
                if intra_near_tie(intra[b, h], tol[b, h], kw["intra_mode"], ip[h]):
                    loose.add((b, h))
    o_idx, o_cnt, tie = orc.select_union(g, p, w.mode, w.params, window=kw.get("window", (-1, -1)),
                                         sink_tokens=kw.get("sink_tokens", 0), intra=intra,
                                         intra_mode=kw.get("intra_mode", 0), intra_params=ip)
    isets = _intra_sets(g, intra, kw.get("intra_mode", 0), ip or [0.0] * g.Hd)
    extras = union_extras(g, kw.get("window", (-1, -1)), kw.get("sink_tokens", 0), isets)
    n_tie = check_union_lists(g, idx, cnt, o_idx, o_cnt, tie, p, w.mode, w.params, extras, loose)
    # window and sink blocks are in every list, near-tie heads included
    base = union_extras(g, kw.get("window", (-1, -1)), kw.get("sink_tokens", 0),
                        [[set() for _ in range(g.Hd)] for _ in range(g.B)])
    gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
    for key, e in base.items():
        assert e <= set(gi[key][:gc[key]].tolist())
    ref = orc.attention(g, qn, kn, vn, gi, gc)
    mx, mean = check_output(to_np(out), ref, w.dtype, f"{name}/{uname}")
    print(f"{name}/{uname}: ties {n_tie}, loose heads {len(loose)}, max_abs {mx:.2e}")


def test_union_none_is_plain_forward(dev):
    w = SMALL["hy_ragged_text"]
    q, k, v = synthetic.make_qkv(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    plan = bsa.plan_for(w, dev)
    out, idx, cnt = plan.forward(qd, kd, vd, w.mode, w.params, return_lists=True)
    out2, idx2, cnt2 = plan.forward_union(qd, kd, vd, w.mode, w.params, bsa.mask_union(w.Hd))
    torch.cuda.synchronize()
    assert torch.equal(out, out2) and torch.equal(cnt, cnt2)


def test_union_rejects_bad_options(dev):
    w = SMALL["hy_ragged_text"]
    plan = bsa.plan_for(w, dev)
    with pytest.raises(bsa.BsaError):
        plan.kmax_for_union(w.mode, w.params, bsa.mask_union(w.Hd, sink_tokens=-1))
    with pytest.raises(bsa.BsaError):
        plan.kmax_for_union(w.mode, w.params, bsa.mask_union(w.Hd, intra_params=1.5))
    qc = torch.zeros(plan.cent_shape, dtype=torch.float32, device=dev)
    with pytest.raises(bsa.BsaError):       # intra requested without scores
        plan.select_union(qc, qc, w.mode, w.params, bsa.mask_union(w.Hd, intra_params=0.2))
    # kmax below the union's bound is refused
    u = bsa.mask_union(w.Hd, window=(2, 2))
    need = plan.kmax_for_union(w.mode, w.params, u)
    assert need > plan.kmax_for(w.mode, w.params)
    with pytest.raises(bsa.BsaError):
        plan.select_union(qc, qc, w.mode, w.params, u, kmax=need - 1)


FULL = {
    "hunyuan": dict(window=(1, 1), sink_tokens=3600, intra_mode=0, intra_params=0.02),
    "wan14_topp": dict(window=(2, 2), sink_tokens=1560, intra_mode=1, intra_params=0.05),
}


@pytest.mark.parametrize("name", list(FULL))
def test_full_workload_forward_union(name, dev):
    w = synthetic.workload(name)
    g = geometry(w)
    q, k, v = synthetic.make_qkv(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    plan = bsa.plan_for(w, dev)
    kw = FULL[name]
    u = _u(plan, kw)
    out, idx, cnt = plan.forward_union(qd, kd, vd, w.mode, w.params, u)
    plan.check_status()
    qn, kn, vn = to_np(q), to_np(k), to_np(v)
    p = orc.scores(g, orc.centroids(g, qn), orc.centroids(g, kn))
    intra = orc.sics(g, kn)
    ip = [float(kw["intra_params"])] * g.Hd
    tol = sics_tol(g, intra)
    loose = {(b, h) for b in range(g.B) for h in range(g.Hd)
             if intra_near_tie(intra[b, h], tol[b, h], kw["intra_mode"], ip[h])}
    o_idx, o_cnt, tie = orc.select_union(g, p, w.mode, w.params, window=kw["window"],
                                         sink_tokens=kw["sink_tokens"], intra=intra,
                                         intra_mode=kw["intra_mode"], intra_params=ip)
    isets = _intra_sets(g, intra, kw["intra_mode"], ip)
    extras = union_extras(g, kw["window"], kw["sink_tokens"], isets)
    n_tie = check_union_lists(g, idx, cnt, o_idx, o_cnt, tie, p, w.mode, w.params, extras, loose)
    rows = sample_rows(g, seed=zlib.crc32(name.encode()) % 1000)
    ref = orc.attention(g, qn, kn, vn, idx.cpu().numpy(), cnt.cpu().numpy(), rows=rows)
    got = out[:, torch.from_numpy(rows).to(dev)]
    mx, mean = check_output(to_np(got), ref, w.dtype, name)
    print(f"{name} union: ties={n_tie} loose heads={len(loose)} mean list "
          f"{float(cnt.float().mean()):.1f} max_abs={mx:.3e}")
