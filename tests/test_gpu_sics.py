"""GPU parity of the intra-block estimator and the blocking-scheme choice
(SPADE §3.2, Eq. (3)-(5)): bsa_sics and bsa_aggregation_scores through the
C ABI against the fp64 oracle on the same seeded inputs.

SICS values are compared with the forward error bound of the fp32 kernel
(parity.sics_tol); the Aggregation Scores with the sum of those bounds; the
choice must be the argmax of the kernel's own scores, and must equal the
oracle's wherever the oracle's best score leads every other candidate by more
than the two bounds together.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_permute_b200 as bsa
import oracle as orc
import synthetic
from parity import check_sics, sics_tol, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bsa.load()
    return torch.device("cuda", 0)


# name: (B, T, H, W, Hd, D, n_text, dtype, candidate block shapes)
CASES = {
    "hy_like_text": (1, 6, 12, 20, 3, 128, 130, "bf16", [(1, 8, 16), (2, 4, 16), (6, 4, 4)]),
    "wan_like_b2_d64": (2, 9, 10, 20, 2, 64, 0, "bf16", [(4, 4, 8), (1, 8, 16), (8, 2, 8)]),
    "f32_d128_ragged": (1, 5, 9, 13, 2, 128, 7, "f32", [(2, 4, 4), (1, 2, 16), (5, 1, 8)]),
    "f32_d64_eight": (1, 4, 8, 16, 2, 64, 0, "f32",
                      [(1, 8, 16), (2, 4, 16), (4, 4, 8), (4, 2, 16), (1, 4, 32), (2, 8, 8),
                       (4, 8, 4), (1, 1, 1)]),
    "one_scheme": (1, 3, 8, 8, 1, 128, 0, "bf16", [(1, 4, 4)]),
}


def _plans(B, T, H, W, Hd, D, n_text, dtype, shapes, dev):
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    return [bsa.Plan(B, T, H, W, bf, br, bc, Hd, D, n_text, dt, dev) for bf, br, bc in shapes]


def _geoms(B, T, H, W, Hd, D, n_text, shapes):
    return [orc.Geometry(B, T, H, W, bf, br, bc, Hd, D, n_text) for bf, br, bc in shapes]


def _as_tol(geoms, ref_sics):
    """Bound on |AS_gpu - AS_ref| per candidate: the sum of the SICS bounds plus
    the double-precision sum of nb fp32 values."""
    out = []
    for g, s in zip(geoms, ref_sics):
        t = sics_tol(g, s).sum(-1)
        out.append(t + 1e-12 * s.sum(-1) * g.nb)
    return np.stack(out)


def _verify(geoms, x_np, sics, as_, choice):
    ref_sics = [orc.sics(g, x_np) for g in geoms]
    worst = 0.0
    for c, g in enumerate(geoms):
        _, w = check_sics(g, sics[c].cpu().numpy(), ref_sics[c], f"candidate {c}")
        worst = max(worst, w)
    ref_as = np.stack([s.sum(-1) for s in ref_sics])              # [n, B, Hd]
    np.testing.assert_allclose(ref_as, np.stack([orc.aggregation_score(g, x_np) for g in geoms]),
                               rtol=1e-12)
    gpu_as = as_.cpu().numpy()
    tol = _as_tol(geoms, ref_sics)
    assert np.all(np.abs(gpu_as - ref_as) <= tol), float(np.abs(gpu_as - ref_as).max())
    # the kernel's AS is the fixed-order double sum of its own SICS values
    own = np.stack([s.cpu().double().numpy().sum(-1) for s in sics])
    np.testing.assert_allclose(gpu_as, own, rtol=1e-12, atol=1e-9)
    gch = choice.cpu().numpy()
    assert np.array_equal(gch, np.argmax(gpu_as, axis=0))
    ref_choice, _ = orc.choose_scheme(geoms, x_np)
    n_clear = 0
    for b in range(gch.shape[0]):
        for h in range(gch.shape[1]):
            best = ref_choice[b, h]
            lead = all(ref_as[best, b, h] - ref_as[c, b, h] > tol[best, b, h] + tol[c, b, h]
                       for c in range(len(geoms)) if c != best)
            if lead:
                n_clear += 1
                assert gch[b, h] == best, (b, h, gch[b, h], best)
            else:   # near-equal candidates: the kernel's pick is one of them
                c = gch[b, h]
                assert ref_as[best, b, h] - ref_as[c, b, h] <= tol[best, b, h] + tol[c, b, h]
    return worst, n_clear


@pytest.mark.parametrize("name", list(CASES))
def test_aggregation_scores_match_oracle(name, dev):
    B, T, H, W, Hd, D, n_text, dtype, shapes = CASES[name]
    q, _, _ = synthetic.make_custom(B, T, H, W, Hd, D, n_text, dtype)
    plans = _plans(B, T, H, W, Hd, D, n_text, dtype, shapes, dev)
    sics, as_, choice = bsa.aggregation_scores(plans, q.to(dev))
    torch.cuda.synchronize()
    geoms = _geoms(B, T, H, W, Hd, D, n_text, shapes)
    worst, n_clear = _verify(geoms, to_np(q), sics, as_, choice)
    print(f"{name}: worst err/bound {worst:.2e}, clear choices {n_clear}/{B * Hd}")


@pytest.mark.parametrize("name", ["hy_like_text", "f32_d128_ragged"])
def test_single_plan_sics_equals_multi(name, dev):
    """bsa_sics of one plan is the candidate's slice of the multi-scheme call."""
    B, T, H, W, Hd, D, n_text, dtype, shapes = CASES[name]
    q, _, _ = synthetic.make_custom(B, T, H, W, Hd, D, n_text, dtype)
    qd = q.to(dev)
    plans = _plans(B, T, H, W, Hd, D, n_text, dtype, shapes, dev)
    sics, _, _ = bsa.aggregation_scores(plans, qd)
    for c, p in enumerate(plans):
        one = p.sics(qd)
        torch.cuda.synchronize()
        assert torch.equal(one, sics[c])


def test_special_rows(dev):
    """Identical directions give n^2, orthogonal rows give n, zero rows count 0
    (values exact in bf16, so both dtypes see the same rows)."""
    B, T, H, W, Hd, D = 1, 2, 4, 16, 3, 128
    n_tok = T * H * W                                   # 128 tokens, two 2x4x8 blocks
    x = torch.zeros((B, n_tok, Hd, D), dtype=torch.float32)
    base = torch.linspace(0.5, 2.0, D).to(torch.bfloat16).float()
    x[0, :, 0, :] = base * (2.0 ** (torch.arange(n_tok) % 8).float())[:, None]
    x[0, :, 1, :] = torch.eye(D)[:n_tok] * 3.0
    x[0, :, 2, :] = x[0, :, 1, :]
    x[0, ::3, 2, :] = 0.0
    n = torch.arange(n_tok)
    blk = (n % W) // 8
    nonzero = x[0, :, 2, :].abs().sum(-1) > 0
    counts = [int(nonzero[blk == j].sum()) for j in range(2)]
    g = orc.Geometry(B, T, H, W, 2, 4, 8, Hd, D, 0)
    ref = orc.sics(g, x.numpy())
    np.testing.assert_allclose(ref[0, 0], [64.0 ** 2] * 2, rtol=1e-12)
    np.testing.assert_allclose(ref[0, 1], [64.0] * 2, rtol=1e-12)
    np.testing.assert_allclose(ref[0, 2], counts, rtol=1e-12)
    for dt in (torch.float32, torch.bfloat16):
        plan = bsa.Plan(B, T, H, W, 2, 4, 8, Hd, D, 0, dt, dev)
        s = plan.sics(x.to(dt).to(dev)).cpu().double().numpy()
        check_sics(g, s, ref, f"special {dt}")


def test_empty_and_invalid_calls(dev):
    plan = bsa.Plan(1, 2, 8, 8, 1, 8, 8, 2, 64, 0, torch.bfloat16, dev)
    other = bsa.Plan(1, 2, 8, 16, 1, 8, 8, 2, 64, 0, torch.bfloat16, dev)
    x = torch.zeros(plan.orig_shape, dtype=torch.bfloat16, device=dev)
    with pytest.raises(bsa.BsaError) as e:
        bsa.aggregation_scores([plan, other], x)
    assert e.value.status == 1
    with pytest.raises(bsa.BsaError):
        bsa.aggregation_scores([plan] * 9, x)
    s = plan.sics(x)                       # all-zero input: every SICS is 0
    torch.cuda.synchronize()
    assert torch.count_nonzero(s).item() == 0


FULL_SCHEMES = {
    "hunyuan": [(1, 8, 16), (4, 4, 8), (16, 1, 8)],
    "wan13": [(4, 4, 8), (1, 8, 16), (8, 2, 8)],
}


@pytest.mark.parametrize("name", list(FULL_SCHEMES))
def test_full_size_aggregation(name, dev):
    """Full workload, one launch over three candidate schemes; the oracle checks
    two sampled heads in full (SICS of every block, AS and choice)."""
    w = synthetic.workload(name)
    q, _, _ = synthetic.make_qkv(w)
    shapes = FULL_SCHEMES[name]
    plans = _plans(w.B, w.T, w.H, w.W, w.Hd, w.D, w.n_text, w.dtype, shapes, dev)
    sics, as_, choice = bsa.aggregation_scores(plans, q.to(dev))
    torch.cuda.synchronize()
    heads = [0, w.Hd - 1]
    geoms = _geoms(w.B, w.T, w.H, w.W, 1, w.D, w.n_text, shapes)
    worst_all = 0.0
    for h in heads:
        xh = to_np(q[:, :, h:h + 1, :].contiguous())
        worst, _ = _verify(geoms, xh, [s[:, h:h + 1].contiguous() for s in sics],
                           as_[:, :, h:h + 1], choice[:, h:h + 1])
        worst_all = max(worst_all, worst)
    print(f"{name}: worst err/bound {worst_all:.2e}; choices {choice.cpu().numpy().ravel().tolist()}")
