"""Shared helpers of the GPU parity tests: CUDA path vs the fp64 oracle.

Tolerances (from the stated bar):
  * layouts, index lists and counts: bit-exact, except rows the oracle
    reports as ties (k-th and (k+1)-th scores, or the Top-P cumulative mass
    at the cut, within 1e-5 relative); such rows must still be a valid
    selection within that tolerance.
  * attention output, bf16 inputs: max-abs <= 2e-2 and mean-abs <= 2e-3.
  * attention output, fp32 inputs: max-abs <= 1e-5.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as orc
import synthetic

TOL_BF16_MAX, TOL_BF16_MEAN = 2e-2, 2e-3
TOL_F32_MAX = 1e-5
TIE_REL = 1e-5


def geometry(w) -> orc.Geometry:
    return orc.Geometry(*w.geometry_args())


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy() if t.dtype == torch.bfloat16 else t.detach().cpu().numpy()


def bound_ties(g, p, tol, mode, params):
    """[B, Hd, nb] rows whose Top-K / Top-P cut could move when every p_ij may
    be off by up to tol_ij (a derived error bound of the kernel's scores)."""
    tie = np.zeros((g.B, g.Hd, g.nb), dtype=np.int32)
    for b in range(g.B):
        for h in range(g.Hd):
            for i in range(g.nb):
                row, t = p[b, h, i], tol[b, h, i]
                order = np.lexsort((np.arange(g.nb), -row))
                v, tv = row[order], t[order]
                if mode == 0:
                    m = orc.k_for_density(params[h], g.nb)
                else:
                    c = np.cumsum(v)
                    m = min(int(np.searchsorted(c, params[h], side="left")) + 1, g.nb)
                    slack = tv.sum()
                    if abs(c[m - 1] - params[h]) <= slack or (m >= 2 and abs(c[m - 2] - params[h]) <= slack):
                        tie[b, h, i] = 1
                if m < g.nb and v[m - 1] - v[m] <= tv[m - 1] + tv[m]:
                    tie[b, h, i] = 1
    return tie


def check_lists(g, gpu_idx, gpu_cnt, o_idx, o_cnt, tie, p, mode, params, tol=None):
    """Bit-exact lists on non-tie rows; valid selections on tie rows. Returns #ties.

    tol (optional, like p): per-score error bounds; tie rows must then be a
    valid selection within those bounds instead of within TIE_REL."""
    gi, gc = gpu_idx.cpu().numpy(), gpu_cnt.cpu().numpy()
    assert gc.shape == o_cnt.shape
    n_tie = 0
    for b in range(g.B):
        for h in range(g.Hd):
            for i in range(g.nb):
                c = int(gc[b, h, i])
                lst = list(gi[b, h, i, :c])
                ref = list(o_idx[b, h, i, :o_cnt[b, h, i]])
                if lst == ref:
                    continue
                assert tie[b, h, i], f"list mismatch at b={b} h={h} i={i}: {lst[:8]}... vs {ref[:8]}..."
                n_tie += 1
                text = list(range(g.nb, g.nb + g.nb_text))
                assert lst[len(lst) - g.nb_text:] == text
                sel = np.array(lst[:len(lst) - g.nb_text], dtype=np.int64)
                assert np.all(np.diff(sel) > 0) and sel.min() >= 0 and sel.max() < g.nb
                row = p[b, h, i]
                uns = np.setdiff1d(np.arange(g.nb), sel)
                if tol is None:
                    if len(uns):
                        assert row[sel].min() >= row[uns].max() * (1 - TIE_REL) - 1e-300
                    if mode == 0:
                        assert len(sel) == orc.k_for_density(params[h], g.nb)
                    else:
                        tau = params[h]
                        mass = row[sel].sum()
                        assert mass >= tau * (1 - TIE_REL)
                        assert mass - row[sel].min() < tau * (1 + TIE_REL)
                else:
                    t = tol[b, h, i]
                    if len(uns):
                        assert (row[sel] + t[sel]).min() >= (row[uns] - t[uns]).max()
                    if mode == 0:
                        assert len(sel) == orc.k_for_density(params[h], g.nb)
                    else:
                        tau, slack = params[h], t.sum()
                        mass = row[sel].sum()
                        assert mass >= tau - slack
                        assert mass - row[sel].min() < tau + slack
    return n_tie


def check_output(gpu, ref, dtype_name, what=""):
    """Elementwise comparison at the stated tolerance; returns (max_abs, mean_abs)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite output"
    err = np.abs(gpu - ref)
    mx, mean = float(err.max()), float(err.mean())
    if dtype_name == "f32":
        assert mx <= TOL_F32_MAX, f"{what}: max-abs {mx:.3e} > {TOL_F32_MAX}"
    else:
        assert mx <= TOL_BF16_MAX, f"{what}: max-abs {mx:.3e} > {TOL_BF16_MAX}"
        assert mean <= TOL_BF16_MEAN, f"{what}: mean-abs {mean:.3e} > {TOL_BF16_MEAN}"
    return mx, mean


def sample_rows(g, seed=0, n_blocks=6, n_text=16):
    """Token rows for sampled comparison: all valid tokens of a few random video
    blocks, always the last (most padded) block, plus some text tokens."""
    rng = np.random.default_rng(seed)
    blocks = set(rng.choice(g.nb, size=min(n_blocks, g.nb), replace=False).tolist())
    blocks.add(g.nb - 1)
    rows = []
    for j in sorted(blocks):
        tb, yb, xb = j // (g.nby * g.nbx), (j // g.nbx) % g.nby, j % g.nbx
        for t in range(tb * g.bf, min(g.T, (tb + 1) * g.bf)):
            for y in range(yb * g.br, min(g.H, (yb + 1) * g.br)):
                for x in range(xb * g.bc, min(g.W, (xb + 1) * g.bc)):
                    rows.append((t * g.H + y) * g.W + x)
    if g.n_text:
        rows += sorted(rng.choice(g.n_text, size=min(n_text, g.n_text), replace=False)
                       + g.n_video)
    return np.array(rows, dtype=np.int64)


def custom_workload(name, B, T, H, W, bf, br, bc, Hd, D, n_text, dtype, mode, param):
    w = synthetic.Workload(name, B, T, H, W, bf, br, bc, Hd, D, dtype, mode, [param] * Hd,
                           n_text=n_text, qk_std=3.0 if dtype == "bf16" else None)
    return w


# ------------------------------------------------------------------ SICS --
U32 = 2.0 ** -24   # unit roundoff of fp32


def valid_counts(g) -> np.ndarray:
    """[nb] number of valid tokens of every video block."""
    j = np.arange(g.nb)
    tb, yb, xb = j // (g.nby * g.nbx), (j // g.nbx) % g.nby, j % g.nbx
    vt = np.minimum(g.bf, g.T - tb * g.bf)
    vy = np.minimum(g.br, g.H - yb * g.br)
    vx = np.minimum(g.bc, g.W - xb * g.bc)
    return (vt * vy * vx).astype(np.float64)


def sics_tol(g, ref) -> np.ndarray:
    """Forward error bound of the fp32 SICS kernel, per block ([..., nb]).

    The kernel forms r = sum_a x_a * rsqrt(|x_a|^2) and returns |r|^2, all in
    fp32, for n <= bs valid rows of D elements.  Each unit row carries a
    relative error of at most (D/2 + 3) u (the D-term sum of squares, rsqrtf's
    2 ulp, the product); the n-term sums of r add n u times sum_a |xhat_a|,
    whose norm is at most n.  So |delta r| <= n (n + D/2 + 3) u =: e and
    |delta |r|^2| <= 2 |r| e + e^2 + (D + 1) u |r|^2, with |r| = sqrt(SICS).
    """
    n = valid_counts(g)
    e = n * (n + g.D / 2 + 3) * U32
    r = np.sqrt(np.maximum(ref, 0.0))
    return 2 * r * e + e * e + (g.D + 1) * U32 * ref + 1e-6


def check_sics(g, gpu, ref, what=""):
    """SICS within the derived bound; returns (max_abs_err, max err/bound)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite SICS"
    tol = sics_tol(g, ref)
    err = np.abs(gpu - ref)
    worst = float((err / tol).max()) if err.size else 0.0
    assert worst <= 1.0, f"{what}: SICS error {float(err.max()):.3e} above its bound (x{worst:.2f})"
    return (float(err.max()) if err.size else 0.0), worst


# ------------------------------------------------------------ mask union --
def union_extras(g, window, sink_tokens, intra_sets):
    """Per (b, h, i): the set of video key blocks the window, sink and intra
    parts add (intra_sets[b][h] = set of key blocks or empty)."""
    wl, wr = window
    sink = set()
    for j in range(g.nb):
        tb, yb, xb = j // (g.nby * g.nbx), (j // g.nbx) % g.nby, j % g.nbx
        first = (tb * g.bf * g.H + yb * g.br) * g.W + xb * g.bc
        if first < sink_tokens:
            sink.add(j)
    out = {}
    for b in range(g.B):
        for h in range(g.Hd):
            for i in range(g.nb):
                win = set()
                if wl >= 0 or wr >= 0:
                    lo = 0 if wl < 0 else i - wl
                    hi = g.nb - 1 if wr < 0 else i + wr
                    win = set(range(max(lo, 0), min(hi, g.nb - 1) + 1))
                out[(b, h, i)] = win | sink | intra_sets[b][h]
    return out


def check_union_lists(g, gpu_idx, gpu_cnt, o_idx, o_cnt, tie, p, mode, params, extras,
                      loose_heads=()):
    """Lists of the mask union: bit-exact on non-tie rows.  On rows the oracle
    flags as inter ties, the list must be E plus a valid inter selection S
    (tie tolerance as check_lists).  Heads in loose_heads (an intra near-tie
    under the SICS error bound) must contain their window and sink blocks.
    Returns the number of tie rows."""
    gi, gc = gpu_idx.cpu().numpy(), gpu_cnt.cpu().numpy()
    n_tie = 0
    text = list(range(g.nb, g.nb + g.nb_text))
    for b in range(g.B):
        for h in range(g.Hd):
            for i in range(g.nb):
                c = int(gc[b, h, i])
                lst = [int(x) for x in gi[b, h, i, :c]]
                ref = [int(x) for x in o_idx[b, h, i, :o_cnt[b, h, i]]]
                if lst == ref:
                    continue
                assert lst[c - g.nb_text:] == text
                L = lst[:c - g.nb_text]
                assert all(x < y for x, y in zip(L, L[1:])) and (not L or (L[0] >= 0 and L[-1] < g.nb))
                if (b, h) in loose_heads:
                    continue
                assert tie[b, h, i], f"union list mismatch at b={b} h={h} i={i}"
                n_tie += 1
                E = extras[(b, h, i)]
                Ls = set(L)
                assert E <= Ls
                row = p[b, h, i]
                must = sorted(Ls - E)
                opt = sorted(Ls & E, key=lambda j: (-row[j], j))
                if mode == 0:
                    k = orc.k_for_density(params[h], g.nb)
                    assert len(must) <= k
                    S = set(must) | set(opt[:k - len(must)])
                    assert len(S) == k
                else:
                    S = set(must)
                    for j in opt:
                        if S and row[sorted(S)].sum() >= params[h] * (1 - TIE_REL):
                            break
                        S.add(j)
                    mass = row[list(S)].sum()
                    assert mass >= params[h] * (1 - TIE_REL)
                    assert mass - row[list(S)].min() < params[h] * (1 + TIE_REL)
                uns = np.setdiff1d(np.arange(g.nb), np.array(sorted(S)))
                if len(uns):
                    assert row[sorted(S)].min() >= row[uns].max() * (1 - TIE_REL) - 1e-300
    return n_tie


def intra_near_tie(values, tol, mode, param):
    """True when the Top-K / Top-P decision on `values` could change within
    per-entry error bounds `tol` (both 1-D)."""
    nb = len(values)
    order = sorted(range(nb), key=lambda j: (-values[j], j))
    v = np.asarray(values, dtype=np.float64)[order]
    t = np.asarray(tol, dtype=np.float64)[order]
    if mode == 0:
        m = orc.k_for_density(param, nb)
    else:
        target = param * v.sum()
        c = np.cumsum(v)
        m = int(np.searchsorted(c, target, side="left")) + 1
        m = min(max(m, 1), nb)
        slack = param * t.sum() + t.sum()
        if abs(c[m - 1] - target) <= slack or (m >= 2 and abs(c[m - 2] - target) <= slack):
            return True
    return m < nb and v[m - 1] - v[m] <= t[m - 1] + t[m]
