"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test ties one oracle function to an independent statement of what the
pages fix: a numpy reshape/transpose formulation of the blocked layout
(SPADE §3.3 layout transform; DecoupAttn Plans README block shapes
"frames x rows x cols"), brute-force means (SPADE §3.1 MEAN-SPADE), scipy's
softmax (SPADE §3.3 inter-block matrix), exhaustive subset search for Top-K
and Top-P (SPADE §3.1 "Top-K/Top-P mode"), torch's fp64 scaled-dot-product
attention, dense (SPADE §2.2 Eq. (1)) and with an explicit token mask
(Eq. (2)), and closed forms (V = 1 gives O = 1; equal keys give the plain
mean of the allowed values).
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers --
def token_table(g):
    """[nb + nb_text, bs] original token id of every slot, -1 for pad.

    Built by padding a (T,H,W) id grid and splitting it with reshape/transpose:
    block (tb,yb,xb) raster, slot (dt,dy,dx) raster; text blocks follow.
    """
    Tp, Hp, Wp = g.nbt * g.bf, g.nby * g.br, g.nbx * g.bc
    ids = np.full((Tp, Hp, Wp), -1, dtype=np.int64)
    ids[:g.T, :g.H, :g.W] = np.arange(g.n_video).reshape(g.T, g.H, g.W)
    blocks = ids.reshape(g.nbt, g.bf, g.nby, g.br, g.nbx, g.bc).transpose(0, 2, 4, 1, 3, 5)
    blocks = blocks.reshape(g.nb, g.bs)
    text = np.full(g.nb_text * g.bs, -1, dtype=np.int64)
    text[:g.n_text] = g.n_video + np.arange(g.n_text)
    return np.concatenate([blocks, text.reshape(g.nb_text, g.bs)], axis=0)


def rand_x(g, seed):
    return np.random.default_rng(seed).standard_normal((g.B, g.n_tot, g.Hd, g.D)).astype(np.float32)


def token_mask(g, idx, cnt):
    """[B, Hd, Ntot, Ntot] boolean: query token may attend key token."""
    tab = token_table(g)
    blk_of = np.empty(g.n_tot, dtype=np.int64)
    for j in range(tab.shape[0]):
        for t in tab[j]:
            if t >= 0:
                blk_of[t] = j
    mask = np.zeros((g.B, g.Hd, g.n_tot, g.n_tot), dtype=bool)
    for b in range(g.B):
        for h in range(g.Hd):
            for qb in range(g.nb):
                keys = np.concatenate([tab[j][tab[j] >= 0] for j in idx[b, h, qb, :cnt[b, h, qb]]])
                qs = tab[qb][tab[qb] >= 0]
                mask[b, h, np.ix_(qs, keys)[0], np.ix_(qs, keys)[1]] = True
            for qb in range(g.nb, g.nb + g.nb_text):
                qs = tab[qb][tab[qb] >= 0]
                mask[b, h, qs, :] = True
    return mask


def sdpa(q, k, v, mask=None):
    """torch fp64 scaled-dot-product attention in the original layout."""
    tq = torch.from_numpy(np.asarray(q, np.float64)).permute(0, 2, 1, 3)
    tk = torch.from_numpy(np.asarray(k, np.float64)).permute(0, 2, 1, 3)
    tv = torch.from_numpy(np.asarray(v, np.float64)).permute(0, 2, 1, 3)
    m = None if mask is None else torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=m)
    return o.permute(0, 2, 1, 3).numpy()


def random_lists(g, seed, max_blocks=None):
    """Random ascending lists of distinct video blocks + all text blocks."""
    rng = np.random.default_rng(seed)
    kmax = g.nb + g.nb_text
    idx = np.full((g.B, g.Hd, g.nb, kmax), -1, dtype=np.int32)
    cnt = np.zeros((g.B, g.Hd, g.nb), dtype=np.int32)
    for b in range(g.B):
        for h in range(g.Hd):
            for i in range(g.nb):
                m = rng.integers(1, (max_blocks or g.nb) + 1)
                sel = np.sort(rng.choice(g.nb, size=m, replace=False))
                lst = list(sel) + list(range(g.nb, g.nb + g.nb_text))
                idx[b, h, i, :len(lst)] = lst
                cnt[b, h, i] = len(lst)
    return idx, cnt


RAGGED = dict(B=2, T=3, H=5, W=7, bf=2, br=4, bc=4, Hd=2, D=16, n_text=5)
EVEN = dict(B=1, T=4, H=8, W=8, bf=2, br=4, bc=4, Hd=2, D=8, n_text=0)


# ------------------------------------------------------------ layout pins --
@pytest.mark.parametrize("geo", [EVEN, RAGGED, dict(B=1, T=5, H=9, W=6, bf=1, br=8, bc=16,
                                                    Hd=3, D=8, n_text=130)])
def test_permute_matches_reshape_layout(geo):
    g = orc.Geometry(**geo)
    x = rand_x(g, 1)
    tab = token_table(g).reshape(-1)
    expect = np.zeros((g.B, g.Hd, g.npad_tot, g.D))
    valid = tab >= 0
    expect[:, :, valid, :] = x[:, tab[valid], :, :].transpose(0, 2, 1, 3)
    got = orc.permute(g, x)
    assert np.array_equal(got, expect)
    # every valid token appears exactly once; pads are exactly zero
    assert np.array_equal(np.sort(tab[valid]), np.arange(g.n_tot))
    assert np.all(got[:, :, ~valid, :] == 0)


@pytest.mark.parametrize("geo", [EVEN, RAGGED])
def test_unpermute_inverts_permute(geo):
    g = orc.Geometry(**geo)
    x = rand_x(g, 2)
    assert np.array_equal(orc.unpermute(g, orc.permute(g, x)), x.astype(np.float64))


def test_permute_dense_even_grid_is_pure_transpose():
    # 1x1x1 blocks: the blocked layout is just [B, Hd, N, D]
    g = orc.Geometry(B=1, T=2, H=3, W=4, bf=1, br=1, bc=1, Hd=2, D=4, n_text=3)
    x = rand_x(g, 3)
    assert np.array_equal(orc.permute(g, x), x.transpose(0, 2, 1, 3).astype(np.float64))


# ----------------------------------------------------------- centroid pin --
@pytest.mark.parametrize("geo", [EVEN, RAGGED])
def test_centroids_are_means_over_valid_tokens(geo):
    g = orc.Geometry(**geo)
    x = rand_x(g, 4)
    Tp, Hp, Wp = g.nbt * g.bf, g.nby * g.br, g.nbx * g.bc
    grid = np.full((g.B, Tp, Hp, Wp, g.Hd, g.D), np.nan)
    grid[:, :g.T, :g.H, :g.W] = x[:, :g.n_video].reshape(g.B, g.T, g.H, g.W, g.Hd, g.D)
    blk = grid.reshape(g.B, g.nbt, g.bf, g.nby, g.br, g.nbx, g.bc, g.Hd, g.D)
    expect = np.nanmean(blk, axis=(2, 4, 6)).reshape(g.B, g.nb, g.Hd, g.D).transpose(0, 2, 1, 3)
    np.testing.assert_allclose(orc.centroids(g, x), expect, rtol=0, atol=1e-12)


# -------------------------------------------------------------- score pin --
def test_scores_are_row_softmax_of_scaled_dots():
    g = orc.Geometry(**RAGGED)
    rng = np.random.default_rng(5)
    qc = rng.standard_normal((g.B, g.Hd, g.nb, g.D))
    kc = rng.standard_normal((g.B, g.Hd, g.nb, g.D))
    expect = scipy.special.softmax(np.einsum("bhid,bhjd->bhij", qc, kc) / math.sqrt(g.D), axis=-1)
    got = orc.scores(g, qc, kc)
    np.testing.assert_allclose(got, expect, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(got.sum(-1), 1.0, rtol=0, atol=1e-12)


# ---------------------------------------------------------- selection pins --
def _golden_k_table():
    rows = []
    with open(os.path.join(GOLDEN, "k_for_density.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rho, nb, k = line.split()
                rows.append((float(rho), int(nb), int(k)))
    return rows


def test_k_for_density_golden():
    rows = _golden_k_table()
    assert len(rows) >= 9
    for rho, nb, k in rows:
        assert orc.k_for_density(rho, nb) == k, (rho, nb, k)


def _rand_p(g, seed, spread=2.0):
    rng = np.random.default_rng(seed)
    s = rng.standard_normal((g.B, g.Hd, g.nb, g.nb)) * spread
    return scipy.special.softmax(s, axis=-1)


@pytest.mark.parametrize("rho", [0.125, 0.25, 0.5, 0.75, 1.0])
def test_topk_is_max_mass_subset(rho):
    g = orc.Geometry(**RAGGED)          # nb = 8, one text block
    p = _rand_p(g, 6)
    idx, cnt, tie = orc.select(g, p, 0, [rho] * g.Hd)
    k = orc.k_for_density(rho, g.nb)
    assert np.all(cnt == k + g.nb_text)
    for b, h, i in itertools.product(range(g.B), range(g.Hd), range(g.nb)):
        best = max(itertools.combinations(range(g.nb), k), key=lambda s: p[b, h, i, list(s)].sum())
        lst = list(idx[b, h, i, :cnt[b, h, i]])
        assert lst == sorted(best) + list(range(g.nb, g.nb + g.nb_text))
        assert tie[b, h, i] == 0


@pytest.mark.parametrize("tau", [0.3, 0.5, 0.9, 0.99, 1.0])
def test_topp_is_shortest_prefix_reaching_tau(tau):
    g = orc.Geometry(**RAGGED)
    p = _rand_p(g, 7)
    idx, cnt, tie = orc.select(g, p, 1, [tau] * g.Hd)
    for b, h, i in itertools.product(range(g.B), range(g.Hd), range(g.nb)):
        if tie[b, h, i]:
            continue
        row = p[b, h, i]
        for m in range(1, g.nb + 1):
            best = max(itertools.combinations(range(g.nb), m), key=lambda s: row[list(s)].sum())
            if row[list(best)].sum() >= tau:
                break
        lst = list(idx[b, h, i, :cnt[b, h, i]])
        assert lst == sorted(best) + list(range(g.nb, g.nb + g.nb_text)), (b, h, i)


def test_topk_ties_break_by_lower_index_and_are_reported():
    g = orc.Geometry(B=1, T=1, H=1, W=8, bf=1, br=1, bc=1, Hd=1, D=4, n_text=0)
    p = np.full((1, 1, 8, 8), 1 / 8.0)
    idx, cnt, tie = orc.select(g, p, 0, [0.25])
    assert np.all(idx[0, 0, :, :2] == [0, 1]) and np.all(tie == 1)


def test_topp_tie_flag_near_threshold():
    g = orc.Geometry(B=1, T=1, H=1, W=4, bf=1, br=1, bc=1, Hd=1, D=4, n_text=0)
    p = np.tile(np.array([0.5, 0.3, 0.15, 0.05]), (1, 1, 4, 1))
    _, cnt, tie = orc.select(g, p, 1, [0.8])
    assert np.all(cnt == 2) and np.all(tie == 1)          # 0.5 + 0.3 == tau
    _, cnt, tie = orc.select(g, p, 1, [0.7])
    assert np.all(cnt == 2) and np.all(tie == 0)


# ---------------------------------------------------------- attention pins --
def test_density_one_equals_dense_attention():
    g = orc.Geometry(**RAGGED)
    q, k, v = rand_x(g, 8), rand_x(g, 9), rand_x(g, 10)
    idx = np.tile(np.arange(g.nb + g.nb_text, dtype=np.int32), (g.B, g.Hd, g.nb, 1))
    cnt = np.full((g.B, g.Hd, g.nb), g.nb + g.nb_text, dtype=np.int32)
    np.testing.assert_allclose(orc.attention(g, q, k, v, idx, cnt), sdpa(q, k, v),
                               rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("geo", [RAGGED, dict(B=1, T=5, H=9, W=6, bf=1, br=8, bc=16, Hd=2, D=8,
                                             n_text=130)])
def test_sparse_attention_equals_masked_sdpa(geo):
    g = orc.Geometry(**geo)
    q, k, v = rand_x(g, 11), rand_x(g, 12), rand_x(g, 13)
    idx, cnt = random_lists(g, 14)
    got = orc.attention(g, q, k, v, idx, cnt)
    np.testing.assert_allclose(got, sdpa(q, k, v, token_mask(g, idx, cnt)), rtol=1e-11, atol=1e-12)


def test_forward_pipeline_equals_masked_sdpa():
    g = orc.Geometry(**RAGGED)
    q, k, v = rand_x(g, 15), rand_x(g, 16), rand_x(g, 17)
    o, idx, cnt, tie, p = orc.forward(g, q, k, v, 0, [0.25] * g.Hd)
    assert np.all(cnt == 2 + g.nb_text)
    np.testing.assert_allclose(o, sdpa(q, k, v, token_mask(g, idx, cnt)), rtol=1e-11, atol=1e-12)


def test_ones_values_give_ones():
    g = orc.Geometry(**RAGGED)
    q, k = rand_x(g, 18), rand_x(g, 19)
    v = np.ones((g.B, g.n_tot, g.Hd, g.D), dtype=np.float32)
    idx, cnt = random_lists(g, 20)
    np.testing.assert_allclose(orc.attention(g, q, k, v, idx, cnt), 1.0, rtol=0, atol=1e-13)


def test_equal_keys_give_plain_mean_of_allowed_values():
    g = orc.Geometry(**RAGGED)
    q, v = rand_x(g, 21), rand_x(g, 22)
    k = np.ones((g.B, g.n_tot, g.Hd, g.D), dtype=np.float32)
    idx, cnt = random_lists(g, 23)
    m = token_mask(g, idx, cnt).astype(np.float64)                 # [B,Hd,Nq,Nk]
    expect = np.einsum("bhqk,bkhd->bqhd", m, v.astype(np.float64)) / m.sum(-1).transpose(0, 2, 1)[..., None]
    np.testing.assert_allclose(orc.attention(g, q, k, v, idx, cnt), expect, rtol=1e-12, atol=1e-13)


def test_row_subset_matches_full_output():
    g = orc.Geometry(**RAGGED)
    q, k, v = rand_x(g, 24), rand_x(g, 25), rand_x(g, 26)
    idx, cnt = random_lists(g, 27)
    full = orc.attention(g, q, k, v, idx, cnt)
    rows = np.array([0, 7, 33, g.n_video - 1, g.n_video, g.n_tot - 1])
    np.testing.assert_array_equal(orc.attention(g, q, k, v, idx, cnt, rows=rows), full[:, rows])


def test_selected_pairs_counts_mask_entries():
    g = orc.Geometry(**RAGGED)
    idx, cnt = random_lists(g, 28)
    assert orc.selected_pairs(g, idx, cnt) == int(token_mask(g, idx, cnt).sum())


# ---------------------------------------------------------- SICS pins (SPADE §3.2)
def test_sics_equals_squared_norm_of_summed_unit_vectors():
    # Eq. (4) sums all pairwise cosines = || sum_k q_k/|q_k| ||^2 (algebra on Eq. (4))
    g = orc.Geometry(**RAGGED)
    x = rand_x(g, 40)
    tab = token_table(g)
    expect = np.zeros((g.B, g.Hd, g.nb))
    for b in range(g.B):
        for h in range(g.Hd):
            for j in range(g.nb):
                toks = tab[j][tab[j] >= 0]
                v = x[b, toks, h, :].astype(np.float64)
                u = v / np.linalg.norm(v, axis=1, keepdims=True)
                expect[b, h, j] = np.sum(u.sum(0) ** 2)
    np.testing.assert_allclose(orc.sics(g, x), expect, rtol=1e-12, atol=1e-10)


def test_sics_online_algorithm_equals_definition():
    g = orc.Geometry(**dict(RAGGED, D=24))
    x = rand_x(g, 41)
    np.testing.assert_allclose(orc.sics_online(g, x), orc.sics(g, x), rtol=1e-12, atol=1e-10)


def test_sics_special_cases():
    # identical directions -> every cosine is 1 -> n^2; mutually orthogonal -> n (the diagonal)
    g = orc.Geometry(B=1, T=1, H=2, W=4, bf=1, br=2, bc=4, Hd=2, D=16, n_text=0)   # one block of 8
    x = np.zeros((1, g.n_tot, 2, 16), dtype=np.float32)
    x[0, :, 0, :] = np.arange(1, 17, dtype=np.float32) * 0.5          # head 0: all the same vector
    x[0, :, 0, :] *= np.arange(1, 9, dtype=np.float32)[:, None]       # ... with different norms
    x[0, :, 1, :] = np.eye(16, dtype=np.float32)[:8] * 3.0             # head 1: orthogonal
    s = orc.sics(g, x)
    assert abs(s[0, 0, 0] - 64.0) < 1e-9 and abs(s[0, 1, 0] - 8.0) < 1e-12
    # a zero vector contributes nothing (reading R15)
    x[0, 3, 1, :] = 0.0
    assert abs(orc.sics(g, x)[0, 1, 0] - 7.0) < 1e-12
    assert abs(orc.sics_online(g, x)[0, 1, 0] - 7.0) < 1e-12


def test_kmax_for_bounds_the_lists():
    # the list width is the longest list the selection can produce: Top-K lists
    # have exactly k_h + nb_text entries, so the widest reaches it; Top-P lists
    # never exceed it
    g = orc.Geometry(B=2, T=4, H=8, W=12, bf=2, br=4, bc=4, Hd=3, D=16, n_text=40)
    q, k = rand_x(g, 5), rand_x(g, 6)
    p = orc.scores(g, orc.centroids(g, q), orc.centroids(g, k))
    dens = [0.1, 0.35, 0.6]
    _, cnt, _ = orc.select(g, p, 0, dens)
    assert orc.kmax_for(g, 0, dens) == int(cnt.max())
    _, cnt, _ = orc.select(g, p, 1, [0.5, 0.9, 1.0])
    assert int(cnt.max()) <= orc.kmax_for(g, 1, [0.5, 0.9, 1.0])


def test_aggregation_score_and_scheme_choice():
    # AS = sum of block SICS (Eq. (3)); the chosen scheme maximises it
    base = dict(B=1, T=4, H=8, W=8, Hd=3, D=16, n_text=0)
    geoms = [orc.Geometry(bf=1, br=8, bc=8, **base), orc.Geometry(bf=4, br=4, bc=4, **base),
             orc.Geometry(bf=2, br=2, bc=16, **base)]
    x = rand_x(geoms[0], 42)
    choice, scores = orc.choose_scheme(geoms, x)
    for gi, g in enumerate(geoms):
        np.testing.assert_allclose(scores[gi], orc.sics(g, x).sum(-1), rtol=1e-13)
    assert np.all(scores[choice[0], 0, np.arange(3)] >= scores.max(0)[0] - 1e-12)


def test_aggregation_score_closed_forms():
    """AS on inputs built so that every block's sum of unit vectors is known:
    the tokens point along coordinate axes (each scaled by a random positive
    factor, which normalisation removes), so a block's SICS is |sum of unit
    vectors|^2 = sum over axes of (signed token count along that axis)^2
    (SPADE §3.2, Eq. (4), diagonal included), and AS (Eq. (3)) sums it over the
    blocks.  Each head's axis pattern follows one blocking scheme, so the
    scheme choice is known too."""
    T, H, W, D = 4, 8, 8, 16
    base = dict(B=1, T=T, H=H, W=W, Hd=5, D=D, n_text=0)
    geoms = [orc.Geometry(bf=1, br=8, bc=8, **base),     # one frame per block
             orc.Geometry(bf=4, br=4, bc=4, **base),     # 4x4x4 cubes
             orc.Geometry(bf=2, br=2, bc=16, **base)]    # 2x2x16, ragged in W (8 real columns)
    rng = np.random.default_rng(5)
    x = np.zeros((1, T * H * W, 5, D), dtype=np.float32)
    for t in range(T):
        for y in range(H):
            for c in range(W):
                n = (t * H + y) * W + c
                s = rng.uniform(0.25, 4.0, size=5).astype(np.float32)
                x[0, n, 0, t] = s[0]                                   # axis = frame
                x[0, n, 1, 2 * (y // 4) + c // 4] = s[1]               # axis = (y, x) quadrant
                x[0, n, 2, 4 * (t // 2) + y // 2] = s[2]               # axis = (frame pair, row pair)
                x[0, n, 3, t] = s[3] * (1 if c % 2 == 0 else -1)       # frame axis, sign by column parity
                if t > 0:
                    x[0, n, 4, t] = s[4]                               # head 0's pattern, frame 0 zero
    # per scheme (rows) and head (columns), from the counts above:
    #  head 0: frame blocks hold 64 tokens on one axis (4 * 64^2); a cube holds
    #          16 per frame on 4 axes (4 blocks * 4 * 16^2); a 2x2x8 block 16 on
    #          each of 2 axes (8 blocks * 2 * 16^2)
    #  head 1: a frame holds 16 tokens on each of 4 axes; a cube 64 on one axis;
    #          a 2x2x8 block 16 on each of 2 axes
    #  head 2: a frame holds 16 on each of 4 axes; a cube 16 on each of 4 axes;
    #          a 2x2x8 block 32 on one axis
    #  head 3: every block holds as many -e as +e tokens on each axis: 0
    #  head 4: head 0 without frame 0 (zero vectors count for nothing):
    #          3 * 64^2; 4 cubes * 3 * 16^2; 4 blocks * 16^2 + 4 blocks * 2 * 16^2
    expect = np.array([[16384, 4096, 4096, 0, 12288],
                       [4096, 16384, 4096, 0, 3072],
                       [4096, 4096, 8192, 0, 3072]], dtype=np.float64)
    choice, scores = orc.choose_scheme(geoms, x)
    np.testing.assert_allclose(scores[:, 0, :], expect, rtol=1e-12, atol=1e-9)
    # head 3 is a three-way tie: the lowest scheme index
    assert list(choice[0]) == [0, 1, 2, 0, 0]


# ------------------------------------------------ mask-union pins (SPADE §3.3)
def _inter_sets(g, p, mode, params):
    idx, cnt, _ = orc.select(g, p, mode, params)
    return {(b, h, i): set(int(j) for j in idx[b, h, i, :cnt[b, h, i] - g.nb_text])
            for b in range(g.B) for h in range(g.Hd) for i in range(g.nb)}


def _max_mass_prefix(v, tau_total):
    """Smallest m whose best m-subset reaches tau_total, by exhaustive search;
    returns that subset (the m largest, ties to the lower index)."""
    nb = len(v)
    for m in range(1, nb + 1):
        best = max(itertools.combinations(range(nb), m), key=lambda c: (sum(v[j] for j in c),
                                                                        [-j for j in c]))
        if sum(v[j] for j in best) >= tau_total:
            return set(best)
    return set(range(nb))


def test_union_window_predicate():
    g = orc.Geometry(**RAGGED)
    p = _rand_p(g, 20)
    inter = _inter_sets(g, p, 0, [0.25, 0.25])
    for window in [(0, 0), (1, 2), (2, -1), (-1, 1), (-1, -1), (100, 100)]:
        idx, cnt, _ = orc.select_union(g, p, 0, [0.25, 0.25], window=window)
        for (b, h, i), s in inter.items():
            lo = -10**9 if window[0] < 0 else i - window[0]
            hi = 10**9 if window[1] < 0 else i + window[1]
            win = set() if window == (-1, -1) else {j for j in range(g.nb) if lo <= j <= hi}
            expect = sorted(s | win) + list(range(g.nb, g.nb + g.nb_text))
            assert list(idx[b, h, i, :cnt[b, h, i]]) == expect, (window, b, h, i)


def test_union_sink_blocks_hold_the_first_tokens():
    g = orc.Geometry(**RAGGED)
    p = _rand_p(g, 21)
    inter = _inter_sets(g, p, 0, [0.25, 0.25])
    tab = token_table(g)[:g.nb]
    for sink in [0, 1, g.W, g.W + 1, g.H * g.W, g.n_video, g.n_tot]:
        blocks = {j for j in range(g.nb) if np.any((tab[j] >= 0) & (tab[j] < sink))}
        idx, cnt, _ = orc.select_union(g, p, 0, [0.25, 0.25], sink_tokens=sink)
        for (b, h, i), s in inter.items():
            assert list(idx[b, h, i, :cnt[b, h, i] - g.nb_text]) == sorted(s | blocks), sink
    assert {j for j in range(g.nb) if np.any((tab[j] >= 0) & (tab[j] < 1))} == {0}


@pytest.mark.parametrize("intra_mode,iparams", [(0, [0.25, 0.5]), (1, [0.3, 0.7]), (0, [1.0, 0.0])])
def test_union_intra_selection_broadcast(intra_mode, iparams):
    g = orc.Geometry(**RAGGED)                       # nb = 8
    p = _rand_p(g, 22)
    inter = _inter_sets(g, p, 1, [0.5, 0.8])
    v = np.random.default_rng(23).random((g.B, g.Hd, g.nb)) * 50.0
    idx, cnt, tie = orc.select_union(g, p, 1, [0.5, 0.8], intra=v, intra_mode=intra_mode,
                                     intra_params=iparams)
    for b in range(g.B):
        for h in range(g.Hd):
            row = v[b, h]
            if iparams[h] <= 0:
                isel = set()
            elif intra_mode == 0:
                k = orc.k_for_density(iparams[h], g.nb)
                isel = set(sorted(range(g.nb), key=lambda j: (-row[j], j))[:k])
            else:
                isel = _max_mass_prefix(row, iparams[h] * row.sum())
            for i in range(g.nb):
                got = list(idx[b, h, i, :cnt[b, h, i] - g.nb_text])
                assert got == sorted(inter[(b, h, i)] | isel), (b, h, i)


def test_union_of_everything_and_dense_cases():
    g = orc.Geometry(**dict(RAGGED, B=1))
    p = _rand_p(g, 24)
    v = np.random.default_rng(25).random((g.B, g.Hd, g.nb))
    full = list(range(g.nb + g.nb_text))
    # any single source at full strength gives dense rows
    for kw in [dict(window=(-1, 10**6)), dict(window=(10**6, -1)), dict(sink_tokens=g.n_video),
               dict(intra=v, intra_mode=0, intra_params=[1.0, 1.0]),
               dict(intra=v, intra_mode=1, intra_params=[1.0, 1.0])]:
        idx, cnt, _ = orc.select_union(g, p, 0, [0.125, 0.125], **kw)
        assert np.all(cnt == g.nb + g.nb_text)
        assert list(idx[0, 1, 3, :cnt[0, 1, 3]]) == full
    # the union is the OR of the separately computed unions
    parts = [orc.select_union(g, p, 0, [0.125, 0.25], window=(1, 0)),
             orc.select_union(g, p, 0, [0.125, 0.25], sink_tokens=9),
             orc.select_union(g, p, 0, [0.125, 0.25], intra=v, intra_params=[0.25, 0.25])]
    idx, cnt, _ = orc.select_union(g, p, 0, [0.125, 0.25], window=(1, 0), sink_tokens=9, intra=v,
                                   intra_params=[0.25, 0.25])
    for h in range(g.Hd):
        for i in range(g.nb):
            u = set()
            for pi, pc, _ in parts:
                u |= set(pi[0, h, i, :pc[0, h, i]].tolist())
            assert list(idx[0, h, i, :cnt[0, h, i]]) == sorted(u)


def test_union_intra_ties_are_flagged():
    g = orc.Geometry(**dict(RAGGED, B=1))
    p = _rand_p(g, 26)
    v = np.arange(g.nb, dtype=np.float64)[None, None, :].repeat(2, axis=1) + 1.0
    v[0, 0, 5] = v[0, 0, 6]                        # k = 2 cut between two equal scores
    _, _, tie = orc.select_union(g, p, 0, [0.25, 0.25], intra=v, intra_params=[0.25, 0.25])
    assert tie[0, 0].all()


# ---------------------------------------- DSA / DSA2 pins (SPADE §3.1, Fig. 4)
@pytest.mark.parametrize("geo", [EVEN, RAGGED])
def test_box_summaries_are_max_and_min_over_valid_tokens(geo):
    g = orc.Geometry(**geo)
    x = rand_x(g, 30)
    Tp, Hp, Wp = g.nbt * g.bf, g.nby * g.br, g.nbx * g.bc
    grid = np.full((g.B, Tp, Hp, Wp, g.Hd, g.D), np.nan)
    grid[:, :g.T, :g.H, :g.W] = x[:, :g.n_video].reshape(g.B, g.T, g.H, g.W, g.Hd, g.D)
    blk = grid.reshape(g.B, g.nbt, g.bf, g.nby, g.br, g.nbx, g.bc, g.Hd, g.D)
    mx = np.nanmax(blk, axis=(2, 4, 6)).reshape(g.B, g.nb, g.Hd, g.D).transpose(0, 2, 1, 3)
    mn = np.nanmin(blk, axis=(2, 4, 6)).reshape(g.B, g.nb, g.Hd, g.D).transpose(0, 2, 1, 3)
    box = orc.box_summaries(g, x)
    assert np.array_equal(box[..., 0], mx) and np.array_equal(box[..., 1], mn)


def _corners(lo, hi):
    """All 2^D corners of the box [lo, hi]."""
    D = len(lo)
    for bits in itertools.product((0, 1), repeat=D):
        yield np.where(np.array(bits) == 1, hi, lo)


def test_dsa_estimate_is_max_over_key_box_corners():
    g = orc.Geometry(B=1, T=2, H=4, W=4, bf=1, br=2, bc=4, Hd=2, D=6, n_text=0)
    x_q, x_k = rand_x(g, 31), rand_x(g, 32)
    qb, kb = orc.box_summaries(g, x_q), orc.box_summaries(g, x_k)
    p = orc.scores_box(g, qb, kb, 1)
    for h in range(g.Hd):
        for i in range(g.nb):
            c = (qb[0, h, i, :, 0] + qb[0, h, i, :, 1]) / 2
            est = np.array([max(c @ k for k in _corners(kb[0, h, j, :, 1], kb[0, h, j, :, 0]))
                            for j in range(g.nb)]) / math.sqrt(g.D)
            np.testing.assert_allclose(p[0, h, i], scipy.special.softmax(est), rtol=1e-12)


def test_dsa2_estimate_is_max_over_both_boxes():
    g = orc.Geometry(B=1, T=2, H=2, W=4, bf=1, br=2, bc=2, Hd=1, D=4, n_text=0)
    x_q, x_k = rand_x(g, 33), rand_x(g, 34)
    qb, kb = orc.box_summaries(g, x_q), orc.box_summaries(g, x_k)
    p = orc.scores_box(g, qb, kb, 2)
    for i in range(g.nb):
        qs = list(_corners(qb[0, 0, i, :, 1], qb[0, 0, i, :, 0]))
        est = np.array([max(qv @ kv for qv in qs for kv in _corners(kb[0, 0, j, :, 1], kb[0, 0, j, :, 0]))
                        for j in range(g.nb)]) / math.sqrt(g.D)
        np.testing.assert_allclose(p[0, 0, i], scipy.special.softmax(est), rtol=1e-12)


def test_box_estimates_bound_the_token_dot_products():
    # DSA2 >= every q_a . k_b of the two blocks; DSA >= every c . k_b
    g = orc.Geometry(**dict(RAGGED, B=1, n_text=0))
    x_q, x_k = rand_x(g, 35), rand_x(g, 36)
    qb, kb = orc.box_summaries(g, x_q), orc.box_summaries(g, x_k)
    tab = token_table(g)
    for h in range(g.Hd):
        for i in range(g.nb):
            qa = x_q[0, tab[i][tab[i] >= 0], h].astype(np.float64)
            c = (qb[0, h, i, :, 0] + qb[0, h, i, :, 1]) / 2
            for j in range(g.nb):
                kk = x_k[0, tab[j][tab[j] >= 0], h].astype(np.float64)
                e1 = np.maximum(c * kb[0, h, j, :, 0], c * kb[0, h, j, :, 1]).sum()
                q4 = np.stack([qb[0, h, i, :, 0] * kb[0, h, j, :, 0], qb[0, h, i, :, 0] * kb[0, h, j, :, 1],
                               qb[0, h, i, :, 1] * kb[0, h, j, :, 0], qb[0, h, i, :, 1] * kb[0, h, j, :, 1]])
                e2 = q4.max(0).sum()
                assert e1 >= (kk @ c).max() - 1e-9
                assert e2 >= (qa @ kk.T).max() - 1e-9
    # one-token blocks: the boxes are points, both estimates are the dot product
    g1 = orc.Geometry(B=1, T=1, H=2, W=3, bf=1, br=1, bc=1, Hd=1, D=5, n_text=0)
    xq, xk = rand_x(g1, 37), rand_x(g1, 38)
    dots = xq[0, :, 0].astype(np.float64) @ xk[0, :, 0].astype(np.float64).T / math.sqrt(5)
    for v in (1, 2):
        p = orc.scores_box(g1, orc.box_summaries(g1, xq), orc.box_summaries(g1, xk), v)
        np.testing.assert_allclose(p[0, 0], scipy.special.softmax(dots, axis=-1), rtol=1e-12)
