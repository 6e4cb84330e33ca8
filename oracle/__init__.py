"""fp64 CPU oracle of 3D block-sparse attention — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product (``block_sparse_attention_permute_b200`` and ``libbsa.so``) never
imports, links or executes it, and it shares no code with them.

Thin ctypes wrapper over ``oracle.cpp`` (plain double-precision C++ loops).
Each function cites the passage it follows; see ``oracle.cpp`` for the
readings taken where the pages are silent.

Parity pins (tests/test_oracle_pins.py) tie every function to something other
than itself: numpy reshape/transpose layouts, brute-force means, scipy
softmax, brute-force subset search for the selections, and torch's fp64
scaled-dot-product attention (dense and with an explicit token mask).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.cpp into liboracle.so (g++ -O2, plain C++17 + threads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        lib.orc_threads.restype = ctypes.c_int
        lib.orc_permute.argtypes = [P, P, P]
        lib.orc_unpermute.argtypes = [P, P, P]
        lib.orc_centroids.argtypes = [P, P, P]
        lib.orc_scores.argtypes = [P, P, P, P]
        lib.orc_k_for_density.argtypes = [ctypes.c_double, ctypes.c_int]
        lib.orc_k_for_density.restype = ctypes.c_int
        lib.orc_select.argtypes = [P, P, ctypes.c_int, P, ctypes.c_int, P, P, P]
        lib.orc_attention.argtypes = [P, P, P, P, P, P, ctypes.c_int, P, ctypes.c_longlong, P]
        lib.orc_select_union.argtypes = [P, P, ctypes.c_int, P, ctypes.c_int, P, ctypes.c_int, P,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_longlong, P, P, P]
        lib.orc_box_summaries.argtypes = [P, P, P]
        lib.orc_scores_box.argtypes = [P, P, P, ctypes.c_int, P]
        lib.orc_sics.argtypes = [P, P, P]
        lib.orc_sics_online.argtypes = [P, P, P]
        lib.orc_aggregation_score.argtypes = [P, P, P]
        lib.orc_selected_pairs.argtypes = [P, P, P, ctypes.c_int]
        lib.orc_selected_pairs.restype = ctypes.c_longlong
        _lib = lib
    return _lib


class Geometry:
    """Problem geometry: batch, grid (T,H,W), block (bf,br,bc), heads, head_dim, text."""

    def __init__(self, B, T, H, W, bf, br, bc, Hd, D, n_text=0):
        self.B, self.T, self.H, self.W = B, T, H, W
        self.bf, self.br, self.bc, self.Hd, self.D, self.n_text = bf, br, bc, Hd, D, n_text
        self.nbt, self.nby, self.nbx = -(-T // bf), -(-H // br), -(-W // bc)
        self.nb = self.nbt * self.nby * self.nbx
        self.bs = bf * br * bc
        self.nb_text = -(-n_text // self.bs)
        self.n_video = T * H * W
        self.n_tot = self.n_video + n_text
        self.npad_tot = (self.nb + self.nb_text) * self.bs
        self.arr = np.array([B, T, H, W, bf, br, bc, Hd, D, n_text], dtype=np.int32)


def _f32(x):
    return np.ascontiguousarray(x, dtype=np.float32)


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def threads() -> int:
    """Threads the oracle uses (ORACLE_THREADS or all host cores)."""
    return _load().orc_threads()


def permute(g: Geometry, x):
    """[B,Ntot,Hd,D] -> blocked [B,Hd,Npad_tot,D] float64 (SPADE §3.3 layout transform)."""
    x = _f32(x)
    out = np.empty((g.B, g.Hd, g.npad_tot, g.D), dtype=np.float64)
    _load().orc_permute(_ptr(g.arr), _ptr(x), _ptr(out))
    return out


def unpermute(g: Geometry, x_blk):
    """Blocked [B,Hd,Npad_tot,D] -> [B,Ntot,Hd,D] float64 (SPADE §3.3 restore layout)."""
    x_blk = np.ascontiguousarray(x_blk, dtype=np.float64)
    out = np.empty((g.B, g.n_tot, g.Hd, g.D), dtype=np.float64)
    _load().orc_unpermute(_ptr(g.arr), _ptr(x_blk), _ptr(out))
    return out


def centroids(g: Geometry, x):
    """Per video block mean over valid tokens, [B,Hd,nb,D] float64 (SPADE §3.1 MEAN-SPADE)."""
    x = _f32(x)
    out = np.empty((g.B, g.Hd, g.nb, g.D), dtype=np.float64)
    _load().orc_centroids(_ptr(g.arr), _ptr(x), _ptr(out))
    return out


def scores(g: Geometry, qc, kc):
    """Row softmax of qbar.kbar/sqrt(D), [B,Hd,nb,nb] float64 (SPADE §3.3 inter-block matrix)."""
    qc = np.ascontiguousarray(qc, dtype=np.float64)
    kc = np.ascontiguousarray(kc, dtype=np.float64)
    out = np.empty((g.B, g.Hd, g.nb, g.nb), dtype=np.float64)
    _load().orc_scores(_ptr(g.arr), _ptr(qc), _ptr(kc), _ptr(out))
    return out


def box_summaries(g: Geometry, x):
    """Per video block and dimension (max, min) over valid tokens, [B,Hd,nb,D,2]
    (SPADE §3.1 DSA / DSA2 summaries)."""
    x = _f32(x)
    out = np.empty((g.B, g.Hd, g.nb, g.D, 2), dtype=np.float64)
    _load().orc_box_summaries(_ptr(g.arr), _ptr(x), _ptr(out))
    return out


def scores_box(g: Geometry, qbox, kbox, variant: int):
    """Row softmax of the DSA (variant 1) or DSA2 (variant 2) estimate / sqrt(D).
    Parity unpinned: the estimator is a reading of SPADE §3.1 / Fig. 4 (the
    equations are not in the text), pinned only to a corner brute force."""
    qbox = np.ascontiguousarray(qbox, dtype=np.float64)
    kbox = np.ascontiguousarray(kbox, dtype=np.float64)
    out = np.empty((g.B, g.Hd, g.nb, g.nb), dtype=np.float64)
    _load().orc_scores_box(_ptr(g.arr), _ptr(qbox), _ptr(kbox), int(variant), _ptr(out))
    return out


def k_for_density(rho: float, nb: int) -> int:
    """ceil(rho*nb - 1e-9) clamped to [1, nb]."""
    return _load().orc_k_for_density(float(rho), int(nb))


def kmax_for(g: Geometry, mode: int, params) -> int:
    if mode == 0:
        return max(k_for_density(r, g.nb) for r in params) + g.nb_text
    return g.nb + g.nb_text


def select(g: Geometry, p, mode: int, params, kmax: int | None = None):
    """Top-K (mode 0, params = densities) or Top-P (mode 1, params = tau) per head.

    Returns (idx [B,Hd,nb,kmax] int32 padded with -1, cnt [B,Hd,nb], tie [B,Hd,nb]).
    """
    params = np.ascontiguousarray(params, dtype=np.float64)
    assert params.shape == (g.Hd,)
    if kmax is None:
        kmax = kmax_for(g, mode, params)
    p = np.ascontiguousarray(p, dtype=np.float64)
    idx = np.full((g.B, g.Hd, g.nb, kmax), -1, dtype=np.int32)
    cnt = np.zeros((g.B, g.Hd, g.nb), dtype=np.int32)
    tie = np.zeros((g.B, g.Hd, g.nb), dtype=np.int32)
    _load().orc_select(_ptr(g.arr), _ptr(p), int(mode), _ptr(params), int(kmax),
                       _ptr(idx), _ptr(cnt), _ptr(tie))
    return idx, cnt, tie


def select_union(g: Geometry, p, mode: int, params, window=(-1, -1), sink_tokens=0,
                 intra=None, intra_mode: int = 0, intra_params=None, kmax: int | None = None):
    """Lists of the mask union (SPADE §3.3): inter Top-K/Top-P of p, united with a
    sliding window over the block sequence, the attention-sink blocks and the
    intra-score selection broadcast over query blocks.  Returns (idx, cnt, tie)."""
    params = np.ascontiguousarray(params, dtype=np.float64)
    assert params.shape == (g.Hd,)
    if kmax is None:
        kmax = g.nb + g.nb_text
    p = np.ascontiguousarray(p, dtype=np.float64)
    ip = None
    if intra is not None:
        intra = np.ascontiguousarray(intra, dtype=np.float64)
        assert intra.shape == (g.B, g.Hd, g.nb)
        ip = np.ascontiguousarray(intra_params, dtype=np.float64)
        assert ip.shape == (g.Hd,)
    idx = np.full((g.B, g.Hd, g.nb, kmax), -1, dtype=np.int32)
    cnt = np.zeros((g.B, g.Hd, g.nb), dtype=np.int32)
    tie = np.zeros((g.B, g.Hd, g.nb), dtype=np.int32)
    _load().orc_select_union(_ptr(g.arr), _ptr(p), int(mode), _ptr(params), int(kmax),
                             None if intra is None else _ptr(intra), int(intra_mode),
                             None if ip is None else _ptr(ip), int(window[0]), int(window[1]),
                             int(sink_tokens), _ptr(idx), _ptr(cnt), _ptr(tie))
    return idx, cnt, tie


def attention(g: Geometry, q, k, v, idx, cnt, rows=None):
    """Exact masked softmax attention per query token, original layout (SPADE Eq. (2)).

    rows=None: output [B,Ntot,Hd,D]; else output [B,len(rows),Hd,D] for those tokens.
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    cnt = np.ascontiguousarray(cnt, dtype=np.int32)
    kmax = idx.shape[-1]
    if rows is None:
        out = np.empty((g.B, g.n_tot, g.Hd, g.D), dtype=np.float64)
        _load().orc_attention(_ptr(g.arr), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(cnt),
                              kmax, None, 0, _ptr(out))
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        out = np.empty((g.B, len(rows), g.Hd, g.D), dtype=np.float64)
        _load().orc_attention(_ptr(g.arr), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(cnt),
                              kmax, _ptr(rows), len(rows), _ptr(out))
    return out


def sics(g: Geometry, x):
    """Sum of intra-block cosine similarities per video block, [B,Hd,nb] (SPADE Eq. (4))."""
    x = _f32(x)
    out = np.empty((g.B, g.Hd, g.nb), dtype=np.float64)
    _load().orc_sics(_ptr(g.arr), _ptr(x), _ptr(out))
    return out


def sics_online(g: Geometry, x):
    """The same by the online form (SPADE Eq. (5), Algorithm 1), [B,Hd,nb]."""
    x = _f32(x)
    out = np.empty((g.B, g.Hd, g.nb), dtype=np.float64)
    _load().orc_sics_online(_ptr(g.arr), _ptr(x), _ptr(out))
    return out


def aggregation_score(g: Geometry, x):
    """AS = sum of SICS over video blocks, [B,Hd] (SPADE Eq. (3))."""
    x = _f32(x)
    out = np.empty((g.B, g.Hd), dtype=np.float64)
    _load().orc_aggregation_score(_ptr(g.arr), _ptr(x), _ptr(out))
    return out


def choose_scheme(geoms, x):
    """Per (b, h): index of the candidate geometry (blocking scheme) with the largest AS,
    lowest index on equality (SPADE §3.2: the Selected Blocking Scheme has max AS)."""
    scores = np.stack([aggregation_score(g, x) for g in geoms])   # [n, B, Hd]
    return np.argmax(scores, axis=0).astype(np.int32), scores


def selected_pairs(g: Geometry, idx, cnt) -> int:
    """Selected valid (query, key) token pairs over all batch elements and heads."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    cnt = np.ascontiguousarray(cnt, dtype=np.int32)
    return int(_load().orc_selected_pairs(_ptr(g.arr), _ptr(idx), _ptr(cnt), idx.shape[-1]))


def forward(g: Geometry, q, k, v, mode: int, params, rows=None, estimator: int = 0):
    """The whole executor: summaries -> scores -> selection -> attention
    (estimator 0 = MEAN, 1 = DSA, 2 = DSA2)."""
    if estimator == 0:
        p = scores(g, centroids(g, q), centroids(g, k))
    else:
        p = scores_box(g, box_summaries(g, q), box_summaries(g, k), estimator)
    idx, cnt, tie = select(g, p, mode, params)
    o = attention(g, q, k, v, idx, cnt, rows=rows)
    return o, idx, cnt, tie, p
