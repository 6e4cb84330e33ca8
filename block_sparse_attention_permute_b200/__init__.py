"""Python binding of libbsa — 3D block-sparse attention for video DiTs on B200.

Argument marshalling only: every step runs in the CUDA kernels of
``libbsa.so`` (built in-tree by ``python -m block_sparse_attention_permute_b200.build``).
There is no fallback: importing works without the library, but every call
raises ``BsaError`` if ``libbsa.so`` is missing or the tensors are not on a
CUDA device.  PyTorch provides device memory and streams.

The calls mirror include/bsa.h (SPADE §3.3 "Head-wise Sparse Attention"):
``Plan.permute``/``unpermute`` (blocked layout), ``Plan.select`` (centroid
scores and Top-K / Top-P), ``Plan.attention`` (flash block-sparse attention)
and ``Plan.forward`` (all four in sequence).
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["Plan", "BsaError", "TOPK", "TOPP", "lib_path", "load"]

TOPK = 0
TOPP = 1
_DT = {torch.float32: 0, torch.bfloat16: 1}
_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libbsa.so")
_lib = None


class BsaError(RuntimeError):
    """A libbsa call returned an error status (or the library is unavailable)."""

    def __init__(self, status: int, msg: str):
        super().__init__(f"libbsa status {status}: {msg}")
        self.status = status


class PlanInfo(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("batch", "T", "H", "W", "bf", "br", "bc", "heads", "head_dim", "n_text", "dtype",
                 "Tp", "Hp", "Wp", "nbt", "nby", "nbx", "nb", "nb_text", "bs")] + \
               [("n_video", ctypes.c_longlong), ("n_tot", ctypes.c_longlong),
                ("npad_tot", ctypes.c_longlong), ("attn_path", ctypes.c_int)]


def lib_path() -> str:
    return _LIB_PATH


def load():
    """Load libbsa.so (raises BsaError if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise BsaError(-1, f"{_LIB_PATH} is missing; build it with "
                           "`python -m block_sparse_attention_permute_b200.build`")
    L = ctypes.CDLL(_LIB_PATH)
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.bsa_last_error_string.restype = ctypes.c_char_p
    L.bsa_version.restype = I
    sigs = {
        "bsa_plan_create": [ctypes.POINTER(P)] + [I] * 11,
        "bsa_plan_destroy": [P],
        "bsa_plan_get_info": [P, ctypes.POINTER(PlanInfo)],
        "bsa_kmax_for": [P, I, P, ctypes.POINTER(I)],
        "bsa_workspace_size": [P, I, ctypes.POINTER(Z), ctypes.POINTER(Z)],
        "bsa_permute": [P, P, P, P, P],
        "bsa_permute_qkv": [P] * 10,
        "bsa_unpermute": [P, P, P, P],
        "bsa_centroids": [P, P, P, P, P, P],
        "bsa_attention_orig": [P, P, P, P, P, P, I, P, P, P],
        "bsa_select": [P, P, P, I, P, I, P, P, P, P, Z, P],
        "bsa_select_centroids": [P, P, P, I, P, I, P, P, P, P],
        "bsa_attention": [P, P, P, P, P, P, I, P, P, P],
        "bsa_forward": [P, P, P, P, I, P, I, P, P, P, P, Z, P, P],
        "bsa_check_status": [P, P],
        "bsa_plan_set_watchdog": [P, ctypes.c_longlong, I],
        "bsa_forward_timed": [P, P, P, P, I, P, I, P, P, P, P, Z, P, P, ctypes.POINTER(Timings)],
        "bsa_sics": [P, P, P, P],
        "bsa_kmax_for_union": [P, I, P, P, ctypes.POINTER(I)],
        "bsa_union_workspace_size": [P, I, P, ctypes.POINTER(Z), ctypes.POINTER(Z)],
        "bsa_select_union": [P, P, P, I, P, P, P, I, P, P, P, P, Z, P],
        "bsa_forward_union": [P, P, P, P, I, P, P, I, P, P, P, P, Z, P, P],
        "bsa_box_summaries": [P, P, P, P, P, P],
        "bsa_select_box": [P, I, P, P, I, P, P, P, I, P, P, P, P, Z, P],
        "bsa_estimator_workspace_size": [P, I, I, P, ctypes.POINTER(Z)],
        "bsa_forward_estimator": [P, P, P, P, I, I, P, P, I, P, P, P, P, Z, P, P],
        "bsa_grouped_workspace_size": [P, I, P, P, ctypes.POINTER(Z)],
        "bsa_pair_workspace_size": [P, I, ctypes.POINTER(Z)],
        "bsa_pair_tiles": [P, P, P, I, P, Z, P],
        "bsa_attention_paired": [P, P, P, P, P, P, I, P, Z, P, P, P],
        "bsa_forward_grouped": [P, I, P, P, P, P, I, P, P, P, P, P, P, P, Z, P, P],
        "bsa_aggregation_scores": [P, I, P, P, P, P, P],
    }
    for name, args in sigs.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = I
    _lib = L
    return L


def _check(status: int):
    if status != 0:
        raise BsaError(status, load().bsa_last_error_string().decode())


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _params(p, heads):
    if isinstance(p, (int, float)):
        p = [float(p)] * heads
    arr = (ctypes.c_double * heads)(*[float(x) for x in p])
    if len(p) != heads:
        raise BsaError(1, f"expected {heads} per-head parameters, got {len(p)}")
    return arr


class Timings(ctypes.Structure):
    """bsa_timings_t: device milliseconds of the phases of one bsa_forward call."""
    _fields_ = [(n, ctypes.c_float) for n in ("summaries_ms", "select_ms", "pairing_ms",
                                               "attention_ms", "unpermute_ms", "total_ms")]

    def as_dict(self):
        return {n: float(getattr(self, n)) for n, _ in self._fields_}


class MaskUnion(ctypes.Structure):
    """bsa_mask_union_t: window (left, right) in blocks, sink tokens, intra rule."""
    _fields_ = [("window_left", ctypes.c_int), ("window_right", ctypes.c_int),
                ("sink_tokens", ctypes.c_longlong), ("intra_mode", ctypes.c_int),
                ("intra_param", ctypes.POINTER(ctypes.c_double))]


def mask_union(heads, window=(-1, -1), sink_tokens=0, intra_mode=0, intra_params=None):
    """A MaskUnion (kept alive with its per-head intra array)."""
    u = MaskUnion(int(window[0]), int(window[1]), int(sink_tokens), int(intra_mode), None)
    if intra_params is not None:
        arr = _params(intra_params, heads) if not isinstance(intra_params, (int, float)) \
            else _params([float(intra_params)] * heads, heads)
        u._keep = arr
        u.intra_param = ctypes.cast(arr, ctypes.POINTER(ctypes.c_double))
    return u


class Plan:
    """One attention problem: grid (T,H,W), block (bf,br,bc), heads, head_dim, text tokens."""

    def __init__(self, batch, T, H, W, bf, br, bc, heads, head_dim, n_text=0,
                 dtype=torch.bfloat16, device=None):
        L = load()
        if dtype not in _DT:
            raise BsaError(1, f"dtype must be float32 or bfloat16, got {dtype}")
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        if self.device.type != "cuda":
            raise BsaError(1, "libbsa runs on CUDA devices only")
        self.dtype = dtype
        self._h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            _check(L.bsa_plan_create(ctypes.byref(self._h), batch, T, H, W, bf, br, bc, heads,
                                     head_dim, n_text, _DT[dtype]))
        info = PlanInfo()
        _check(L.bsa_plan_get_info(self._h, ctypes.byref(info)))
        self.info = info

    def __del__(self):
        h = getattr(self, "_h", None)
        if h and _lib is not None:
            try:
                with torch.cuda.device(self.device):
                    _lib.bsa_plan_destroy(h)
            except Exception:
                pass
            self._h = None

    # ---------------------------------------------------------------- sizes
    @property
    def orig_shape(self):
        i = self.info
        return (i.batch, i.n_tot, i.heads, i.head_dim)

    @property
    def blk_shape(self):
        i = self.info
        return (i.batch, i.heads, i.npad_tot, i.head_dim)

    @property
    def cent_shape(self):
        i = self.info
        return (i.batch, i.heads, i.nb, i.head_dim)

    def kmax_for(self, mode, params) -> int:
        k = ctypes.c_int()
        _check(load().bsa_kmax_for(self._h, mode, _params(params, self.info.heads), ctypes.byref(k)))
        return k.value

    def workspace_size(self, kmax):
        a, b = ctypes.c_size_t(), ctypes.c_size_t()
        _check(load().bsa_workspace_size(self._h, kmax, ctypes.byref(a), ctypes.byref(b)))
        return a.value, b.value

    def _new(self, shape, dtype=None):
        return torch.empty(shape, dtype=dtype or self.dtype, device=self.device)

    def _check_tensor(self, t, shape, dtype=None, name="tensor"):
        dtype = dtype or self.dtype
        if not isinstance(t, torch.Tensor) or t.device != self.device:
            raise BsaError(1, f"{name} must be a tensor on {self.device}")
        if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
            raise BsaError(1, f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)}, "
                              f"got {t.dtype} {tuple(t.shape)}")

    # ---------------------------------------------------------------- calls
    def permute(self, x, centroids=False, out=None):
        self._check_tensor(x, self.orig_shape, name="x")
        out = self._new(self.blk_shape) if out is None else out
        cent = self._new(self.cent_shape, torch.float32) if centroids else None
        _check(load().bsa_permute(self._h, _ptr(x), _ptr(out), _ptr(cent), _stream(self.device)))
        return (out, cent) if centroids else out

    def permute_qkv(self, q, k, v):
        for t, n in ((q, "q"), (k, "k"), (v, "v")):
            self._check_tensor(t, self.orig_shape, name=n)
        qb, kb, vb = (self._new(self.blk_shape) for _ in range(3))
        qc, kc = (self._new(self.cent_shape, torch.float32) for _ in range(2))
        _check(load().bsa_permute_qkv(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(qb), _ptr(kb),
                                      _ptr(vb), _ptr(qc), _ptr(kc), _stream(self.device)))
        return qb, kb, vb, qc, kc

    def centroids(self, q, k):
        """Q and K block centroids straight from the original layout (bsa_centroids)."""
        self._check_tensor(q, self.orig_shape, name="q")
        self._check_tensor(k, self.orig_shape, name="k")
        qc, kc = (self._new(self.cent_shape, torch.float32) for _ in range(2))
        _check(load().bsa_centroids(self._h, _ptr(q), _ptr(k), _ptr(qc), _ptr(kc),
                                    _stream(self.device)))
        return qc, kc

    def sics(self, x, out=None):
        """Sum of intra-block cosine similarities per video block, [B,Hd,nb] fp32 (bsa_sics)."""
        self._check_tensor(x, self.orig_shape, name="x")
        i = self.info
        out = self._new((i.batch, i.heads, i.nb), torch.float32) if out is None else out
        self._check_tensor(out, (i.batch, i.heads, i.nb), torch.float32, "out")
        _check(load().bsa_sics(self._h, _ptr(x), _ptr(out), _stream(self.device)))
        return out

    def pair_tiles(self, idx, cnt):
        """bsa_pair_tiles: the pairing workspace (a uint8 tensor) for these lists."""
        z = ctypes.c_size_t()
        kmax = idx.shape[-1]
        _check(load().bsa_pair_workspace_size(self._h, kmax, ctypes.byref(z)))
        ws = self._new((max(z.value, 1),), torch.uint8)
        _check(load().bsa_pair_tiles(self._h, _ptr(idx), _ptr(cnt), kmax, _ptr(ws), ws.numel(),
                                     _stream(self.device)))
        return ws

    def attention_paired(self, q, k, v, idx, cnt, ws, out=None, dev_status=None):
        """bsa_attention_paired on the schedule of pair_tiles(idx, cnt)."""
        for t, n in ((q, "q"), (k, "k"), (v, "v")):
            self._check_tensor(t, self.orig_shape, name=n)
        out = self._new(self.orig_shape) if out is None else out
        _check(load().bsa_attention_paired(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(cnt),
                                           idx.shape[-1], _ptr(ws), ws.numel(), _ptr(out),
                                           _ptr(dev_status), _stream(self.device)))
        return out

    def attention_orig(self, q, k, v, idx, cnt, out=None, dev_status=None):
        """Attention on the original layout; the layout transform is fused (bsa_attention_orig)."""
        for t, n in ((q, "q"), (k, "k"), (v, "v")):
            self._check_tensor(t, self.orig_shape, name=n)
        i = self.info
        kmax = idx.shape[-1]
        self._check_tensor(idx, (i.batch, i.heads, i.nb, kmax), torch.int32, "idx")
        self._check_tensor(cnt, (i.batch, i.heads, i.nb), torch.int32, "cnt")
        out = self._new(self.orig_shape) if out is None else out
        _check(load().bsa_attention_orig(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(cnt),
                                         kmax, _ptr(out), _ptr(dev_status), _stream(self.device)))
        return out

    def unpermute(self, o_blk, out=None):
        self._check_tensor(o_blk, self.blk_shape, name="o_blk")
        out = self._new(self.orig_shape) if out is None else out
        _check(load().bsa_unpermute(self._h, _ptr(o_blk), _ptr(out), _stream(self.device)))
        return out

    def _lists(self, kmax):
        i = self.info
        return (self._new((i.batch, i.heads, i.nb, kmax), torch.int32),
                self._new((i.batch, i.heads, i.nb), torch.int32))

    def select(self, q_blk, k_blk, mode, params, kmax=None, scores=False):
        self._check_tensor(q_blk, self.blk_shape, name="q_blk")
        self._check_tensor(k_blk, self.blk_shape, name="k_blk")
        kmax = self.kmax_for(mode, params) if kmax is None else kmax
        idx, cnt = self._lists(kmax)
        i = self.info
        sc = self._new((i.batch, i.heads, i.nb, i.nb), torch.float32) if scores else None
        ws = self._new((max(self.workspace_size(kmax)[0], 1),), torch.uint8)
        _check(load().bsa_select(self._h, _ptr(q_blk), _ptr(k_blk), mode,
                                 _params(params, i.heads), kmax, _ptr(idx), _ptr(cnt), _ptr(sc),
                                 _ptr(ws), ws.numel(), _stream(self.device)))
        return (idx, cnt, sc) if scores else (idx, cnt)

    def select_centroids(self, q_cent, k_cent, mode, params, kmax=None, scores=False):
        self._check_tensor(q_cent, self.cent_shape, torch.float32, "q_cent")
        self._check_tensor(k_cent, self.cent_shape, torch.float32, "k_cent")
        kmax = self.kmax_for(mode, params) if kmax is None else kmax
        idx, cnt = self._lists(kmax)
        i = self.info
        sc = self._new((i.batch, i.heads, i.nb, i.nb), torch.float32) if scores else None
        _check(load().bsa_select_centroids(self._h, _ptr(q_cent), _ptr(k_cent), mode,
                                           _params(params, i.heads), kmax, _ptr(idx), _ptr(cnt),
                                           _ptr(sc), _stream(self.device)))
        return (idx, cnt, sc) if scores else (idx, cnt)

    def attention(self, q_blk, k_blk, v_blk, idx, cnt, out=None, dev_status=None):
        for t, n in ((q_blk, "q_blk"), (k_blk, "k_blk"), (v_blk, "v_blk")):
            self._check_tensor(t, self.blk_shape, name=n)
        i = self.info
        kmax = idx.shape[-1]
        self._check_tensor(idx, (i.batch, i.heads, i.nb, kmax), torch.int32, "idx")
        self._check_tensor(cnt, (i.batch, i.heads, i.nb), torch.int32, "cnt")
        out = self._new(self.blk_shape) if out is None else out
        _check(load().bsa_attention(self._h, _ptr(q_blk), _ptr(k_blk), _ptr(v_blk), _ptr(idx),
                                    _ptr(cnt), kmax, _ptr(out), _ptr(dev_status),
                                    _stream(self.device)))
        return out

    def forward(self, q, k, v, mode, params, kmax=None, out=None, workspace=None,
                return_lists=False):
        for t, n in ((q, "q"), (k, "k"), (v, "v")):
            self._check_tensor(t, self.orig_shape, name=n)
        kmax = self.kmax_for(mode, params) if kmax is None else kmax
        out = self._new(self.orig_shape) if out is None else out
        need = self.workspace_size(kmax)[1]
        ws = self._new((need,), torch.uint8) if workspace is None else workspace
        idx, cnt = self._lists(kmax) if return_lists else (None, None)
        _check(load().bsa_forward(self._h, _ptr(q), _ptr(k), _ptr(v), mode,
                                  _params(params, self.info.heads), kmax, _ptr(out), _ptr(idx),
                                  _ptr(cnt), _ptr(ws), ws.numel(), None, _stream(self.device)))
        return (out, idx, cnt) if return_lists else out

    def forward_timed(self, q, k, v, mode, params, kmax=None, out=None, workspace=None):
        """bsa_forward_timed: the forward plus the device time of each phase
        (synchronises); returns (out, dict of milliseconds)."""
        for t, n in ((q, "q"), (k, "k"), (v, "v")):
            self._check_tensor(t, self.orig_shape, name=n)
        kmax = self.kmax_for(mode, params) if kmax is None else kmax
        out = self._new(self.orig_shape) if out is None else out
        need = self.workspace_size(kmax)[1]
        ws = self._new((need,), torch.uint8) if workspace is None else workspace
        t = Timings()
        _check(load().bsa_forward_timed(self._h, _ptr(q), _ptr(k), _ptr(v), mode,
                                        _params(params, self.info.heads), kmax, _ptr(out), None,
                                        None, _ptr(ws), ws.numel(), None, _stream(self.device),
                                        ctypes.byref(t)))
        return out, t.as_dict()

    # --------------------------------------------------------- mask union
    def kmax_for_union(self, mode, params, union) -> int:
        k = ctypes.c_int()
        _check(load().bsa_kmax_for_union(self._h, mode, _params(params, self.info.heads),
                                         ctypes.byref(union) if union is not None else None,
                                         ctypes.byref(k)))
        return k.value

    def union_workspace_size(self, kmax, union):
        a, b = ctypes.c_size_t(), ctypes.c_size_t()
        _check(load().bsa_union_workspace_size(self._h, kmax,
                                               ctypes.byref(union) if union is not None else None,
                                               ctypes.byref(a), ctypes.byref(b)))
        return a.value, b.value

    def select_union(self, q_cent, k_cent, mode, params, union, intra_scores=None, kmax=None,
                     scores=False):
        """bsa_select_union: Top-K/Top-P lists united with window, sink and intra blocks."""
        i = self.info
        self._check_tensor(q_cent, self.cent_shape, torch.float32, "q_cent")
        self._check_tensor(k_cent, self.cent_shape, torch.float32, "k_cent")
        if intra_scores is not None:
            self._check_tensor(intra_scores, (i.batch, i.heads, i.nb), torch.float32, "intra_scores")
        kmax = kmax or self.kmax_for_union(mode, params, union)
        idx, cnt = self._lists(kmax)
        sc = self._new((i.batch, i.heads, i.nb, i.nb), torch.float32) if scores else None
        sel_ws, _ = self.union_workspace_size(kmax, union)
        ws = self._new((max(sel_ws, 1),), torch.uint8)
        _check(load().bsa_select_union(self._h, _ptr(q_cent), _ptr(k_cent), mode,
                                       _params(params, i.heads), ctypes.byref(union),
                                       _ptr(intra_scores), kmax, _ptr(idx), _ptr(cnt), _ptr(sc),
                                       _ptr(ws), ws.numel(), _stream(self.device)))
        return (idx, cnt, sc) if scores else (idx, cnt)

    def forward_union(self, q, k, v, mode, params, union, kmax=None, out=None, workspace=None,
                      dev_status=None):
        """bsa_forward_union: the whole path with the mask union; returns (o, idx, cnt)."""
        for t, n in ((q, "q"), (k, "k"), (v, "v")):
            self._check_tensor(t, self.orig_shape, name=n)
        kmax = kmax or self.kmax_for_union(mode, params, union)
        idx, cnt = self._lists(kmax)
        out = self._new(self.orig_shape) if out is None else out
        _, fwd_ws = self.union_workspace_size(kmax, union)
        ws = workspace if workspace is not None else self._new((max(fwd_ws, 1),), torch.uint8)
        _check(load().bsa_forward_union(self._h, _ptr(q), _ptr(k), _ptr(v), mode,
                                        _params(params, self.info.heads),
                                        ctypes.byref(union) if union is not None else None, kmax,
                                        _ptr(out), _ptr(idx), _ptr(cnt), _ptr(ws), ws.numel(),
                                        _ptr(dev_status), _stream(self.device)))
        return out, idx, cnt

    # ---------------------------------------------------- box estimators
    @property
    def box_shape(self):
        i = self.info
        return (i.batch, i.heads, i.nb, i.head_dim, 2)

    def box_summaries(self, q, k):
        """(max, min) per video block and dimension of Q and K (bsa_box_summaries)."""
        self._check_tensor(q, self.orig_shape, name="q")
        self._check_tensor(k, self.orig_shape, name="k")
        qb, kb = (self._new(self.box_shape, torch.float32) for _ in range(2))
        _check(load().bsa_box_summaries(self._h, _ptr(q), _ptr(k), _ptr(qb), _ptr(kb),
                                        _stream(self.device)))
        return qb, kb

    def select_box(self, est, q_box, k_box, mode, params, union=None, intra_scores=None,
                   kmax=None, scores=False):
        """bsa_select_box: lists from the DSA (est 1) or DSA2 (est 2) estimator."""
        i = self.info
        self._check_tensor(q_box, self.box_shape, torch.float32, "q_box")
        self._check_tensor(k_box, self.box_shape, torch.float32, "k_box")
        kmax = kmax or self.kmax_for_union(mode, params, union)
        idx, cnt = self._lists(kmax)
        sc = self._new((i.batch, i.heads, i.nb, i.nb), torch.float32) if scores else None
        sel_ws = self.union_workspace_size(kmax, union)[0] if union is not None else 0
        ws = self._new((max(sel_ws, 1),), torch.uint8)
        _check(load().bsa_select_box(self._h, est, _ptr(q_box), _ptr(k_box), mode,
                                     _params(params, i.heads),
                                     ctypes.byref(union) if union is not None else None,
                                     _ptr(intra_scores), kmax, _ptr(idx), _ptr(cnt), _ptr(sc),
                                     _ptr(ws), ws.numel(), _stream(self.device)))
        return (idx, cnt, sc) if scores else (idx, cnt)

    def forward_estimator(self, q, k, v, est, mode, params, union=None, kmax=None, out=None,
                          dev_status=None):
        """bsa_forward_estimator: the whole path with MEAN / DSA / DSA2; returns (o, idx, cnt)."""
        for t, n in ((q, "q"), (k, "k"), (v, "v")):
            self._check_tensor(t, self.orig_shape, name=n)
        kmax = kmax or self.kmax_for_union(mode, params, union)
        idx, cnt = self._lists(kmax)
        out = self._new(self.orig_shape) if out is None else out
        z = ctypes.c_size_t()
        u = ctypes.byref(union) if union is not None else None
        _check(load().bsa_estimator_workspace_size(self._h, est, kmax, u, ctypes.byref(z)))
        ws = self._new((max(z.value, 1),), torch.uint8)
        _check(load().bsa_forward_estimator(self._h, _ptr(q), _ptr(k), _ptr(v), est, mode,
                                            _params(params, self.info.heads), u, kmax, _ptr(out),
                                            _ptr(idx), _ptr(cnt), _ptr(ws), ws.numel(),
                                            _ptr(dev_status), _stream(self.device)))
        return out, idx, cnt

    def check_status(self):
        """Synchronise the current stream and raise if a kernel recorded an error."""
        _check(load().bsa_check_status(self._h, _stream(self.device)))

    def set_watchdog(self, wait_limit_cycles=0, withhold_copy=0):
        """Bound of the attention kernel's in-kernel waits (0 = default, about a
        second) and the timeout path's test hook (bsa_plan_set_watchdog)."""
        _check(load().bsa_plan_set_watchdog(self._h, int(wait_limit_cycles), int(withhold_copy)))


def aggregation_scores(plans, x):
    """Aggregation evaluation over candidate blocking schemes (bsa_aggregation_scores).

    plans: 1..8 Plans that differ only in block shape.  Returns (sics, as_, choice):
    sics[c] [B,Hd,nb_c] fp32, as_ [n,B,Hd] float64, choice [B,Hd] int32.
    """
    plans = list(plans)
    n = len(plans)
    p0 = plans[0]
    p0._check_tensor(x, p0.orig_shape, name="x")
    i = p0.info
    sics = [p._new((i.batch, i.heads, p.info.nb), torch.float32) for p in plans]
    as_ = p0._new((n, i.batch, i.heads), torch.float64)
    choice = p0._new((i.batch, i.heads), torch.int32)
    handles = (ctypes.c_void_p * n)(*[p._h.value for p in plans])
    outs = (ctypes.c_void_p * n)(*[t.data_ptr() for t in sics])
    _check(load().bsa_aggregation_scores(handles, n, _ptr(x), outs, _ptr(as_), _ptr(choice),
                                         _stream(p0.device)))
    return sics, as_, choice


def forward_grouped(plans, head_plan, q, k, v, mode, params, union=None, kmax=None, out=None):
    """bsa_forward_grouped: each (b, h) served by plans[head_plan[b*Hd + h]].

    head_plan: sequence or int tensor of B*Hd plan indices (host values).
    Returns (o, lists) with lists[c] = (idx, cnt) of plan c (only its heads written).
    """
    plans = list(plans)
    n = len(plans)
    p0 = plans[0]
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        p0._check_tensor(t, p0.orig_shape, name=nm)
    hp = [int(x) for x in (head_plan.flatten().tolist() if isinstance(head_plan, torch.Tensor)
                           else head_plan)]
    hp_arr = (ctypes.c_int32 * len(hp))(*hp)
    kmaxes = kmax or [p.kmax_for_union(mode, params, union) for p in plans]
    km_arr = (ctypes.c_int * n)(*kmaxes)
    lists = [p._lists(km) for p, km in zip(plans, kmaxes)]
    for idx, cnt in lists:
        cnt.zero_()
    idx_arr = (ctypes.c_void_p * n)(*[l[0].data_ptr() for l in lists])
    cnt_arr = (ctypes.c_void_p * n)(*[l[1].data_ptr() for l in lists])
    handles = (ctypes.c_void_p * n)(*[p._h.value for p in plans])
    u = ctypes.byref(union) if union is not None else None
    z = ctypes.c_size_t()
    _check(load().bsa_grouped_workspace_size(handles, n, km_arr, u, ctypes.byref(z)))
    ws = p0._new((max(z.value, 1),), torch.uint8)
    out = p0._new(p0.orig_shape) if out is None else out
    _check(load().bsa_forward_grouped(handles, n, hp_arr, _ptr(q), _ptr(k), _ptr(v), mode,
                                      _params(params, p0.info.heads), u, km_arr, _ptr(out),
                                      idx_arr, cnt_arr, _ptr(ws), ws.numel(), None,
                                      _stream(p0.device)))
    return out, lists


def plan_for(w, device=None) -> Plan:
    """A Plan for a synthetic Workload-like object (attributes B,T,H,W,bf,br,bc,Hd,D,n_text,dtype)."""
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    return Plan(w.B, w.T, w.H, w.W, w.bf, w.br, w.bc, w.Hd, w.D, w.n_text, dt, device)
