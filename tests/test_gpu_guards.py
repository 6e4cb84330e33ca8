"""Guard bands around every buffer a call writes (the stand-in for a memory
checker, which is not available on the test machines).

Each output (O, the index lists and counts, the workspace) is carved from the
middle of a larger allocation whose 4 KB margins on both sides hold a byte
pattern; after the call the margins must be unchanged, so no kernel wrote
past the end (or before the start) of what it was given.  Covered: the fused
tensor-core forward (paired tiles, text blocks, both head dims), the SIMT
forward (fp32 and bf16 with 32-token blocks), the blocked four-call pipeline,
the grouped forward with mixed block shapes, and one full workload.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_permute_b200 as bsa
import synthetic
from parity import custom_workload

pytestmark = pytest.mark.gpu

GUARD = 4096
PATTERN = 0xA5


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    bsa.load()
    return torch.device("cuda", 0)


class Guarded:
    """A tensor of `shape`/`dtype` inside a byte buffer with patterned margins."""

    def __init__(self, shape, dtype, dev, fill=None):
        nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8, device=dev)
        self.n = nbytes
        body = self.raw[GUARD:GUARD + nbytes]
        self.t = body.view(dtype).view(shape)
        if fill is not None:
            self.t.fill_(fill)
        assert self.t.data_ptr() % 256 == 0

    def check(self, what):
        torch.cuda.synchronize()
        lo = self.raw[:GUARD]
        hi = self.raw[GUARD + self.n:]
        assert bool(torch.all(lo == PATTERN)), f"{what}: bytes written before the buffer"
        assert bool(torch.all(hi == PATTERN)), f"{what}: bytes written past the buffer"


def _forward_guarded(plan, w, qd, kd, vd, dev):
    L = bsa.load()
    i = plan.info
    kmax = plan.kmax_for(w.mode, w.params)
    _, wsz = plan.workspace_size(kmax)
    out = Guarded(plan.orig_shape, plan.dtype, dev)
    idx = Guarded((i.batch, i.heads, i.nb, kmax), torch.int32, dev)
    cnt = Guarded((i.batch, i.heads, i.nb), torch.int32, dev)
    ws = Guarded((wsz,), torch.uint8, dev)
    P = bsa._ptr
    bsa._check(L.bsa_forward(plan._h, P(qd), P(kd), P(vd), w.mode, bsa._params(w.params, i.heads),
                             kmax, P(out.t), P(idx.t), P(cnt.t), P(ws.t), wsz, None,
                             bsa._stream(dev)))
    plan.check_status()
    for b, nm in ((out, "out"), (idx, "idx"), (cnt, "cnt"), (ws, "workspace")):
        b.check(f"{w.name} {nm}")
    return out.t


CASES = {
    "hy_ragged_text": custom_workload("hy_ragged_text", 1, 6, 12, 20, 1, 8, 16, 3, 128, 130,
                                      "bf16", 0, 0.3),
    "d64_text": custom_workload("d64_text", 1, 5, 12, 20, 1, 8, 16, 3, 64, 200, "bf16", 0, 0.35),
    "wan_topp": custom_workload("wan_topp", 1, 9, 10, 20, 4, 4, 8, 3, 128, 0, "bf16", 1, 0.9),
    "tiny": synthetic.workload("tiny"),
    "simt_bf16_bs32": custom_workload("simt_bf16_bs32", 1, 5, 9, 12, 2, 4, 4, 2, 128, 40, "bf16",
                                      0, 0.3),
    "f32_bs128": custom_workload("f32_bs128", 1, 6, 12, 20, 1, 8, 16, 2, 64, 0, "f32", 0, 0.3),
}


@pytest.mark.parametrize("name", list(CASES))
def test_forward_writes_only_its_buffers(name, dev):
    w = CASES[name]
    q, k, v = synthetic.make_qkv(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    plan = bsa.plan_for(w, dev)
    got = _forward_guarded(plan, w, qd, kd, vd, dev)
    ref = plan.forward(qd, kd, vd, w.mode, w.params)
    plan.check_status()
    assert torch.equal(got, ref)


def test_blocked_pipeline_writes_only_its_buffers(dev):
    w = CASES["hy_ragged_text"]
    q, k, v = synthetic.make_qkv(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    plan = bsa.plan_for(w, dev)
    L = bsa.load()
    P = bsa._ptr
    i = plan.info
    S = bsa._stream(dev)
    blk = [Guarded(plan.blk_shape, plan.dtype, dev) for _ in range(4)]
    cent = [Guarded(plan.cent_shape, torch.float32, dev) for _ in range(2)]
    kmax = plan.kmax_for(w.mode, w.params)
    idx = Guarded((i.batch, i.heads, i.nb, kmax), torch.int32, dev)
    cnt = Guarded((i.batch, i.heads, i.nb), torch.int32, dev)
    sc = Guarded((i.batch, i.heads, i.nb, i.nb), torch.float32, dev)
    out = Guarded(plan.orig_shape, plan.dtype, dev)
    bsa._check(L.bsa_permute_qkv(plan._h, P(qd), P(kd), P(vd), P(blk[0].t), P(blk[1].t),
                                 P(blk[2].t), P(cent[0].t), P(cent[1].t), S))
    bsa._check(L.bsa_select_centroids(plan._h, P(cent[0].t), P(cent[1].t), w.mode,
                                      bsa._params(w.params, i.heads), kmax, P(idx.t), P(cnt.t),
                                      P(sc.t), S))
    bsa._check(L.bsa_attention(plan._h, P(blk[0].t), P(blk[1].t), P(blk[2].t), P(idx.t), P(cnt.t),
                               kmax, P(blk[3].t), None, S))
    bsa._check(L.bsa_unpermute(plan._h, P(blk[3].t), P(out.t), S))
    plan.check_status()
    for b, nm in zip(blk + cent + [idx, cnt, sc, out],
                     ["q_blk", "k_blk", "v_blk", "o_blk", "q_cent", "k_cent", "idx", "cnt",
                      "scores", "out"]):
        b.check(nm)
    # the same four calls on plain buffers give the same bytes
    qb, kb, vb, qc, kc = plan.permute_qkv(qd, kd, vd)
    idx2, cnt2 = plan.select_centroids(qc, kc, w.mode, w.params, kmax=kmax)
    ref = plan.unpermute(plan.attention(qb, kb, vb, idx2, cnt2))
    plan.check_status()
    assert torch.equal(out.t, ref)


def test_grouped_forward_writes_only_its_buffers(dev):
    w = custom_workload("grouped", 1, 8, 16, 32, 1, 8, 16, 4, 128, 0, "bf16", 0, 0.3)
    q, k, v = synthetic.make_qkv(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    shapes = [(1, 8, 16), (2, 8, 8), (4, 4, 8)]
    plans = [bsa.Plan(w.B, w.T, w.H, w.W, a, b, c, w.Hd, w.D, 0, torch.bfloat16, dev)
             for a, b, c in shapes]
    head_plan = [0, 1, 2, 1]
    L = bsa.load()
    P = bsa._ptr
    n = len(plans)
    kmaxes = [p.kmax_for(w.mode, w.params) for p in plans]
    lists = [(Guarded((1, w.Hd, p.info.nb, km), torch.int32, dev),
              Guarded((1, w.Hd, p.info.nb), torch.int32, dev, fill=0)) for p, km in zip(plans, kmaxes)]
    hs = (ctypes.c_void_p * n)(*[p._h.value for p in plans])
    km = (ctypes.c_int * n)(*kmaxes)
    z = ctypes.c_size_t()
    bsa._check(L.bsa_grouped_workspace_size(hs, n, km, None, ctypes.byref(z)))
    ws = Guarded((z.value,), torch.uint8, dev)
    out = Guarded(plans[0].orig_shape, torch.bfloat16, dev)
    hp = (ctypes.c_int32 * w.Hd)(*head_plan)
    ia = (ctypes.c_void_p * n)(*[l[0].t.data_ptr() for l in lists])
    ca = (ctypes.c_void_p * n)(*[l[1].t.data_ptr() for l in lists])
    bsa._check(L.bsa_forward_grouped(hs, n, hp, P(qd), P(kd), P(vd), w.mode,
                                     bsa._params(w.params, w.Hd), None, km, P(out.t), ia, ca,
                                     P(ws.t), z.value, None, bsa._stream(dev)))
    plans[0].check_status()
    for c, (ib, cb) in enumerate(lists):
        ib.check(f"idx of plan {c}")
        cb.check(f"cnt of plan {c}")
    ws.check("workspace")
    out.check("out")
    ref, _ = bsa.forward_grouped(plans, head_plan, qd, kd, vd, w.mode, w.params)
    plans[0].check_status()
    assert torch.equal(out.t, ref)


def test_full_workload_writes_only_its_buffers(dev):
    w = synthetic.workload("hunyuan")
    q, k, v = synthetic.make_qkv(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    plan = bsa.plan_for(w, dev)
    _forward_guarded(plan, w, qd, kd, vd, dev)
