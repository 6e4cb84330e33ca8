"""Benchmark of the block-sparse attention executor on one node.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one bsa_forward over one batch of synthetic input already resident
in HBM: on the tensor-core plans that is centroids -> selection -> attention
with the layout transform (permute) and its inverse fused into the
attention's TMA loads and stores.  Default workload: the
HunyuanVideo 720p 61-frame shape (16x45x80 latent grid + 256 text tokens,
24 heads, head_dim 128, bf16, 1x8x16 blocks, density 0.15).

Printed: one JSON line on rank 0.  value = effective TFLOP/s of the whole job
= 4 x selected valid (query, key) pairs x head_dim (summed over heads and
ranks) / max-over-ranks device time.  Per-phase times come from a second loop
that issues bsa_forward's calls separately, with CUDA events on the launching
stream; a third loop times the unfused pipeline (bsa_permute_qkv,
selection, bsa_attention on the blocked layout, bsa_unpermute) for reference.  Under torchrun every rank runs its own replica of the
workload (weak scaling, no collective on the data path).

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

METRIC = "sparse-attn ms/call + effective TFLOP/s (% bf16 TC peak), 57.6k-token shape"
L2_BYTES = 126 * 1024 * 1024


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def peaks():
    """bf16 tensor peaks and HBM bandwidth: (burst TFLOP/s, sustained TFLOP/s,
    HBM GB/s, source).  The burst figure is cuBLAS timed alone at full clock,
    the sustained one a seconds-long back-to-back loop under the power cap.
    Every loop this bench times is event-timed and well under a second, so
    fractions are quoted against the burst peak."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        burst = d.get("bf16_tflops")
        return burst, d.get("bf16_tflops_sustained", burst), d.get("hbm_gbs"), "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


def attn_source_sha() -> str:
    """Hash of the attention kernel's code: its sources with // comments and
    whitespace removed (none of them has // inside a string literal), so that
    an edit to a comment does not void a profile taken on the same code."""
    h = hashlib.sha256()
    for name in ("attn.cu", "common.cuh", "kernels.cuh"):
        with open(os.path.join(ROOT, "block_sparse_attention_permute_b200", "csrc", name)) as f:
            for line in f:
                code = "".join(line.split("//", 1)[0].split())
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per attention launch of `workload`, from the ncu figures kept
    in profiles/attn_traffic.json, if they were captured on the current
    attention source (else None)."""
    path = os.path.join(ROOT, "profiles", "attn_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(workload)
    if not rec or rec.get("attn_source_sha") != attn_source_sha():
        return None
    return float(rec["dram_bytes_per_launch"])


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.5)            # let the sampler start before the timed region
        except (FileNotFoundError, OSError):
            self.proc = None
        self.t_start = self.t_end = None
        return self

    def mark_start(self):
        self.t_start = time.time()

    def mark_end(self):
        self.t_end = time.time()

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        """Median SM clock and throttle reasons over the samples taken inside the
        timed region (timestamps between mark_start and mark_end)."""
        from datetime import datetime
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                clk, clk_max = float(parts[2]), float(parts[3])
            except ValueError:
                continue
            if self.t_start is not None and not (self.t_start <= ts <= (self.t_end or ts)):
                continue
            sm.append(clk)
            mx = clk_max
            for n, v in zip(names, parts[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def reduce_max(vals, device="cpu"):
    """Element-wise max of per-rank values over all ranks (identity on one rank)."""
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_tflops(world: int, flops_per_rank_step: float, step_ms: float) -> float:
    """Whole-job throughput: every rank processes one replica per step."""
    return world * flops_per_rank_step / (step_ms * 1e-3) / 1e12


def effective_pairs(plan, idx, cnt) -> int:
    """Selected valid (query, key) token pairs, summed over batch and heads."""
    i = plan.info
    nbk = i.nb + i.nb_text
    valid = np.zeros(nbk, dtype=np.int64)
    for j in range(i.nb):
        tb, yb, xb = j // (i.nby * i.nbx), (j // i.nbx) % i.nby, j % i.nbx
        valid[j] = (min(i.bf, i.T - tb * i.bf) * min(i.br, i.H - yb * i.br)
                    * min(i.bc, i.W - xb * i.bc))
    for t in range(i.nb_text):
        valid[i.nb + t] = min(i.bs, i.n_text - t * i.bs)
    vd = torch.from_numpy(valid).to(idx.device)
    kmax = idx.shape[-1]
    ar = torch.arange(kmax, device=idx.device)
    sel = (ar[None, None, None, :] < cnt[..., None])
    keys = torch.where(sel, vd[idx.clamp(0, nbk - 1).long()], torch.zeros_like(idx, dtype=torch.long))
    keys_per_row = keys.sum(-1)                                  # [B,Hd,nb]
    video = int((keys_per_row * vd[:i.nb][None, None, :]).sum())
    text = int(valid[i.nb:].sum()) * i.n_tot * i.batch * i.heads
    return video + text


# Mask union timed beside the plain step: a window of one block on each side,
# the blocks of the first latent frame as attention sink, and the 2% of key
# blocks with the largest SICS (intra Top-K).
UNION = dict(window=(1, 1), sink_frames=1, intra_mode=0, intra_density=0.02)


def time_union_forward(bsa, w, plan, qd, kd, vd, out, dev, args, barrier):
    """CUDA-event timing of bsa_forward_union over --steps steps."""
    L = bsa.load()
    u = bsa.mask_union(w.Hd, window=UNION["window"], sink_tokens=UNION["sink_frames"] * w.H * w.W,
                       intra_mode=UNION["intra_mode"], intra_params=UNION["intra_density"])
    kmax = plan.kmax_for_union(w.mode, w.params, u)
    _, fwd_ws = plan.union_workspace_size(kmax, u)
    ws = torch.empty(fwd_ws, dtype=torch.uint8, device=dev)
    idx = torch.empty((w.B, w.Hd, plan.info.nb, kmax), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.B, w.Hd, plan.info.nb), dtype=torch.int32, device=dev)
    params = bsa._params(w.params, w.Hd)
    P = bsa._ptr
    stream = torch.cuda.current_stream(dev)

    def step():
        bsa._check(L.bsa_forward_union(plan._h, P(qd), P(kd), P(vd), w.mode, params, ctypes.byref(u),
                                       kmax, P(out), P(idx), P(cnt), P(ws), ws.numel(), None,
                                       bsa._stream(dev)))

    for _ in range(args.warmup):
        step()
    barrier()
    plan.check_status()
    pairs = effective_pairs(plan, idx, cnt)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    barrier()
    plan.check_status()
    ms = e0.elapsed_time(e1) / args.steps
    flops = 4.0 * pairs * w.D
    return {"window": list(UNION["window"]), "sink_tokens": UNION["sink_frames"] * w.H * w.W,
            "intra": f"top-k density {UNION['intra_density']} of K-block SICS",
            "ms_per_step": round(ms, 4), "effective_tflop_per_step": round(flops / 1e12, 4),
            "tflops": round(flops / (ms * 1e-3) / 1e12, 2),
            "mean_list_len": round(float(cnt.float().mean()), 2), "selected_pairs": pairs}


def time_estimators(bsa, w, plan, qd, kd, vd, out, dev, args, barrier):
    """Per box estimator (DSA, DSA2): CUDA-event times of the whole
    bsa_forward_estimator step and of its summarizer and selection phases."""
    L = bsa.load()
    P = bsa._ptr
    params = bsa._params(w.params, w.Hd)
    kmax = plan.kmax_for(w.mode, w.params)
    idx = torch.empty((w.B, w.Hd, plan.info.nb, kmax), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.B, w.Hd, plan.info.nb), dtype=torch.int32, device=dev)
    qb, kb = (torch.empty(plan.box_shape, dtype=torch.float32, device=dev) for _ in range(2))
    stream = torch.cuda.current_stream(dev)
    res = {}
    for name, est in (("dsa", 1), ("dsa2", 2)):
        z = ctypes.c_size_t()
        bsa._check(L.bsa_estimator_workspace_size(plan._h, est, kmax, None, ctypes.byref(z)))
        ws = torch.empty(z.value, dtype=torch.uint8, device=dev)
        calls = [
            lambda: L.bsa_box_summaries(plan._h, P(qd), P(kd), P(qb), P(kb), bsa._stream(dev)),
            lambda: L.bsa_select_box(plan._h, est, P(qb), P(kb), w.mode, params, None, None, kmax,
                                     P(idx), P(cnt), None, None, 0, bsa._stream(dev)),
            lambda: L.bsa_forward_estimator(plan._h, P(qd), P(kd), P(vd), est, w.mode, params, None,
                                            kmax, P(out), P(idx), P(cnt), P(ws), ws.numel(), None,
                                            bsa._stream(dev)),
        ]
        times = []
        for c in calls:
            for _ in range(args.warmup):
                bsa._check(c())
            barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                bsa._check(c())
            e1.record(stream)
            barrier()
            times.append(e0.elapsed_time(e1) / args.steps)
        plan.check_status()
        pairs = effective_pairs(plan, idx, cnt)
        res[name] = {"summaries_ms": round(times[0], 4), "select_ms": round(times[1], 4),
                     "ms_per_step": round(times[2], 4),
                     "tflops": round(4.0 * pairs * w.D / (times[2] * 1e-3) / 1e12, 2)}
        del ws
    return res


def time_grouped_forward(bsa, w, qd, kd, vd, dev, args, barrier):
    """Per-head blocking schemes: the aggregation-score choice among three
    candidate block shapes (computed once), then CUDA-event timing of
    bsa_forward_grouped over --steps steps."""
    shapes = [(w.bf, w.br, w.bc)] + [s for s in CANDIDATE_SHAPES if s != (w.bf, w.br, w.bc)][:2]
    plans = [bsa.Plan(w.B, w.T, w.H, w.W, a, b, c, w.Hd, w.D, w.n_text, qd.dtype, dev)
             for a, b, c in shapes]
    if any(p.info.attn_path != 1 for p in plans):
        return {"skipped": "grouped forward needs tensor-core plans"}
    _, _, choice = bsa.aggregation_scores(plans, qd)
    head_plan = choice.cpu().flatten().tolist()
    L = bsa.load()
    n = len(plans)
    kmaxes = [p.kmax_for(w.mode, w.params) for p in plans]
    lists = [p._lists(km) for p, km in zip(plans, kmaxes)]
    for _, cnt in lists:
        cnt.zero_()
    hp = (ctypes.c_int32 * len(head_plan))(*head_plan)
    km = (ctypes.c_int * n)(*kmaxes)
    hs = (ctypes.c_void_p * n)(*[p._h.value for p in plans])
    ia = (ctypes.c_void_p * n)(*[l[0].data_ptr() for l in lists])
    ca = (ctypes.c_void_p * n)(*[l[1].data_ptr() for l in lists])
    z = ctypes.c_size_t()
    bsa._check(L.bsa_grouped_workspace_size(hs, n, km, None, ctypes.byref(z)))
    ws = torch.empty(z.value, dtype=torch.uint8, device=dev)
    out = torch.empty_like(qd)
    params = bsa._params(w.params, w.Hd)
    P = bsa._ptr
    stream = torch.cuda.current_stream(dev)

    def step():
        bsa._check(L.bsa_forward_grouped(hs, n, hp, P(qd), P(kd), P(vd), w.mode, params, None, km,
                                         P(out), ia, ca, P(ws), ws.numel(), None, bsa._stream(dev)))

    for _ in range(args.warmup):
        step()
    barrier()
    plans[0].check_status()
    i0 = plans[0].info
    text = sum(min(i0.bs, i0.n_text - t * i0.bs) for t in range(i0.nb_text)) * i0.n_tot * w.B * w.Hd
    pairs = text + sum(effective_pairs(p, idx, cnt) - text for p, (idx, cnt) in zip(plans, lists))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    barrier()
    ms = e0.elapsed_time(e1) / args.steps
    return {"candidates": [f"{a}x{b}x{c}" for a, b, c in shapes],
            "heads_per_scheme": [head_plan.count(c) for c in range(n)],
            "ms_per_step": round(ms, 4), "effective_tflop_per_step": round(4.0 * pairs * w.D / 1e12, 4),
            "tflops": round(4.0 * pairs * w.D / (ms * 1e-3) / 1e12, 2), "selected_pairs": pairs}


CANDIDATE_SHAPES = [(1, 8, 16), (4, 4, 8), (16, 1, 8), (2, 8, 8), (8, 2, 8)]


def time_scheme_generation(bsa, w, qd, dev, args, barrier):
    """CUDA-event timing of bsa_aggregation_scores over three candidate block
    shapes (the workload's own first), inputs resident (larger than L2)."""
    shapes = [(w.bf, w.br, w.bc)] + [s for s in CANDIDATE_SHAPES if s != (w.bf, w.br, w.bc)][:2]
    plans = [bsa.Plan(w.B, w.T, w.H, w.W, bf, br, bc, w.Hd, w.D, w.n_text, qd.dtype, dev)
             for bf, br, bc in shapes]
    L = bsa.load()
    n = len(plans)
    sics = [torch.empty((w.B, w.Hd, p.info.nb), dtype=torch.float32, device=dev) for p in plans]
    as_ = torch.empty((n, w.B, w.Hd), dtype=torch.float64, device=dev)
    choice = torch.empty((w.B, w.Hd), dtype=torch.int32, device=dev)
    handles = (ctypes.c_void_p * n)(*[p._h.value for p in plans])
    outs = (ctypes.c_void_p * n)(*[t.data_ptr() for t in sics])
    stream = torch.cuda.current_stream(dev)

    def call():
        bsa._check(L.bsa_aggregation_scores(handles, n, bsa._ptr(qd), outs, bsa._ptr(as_),
                                            bsa._ptr(choice), bsa._stream(dev)))

    for _ in range(args.warmup):
        call()
    barrier()
    # replayed from a CUDA graph of 10 calls, so host launch gaps do not count
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(10):
            call()
    graph.replay()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = max(1, args.steps // 10)
    e0.record(stream)
    for _ in range(reps):
        graph.replay()
    e1.record(stream)
    barrier()
    ms = e0.elapsed_time(e1) / (10 * reps)
    del graph
    x_bytes = qd.numel() * qd.element_size()
    return {"candidates": [f"{a}x{b}x{c}" for a, b, c in shapes], "ms": round(ms, 4),
            "algorithmic_bytes": x_bytes,
            "achieved_gbs": round(x_bytes / (ms * 1e-3) / 1e9, 1),
            "choice_histogram": torch.bincount(choice.flatten().long(), minlength=n).tolist()}


# The other workloads of the suite, each timed in its own loop beside the
# headline: the 4x8x8 fp32 case, Wan2.1-1.3B, HunyuanVideo at the 20% target
# density, Wan2.1-14B (mixed per-head density, then Top-P tau = 0.9) and the
# 333-frame Long shape.
SUITE = ["tiny", "wan13", "hunyuan20", "wan14", "wan14_topp", "long"]


def _inputs_key(w):
    return (w.B, w.T, w.H, w.W, w.Hd, w.D, w.n_text, w.dtype, w.qk_std)


def time_workload(bsa, name, dev, barrier, args, cache, peak_burst, peak_sust):
    """One workload of the suite: bsa_forward steps timed with CUDA events over
    at least ~0.6 s (so the clock sampler sees the loop), its phases timed in a
    second loop, SM clocks sampled during the first.  Inputs (CPU, seeded) are
    shared between workloads of the same shape through `cache`."""
    w = synthetic.workload(name)
    key = _inputs_key(w)
    if key not in cache:
        cache.clear()
        cache[key] = synthetic.make_qkv(w)
    q, k, v = cache[key]
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    plan = bsa.plan_for(w, dev)
    L = bsa.load()
    P = bsa._ptr
    params = bsa._params(w.params, w.Hd)
    kmax = plan.kmax_for(w.mode, w.params)
    _, fwd_ws = plan.workspace_size(kmax)
    ws = torch.empty(fwd_ws, dtype=torch.uint8, device=dev)
    out = torch.empty_like(qd)
    idx = torch.empty((w.B, w.Hd, plan.info.nb, kmax), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.B, w.Hd, plan.info.nb), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    S = lambda: bsa._stream(dev)

    def forward():
        bsa._check(L.bsa_forward(plan._h, P(qd), P(kd), P(vd), w.mode, params, kmax, P(out), P(idx),
                                 P(cnt), P(ws), ws.numel(), None, S()))

    for _ in range(args.warmup):
        forward()
    barrier()
    plan.check_status()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(3):
        forward()
    e1.record(stream)
    barrier()
    est_ms = e0.elapsed_time(e1) / 3
    n = int(min(20000, max(args.steps, -(-600.0 // max(est_ms, 1e-3)))))
    pairs = effective_pairs(plan, idx, cnt)
    flops = 4.0 * pairs * w.D
    with ClockSampler(dev.index) as clk:
        clk.mark_start()
        e0.record(stream)
        for _ in range(n):
            forward()
        e1.record(stream)
        barrier()
        clk.mark_end()
    plan.check_status()
    step_ms = e0.elapsed_time(e1) / n
    clocks = clk.summary()

    qc, kc = (torch.empty(plan.cent_shape, dtype=torch.float32, device=dev) for _ in range(2))
    if plan.info.attn_path == 1:
        pz = ctypes.c_size_t()
        bsa._check(L.bsa_pair_workspace_size(plan._h, kmax, ctypes.byref(pz)))
        pws = torch.empty(pz.value, dtype=torch.uint8, device=dev)
        paired = plan.info.nb <= 1536
        names = ["centroids", "select"] + (["pairing"] if paired else []) + ["attention"]
        calls = [lambda: L.bsa_centroids(plan._h, P(qd), P(kd), P(qc), P(kc), S()),
                 lambda: L.bsa_select_centroids(plan._h, P(qc), P(kc), w.mode, params, kmax, P(idx),
                                                P(cnt), None, S())]
        if paired:
            calls += [lambda: L.bsa_pair_tiles(plan._h, P(idx), P(cnt), kmax, P(pws), pws.numel(), S()),
                      lambda: L.bsa_attention_paired(plan._h, P(qd), P(kd), P(vd), P(idx), P(cnt), kmax,
                                                     P(pws), pws.numel(), P(out), None, S())]
        else:
            calls += [lambda: L.bsa_attention_orig(plan._h, P(qd), P(kd), P(vd), P(idx), P(cnt), kmax,
                                                   P(out), None, S())]
        # per bsa_forward step: centroids, select, 3 pairing kernels, attention, text merge
        launches = 3 + (3 if paired else 0) + (1 if paired and plan.info.nb_text > 0 else 0)
    else:
        qb, kb, vb, ob = (torch.empty(plan.blk_shape, dtype=plan.dtype, device=dev) for _ in range(4))
        names = ["permute", "select", "attention", "unpermute"]
        calls = [lambda: L.bsa_permute_qkv(plan._h, P(qd), P(kd), P(vd), P(qb), P(kb), P(vb), P(qc),
                                           P(kc), S()),
                 lambda: L.bsa_select_centroids(plan._h, P(qc), P(kc), w.mode, params, kmax, P(idx),
                                                P(cnt), None, S()),
                 lambda: L.bsa_attention(plan._h, P(qb), P(kb), P(vb), P(idx), P(cnt), kmax, P(ob),
                                         None, S()),
                 lambda: L.bsa_unpermute(plan._h, P(ob), P(out), S())]
        launches = 4
    for _ in range(args.warmup):
        for c in calls:
            bsa._check(c())
    m = max(3, min(n, 50))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(m)]
    barrier()
    for si in range(m):
        evs[si][0].record(stream)
        for ci, c in enumerate(calls):
            bsa._check(c())
            evs[si][ci + 1].record(stream)
    barrier()
    plan.check_status()
    ph = {nm: sum(evs[si][ci].elapsed_time(evs[si][ci + 1]) for si in range(m)) / m
          for ci, nm in enumerate(names)}
    attn_tf = flops / (ph["attention"] * 1e-3) / 1e12
    pre_calls = ph.get("centroids", ph.get("permute", 0.0)) + ph["select"] + ph.get("pairing", 0.0)
    # the same split inside bsa_forward as it runs (events at its phase
    # boundaries; the selection there also hands the pairing its bit sets)
    splits = [plan.forward_timed(qd, kd, vd, w.mode, w.params, kmax=kmax, out=out, workspace=ws)[1]
              for _ in range(max(5, min(m, 15)))]
    plan.check_status()
    fs = {key: statistics.median(sp[key] for sp in splits) for key in splits[0]}
    pre = fs["summaries_ms"] + fs["select_ms"] + fs["pairing_ms"]
    res = {
        "shape": workload_config(w)["shape"],
        "selection": workload_config(w)["selection"],
        "steps": n,
        "ms_per_step": round(step_ms, 4),
        "step_tflops": round(flops / (step_ms * 1e-3) / 1e12, 2),
        "effective_tflop_per_step": round(flops / 1e12, 4),
        "mean_list_len": round(float(cnt.float().mean()), 2),
        "phases_ms": {nm: round(t, 4) for nm, t in ph.items()},
        "attn_ms": round(ph["attention"], 4),
        "attn_tflops": round(attn_tf, 2),
        "phases_ms_in_forward": {key: round(t, 4) for key, t in fs.items()},
        "pre_attention_share": round(pre / fs["attention_ms"], 4),
        "pre_attention_share_of": "summaries + select + pairing over attention, inside bsa_forward_timed",
        "pre_attention_share_calls": round(pre_calls / ph["attention"], 4),
        "pre_attention_phases": [nm for nm in names if nm not in ("attention", "unpermute")],
        "clocks": clocks,
        "gpu_launches_per_step": launches,
    }
    if plan.info.attn_path == 1:
        res["attn_frac_of_burst"] = round(attn_tf / peak_burst, 4)
        res["attn_frac_of_sustained"] = round(attn_tf / peak_sust, 4)
    else:
        res["attn_bound"] = "alu (fp32 SIMT kernel)"
        res["attn_frac_of_fp32_peak"] = round(attn_tf / FP32_PEAK_TFLOPS, 4)
    traffic = profiled_traffic(name)
    if traffic is not None:
        res["attn_dram_bytes_per_launch"] = traffic
    del qd, kd, vd, out, ws
    torch.cuda.empty_cache()
    return res


def run_ours(args, rank, world, local):
    import block_sparse_attention_permute_b200 as bsa

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=dev)
    w = synthetic.workload(args.workload)
    if args.heads:
        reps = args.heads // len(w.params) + 1
        w.Hd, w.params = args.heads, (w.params * reps)[:args.heads]
        w.name = f"{w.name}_{args.heads}heads"
    q, k, v = synthetic.make_qkv(w)
    plan = bsa.plan_for(w, dev)
    kmax = plan.kmax_for(w.mode, w.params)
    sel_ws, fwd_ws = plan.workspace_size(kmax)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    out = torch.empty_like(qd)
    ws = torch.empty(fwd_ws, dtype=torch.uint8, device=dev)
    idx = torch.empty((w.B, w.Hd, plan.info.nb, kmax), dtype=torch.int32, device=dev)
    cnt = torch.empty((w.B, w.Hd, plan.info.nb), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    L = bsa.load()
    params = bsa._params(w.params, w.Hd)
    P = bsa._ptr

    def forward():
        bsa._check(L.bsa_forward(plan._h, P(qd), P(kd), P(vd), w.mode, params, kmax, P(out), P(idx),
                                 P(cnt), P(ws), ws.numel(), None, bsa._stream(dev)))

    def barrier():
        torch.cuda.synchronize(dev)
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        forward()
    plan.check_status()
    pairs = effective_pairs(plan, idx, cnt)
    flops = 4.0 * pairs * w.D

    # ---- main timed loop: K whole steps
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev_step = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    with ClockSampler(local) as clk:
        clk.mark_start()
        ev0.record(stream)
        for i in range(args.steps):
            forward()
            ev_step[i].record(stream)
        ev1.record(stream)
        barrier()
        clk.mark_end()
    plan.check_status()
    step_ms = ev0.elapsed_time(ev1) / args.steps
    per_step = [ev0.elapsed_time(ev_step[0])] + [ev_step[i - 1].elapsed_time(ev_step[i])
                                                for i in range(1, args.steps)]
    step_stats = {"min": round(min(per_step), 4), "median": round(statistics.median(per_step), 4),
                  "max": round(max(per_step), 4)}
    clocks = clk.summary()

    # ---- phase loops (CUDA events on the launching stream)
    def time_phases(names, calls):
        for _ in range(args.warmup):
            for c in calls:
                bsa._check(c())
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)]
               for _ in range(args.steps)]
        barrier()
        for st_i in range(args.steps):
            evs[st_i][0].record(stream)
            for ci, c in enumerate(calls):
                bsa._check(c())
                evs[st_i][ci + 1].record(stream)
        barrier()
        plan.check_status()
        return {n: sum(evs[si][ci].elapsed_time(evs[si][ci + 1]) for si in range(args.steps)) / args.steps
                for ci, n in enumerate(names)}

    # ---- the same split from inside the library: one bsa_forward_timed call
    # (events at its phase boundaries), median of a few calls
    splits = [plan.forward_timed(qd, kd, vd, w.mode, w.params, kmax=kmax, out=out, workspace=ws)[1]
              for _ in range(5)]
    library_split = {key: round(statistics.median(sp[key] for sp in splits), 4) for key in splits[0]}
    plan.check_status()

    qc, kc = (torch.empty(plan.cent_shape, dtype=torch.float32, device=dev) for _ in range(2))
    S = lambda: bsa._stream(dev)
    if plan.info.attn_path == 1:
        # what bsa_forward runs on this plan: the layout transform is fused into
        # the attention, whose query tiles are paired by shared key blocks
        pz = ctypes.c_size_t()
        bsa._check(L.bsa_pair_workspace_size(plan._h, kmax, ctypes.byref(pz)))
        pws = torch.empty(pz.value, dtype=torch.uint8, device=dev)
        fused = time_phases(
            ["centroids", "select", "pairing", "attention", "attention_unpaired"],
            [lambda: L.bsa_centroids(plan._h, P(qd), P(kd), P(qc), P(kc), S()),
             lambda: L.bsa_select_centroids(plan._h, P(qc), P(kc), w.mode, params, kmax, P(idx),
                                            P(cnt), None, S()),
             lambda: L.bsa_pair_tiles(plan._h, P(idx), P(cnt), kmax, P(pws), pws.numel(), S()),
             lambda: L.bsa_attention_paired(plan._h, P(qd), P(kd), P(vd), P(idx), P(cnt), kmax,
                                            P(pws), pws.numel(), P(out), None, S()),
             # the same lists without pairing, for comparison (not part of the step)
             lambda: L.bsa_attention_orig(plan._h, P(qd), P(kd), P(vd), P(idx), P(cnt), kmax, P(out),
                                          None, S())])
    else:
        fused = None
    qb, kb, vb, ob = (torch.empty(plan.blk_shape, dtype=plan.dtype, device=dev) for _ in range(4))
    unfused = time_phases(
        ["permute", "select", "attention", "unpermute"],
        [lambda: L.bsa_permute_qkv(plan._h, P(qd), P(kd), P(vd), P(qb), P(kb), P(vb), P(qc), P(kc), S()),
         lambda: L.bsa_select_centroids(plan._h, P(qc), P(kc), w.mode, params, kmax, P(idx), P(cnt),
                                        None, S()),
         lambda: L.bsa_attention(plan._h, P(qb), P(kb), P(vb), P(idx), P(cnt), kmax, P(ob), None, S()),
         lambda: L.bsa_unpermute(plan._h, P(ob), P(out), S())])
    del qb, kb, vb, ob
    phase_ms = fused if fused is not None else unfused

    # ---- the DSA / DSA2 box estimators in place of MEAN
    estimators = time_estimators(bsa, w, plan, qd, kd, vd, out, dev, args, barrier)

    # ---- forward with the mask union (window, sink, intra blocks added)
    union = time_union_forward(bsa, w, plan, qd, kd, vd, out, dev, args, barrier)

    # ---- per-head blocking schemes: grouped forward on the aggregation choice
    grouped = time_grouped_forward(bsa, w, qd, kd, vd, dev, args, barrier)

    # ---- scheme generation (aggregation evaluation over candidate blockings):
    # one launch evaluates three candidate schemes of Q; timed alone.
    scheme = time_scheme_generation(bsa, w, qd, dev, args, barrier)

    # ---- end to end: pinned host buffers, copies inside the timed region.
    # Serial: upload, forward, download on one stream.  Pipelined: three
    # streams and double-buffered device tensors, so step i+1's upload runs
    # while step i computes and step i-1's output downloads; every step still
    # moves its own inputs up and its own output down.
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    ohs = [torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(2)]
    h2d = 3 * q.numel() * q.element_size()
    d2h = q.numel() * q.element_size()

    def upload(dst):
        for d_t, h_t in zip(dst, (qh, kh, vh)):
            d_t.copy_(h_t, non_blocking=True)

    for _ in range(2):
        upload((qd, kd, vd)); forward(); ohs[0].copy_(out, non_blocking=True)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        upload((qd, kd, vd)); forward(); ohs[0].copy_(out, non_blocking=True)
    e1.record(stream)
    barrier()
    e2e_serial_ms = e0.elapsed_time(e1) / args.steps
    ref_out = ohs[0].clone()

    ins = [(qd, kd, vd), tuple(torch.empty_like(t) for t in (qd, kd, vd))]
    outs = [out, torch.empty_like(out)]
    s_up, s_dn = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_dn = [torch.cuda.Event() for _ in range(2)]

    def run_pipelined(n_steps, first_event=None):
        for i in range(n_steps):
            bi = i % 2
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(ev_done[bi])            # compute i-2 finished reading ins[bi]
                if i == 0 and first_event is not None:
                    first_event.record(s_up)
                upload(ins[bi])
                ev_in[bi].record(s_up)
            stream.wait_event(ev_in[bi])
            if i >= 2:
                stream.wait_event(ev_dn[bi])                 # download i-2 finished reading outs[bi]
            qi, ki, vi = ins[bi]
            bsa._check(L.bsa_forward(plan._h, P(qi), P(ki), P(vi), w.mode, params, kmax,
                                     P(outs[bi]), P(idx), P(cnt), P(ws), ws.numel(), None,
                                     bsa._stream(dev)))
            ev_done[bi].record(stream)
            with torch.cuda.stream(s_dn):
                s_dn.wait_event(ev_done[bi])
                ohs[bi].copy_(outs[bi], non_blocking=True)
                ev_dn[bi].record(s_dn)

    run_pipelined(3)
    barrier()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run_pipelined(args.steps, first_event=p0)
    p1.record(s_dn)
    barrier()
    e2e_ms = p0.elapsed_time(p1) / args.steps
    # the overlapped steps did all their work: the last downloaded output equals
    # the serial loop's (same inputs, deterministic kernels)
    assert torch.equal(ohs[(args.steps - 1) % 2], ref_out), "pipelined e2e output differs"

    # ---- the other workloads of the suite, one loop each (one GPU only: the
    # replicas of a multi-GPU run would only repeat them)
    suite = {}
    if world == 1 and not args.no_suite:
        peak_b, peak_s, _, _ = peaks()
        del ins, outs
        cache = {_inputs_key(w): (q, k, v)}
        for name in SUITE:
            if name != w.name:
                suite[name] = time_workload(bsa, name, dev, barrier, args, cache, peak_b, peak_s)
        cache.clear()

    step_ms, e2e_ms, e2e_serial_ms, attn_ms = reduce_max(
        [step_ms, e2e_ms, e2e_serial_ms, phase_ms["attention"]], dev)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()

    if rank != 0:
        return
    peak_tf, peak_sust, hbm_gbs, peak_src = peaks()
    phase_roof = phase_rooflines(w, plan, fused, unfused, hbm_gbs)
    value = job_tflops(world, flops, step_ms)
    attn_tf = flops / (attn_ms * 1e-3) / 1e12
    traffic = profiled_traffic(args.workload)
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4),
        "ms_per_step_stats": step_stats,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": {
            **workload_config(w),
            "parallelism": f"replicas x{world} (no collective)",
            "l2": f"inputs {3 * q.numel() * q.element_size() / 1e9:.2f} GB > 126 MB L2 (no flush)",
            "effective_tflop_per_step": round(flops / 1e12, 4),
            "selected_pairs": pairs,
        },
        "phases_ms": {n: round(t, 4) for n, t in phase_ms.items()},
        "phases_ms_in_forward": library_split,
        "phases_ms_unfused": {n: round(t, 4) for n, t in unfused.items()},
        "attn_tflops": round(attn_tf, 2),
        "attn_frac_of_peak": round(attn_tf / peak_tf, 4),
        "phase_rooflines": phase_roof,
        "permute_select_share_of_attn": round(
            (phase_ms.get("centroids", phase_ms.get("permute", 0.0)) + phase_ms["select"]
             + phase_ms.get("pairing", 0.0)) / phase_ms["attention"], 4),
        "permute_select_share_of_attn_in_forward": round(
            (library_split["summaries_ms"] + library_split["select_ms"] + library_split["pairing_ms"])
            / library_split["attention_ms"], 4),
        "permute_select_share_of_attn_unfused": round(
            (unfused["permute"] + unfused["select"]) / unfused["attention"], 4),
        "roofline": {
            "bound": "tensor",
            "kernel": "attn_tc_kernel<128, original layout, paired tiles>" if plan.info.attn_path == 1
                      else "attn_simt_kernel",
            "achieved": round(attn_tf, 2),
            "peak": peak_tf,
            "peak_source": f"{peak_src} bf16_tflops (burst: cuBLAS timed alone; this loop is "
                           f"event-timed and well under a second, at the sampled clocks below)",
            "unit": "TFLOP/s",
            "frac": round(attn_tf / peak_tf, 4),
            "peak_sustained": peak_sust,
            "frac_of_sustained": round(attn_tf / peak_sust, 4),
            "traffic": traffic,
        },
        "e2e": {"value": round(job_tflops(world, flops, e2e_ms), 2), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "mode": "pipelined across steps (upload / compute / download streams, "
                        "double-buffered device tensors)",
                "serial": {"value": round(job_tflops(world, flops, e2e_serial_ms), 2),
                           "ms_per_step": round(e2e_serial_ms, 3)}},
        "mask_union": dict(union, frac_of_peak=round(union["tflops"] / peak_tf, 4)),
        "estimators": estimators,
        "scheme_adaptive": dict(grouped, frac_of_peak=round(grouped["tflops"] / peak_tf, 4)),
        "scheme_generation": dict(scheme, share_of_attn=round(scheme["ms"] / phase_ms["attention"], 4),
                                  frac=round(scheme["achieved_gbs"] / hbm_gbs, 4),
                                  peak_gbs=hbm_gbs, bound="hbm"),
        # per bsa_forward step, tensor-core plans: centroids, select (which also
        # writes the lists' bit sets), 3 pairing kernels (candidates, matching,
        # reordered lists; none beyond 1536 video blocks), attention, and with
        # text tokens the merge of the text chunks; other plans: permute,
        # select, attention, unpermute
        "gpu_launches": ((3 + (3 if plan.info.nb <= 1536 else 0)
                          + (1 if plan.info.nb <= 1536 and plan.info.nb_text > 0 else 0))
                         if plan.info.attn_path == 1 else 4) * args.steps,
        "clocks": clocks,
        "workloads": suite,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, q, k, v, budget_s=args.cpu_seconds)
    print(json.dumps(line), flush=True)


# fp32 FMA peak of the selection's score GEMM: 148 SMs x 128 FMA lanes x 2 FLOP
# x the 1965 MHz maximum SM clock (derived from the unit counts, not measured)
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def phase_rooflines(w, plan, fused, unfused, hbm_gbs):
    """Achieved rate of every non-attention phase against its roofline, from
    the phases' CUDA-event times: HBM phases by their algorithmic bytes (each
    input byte read once, each output byte written once), the selection by the
    fp32 FLOP of its score GEMM."""
    e = 2 if w.dtype == "bf16" else 4
    info = plan.info
    row = w.Hd * w.D * e * w.B                       # bytes of one token of Q, K or V
    n_tot, n_pad = info.n_tot, info.npad_tot
    cent_out = 2 * w.B * w.Hd * info.nb * w.D * 4
    out = {}

    def hbm(name, ms, nbytes):
        if ms and ms > 0:
            gbs = nbytes / (ms * 1e-3) / 1e9
            out[name] = {"bound": "hbm", "bytes": int(nbytes), "ms": round(ms, 4),
                         "achieved_gbs": round(gbs, 1), "peak_gbs": hbm_gbs,
                         "frac": round(gbs / hbm_gbs, 3)}

    if fused is not None:
        hbm("centroids", fused["centroids"], 2 * info.n_video * row + cent_out)   # video tokens only
    hbm("permute_qkv", unfused["permute"], 3 * n_tot * row + 3 * n_pad * row + cent_out)
    hbm("unpermute", unfused["unpermute"], n_pad * row + n_tot * row)
    sel_ms = (fused or unfused)["select"]
    sel_flop = 2.0 * w.B * w.Hd * info.nb * info.nb * w.D
    tf = sel_flop / (sel_ms * 1e-3) / 1e12
    out["select"] = {"bound": "alu", "flop": sel_flop, "ms": round(sel_ms, 4),
                     "achieved_tflops": round(tf, 2), "peak_tflops": round(FP32_PEAK_TFLOPS, 1),
                     "peak_source": "derived: 148 SMs x 128 fp32 FMA/clk x 2 x 1965 MHz",
                     "frac": round(tf / FP32_PEAK_TFLOPS, 3)}
    return out


def workload_config(w):
    """The workload keys shared by both arms' config."""
    return {
        "workload": w.name,
        "shape": f"grid {w.T}x{w.H}x{w.W} + {w.n_text} text, block {w.bf}x{w.br}x{w.bc}, "
                 f"{w.Hd} heads, head_dim {w.D}, batch {w.B}",
        "selection": ("top-k density " if w.mode == 0 else "top-p tau ") +
                     (str(w.params[0]) if len(set(w.params)) == 1 else "per-head mix"),
    }


class OracleSampler:
    """The fp64 oracle, as it stands, on bounded samples of a workload: the
    selection of the whole workload once, then attention on whole random query
    blocks (all heads) for a time budget per sample."""

    def __init__(self, w, q, k, v):
        import oracle as orc
        self.orc, self.w = orc, w
        self.g = orc.Geometry(*w.geometry_args())
        self.qn, self.kn, self.vn = (t.float().numpy() for t in (q, k, v))
        t0 = time.perf_counter()
        p = orc.scores(self.g, orc.centroids(self.g, self.qn), orc.centroids(self.g, self.kn))
        self.idx, self.cnt, _ = orc.select(self.g, p, w.mode, w.params)
        self.t_sel = time.perf_counter() - t0
        self.full_flop = 4.0 * orc.selected_pairs(self.g, self.idx, self.cnt) * self.g.D
        self.rng = np.random.default_rng(0)
        self.valid_tab = {}

    def sample(self, budget_s, chunk=None):
        """Effective FLOP and seconds of oracle attention over random query
        blocks (all heads; `chunk` rows of each if given), at least one block.
        Whole blocks keep the oracle's threads as busy as a full run would."""
        g = self.g
        pairs, t_att, nblk = 0, 0.0, 0
        while True:
            j = int(self.rng.integers(g.nb))
            tb, yb, xb = j // (g.nby * g.nbx), (j // g.nbx) % g.nby, j % g.nbx
            rows = [(t * g.H + y) * g.W + x
                    for t in range(tb * g.bf, min(g.T, (tb + 1) * g.bf))
                    for y in range(yb * g.br, min(g.H, (yb + 1) * g.br))
                    for x in range(xb * g.bc, min(g.W, (xb + 1) * g.bc))]
            if chunk is not None:
                c0 = int(self.rng.integers(max(1, len(rows) - chunk + 1)))
                rows = rows[c0:c0 + chunk]
            t1 = time.perf_counter()
            self.orc.attention(g, self.qn, self.kn, self.vn, self.idx, self.cnt, rows=np.array(rows))
            t_att += time.perf_counter() - t1
            nblk += 1
            for b in range(g.B):
                for h in range(g.Hd):
                    keys = 0
                    for jj in self.idx[b, h, j, :self.cnt[b, h, j]]:
                        if jj not in self.valid_tab:
                            self.valid_tab[jj] = _valid_count(g, int(jj))
                        keys += self.valid_tab[jj]
                    pairs += keys * len(rows)
            if t_att >= budget_s:
                return 4.0 * pairs * g.D, t_att, nblk

    def baseline(self, flop, t_att, nblk):
        return {"value": flop / t_att / 1e12, "unit": "TFLOP/s", "cores": self.orc.threads(),
                "kind": "oracle", "full_step_flop": self.full_flop,
                "sample": f"oracle centroids+scores+selection on the full workload "
                          f"({self.t_sel:.1f} s, once), attention on {nblk} random query blocks "
                          f"x all {self.g.Hd} heads ({t_att:.1f} s); value = effective FLOP of "
                          f"the sampled attention / its time"}


def cpu_baseline(w, q, k, v, budget_s=20.0):
    """The fp64 oracle, as it stands, on a bounded sample of the workload."""
    o = OracleSampler(w, q, k, v)
    return o.baseline(*o.sample(max(0.0, budget_s - o.t_sel)))


def _valid_count(g, j):
    if j >= g.nb:
        return min(g.bs, g.n_text - (j - g.nb) * g.bs)
    tb, yb, xb = j // (g.nby * g.nbx), (j // g.nbx) % g.nby, j % g.nbx
    return (min(g.bf, g.T - tb * g.bf) * min(g.br, g.H - yb * g.br) * min(g.bc, g.W - xb * g.bc))


def run_reference(args, rank, world):
    if rank != 0:
        return
    w = synthetic.workload(args.workload)
    q, k, v = synthetic.make_qkv(w)
    o = OracleSampler(w, q, k, v)
    # every step a bounded sample (at least one query block, all heads): about
    # a minute of oracle attention in all, or one block per step when steps
    # are many (about 0.7 s each on 16 host cores for the HunyuanVideo shape)
    per_step = 60.0 / max(1, args.steps + args.warmup)
    flop = t_att = 0.0
    nblk = 0
    for s_i in range(args.warmup + args.steps):
        f, t, n = o.sample(per_step)
        if s_i >= args.warmup:
            flop, t_att, nblk = flop + f, t_att + t, nblk + n
    cb = o.baseline(flop, t_att, nblk)
    value = cb["value"]
    # one whole step of the workload at the sampled rate
    ms_full = cb["full_step_flop"] / (value * 1e12) * 1e3
    config = workload_config(w)
    config["parallelism"] = f"host cores ({cb['cores']} oracle threads)"
    config["ms_per_step_note"] = "one full step extrapolated from the sampled rate"
    line = {
        "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_full, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": config,
        "cpu_baseline": cb,
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="hunyuan", choices=synthetic.WORKLOADS)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-suite", action="store_true",
                    help="time the headline workload only (skip the other workloads' loops)")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the workload's head count (smaller profiling cases)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)   # at least 3 untimed warm-up steps
    rank, world, local = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
