"""Seeded synthetic workloads shared by the tests, the smoke check and the bench.

This module holds workload shapes and the input recipe only — none of the
attention method's arithmetic.  Both the CUDA path and the CPU oracle receive
the tensors it makes; neither imports the other.

Input recipe (stands in for the pages' model workloads — VBench-2.0 and
MovieGen prompts through Wan and HunyuanVideo — which need datasets and
trained weights; the shapes are those models' latent grids):
  * For each tensor (Q seed 1, K seed 2, V seed 3), batch element b, head h
    and channel c: 8 frequency triples (f_t, f_y, f_x) ~ U[0, 3) cycles over
    the grid extent of each axis, a phase ~ U[0, 2*pi) and an amplitude
    a ~ N(0, 1).  field(t,y,x) = sum_k a_k cos(2*pi*(f_t t/T + f_y y/H +
    f_x x/W) + phase_k), divided by sqrt(sum_k a_k^2 / 2) (unit variance).
  * x = 0.7 * field + 0.3 * N(0, 1).
  * Text tokens: 0.7 * (a per batch/head/channel constant ~ N(0, 1)) +
    0.3 * N(0, 1).
  * bf16 workloads: Q and K (text included) are multiplied by a common
    per-head factor s so that the standard deviation of q.k/sqrt(D) over 4096
    seeded random (video query, video key) pairs is 3 (factor 1 when those
    pairs have no spread, e.g. a one-token grid); V is not scaled.  The result
    is rounded to bf16 (round to nearest even).
  * Per-head mixed density (Wan2.1-14B shape): u ~ U[0, 1) per head (seed 4);
    rho = 0.03 if u < 0.35, 0.05 if u < 0.50, else 0.10.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field as dc_field

import numpy as np
import torch


@dataclass
class Workload:
    name: str
    B: int
    T: int
    H: int
    W: int
    bf: int
    br: int
    bc: int
    Hd: int
    D: int
    dtype: str            # "f32" | "bf16"
    mode: int             # 0 = top-k (params are densities), 1 = top-p (params are tau)
    params: list = dc_field(default_factory=list)   # per head
    n_text: int = 0
    qk_std: float | None = 3.0   # target std of q.k/sqrt(D); None = unscaled
    note: str = ""

    @property
    def bs(self):
        return self.bf * self.br * self.bc

    @property
    def nb(self):
        return -(-self.T // self.bf) * -(-self.H // self.br) * -(-self.W // self.bc)

    @property
    def nb_text(self):
        return -(-self.n_text // self.bs)

    @property
    def n_tot(self):
        return self.T * self.H * self.W + self.n_text

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def geometry_args(self):
        return (self.B, self.T, self.H, self.W, self.bf, self.br, self.bc, self.Hd, self.D,
                self.n_text)


def mixed_densities(Hd: int, seed: int = 4) -> list:
    """Per-head density draw of the Wan2.1-14B workload (probabilities .35/.15/.50)."""
    u = np.random.default_rng(seed).random(Hd)
    return [0.03 if x < 0.35 else (0.05 if x < 0.50 else 0.10) for x in u]


def workload(name: str) -> Workload:
    """The five workloads (plus the 20%-density Hunyuan point and the top-p pass)."""
    if name == "tiny":
        return Workload("tiny", 1, 4, 8, 8, 2, 4, 4, 2, 64, "f32", 0, [0.25] * 2, qk_std=None,
                        note="4x8x8 grid, block 2x4x4, 2 heads, D=64, fp32, density 0.25")
    if name == "wan13":
        return Workload("wan13", 1, 21, 30, 52, 4, 4, 8, 12, 128, "bf16", 0, [0.20] * 12,
                        note="Wan2.1-1.3B 480p 81f: 21x30x52, block 4x4x8, 12 heads, density 0.20")
    if name in ("hunyuan", "hunyuan20"):
        rho = 0.15 if name == "hunyuan" else 0.20
        return Workload(name, 1, 16, 45, 80, 1, 8, 16, 24, 128, "bf16", 0, [rho] * 24,
                        n_text=256,
                        note=f"HunyuanVideo 720p 61f: 16x45x80 + 256 text, block 1x8x16, "
                             f"24 heads, density {rho}")
    if name == "wan14":
        return Workload("wan14", 1, 21, 30, 52, 4, 4, 8, 40, 128, "bf16", 0, mixed_densities(40),
                        note="Wan2.1-14B 480p 81f: 21x30x52, block 4x4x8, 40 heads, "
                             "per-head density {.03,.05,.10}")
    if name == "wan14_topp":
        return Workload("wan14_topp", 1, 21, 30, 52, 4, 4, 8, 40, 128, "bf16", 1, [0.90] * 40,
                        note="Wan2.1-14B shape, cumulative threshold tau=0.90")
    if name == "long":
        return Workload("long", 1, 84, 30, 52, 4, 4, 8, 12, 128, "bf16", 0, [0.10] * 12,
                        note="4x Wan-1.3B (333 frames): 84x30x52, block 4x4x8, 12 heads, "
                             "density 0.10")
    raise KeyError(name)


WORKLOADS = ["tiny", "wan13", "hunyuan", "hunyuan20", "wan14", "wan14_topp", "long"]


def _field_tensor(B, T, H, W, Hd, D, n_text, seed) -> torch.Tensor:
    """0.7*unit-variance Fourier field + 0.3*N(0,1), float32 [B, Ntot, Hd, D]."""
    rng = np.random.default_rng(seed)
    f = rng.random((B, Hd, D, 8, 3)) * 3.0
    ph = rng.random((B, Hd, D, 8)) * 2.0 * math.pi
    amp = rng.standard_normal((B, Hd, D, 8))
    text_const = rng.standard_normal((B, Hd, D))
    norm = np.sqrt((amp ** 2).sum(-1) / 2.0)                      # [B,Hd,D]
    gen = torch.Generator().manual_seed(1000 + seed)
    n_video = T * H * W
    out = torch.empty((B, n_video + n_text, Hd, D), dtype=torch.float32)
    t = torch.arange(T, dtype=torch.float64)
    y = torch.arange(H, dtype=torch.float64)
    x = torch.arange(W, dtype=torch.float64)
    for b in range(B):
        for h in range(Hd):
            ft = torch.from_numpy(f[b, h, :, :, 0])               # [D,8]
            fy = torch.from_numpy(f[b, h, :, :, 1])
            fx = torch.from_numpy(f[b, h, :, :, 2])
            a = torch.from_numpy(amp[b, h] / norm[b, h][:, None])  # [D,8]
            # angle = A(t,y) + Bx(x): cos(A+Bx) = cosA cosBx - sinA sinBx
            A = 2 * math.pi * (ft[:, None, None, :] * t[None, :, None, None] / T
                               + fy[:, None, None, :] * y[None, None, :, None] / H) \
                + torch.from_numpy(ph[b, h])[:, None, None, :]     # [D,T,H,8]
            Bx = 2 * math.pi * fx[:, None, :] * x[None, :, None] / W  # [D,W,8]
            cA = (torch.cos(A) * a[:, None, None, :]).reshape(D, T * H, 8)
            sA = (torch.sin(A) * a[:, None, None, :]).reshape(D, T * H, 8)
            fld = torch.bmm(cA, torch.cos(Bx).transpose(1, 2)) \
                - torch.bmm(sA, torch.sin(Bx).transpose(1, 2))      # [D, T*H, W]
            out[b, :n_video, h, :] = (0.7 * fld.reshape(D, n_video).T).to(torch.float32)
            if n_text:
                out[b, n_video:, h, :] = torch.from_numpy(0.7 * text_const[b, h]).float()
    out += 0.3 * torch.randn(out.shape, generator=gen, dtype=torch.float32)
    return out


def make_qkv(w: Workload):
    """Seeded (q, k, v) CPU tensors [B, Ntot, Hd, D] in the workload's dtype."""
    return make_custom(w.B, w.T, w.H, w.W, w.Hd, w.D, w.n_text, w.dtype, w.qk_std)


def make_custom(B, T, H, W, Hd, D, n_text=0, dtype="bf16", qk_std=3.0, seed_base=0):
    """The recipe on an arbitrary grid: (q, k, v) CPU tensors [B, Ntot, Hd, D].

    seed_base=0 reproduces the workload seeds (Q 1, K 2, V 3, pair sample 7).
    """
    q = _field_tensor(B, T, H, W, Hd, D, n_text, 1 + 10 * seed_base)
    k = _field_tensor(B, T, H, W, Hd, D, n_text, 2 + 10 * seed_base)
    v = _field_tensor(B, T, H, W, Hd, D, n_text, 3 + 10 * seed_base)
    if qk_std is not None:
        rng = np.random.default_rng(7 + seed_base)
        n_video = T * H * W
        qi = torch.from_numpy(rng.integers(0, n_video, 4096))
        ki = torch.from_numpy(rng.integers(0, n_video, 4096))
        for b in range(B):
            for h in range(Hd):
                dots = (q[b, qi, h, :].double() * k[b, ki, h, :].double()).sum(-1) / math.sqrt(D)
                sd = float(dots.std())
                # a grid of one token (every sampled pair is the same pair) has no spread
                s = math.sqrt(qk_std / sd) if sd > 1e-3 else 1.0
                q[b, :, h, :] *= s
                k[b, :, h, :] *= s
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    return q.to(dt).contiguous(), k.to(dt).contiguous(), v.to(dt).contiguous()
