"""Seeded synthetic inputs for the FVAttn single-GPU hot path.

This module only draws random numbers and lays them out.  It holds none of
the method's arithmetic (no reorder, pooling, scoring, selection or
attention), so that both the CUDA path and the CPU oracle can be fed the
same tensors from it without sharing any of the computation.

The workloads stand in for the step-distilled Wan2.2 I2V attention layers
that the FVAttn pages evaluate on ("FVAttn: Adaptive Sparse Attention with
Runtime Load Balancing for Video Generation", paperlayer.ai summary, section
4 Experiments).  The pages give no activation statistics, so the shapes are
Wan2.2 latent shapes (40 heads, head dim 128, 21 latent frames) and the
values are Gaussian with per-head query scales, which set how concentrated
each head's block-score distribution is (section 2 Background: Top-p keeps
fewer blocks for concentrated heads and more for flat ones).

Recipe (all draws in this order from one torch Generator seeded per config):
  1. X_q, X_k, X_v ~ N(0, 1) in fp32, laid out raster [B, N, H, D] with
     N = F*Hs*Ws tokens ordered (frame, row, col).
  2. Per-head query scales s_h (shape [H]).
  3. 720p-shaped layers only: a shared rank-8 spatio-temporal component
     Lr[n, :] = sum_r a_r(f, y, x) * w_r / sqrt(8),
     a_r = cos(2*pi*(alpha_r*f/F + beta_r*y/Hs + gamma_r*x/Ws) + phi_r),
     alpha, beta, gamma integers in {0, 1, 2}, phi_r ~ U(0, 2*pi),
     w_r ~ N(0, I_D); the same for every head and batch entry.
  Then Q = s_h * (X_q + 0.5*Lr), K = X_k + 0.5*Lr, V = X_v, each rounded
  to bf16 (round to nearest even).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, asdict
from typing import Optional

import torch


@dataclass
class Workload:
    """One attention layer's shape, routing parameters and input recipe."""
    name: str
    B: int
    H: int
    D: int
    F: int
    Hs: int
    Ws: int
    tf: int
    th: int
    tw: int
    p: float
    k: int
    seed: int
    qscale: str = "loguniform"     # "fixed", "loguniform" or "skew"
    qscale_values: tuple = ()      # used when qscale == "fixed"
    lowrank: bool = False
    lowrank_weight: float = 0.5
    lowrank_rank: int = 8
    layers: int = 1
    p_sweep: tuple = ()
    order: str = "raster"          # block order: "raster" tile order or "hilbert"

    @property
    def N(self) -> int:
        return self.F * self.Hs * self.Ws

    def as_dict(self) -> dict:
        return asdict(self)


WORKLOADS = {
    # Small enough for the oracle to finish in seconds.
    "tiny": Workload("tiny", B=1, H=2, D=64, F=2, Hs=8, Ws=8, tf=2, th=2, tw=4,
                     p=0.9, k=2, seed=0, qscale="fixed", qscale_values=(0.5, 3.0)),
    # Wan2.2 480p latent (21 x 30 x 52), 2x8x8 = 128-token blocks.
    "480p": Workload("480p", B=1, H=40, D=128, F=21, Hs=30, Ws=52, tf=2, th=8, tw=8,
                     p=0.9, k=8, seed=480),
    # Wan2.2 720p latent (21 x 45 x 80) with a shared low-rank component.
    "720p": Workload("720p", B=1, H=40, D=128, F=21, Hs=45, Ws=80, tf=2, th=8, tw=8,
                     p=0.9, k=16, seed=720, lowrank=True),
    # 480p geometry, half the heads concentrated, half flat; p is swept.
    "skew": Workload("skew", B=1, H=40, D=128, F=21, Hs=30, Ws=52, tf=2, th=8, tw=8,
                     p=0.9, k=8, seed=4800, qscale="skew",
                     p_sweep=(0.5, 0.7, 0.9, 0.95, 0.99)),
    # Classifier-free-guidance batch (B=2) at 720p, 1x8x8 = 64-token blocks,
    # 40 independent seeded layers (seed 7200 + layer).
    "cfg720p": Workload("cfg720p", B=2, H=40, D=128, F=21, Hs=45, Ws=80, tf=1, th=8, tw=8,
                        p=0.95, k=32, seed=7200, layers=40),
}


def custom_workload(**kw) -> Workload:
    """A workload with explicit fields (used for small test geometries)."""
    base = dict(name="custom", B=1, H=2, D=64, F=2, Hs=8, Ws=8, tf=2, th=2, tw=4,
                p=0.9, k=2, seed=1)
    base.update(kw)
    return Workload(**base)


def _head_scales(w: Workload, gen: torch.Generator, device) -> torch.Tensor:
    if w.qscale == "fixed":
        vals = list(w.qscale_values)
        assert len(vals) > 0
        s = torch.tensor([vals[h % len(vals)] for h in range(w.H)], dtype=torch.float32)
        return s.to(device)
    if w.qscale == "loguniform":
        u = torch.rand(w.H, generator=gen, device=device, dtype=torch.float32)
        lo, hi = math.log(0.25), math.log(4.0)
        return torch.exp(lo + (hi - lo) * u)
    if w.qscale == "skew":
        s = torch.empty(w.H, dtype=torch.float32, device=device)
        s[: w.H // 2] = 4.0
        s[w.H // 2:] = 0.25
        return s
    raise ValueError(f"unknown qscale recipe {w.qscale!r}")


def _lowrank(w: Workload, gen: torch.Generator, device) -> torch.Tensor:
    """The shared rank-r spatio-temporal component, [N, D] fp32."""
    r = w.lowrank_rank
    freqs = torch.randint(0, 3, (r, 3), generator=gen, device=device).to(torch.float32)
    phi = torch.rand(r, generator=gen, device=device, dtype=torch.float32) * (2 * math.pi)
    wr = torch.randn(r, w.D, generator=gen, device=device, dtype=torch.float32)
    f = torch.arange(w.F, device=device, dtype=torch.float32).view(w.F, 1, 1) / w.F
    y = torch.arange(w.Hs, device=device, dtype=torch.float32).view(1, w.Hs, 1) / w.Hs
    x = torch.arange(w.Ws, device=device, dtype=torch.float32).view(1, 1, w.Ws) / w.Ws
    out = torch.zeros(w.N, w.D, device=device, dtype=torch.float32)
    for i in range(r):
        a = torch.cos(2 * math.pi * (freqs[i, 0] * f + freqs[i, 1] * y + freqs[i, 2] * x) + phi[i])
        out += a.reshape(w.N, 1) * wr[i].view(1, w.D)
    return out / math.sqrt(r)


def make_qkv(w: Workload, layer: int = 0, device="cpu", seed: Optional[int] = None,
             head_scales: Optional[torch.Tensor] = None):
    """Draw raster Q, K, V ([B, N, H, D], bf16) for one layer of workload w.

    The seed is w.seed + layer unless given.  The generator lives on
    `device`, so CPU and CUDA draws differ; parity tests always hand the
    same tensors to both sides.  Returns (q, k, v, s_h).
    """
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed + layer if seed is None else seed)
    shape = (w.B, w.N, w.H, w.D)
    xq = torch.randn(shape, generator=gen, device=dev, dtype=torch.float32)
    xk = torch.randn(shape, generator=gen, device=dev, dtype=torch.float32)
    xv = torch.randn(shape, generator=gen, device=dev, dtype=torch.float32)
    s = _head_scales(w, gen, dev)
    if head_scales is not None:
        s = head_scales.to(dev, torch.float32)
    if w.lowrank:
        lr = _lowrank(w, gen, dev).view(1, w.N, 1, w.D) * w.lowrank_weight
        xq += lr
        xk += lr
    xq *= s.view(1, 1, w.H, 1)
    q = xq.to(torch.bfloat16)
    del xq
    k = xk.to(torch.bfloat16)
    del xk
    v = xv.to(torch.bfloat16)
    del xv
    return q, k, v, s


def bf16_bits(t: torch.Tensor):
    """The raw 16-bit patterns of a bf16 tensor, as a numpy uint16 array."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


def sample_items(n_items_total: int, count: int, seed: int):
    """A sorted, seeded sample of distinct flat item ids in [0, n_items_total)."""
    g = torch.Generator()
    g.manual_seed(seed)
    count = min(count, n_items_total)
    perm = torch.randperm(n_items_total, generator=g)[:count]
    return sorted(int(i) for i in perm)
