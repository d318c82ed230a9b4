"""Seeded synthetic video-DiT attention inputs (shared by the CUDA path's tests and the oracle).

This module only draws inputs; it holds none of the method's arithmetic. Both the
CUDA path and the CPU oracle receive the very same tensors from here.

Token order is frame-major: token t = f*Hf*Wf + y*Wf + x, tensors are [B, H, T, d] bf16.

Recipe (per (b, h, channel) and per tensor Q, K, V independently):
  * a smooth field: an N(0,1) grid of (ceil(Hf/8)+1) x (ceil(Wf/8)+1) points per frame,
    sampled bilinearly at (y/8, x/8) (grid point (gy, gx) sits on token (8gy, 8gx));
  * plus i.i.d. N(0, 0.3^2) noise;
  * optional attention sinks: `sinks` seeded token positions per frame; at those tokens
    K <- 4 K + 2 sqrt(d) u_h, and every query gets + 0.25 u_h (u_h a seeded unit vector
    per head), so that the sinks draw a large share of attention;
  * optional per-head temperature: Q of head h scaled by 0.5 * 4^(h/(H-1)) (0.5 ... 2.0);
  * rounded to bf16 (round-to-nearest-even).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, asdict, replace

import torch


@dataclass(frozen=True)
class Workload:
    """One attention call: shapes, pooling window and precision budgets (percent)."""
    name: str
    B: int
    H: int
    d: int
    F: int
    Hf: int
    Wf: int
    ph: int
    pw: int
    pct_fp8: int
    pct_fp4: int
    sinks: int = 0
    temperature: bool = False
    seed: int = 0
    pct_mix: int = 0     # percent of KV blocks with E4M3 scores and E2M1 P V (between FP8 and FP4)
    adapt_tau: float = 0.0   # > 0: skipped blocks with draft score >= adapt_tau join FP4 ...
    pct_fp4_max: int = 0     # ... up to this FP4 budget (percent)
    pct_bf16: int = 0        # percent of KV blocks in the bf16 tier above FP8 (the oracle only)

    @property
    def T(self) -> int:
        return self.F * self.Hf * self.Wf

    def as_dict(self) -> dict:
        return asdict(self)


# The five workloads: a tiny CPU-checkable case, Wan2.1-14B-like 480p and 720p layers,
# a HunyuanVideo-like 129-frame 720p layer and a budget sweep on the 720p shape (B=2).
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 64, 4, 16, 32, 4, 8, 15, 35, 0, False, 1000),
    "wan480": Workload("wan480", 1, 40, 128, 21, 30, 52, 8, 8, 10, 30, 4, False, 1001),
    "wan720": Workload("wan720", 1, 40, 128, 21, 45, 80, 8, 16, 10, 30, 4, False, 1002),
    "hunyuan720": Workload("hunyuan720", 1, 24, 128, 33, 45, 80, 8, 16, 5, 25, 0, True, 1003),
}
# The 720p layer with the mixed class between FP8 and FP4 (FP8 10 / mixed 10 / FP4 20 / skip 60).
WORKLOADS["wan720mix"] = Workload("wan720mix", 1, 40, 128, 21, 45, 80, 8, 16, 10, 20, 4, False, 1002, 10)
# The 720p layer with the error-bound-driven FP4 budget: FP8 10 / FP4 20, skipped blocks
# whose draft score reaches 0.002 recovered at FP4 up to 40 %.
WORKLOADS["wan720adapt"] = Workload("wan720adapt", 1, 40, 128, 21, 45, 80, 8, 16, 10, 20, 4, False, 1002, 0,
                                    0.002, 40)
SWEEP_BUDGETS = [(100, 0), (0, 100), (25, 0), (10, 30), (5, 45)]
for _i, (_p8, _p4) in enumerate(SWEEP_BUDGETS):
    WORKLOADS[f"sweep{_i}"] = Workload(f"sweep{_i}", 2, 40, 128, 21, 45, 80, 8, 16,
                                       _p8, _p4, 4, False, 1004)


def scaled(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (smaller test variants)."""
    return replace(w, **kw)


def _smooth_field(gen, B, H, F, Hf, Wf, d, device):
    gy, gx = math.ceil(Hf / 8) + 1, math.ceil(Wf / 8) + 1
    grid = torch.randn((B, H, F, gy, gx, d), generator=gen, device=device, dtype=torch.float32)
    ys = torch.arange(Hf, device=device)
    xs = torch.arange(Wf, device=device)
    y0, x0 = ys // 8, xs // 8
    wy = ((ys % 8).to(torch.float32) / 8.0).view(Hf, 1, 1)
    wx = ((xs % 8).to(torch.float32) / 8.0).view(1, Wf, 1)
    g00 = grid[:, :, :, y0][:, :, :, :, x0]
    g01 = grid[:, :, :, y0][:, :, :, :, x0 + 1]
    g10 = grid[:, :, :, y0 + 1][:, :, :, :, x0]
    g11 = grid[:, :, :, y0 + 1][:, :, :, :, x0 + 1]
    top = g00 * (1 - wx) + g01 * wx
    bot = g10 * (1 - wx) + g11 * wx
    return top * (1 - wy) + bot * wy  # [B, H, F, Hf, Wf, d]


def generate(w: Workload, device="cpu", seed: int | None = None):
    """Return (q, k, v) bf16 tensors of shape [B, H, T, d] on `device`.

    The stream of random numbers depends on the device's generator, so the CPU and a
    GPU give different (equally valid) draws for one seed; a parity check always hands
    the same tensors to both sides.
    """
    seed = w.seed if seed is None else seed
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    B, H, F, Hf, Wf, d = w.B, w.H, w.F, w.Hf, w.Wf, w.d
    out = []
    for _ in range(3):
        x = _smooth_field(gen, B, H, F, Hf, Wf, d, device)
        x = x + 0.3 * torch.randn(x.shape, generator=gen, device=device, dtype=torch.float32)
        out.append(x.reshape(B, H, F * Hf * Wf, d))
    q, k, v = out
    if w.sinks > 0:
        u = torch.randn((H, d), generator=gen, device=device, dtype=torch.float32)
        u = u / u.norm(dim=1, keepdim=True)
        HW = Hf * Wf
        pos = torch.stack([torch.randperm(HW, generator=gen, device=device)[: w.sinks]
                           for _ in range(F)])                       # [F, sinks]
        tok = (pos + torch.arange(F, device=device).view(F, 1) * HW).reshape(-1)
        k[:, :, tok, :] = 4.0 * k[:, :, tok, :] + 2.0 * math.sqrt(d) * u.view(1, H, 1, d)
        q = q + 0.25 * u.view(1, H, 1, d)
    if w.temperature and H > 1:
        t = 0.5 * torch.pow(torch.tensor(4.0, device=device),
                            torch.arange(H, device=device, dtype=torch.float32) / (H - 1))
        q = q * t.view(1, H, 1, 1)
    return tuple(x.to(torch.bfloat16).contiguous() for x in (q, k, v))
