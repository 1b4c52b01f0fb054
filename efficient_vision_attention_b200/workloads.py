"""Seeded synthetic workloads for the Agent Attention forward pass.

This module only draws random numbers and names shapes; it holds none of the
method's arithmetic.  Both the CUDA path (through the tests and ``bench.py``)
and the fp64 oracle (through the tests) consume what it returns.

The shapes stand in for the pages' workloads, whose data and weights are not
available here (ImageNet-1K, DeiT / PVT / Swin backbones, Stable Diffusion
latents): DeiT-Tiny at 224^2 (14x14 tokens, 7x7 = 49 agents, the agent count
the jsqmd.com article's §2 tip binds to grid positions), a PVT/Swin stage-1 map
at 56x56, a Stable-Diffusion 1024^2 latent (128x128 tokens, 16x16 = 256 agents,
the 512^2 -> 256 agents row of the coreui.cn article's §3.1 table) and a
256x256 very-high-resolution sweep.

Recipe: a ``torch.Generator`` seeded with the workload's seed draws Q, K and V
(in that order) as i.i.d. N(0, 1) float32, multiplies each by the workload's
value scale, and casts to the run dtype (round-to-nearest-even for bf16).
Learnable agents, when the workload has them, are drawn afterwards from the
same generator as N(0, 0.02^2) with every value outside +-2 sigma redrawn (the
truncated-normal init of the jsqmd.com article's §2 tuning notes), then cast.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    grid_h: int
    grid_w: int
    d: int
    pool_h: int
    pool_w: int
    dtype: str            # "fp32" or "bf16"
    value_scale: float
    seed: int
    learnable_agents: int = 0   # > 0: that many externally supplied agents, pooling skipped

    @property
    def N(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def n_agents(self) -> int:
        return self.learnable_agents if self.learnable_agents else self.pool_h * self.pool_w

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "fp32" else 2

    def describe(self) -> dict:
        return {"workload": self.name, "B": self.B, "H": self.H, "N": self.N,
                "grid": [self.grid_h, self.grid_w], "d": self.d,
                "n_agents": self.n_agents,
                "agents": ("learnable" if self.learnable_agents
                           else f"avgpool {self.pool_h}x{self.pool_w}"),
                "dtype": self.dtype, "seed": self.seed}


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_fp32", 1, 1, 8, 8, 32, 2, 2, "fp32", 1.0, 0),
        Workload("deit_tiny_224", 64, 3, 14, 14, 64, 7, 7, "bf16", 0.5, 1),
        Workload("pvt_stage1_56", 16, 2, 56, 56, 32, 7, 7, "bf16", 1.0, 2),
        Workload("sd_latent_1024", 2, 8, 128, 128, 40, 16, 16, "bf16", 1.0, 3),
        Workload("highres_256_k64", 1, 8, 256, 256, 64, 8, 8, "bf16", 1.0, 4),
        Workload("highres_256_k144", 1, 8, 256, 256, 64, 12, 12, "bf16", 1.0, 4),
        Workload("highres_256_k256", 1, 8, 256, 256, 64, 16, 16, "bf16", 1.0, 4),
        Workload("highres_256_learnable256", 1, 8, 256, 256, 64, 16, 16, "bf16", 1.0, 4,
                 learnable_agents=256),
    ]
}

# The workload the benchmark times by default: the Stable-Diffusion 1024^2
# latent shape, the larger of the two workloads the HBM-roofline target is
# stated on.
BENCH_WORKLOAD = "sd_latent_1024"


def truncated_normal(shape, std: float, gen: torch.Generator) -> torch.Tensor:
    """N(0, std^2) with every draw outside +-2 std redrawn (float32)."""
    out = torch.randn(shape, generator=gen) * std
    bad = out.abs() > 2 * std
    while bool(bad.any()):
        out[bad] = torch.randn(int(bad.sum()), generator=gen) * std
        bad = out.abs() > 2 * std
    return out


def make_inputs(w: Workload, seed: int | None = None, B: int | None = None) -> dict:
    """Returns CPU tensors q, k, v ([B, H, N, d]) and agents ([H, k, d] or None),
    already cast to the run dtype.  ``B`` overrides the batch (sharding)."""
    gen = torch.Generator().manual_seed(w.seed if seed is None else seed)
    b = w.B if B is None else B
    shape = (b, w.H, w.N, w.d)
    q = torch.randn(shape, generator=gen) * w.value_scale
    k = torch.randn(shape, generator=gen) * w.value_scale
    v = torch.randn(shape, generator=gen) * w.value_scale
    agents = None
    if w.learnable_agents:
        agents = truncated_normal((w.H, w.learnable_agents, w.d), 0.02, gen).to(w.torch_dtype)
    dt = w.torch_dtype
    return {"q": q.to(dt), "k": k.to(dt), "v": v.to(dt), "agents": agents}


def random_qkv(shape, seed: int, dtype: torch.dtype = torch.float32, scale: float = 1.0):
    """Small seeded i.i.d. N(0, scale^2) q, k, v of the given shape (tests)."""
    gen = torch.Generator().manual_seed(seed)
    return tuple((torch.randn(shape, generator=gen) * scale).to(dtype) for _ in range(3))
