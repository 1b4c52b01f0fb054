"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare it with the fp64 oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import efficient_vision_attention_b200 as eva
import oracle

BF16_MAX_ABS = 2e-2     # bf16 inputs, fp32 accumulate
BF16_REL_L2 = 5e-3
FP32_MAX_ABS = 1e-5


def dtype_code(t: torch.dtype) -> int:
    return eva.AA_FP32 if t == torch.float32 else eva.AA_BF16


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def errors(gpu: np.ndarray, ref: np.ndarray) -> tuple[float, float]:
    diff = gpu.astype(np.float64) - ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(diff)) / den if den > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_close(gpu: np.ndarray, ref: np.ndarray, dtype: torch.dtype, what: str = "",
                 max_abs: float | None = None, rel_l2: float | None = None):
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    ma, rl = errors(gpu, ref)
    if dtype == torch.float32:
        lim_a = FP32_MAX_ABS if max_abs is None else max_abs
        assert ma <= lim_a, f"{what}: max-abs {ma:.3e} > {lim_a:.1e} (rel-L2 {rl:.3e})"
        if rel_l2 is not None:
            assert rl <= rel_l2, f"{what}: rel-L2 {rl:.3e} > {rel_l2:.1e}"
    else:
        lim_a = BF16_MAX_ABS if max_abs is None else max_abs
        lim_r = BF16_REL_L2 if rel_l2 is None else rel_l2
        assert ma <= lim_a and rl <= lim_r, \
            f"{what}: max-abs {ma:.3e} (<= {lim_a:.1e}), rel-L2 {rl:.3e} (<= {lim_r:.1e})"
    return ma, rl


def run_forward(q, k, v, grid_h, grid_w, pool_h, pool_w, scale, agents=None, guard=0):
    """Pooled-agents forward on the GPU; q/k/v CPU tensors [B, H, N, d].
    With guard > 0 the output sits inside a larger buffer whose margins are
    checked for stray writes.  Returns the output as a CPU tensor."""
    B, H, N, d = q.shape
    dev = torch.device("cuda")
    qd, kd, vd = (t.to(dev).contiguous() for t in (q, k, v))
    ad = agents.to(dev).contiguous() if agents is not None else None
    n = q.numel()
    fill = float("nan") if q.dtype == torch.float32 else 12288.0   # exact in bf16
    buf = torch.full((n + 2 * guard,), fill, dtype=q.dtype, device=dev)
    out = buf[guard:guard + n].view(B, H, N, d)
    eva.agent_attn_forward(qd, kd, vd, ad, out, B, H, N, d, grid_h, grid_w, pool_h, pool_w,
                           scale, dtype_code(q.dtype))
    torch.cuda.synchronize()
    eva.agent_attn_check_device_error()          # raises if an in-kernel wait timed out
    if guard:
        g = torch.cat([buf[:guard], buf[guard + n:]]).cpu().float()
        if q.dtype == torch.float32:
            assert torch.isnan(g).all(), "stray write into the guard band"
        else:
            assert (g == 12288.0).all(), "stray write into the guard band"
    return out.cpu()


def run_forward_agents(q, k, v, agents, scale, batch_stride=0):
    B, H, N, d = q.shape
    dev = torch.device("cuda")
    qd, kd, vd, ad = (t.to(dev).contiguous() for t in (q, k, v, agents))
    out = torch.empty_like(qd)
    eva.agent_attn_forward_agents(qd, kd, vd, ad, agents.shape[-2], batch_stride, out, B, H, N, d,
                                  scale, dtype_code(q.dtype))
    torch.cuda.synchronize()
    eva.agent_attn_check_device_error()
    return out.cpu()


def oracle_slices(q, k, v, grid_h, grid_w, pool_h, pool_w, scale, slices, agents=None):
    """Oracle output for the (b, h) slices listed, as [len(slices), N, d]."""
    outs = []
    for (b, h) in slices:
        ag = None
        if agents is not None:
            ag = f64(agents[h] if agents.dim() == 3 else agents[b, h])[None]
        outs.append(oracle.agent_attn(f64(q[b, h])[None], f64(k[b, h])[None], f64(v[b, h])[None],
                                      grid_h, grid_w, pool_h, pool_w, scale, agents=ag)[0])
    return np.stack(outs)
