"""GPU parity of the backward pass (dQ, dK, dV and the agents' gradient)
against the fp64 oracle's derivatives."""
import math

import numpy as np
import pytest
import torch

import efficient_vision_attention_b200 as eva
import oracle
from efficient_vision_attention_b200.workloads import random_qkv
from gpu_helpers import dtype_code, f64

pytestmark = pytest.mark.gpu


def close(got, want, dtype, what):
    assert np.isfinite(got).all(), f"{what}: non-finite"
    den = np.linalg.norm(want)
    rel = np.linalg.norm(got - want) / den if den > 0 else np.linalg.norm(got - want)
    lim_rel = 1e-5 if dtype == torch.float32 else 1e-2
    scale = np.abs(want).max() if want.size else 1.0
    lim_abs = (1e-5 if dtype == torch.float32 else 2e-2) * max(1.0, scale)
    err = np.abs(got - want).max()
    assert rel <= lim_rel and err <= lim_abs, f"{what}: rel-L2 {rel:.2e}, max-abs {err:.2e}"


def run_backward(q, k, v, dout, gh, gw, ph, pw, scale, agents=None):
    B, H, N, d = q.shape
    dev = "cuda"
    dq, dk, dv = (torch.empty_like(q, device=dev) for _ in range(3))
    da = torch.empty((B, H, ph * pw, d), dtype=torch.float32, device=dev)
    eva.agent_attn_backward(q.to(dev), k.to(dev), v.to(dev),
                            None if agents is None else agents.to(dev), dout.to(dev), dq, dk, dv,
                            da, B, H, N, d, gh, gw, ph, pw, scale, dtype_code(q.dtype))
    torch.cuda.synchronize()
    assert eva.agent_attn_check_device_error(check=False) == 0
    return dq, dk, dv, da


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,H,gh,gw,ph,pw,d", [(1, 1, 8, 8, 2, 2, 32), (2, 3, 14, 14, 7, 7, 64),
                                               (1, 2, 13, 11, 4, 3, 40), (1, 1, 32, 32, 16, 16, 16),
                                               (1, 2, 9, 20, 1, 1, 8), (1, 1, 12, 12, 3, 3, 128),
                                               (1, 1, 50, 37, 12, 9, 16)])
def test_backward_matches_oracle(dtype, B, H, gh, gw, ph, pw, d):
    N = gh * gw
    q, k, v = random_qkv((B, H, N, d), seed=N + 7 * d, dtype=dtype)
    dout = (torch.randn((B, H, N, d), generator=torch.Generator().manual_seed(3))).to(dtype)
    scale = 1 / math.sqrt(d)
    dq, dk, dv, da = run_backward(q, k, v, dout, gh, gw, ph, pw, scale)
    rq, rk, rv, ra = oracle.agent_attn_backward(f64(q), f64(k), f64(v), f64(dout), gh, gw, ph, pw,
                                                scale)
    for got, want, name in ((dq, rq, "dQ"), (dk, rk, "dK"), (dv, rv, "dV"), (da, ra, "dA")):
        close(f64(got), want, dtype, name)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_backward_with_given_agents(dtype):
    B, H, gh, gw, ph, pw, d = 2, 2, 16, 16, 8, 8, 32
    N = gh * gw
    q, k, v = random_qkv((B, H, N, d), seed=11, dtype=dtype)
    agents = (torch.randn((H, ph * pw, d), generator=torch.Generator().manual_seed(12)) * 0.5).to(dtype)
    dout = torch.randn((B, H, N, d), generator=torch.Generator().manual_seed(13)).to(dtype)
    scale = 1 / math.sqrt(d)
    dq, dk, dv, da = run_backward(q, k, v, dout, gh, gw, ph, pw, scale, agents=agents)
    rq, rk, rv, ra = oracle.agent_attn_backward(f64(q), f64(k), f64(v), f64(dout), gh, gw, ph, pw,
                                                scale, agents=f64(agents))
    for got, want, name in ((dq, rq, "dQ"), (dk, rk, "dK"), (dv, rv, "dV"), (da, ra, "dA")):
        close(f64(got), want, dtype, name)


def test_backward_at_the_sd_latent_size():
    """The bench's backward configuration (2 x 8 slices, N = 16384 on a
    128 x 128 grid, k = 256 pooled agents, d = 40, bf16): the gradient sums over
    16384 keys and the per-agent accumulation over 128 query tiles differ most
    from the small cases; three whole slices are compared with the oracle."""
    from efficient_vision_attention_b200.workloads import WORKLOADS, make_inputs
    w = WORKLOADS["sd_latent_1024"]
    inp = make_inputs(w)
    q, k, v = inp["q"], inp["k"], inp["v"]
    dout = torch.randn(q.shape, generator=torch.Generator().manual_seed(5)).to(q.dtype)
    dq, dk, dv, da = run_backward(q, k, v, dout, w.grid_h, w.grid_w, w.pool_h, w.pool_w,
                                  w.scale)
    for (b, h) in ((0, 0), (0, 7), (1, 3)):
        sl = lambda t: f64(t[b:b + 1, h:h + 1])
        rq, rk, rv, ra = oracle.agent_attn_backward(sl(q), sl(k), sl(v), sl(dout), w.grid_h,
                                                    w.grid_w, w.pool_h, w.pool_w, w.scale)
        for got, want, name in ((dq, rq, "dQ"), (dk, rk, "dK"), (dv, rv, "dV"), (da, ra, "dA")):
            close(sl(got), want, q.dtype, f"{name} slice ({b}, {h})")
