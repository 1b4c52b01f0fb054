"""GPU parity of the forward pass with agent bias (row, column and block
components in both softmaxes) against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import efficient_vision_attention_b200 as eva
import oracle
from efficient_vision_attention_b200.workloads import random_qkv
from gpu_helpers import assert_close, dtype_code, f64

pytestmark = pytest.mark.gpu


def parts(H, k, gh, gw, seed, scale=0.5, drop=()):
    g = torch.Generator().manual_seed(seed)
    out = []
    for name, n in (("row", gh), ("col", gw), ("block", k)):
        t = torch.randn((H, k, n), generator=g) * scale
        out.append(None if name in drop else t)
    return out


def run(q, k, v, gh, gw, ph, pw, scale, b1, b2, dtype):
    B, H, N, d = q.shape
    out = torch.empty((B, H, N, d), dtype=dtype, device="cuda")
    dev = lambda t: None if t is None else t.cuda()
    eva.agent_attn_forward_bias(q.cuda(), k.cuda(), v.cuda(), None,
                                None if b1 is None else [dev(t) for t in b1],
                                None if b2 is None else [dev(t) for t in b2], out, B, H, N, d,
                                gh, gw, ph, pw, scale, dtype_code(dtype))
    torch.cuda.synchronize()
    return out


def full(b, gh, gw, ph, pw):
    if b is None:
        return None
    return oracle.agent_bias(*[None if t is None else f64(t) for t in b], gh, gw, ph, pw)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,H,gh,gw,ph,pw,d", [(2, 2, 8, 8, 2, 2, 32), (2, 3, 14, 14, 7, 7, 64),
                                               (1, 2, 32, 32, 8, 8, 40), (1, 2, 13, 11, 4, 3, 16)])
@pytest.mark.parametrize("drop1,drop2", [((), ()), (("col",), ("row", "block")),
                                         (("row", "col", "block"), ())])
def test_bias_matches_oracle(dtype, B, H, gh, gw, ph, pw, d, drop1, drop2):
    N, k = gh * gw, ph * pw
    q, kk, v = random_qkv((B, H, N, d), seed=N + d, dtype=dtype)
    b1 = parts(H, k, gh, gw, 21, drop=drop1)
    b2 = parts(H, k, gh, gw, 22, drop=drop2)
    b1 = None if all(t is None for t in b1) else b1
    scale = 1 / math.sqrt(d)
    out = run(q, kk, v, gh, gw, ph, pw, scale, b1, b2, dtype)
    ref = oracle.agent_attn_bias(f64(q), f64(kk), f64(v), gh, gw, ph, pw, scale,
                                 full(b1, gh, gw, ph, pw), full(b2, gh, gw, ph, pw))
    assert_close(f64(out), ref, dtype, "biased O")


@pytest.mark.parametrize("dtype,mask", [(torch.float32, -1e4), (torch.bfloat16, -1e4),
                                        (torch.bfloat16, -1e6)])
def test_bias_admitting_one_token_selects_its_value_on_gpu(dtype, mask):
    """B1 = mask everywhere but one token: every agent's V_A is that token's
    V row, and so is every output row.  bf16 holds B1 * log2(e) in fp16: -1e4
    components (sum -2e4) lie inside its range, -1e6 saturate at -65504 and
    still give the admitted token all the weight."""
    gh, gw, ph, pw, d, ys, xs = 9, 7, 3, 3, 16, 4, 2
    q, kk, v = random_qkv((1, 2, gh * gw, d), seed=3, dtype=dtype)
    row = torch.full((2, 9, gh), mask)
    row[:, :, ys] = 0.0
    col = torch.full((2, 9, gw), mask)
    col[:, :, xs] = 0.0
    out = run(q, kk, v, gh, gw, ph, pw, 0.25, [row, col, None], parts(2, 9, gh, gw, 5), dtype)
    want = v[:, :, ys * gw + xs][:, :, None, :].expand_as(out.cpu())
    atol = 1e-6 if dtype == torch.float32 else 1e-2
    assert torch.allclose(out.cpu().float(), want.float(), atol=atol, rtol=0)


def test_bias_at_the_sd_latent_size_on_sampled_slices():
    """The SD-latent workload (B=2, H=8, N=16384, d=40, k=256) with all six bias
    components, checked on two sampled (b, h) slices."""
    from efficient_vision_attention_b200.workloads import WORKLOADS, make_inputs
    w = WORKLOADS["sd_latent_1024"]
    inp = make_inputs(w)
    q, kk, v = inp["q"], inp["k"], inp["v"]
    b1 = parts(w.H, w.n_agents, w.grid_h, w.grid_w, 31)
    b2 = parts(w.H, w.n_agents, w.grid_h, w.grid_w, 32)
    out = run(q, kk, v, w.grid_h, w.grid_w, w.pool_h, w.pool_w, w.scale, b1, b2, w.torch_dtype)
    for (b, h) in [(0, 0), (1, 7)]:
        sl = lambda t: t[b:b + 1, h:h + 1]
        hb = lambda trip: [t[h:h + 1] for t in trip]
        ref = oracle.agent_attn_bias(f64(sl(q)), f64(sl(kk)), f64(sl(v)), w.grid_h, w.grid_w,
                                     w.pool_h, w.pool_w, w.scale,
                                     full(hb(b1), w.grid_h, w.grid_w, w.pool_h, w.pool_w),
                                     full(hb(b2), w.grid_h, w.grid_w, w.pool_h, w.pool_w))
        assert_close(f64(out[b, h]), ref[0, 0], w.torch_dtype, f"biased O slice {(b, h)}")


@pytest.mark.parametrize("dtype", [torch.bfloat16])
def test_bias_with_a_column_component_on_a_4_byte_boundary(dtype):
    """A column component that starts 4 bytes past an 8-byte boundary (the
    boundary the entry point accepts) reads correctly."""
    B, H, gh, gw, ph, pw, d = 1, 2, 16, 16, 4, 4, 32
    N, k = gh * gw, ph * pw
    q, kk, v = random_qkv((B, H, N, d), seed=5, dtype=dtype)
    b1 = parts(H, k, gh, gw, 31)
    b2 = parts(H, k, gh, gw, 32)
    col = b1[1]
    buf = torch.zeros(col.numel() + 1, device="cuda")
    shifted = buf[1:].view(col.shape)
    shifted.copy_(col.cuda())
    assert shifted.data_ptr() % 8 == 4
    out = torch.empty((B, H, N, d), dtype=dtype, device="cuda")
    eva.agent_attn_forward_bias(q.cuda(), kk.cuda(), v.cuda(), None,
                                [b1[0].cuda(), shifted, b1[2].cuda()],
                                [t.cuda() for t in b2], out, B, H, N, d, gh, gw, ph, pw,
                                1 / math.sqrt(d), dtype_code(dtype))
    torch.cuda.synchronize()
    ref = oracle.agent_attn_bias(f64(q), f64(kk), f64(v), gh, gw, ph, pw, 1 / math.sqrt(d),
                                 full(b1, gh, gw, ph, pw), full(b2, gh, gw, ph, pw))
    assert_close(f64(out), ref, dtype, "biased O")


def test_bias_on_a_grid_wider_than_4096_tokens():
    """A 2 x 4100 grid (8200 tokens, 1 x 4 agent cells, odd cell widths of
    1025 tokens) takes the tensor-core kernels with the dense bias copies; the
    B1 rows (8200 tokens) and B2 rows (4 agents, padded to 16) end mid-tile."""
    B, H, gh, gw, ph, pw, d = 1, 2, 2, 4100, 1, 4, 16
    N = gh * gw
    q, kk, v = random_qkv((B, H, N, d), seed=9, dtype=torch.bfloat16)
    b1 = parts(H, ph * pw, gh, gw, 41)
    b2 = parts(H, ph * pw, gh, gw, 42)
    out = run(q, kk, v, gh, gw, ph, pw, 1 / math.sqrt(d), b1, b2, torch.bfloat16)
    ref = oracle.agent_attn_bias(f64(q), f64(kk), f64(v), gh, gw, ph, pw, 1 / math.sqrt(d),
                                 full(b1, gh, gw, ph, pw), full(b2, gh, gw, ph, pw))
    assert_close(f64(out), ref, torch.bfloat16, "biased O")
