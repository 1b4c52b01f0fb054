"""GPU parity of the depth-wise convolution term (the full module's DWC term)
and of the full module output, against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

import efficient_vision_attention_b200 as eva
import oracle
from efficient_vision_attention_b200.workloads import random_qkv
from gpu_helpers import assert_close, dtype_code, f64

pytestmark = pytest.mark.gpu


def dwc_params(H, d, seed, with_bias=True):
    g = torch.Generator().manual_seed(seed)
    w = torch.randn((H, d, 3, 3), generator=g) * 0.3
    b = torch.randn((H, d), generator=g) * 0.1 if with_bias else None
    return w, b


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,H,gh,gw,d", [(2, 3, 7, 9, 8), (1, 2, 1, 17, 16), (1, 1, 13, 1, 32),
                                         (2, 2, 56, 56, 32), (1, 8, 128, 128, 40),
                                         (1, 2, 5, 5, 128), (1, 1, 1, 1, 8),
                                         (1, 2, 9, 50, 128), (2100, 32, 2, 3, 8)])
@pytest.mark.parametrize("with_bias,accumulate", [(True, False), (False, True), (True, True)])
def test_dwc_matches_oracle(dtype, B, H, gh, gw, d, with_bias, accumulate):
    N = gh * gw
    _, _, v = random_qkv((B, H, N, d), seed=N + d, dtype=dtype)
    w, b = dwc_params(H, d, 7, with_bias)
    init = (torch.randn((B, H, N, d), generator=torch.Generator().manual_seed(9))).to(dtype)
    guard = 4096
    fill = float("nan") if dtype == torch.float32 else 12288.0
    buf = torch.full((v.numel() + 2 * guard,), fill, dtype=dtype, device="cuda")
    out = buf[guard:guard + v.numel()].view(B, H, N, d)
    out.copy_(init.cuda())
    eva.agent_attn_dwc(v.cuda(), w.cuda(), None if b is None else b.cuda(), out, B, H, gh, gw, d,
                       dtype_code(dtype), accumulate)
    torch.cuda.synchronize()
    ref = oracle.dwc(f64(v), f64(w), None if b is None else f64(b), gh, gw)
    if accumulate:
        ref = ref + f64(init)
    assert_close(f64(out), ref, dtype, "DWC")
    g = buf.cpu()
    margin = torch.cat([g[:guard], g[guard + v.numel():]]).float()
    if dtype == torch.float32:
        assert torch.isnan(margin).all(), "stray write outside the output"
    else:
        assert (margin == fill).all(), "stray write outside the output"


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,H,gh,gw,ph,pw,d", [(2, 3, 14, 14, 7, 7, 64), (2, 2, 56, 56, 7, 7, 32),
                                               (1, 2, 32, 32, 16, 16, 40)])
def test_full_module_output_matches_oracle(dtype, B, H, gh, gw, ph, pw, d):
    N = gh * gw
    q, k, v = random_qkv((B, H, N, d), seed=3 * N + d, dtype=dtype)
    w, b = dwc_params(H, d, 11)
    out = torch.empty((B, H, N, d), dtype=dtype, device="cuda")
    scale = 1 / math.sqrt(d)
    eva.agent_attn_forward_dwc(q.cuda(), k.cuda(), v.cuda(), None, w.cuda(), b.cuda(), out, B, H,
                               N, d, gh, gw, ph, pw, scale, dtype_code(dtype))
    torch.cuda.synchronize()
    assert eva.agent_attn_check_device_error(check=False) == 0
    ref = oracle.agent_attn_dwc(f64(q), f64(k), f64(v), gh, gw, ph, pw, scale, f64(w), f64(b))
    assert_close(f64(out), ref, dtype, "attention + DWC")


def test_identity_kernel_adds_v_exactly_in_fp32():
    """A unit centre tap and no bias: out = init + V, exactly (one fp32 add)."""
    B, H, gh, gw, d = 1, 2, 9, 11, 16
    _, _, v = random_qkv((B, H, gh * gw, d), seed=5)
    w = torch.zeros((H, d, 3, 3))
    w[:, :, 1, 1] = 1.0
    init = torch.randn((B, H, gh * gw, d), generator=torch.Generator().manual_seed(6))
    out = init.cuda()
    eva.agent_attn_dwc(v.cuda(), w.cuda(), None, out, B, H, gh, gw, d, eva.AA_FP32, True)
    torch.cuda.synchronize()
    assert torch.equal(out.cpu(), init + v)


# The full module output through its own entry point on bf16 shapes that take
# the tensor-core forward pass (the convolution kernel follows it): ragged
# last tiles (N % 128 != 0), tiles spanning many grid rows (narrow grids), a
# single grid row and a single column, grid rows wider than a query tile,
# more tiles than SMs (CTAs crossing slices and heads), d from 8 to 64, k from
# 1 to 256.
@pytest.mark.parametrize("B,H,gh,gw,ph,pw,d", [
    (1, 3, 37, 23, 5, 4, 16),      # N = 851: tiles cross 6 grid rows, ragged tail
    (2, 1, 1, 700, 1, 7, 8),       # one grid row
    (1, 2, 300, 1, 3, 1, 24),      # one grid column: the taps are tokens n-1, n, n+1
    (1, 2, 5, 300, 5, 6, 32),      # grid rows of 300 tokens
    (6, 7, 32, 64, 4, 4, 48),      # 672 tiles: CTAs cross slices and heads
    (6, 7, 32, 64, 4, 4, 64),
    (1, 2, 20, 20, 1, 1, 40),      # k = 1: the attention term is V's mean
    (1, 8, 128, 128, 16, 16, 40),  # the SD-latent slice shape, k = 256
])
def test_full_module_tc_shapes_match_oracle(B, H, gh, gw, ph, pw, d):
    N = gh * gw
    dtype = torch.bfloat16
    q, k, v = random_qkv((B, H, N, d), seed=5 * N + d, dtype=dtype)
    w, b = dwc_params(H, d, 13 + d)
    guard = 4096
    buf = torch.full((q.numel() + 2 * guard,), 12288.0, dtype=dtype, device="cuda")
    out = buf[guard:guard + q.numel()].view(B, H, N, d)
    scale = 1 / math.sqrt(d)
    eva.agent_attn_forward_dwc(q.cuda(), k.cuda(), v.cuda(), None, w.cuda(), b.cuda(), out, B, H,
                               N, d, gh, gw, ph, pw, scale, dtype_code(dtype))
    torch.cuda.synchronize()
    assert eva.agent_attn_check_device_error(check=False) == 0
    ref = oracle.agent_attn_dwc(f64(q), f64(k), f64(v), gh, gw, ph, pw, scale, f64(w), f64(b))
    assert_close(f64(out), ref, dtype, "attention + DWC")
    g = buf.cpu()
    assert (torch.cat([g[:guard], g[guard + q.numel():]]) == 12288.0).all(), \
        "stray write outside the output"


def test_full_module_without_bias_and_with_given_agents():
    """Given agents [H, k, d], no DWC bias: the full module entry point against
    the oracle, and bit for bit against its composition (the forward pass,
    then the DWC kernel accumulating into its output)."""
    B, H, gh, gw, ph, pw, d = 2, 4, 48, 40, 8, 8, 32
    N, nk = gh * gw, ph * pw
    dtype = torch.bfloat16
    q, k, v = random_qkv((B, H, N, d), seed=21, dtype=dtype)
    gen = torch.Generator().manual_seed(22)
    agents = (torch.randn((H, nk, d), generator=gen) * 0.5).to(dtype)
    w, _ = dwc_params(H, d, 23, with_bias=False)
    scale = 1 / math.sqrt(d)
    qd, kd, vd, ad, wd = (t.cuda() for t in (q, k, v, agents, w))
    out = torch.empty((B, H, N, d), dtype=dtype, device="cuda")
    eva.agent_attn_forward_dwc(qd, kd, vd, ad, wd, None, out, B, H, N, d, gh, gw, ph, pw, scale,
                               dtype_code(dtype))
    two = torch.empty_like(out)
    eva.agent_attn_forward(qd, kd, vd, ad, two, B, H, N, d, gh, gw, ph, pw, scale,
                           dtype_code(dtype))
    eva.agent_attn_dwc(vd, wd, None, two, B, H, gh, gw, d, dtype_code(dtype), True)
    torch.cuda.synchronize()
    ref = oracle.agent_attn_dwc(f64(q), f64(k), f64(v), gh, gw, ph, pw, scale, f64(w), None,
                                agents=f64(agents))
    assert_close(f64(out), ref, dtype, "attention + DWC, given agents")
    assert torch.equal(out, two)
