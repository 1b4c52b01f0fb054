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
