"""The exponential the tensor-core softmax kernels take on the FMA pipe for
part of each score row (Cody-Waite split plus a fitted degree-3 polynomial,
tc_primitives.cuh) against CUDA's exp2f: relative error at most 1e-4 over the
arguments the kernels produce (x <= 8; below -125 the result is about 2^-125,
negligible against the row maximum's weight of 1)."""
import numpy as np
import pytest
import torch

import efficient_vision_attention_b200 as eva

pytestmark = pytest.mark.gpu


def run(x: torch.Tensor):
    x = x.cuda().contiguous()
    y_fma = torch.empty_like(x)
    y_ref = torch.empty_like(x)
    eva.agent_attn_selftest_exp2(x, y_fma, y_ref, x.numel())
    torch.cuda.synchronize()
    return y_fma.cpu().double().numpy(), y_ref.cpu().double().numpy()


def test_fma_exp2_matches_exp2f():
    x = torch.cat([torch.linspace(-125.0, 8.0, 4_000_001),
                   torch.linspace(-1.0, 1.0, 200_001),            # around 2^0 and the f split
                   torch.arange(-125, 9, dtype=torch.float32) + 0.5,
                   torch.arange(-125, 9, dtype=torch.float32)])
    y, ref = run(x)
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= 1e-4, f"max relative error {rel.max():.3e} at x = {x[rel.argmax()]}"


def test_fma_exp2_of_masked_scores_is_negligible():
    x = torch.tensor([-float("inf"), -1e30, -500.0, -126.0, -125.5], dtype=torch.float32)
    y, ref = run(x)
    assert np.isfinite(y).all() and (y >= 0).all()
    assert (y <= 2.0 ** -124).all()
