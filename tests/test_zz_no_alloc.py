"""The allocation-free aggregation entry point.

Some callers may not allocate device memory (a plugin inside a framework that
owns the device memory, a loop that forbids allocation after start-up).  For
them agent_attn_stage_aggregate_static keeps its split partials in a fixed
array inside the library.  This file checks it through the C ABI against the
regular aggregation entry point on the same inputs, on two calls in a row.  It
is collected last so that a failure here cannot hide any other test.
"""
import math

import pytest
import torch

import efficient_vision_attention_b200 as eva
import oracle
from efficient_vision_attention_b200.workloads import random_qkv
from gpu_helpers import assert_close, dtype_code, f64

pytestmark = pytest.mark.gpu


def aggregate(fn, agents, k, v, n_agents, dtype):
    B, H, N, d = k.shape
    va32 = torch.full((B, H, n_agents, d), float("nan"), dtype=torch.float32, device="cuda")
    valow = torch.zeros((B, H, n_agents, d), dtype=dtype, device="cuda")
    fn(agents, H * n_agents * d, k, v, va32, valow, B, H, N, d, n_agents, 1 / math.sqrt(d),
       dtype_code(dtype))
    torch.cuda.synchronize()
    return va32, valow


@pytest.mark.parametrize("dtype,B,H,N,n_agents,d", [
    (torch.bfloat16, 2, 8, 16384, 256, 40),     # the SD-latent aggregation shape
    (torch.bfloat16, 4, 3, 196, 49, 64),
    (torch.float32, 1, 2, 1000, 64, 32),
])
def test_static_scratch_matches_regular_entry_point(dtype, B, H, N, n_agents, d):
    _, k, v = random_qkv((B, H, N, d), seed=N + d, dtype=dtype)
    g = torch.Generator().manual_seed(21)
    agents = (torch.randn((B, H, n_agents, d), generator=g) * 0.5).to(dtype).cuda()
    k, v = k.cuda(), v.cuda()
    ref32, reflow = aggregate(eva.agent_attn_stage_aggregate, agents, k, v, n_agents, dtype)
    want = oracle.agent_aggregate(f64(agents), f64(k), f64(v), 1 / math.sqrt(d))
    for _ in range(2):                     # two calls in a row share the fixed array
        got32, gotlow = aggregate(eva.agent_attn_stage_aggregate_static, agents, k, v,
                                  n_agents, dtype)
        assert_close(f64(got32), f64(ref32), dtype, "static-scratch V_A vs regular call")
        assert_close(f64(got32), want, dtype, "static-scratch V_A vs oracle")
        if dtype != torch.float32:
            # the run-dtype copy feeds the broadcast: the same bits as the
            # regular call's, and the fp32 result rounded once
            assert torch.equal(gotlow, reflow), "static-scratch bf16 V_A differs"
            assert_close(f64(gotlow), want, dtype, "static-scratch bf16 V_A vs oracle")
    assert eva.agent_attn_check_device_error(check=False) == 0


def test_static_scratch_rejects_oversized_problems():
    # 4096 slices x 256 agents x d=128 fp32: at least one partial per slice,
    # 512 MiB, far beyond the fixed array whatever the SM count.  The fake
    # pointers are never dereferenced: the size check precedes any launch.
    B, H, N, d, n_agents = 64, 64, 4096, 128, 256
    status = eva.agent_attn_stage_aggregate_static(
        1 << 20, 0, 1 << 20, 1 << 20, 1 << 20, None, B, H, N, d, n_agents, 0.1, eva.AA_FP32, 0,
        check=False)
    assert status == 5          # AA_ERR_WORKSPACE, before any launch
