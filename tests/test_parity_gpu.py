"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.  bf16: max-abs <= 2e-2 and rel-L2 <= 5e-3; fp32: max-abs
<= 1e-5.  Full-size workloads compare whole (b, h) slices the oracle can
evaluate in seconds (every slice of every workload); smaller cases compare
every output."""
import math

import numpy as np
import pytest
import torch

import efficient_vision_attention_b200 as eva
import oracle
from efficient_vision_attention_b200.workloads import WORKLOADS, make_inputs, random_qkv
from gpu_helpers import (assert_close, dtype_code, f64, oracle_slices, run_forward,
                         run_forward_agents)

pytestmark = pytest.mark.gpu


def sample_slices(B, H, max_slices):
    all_s = [(b, h) for b in range(B) for h in range(H)]
    if len(all_s) <= max_slices:
        return all_s
    rng = np.random.default_rng(7)
    pick = {0, len(all_s) - 1}
    while len(pick) < max_slices:
        pick.add(int(rng.integers(len(all_s))))
    return [all_s[i] for i in sorted(pick)]


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_workload_matches_oracle(name):
    w = WORKLOADS[name]
    inp = make_inputs(w)
    q, k, v, agents = inp["q"], inp["k"], inp["v"], inp["agents"]
    if agents is None:
        out = run_forward(q, k, v, w.grid_h, w.grid_w, w.pool_h, w.pool_w, w.scale, guard=4096)
    else:
        out = run_forward_agents(q, k, v, agents, w.scale)
    # every (b, h) slice: the tensor-core aggregation gives each slice its own
    # split count and partial slots, so a scheduling or merge error can hit any
    slices = [(b, h) for b in range(w.B) for h in range(w.H)]
    ref = oracle_slices(q, k, v, w.grid_h, w.grid_w, w.pool_h, w.pool_w, w.scale, slices,
                        agents=agents)
    got = np.stack([f64(out[b, h]) for (b, h) in slices])
    assert_close(got, ref, w.torch_dtype, name)


@pytest.mark.parametrize("B,H,gh,gw,ph,pw,d", [
    (4, 3, 14, 14, 7, 7, 64),      # DeiT-shaped slices: N = 196, k = 49
    (2, 2, 13, 11, 4, 3, 40),      # N = 143, overlapping bins, d = 40
    (1, 3, 9, 20, 1, 1, 8),        # one agent, d = 8
    (2, 1, 16, 16, 16, 8, 64),     # k = 128 (the tile), N = 256 (the limit)
    (3, 2, 10, 10, 10, 10, 32),    # k = N = 100: every token an agent
    (1, 2, 7, 7, 3, 3, 16),        # N = 49, bins 3x3 over 7 tokens
    (5, 1, 12, 15, 5, 4, 24),      # N = 180, k = 20, non-dividing bins
])
def test_fused_small_slices_match_oracle(B, H, gh, gw, ph, pw, d):
    """bf16 slices of at most 256 tokens with at most 128 pooled agents and
    d <= 64 run the whole pass in one CTA per slice (agent_fused_small_tc):
    every output against the oracle, and twice in a row bit-identical."""
    N = gh * gw
    q, k, v = random_qkv((B, H, N, d), seed=3 * N + d, dtype=torch.bfloat16)
    scale = 1 / math.sqrt(d)
    out = run_forward(q, k, v, gh, gw, ph, pw, scale, guard=1024)
    again = run_forward(q, k, v, gh, gw, ph, pw, scale, guard=1024)
    assert torch.equal(out, again)
    ref = oracle.agent_attn(f64(q), f64(k), f64(v), gh, gw, ph, pw, scale)
    assert_close(f64(out), ref, torch.bfloat16, f"{B}x{H} {gh}x{gw}->{ph}x{pw} d={d}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,H,gh,gw,ph,pw,d", [
    (1, 1, 8, 8, 2, 2, 32),        # tiny
    (2, 3, 13, 11, 4, 3, 40),      # ragged N = 143, overlapping bins
    (1, 2, 9, 20, 1, 1, 16),       # one agent
    (1, 1, 16, 16, 16, 16, 64),    # k = N = 256 (every token an agent)
    (3, 1, 33, 7, 5, 7, 8),        # d = 8
    (1, 2, 12, 12, 3, 3, 128),     # d = 128
    (2, 1, 40, 40, 12, 12, 64),    # k = 144
    (1, 1, 64, 64, 16, 16, 48),    # k = 256, N = 4096
    (1, 1, 1, 300, 1, 7, 24),      # a 1-row grid
])
def test_shapes_and_edges(dtype, B, H, gh, gw, ph, pw, d):
    N = gh * gw
    q, k, v = random_qkv((B, H, N, d), seed=N + d, dtype=dtype)
    scale = 1 / math.sqrt(d)
    out = run_forward(q, k, v, gh, gw, ph, pw, scale, guard=1024)
    ref = oracle.agent_attn(f64(q), f64(k), f64(v), gh, gw, ph, pw, scale)
    assert_close(f64(out), ref, dtype, f"{B}x{H} {gh}x{gw}->{ph}x{pw} d={d}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_stage_pool(dtype):
    B, H, gh, gw, d = 2, 3, 56, 56, 32
    # uniform bins (8x8, 4x4, 14x1, 7x8 tokens) take the band kernel for bf16;
    # the others the staged kernel
    for ph, pw in [(7, 7), (12, 5), (16, 16), (1, 1), (3, 56), (14, 14), (4, 56), (8, 7)]:
        q, _, _ = random_qkv((B, H, gh * gw, d), seed=ph * 31 + pw, dtype=dtype)
        qd = q.cuda()
        a32 = torch.empty((B, H, ph * pw, d), dtype=torch.float32, device="cuda")
        alow = torch.empty((B, H, ph * pw, d), dtype=dtype, device="cuda")
        eva.agent_attn_stage_pool(qd, a32, alow, B, H, gh * gw, d, gh, gw, ph, pw,
                                  dtype_code(dtype))
        torch.cuda.synchronize()
        ref = oracle.agent_pool(f64(q), gh, gw, ph, pw)
        np.testing.assert_allclose(f64(a32), ref, rtol=0, atol=2e-6)
        if dtype == torch.bfloat16:
            # the kernel rounds its fp32 mean to bf16; the exact mean rounded to
            # bf16 can land one bf16 ulp (2^-7 relative at most) away
            np.testing.assert_allclose(f64(alow), f64(torch.from_numpy(ref).to(dtype)),
                                       rtol=2 ** -7, atol=1e-6)


@pytest.mark.parametrize("gh,gw,ph,pw,d", [(128, 128, 16, 16, 40), (256, 256, 16, 16, 64),
                                         (14, 14, 7, 7, 64), (48, 96, 3, 32, 8),
                                         (256, 256, 8, 8, 64), (120, 40, 2, 5, 16)])
def test_stage_pool_uniform_bins(gh, gw, ph, pw, d):
    """Grids that the bins divide exactly (the band kernel for bf16): the SD
    latent, high-res (16- and 32-row bins), DeiT shapes, one with 16x3-token
    bins and d = 8 and one with 60-row bins (four batches of row loads)."""
    B, H = 2, 3
    q, _, _ = random_qkv((B, H, gh * gw, d), seed=gh + pw + d, dtype=torch.bfloat16)
    a32 = torch.empty((B, H, ph * pw, d), dtype=torch.float32, device="cuda")
    alow = torch.empty((B, H, ph * pw, d), dtype=torch.bfloat16, device="cuda")
    eva.agent_attn_stage_pool(q.cuda(), a32, alow, B, H, gh * gw, d, gh, gw, ph, pw, eva.AA_BF16)
    torch.cuda.synchronize()
    ref = oracle.agent_pool(f64(q), gh, gw, ph, pw)
    np.testing.assert_allclose(f64(a32), ref, rtol=0, atol=2e-6)
    np.testing.assert_allclose(f64(alow), f64(torch.from_numpy(ref).to(torch.bfloat16)),
                               rtol=2 ** -7, atol=1e-6)


@pytest.mark.parametrize("gh,gw,ph,pw,d", [(256, 256, 12, 12, 64), (128, 16, 2, 3, 24),
                                         (50, 37, 12, 9, 16), (3, 300, 3, 7, 8),
                                         (130, 20, 2, 3, 8)])
def test_stage_pool_adaptive_bins(gh, gw, ph, pw, d):
    """Bins that do not divide the grid (adaptive bounds, neighbours sharing a
    token row or column): the high-res 256/12 shape (21-22-token bins), 64-row
    bins (the band kernel's limit) with overlapping columns, many small
    overlapping bins, one-row bins, and 65-row bins (past the band kernel's
    limit: the fallback kernel)."""
    B, H = 2, 2
    q, _, _ = random_qkv((B, H, gh * gw, d), seed=gh * pw + d, dtype=torch.bfloat16)
    a32 = torch.empty((B, H, ph * pw, d), dtype=torch.float32, device="cuda")
    alow = torch.empty((B, H, ph * pw, d), dtype=torch.bfloat16, device="cuda")
    eva.agent_attn_stage_pool(q.cuda(), a32, alow, B, H, gh * gw, d, gh, gw, ph, pw, eva.AA_BF16)
    torch.cuda.synchronize()
    ref = oracle.agent_pool(f64(q), gh, gw, ph, pw)
    np.testing.assert_allclose(f64(a32), ref, rtol=0, atol=2e-6)
    np.testing.assert_allclose(f64(alow), f64(torch.from_numpy(ref).to(torch.bfloat16)),
                               rtol=2 ** -7, atol=1e-6)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N,n_agents,d", [(3136, 49, 32), (1000, 256, 40), (196, 49, 64),
                                          (4100, 144, 64), (77, 3, 16)])
def test_stage_aggregate(dtype, N, n_agents, d):
    B, H = 2, 2
    q, k, v = random_qkv((B, H, N, d), seed=N + n_agents, dtype=dtype)
    agents = (torch.randn((B, H, n_agents, d), generator=torch.Generator().manual_seed(5)) * 0.5)
    agents = agents.to(dtype)
    va32 = torch.empty((B, H, n_agents, d), dtype=torch.float32, device="cuda")
    valow = torch.empty((B, H, n_agents, d), dtype=dtype, device="cuda")
    scale = 1 / math.sqrt(d)
    eva.agent_attn_stage_aggregate(agents.cuda(), H * n_agents * d, k.cuda(), v.cuda(), va32,
                                   valow, B, H, N, d, n_agents, scale, dtype_code(dtype))
    torch.cuda.synchronize()
    ref = oracle.agent_aggregate(f64(agents), f64(k), f64(v), scale)
    assert_close(f64(va32), ref, dtype, "V_A")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("N,n_agents,d", [(3136, 49, 32), (1000, 256, 40), (300, 144, 64),
                                          (129, 1, 16)])
def test_stage_broadcast(dtype, N, n_agents, d):
    B, H = 2, 2
    q, _, _ = random_qkv((B, H, N, d), seed=N * 3 + n_agents, dtype=dtype)
    g = torch.Generator().manual_seed(11)
    agents = torch.randn((H, n_agents, d), generator=g).to(dtype)      # shared over B
    va = torch.randn((B, H, n_agents, d), generator=g).to(dtype)
    out = torch.empty((B, H, N, d), dtype=dtype, device="cuda")
    scale = 1 / math.sqrt(d)
    eva.agent_attn_stage_broadcast(q.cuda(), agents.cuda(), 0, va.cuda(), out, B, H, N, d,
                                   n_agents, scale, dtype_code(dtype))
    torch.cuda.synchronize()
    ag = np.broadcast_to(f64(agents)[None], (B, H, n_agents, d))
    ref = oracle.agent_broadcast(f64(q), ag, f64(va), scale)
    assert_close(f64(out.cpu()), ref, dtype, "O")


@pytest.mark.parametrize("B,H,N,n_agents,d", [(16, 2, 3136, 49, 32), (2, 4, 8192, 144, 64),
                                              (2, 8, 16384, 256, 40), (64, 3, 196, 49, 64)])
def test_tensor_core_stages_are_repeatable(B, H, N, n_agents, d):
    """Repeated launches of the bf16 aggregation and broadcast give bit-identical
    results: many key tiles per CTA, agent counts that leave some softmax warps
    without rows (49, 144) and both agent-tile modes.  A missing dependency
    between the softmax warps, the MMA issuers and the TMEM buffers shows up
    as run-to-run drift even when each run stays inside the tolerance."""
    q, k, v = (t.cuda() for t in random_qkv((B, H, N, d), seed=N + d, dtype=torch.bfloat16))
    g = torch.Generator().manual_seed(17)
    agents = (torch.randn((B, H, n_agents, d), generator=g) * 0.5).to(torch.bfloat16).cuda()
    scale = 1 / math.sqrt(d)
    vas, outs = [], []
    for _ in range(6):
        va = torch.full((B, H, n_agents, d), 3.0, dtype=torch.bfloat16, device="cuda")
        eva.agent_attn_stage_aggregate(agents, H * n_agents * d, k, v, None, va, B, H, N, d,
                                       n_agents, scale, eva.AA_BF16)
        out = torch.full_like(q, 3.0)
        eva.agent_attn_stage_broadcast(q, agents, H * n_agents * d, va, out, B, H, N, d,
                                       n_agents, scale, eva.AA_BF16)
        torch.cuda.synchronize()
        vas.append(va)
        outs.append(out)
    assert eva.agent_attn_check_device_error(check=False) == 0
    for r in range(1, 6):
        assert torch.equal(vas[r], vas[0]), f"V_A differs in run {r}"
        assert torch.equal(outs[r], outs[0]), f"O differs in run {r}"


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_learnable_agents_batch_stride_and_permutation(dtype):
    B, H, gh, gw, d, n_ag = 2, 2, 20, 20, 32, 40
    q, k, v = random_qkv((B, H, gh * gw, d), seed=3, dtype=dtype)
    agents = (torch.randn((B, H, n_ag, d), generator=torch.Generator().manual_seed(4)) * 0.3)
    agents = agents.to(dtype)
    scale = 1 / math.sqrt(d)
    out = run_forward_agents(q, k, v, agents, scale, batch_stride=H * n_ag * d)
    ref = oracle.agent_attn(f64(q), f64(k), f64(v), gh, gw, 1, 1, scale, agents=f64(agents))
    assert_close(f64(out), ref, dtype, "per-batch agents")
    perm = torch.randperm(n_ag, generator=torch.Generator().manual_seed(6))
    out_p = run_forward_agents(q, k, v, agents[:, :, perm].contiguous(), scale,
                               batch_stride=H * n_ag * d)
    assert_close(f64(out_p), ref, dtype, "permuted agents")


@pytest.mark.parametrize("shared", [True, False])
@pytest.mark.parametrize("N,n_ag,d", [(196, 49, 64), (143, 100, 40), (256, 128, 16)])
def test_fused_small_slices_with_given_agents(shared, N, n_ag, d):
    """Small bf16 slices with learnable agents (shared over the batch, or one
    set per batch through the batch stride) also run as the one-kernel pass:
    every output against the oracle."""
    B, H = 2, 3
    q, k, v = random_qkv((B, H, N, d), seed=N + n_ag, dtype=torch.bfloat16)
    g = torch.Generator().manual_seed(N + 1)
    if shared:
        agents = (torch.randn((H, n_ag, d), generator=g) * 0.3).to(torch.bfloat16)
        out = run_forward_agents(q, k, v, agents, 1 / math.sqrt(d), batch_stride=0)
        ag_ref = agents.unsqueeze(0).expand(B, H, n_ag, d)
    else:
        agents = (torch.randn((B, H, n_ag, d), generator=g) * 0.3).to(torch.bfloat16)
        out = run_forward_agents(q, k, v, agents, 1 / math.sqrt(d), batch_stride=H * n_ag * d)
        ag_ref = agents
    ref = oracle.agent_attn(f64(q), f64(k), f64(v), N, 1, 1, 1, 1 / math.sqrt(d),
                            agents=f64(ag_ref.contiguous()))
    assert_close(f64(out), ref, torch.bfloat16, f"given agents N={N} k={n_ag} d={d}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_joint_key_value_permutation(dtype):
    B, H, gh, gw, d = 1, 2, 30, 30, 64
    q, k, v = random_qkv((B, H, gh * gw, d), seed=8, dtype=dtype)
    perm = torch.randperm(gh * gw, generator=torch.Generator().manual_seed(9))
    o1 = run_forward(q, k, v, gh, gw, 5, 5, 0.125)
    o2 = run_forward(q, k[:, :, perm], v[:, :, perm], gh, gw, 5, 5, 0.125)
    assert_close(f64(o2), f64(o1).astype(np.float64), dtype, "K/V permutation",
                 max_abs=1e-5 if dtype == torch.float32 else 2e-2)


def test_sharp_logits_fp32():
    """Scale 1 and inputs x4: peaked softmaxes exercise the running max and the
    log-sum-exp merge across splits."""
    B, H, gh, gw, d = 1, 2, 40, 40, 32
    q, k, v = random_qkv((B, H, gh * gw, d), seed=12, scale=4.0)
    out = run_forward(q, k, v, gh, gw, 4, 4, 1.0)
    ref = oracle.agent_attn(f64(q), f64(k), f64(v), gh, gw, 4, 4, 1.0)
    assert_close(f64(out), ref, torch.float32, "sharp fp32", max_abs=2e-4)


def test_sharp_logits_bf16_same_agents():
    """bf16 with peaked softmaxes.  Rounding pooled agents to bf16 moves logits in
    the thousands by whole units, so both sides take the same bf16 agents
    (oracle pool, rounded) through the learnable-agents entry point."""
    B, H, gh, gw, d = 1, 2, 48, 48, 64
    q, k, v = random_qkv((B, H, gh * gw, d), seed=13, dtype=torch.bfloat16, scale=4.0)
    a = torch.from_numpy(oracle.agent_pool(f64(q), gh, gw, 8, 8)).to(torch.bfloat16)
    out = run_forward_agents(q, k, v, a, 1.0, batch_stride=H * 64 * d)
    ref = oracle.agent_attn(f64(q), f64(k), f64(v), gh, gw, 1, 1, 1.0, agents=f64(a))
    assert_close(f64(out), ref, torch.bfloat16, "sharp bf16", max_abs=8e-2, rel_l2=1e-2)


def test_huge_logits_stay_finite_and_convex():
    B, H, gh, gw, d = 1, 1, 32, 32, 32
    q, k, v = random_qkv((B, H, gh * gw, d), seed=14, scale=100.0)
    out = f64(run_forward(q, k, v, gh, gw, 4, 4, 1.0))
    assert np.isfinite(out).all()
    vv = f64(v)
    assert (out >= vv.min(axis=2, keepdims=True) - 1e-3).all()
    assert (out <= vv.max(axis=2, keepdims=True) + 1e-3).all()


def test_equal_keys_and_constant_values_on_gpu():
    B, H, gh, gw, d = 2, 2, 24, 24, 32
    q, k, v = random_qkv((B, H, gh * gw, d), seed=15, dtype=torch.bfloat16)
    k_eq = k[:, :, :1].expand_as(k).contiguous()
    out = f64(run_forward(q, k_eq, v, gh, gw, 6, 6, 1 / math.sqrt(d)))
    mean_v = f64(v).mean(axis=2, keepdims=True)
    assert np.abs(out - mean_v).max() < 1e-2
    c = torch.linspace(-2, 2, d).to(torch.bfloat16)
    v_c = c.expand_as(v).contiguous()
    out_c = f64(run_forward(q, k, v_c, gh, gw, 6, 6, 1 / math.sqrt(d)))
    assert np.abs(out_c - f64(c)).max() < 2e-2


def test_workspace_variant_and_determinism():
    w = WORKLOADS["pvt_stage1_56"]
    inp = make_inputs(w)
    q, k, v = (inp[n].cuda() for n in "qkv")
    B, H, N, d = q.shape
    ws_bytes = eva.agent_attn_workspace_bytes(B, H, N, d, w.n_agents, eva.AA_BF16)
    assert ws_bytes > 0
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    o1 = torch.empty_like(q)
    o2 = torch.empty_like(q)
    args = (B, H, N, d, w.grid_h, w.grid_w, w.pool_h, w.pool_w, w.scale, eva.AA_BF16)
    eva.agent_attn_forward_ws(q, k, v, None, o1, *args, ws, ws_bytes)
    eva.agent_attn_forward(q, k, v, None, o2, *args)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    status = eva.agent_attn_forward_ws(q, k, v, None, o1, *args, ws, ws_bytes - 256, check=False)
    assert status == 5
    status = eva.agent_attn_forward_ws(q, k, v, None, o1, *args, ws[1:], ws_bytes - 1,
                                       check=False)
    assert status == 4


@pytest.mark.parametrize("name", ["deit_tiny_224", "sd_latent_1024", "highres_256_learnable256"])
def test_host_buffer_entry_point(name):
    """The host-buffer call pipelines chunks of slices over two streams; each
    chunk is its own forward pass, so the split-over-keys schedule (and with
    it the rounding order) differs from one call over all slices: compare with
    the device call at rounding level and with the oracle on sampled slices."""
    w = WORKLOADS[name]
    inp = make_inputs(w)
    q, k, v = (inp[n].pin_memory() for n in "qkv")
    ag = inp["agents"].pin_memory() if inp["agents"] is not None else None
    out = torch.empty_like(q).pin_memory()
    B, H, N, d = q.shape
    eva.agent_attn_forward_host(q, k, v, ag, out, B, H, N, d, w.grid_h, w.grid_w, w.pool_h,
                                w.pool_w, w.scale, eva.AA_BF16)
    if ag is None:
        dev = run_forward(inp["q"], inp["k"], inp["v"], w.grid_h, w.grid_w, w.pool_h, w.pool_w,
                          w.scale)
    else:
        dev = run_forward_agents(inp["q"], inp["k"], inp["v"], inp["agents"], w.scale)
    assert_close(f64(out), f64(dev), torch.bfloat16, "host vs device", max_abs=4e-3,
                 rel_l2=2e-3)
    slices = sample_slices(B, H, 2)
    ref = oracle_slices(inp["q"], inp["k"], inp["v"], w.grid_h, w.grid_w, w.pool_h, w.pool_w,
                        w.scale, slices, agents=inp["agents"])
    got = np.stack([f64(out[b, h]) for (b, h) in slices])
    assert_close(got, ref, torch.bfloat16, "host vs oracle")
