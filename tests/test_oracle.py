"""Pins for the fp64 CPU oracle (no GPU).

The oracle is checked against things that do not come from itself: library
routines (torch's adaptive average pool and scaled-dot-product attention in
float64, scipy's softmax), the generalized-linear-attention identity of
arXiv:2312.08874v3 (summary §4), closed forms, exact invariants, and the
hand-derived worked examples in ``tests/golden/``.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

import oracle
from oracle import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def torch_pool(q, gh, gw, ph, pw):
    """Library adaptive average pool of q [BH, N, d] over the (gh, gw) grid."""
    t = torch.from_numpy(q).reshape(q.shape[0], gh, gw, q.shape[-1]).permute(0, 3, 1, 2)
    a = F.adaptive_avg_pool2d(t, (ph, pw))
    return a.permute(0, 2, 3, 1).reshape(q.shape[0], ph * pw, q.shape[-1]).numpy()


def sdpa(q, k, v, scale):
    """Library scaled-dot-product attention in float64."""
    return F.scaled_dot_product_attention(torch.from_numpy(q), torch.from_numpy(k),
                                          torch.from_numpy(v), scale=scale).numpy()


# ---------------------------------------------------------------- pooling

@pytest.mark.parametrize("gh,gw,ph,pw", [
    (8, 8, 2, 2), (14, 14, 7, 7), (56, 56, 7, 7), (13, 5, 5, 3),   # 13/5 and 5/3 overlap
    (6, 10, 4, 3), (9, 9, 9, 9), (7, 4, 1, 1), (256, 16, 12, 16)])
def test_pool_matches_library_adaptive_avg_pool(gh, gw, ph, pw):
    q = rnd((3, gh * gw, 5), seed=gh * 100 + pw)
    np.testing.assert_allclose(oracle.agent_pool(q, gh, gw, ph, pw),
                               torch_pool(q, gh, gw, ph, pw), rtol=0, atol=1e-13)


def test_pool_integer_grid_256_to_12_overlap():
    """Q[n] = y*grid_w + x on a 256x256 grid pooled to 12x12: bins are 21 or 22
    wide and neighbours share a row; compare with the library pool exactly."""
    g, p = 256, 12
    y, x = np.meshgrid(np.arange(g), np.arange(g), indexing="ij")
    q = (y * g + x).reshape(1, g * g, 1).astype(np.float64)
    a = oracle.agent_pool(q, g, g, p, p)
    np.testing.assert_allclose(a, torch_pool(q, g, g, p, p), rtol=1e-15, atol=1e-9)
    # bin of agent (0, 1) along x: [floor(256/12), ceil(512/12)) = [21, 43)
    assert math.isclose(a[0, 1, 0], np.mean((y * g + x)[0:22, 21:43]), rel_tol=1e-15)


# ----------------------------------------------------- whole-pass identities

@pytest.mark.parametrize("seed,gh,gw,ph,pw,d,scale", [
    (0, 6, 6, 3, 2, 5, 0.45), (1, 4, 8, 2, 2, 8, 1.0), (2, 5, 5, 5, 5, 3, 0.7),
    (3, 8, 8, 2, 2, 32, 1 / math.sqrt(32)), (4, 3, 7, 2, 3, 4, 2.5)])
def test_brute_force_generalized_linear_attention(seed, gh, gw, ph, pw, d, scale):
    """O equals M V with the explicit N x N matrix M = softmax(QA^T s) softmax(AK^T s),
    whose rows sum to one (arXiv:2312.08874v3 summary §4)."""
    n = gh * gw
    q, k, v = (rnd((2, n, d), seed + 10 * i) for i in range(3))
    o = oracle.agent_attn(q, k, v, gh, gw, ph, pw, scale)
    a_lib = torch_pool(q, gh, gw, ph, pw)
    for bh in range(2):
        o_b, m = brute.agent_attn_brute(q[bh], a_lib[bh], k[bh], v[bh], scale)
        np.testing.assert_allclose(m.sum(axis=1), 1.0, rtol=0, atol=1e-12)
        assert (m >= 0).all()
        np.testing.assert_allclose(o[bh], o_b, rtol=0, atol=1e-12)


def test_pool_equal_grid_reduces_to_softmax_attention():
    """pool = grid: every token is its own agent (A = Q), so aggregation is plain
    softmax attention SDPA(Q, K, V) and broadcast is SDPA(Q, Q, V_A)."""
    gh, gw, d, scale = 5, 6, 7, 0.6
    q, k, v = (rnd((3, gh * gw, d), 40 + i) for i in range(3))
    a = oracle.agent_pool(q, gh, gw, gh, gw)
    np.testing.assert_allclose(a, q, rtol=0, atol=1e-15)
    va = oracle.agent_aggregate(a, k, v, scale)
    np.testing.assert_allclose(va, sdpa(q, k, v, scale), rtol=0, atol=1e-13)
    o = oracle.agent_broadcast(q, a, va, scale)
    np.testing.assert_allclose(o, sdpa(q, q, va, scale), rtol=0, atol=1e-13)
    np.testing.assert_allclose(oracle.agent_attn(q, k, v, gh, gw, gh, gw, scale), o,
                               rtol=0, atol=1e-15)


def test_single_agent_closed_form():
    """pool 1x1: A = mean(Q); one agent takes all broadcast weight, so every output
    row equals softmax(s mean(Q) K^T) V, a one-query SDPA."""
    gh, gw, d, scale = 6, 5, 8, 0.8
    q, k, v = (rnd((2, gh * gw, d), 50 + i) for i in range(3))
    o = oracle.agent_attn(q, k, v, gh, gw, 1, 1, scale)
    mean_q = q.mean(axis=1, keepdims=True)
    row = sdpa(mean_q, k, v, scale)                      # [2, 1, d]
    np.testing.assert_allclose(o, np.broadcast_to(row, o.shape), rtol=0, atol=1e-13)


def test_equal_keys_give_mean_of_values():
    gh, gw, d = 7, 7, 6
    q, _, v = (rnd((2, gh * gw, d), 60 + i) for i in range(3))
    k = np.broadcast_to(rnd((2, 1, d), 63), q.shape).copy()
    o = oracle.agent_attn(q, k, v, gh, gw, 3, 3, 0.9)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=1, keepdims=True), o.shape),
                               rtol=0, atol=1e-13)


def test_constant_values_give_constant_output():
    gh, gw, d = 6, 6, 4
    q, k, _ = (rnd((2, gh * gw, d), 70 + i, scale=3.0) for i in range(3))
    c = np.array([1.5, -2.0, 0.25, 7.0])
    v = np.broadcast_to(c, q.shape).copy()
    o = oracle.agent_attn(q, k, v, gh, gw, 2, 3, 1.0)
    np.testing.assert_allclose(o, np.broadcast_to(c, o.shape), rtol=0, atol=1e-12)


def test_affine_values_and_key_shift():
    gh, gw, d, scale = 6, 8, 5, 0.7
    q, k, v = (rnd((2, gh * gw, d), 80 + i) for i in range(3))
    o = oracle.agent_attn(q, k, v, gh, gw, 3, 4, scale)
    alpha, shift = -1.75, rnd((d,), 84)
    o2 = oracle.agent_attn(q, k, alpha * v + shift, gh, gw, 3, 4, scale)
    np.testing.assert_allclose(o2, alpha * o + shift, rtol=0, atol=1e-12)
    u = rnd((d,), 85, scale=5.0)           # the same vector added to every key
    o3 = oracle.agent_attn(q, k + u, v, gh, gw, 3, 4, scale)
    np.testing.assert_allclose(o3, o, rtol=0, atol=1e-12)


def test_convex_hull_of_values():
    gh, gw, d = 9, 9, 6
    q, k, v = (rnd((3, gh * gw, d), 90 + i, scale=2.0) for i in range(3))
    o = oracle.agent_attn(q, k, v, gh, gw, 3, 3, 1.0)
    lo, hi = v.min(axis=1, keepdims=True), v.max(axis=1, keepdims=True)
    assert (o >= lo - 1e-12).all() and (o <= hi + 1e-12).all()


def test_joint_permutation_of_keys_and_values():
    gh, gw, d = 8, 6, 5
    q, k, v = (rnd((2, gh * gw, d), 100 + i) for i in range(3))
    perm = np.random.default_rng(103).permutation(gh * gw)
    o = oracle.agent_attn(q, k, v, gh, gw, 2, 3, 0.8)
    o_p = oracle.agent_attn(q, k[:, perm], v[:, perm], gh, gw, 2, 3, 0.8)
    np.testing.assert_allclose(o_p, o, rtol=0, atol=1e-13)


def test_learnable_agents_and_agent_permutation():
    """Externally supplied agents [H, k, d] shared over the batch; the output does
    not depend on agent order."""
    B, H, gh, gw, d, n_ag = 2, 3, 5, 6, 8, 7
    q, k, v = (rnd((B, H, gh * gw, d), 110 + i) for i in range(3))
    agents = rnd((H, n_ag, d), 113, scale=0.7)
    o = oracle.agent_attn(q, k, v, gh, gw, 1, 1, 0.5, agents=agents)
    perm = np.random.default_rng(114).permutation(n_ag)
    o_p = oracle.agent_attn(q, k, v, gh, gw, 1, 1, 0.5, agents=agents[:, perm])
    np.testing.assert_allclose(o_p, o, rtol=0, atol=1e-13)
    # the shared agents equal an explicit per-batch copy, and match the brute force
    full = np.broadcast_to(agents, (B,) + agents.shape)
    o_full = oracle.agent_attn(q, k, v, gh, gw, 1, 1, 0.5, agents=full)
    np.testing.assert_allclose(o_full, o, rtol=0, atol=0)
    o_b, _ = brute.agent_attn_brute(q[1, 2], agents[2], k[1, 2], v[1, 2], 0.5)
    np.testing.assert_allclose(o[1, 2], o_b, rtol=0, atol=1e-12)


def test_scale_to_zero_gives_mean_of_values():
    gh, gw, d = 6, 6, 4
    q, k, v = (rnd((2, gh * gw, d), 120 + i) for i in range(3))
    o = oracle.agent_attn(q, k, v, gh, gw, 3, 3, 1e-12)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=1, keepdims=True), o.shape),
                               rtol=0, atol=1e-9)


@pytest.mark.parametrize("mult", [4.0, 100.0])
def test_sharp_logits_match_library_softmax(mult):
    """Scale 1 and inputs x4 or x100 (logits in the thousands): stage outputs match
    scipy's softmax and stay finite."""
    gh, gw, d = 6, 6, 8
    q, k, v = (rnd((2, gh * gw, d), 130 + i, scale=mult) for i in range(3))
    a = oracle.agent_pool(q, gh, gw, 2, 2)
    va = oracle.agent_aggregate(a, k, v, 1.0)
    ref_va = scipy.special.softmax(np.einsum("bjc,bnc->bjn", a, k), axis=-1) @ v
    np.testing.assert_allclose(va, ref_va, rtol=1e-12, atol=1e-12 * mult)
    o = oracle.agent_broadcast(q, a, va, 1.0)
    ref_o = scipy.special.softmax(np.einsum("bnc,bjc->bnj", q, a), axis=-1) @ va
    np.testing.assert_allclose(o, ref_o, rtol=1e-12, atol=1e-12 * mult)
    assert np.isfinite(o).all()


# ------------------------------------------------------ worked examples

def _eval(x):
    if isinstance(x, str):
        return float(eval(x, {"__builtins__": {}}, {"e": math.e, "log": math.log}))
    return float(x)


def _mat(rows):
    return np.array([[_eval(x) for x in r] for r in rows], dtype=np.float64)


def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_hand_derived_worked_examples(case):
    gh, gw = case["grid"]
    ph, pw = case["pool"]
    q, k, v = (_mat(case[n])[None] for n in ("q", "k", "v"))
    a = oracle.agent_pool(q, gh, gw, ph, pw)
    np.testing.assert_allclose(a[0], _mat(case["expected_agents"]), rtol=0, atol=1e-14)
    va = oracle.agent_aggregate(a, k, v, case["scale"])
    np.testing.assert_allclose(va[0], _mat(case["expected_va"]), rtol=0, atol=1e-13)
    o = oracle.agent_attn(q, k, v, gh, gw, ph, pw, case["scale"])
    np.testing.assert_allclose(o[0], _mat(case["expected_o"]), rtol=0, atol=1e-13)


def test_oracle_is_fp64_and_deterministic():
    q, k, v = (rnd((1, 64, 32), 140 + i) for i in range(3))
    o1 = oracle.agent_attn(q, k, v, 8, 8, 2, 2, 0.2)
    o2 = oracle.agent_attn(q, k, v, 8, 8, 2, 2, 0.2)
    assert o1.dtype == np.float64
    np.testing.assert_array_equal(o1, o2)


# ---------------------------------------------------------------- DWC term
def torch_dwc(v, w, bias, gh, gw):
    """Library depth-wise convolution (float64 conv2d, one group per channel)."""
    B, H, N, d = v.shape
    t = torch.from_numpy(v).reshape(B, H, gh, gw, d).permute(0, 1, 4, 2, 3).reshape(B, H * d, gh, gw)
    wt = torch.from_numpy(w).reshape(H * d, 1, 3, 3)
    bt = None if bias is None else torch.from_numpy(bias).reshape(H * d)
    o = F.conv2d(t, wt, bt, padding=1, groups=H * d)
    return o.reshape(B, H, d, gh, gw).permute(0, 1, 3, 4, 2).reshape(B, H, N, d).numpy()


@pytest.mark.parametrize("gh,gw,d", [(5, 7, 3), (1, 9, 2), (6, 1, 4), (8, 8, 8)])
def test_dwc_matches_library_depthwise_conv(gh, gw, d):
    B, H = 2, 3
    v = rnd((B, H, gh * gw, d), 31)
    w = rnd((H, d, 3, 3), 32)
    bias = rnd((H, d), 33)
    np.testing.assert_allclose(oracle.dwc(v, w, bias, gh, gw), torch_dwc(v, w, bias, gh, gw),
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.dwc(v, w, None, gh, gw), torch_dwc(v, w, None, gh, gw),
                               rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("ty,tx", [(0, 0), (0, 1), (0, 2), (1, 0), (1, 1), (1, 2), (2, 0), (2, 1),
                                   (2, 2)])
def test_dwc_single_tap_is_a_zero_filled_shift(ty, tx):
    """A kernel with one unit tap at (ty, tx) reads V at (y + ty - 1, x + tx - 1)."""
    gh, gw, d = 4, 6, 2
    v = rnd((1, 2, gh * gw, d), 34)
    w = np.zeros((2, d, 3, 3))
    w[:, :, ty, tx] = 1.0
    grid = v.reshape(1, 2, gh, gw, d)
    want = np.zeros_like(grid)
    dy, dx = ty - 1, tx - 1
    ys, xs = slice(max(0, -dy), gh - max(0, dy)), slice(max(0, -dx), gw - max(0, dx))
    ys2, xs2 = slice(max(0, dy), gh - max(0, -dy)), slice(max(0, dx), gw - max(0, -dx))
    want[:, :, ys, xs] = grid[:, :, ys2, xs2]
    np.testing.assert_array_equal(oracle.dwc(v, w, None, gh, gw), want.reshape(v.shape))


def test_dwc_constant_values_count_the_taps_inside_the_grid():
    gh, gw, d, c = 5, 4, 3, 1.75
    v = np.full((1, 1, gh * gw, d), c)
    w = rnd((1, d, 3, 3), 35)
    out = oracle.dwc(v, w, None, gh, gw).reshape(gh, gw, d)
    for y in range(gh):
        for x in range(gw):
            inside = np.zeros((3, 3))
            for ty in range(3):
                for tx in range(3):
                    inside[ty, tx] = 0 <= y + ty - 1 < gh and 0 <= x + tx - 1 < gw
            want = c * (w[0] * inside).sum(axis=(1, 2))
            np.testing.assert_allclose(out[y, x], want, rtol=1e-14, atol=1e-14)


def test_dwc_is_linear_and_bias_only_is_a_broadcast():
    gh, gw, d = 3, 5, 4
    v1, v2 = rnd((2, 2, gh * gw, d), 36), rnd((2, 2, gh * gw, d), 37)
    w = rnd((2, d, 3, 3), 38)
    lhs = oracle.dwc(2.5 * v1 + v2, w, None, gh, gw)
    rhs = 2.5 * oracle.dwc(v1, w, None, gh, gw) + oracle.dwc(v2, w, None, gh, gw)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-12)
    bias = rnd((2, d), 39)
    out = oracle.dwc(v1, np.zeros((2, d, 3, 3)), bias, gh, gw)
    np.testing.assert_array_equal(out, np.broadcast_to(bias[None, :, None, :], out.shape))


def test_full_module_output_is_attention_plus_dwc():
    gh, gw, d = 6, 6, 4
    q, k, v = (rnd((1, 2, gh * gw, d), s) for s in (40, 41, 42))
    w = rnd((2, d, 3, 3), 43)
    full = oracle.agent_attn_dwc(q, k, v, gh, gw, 3, 3, 0.5, w)
    np.testing.assert_allclose(full - oracle.agent_attn(q, k, v, gh, gw, 3, 3, 0.5),
                               torch_dwc(v, w, None, gh, gw), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- agent bias
def bias_parts(H, k, gh, gw, nb, seed, scale=1.0):
    return (rnd((H, k, gh), seed, scale), rnd((H, k, gw), seed + 1, scale),
            rnd((H, k, nb), seed + 2, scale))


def test_bias_components_build_the_full_matrix_by_grid_cell():
    """Row, column and block components land on the token's grid row, grid
    column and cell of the floor partition into pool_h x pool_w blocks."""
    H, k, gh, gw, ph, pw = 2, 3, 7, 5, 3, 2
    row, col, block = bias_parts(H, k, gh, gw, ph * pw, 50)
    full = oracle.agent_bias(row, col, block, gh, gw, ph, pw)
    for y in range(gh):
        for x in range(gw):
            cell = (y * ph // gh) * pw + (x * pw // gw)
            np.testing.assert_array_equal(full[:, :, y * gw + x],
                                          row[:, :, y] + col[:, :, x] + block[:, :, cell])
    # a one-hot block component marks exactly the tokens of that block
    onehot = np.zeros((1, 1, ph * pw))
    onehot[0, 0, 4] = 1.0
    marked = oracle.agent_bias(None, None, onehot, gh, gw, ph, pw).reshape(gh, gw)
    ys, xs = np.nonzero(marked)
    assert set(ys * ph // gh) == {4 // pw} and set(xs * pw // gw) == {4 % pw}


@pytest.mark.parametrize("gh,gw,ph,pw", [
    (13, 11, 4, 3), (256, 256, 12, 12), (7, 5, 3, 2), (128, 128, 16, 16), (5, 9, 5, 2),
    (31, 17, 6, 4)])
def test_bias_matches_library_nearest_upsampling(gh, gw, ph, pw):
    """The bias matrix against library routines: the block component is the
    pool_h x pool_w grid of block values upsampled to the token grid by torch's
    nearest-neighbour interpolation (source cell floor(y * pool_h / grid_h),
    floor(x * pool_w / grid_w)), the row and column components are torch
    broadcasts along the other grid axis.  Non-square pools and non-dividing
    grids make a swapped pool_h / pool_w, a ceil instead of a floor, or a token
    assigned to the later of two overlapping adaptive-pool bins fail."""
    # torch computes the source index in single precision; for these sizes it
    # agrees with the exact integer floor, which is asserted first
    for g, p in ((gh, ph), (gw, pw)):
        idx = F.interpolate(torch.arange(p, dtype=torch.float64).reshape(1, 1, p), size=g,
                            mode="nearest")[0, 0].numpy().astype(int)
        assert (idx == (np.arange(g) * p) // g).all()
    H, k = 2, 3
    row, col, block = bias_parts(H, k, gh, gw, ph * pw, 61)
    t_row = torch.from_numpy(row)[:, :, :, None].expand(H, k, gh, gw)
    t_col = torch.from_numpy(col)[:, :, None, :].expand(H, k, gh, gw)
    t_blk = F.interpolate(torch.from_numpy(block).reshape(H * k, 1, ph, pw), size=(gh, gw),
                          mode="nearest").reshape(H, k, gh, gw)
    want = (torch.zeros(H, k, gh, gw, dtype=torch.float64) + t_row + t_col + t_blk).numpy()
    got = oracle.agent_bias(row, col, block, gh, gw, ph, pw).reshape(H, k, gh, gw)
    np.testing.assert_array_equal(got, want)
    # each component alone, through the same library routines
    np.testing.assert_array_equal(
        oracle.agent_bias(None, None, block, gh, gw, ph, pw).reshape(H, k, gh, gw),
        t_blk.numpy())
    np.testing.assert_array_equal(
        oracle.agent_bias(row, None, None, gh, gw, ph, pw).reshape(H, k, gh, gw),
        t_row.numpy())
    np.testing.assert_array_equal(
        oracle.agent_bias(None, col, None, gh, gw, ph, pw).reshape(H, k, gh, gw),
        t_col.numpy())


def test_zero_bias_is_the_plain_forward_pass():
    q, k, v = (rnd((2, 2, 30, 4), s) for s in (51, 52, 53))
    z = np.zeros((2, 4, 30))
    np.testing.assert_array_equal(oracle.agent_attn_bias(q, k, v, 5, 6, 2, 2, 0.4, z, z),
                                  oracle.agent_attn(q, k, v, 5, 6, 2, 2, 0.4))


def test_bias_matches_the_brute_force_mixing_matrix():
    gh, gw, ph, pw, d = 4, 5, 2, 2, 3
    q, k, v = (rnd((1, 2, gh * gw, d), s) for s in (54, 55, 56))
    b1 = oracle.agent_bias(*bias_parts(2, 4, gh, gw, 4, 57), gh, gw, ph, pw)
    b2 = oracle.agent_bias(*bias_parts(2, 4, gh, gw, 4, 60), gh, gw, ph, pw)
    got = oracle.agent_attn_bias(q, k, v, gh, gw, ph, pw, 0.7, b1, b2)
    a = torch_pool(q[0], gh, gw, ph, pw)
    for h in range(2):
        o, m = brute.agent_attn_brute_bias(q[0, h], a[h], k[0, h], v[0, h], 0.7, b1[h], b2[h])
        np.testing.assert_allclose(m.sum(axis=1), 1.0, rtol=0, atol=1e-12)
        np.testing.assert_allclose(got[0, h], o, rtol=1e-11, atol=1e-12)


def test_bias_constant_along_the_softmax_axis_changes_nothing():
    """A per-agent constant in B1 (over keys) and a per-query constant in B2
    (over agents) cancel in their softmaxes."""
    gh, gw, ph, pw = 6, 6, 3, 3
    q, k, v = (rnd((2, 2, 36, 4), s) for s in (63, 64, 65))
    row1 = np.broadcast_to(rnd((2, 9, 1), 66), (2, 9, gh))           # depends on the agent only
    b1 = oracle.agent_bias(row1, None, None, gh, gw, ph, pw)
    row2 = np.broadcast_to(rnd((2, 1, gh), 67), (2, 9, gh))          # depends on the query only
    col2 = np.broadcast_to(rnd((2, 1, gw), 68), (2, 9, gw))
    b2 = oracle.agent_bias(row2, col2, None, gh, gw, ph, pw)
    np.testing.assert_allclose(oracle.agent_attn_bias(q, k, v, gh, gw, ph, pw, 0.5, b1, b2),
                               oracle.agent_attn(q, k, v, gh, gw, ph, pw, 0.5),
                               rtol=1e-12, atol=1e-12)


def test_bias_that_admits_one_token_selects_its_value():
    """B1 = -1e4 everywhere except token (y*, x*): every agent aggregates exactly
    V[n*], so every query reads V[n*] whatever B2 is."""
    gh, gw, ph, pw, ys, xs = 5, 4, 2, 2, 3, 1
    q, k, v = (rnd((1, 2, gh * gw, 3), s) for s in (69, 70, 71))
    row = np.full((2, 4, gh), -1e4)
    row[:, :, ys] = 0.0
    col = np.full((2, 4, gw), -1e4)
    col[:, :, xs] = 0.0
    b1 = oracle.agent_bias(row, col, None, gh, gw, ph, pw)
    b2 = oracle.agent_bias(*bias_parts(2, 4, gh, gw, 4, 72), gh, gw, ph, pw)
    got = oracle.agent_attn_bias(q, k, v, gh, gw, ph, pw, 0.5, b1, b2)
    want = np.broadcast_to(v[:, :, ys * gw + xs][:, :, None, :], got.shape)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- backward
def torch_forward(q, k, v, gh, gw, ph, pw, scale, agents=None):
    """The forward pass written with torch library ops (float64), for autograd."""
    B, H, N, d = q.shape
    if agents is None:
        t = q.reshape(B * H, gh, gw, d).permute(0, 3, 1, 2)
        a = F.adaptive_avg_pool2d(t, (ph, pw)).permute(0, 2, 3, 1).reshape(B, H, ph * pw, d)
    else:
        a = agents
    va = torch.softmax(scale * a @ k.transpose(-1, -2), dim=-1) @ v
    return torch.softmax(scale * q @ a.transpose(-1, -2), dim=-1) @ va


@pytest.mark.parametrize("learnable", [False, True])
def test_backward_matches_autograd_of_library_ops(learnable):
    B, H, gh, gw, ph, pw, d, scale = 2, 2, 5, 6, 2, 3, 4, 0.6
    q, k, v, do = (rnd((B, H, gh * gw, d), s) for s in (80, 81, 82, 83))
    ag = rnd((B, H, ph * pw, d), 84) if learnable else None
    tq, tk, tv = (torch.from_numpy(x).requires_grad_() for x in (q, k, v))
    ta = torch.from_numpy(ag).requires_grad_() if learnable else None
    out = torch_forward(tq, tk, tv, gh, gw, ph, pw, scale, ta)
    out.backward(torch.from_numpy(do))
    dq, dk, dv, da = oracle.agent_attn_backward(q, k, v, do, gh, gw, ph, pw, scale, agents=ag)
    for got, want in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        np.testing.assert_allclose(got, want.numpy(), rtol=1e-10, atol=1e-12)
    if learnable:
        np.testing.assert_allclose(da, ta.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_backward_matches_central_differences():
    """<dO, O(x + eU)> - <dO, O(x - eU)> over 2e equals <grad, U>, for random
    directions U of q, k and v, with the oracle's own forward pass."""
    B, H, gh, gw, ph, pw, d, scale = 1, 2, 4, 5, 2, 2, 3, 0.8
    x = {n: rnd((B, H, gh * gw, d), s) for n, s in (("q", 90), ("k", 91), ("v", 92))}
    do = rnd((B, H, gh * gw, d), 93)
    grads = dict(zip("qkv", oracle.agent_attn_backward(x["q"], x["k"], x["v"], do, gh, gw, ph,
                                                        pw, scale)[:3]))
    eps = 1e-5
    for name, s in (("q", 94), ("k", 95), ("v", 96)):
        u = rnd(x[name].shape, s)

        def loss(sign):
            y = dict(x)
            y[name] = x[name] + sign * eps * u
            return float((do * oracle.agent_attn(y["q"], y["k"], y["v"], gh, gw, ph, pw,
                                                 scale)).sum())
        fd = (loss(1) - loss(-1)) / (2 * eps)
        assert abs(fd - float((grads[name] * u).sum())) < 1e-7 * max(1.0, abs(fd))


def test_backward_sums_follow_the_forward_invariances():
    """O(K + u) = O(K) gives sum_n dK_n = 0; O(V + c) = O(V) + c gives
    sum_n dV_n = sum_n dO_n."""
    q, k, v, do = (rnd((2, 3, 24, 5), s) for s in (97, 98, 99, 100))
    _, dk, dv, _ = oracle.agent_attn_backward(q, k, v, do, 4, 6, 2, 3, 0.5)
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
    np.testing.assert_allclose(dv.sum(axis=2), do.sum(axis=2), rtol=1e-12, atol=1e-12)


# ------------------------------------------- the kernels' FMA-pipe exponential
def test_fma_exp2_polynomial_constants_meet_their_bound():
    """The degree-3 coefficients compiled into the tensor-core kernels,
    evaluated in fp32 Horner form as the kernels do, approximate 2^f on
    [-1/2, 1/2] to a relative error below 1e-4 (the fit reports 7.5e-5); a
    dropped or mistyped coefficient fails."""
    import re
    src = open(os.path.join(os.path.dirname(os.path.dirname(__file__)),
                            "efficient_vision_attention_b200", "csrc",
                            "tc_primitives.cuh")).read()
    coef = [np.float32(re.search(rf"kExp2C{i} = ([0-9.e+-]+)f;", src).group(1))
            for i in range(4)]
    f = np.linspace(-0.5, 0.5, 1_000_001).astype(np.float32)
    p = np.full_like(f, coef[3])
    for c in coef[2::-1]:
        p = (p * f + c).astype(np.float32)
    rel = np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    assert rel.max() < 1e-4
    # whole arguments: rint split, exponent insertion (2^j exactly) times p(f)
    x = np.linspace(-125.0, 8.0, 200_001).astype(np.float32)
    j = np.rint(x)
    fx = (x - j).astype(np.float32)
    px = np.full_like(fx, coef[3])
    for c in coef[2::-1]:
        px = (px * fx + c).astype(np.float32)
    y = px.astype(np.float64) * np.exp2(j)
    assert np.abs(y / np.exp2(x.astype(np.float64)) - 1.0).max() < 1e-4
