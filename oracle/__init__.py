"""Agent Attention forward pass: fp64 CPU oracle (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or executes anything here, and this
package imports nothing from the product.

The arithmetic lives in ``agent_attn_oracle.c`` (plain fp64 loops, OpenMP over
independent rows), compiled with ``gcc -O2 -fopenmp`` without fast-math.  This
module only marshals numpy arrays.  ``brute.py`` holds the independent N x N
brute force (the generalized-linear-attention form of the same operator).

Every function here is pinned by ``tests/test_oracle.py`` against facts that
do not come from the oracle itself: library routines (torch's adaptive average
pool and scaled-dot-product attention in float64, scipy's softmax), closed
forms, exact invariants and hand-derived worked examples in ``tests/golden/``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "agent_attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, -O2, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        i64 = ctypes.c_int64
        lib.oracle_agent_pool.argtypes = [dp, i64, i64, i64, i64, i64, i64, i64, dp]
        lib.oracle_agent_aggregate.argtypes = [dp, dp, dp, i64, i64, i64, i64, ctypes.c_double, dp]
        lib.oracle_agent_broadcast.argtypes = [dp, dp, dp, i64, i64, i64, i64, ctypes.c_double, dp]
        lib.oracle_agent_attn.argtypes = [dp, dp, dp, dp, i64, i64, i64, i64, i64, i64, i64, i64,
                                          ctypes.c_double, dp, dp, dp]
        lib.oracle_dwc.argtypes = [dp, dp, dp, i64, i64, i64, i64, i64, dp]
        lib.oracle_agent_attn_backward.argtypes = [dp, dp, dp, dp, dp, i64, i64, i64, i64, i64,
                                                   i64, i64, i64, ctypes.c_double, dp, dp, dp,
                                                   dp]
        lib.oracle_agent_attn_bias.argtypes = [dp, dp, dp, dp, dp, dp, i64, i64, i64, i64, i64,
                                               i64, i64, i64, i64, ctypes.c_double, dp, dp, dp]
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(x: np.ndarray):
    return x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _bh_view(x: np.ndarray, rank: int = 3):
    """Collapse leading batch/head axes: returns (array [BH, rows, d], leading shape)."""
    x = _f64(x)
    lead = x.shape[:-2]
    return x.reshape((-1,) + x.shape[-2:]), lead


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def agent_pool(q, grid_h: int, grid_w: int, pool_h: int, pool_w: int) -> np.ndarray:
    """Adaptive average pool of Q [..., N, d] over its grid -> agents [..., pool_h*pool_w, d]."""
    q3, lead = _bh_view(q)
    bh, n, d = q3.shape
    if n != grid_h * grid_w:
        raise ValueError("N must equal grid_h * grid_w")
    if not (1 <= pool_h <= grid_h and 1 <= pool_w <= grid_w):
        raise ValueError("pool size must lie in [1, grid]")
    a = np.empty((bh, pool_h * pool_w, d), dtype=np.float64)
    _load().oracle_agent_pool(_ptr(q3), bh, n, d, grid_h, grid_w, pool_h, pool_w, _ptr(a))
    return a.reshape(lead + a.shape[1:])


def agent_aggregate(a, k, v, scale: float) -> np.ndarray:
    """V_A = softmax(A K^T * scale) V per (batch, head) slice."""
    a3, lead = _bh_view(a)
    k3, _ = _bh_view(k)
    v3, _ = _bh_view(v)
    bh, n_agents, d = a3.shape
    n = k3.shape[1]
    assert k3.shape == (bh, n, d) and v3.shape == (bh, n, d)
    va = np.empty_like(a3)
    _load().oracle_agent_aggregate(_ptr(a3), _ptr(k3), _ptr(v3), bh, n, d, n_agents,
                                   float(scale), _ptr(va))
    return va.reshape(lead + va.shape[1:])


def agent_broadcast(q, a, va, scale: float) -> np.ndarray:
    """O = softmax(Q A^T * scale) V_A per (batch, head) slice."""
    q3, lead = _bh_view(q)
    a3, _ = _bh_view(a)
    va3, _ = _bh_view(va)
    bh, n, d = q3.shape
    n_agents = a3.shape[1]
    assert a3.shape == (bh, n_agents, d) and va3.shape == (bh, n_agents, d)
    o = np.empty_like(q3)
    _load().oracle_agent_broadcast(_ptr(q3), _ptr(a3), _ptr(va3), bh, n, d, n_agents,
                                   float(scale), _ptr(o))
    return o.reshape(lead + o.shape[1:])


def agent_attn(q, k, v, grid_h: int, grid_w: int, pool_h: int, pool_w: int,
               scale: float, agents=None) -> np.ndarray:
    """Whole forward pass on [B, H, N, d] (or [BH, N, d]) inputs.

    ``agents`` (learnable agents) may be [H, k, d] (shared over the batch),
    [B, H, k, d] or None (agents pooled from Q).
    """
    q3, lead = _bh_view(q)
    k3, _ = _bh_view(k)
    v3, _ = _bh_view(v)
    bh, n, d = q3.shape
    if agents is None:
        n_agents = pool_h * pool_w
        a3 = None
    else:
        ag = _f64(agents)
        n_agents = ag.shape[-2]
        if ag.ndim == 3 and len(lead) == 2:            # [H, k, d] shared over B
            ag = np.broadcast_to(ag[None], lead[:1] + ag.shape)
        a3 = np.ascontiguousarray(ag.reshape(bh, n_agents, d))
    scratch_a = np.empty((bh, n_agents, d), dtype=np.float64)
    scratch_va = np.empty((bh, n_agents, d), dtype=np.float64)
    o = np.empty_like(q3)
    lib = _load()
    lib.oracle_agent_attn(_ptr(q3), _ptr(k3), _ptr(v3), _ptr(a3) if a3 is not None else None,
                          bh, n, d, grid_h, grid_w, pool_h, pool_w, n_agents, float(scale),
                          _ptr(scratch_a), _ptr(scratch_va), _ptr(o))
    return o.reshape(lead + o.shape[1:])


def dwc(v, w, bias, grid_h: int, grid_w: int) -> np.ndarray:
    """Depth-wise 3x3 convolution of V [B, H, N, d] over its token grid with
    per-(head, channel) kernels w [H, d, 3, 3] and optional bias [H, d]
    (zero padding, output on the same grid)."""
    v = _f64(v)
    B, H, n, d = v.shape
    if n != grid_h * grid_w:
        raise ValueError("N must equal grid_h * grid_w")
    w = _f64(w)
    assert w.shape == (H, d, 3, 3)
    b = None if bias is None else _f64(bias)
    if b is not None:
        assert b.shape == (H, d)
    out = np.empty_like(v)
    _load().oracle_dwc(_ptr(v), _ptr(w), _ptr(b) if b is not None else None, B * H, H, grid_h,
                       grid_w, d, _ptr(out))
    return out


def agent_attn_dwc(q, k, v, grid_h: int, grid_w: int, pool_h: int, pool_w: int, scale: float,
                   w, bias=None, agents=None) -> np.ndarray:
    """The full module's output: the Agent Attention forward pass plus the
    depth-wise convolution term of V."""
    return (agent_attn(q, k, v, grid_h, grid_w, pool_h, pool_w, scale, agents=agents)
            + dwc(v, w, bias, grid_h, grid_w))


def agent_bias(row, col, block, grid_h: int, grid_w: int, pool_h: int, pool_w: int) -> np.ndarray:
    """Full agent-bias matrix [H, k, N] from its components (the reading of the
    pages' "column, row and block components"): for agent j and token
    n = y*grid_w + x,
        B[h, j, n] = row[h, j, y] + col[h, j, x] + block[h, j, b(y, x)],
    where b(y, x) = floor(y*pool_h/grid_h)*pool_w + floor(x*pool_w/grid_w) is
    the cell of the pool_h x pool_w partition of the grid holding the token.
    row: [H, k, grid_h], col: [H, k, grid_w], block: [H, k, pool_h*pool_w];
    a component given as None contributes zero (at least one is required)."""
    parts = [x for x in (row, col, block) if x is not None]
    H, k = _f64(parts[0]).shape[:2]
    out = np.zeros((H, k, grid_h, grid_w))
    if row is not None:
        out += _f64(row)[:, :, :, None]
    if col is not None:
        out += _f64(col)[:, :, None, :]
    if block is not None:
        by = (np.arange(grid_h) * pool_h) // grid_h
        bx = (np.arange(grid_w) * pool_w) // grid_w
        cell = by[:, None] * pool_w + bx[None, :]
        out += _f64(block)[:, :, cell]
    return out.reshape(H, k, grid_h * grid_w)


def agent_attn_bias(q, k, v, grid_h: int, grid_w: int, pool_h: int, pool_w: int, scale: float,
                    b1=None, b2=None, agents=None) -> np.ndarray:
    """Forward pass with agent bias: b1 [H, k, N] is added to the aggregation
    logits (agent j, key n), b2 [H, k, N] to the broadcast logits (query n,
    agent j); either may be None.  Inputs [B, H, N, d]."""
    q = _f64(q)
    B, H, n, d = q.shape
    k3 = _f64(k).reshape(B * H, n, d)
    v3 = _f64(v).reshape(B * H, n, d)
    q3 = q.reshape(B * H, n, d)
    if agents is None:
        n_agents = pool_h * pool_w
        a3 = None
    else:
        ag = _f64(agents)
        n_agents = ag.shape[-2]
        if ag.ndim == 3:
            ag = np.broadcast_to(ag[None], (B,) + ag.shape)
        a3 = np.ascontiguousarray(ag.reshape(B * H, n_agents, d))
    b1 = None if b1 is None else np.ascontiguousarray(_f64(b1))
    b2 = None if b2 is None else np.ascontiguousarray(_f64(b2))
    for b in (b1, b2):
        if b is not None:
            assert b.shape == (H, n_agents, n)
    scratch_a = np.empty((B * H, n_agents, d))
    scratch_va = np.empty((B * H, n_agents, d))
    o = np.empty_like(q3)
    _load().oracle_agent_attn_bias(
        _ptr(q3), _ptr(k3), _ptr(v3), _ptr(a3) if a3 is not None else None,
        _ptr(b1) if b1 is not None else None, _ptr(b2) if b2 is not None else None,
        B * H, H, n, d, grid_h, grid_w, pool_h, pool_w, n_agents, float(scale),
        _ptr(scratch_a), _ptr(scratch_va), _ptr(o))
    return o.reshape(B, H, n, d)


def agent_attn_backward(q, k, v, dout, grid_h: int, grid_w: int, pool_h: int, pool_w: int,
                        scale: float, agents=None):
    """Gradients (dq, dk, dv, dagents) of the forward pass for the output
    gradient dout; inputs [B, H, N, d].  agents: None (pooled from Q; dq then
    includes the pooling adjoint) or [H, k, d] / [B, H, k, d] given agents.
    dagents is [B, H, k, d] (per slice, before any sum over a shared batch)."""
    q = _f64(q)
    B, H, n, d = q.shape
    k3, v3, do3 = (_f64(t).reshape(B * H, n, d) for t in (k, v, dout))
    q3 = q.reshape(B * H, n, d)
    if agents is None:
        n_agents = pool_h * pool_w
        a3 = None
    else:
        ag = _f64(agents)
        n_agents = ag.shape[-2]
        if ag.ndim == 3:
            ag = np.broadcast_to(ag[None], (B,) + ag.shape)
        a3 = np.ascontiguousarray(ag.reshape(B * H, n_agents, d))
    dq, dk, dv = (np.empty((B * H, n, d)) for _ in range(3))
    da = np.empty((B * H, n_agents, d))
    _load().oracle_agent_attn_backward(
        _ptr(q3), _ptr(k3), _ptr(v3), _ptr(a3) if a3 is not None else None, _ptr(do3), B * H, n,
        d, grid_h, grid_w, pool_h, pool_w, n_agents, float(scale), _ptr(dq), _ptr(dk), _ptr(dv),
        _ptr(da))
    shape = (B, H, n, d)
    return dq.reshape(shape), dk.reshape(shape), dv.reshape(shape), da.reshape(B, H, n_agents, d)
