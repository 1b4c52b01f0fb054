"""N x N brute force of the Agent Attention forward pass (test infrastructure only).

The summary of arXiv:2312.08874v3 ("Agent Attention: On the Integration of
Softmax and Linear Attention", §4 "Agent Attention") states that the module is
a generalized linear attention: O = sigma(Q A^T) sigma(A K^T) V, i.e. the two
softmax attentions collapse into one N x N mixing matrix
M = softmax_rows(Q A^T s) @ softmax_rows(A K^T s).  Each factor is row
stochastic, so every row of M sums to one.  This module builds M explicitly
(float64, numpy) for tiny inputs; it is an independent formulation of the same
operator that the C oracle evaluates stage by stage.
"""
from __future__ import annotations

import numpy as np


def _softmax_rows(x: np.ndarray) -> np.ndarray:
    x = x - x.max(axis=-1, keepdims=True)
    e = np.exp(x)
    return e / e.sum(axis=-1, keepdims=True)


def mixing_matrix(q: np.ndarray, a: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """M = softmax_rows(Q A^T s) @ softmax_rows(A K^T s) for one slice: [N, N]."""
    q = np.asarray(q, np.float64)
    a = np.asarray(a, np.float64)
    k = np.asarray(k, np.float64)
    left = _softmax_rows(scale * q @ a.T)        # [N, n_agents]
    right = _softmax_rows(scale * a @ k.T)       # [n_agents, N]
    return left @ right


def agent_attn_brute(q, a, k, v, scale: float):
    """Returns (O, M) for one slice; O = M @ V."""
    m = mixing_matrix(q, a, k, scale)
    return m @ np.asarray(v, np.float64), m


def agent_attn_brute_bias(q, a, k, v, scale: float, b1=None, b2=None):
    """Biased twin for one slice: M = softmax_rows(Q A^T s + B2^T) @
    softmax_rows(A K^T s + B1) with b1, b2 given as [n_agents, N]; O = M @ V."""
    q = np.asarray(q, np.float64)
    a = np.asarray(a, np.float64)
    k = np.asarray(k, np.float64)
    n_agents, n = a.shape[0], q.shape[0]
    b1 = np.zeros((n_agents, n)) if b1 is None else np.asarray(b1, np.float64)
    b2 = np.zeros((n_agents, n)) if b2 is None else np.asarray(b2, np.float64)
    left = _softmax_rows(scale * q @ a.T + b2.T)
    right = _softmax_rows(scale * a @ k.T + b1)
    m = left @ right
    return m @ np.asarray(v, np.float64), m
