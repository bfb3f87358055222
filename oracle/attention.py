"""Exact softmax attention in fp64.

Definition followed: [P1] sections 2 and 6, [P4] and the [P3] passage on
bidirectional attention -- every packed row attends to every packed row
(full, non-causal, no mask, no segment masking).  Per head:

    s_ij = q_i . k_j * scale           (scale = 1/sqrt(D) unless given)
    o_i  = sum_j softmax_j(s_i) v_j
    lse_i = log sum_j exp(s_ij)

The softmax subtracts the row maximum before exponentiating (the same value
in exact arithmetic).  Matrix products use numpy's matmul.
"""
from __future__ import annotations

import numpy as np


def attention_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float | None = None,
                   chunk: int = 512):
    """q [M, D], k [N, D], v [N, Dv] (fp64) -> (o [M, Dv], lse [M])."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    if scale is None:
        scale = 1.0 / np.sqrt(q.shape[-1])
    M = q.shape[0]
    o = np.empty((M, v.shape[1]), np.float64)
    lse = np.empty(M, np.float64)
    for r0 in range(0, M, chunk):
        s = (q[r0:r0 + chunk] @ k.T) * scale
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        l = p.sum(axis=1, keepdims=True)
        o[r0:r0 + chunk] = (p @ v) / l
        lse[r0:r0 + chunk] = (m + np.log(l))[:, 0]
    return o, lse


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float | None = None):
    """q [M, H, D], k/v [N, H, D] -> o [M, H, D], lse [H, M]."""
    M, H, _ = q.shape
    o = np.empty((M, H, v.shape[2]), np.float64)
    lse = np.empty((H, M), np.float64)
    for h in range(H):
        o[:, h], lse[h] = attention_head(q[:, h], k[:, h], v[:, h], scale)
    return o, lse
