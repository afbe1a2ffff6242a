"""Dense softmax attention in float64: the reference for the in-library softmax baseline.

Test infrastructure only. P = softmax(scale * Q K^T) over the allowed keys (j <= i when causal),
O = P V, lse = log sum_j exp(scale * q_i . k_j); backward dS = P * (dO V^T - rowsum(dO * O)),
dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO.
"""
from __future__ import annotations

import numpy as np

from .attention import allowed, scores


def forward(Q, K, V, causal, scale=None, chunk=256):
    Q = np.asarray(Q)
    B, H, n, d = Q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    O = np.zeros((B, H, n, np.asarray(V).shape[-1]))
    lse = np.zeros((B, H, n))
    for b in range(B):
        for h in range(H):
            for c0 in range(0, n, chunk):
                rows = np.arange(c0, min(n, c0 + chunk))
                s = np.where(allowed(rows, n, causal), scores(Q[b, h][rows], K[b, h], scale), -np.inf)
                m = s.max(axis=1, keepdims=True)
                e = np.exp(s - m)
                l = e.sum(axis=1, keepdims=True)
                O[b, h, rows] = (e / l) @ np.asarray(V[b, h], np.float64)
                lse[b, h, rows] = (m + np.log(l))[:, 0]
    return O, lse


def backward(Q, K, V, dO, causal, scale=None, chunk=256):
    Q = np.asarray(Q)
    B, H, n, d = Q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    dQ = np.zeros((B, H, n, d))
    dK = np.zeros((B, H, n, d))
    dV = np.zeros((B, H, n, np.asarray(V).shape[-1]))
    for b in range(B):
        for h in range(H):
            q = np.asarray(Q[b, h], np.float64)
            k = np.asarray(K[b, h], np.float64)
            v = np.asarray(V[b, h], np.float64)
            do = np.asarray(dO[b, h], np.float64)
            for c0 in range(0, n, chunk):
                rows = np.arange(c0, min(n, c0 + chunk))
                s = np.where(allowed(rows, n, causal), scores(q[rows], k, scale), -np.inf)
                e = np.exp(s - s.max(axis=1, keepdims=True))
                p = e / e.sum(axis=1, keepdims=True)
                o = p @ v
                g = do[rows] @ v.T
                ds = p * (g - (do[rows] * o).sum(axis=1, keepdims=True))
                dQ[b, h, rows] = scale * (ds @ k)
                dK[b, h] += scale * (ds.T @ q[rows])
                dV[b, h] += p.T @ do[rows]
    return dQ, dK, dV
