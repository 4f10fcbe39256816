"""fp64 gradients of attention (TEST INFRASTRUCTURE ONLY; see package docstring).

The backward pass the pages plan for the forward's saved statistics: no
intermediate is stored, S and P are recomputed from Q, K and the per-row
log-sum-exp ("从理论到实现：基于Triton剖析FlashAttention三代的演进与优化" §2.2,
重计算机制: intermediate results are recomputed in backpropagation rather than
stored).  For O = softmax(S) V with S = scale * Q K^T (causal: j <= i):

    P   = exp(S - LSE)                      (rows of P sum to 1)
    dV  = P^T dO
    dP  = dO V^T
    D_i = sum_c dO_ic O_ic                  (= sum_j P_ij dP_ij)
    dS  = P * (dP - D)                      (softmax Jacobian, row-wise)
    dQ  = scale * dS K
    dK  = scale * dS^T Q

These are the chain rule through the plain definition; the oracle writes them
out per (batch, head) with materialised matrices.
"""

from __future__ import annotations

import numpy as np

from .attention import _as_f64


def attention_bwd_ref(q, k, v, do, scale: float, causal: bool):
    """Returns (dq, dk, dv) in fp64 for [B, H, N, d] inputs and upstream dO."""
    q, k, v, do = (_as_f64(t) for t in (q, k, v, do))
    B, H, N, d = q.shape
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    keys = np.arange(N)[None, :]
    rows = np.arange(N)[:, None]
    for b in range(B):
        for h in range(H):
            s = scale * (q[b, h] @ k[b, h].T)
            if causal:
                s = np.where(keys <= rows, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            p = e / e.sum(axis=1, keepdims=True)
            o = p @ v[b, h]
            dv[b, h] = p.T @ do[b, h]
            dp = do[b, h] @ v[b, h].T
            dd = np.sum(do[b, h] * o, axis=1, keepdims=True)
            ds = p * (dp - dd)
            dq[b, h] = scale * (ds @ k[b, h])
            dk[b, h] = scale * (ds.T @ q[b, h])
    return dq, dk, dv


def attention_bwd_d(o, do) -> np.ndarray:
    """D = rowsum(dO * O) in fp64, [B, H, N] (the backward's pre-pass)."""
    return np.sum(_as_f64(o) * _as_f64(do), axis=-1)
