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


def attention_bwd_rows(q, k, v, do, scale: float, causal: bool, b: int, h: int, q_rows, k_rows):
    """The same gradients of head (b, h) for chosen rows only, for checking
    full-size results on a sample: dQ at the query rows ``q_rows``, dK and dV
    at the key rows ``k_rows``.

    A dQ row needs only its own row of P and dS; a dK or dV row needs only its
    column of them.  LSE and D of every query row come from the forward written
    out row chunk by row chunk (the plain definition, as in attention_ref).
    Returns (dq [len(q_rows), d], dk [len(k_rows), d], dv [len(k_rows), d])."""
    from .attention import attention_ref

    q_rows = np.asarray(q_rows, dtype=np.int64)
    k_rows = np.asarray(k_rows, dtype=np.int64)
    qh, kh, vh, gh = (_as_f64(t[b:b + 1, h:h + 1]) for t in (q, k, v, do))
    o, lse = attention_ref(qh, kh, vh, scale, causal)
    qh, kh, vh, gh, o, lse = qh[0, 0], kh[0, 0], vh[0, 0], gh[0, 0], o[0, 0], lse[0, 0]
    n = qh.shape[0]
    dd = np.sum(gh * o, axis=1)                               # D_i = sum_c dO_ic O_ic
    # dQ rows: P and dS along the row
    s = scale * (qh[q_rows] @ kh.T)
    if causal:
        s = np.where(np.arange(n)[None, :] <= q_rows[:, None], s, -np.inf)
    p = np.exp(s - lse[q_rows, None])
    ds = p * (gh[q_rows] @ vh.T - dd[q_rows, None])
    dq = scale * ds @ kh
    # dK, dV rows: P and dS down the column
    st = scale * (qh @ kh[k_rows].T)                          # [n, len(k_rows)]
    if causal:
        st = np.where(np.arange(n)[:, None] >= k_rows[None, :], st, -np.inf)
    pt = np.exp(st - lse[:, None])
    dst = pt * (gh @ vh[k_rows].T - dd[:, None])
    dv = pt.T @ gh
    dk = scale * dst.T @ qh
    return dq, dk, dv
