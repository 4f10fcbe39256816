"""Plain-definition attention in fp64 (TEST INFRASTRUCTURE ONLY; see package docstring).

Follows the definition printed on the "Flash Attention" tag page (guijiagi.com),
excerpt "Flash Attention解决了什么问题", section 算法原理:
    S = Q K^T * scale,  P = softmax(S) row-wise,  O = P V,
with tensors laid out (batch, heads, seq, dim) as in the excerpt
"Flash Attention 系列回顾" (comment on standard_attention).

Causal masking follows "从理论到实现：基于Triton剖析FlashAttention三代的演进与优化"
§3.1: a score (query i, key j) is kept when the query position is at or past
the key position (i >= j), otherwise it is set to -inf.  The comparison
operator is lost in the page text; i >= j is the reading under which causal
row 0 attends to key 0 only.

The log-sum-exp per row is LSE_i = m_i + log(sum_j exp(S_ij - m_i)) in natural
log units, m_i = max_j S_ij.  The pages do not name it; it is the quantity a
recomputing backward pass (same article, §2.2) needs, and the two-pass softmax
below produces it directly.

The score matrix is materialised per (batch, head) in row chunks only to bound
memory; each chunk is the textbook two-pass softmax (max, then exp and sum),
not a tiling of the method.
"""

from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

try:  # keep BLAS single-threaded inside the worker threads
    from threadpoolctl import threadpool_limits
except Exception:  # pragma: no cover - threadpoolctl is in the image
    threadpool_limits = None


def _as_f64(x) -> np.ndarray:
    """Exact widening of bf16/fp16/fp32 tensors or arrays to fp64."""
    if hasattr(x, "detach"):  # torch tensor (CPU); bf16 has no numpy dtype
        import torch

        x = x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def _rows_two_pass(qr, k, v, scale, causal, row_ids):
    """Two-pass softmax attention for the query rows ``row_ids`` of one head.

    qr: [r, d] fp64, k, v: [N, d] fp64.  Returns (o [r, dv], lse [r]).
    """
    s = (qr @ k.T) * scale                       # S = scale * Q K^T
    if causal:
        keys = np.arange(k.shape[0])[None, :]
        s = np.where(keys <= row_ids[:, None], s, -np.inf)   # keep j <= i
    m = s.max(axis=1)                             # pass 1: row max
    e = np.exp(s - m[:, None])                    # pass 2: exponentials
    denom = e.sum(axis=1)
    p = e / denom[:, None]                        # P = softmax(S)
    o = p @ v                                     # O = P V
    lse = m + np.log(denom)
    return o, lse


def attention_ref(q, k, v, scale: float, causal: bool, row_chunk: int = 512,
                  workers: int | None = None):
    """O = softmax(scale * Q K^T [+ causal]) V and LSE, in fp64.

    q, k, v: [B, H, N, d] (numpy or CPU torch, any float dtype; widened to fp64
    exactly).  Returns (o [B, H, N, d] fp64, lse [B, H, N] fp64).
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, H, N, d = q.shape
    o = np.empty((B, H, N, v.shape[-1]), dtype=np.float64)
    lse = np.empty((B, H, N), dtype=np.float64)
    jobs = [(b, h, r0) for b in range(B) for h in range(H)
            for r0 in range(0, N, row_chunk)]

    def run(job):
        b, h, r0 = job
        r1 = min(N, r0 + row_chunk)
        rows = np.arange(r0, r1)
        ob, lb = _rows_two_pass(q[b, h, r0:r1], k[b, h], v[b, h], scale, causal, rows)
        o[b, h, r0:r1] = ob
        lse[b, h, r0:r1] = lb

    workers = workers or os.cpu_count() or 1
    if workers == 1 or len(jobs) == 1:
        for j in jobs:
            run(j)
    else:
        if threadpool_limits is not None:
            with threadpool_limits(limits=1), ThreadPoolExecutor(max_workers=workers) as ex:
                list(ex.map(run, jobs))
        else:
            with ThreadPoolExecutor(max_workers=workers) as ex:
                list(ex.map(run, jobs))
    return o, lse


def attention_rows(q, k, v, scale: float, causal: bool, b: int, h: int, rows):
    """The same definition for a chosen set of query rows of head (b, h).

    Used to check full-size GPU outputs on sampled rows.  Returns
    (o [len(rows), d] fp64, lse [len(rows)] fp64).
    """
    rows = np.asarray(rows, dtype=np.int64)
    qr = _as_f64(q[b, h][rows]) if not hasattr(q, "detach") else _as_f64(q[b, h][rows.tolist()])
    kk = _as_f64(k[b, h])
    vv = _as_f64(v[b, h])
    return _rows_two_pass(qr, kk, vv, scale, causal, rows)


def attention_flops(B: int, H: int, N: int, d: int, causal: bool) -> float:
    """Algorithmic FLOPs of one forward: two GEMMs of 2*N*N*d each per head.

    The per-GEMM count 2*n^2*d matches the IO analysis on the "Flash Attention"
    tag page (excerpt "为什么需要 Flash Attention"): about 16 GFLOP per GEMM at
    n = 8192, d = 128.  Causal attention does half the work (the masked upper
    triangle is never computed).
    """
    f = 4.0 * B * H * float(N) * float(N) * d
    return f / 2.0 if causal else f
