"""The pages' online-softmax recurrence, block by block, in fp64.

TEST INFRASTRUCTURE ONLY (see package docstring).  This is not the oracle the
GPU is compared with; it exists so the tests can check that the recurrence the
kernel implements reaches the plain two-pass definition.

Recurrence, as stated in "从理论到实现：基于Triton剖析FlashAttention三代的演进与优化"
§2.1 (operators lost in the page text are restored as the only readings that
type-check), and in block form on the "Flash Attention" tag page, excerpt
"注意力计算的性能瓶颈", paragraph 在线Softmax:

    m_new = max(m, rowmax(S_blk))
    alpha = exp(m - m_new)                # rescale of everything so far
    beta  = exp(S_blk - m_new)            # this block's exponentials
    l     = alpha * l + rowsum(beta)
    acc   = alpha * acc + beta @ V_blk
    O     = acc / l                       # once, at the end

The division by l is deferred to the end, the order the tag page attributes to
FlashAttention V2 (paragraph 减少非矩阵乘法运算).

``tau`` adds the deferred-rescale rule: the running max is only moved when the
block max exceeds it by more than ``tau`` (natural-log units); otherwise the
block is exponentiated against the stale max.  acc and l share that stale
reference, so O = acc / l is unchanged in exact arithmetic; tau = 0 is the
plain recurrence above.
"""

from __future__ import annotations

import numpy as np


def online_attention(q, k, v, scale: float, causal: bool, block: int, tau: float = 0.0):
    """Block-by-block online softmax for one head.

    q: [N, d], k: [N, d], v: [N, dv] (fp64 arrays).  Keys are visited in blocks
    of ``block``; every query row is processed at once (the recurrence is per
    row, so the query blocking does not change any value).  Returns (o, lse).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n_q, n_k = q.shape[0], k.shape[0]
    rows = np.arange(n_q)[:, None]
    m = np.full(n_q, -np.inf)
    l = np.zeros(n_q)
    acc = np.zeros((n_q, v.shape[1]))
    for j0 in range(0, n_k, block):
        j1 = min(n_k, j0 + block)
        s = (q @ k[j0:j1].T) * scale
        if causal:
            keys = np.arange(j0, j1)[None, :]
            s = np.where(keys <= rows, s, -np.inf)
        blk_max = s.max(axis=1)
        cand = np.maximum(m, blk_max)
        # deferred rule: move the max only when it grew by more than tau
        # (always on the first finite block, where m is still -inf)
        move = (cand - m > tau) | np.isneginf(m)
        m_new = np.where(move, cand, m)
        # alpha = exp(m - m_new); m = -inf (nothing accumulated yet) gives 0
        with np.errstate(invalid="ignore"):
            alpha = np.where(np.isneginf(m), 0.0, np.exp(m - m_new))
        # rows with every key of this block masked keep m_new = -inf and
        # contribute nothing
        with np.errstate(invalid="ignore"):
            beta = np.where(np.isneginf(s), 0.0, np.exp(s - m_new[:, None]))
        l = alpha * l + beta.sum(axis=1)
        acc = alpha[:, None] * acc + beta @ v[j0:j1]
        m = m_new
    o = acc / l[:, None]
    lse = m + np.log(l)
    return o, lse
