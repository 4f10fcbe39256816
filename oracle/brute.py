"""Pure-Python brute-force attention for tiny inputs.

TEST INFRASTRUCTURE ONLY (see package docstring).  It restates the plain
definition from the "Flash Attention" tag page (excerpt "Flash Attention解决了
什么问题", section 算法原理: S = QK^T * scale, P = softmax(S), O = PV) with
Python floats and explicit loops, with no numpy, so that the fp64 oracle can be
checked against code that shares nothing with it.  Causal keeps key j for
query i when i >= j ("从理论到实现…" §3.1).
"""

from __future__ import annotations

import math


def brute_attention(q, k, v, scale: float, causal: bool, keep=None):
    """q, k, v: nested lists [N][d] of floats.  Returns (o [N][dv], lse [N]).

    ``keep(i, j)``, when given, further restricts which keys query i sees
    (block-sparse attention); a query that sees no key gets a zero row and
    LSE = -inf (an empty softmax)."""
    n_q, n_k = len(q), len(k)
    d = len(q[0])
    dv = len(v[0])
    o, lse = [], []
    for i in range(n_q):
        scores = []
        for j in range(n_k):
            if causal and j > i:
                continue
            if keep is not None and not keep(i, j):
                continue
            dot = 0.0
            for c in range(d):
                dot += q[i][c] * k[j][c]
            scores.append((j, dot * scale))
        if not scores:
            o.append([0.0] * dv)
            lse.append(-math.inf)
            continue
        big = max(s for _, s in scores)
        weights = [(j, math.exp(s - big)) for j, s in scores]
        total = sum(w for _, w in weights)
        row = [0.0] * dv
        for j, w in weights:
            for c in range(dv):
                row[c] += (w / total) * v[j][c]
        o.append(row)
        lse.append(big + math.log(total))
    return o, lse
