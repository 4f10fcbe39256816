"""fp64 merge of partial attention results (TEST INFRASTRUCTURE ONLY; see the
package docstring).

Ring attention ("深度解析注意力机制的变体与演进", section Ring Attention) splits
the sequence over devices: each one attends its query block to one key/value
block at a time and combines the partial results.  Combining is the online
softmax renormalisation ("从理论到实现：基于Triton剖析FlashAttention三代的演进与优化"
§2.1, and "FlashAttention速度提升的核心原理" §1.3) applied to whole blocks: a
partial result over key set A is (O_A, LSE_A) with O_A = softmax over A
applied to V_A and LSE_A = log sum_{j in A} exp(S_ij); for disjoint A and B

    LSE = log(exp(LSE_A) + exp(LSE_B))
    O   = exp(LSE_A - LSE) * O_A + exp(LSE_B - LSE) * O_B

which is the renormalisation step with m replaced by the log-sum-exp.  An
empty key set has LSE = -inf and contributes nothing.
"""

from __future__ import annotations

import numpy as np

from .attention import _as_f64


def merge_partials_ref(o_a, lse_a, o_b, lse_b):
    """Merge two partial results ([..., d] outputs, [...] LSEs) in fp64."""
    o_a, o_b = _as_f64(o_a), _as_f64(o_b)
    lse_a, lse_b = _as_f64(lse_a), _as_f64(lse_b)
    hi = np.maximum(lse_a, lse_b)
    both_empty = np.isneginf(hi)
    safe_hi = np.where(both_empty, 0.0, hi)
    w_a = np.exp(lse_a - safe_hi)                 # exp(-inf) = 0 for an empty side
    w_b = np.exp(lse_b - safe_hi)
    total = w_a + w_b
    lse = np.where(both_empty, -np.inf, safe_hi + np.log(np.where(both_empty, 1.0, total)))
    norm = np.where(both_empty, 1.0, total)
    o = (w_a / norm)[..., None] * o_a + (w_b / norm)[..., None] * o_b
    o = np.where(both_empty[..., None], 0.0, o)
    return o, lse


def ring_schedule(rank: int, world: int, causal: bool):
    """The K/V block each ring step brings to `rank`, and how it is attended.

    Step s holds the block that started on rank (rank - s) mod world (blocks
    travel to the next rank each step).  With equal contiguous sequence blocks
    and the causal mask, a block from an earlier rank is attended in full,
    the rank's own block with the causal mask, and a later one not at all.
    Returns [(step, source_rank, mode)] with mode in {"full", "causal", "skip"}.
    """
    out = []
    for s in range(world):
        src = (rank - s) % world
        if not causal:
            mode = "full"
        elif src < rank:
            mode = "full"
        elif src == rank:
            mode = "causal"
        else:
            mode = "skip"
        out.append((s, src, mode))
    return out
