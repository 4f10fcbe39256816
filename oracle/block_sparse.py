"""Block-sparse attention in fp64 (TEST INFRASTRUCTURE ONLY; see package docstring).

Follows "深度解析注意力机制的变体与演进", section "Block Sparse Attention": the
attention matrix is cut into fixed-size blocks and only some of the blocks are
computed, with full attention inside a computed block and none through a
skipped one.  The page gives neither the block size nor how the chosen blocks
are described; the reading used here:

  * a boolean block mask M of shape [B, H, ceil(N / bs), ceil(N / bs)];
  * the score of (query i, key j) is kept when M[b, h, i // bs, j // bs] is
    set and, with the causal flag, when i >= j (the causal reading of
    "从理论到实现：基于Triton剖析FlashAttention三代的演进与优化" §3.1); every other
    score is -inf before the softmax;
  * a row that keeps no score has an empty softmax: its output row is zero and
    its log-sum-exp is -inf.

Otherwise the definition is the plain one of the "Flash Attention" tag page
(excerpt "Flash Attention解决了什么问题", 算法原理): S = scale * Q K^T,
P = softmax(S) row-wise, O = P V, and LSE_i = m_i + log sum_j exp(S_ij - m_i).
"""

from __future__ import annotations

import numpy as np

from .attention import _as_f64


def _keep_matrix(mask_bh: np.ndarray, rows: np.ndarray, n_keys: int, block: int, causal: bool) -> np.ndarray:
    """Element-level keep matrix [len(rows), n_keys] of one head."""
    keys = np.arange(n_keys)
    keep = mask_bh[rows[:, None] // block, keys[None, :] // block].astype(bool)
    if causal:
        keep &= keys[None, :] <= rows[:, None]
    return keep


def _rows(qr, k, v, scale, keep):
    s = (qr @ k.T) * scale
    s = np.where(keep, s, -np.inf)
    o = np.zeros((qr.shape[0], v.shape[1]))
    lse = np.full(qr.shape[0], -np.inf)
    live = keep.any(axis=1)
    if live.any():
        sl = s[live]
        m = sl.max(axis=1)                        # pass 1: row max
        e = np.exp(sl - m[:, None])               # pass 2: exponentials
        denom = e.sum(axis=1)
        o[live] = (e / denom[:, None]) @ v        # O = softmax(S) V
        lse[live] = m + np.log(denom)
    return o, lse


def attention_block_sparse_ref(q, k, v, scale: float, causal: bool, block_mask, block: int = 128,
                               row_chunk: int = 512):
    """O and LSE in fp64 for [B, H, N, d] inputs and a [B, H, nb, nb] block mask
    (any dtype; nonzero = computed block).  Returns (o, lse)."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    mask = np.asarray(block_mask.cpu().numpy() if hasattr(block_mask, "cpu") else block_mask) != 0
    B, H, N, _ = q.shape
    nb = -(-N // block)
    assert mask.shape == (B, H, nb, nb), (mask.shape, (B, H, nb, nb))
    o = np.empty((B, H, N, v.shape[-1]))
    lse = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            for r0 in range(0, N, row_chunk):
                rows = np.arange(r0, min(N, r0 + row_chunk))
                keep = _keep_matrix(mask[b, h], rows, N, block, causal)
                o[b, h, rows], lse[b, h, rows] = _rows(q[b, h, rows], k[b, h], v[b, h], scale, keep)
    return o, lse


def attention_block_sparse_rows(q, k, v, scale: float, causal: bool, block_mask, b: int, h: int, rows,
                                block: int = 128):
    """The same definition for chosen query rows of head (b, h) (sampled checks
    of full-size outputs).  Returns (o [len(rows), d], lse [len(rows)])."""
    rows = np.asarray(rows, dtype=np.int64)
    mask = np.asarray(block_mask.cpu().numpy() if hasattr(block_mask, "cpu") else block_mask) != 0
    qr = _as_f64(q[b, h][rows.tolist()] if hasattr(q, "detach") else q[b, h][rows])
    kk, vv = _as_f64(k[b, h]), _as_f64(v[b, h])
    keep = _keep_matrix(mask[b, h], rows, kk.shape[0], block, causal)
    return _rows(qr, kk, vv, scale, keep)


def block_sparse_flops(block_mask, N: int, d: int, causal: bool, block: int = 128) -> float:
    """Algorithmic FLOPs: 4 * d per kept (query, key) pair (two GEMMs of
    2 * d each), counted exactly from the mask and the causal predicate."""
    mask = np.asarray(block_mask.cpu().numpy() if hasattr(block_mask, "cpu") else block_mask) != 0
    nb = mask.shape[-1]
    sizes = np.minimum(block, N - np.arange(nb) * block)          # rows (or keys) per block
    full = sizes[:, None] * sizes[None, :]
    if causal:
        # diagonal blocks keep the lower triangle with the diagonal; blocks
        # above the diagonal keep nothing
        pairs = np.where(np.arange(nb)[:, None] > np.arange(nb)[None, :], full, 0).astype(np.float64)
        diag = sizes * (sizes + 1) / 2.0
        pairs[np.arange(nb), np.arange(nb)] = diag
    else:
        pairs = full.astype(np.float64)
    kept = (mask * pairs[None, None]).sum()
    return 4.0 * d * float(kept)
