"""Pins for the block-sparse oracle ("深度解析注意力机制的变体与演进", Block
Sparse Attention): brute force with an explicit keep predicate, reductions to
the dense oracle, independence of block-diagonal problems, empty rows, and the
exact FLOP count."""

import math

import numpy as np
import pytest

from oracle import attention_ref, brute_attention
from oracle.block_sparse import attention_block_sparse_ref, attention_block_sparse_rows, block_sparse_flops


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,d,bs", [(7, 3, 2), (12, 4, 4), (10, 2, 3), (9, 5, 1)])
def test_matches_brute_force(n, d, bs, causal):
    q, k, v = (_rand((1, 1, n, d), s) for s in (21, 22, 23))
    nb = -(-n // bs)
    mask = np.random.default_rng(n * 7 + bs).random((1, 1, nb, nb)) < 0.5
    mask[0, 0, 0, 0] = True
    o, lse = attention_block_sparse_ref(q, k, v, 0.6, causal, mask, block=bs, row_chunk=3)
    keep = lambda i, j: bool(mask[0, 0, i // bs, j // bs])  # noqa: E731
    ob, lb = brute_attention(q[0, 0].tolist(), k[0, 0].tolist(), v[0, 0].tolist(), 0.6, causal, keep=keep)
    assert np.max(np.abs(o[0, 0] - np.array(ob))) <= 1e-12
    lb = np.array(lb)
    assert np.array_equal(np.isinf(lse[0, 0]), np.isinf(lb))
    fin = np.isfinite(lb)
    assert np.max(np.abs(lse[0, 0][fin] - lb[fin]), initial=0.0) <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_all_blocks_equals_dense(causal):
    q, k, v = (_rand((2, 2, 70, 6), s) for s in (1, 2, 3))
    mask = np.ones((2, 2, 5, 5), dtype=np.uint8)
    o, lse = attention_block_sparse_ref(q, k, v, 0.4, causal, mask, block=16)
    od, ld = attention_ref(q, k, v, 0.4, causal, workers=1)
    assert np.max(np.abs(o - od)) <= 1e-12 and np.max(np.abs(lse - ld)) <= 1e-12


def test_block_diagonal_is_independent_problems():
    """With only the diagonal blocks computed, each block of rows is a separate
    attention problem over its own keys."""
    n, bs = 50, 16
    q, k, v = (_rand((1, 1, n, 4), s) for s in (4, 5, 6))
    nb = -(-n // bs)
    mask = np.eye(nb, dtype=bool)[None, None]
    for causal in (False, True):
        o, lse = attention_block_sparse_ref(q, k, v, 0.5, causal, mask, block=bs)
        for r0 in range(0, n, bs):
            sl = slice(r0, min(n, r0 + bs))
            od, ld = attention_ref(q[:, :, sl], k[:, :, sl], v[:, :, sl], 0.5, causal, workers=1)
            assert np.max(np.abs(o[:, :, sl] - od)) <= 1e-12
            assert np.max(np.abs(lse[:, :, sl] - ld)) <= 1e-12


def test_first_key_block_only():
    """Every row keeps key block 0 only: dense attention over the first bs keys."""
    n, bs = 40, 8
    q, k, v = (_rand((1, 1, n, 3), s) for s in (7, 8, 9))
    mask = np.zeros((1, 1, 5, 5), dtype=bool)
    mask[..., 0] = True
    o, lse = attention_block_sparse_ref(q, k, v, 1.0, False, mask, block=bs)
    od, ld = attention_ref(q, k[:, :, :bs], v[:, :, :bs], 1.0, False, workers=1)
    assert np.max(np.abs(o - od)) <= 1e-12 and np.max(np.abs(lse - ld)) <= 1e-12


def test_empty_rows_are_zero_with_minus_inf_lse():
    n, bs = 20, 4
    q, k, v = (_rand((1, 1, n, 3), s) for s in (10, 11, 12))
    mask = np.ones((1, 1, 5, 5), dtype=bool)
    mask[0, 0, 2, :] = False             # rows 8..11 keep nothing
    mask[0, 0, 4, 4] = False             # causal: rows 16..19 still keep blocks 0..3
    for causal in (False, True):
        o, lse = attention_block_sparse_ref(q, k, v, 1.0, causal, mask, block=bs)
        assert np.all(o[0, 0, 8:12] == 0.0) and np.all(np.isneginf(lse[0, 0, 8:12]))
        assert np.all(np.isfinite(lse[0, 0, :8])) and np.all(np.isfinite(lse[0, 0, 12:]))
    # causal with the diagonal block of row block 0 removed: rows 0..3 keep nothing
    mask = np.ones((1, 1, 5, 5), dtype=bool)
    mask[0, 0, 0, 0] = False
    o, lse = attention_block_sparse_ref(q, k, v, 1.0, True, mask, block=bs)
    assert np.all(o[0, 0, :4] == 0.0) and np.all(np.isneginf(lse[0, 0, :4]))


def test_rows_helper_matches_full():
    q, k, v = (_rand((1, 2, 37, 4), s) for s in (13, 14, 15))
    mask = np.random.default_rng(3).random((1, 2, 5, 5)) < 0.6
    o, lse = attention_block_sparse_ref(q, k, v, 0.7, True, mask, block=8)
    rows = [0, 5, 17, 36]
    orow, lrow = attention_block_sparse_rows(q, k, v, 0.7, True, mask, 0, 1, rows, block=8)
    assert np.array_equal(orow, o[0, 1, rows]) and np.array_equal(lrow, lse[0, 1, rows])


@pytest.mark.parametrize("causal", [False, True])
def test_flop_count_by_enumeration(causal):
    n, bs, d = 23, 5, 3
    nb = -(-n // bs)
    mask = np.random.default_rng(9).random((1, 2, nb, nb)) < 0.5
    kept = 0
    for h in range(2):
        for i in range(n):
            for j in range(n):
                if mask[0, h, i // bs, j // bs] and (not causal or j <= i):
                    kept += 1
    assert block_sparse_flops(mask, n, d, causal, block=bs) == 4.0 * d * kept
    full = np.ones((1, 1, nb, nb))
    assert block_sparse_flops(full, n, d, False, block=bs) == 4.0 * d * n * n
    assert block_sparse_flops(full, n, d, True, block=bs) == 4.0 * d * n * (n + 1) / 2


def _mutant_keep(kind, mask, block, causal, n):
    """Plausible mistakes in the block-sparse keep matrix."""
    rows = np.arange(n)[:, None]
    keys = np.arange(n)[None, :]
    if kind == "transposed_mask":
        keep = mask[keys // block, rows // block]
    elif kind == "block_of_row_for_key":
        keep = mask[rows // block, rows // block] & np.ones_like(keys, dtype=bool)
    elif kind == "off_by_one_block":
        keep = mask[np.minimum(rows // block + 1, mask.shape[0] - 1), keys // block]
    else:
        keep = mask[rows // block, keys // block]
    if causal and kind != "drop_causal":
        keep = keep & (keys <= rows)
    return keep


@pytest.mark.parametrize("kind", ["transposed_mask", "block_of_row_for_key", "off_by_one_block", "drop_causal"])
def test_brute_force_pin_rejects_mutant(kind):
    """A mutated keep rule inside the oracle's row routine disagrees with the
    brute force on some seeded case."""
    from oracle.block_sparse import _rows
    n, bs, d = 12, 4, 3
    q, k, v = (_rand((n, d), s) for s in (31, 32, 33))
    rejected = False
    for seed in range(4):
        mask = np.random.default_rng(seed).random((3, 3)) < 0.5
        mask[:, 0] = True
        for causal in (False, True):
            keep = _mutant_keep(kind, mask, bs, causal, n)
            o, _ = _rows(q, k, v, 0.8, keep)
            ob, _ = brute_attention(q.tolist(), k.tolist(), v.tolist(), 0.8, causal,
                                    keep=lambda i, j: bool(mask[i // bs, j // bs]))
            if np.max(np.abs(o - np.array(ob))) > 1e-9:
                rejected = True
    assert rejected, kind
