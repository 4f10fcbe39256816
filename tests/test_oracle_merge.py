"""Pins for the partial-result merge and the ring schedule of the oracle
(Ring Attention in "深度解析注意力机制的变体与演进"; the block form of the online
softmax renormalisation of "从理论到实现…" §2.1): merging attention over
disjoint key chunks must give attention over all keys, and a simulated ring
must give the plain (causal) attention of each rank's rows."""

import numpy as np
import pytest

from oracle import attention_ref
from oracle.merge import merge_partials_ref, ring_schedule


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


@pytest.mark.parametrize("chunks", [2, 3, 4])
def test_merging_key_chunks_gives_full_attention(chunks):
    n, d = 24, 5
    q, k, v = (_rand((1, 2, n, d), s) for s in (1, 2, 3))
    full_o, full_l = attention_ref(q, k, v, 0.7, False, workers=1)
    bounds = np.linspace(0, n, chunks + 1).astype(int)
    o = lse = None
    for a, b in zip(bounds[:-1], bounds[1:]):
        po, pl = attention_ref(q, k[:, :, a:b], v[:, :, a:b], 0.7, False, workers=1)
        o, lse = (po, pl) if o is None else merge_partials_ref(o, lse, po, pl)
    assert np.max(np.abs(o - full_o)) <= 1e-12
    assert np.max(np.abs(lse - full_l)) <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("world", [1, 2, 3, 5])
def test_simulated_ring_gives_plain_attention(world, causal):
    n_local, d = 6, 4
    n = world * n_local
    q, k, v = (_rand((1, 1, n, d), s) for s in (4, 5, 6))
    ref_o, ref_l = attention_ref(q, k, v, 0.5, causal, workers=1)
    blk = lambda t, r: t[:, :, r * n_local:(r + 1) * n_local]  # noqa: E731
    for rank in range(world):
        o = lse = None
        for _, src, mode in ring_schedule(rank, world, causal):
            if mode == "skip":
                continue
            po, pl = attention_ref(blk(q, rank), blk(k, src), blk(v, src), 0.5, mode == "causal", workers=1)
            o, lse = (po, pl) if o is None else merge_partials_ref(o, lse, po, pl)
        assert np.max(np.abs(o - blk(ref_o, rank))) <= 1e-12
        assert np.max(np.abs(lse - ref_l[:, :, rank * n_local:(rank + 1) * n_local])) <= 1e-12


def test_schedule_visits_every_block_once():
    for world in (1, 2, 4, 7):
        for rank in range(world):
            srcs = [src for _, src, _ in ring_schedule(rank, world, False)]
            assert sorted(srcs) == list(range(world)) and srcs[0] == rank
            modes = {src: m for _, src, m in ring_schedule(rank, world, True)}
            assert all(modes[s] == ("full" if s < rank else "causal" if s == rank else "skip") for s in srcs)


def test_empty_side_and_symmetry():
    o_a, o_b = _rand((3, 4), 7), _rand((3, 4), 8)
    l_a, l_b = _rand(3, 9), _rand(3, 10)
    empty = np.full(3, -np.inf)
    o, l = merge_partials_ref(o_a, l_a, np.zeros((3, 4)), empty)
    assert np.array_equal(o, o_a) and np.array_equal(l, l_a)
    o, l = merge_partials_ref(np.zeros((3, 4)), empty, np.zeros((3, 4)), empty)
    assert np.all(o == 0) and np.all(np.isneginf(l))
    o1, l1 = merge_partials_ref(o_a, l_a, o_b, l_b)
    o2, l2 = merge_partials_ref(o_b, l_b, o_a, l_a)
    assert np.max(np.abs(o1 - o2)) <= 1e-15 and np.max(np.abs(l1 - l2)) <= 1e-15
    # equal LSEs average the outputs and add log 2
    o, l = merge_partials_ref(o_a, l_a, o_b, l_a)
    assert np.max(np.abs(o - (o_a + o_b) / 2)) <= 1e-15 and np.max(np.abs(l - (l_a + np.log(2)))) <= 1e-15


@pytest.mark.parametrize("kind", ["swapped_weights", "no_renormalise", "max_instead_of_lse"])
def test_chunk_pin_rejects_mutant(kind):
    """Planted mistakes in a copy of the merge are caught by the chunk pin."""
    def mutant(o_a, l_a, o_b, l_b):
        hi = np.maximum(l_a, l_b)
        w_a, w_b = np.exp(l_a - hi), np.exp(l_b - hi)
        if kind == "swapped_weights":
            w_a, w_b = w_b, w_a
        tot = w_a + w_b
        if kind == "no_renormalise":
            tot = np.ones_like(tot)
        lse = hi if kind == "max_instead_of_lse" else hi + np.log(w_a + w_b)
        return (w_a / tot)[..., None] * o_a + (w_b / tot)[..., None] * o_b, lse
    n, d = 16, 3
    q, k, v = (_rand((1, 1, n, d), s) for s in (11, 12, 13))
    full_o, full_l = attention_ref(q, k, v, 1.0, False, workers=1)
    po, pl = attention_ref(q, k[:, :, :7], v[:, :, :7], 1.0, False, workers=1)
    so, sl = attention_ref(q, k[:, :, 7:], v[:, :, 7:], 1.0, False, workers=1)
    o, lse = mutant(po, pl, so, sl)
    assert np.max(np.abs(o - full_o)) > 1e-6 or np.max(np.abs(lse - full_l)) > 1e-6
