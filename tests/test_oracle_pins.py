"""Pins for the fp64 oracle: brute force, closed forms and invariants.

Each test ties the oracle to something other than itself: a pure-Python
restatement, a closed form, or an invariant the pages' method must satisfy.
"""

import math

import numpy as np
import pytest

from oracle import attention_ref, attention_rows, brute_attention, online_attention


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n,d", [(1, 1), (3, 2), (7, 5), (16, 8), (11, 3)])
def test_oracle_matches_brute_force(n, d, causal):
    q, k, v = (_rand((1, 1, n, d), s) for s in (1, 2, 3))
    scale = 1.0 / math.sqrt(d)
    o, lse = attention_ref(q, k, v, scale, causal, row_chunk=4, workers=2)
    ob, lb = brute_attention(q[0, 0].tolist(), k[0, 0].tolist(), v[0, 0].tolist(), scale, causal)
    assert np.max(np.abs(o[0, 0] - np.array(ob))) <= 1e-12
    assert np.max(np.abs(lse[0, 0] - np.array(lb))) <= 1e-12


def test_brute_force_values_by_hand():
    # two keys, one query: weights e^{s}/(e^{s0}+e^{s1}) worked out by hand
    q = [[1.0, 0.0]]
    k = [[2.0, 0.0], [0.0, 5.0]]
    v = [[10.0], [20.0]]
    o, lse = brute_attention(q, k, v, 1.0, False)
    w0 = math.exp(2.0) / (math.exp(2.0) + math.exp(0.0))
    assert abs(o[0][0] - (10 * w0 + 20 * (1 - w0))) < 1e-14
    assert abs(lse[0] - math.log(math.exp(2.0) + 1.0)) < 1e-14


@pytest.mark.parametrize("causal", [False, True])
def test_rows_sum_to_one(causal):
    """softmax rows sum to 1: a V column of ones comes back as ones."""
    q, k = _rand((2, 2, 40, 8), 4), _rand((2, 2, 40, 8), 5)
    v = _rand((2, 2, 40, 8), 6)
    v[..., 0] = 1.0
    o, _ = attention_ref(q, k, v, 0.3, causal, row_chunk=16)
    assert np.max(np.abs(o[..., 0] - 1.0)) <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_identical_v_rows_return_that_row(causal):
    q, k = _rand((1, 2, 33, 4), 7, 3.0), _rand((1, 2, 33, 4), 8, 3.0)
    row = _rand((4,), 9)
    v = np.broadcast_to(row, (1, 2, 33, 4)).copy()
    o, _ = attention_ref(q, k, v, 0.5, causal)
    assert np.max(np.abs(o - row)) <= 1e-12


def test_causal_row_zero_is_v0():
    q, k, v = (_rand((1, 3, 20, 6), s) for s in (10, 11, 12))
    o, lse = attention_ref(q, k, v, 0.4, True)
    assert np.array_equal(o[:, :, 0], v[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], 0.4 * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0]),
                               rtol=0, atol=1e-13)


@pytest.mark.parametrize("zero", ["q", "k"])
def test_zero_q_or_k_gives_uniform_weights(zero):
    n, d = 25, 4
    q, k, v = (_rand((1, 1, n, d), s) for s in (13, 14, 15))
    if zero == "q":
        q[:] = 0
    else:
        k[:] = 0
    o, lse = attention_ref(q, k, v, 1.0, False)
    assert np.max(np.abs(o[0, 0] - v[0, 0].mean(axis=0))) <= 1e-12
    assert np.max(np.abs(lse - math.log(n))) <= 1e-12
    o, lse = attention_ref(q, k, v, 1.0, True)
    prefix = np.cumsum(v[0, 0], axis=0) / np.arange(1, n + 1)[:, None]
    assert np.max(np.abs(o[0, 0] - prefix)) <= 1e-12
    assert np.max(np.abs(lse[0, 0] - np.log(np.arange(1, n + 1)))) <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("block", [1, 7, 64, 128])
@pytest.mark.parametrize("tau", [0.0, 8.0 * math.log(2.0)])
def test_online_recurrence_equals_two_pass(causal, block, tau):
    n, d = 300, 16
    q, k, v = (_rand((n, d), s, 2.0) for s in (16, 17, 18))
    o1, l1 = online_attention(q, k, v, 0.25, causal, block, tau)
    o2, l2 = attention_ref(q[None, None], k[None, None], v[None, None], 0.25, causal)
    assert np.max(np.abs(o1 - o2[0, 0])) <= 1e-12
    assert np.max(np.abs(l1 - l2[0, 0])) <= 1e-12


def test_online_lazy_rule_really_defers():
    """With a large tau the running max stays stale, yet the result is unchanged."""
    n, d = 64, 4
    q = np.ones((n, d))
    k = np.zeros((n, d))
    k[np.arange(n), 0] = np.linspace(0, 5, n)   # scores grow along the keys
    v = _rand((n, d), 19)
    o_eager, _ = online_attention(q, k, v, 1.0, False, block=8, tau=0.0)
    o_lazy, _ = online_attention(q, k, v, 1.0, False, block=8, tau=100.0)
    assert np.max(np.abs(o_eager - o_lazy)) <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_lse_bounds(causal):
    n, d = 50, 8
    q, k, v = (_rand((1, 1, n, d), s) for s in (20, 21, 22))
    _, lse = attention_ref(q, k, v, 0.7, causal)
    s = 0.7 * q[0, 0] @ k[0, 0].T
    if causal:
        s = np.where(np.tril(np.ones((n, n))) > 0, s, -np.inf)
    mx = s.max(axis=1)
    count = np.isfinite(s).sum(axis=1)
    assert np.all(lse[0, 0] >= mx - 1e-12)
    assert np.all(lse[0, 0] <= mx + np.log(count) + 1e-12)
    assert lse[0, 0, 0] >= s[0, 0] - 1e-12
    if causal:
        assert abs(lse[0, 0, 0] - s[0, 0]) <= 1e-13


def test_large_scores_are_stable_and_pick_the_argmax():
    n, d = 40, 16
    q, k, v = (_rand((1, 1, n, d), s) for s in (23, 24, 25))
    o, lse = attention_ref(q * 100, k * 100, v, 1.0 / 4.0, False)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    s = (q[0, 0] * 100) @ (k[0, 0] * 100).T / 4.0
    top = s.argmax(axis=1)
    gap = np.sort(s, axis=1)[:, -1] - np.sort(s, axis=1)[:, -2]
    sure = gap > 50          # rows whose winner leads by e^50
    assert sure.sum() > n // 2
    assert np.max(np.abs(o[0, 0][sure] - v[0, 0][top[sure]])) <= 1e-12


def test_single_key_returns_v():
    q, k, v = (_rand((2, 3, 1, 8), s) for s in (26, 27, 28))
    for causal in (False, True):
        o, lse = attention_ref(q, k, v, 0.3, causal)
        assert np.array_equal(o, v)
        np.testing.assert_allclose(lse, 0.3 * np.sum(q * k, axis=-1), rtol=0, atol=1e-13)


def test_noncausal_is_invariant_to_key_order():
    """Permuting keys and values together changes nothing (catches K/V index slips)."""
    n, d = 37, 8
    q, k, v = (_rand((1, 1, n, d), s) for s in (29, 30, 31))
    perm = np.random.default_rng(32).permutation(n)
    o1, l1 = attention_ref(q, k, v, 0.5, False)
    o2, l2 = attention_ref(q, k[:, :, perm], v[:, :, perm], 0.5, False)
    assert np.max(np.abs(o1 - o2)) <= 1e-12 and np.max(np.abs(l1 - l2)) <= 1e-12


def test_sampled_rows_match_full_oracle():
    q, k, v = (_rand((2, 2, 300, 16), s) for s in (33, 34, 35))
    o, lse = attention_ref(q, k, v, 0.25, True, row_chunk=64)
    rows = [0, 1, 127, 128, 255, 299]
    orr, lr = attention_rows(q, k, v, 0.25, True, 1, 1, rows)
    assert np.max(np.abs(orr - o[1, 1, rows])) <= 1e-13
    assert np.max(np.abs(lr - lse[1, 1, rows])) <= 1e-13


def test_oracle_accepts_torch_bf16_exactly():
    import torch

    from tiled_attention_12_b200.synth import WORKLOADS, make_qkv

    case = WORKLOADS["tiny"].cases[0]
    q, k, v = make_qkv(case)
    assert q.dtype == torch.bfloat16
    o, lse = attention_ref(q[:, :, :32], k[:, :, :32], v[:, :, :32], case.softmax_scale, False)
    o2, _ = attention_ref(q[:, :, :32].float().numpy(), k[:, :, :32].float().numpy(),
                          v[:, :, :32].float().numpy(), case.softmax_scale, False)
    assert np.array_equal(o, o2)
