"""Pins for the fp64 backward oracle: central finite differences of the
forward definition, closed forms, and identities the gradients satisfy."""

import math

import numpy as np
import pytest

from oracle import attention_bwd_d, attention_bwd_ref, attention_ref, brute_attention


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _loss(q, k, v, g, scale, causal):
    """L = sum(O * G) through the pure-Python brute force (independent of the
    numpy oracle)."""
    o, _ = brute_attention(q.tolist(), k.tolist(), v.tolist(), scale, causal)
    return float(np.sum(np.array(o) * g))


@pytest.mark.parametrize("causal", [False, True])
def test_gradients_match_finite_differences(causal):
    n, d = 6, 4
    q, k, v = (_rand((n, d), s) for s in (1, 2, 3))
    g = _rand((n, d), 4)
    scale = 0.7
    dq, dk, dv = attention_bwd_ref(q[None, None], k[None, None], v[None, None], g[None, None], scale, causal)
    eps = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            num[idx] = (_loss(args_p["q"], args_p["k"], args_p["v"], g, scale, causal)
                        - _loss(args_m["q"], args_m["k"], args_m["v"], g, scale, causal)) / (2 * eps)
        assert np.max(np.abs(num - grad[0, 0])) < 1e-6, name


def test_dv_closed_form_for_zero_q():
    """Q = 0 makes P uniform over each row's visible keys, so
    causal: dV_j = sum_{i >= j} dO_i / (i + 1);  non-causal: dV_j = sum_i dO_i / n."""
    n, d = 9, 3
    k, v, g = (_rand((1, 1, n, d), s) for s in (5, 6, 7))
    q = np.zeros((1, 1, n, d))
    _, _, dv = attention_bwd_ref(q, k, v, g, 1.0, True)
    w = 1.0 / np.arange(1, n + 1)
    expect = np.array([np.sum(g[0, 0, j:] * w[j:, None], axis=0) for j in range(n)])
    assert np.max(np.abs(dv[0, 0] - expect)) < 1e-12
    _, _, dv = attention_bwd_ref(q, k, v, g, 1.0, False)
    assert np.max(np.abs(dv[0, 0] - np.sum(g[0, 0], axis=0) / n)) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_single_key_closed_form(causal):
    """N = 1: O = V, so dV = dO; P = 1 makes dS = P (dP - D) = dO.V - dO.V = 0,
    so dQ = dK = 0 exactly, whatever Q, K and the scale."""
    q, k, v, g = (_rand((2, 3, 1, 5), s) for s in (11, 12, 13, 14))
    dq, dk, dv = attention_bwd_ref(q, k, v, g, 0.9, causal)
    assert np.max(np.abs(dv - g)) < 1e-15
    assert np.max(np.abs(dq)) < 1e-15 and np.max(np.abs(dk)) < 1e-15


def test_gradient_identities():
    """Adding a constant to every score of a row leaves softmax unchanged, so
    each row of dS sums to zero and therefore sum_j dK_j = scale * dS^T Q
    summed over keys = 0.  And since every row of P sums to 1, the columns of
    dV = P^T dO sum like the columns of dO."""
    n, d = 12, 5
    q, k, v, g = (_rand((1, 2, n, d), s) for s in (8, 9, 10, 11))
    for causal in (False, True):
        _, dk, dv = attention_bwd_ref(q, k, v, g, 0.3, causal)
        assert np.max(np.abs(dk.sum(axis=2))) < 1e-12
        assert np.max(np.abs(dv.sum(axis=2) - g.sum(axis=2))) < 1e-12


def test_d_prepass_equals_rowsum_of_p_dp():
    n, d = 10, 4
    q, k, v, g = (_rand((1, 1, n, d), s) for s in (12, 13, 14, 15))
    o, _ = attention_ref(q, k, v, 0.5, True)
    dd = attention_bwd_d(o, g)
    s = 0.5 * q[0, 0] @ k[0, 0].T
    s = np.where(np.tril(np.ones((n, n))) > 0, s, -np.inf)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    dp = g[0, 0] @ v[0, 0].T
    assert np.max(np.abs(dd[0, 0] - np.sum(p * dp, axis=1))) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_sampled_rows_match_full_backward(causal):
    """The row-sampled gradients equal the full ones at the sampled rows."""
    from oracle.backward import attention_bwd_rows
    n, d = 37, 6
    q, k, v, g = (_rand((2, 3, n, d), s) for s in (21, 22, 23, 24))
    dq, dk, dv = attention_bwd_ref(q, k, v, g, 0.4, causal)
    rows = [0, 5, 17, 36]
    for b, h in ((0, 0), (1, 2)):
        rq, rk, rv = attention_bwd_rows(q, k, v, g, 0.4, causal, b, h, rows, rows[::-1])
        assert np.max(np.abs(rq - dq[b, h, rows])) < 1e-12
        assert np.max(np.abs(rk - dk[b, h, rows[::-1]])) < 1e-12
        assert np.max(np.abs(rv - dv[b, h, rows[::-1]])) < 1e-12
