"""Plant plausible mistakes in a copy of the oracle's arithmetic (on the CPU)
and check that the pins reject every one of them."""

import math

import numpy as np
import pytest

from oracle import brute_attention


def _mutant(kind):
    def f(q, k, v, scale, causal):
        s = q @ k.T
        if kind != "no_scale":
            s = s * scale
        if kind == "transposed_k":
            s = (q @ k.T).T * scale
        n = k.shape[0]
        if causal:
            keys = np.arange(n)[None, :]
            rows = np.arange(q.shape[0])[:, None]
            keep = keys < rows if kind == "strict_causal" else keys <= rows
            s = np.where(keep, s, -np.inf)
        m = s.max(axis=1)
        if kind == "sign":
            e = np.exp(m[:, None] - s)
        else:
            e = np.exp(s - m[:, None])
        e[~np.isfinite(e)] = 0.0
        den = e.sum(axis=1)
        p = e if kind == "no_normalise" else e / den[:, None]
        o = p @ (k if kind == "uses_k" else v)
        lse = m + (np.log(den) if kind != "lse_drop_log" else 0.0)
        return o, lse
    return f


@pytest.mark.parametrize("kind", ["no_scale", "transposed_k", "strict_causal", "sign",
                                  "no_normalise", "uses_k", "lse_drop_log"])
def test_pins_reject_mutant(kind):
    rng = np.random.default_rng(0)
    n, d = 9, 9
    q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
    scale = 1 / math.sqrt(d)
    rejected = False
    for causal in (False, True):
        with np.errstate(all="ignore"):
            o, lse = _mutant(kind)(q, k, v, scale, causal)
        ob, lb = brute_attention(q.tolist(), k.tolist(), v.tolist(), scale, causal)
        bad = (not np.all(np.isfinite(o))) or np.max(np.abs(o - np.array(ob))) > 1e-9 \
            or np.max(np.abs(lse - np.array(lb))) > 1e-9
        rejected |= bad
    assert rejected
