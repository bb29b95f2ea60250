"""Pins of the oracle's batch pre-gating (one routing decision for a decode
batch that shares one merged weight).

The pages route one token at a time (gist.science technical summary, section
2-ga).  The reading for a batch is the token rule applied to the mean of the
tokens' router logits; since the logits are linear in h, that is the token
rule applied to the mean hidden state.  These tests pin the oracle to that
statement through things other than itself: hand-worked fixtures, numpy's
fp64 matmul with a stable sort, exact rational brute force over tied integer
routers, and invariances of a mean.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "batch_route.json")


def _f32_close(got, want, ulps=1):
    got = np.asarray(got, np.float32)
    want = np.asarray(want, np.float64).astype(np.float32)
    gi = got.view(np.int32).astype(np.int64)
    wi = want.view(np.int32).astype(np.int64)
    return np.all(np.abs(gi - wi) <= ulps)


def test_batch_golden_fixtures(oracle_mod):
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        h = np.array(c["h"], np.float32)
        Wr = np.array(c["Wr"], np.float32)
        for k, want in c["k"].items():
            idx, gate, zbar = oracle_mod.pregate_batch(h, Wr, int(k), return_logits=True)
            assert np.array_equal(idx, want["idx"]), (c["name"], k, idx)
            assert _f32_close(gate, want["gate"]), (c["name"], k, gate)
            assert np.array_equal(zbar, np.array(c["zbar"])), (c["name"], zbar)


@pytest.mark.parametrize("T,d,E,k", [(7, 64, 8, 2), (33, 40, 5, 3), (2, 8, 16, 4), (64, 128, 8, 1)])
def test_batch_route_is_the_token_rule_on_the_mean_hidden_state(oracle_mod, T, d, E, k):
    rng = np.random.default_rng(1000 + T)
    h = rng.normal(size=(T, d)).astype(np.float32)
    Wr = (0.05 * rng.normal(size=(d, E))).astype(np.float32)
    idx, gate, zbar = oracle_mod.pregate_batch(h, Wr, k, return_logits=True)
    # numpy: logits of the mean hidden state, stable sort for (z desc, index asc)
    z = h.astype(np.float64).mean(axis=0) @ Wr.astype(np.float64)
    np.testing.assert_allclose(zbar, z, rtol=1e-12, atol=1e-12)
    order = np.argsort(-z, kind="stable")[:k]
    srt = np.sort(z)[::-1]
    assert np.all(np.diff(srt[:k + 1]) < -1e-9)     # no near ties in this data
    assert np.array_equal(idx[:min(k, E)], order[:min(k, E)])
    ez = np.exp(z[order] - z[order[0]])
    np.testing.assert_allclose(gate[:len(order)], ez / ez.sum(), rtol=2e-7)


@pytest.mark.parametrize("seed", range(6))
def test_batch_tie_rule_brute_force_exact(oracle_mod, seed):
    """Small integer routers with many exact ties: the picks are the experts
    sorted by (mean logit descending, index ascending), computed with exact
    rationals."""
    rng = np.random.default_rng(seed)
    T, d, E = int(rng.integers(1, 5)), int(rng.integers(1, 4)), int(rng.integers(1, 9))
    h = rng.integers(-2, 3, size=(T, d)).astype(np.float32)
    Wr = rng.integers(-1, 2, size=(d, E)).astype(np.float32)
    zbar = [Fraction(int(sum(h[t, i] * Wr[i, e] for t in range(T) for i in range(d))), T)
            for e in range(E)]
    ranked = sorted(range(E), key=lambda e: (-zbar[e], e))
    for k in range(1, 5):
        idx, gate = oracle_mod.pregate_batch(h, Wr, k)
        want = ranked[:k] + [-1] * max(0, k - E)
        assert list(idx) == want, (seed, k, list(idx), want, zbar)
        assert np.all(gate[np.asarray(want) < 0] == 0.0)
        assert abs(float(gate[np.asarray(want) >= 0].sum()) - 1.0) < 1e-6


def test_batch_of_one_token_is_the_token_route(oracle_mod):
    rng = np.random.default_rng(7)
    h = rng.normal(size=(5, 96)).astype(np.float32)
    Wr = (0.05 * rng.normal(size=(96, 8))).astype(np.float32)
    for t in range(5):
        for k in range(1, 5):
            idx, gate = oracle_mod.pregate_batch(h[t:t + 1], Wr, k)
            i2, g2 = oracle_mod.pregate_topk(h[t:t + 1], Wr, k)
            assert np.array_equal(idx, i2[0]) and np.array_equal(gate, g2[0])


def test_batch_is_order_and_duplicate_invariant(oracle_mod):
    rng = np.random.default_rng(8)
    h = rng.normal(size=(9, 48)).astype(np.float32)
    Wr = (0.05 * rng.normal(size=(48, 6))).astype(np.float32)
    idx, gate = oracle_mod.pregate_batch(h, Wr, 3)
    idx2, gate2 = oracle_mod.pregate_batch(h[rng.permutation(9)], Wr, 3)
    assert np.array_equal(idx, idx2) and _f32_close(gate, gate2)
    # a batch of copies of one token routes like the token
    one = h[4:5]
    idx3, gate3 = oracle_mod.pregate_batch(np.repeat(one, 5, axis=0), Wr, 3)
    idx4, gate4 = oracle_mod.pregate_batch(one, Wr, 3)
    assert np.array_equal(idx3, idx4) and _f32_close(gate3, gate4)
