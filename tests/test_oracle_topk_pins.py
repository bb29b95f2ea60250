"""Pins for the oracle's top-k widening of the router and the switch.

The AdaFuse pages use a top-2 router (gist.science technical summary, section
2-ga); the top-k router picks k in [1, 4] experts by the same rule (logit
descending, index ascending) and renormalises the full softmax over the k
picks, and the switch (section 2-na) then un-merges up to k experts and merges
up to k.  Each test ties the widened oracle to something other than itself:
the top-2 oracle, numpy's stable argsort, brute force over ordered k-tuples,
the closed form of the renormalised softmax, and numpy's fp64 matmul.
"""
import ctypes
import itertools
import math

import numpy as np
import pytest

from .test_oracle_pins import _rand_lora, bf16_bits_of, f64


def _rand_router(rng, T, d, E, scale=1.0):
    h = (rng.standard_normal((T, d)) * scale).astype(np.float32)
    Wr = (rng.standard_normal((d, E)) * 0.05 * scale).astype(np.float32)
    return h, Wr


def test_topk_with_k2_is_the_top2_router(oracle_mod):
    rng = np.random.default_rng(40)
    for E in (2, 3, 8, 16):
        h, Wr = _rand_router(rng, 96, 64, E)
        i2, g2 = oracle_mod.pregate(h, Wr)
        ik, gk = oracle_mod.pregate_topk(h, Wr, 2)
        np.testing.assert_array_equal(ik, i2)
        np.testing.assert_array_equal(gk.view(np.uint32), g2.view(np.uint32))


@pytest.mark.parametrize("k", [1, 2, 3, 4])
@pytest.mark.parametrize("E", [4, 6, 9])
def test_topk_matches_numpy_stable_argsort(oracle_mod, k, E):
    rng = np.random.default_rng(41 + 7 * k + E)
    h, Wr = _rand_router(rng, 64, 48, E)
    idx, gate, z = oracle_mod.pregate_topk(h, Wr, k, return_logits=True)
    z_np = h.astype(np.float64) @ Wr.astype(np.float64)
    np.testing.assert_allclose(z, z_np, rtol=1e-12, atol=1e-12)
    for t in range(h.shape[0]):
        order = np.argsort(-z[t], kind="stable")
        assert list(idx[t]) == list(order[:k])


def test_topk_brute_force_on_tied_routers(oracle_mod):
    """Every ordered k-tuple enumerated; exactly one is the top-k under
    (logit desc, index asc): its members in order, each before every expert
    left out."""
    rng = np.random.default_rng(42)
    for E in (3, 4, 5):
        h = rng.integers(-2, 3, size=(120, 3)).astype(np.float32)
        Wr = rng.integers(-1, 2, size=(3, E)).astype(np.float32)
        z = h.astype(np.float64) @ Wr.astype(np.float64)
        for k in range(1, min(4, E) + 1):
            idx, _ = oracle_mod.pregate_topk(h, Wr, k)
            for t in range(h.shape[0]):
                def before(a, b):
                    return (z[t, a] > z[t, b]) or (z[t, a] == z[t, b] and a < b)
                found = []
                for tup in itertools.permutations(range(E), k):
                    in_order = all(before(tup[j], tup[j + 1]) for j in range(k - 1))
                    beats_rest = all(before(tup[-1], c) for c in range(E) if c not in tup)
                    if in_order and beats_rest:
                        found.append(tup)
                assert len(found) == 1
                assert tuple(idx[t]) == found[0]


@pytest.mark.parametrize("k", [2, 3, 4])
def test_topk_gates_closed_form(oracle_mod, k):
    """g_j = exp(z_j - z_0) / sum_i exp(z_i - z_0) over the picks (the full
    softmax renormalised over them); gates sum to one and do not increase."""
    rng = np.random.default_rng(43 + k)
    h, Wr = _rand_router(rng, 128, 64, 8)
    idx, gate, z = oracle_mod.pregate_topk(h, Wr, k, return_logits=True)
    zp = np.take_along_axis(z, idx.astype(np.int64), axis=1)
    x = np.exp(zp - zp[:, :1])
    want = x / x.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(gate, want, rtol=2e-7, atol=1e-8)
    np.testing.assert_allclose(gate.astype(np.float64).sum(axis=1), 1.0, rtol=0, atol=4e-7)
    assert np.all(np.diff(gate, axis=1) <= 0)


def test_topk_k1_has_gate_one(oracle_mod):
    rng = np.random.default_rng(44)
    h, Wr = _rand_router(rng, 32, 32, 5)
    idx, gate, z = oracle_mod.pregate_topk(h, Wr, 1, return_logits=True)
    assert np.all(gate == np.float32(1.0))
    np.testing.assert_array_equal(idx[:, 0], np.argmax(z, axis=1))


def test_topk_more_slots_than_experts(oracle_mod):
    rng = np.random.default_rng(45)
    h, Wr = _rand_router(rng, 16, 32, 2)
    idx, gate = oracle_mod.pregate_topk(h, Wr, 4)
    assert np.all(idx[:, 2:] == -1) and np.all(gate[:, 2:] == 0.0)
    i2, g2 = oracle_mod.pregate(h, Wr)
    np.testing.assert_array_equal(idx[:, :2], i2)
    np.testing.assert_array_equal(gate[:, :2], g2)


def test_topk_large_logits_do_not_overflow(oracle_mod):
    rng = np.random.default_rng(46)
    h, Wr = _rand_router(rng, 16, 64, 8, scale=2000.0)
    idx, gate = oracle_mod.pregate_topk(h, Wr, 4)
    assert np.all(np.isfinite(gate)) and np.all(gate[:, 0] > 0)


# --------------------------------------------------------------------------
# switch with k-slot routes


def _route_k(idx, gate):
    return (np.array(idx, np.int32), np.array(gate, np.float32))


@pytest.mark.parametrize("k", [3, 4])
def test_switch_k_slots_matches_numpy_matmul(oracle_mod, k):
    rng = np.random.default_rng(50 + k)
    out, inn, E, r, s = 24, 40, 9, 6, 2.0
    W, A, B = _rand_lora(rng, out, inn, E, r)
    pi = [7, 0, 3, 5][:k]
    pg = [0.4, 0.3, 0.2, 0.1][:k]
    ci = [3, 8, 1, 2][:k]            # expert 3 is in both routes
    cg = [0.5, 0.25, 0.15, 0.1][:k]
    prev, cur = _route_k(pi, pg), _route_k(ci, cg)
    _, Wx = oracle_mod.switch(W, A, B, s, prev, cur, exact=True)
    A64, B64, W64 = f64(A), f64(B), f64(W)
    g = lambda v: float(np.float32(v))
    plus = sum(g(cg[j]) * (B64[ci[j]] @ A64[ci[j]]) for j in range(k))
    minus = sum(g(pg[j]) * (B64[pi[j]] @ A64[pi[j]]) for j in range(k))
    np.testing.assert_allclose(Wx, W64 + s * plus - s * minus, rtol=1e-13, atol=1e-16)


def test_switch_k_slots_equal_routes_are_identity(oracle_mod):
    rng = np.random.default_rng(55)
    W, A, B = _rand_lora(rng, 16, 24, 6, 4)
    rt = _route_k([5, 2, 0, 4], [0.4, 0.3, 0.2, 0.1])
    Wn, Wx = oracle_mod.switch(W, A, B, 2.0, rt, rt, exact=True)
    np.testing.assert_array_equal(Wn, W)
    np.testing.assert_array_equal(Wx, f64(W))


def test_switch_k_slots_empty_slots_contribute_nothing(oracle_mod):
    rng = np.random.default_rng(56)
    W, A, B = _rand_lora(rng, 16, 24, 6, 4)
    full = oracle_mod.switch(W, A, B, 2.0, None, _route_k([1, 3, -1, -1], [0.6, 0.4, 0.9, 0.9]))
    two = oracle_mod.switch(W, A, B, 2.0, None, _route_k([1, 3], [0.6, 0.4]))
    np.testing.assert_array_equal(full, two)


def test_switch_two_slot_path_equals_general_path(oracle_mod):
    """The k = 2 entry and the k-slot entry with two slots agree bitwise."""
    rng = np.random.default_rng(57)
    W, A, B = _rand_lora(rng, 12, 16, 5, 3)
    E, r, inn = A.shape
    out = W.shape[0]
    prev = _route_k([4, 1], [0.55, 0.45])
    cur = _route_k([1, 0], [0.7, 0.3])
    want = oracle_mod.switch(W, A, B, 2.0, prev, cur)
    lib = oracle_mod._load()
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    rows = np.arange(out, dtype=np.int64)
    got = np.empty_like(W)
    lib.orc_switch_rows_k(ptr(W), ptr(rows), out, out, inn, ptr(A), ptr(B), r, 2.0, 2,
                          ptr(prev[0]), ptr(prev[1]), ptr(cur[0]), ptr(cur[1]), ptr(got), None)
    np.testing.assert_array_equal(got, want)


def test_switch_k_slots_merge_then_unmerge_restores(oracle_mod):
    """Merging a top-4 route then un-merging it returns W to within the two
    roundings' half-steps."""
    rng = np.random.default_rng(58)
    W0, A, B = _rand_lora(rng, 32, 48, 8, 8)
    rt = _route_k([6, 1, 3, 0], [0.4, 0.3, 0.2, 0.1])
    W1 = oracle_mod.switch(W0, A, B, 2.0, None, rt)
    W2 = oracle_mod.switch(W1, A, B, 2.0, rt, None)
    step = lambda b: np.ldexp(1.0, np.where(((b >> 7) & 0xFF) == 0, -133,
                                            ((b.astype(np.int32) >> 7) & 0xFF) - 134))
    assert np.any(W1 != W0)
    assert np.all(np.abs(f64(W2) - f64(W0)) <= 0.5 * step(W1) + 0.5 * step(W2) + 1e-30)
