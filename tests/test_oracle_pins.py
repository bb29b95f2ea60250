"""Pins for the CPU oracle: it is checked against things other than itself.

Each test ties one oracle function to a closed form, a library routine, a
brute-force enumeration or a hand-worked fixture, so that a dropped term, a
wrong sign, a wrong index or a transposed operand fails at least one of them.
The AdaFuse pages (gist.science technical summary, sections 2-ga and 2-na)
print no worked example, so the fixtures are worked by hand from the formula
W <- W - s*sum_prev g B A + s*sum_cur g B A.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f64(b):
    import oracle
    return oracle.bf16_to_f64(b)


def bf16_bits_of(x):
    """bf16 bit patterns of fp32-representable values, via torch's RNE cast."""
    t = torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_step(bits):
    """Spacing of bf16 values at the given bit patterns (2^-133 when subnormal)."""
    e = (bits.astype(np.int32) >> 7) & 0xFF
    return np.ldexp(1.0, np.where(e == 0, -133, e - 127 - 7))


def ulp_dist(a, b):
    """Distance in bf16 steps between bit patterns (+0 and -0 are equal)."""
    def ordered(u):
        u = u.astype(np.int32)
        return np.where(u & 0x8000, -(u & 0x7FFF), u)
    return np.abs(ordered(a) - ordered(b))


# --------------------------------------------------------------------------
# bf16 rounding

def _exact_nearest_bf16(x: float) -> int:
    """Brute force: compare x exactly (Fractions) with every candidate bf16
    value near it and pick the nearest, ties to the even bit pattern."""
    fx = Fraction(x)
    f32 = np.float32(x)
    base = int(np.array([f32]).view(np.uint32)[0] >> 16)
    best = None
    for cand in range(max(0, (base & 0x7FFF) - 2), min(0x7F80, (base & 0x7FFF) + 3)):
        bits = cand | (base & 0x8000)
        val = Fraction(float(np.array([bits << 16], dtype=np.uint32).view(np.float32)[0]))
        dist = abs(val - fx)
        key = (dist, bits & 1)
        if best is None or key < best[0]:
            best = (key, bits)
    return best[1]


def test_bf16_rounding_matches_torch_on_fp32_inputs(oracle_mod):
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 0.02,
        rng.standard_normal(2000).astype(np.float32) * 1e30,
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),   # subnormals
        np.array([0.0, -0.0, 1.0, -1.0, 3.3895313892515355e38, 3.4e38, -3.4e38,
                  np.inf, -np.inf, 1.00390625, 1.01171875, 9.183549615799121e-41],
                 dtype=np.float32),
    ])
    # exact ties: bf16 value + half a step
    u = rng.integers(0x0001, 0x7F00, size=4000).astype(np.uint32)
    ties = ((u << 16) | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, -ties])
    got = oracle_mod.bf16_from_f64(x.astype(np.float64))
    want = bf16_bits_of(x)
    assert np.array_equal(got, want)


def test_bf16_rounding_is_one_step_from_fp64(oracle_mod):
    # 1 + 2^-8 + 2^-30: via fp32 it collapses onto the tie 1 + 2^-8 and would
    # round to 1.0; rounded once it is above the midpoint -> 1 + 2^-7.
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert oracle_mod.bf16_from_f64(np.array([x]))[0] == 0x3F81
    assert oracle_mod.bf16_from_f64(np.array([-x]))[0] == 0xBF81
    rng = np.random.default_rng(2)
    xs = rng.standard_normal(3000) * 10.0 ** rng.integers(-42, 38, size=3000)
    got = oracle_mod.bf16_from_f64(xs)
    want = np.array([_exact_nearest_bf16(float(v)) for v in xs], dtype=np.uint16)
    assert np.array_equal(got, want)


def test_bf16_overflow_and_nan(oracle_mod):
    # largest finite bf16 is (2 - 2^-7) * 2^127; the midpoint to 2^128 is
    # (2 - 2^-8) * 2^127 = 3.39617e38
    mid = (2.0 - 2.0 ** -8) * 2.0 ** 127
    big = np.array([mid * (1 - 1e-9), mid, mid * (1 + 1e-9), 1e39, -1e300, np.nan])
    got = oracle_mod.bf16_from_f64(big)
    assert got[0] == 0x7F7F                     # below the midpoint: largest finite
    assert got[1] == 0x7F80                     # tie: the even neighbour is 2^128 -> inf
    assert got[2] == 0x7F80 and got[3] == 0x7F80 and got[4] == 0xFF80
    assert (got[5] & 0x7F80) == 0x7F80 and (got[5] & 0x7F) != 0


# --------------------------------------------------------------------------
# pre-gating (gist.science technical summary, section 2-ga)

def _rand_router(rng, T, d, E, scale=1.0):
    h = rng.standard_normal((T, d)).astype(np.float32) * np.float32(scale)
    Wr = (rng.standard_normal((d, E)) * 0.05).astype(np.float32)
    return h, Wr


@pytest.mark.parametrize("E", [2, 3, 4, 8, 16])
def test_pregate_matches_numpy_stable_argsort(oracle_mod, E):
    rng = np.random.default_rng(10 + E)
    h, Wr = _rand_router(rng, 64, 96, E)
    idx, gate, z = oracle_mod.pregate(h, Wr, return_logits=True)
    z_np = h.astype(np.float64) @ Wr.astype(np.float64)
    np.testing.assert_allclose(z, z_np, rtol=1e-12, atol=1e-12)
    for t in range(h.shape[0]):
        order = np.argsort(-z[t], kind="stable")
        assert list(idx[t]) == list(order[:2])


def test_pregate_brute_force_top2(oracle_mod):
    """All ordered pairs enumerated on tiny routers; the picked pair must beat
    every other expert under (logit desc, index asc)."""
    rng = np.random.default_rng(3)
    for E in (2, 3, 4, 5):
        # coarse values so that exact ties occur often
        h = rng.integers(-2, 3, size=(200, 4)).astype(np.float32)
        Wr = rng.integers(-2, 3, size=(4, E)).astype(np.float32)
        idx, _ = oracle_mod.pregate(h, Wr)
        z = h.astype(np.float64) @ Wr.astype(np.float64)
        for t in range(h.shape[0]):
            def before(a, b):
                return (z[t, a] > z[t, b]) or (z[t, a] == z[t, b] and a < b)
            best = None
            for a in range(E):
                for b in range(E):
                    if a == b or not before(a, b):
                        continue
                    if all(before(b, c) for c in range(E) if c not in (a, b)) and \
                       all(before(a, c) for c in range(E) if c != a):
                        assert best is None
                        best = (a, b)
            assert tuple(idx[t]) == best


def test_pregate_gates_closed_form(oracle_mod):
    rng = np.random.default_rng(4)
    h, Wr = _rand_router(rng, 128, 64, 8)
    idx, gate, z = oracle_mod.pregate(h, Wr, return_logits=True)
    z0 = z[np.arange(128), idx[:, 0]]
    z1 = z[np.arange(128), idx[:, 1]]
    g0 = 1.0 / (1.0 + np.exp(z1 - z0))
    np.testing.assert_allclose(gate[:, 0], g0, rtol=1e-7)
    np.testing.assert_allclose(gate[:, 1], 1.0 - g0, rtol=2e-6, atol=1e-7)
    assert np.all(gate[:, 0] >= gate[:, 1])


def test_pregate_large_logits_do_not_overflow(oracle_mod):
    rng = np.random.default_rng(5)
    h, Wr = _rand_router(rng, 16, 64, 8, scale=2000.0)
    idx, gate, z = oracle_mod.pregate(h, Wr, return_logits=True)
    assert np.all(np.isfinite(gate))
    z0 = z[np.arange(16), idx[:, 0]]
    z1 = z[np.arange(16), idx[:, 1]]
    np.testing.assert_allclose(gate[:, 0], 1.0 / (1.0 + np.exp(z1 - z0)), rtol=1e-7)


def test_pregate_duplicate_columns_tie_to_lower_index(oracle_mod):
    rng = np.random.default_rng(6)
    h, Wr = _rand_router(rng, 32, 48, 6)
    Wr[:, 4] = Wr[:, 1]
    Wr[:, 1] += 10.0 * np.abs(Wr).max()   # make the pair (1, 4) win everywhere h.sum>0
    Wr[:, 4] = Wr[:, 1]
    h = np.abs(h)
    idx, gate = oracle_mod.pregate(h, Wr)
    assert np.all(idx[:, 0] == 1) and np.all(idx[:, 1] == 4)
    np.testing.assert_array_equal(gate, np.full_like(gate, 0.5))


def test_pregate_single_expert(oracle_mod):
    rng = np.random.default_rng(7)
    h, Wr = _rand_router(rng, 4, 16, 1)
    idx, gate = oracle_mod.pregate(h, Wr)
    assert np.all(idx == np.array([0, -1])) and np.all(gate == np.array([1.0, 0.0], np.float32))


# --------------------------------------------------------------------------
# switch (gist.science technical summary, section 2-na)

def _rand_lora(rng, out, inn, E, r, w_std=0.02, a_std=None, b_std=0.01):
    a_std = a_std or 1.0 / math.sqrt(inn)
    W = bf16_bits_of(rng.standard_normal((out, inn)) * w_std)
    A = bf16_bits_of(rng.standard_normal((E, r, inn)) * a_std)
    B = bf16_bits_of(rng.standard_normal((E, out, r)) * b_std)
    return W, A, B


def _route(i0, i1, g0, g1):
    return (np.array([i0, i1], np.int32), np.array([g0, g1], np.float32))


def test_switch_matches_numpy_matmul(oracle_mod):
    """dW against numpy's fp64 matmul of the widened operands (library routine)."""
    rng = np.random.default_rng(20)
    out, inn, E, r, s = 24, 40, 5, 6, 2.0
    W, A, B = _rand_lora(rng, out, inn, E, r)
    prev, cur = _route(3, 0, 0.7, 0.3), _route(1, 4, 0.6, 0.4)
    _, Wx = oracle_mod.switch(W, A, B, s, prev, cur, exact=True)
    A64, B64, W64 = f64(A), f64(B), f64(W)
    want = W64 + s * (0.6 * (B64[1] @ A64[1]) + 0.4 * (B64[4] @ A64[4])) \
               - s * (0.7 * (B64[3] @ A64[3]) + 0.3 * (B64[0] @ A64[0]))
    # gates as the fp32 values the route holds
    g = lambda v: float(np.float32(v))
    want = W64 + s * (g(0.6) * (B64[1] @ A64[1]) + g(0.4) * (B64[4] @ A64[4])) \
               - s * (g(0.7) * (B64[3] @ A64[3]) + g(0.3) * (B64[0] @ A64[0]))
    np.testing.assert_allclose(Wx, want, rtol=1e-13, atol=1e-16)


def test_switch_forward_identity(oracle_mod):
    """W'x == Wx + s*sum g B (A x), evaluated right-to-left, before rounding."""
    rng = np.random.default_rng(21)
    out, inn, E, r, s = 48, 32, 4, 8, 2.0
    W, A, B = _rand_lora(rng, out, inn, E, r)
    cur = _route(2, 1, 0.625, 0.375)
    _, Wx = oracle_mod.switch(W, A, B, s, None, cur, exact=True)
    x = rng.standard_normal(inn)
    A64, B64, W64 = f64(A), f64(B), f64(W)
    want = W64 @ x + s * (0.625 * (B64[2] @ (A64[2] @ x)) + 0.375 * (B64[1] @ (A64[1] @ x)))
    np.testing.assert_allclose(Wx @ x, want, rtol=1e-11, atol=1e-14)


def test_switch_non_square_uses_right_operands(oracle_mod):
    """out != in != r: a transposed operand or a swapped A/B index cannot fit."""
    rng = np.random.default_rng(22)
    out, inn, E, r, s = 7, 13, 3, 2, 1.5
    W, A, B = _rand_lora(rng, out, inn, E, r)
    _, Wx = oracle_mod.switch(W, A, B, s, None, _route(2, -1, 1.0, 0.0), exact=True)
    A64, B64, W64 = f64(A), f64(B), f64(W)
    for i in range(out):
        for j in range(inn):
            want = W64[i, j] + s * sum(B64[2, i, k] * A64[2, k, j] for k in range(r))
            assert abs(Wx[i, j] - want) <= 1e-15 * max(1.0, abs(want))


def test_switch_merge_then_unmerge_restores(oracle_mod):
    rng = np.random.default_rng(23)
    out, inn, E, r, s = 64, 64, 4, 8, 2.0
    W0, A, B = _rand_lora(rng, out, inn, E, r)
    cur = _route(0, 3, 0.55, 0.45)
    W1 = oracle_mod.switch(W0, A, B, s, None, cur)
    assert ulp_dist(W1, W0).max() > 0          # the merge did something
    W2 = oracle_mod.switch(W1, A, B, s, cur, None)
    # W1 = W0 + dW + e1 and W2 = W1 - dW + e2 with each e at most half a bf16
    # step of the value it rounded to: the round trip is off by at most those
    # two half-steps (more than one step of W0 where |dW| >> |W0|).
    err = np.abs(f64(W2) - f64(W0))
    bound = 0.5 * bf16_step(W1) + 0.5 * bf16_step(W2)
    assert np.all(err <= bound)
    # where |W0| is not small against dW this is within one step of W0
    big = np.abs(f64(W0)) >= 4 * np.abs(f64(W1) - f64(W0))
    assert big.mean() > 0.5 and ulp_dist(W2[big], W0[big]).max() <= 1


def test_switch_prev_equals_cur_is_identity(oracle_mod):
    rng = np.random.default_rng(24)
    W0, A, B = _rand_lora(rng, 32, 48, 4, 4)
    rt = _route(1, 2, 0.8, 0.2)
    assert np.array_equal(oracle_mod.switch(W0, A, B, 2.0, rt, rt), W0)
    swapped = _route(2, 1, 0.2, 0.8)
    assert np.array_equal(oracle_mod.switch(W0, A, B, 2.0, rt, swapped), W0)


def test_switch_zero_coefficients_is_identity(oracle_mod):
    rng = np.random.default_rng(25)
    W0, A, B = _rand_lora(rng, 16, 24, 3, 4)
    assert np.array_equal(oracle_mod.switch(W0, A, B, 2.0, None, None), W0)
    zero = _route(0, 2, 0.0, 0.0)
    assert np.array_equal(oracle_mod.switch(W0, A, B, 2.0, None, zero), W0)
    assert np.array_equal(oracle_mod.switch(W0, A, B, 2.0, zero, None), W0)


def test_switch_sign_merge_adds_unmerge_subtracts(oracle_mod):
    out, inn, E, r = 4, 4, 1, 1
    W = bf16_bits_of(np.ones((out, inn)))
    A = bf16_bits_of(np.full((E, r, inn), 0.5))
    B = bf16_bits_of(np.full((E, out, r), 0.5))
    up = oracle_mod.switch(W, A, B, 2.0, None, _route(0, -1, 1.0, 0.0))
    down = oracle_mod.switch(W, A, B, 2.0, _route(0, -1, 1.0, 0.0), None)
    assert np.all(f64(up) == 1.5) and np.all(f64(down) == 0.5)


def test_switch_shared_expert_nets_out(oracle_mod):
    """prev=(a,b), cur=(a,c) with the same gate on a: only b leaves and c enters."""
    rng = np.random.default_rng(26)
    out, inn, E, r, s = 32, 40, 4, 4, 2.0
    W, A, B = _rand_lora(rng, out, inn, E, r)
    _, Wx = oracle_mod.switch(W, A, B, s, _route(0, 1, 0.5, 0.5), _route(0, 3, 0.5, 0.5),
                              exact=True)
    A64, B64, W64 = f64(A), f64(B), f64(W)
    want = W64 + s * 0.5 * (B64[3] @ A64[3]) - s * 0.5 * (B64[1] @ A64[1])
    np.testing.assert_allclose(Wx, want, rtol=1e-13, atol=1e-17)


def test_switch_rows_subset_matches_full(oracle_mod):
    rng = np.random.default_rng(27)
    out, inn, E, r, s = 40, 24, 4, 4, 2.0
    W, A, B = _rand_lora(rng, out, inn, E, r)
    prev, cur = _route(1, 2, 0.6, 0.4), _route(3, 0, 0.9, 0.1)
    full = oracle_mod.switch(W, A, B, s, prev, cur)
    rows = np.array([0, 5, 39, 17], dtype=np.int64)
    sub = oracle_mod.switch_rows(W[rows], rows, out, A, B, s, prev, cur)
    assert np.array_equal(sub, full[rows])


def test_switch_golden_rank1_fixtures(oracle_mod):
    with open(os.path.join(GOLDEN, "rank1_switch.json")) as f:
        fx = json.load(f)
    for case in fx["cases"]:
        W = bf16_bits_of(np.array(case["W"]))
        A = bf16_bits_of(np.array(case["A"]).reshape(1, 1, -1))
        B = bf16_bits_of(np.array(case["B"]).reshape(1, -1, 1))
        s = case["alpha"] / case["rank"]
        rt = lambda k: None if k not in case else _route(*case[k]["idx"], *case[k]["gate"])
        got = oracle_mod.switch(W, A, B, s, rt("prev"), rt("cur"))
        want = bf16_bits_of(np.array(case["expected"]))
        assert np.array_equal(got, want), case["name"]
