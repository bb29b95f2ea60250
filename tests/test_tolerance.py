"""The switch's parity tolerance, checked on the CPU.

An fp32 emulation of the GPU arithmetic (per-expert fp32 sums of rank
products, coefficients applied in fp32, one add to W, one bf16 rounding)
must pass the test's comparison with the oracle -- including elements where
W and dW cancel to far below either -- and planted mistakes must fail it.
"""
import numpy as np
import pytest
import torch

from .util import bf16_to_f64, check_switch_rows, ulp_dist


def _bf16(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def emulate_fp32_switch(W, A, B, s, prev, cur, drop_expert=None, sign=1.0):
    """fp32 arithmetic in the order the CUDA kernels use (not the oracle)."""
    coef = {}
    for side, rt in ((1.0, cur), (-1.0, prev)):
        if rt is None:
            continue
        for e, g in zip(rt[0], rt[1]):
            if e >= 0:
                coef[int(e)] = np.float32(coef.get(int(e), np.float32(0)) + np.float32(side * g))
    Wf = bf16_to_f64(W).astype(np.float32)
    Af = bf16_to_f64(A).astype(np.float32)
    Bf = bf16_to_f64(B).astype(np.float32)
    tot = np.zeros_like(Wf)
    for e, u in coef.items():
        c = np.float32(s) * u
        if c == 0 or e == drop_expert:
            continue
        acc = np.zeros_like(Wf)
        for k in range(A.shape[1]):
            acc = (acc + np.outer(Bf[e][:, k], Af[e][k])).astype(np.float32)
        tot = (tot + np.float32(sign) * c * acc).astype(np.float32)
    return _bf16((Wf + tot).astype(np.float32))


def _case(seed, cancel=True):
    rng = np.random.default_rng(seed)
    out, inn, E, r, s = 64, 96, 4, 8, 2.0
    W = _bf16(rng.standard_normal((out, inn)) * 0.02)
    A = _bf16(rng.standard_normal((E, r, inn)) * 0.125)
    B = _bf16(rng.standard_normal((E, out, r)) * 0.01)
    prev = (np.array([0, 1], np.int32), np.array([0.6, 0.4], np.float32))
    cur = (np.array([2, 3], np.int32), np.array([0.7, 0.3], np.float32))
    if cancel:
        # make a few W elements the bf16 negation of their exact dW
        import oracle
        _, ex = oracle.switch(np.zeros_like(W), A, B, s, prev, cur, exact=True)
        idx = rng.choice(W.size, size=200, replace=False)
        Wflat = W.reshape(-1)
        Wflat[idx] = _bf16(-ex.reshape(-1)[idx])
    return W, A, B, s, prev, cur


def test_fp32_emulation_passes_with_cancellations(oracle_mod):
    hits = 0
    for seed in range(6):
        W, A, B, s, prev, cur = _case(seed)
        got = emulate_fp32_switch(W, A, B, s, prev, cur)
        rows = np.arange(W.shape[0], dtype=np.int64)
        worst, ncancel = check_switch_rows(got, W, rows, W.shape[0], A, B, s, prev, cur)
        assert worst <= 1
        hits += ncancel
    # the planted cancellations really needed the fp32 clause
    assert hits > 0


@pytest.mark.parametrize("mistake", ["drop_expert", "sign"])
def test_planted_mistakes_fail(oracle_mod, mistake):
    W, A, B, s, prev, cur = _case(11, cancel=False)
    kw = {"drop_expert": 3} if mistake == "drop_expert" else {"sign": -1.0}
    got = emulate_fp32_switch(W, A, B, s, prev, cur, **kw)
    rows = np.arange(W.shape[0], dtype=np.int64)
    with pytest.raises(AssertionError):
        check_switch_rows(got, W, rows, W.shape[0], A, B, s, prev, cur)


def test_one_step_off_everywhere_is_caught_only_beyond_one_step(oracle_mod):
    W, A, B, s, prev, cur = _case(12, cancel=False)
    import oracle
    want = oracle.switch(W, A, B, s, prev, cur)
    off1 = (want.astype(np.int32) + 1).astype(np.uint16)      # one step in magnitude
    off2 = (want.astype(np.int32) + 2).astype(np.uint16)
    rows = np.arange(W.shape[0], dtype=np.int64)
    assert ulp_dist(off1, want).max() == 1
    check_switch_rows(off1, W, rows, W.shape[0], A, B, s, prev, cur)
    with pytest.raises(AssertionError):
        check_switch_rows(off2, W, rows, W.shape[0], A, B, s, prev, cur)
