"""Host logic of bench.py that decides which switches count as W-moving.

The end-to-end leg pre-gates tokens the timed loop never reached; the number
of W-moving switches it reports must come from the routes that leg computed,
read back after its own loop.  A stub router stands in for the GPU.
"""
import numpy as np

import bench


def _stub_route(t, E=8):
    # distinct consecutive routes: the pair (t, t + 3) mod E with fixed gates
    return np.array([t % E, (t + 3) % E, 0, 0], dtype=np.int32)


def test_e2e_leg_counts_the_routes_it_computed():
    T, warmup, steps = 64, 5, 20
    routes = np.zeros((T, 4), dtype=np.int32)
    # the timed loop filled tokens warmup .. warmup+steps-1
    for t in range(warmup + steps):
        routes[t] = _stub_route(t)
    before = routes.copy()             # a snapshot taken before the e2e loop
    prev_t = (warmup + steps - 1) % T
    seq = [(warmup + steps + k) % T for k in range(steps)]
    calls = []

    def run_step(pe, t):
        calls.append((pe, t))
        routes[t] = _stub_route(t)     # the router writes the token's route

    ms, flags, last = bench.e2e_leg(seq, prev_t, run_step, lambda: None, lambda: 4.7 * steps,
                                    lambda: routes.copy())
    assert ms == 4.7 * steps
    assert sum(flags) == steps         # every one of the 20 switches moves W
    assert last == seq[-1]
    assert calls[0] == (prev_t, seq[0]) and [c[1] for c in calls] == seq
    # the stale snapshot would have seen 19 identity switches among zero rows
    assert sum(bench.moving_steps(before, seq, prev_t)) == 1


def test_moving_steps_identity_and_rebase():
    r = np.array([[1, 2, 7, 9], [1, 2, 7, 9], [1, 2, 7, 8], [3, 2, 7, 8]], dtype=np.int32)
    # first switch (no previous route) moves W; bitwise-equal routes do not;
    # equal indices with a different gate do
    assert bench.moving_steps(r, [0, 1, 2, 3], None) == [True, False, True, True]
    assert bench.moving_steps(r, [1], 0) == [False]
    # a re-base writes W every time
    assert bench.moving_steps(r, [0, 1], 0, rebase=True) == [True, True]


def test_route_buffer_synthesised_workloads():
    from weight_merge_b200 import workloads as wl
    cfg = wl.CONFIGS["7b-r64"]
    buf = bench.route_buffer(cfg, 16, False, "cpu").numpy()
    idx, gate = wl.synth_routes(cfg, T=16)
    assert np.array_equal(buf[:, :2], idx)
    assert np.array_equal(buf[:, 2:].view(np.float32), gate)
    buf4 = bench.route_buffer(cfg, 16, True, "cpu").numpy()
    assert np.array_equal(buf4[:, :2], idx) and np.all(buf4[:, 2:4] == -1)
    assert np.array_equal(buf4[:, 4:6].view(np.float32), gate)
    assert np.all(buf4[:, 6:].view(np.float32) == 0)
    assert bench.route_buffer(wl.CONFIGS["7b"], 16, False, "cpu") is None


def test_effective_schedule_follows_the_auto_rule():
    """ADAFUSE_SCHEDULE_AUTO: dynamic for the single-CTA tensor-core kernel
    (2), static for the pair kernel (3); an explicit choice applies to both;
    the other kernels are static."""
    assert bench.effective_schedule("auto", 2) == "dynamic"
    assert bench.effective_schedule("auto", 3) == "static"
    assert bench.effective_schedule("dynamic", 3) == "dynamic"
    assert bench.effective_schedule("static", 2) == "static"
    for k in (1, 4):
        assert bench.effective_schedule("dynamic", k) == "static"
