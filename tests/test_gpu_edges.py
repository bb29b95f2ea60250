"""GPU edge cases of the switch and the pre-gate, against the fp64 oracle.

Degenerate and extreme inputs the AdaFuse switch (gist.science technical
summary, section 2-na) must still get right: results in the bf16 subnormal
range, W values at the edge of overflow, an empty token batch, and the
pre-gate + switch pair captured into a CUDA graph and replayed.
"""
import numpy as np
import pytest
import torch

import oracle
from weight_merge_b200 import binding as Bnd
from weight_merge_b200 import workloads as wl

from .util import (bf16_to_f64, bits, check_switch_rows, fp32_accum_gamma, make_routes,
                   route_tuple, routes_to_np, ulp_dist)

pytestmark = pytest.mark.gpu

MMA, TC, TC2, TF = (Bnd.ADAFUSE_KERNEL_MMA_SYNC, Bnd.ADAFUSE_KERNEL_TCGEN05,
                    Bnd.ADAFUSE_KERNEL_TCGEN05_PAIR, Bnd.ADAFUSE_KERNEL_TCGEN05_FOLD)
# each kernel at a rank it takes
KERNEL_RANKS = [(MMA, 8), (TC, 8), (TC, 4), (TF, 8), (TF, 4), (TC2, 16)]


@pytest.fixture(scope="module", autouse=True)
def built():
    from weight_merge_b200 import build
    build.build()
    oracle.build()


def stream():
    return torch.cuda.current_stream().cuda_stream


def _model(kernel, scale_w=1.0, scale_a=1.0, scale_b=1.0, seed=0, r=8):
    cfg = wl.custom("edge", 2, [("a", 136, 264), ("b", 256, 128)], n_experts=4, rank=r,
                    alpha=2.0 * r, n_tokens=2, d=264)
    m = wl.make_model(cfg, device="cuda", seed=seed)
    with torch.no_grad():
        for w in m.W:
            w.copy_((w.float() * scale_w).to(torch.bfloat16))
        for a in m.A:
            a.copy_((a.float() * scale_a).to(torch.bfloat16))
        for b in m.B:
            b.copy_((b.float() * scale_b).to(torch.bfloat16))
    sw = Bnd.Switcher(m.W, m.A, m.B, cfg.n_layers, len(cfg.targets), cfg.n_experts, cfg.rank,
                      cfg.alpha, device=torch.cuda.current_device())
    sw.set_kernel(kernel)
    return cfg, m, sw


def _switch_and_check(cfg, m, sw, routes, steps):
    r_np = routes_to_np(routes)
    A_h = [bits(a) for a in m.A]
    B_h = [bits(b) for b in m.B]
    for p, c in steps:
        before = [bits(w) for w in m.W]
        sw.switch(None if p is None else Bnd.Switcher.route_ptr(routes, p),
                  None if c is None else Bnd.Switcher.route_ptr(routes, c), stream())
        torch.cuda.synchronize()
        assert sw.status(stream()) == 0
        for i, w in enumerate(m.W):
            rows = np.arange(w.shape[0], dtype=np.int64)
            check_switch_rows(bits(w), before[i], rows, w.shape[0], A_h[i], B_h[i], cfg.scale,
                              None if p is None else route_tuple(r_np, p),
                              None if c is None else route_tuple(r_np, c))


@pytest.mark.parametrize("kernel,r", KERNEL_RANKS)
def test_subnormal_results(kernel, r):
    """W ~ 1e-39 and dW of the same size: every result is a bf16 subnormal
    (below 2^-126), which fp32 arithmetic without flush-to-zero keeps."""
    # W ~ N(0, .02) * 5e-38 -> ~1e-39; B ~ .01 * 1e-37, A ~ .06 -> B*A ~ 6e-41 per term
    cfg, m, sw = _model(kernel, scale_w=5e-38, scale_b=1e-37, seed=3, r=r)
    sub = sum(int(((bits(w) & 0x7F80) == 0).sum()) for w in m.W)
    assert sub > 0.9 * sum(w.numel() for w in m.W)
    routes = make_routes(np.array([[0, 2], [3, 1]], np.int32),
                         np.array([[0.7, 0.3], [0.6, 0.4]], np.float32))
    _switch_and_check(cfg, m, sw, routes, [(None, 0), (0, 1), (1, None)])


@pytest.mark.parametrize("kernel,r", KERNEL_RANKS)
def test_overflow_to_infinity(kernel, r):
    """W at the largest bf16 magnitudes plus a same-signed dW rounds to +-inf,
    as the oracle's round-to-nearest-even does.

    Under round-to-nearest-even a magnitude rounds to inf from
    2^128 - 2^119 up (half a step above the largest finite bf16, the tie
    going to the even pattern, inf).  Where the exact fp64 value lies within
    the fp32 accumulation bound of that threshold either side is a correct
    rounding of an fp32 sum, so there the 1-step parity bar decides; every
    other element must land on the oracle's side of it."""
    cfg, m, sw = _model(kernel, seed=4, r=r)
    with torch.no_grad():
        for w in m.W:
            w.copy_(torch.where(w >= 0, 3.3895e38, -3.3895e38).to(torch.bfloat16))
        # |B| ~ 2e36, |A| ~ 0.05: dW ~ r * 1.3e35, against half a bf16 step at
        # 3.39e38 (6.6e35); positive everywhere, every fp32 partial finite
        for b in m.B:
            b.abs_().mul_(3e38)
        for a in m.A:
            a.abs_()
    Bnd.adafuse_refresh_adapters(sw.ctx, stream())   # B changed after create (rank < 8 copy)
    routes = make_routes(np.array([[0, 1]], np.int32), np.array([[0.5, 0.5]], np.float32))
    before = [bits(w) for w in m.W]
    sw.switch(None, Bnd.Switcher.route_ptr(routes, 0), stream())
    torch.cuda.synchronize()
    A_h = [bits(a) for a in m.A]
    B_h = [bits(b) for b in m.B]
    r_np = routes_to_np(routes)
    thr = 2.0 ** 128 - 2.0 ** 119
    gamma = fp32_accum_gamma(r, 2)
    for i, w in enumerate(m.W):
        got = bits(w)
        want, exact = oracle.switch(before[i], A_h[i], B_h[i], cfg.scale, None,
                                    route_tuple(r_np, 0), exact=True)
        M = np.abs(bf16_to_f64(before[i]))
        for e, g in zip(*route_tuple(r_np, 0)):
            M += cfg.scale * float(g) * (np.abs(bf16_to_f64(B_h[i][e])) @ np.abs(bf16_to_f64(A_h[i][e])))
        margin = gamma * M
        over = np.abs(exact) >= thr + margin
        under = np.abs(exact) < thr - margin
        is_inf = (got & 0x7FFF) == 0x7F80
        assert over.sum() > 0                           # some really overflow
        assert np.array_equal(got[over], want[over])    # to inf of the right sign
        assert not is_inf[under].any()                  # the rest stays finite
        assert not is_inf[(before[i] & 0x8000) != 0].any()   # negative W moves away
        assert ulp_dist(got, want).max() <= 1


def test_pregate_empty_batch_is_a_noop():
    cfg, m, sw = _model(TC)
    h = torch.empty((0, cfg.d), device="cuda")
    routes = torch.full((1, 4), 7, dtype=torch.int32, device="cuda")
    sw.pregate(h, m.Wr, routes, stream())
    torch.cuda.synchronize()
    assert torch.all(routes == 7)


@pytest.mark.parametrize("kernel,r,schedule",
                         [(k, r, Bnd.ADAFUSE_SCHEDULE_AUTO) for (k, r) in KERNEL_RANKS] +
                         [(TC2, 16, Bnd.ADAFUSE_SCHEDULE_DYNAMIC),
                          (TC, 8, Bnd.ADAFUSE_SCHEDULE_STATIC)])
def test_cuda_graph_capture_of_pregate_and_switch(kernel, r, schedule):
    """One decode step (pre-gate the token, switch prev -> cur, keep cur as the
    next prev) captured once and replayed gives the same W, bit for bit, as
    the same calls made eagerly (both tile schedules: a dynamic launch leaves
    its ticket counter at zero for the next replay)."""
    cfg, m1, s1 = _model(kernel, seed=9, r=r)
    _, m2, s2 = _model(kernel, seed=9, r=r)
    s1.set_schedule(schedule)
    s2.set_schedule(schedule)
    g = torch.Generator(device="cuda").manual_seed(5)
    T = 4
    hs = torch.randn((T, cfg.d), generator=g, device="cuda")
    # eager
    r1 = torch.zeros((T, 4), dtype=torch.int32, device="cuda")
    for t in range(T):
        s1.pregate(hs[t:t + 1], m1.Wr, r1[t:t + 1], stream())
        s1.switch(None if t == 0 else Bnd.Switcher.route_ptr(r1, t - 1),
                  Bnd.Switcher.route_ptr(r1, t), stream())
    # graph: fixed buffers for the token, the previous and the current route
    h_slot = torch.empty((1, cfg.d), device="cuda")
    prev = torch.zeros((1, 4), dtype=torch.int32, device="cuda")
    cur = torch.zeros((1, 4), dtype=torch.int32, device="cuda")
    h_slot.copy_(hs[0:1])
    s2.pregate(h_slot, m2.Wr, cur, stream())          # token 0, eagerly (no prev)
    s2.switch(None, Bnd.Switcher.route_ptr(cur, 0), stream())
    prev.copy_(cur)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            sh = side.cuda_stream
            s2.pregate(h_slot, m2.Wr, cur, sh)
            s2.switch(Bnd.Switcher.route_ptr(prev, 0), Bnd.Switcher.route_ptr(cur, 0), sh)
            prev.copy_(cur)
    for t in range(1, T):
        h_slot.copy_(hs[t:t + 1])
        graph.replay()
    torch.cuda.synchronize()
    assert s2.status(stream()) == 0
    for a, b in zip(m1.W, m2.W):
        assert torch.equal(a, b)
    assert torch.equal(r1[T - 1:T], cur)


@pytest.mark.parametrize("kernel,r", [(TC, 8), (TC, 16), (TF, 8), (TC2, 16), (TC2, 64)])
def test_bounded_wait_timeout_reports_status_and_context_stays_usable(kernel, r):
    """Failure detection without a GPU fault: the test hook makes each CTA's
    first operand stage wait for 16 bytes that never arrive.  The MMA warp's
    bounded wait (1 s) runs out, the launch raises ADAFUSE_STATUS_TIMEOUT and
    every warp leaves through its own bounded waits before any MMA completes,
    so W is untouched; the next switch on the same context is exact."""
    cfg, m, sw = _model(kernel, seed=21, r=r)
    assert sw.kernel == kernel
    W0 = [bits(w) for w in m.W]
    routes = make_routes(np.array([[0, 2], [3, 1]], np.int32),
                         np.array([[0.7, 0.3], [0.6, 0.4]], np.float32))
    Bnd.adafuse_debug_stall_next_switch(sw.ctx)
    sw.switch(None, Bnd.Switcher.route_ptr(routes, 0), stream())
    assert sw.status(stream()) == Bnd.ADAFUSE_STATUS_TIMEOUT
    for w, w0 in zip(m.W, W0):
        assert np.array_equal(bits(w), w0)
    _switch_and_check(cfg, m, sw, routes, [(None, 0), (0, 1)])


MID_SHAPES = {"blocked": [("q", 1024, 1024), ("o", 1280, 768)],
              "plain": [("q", 1024, 1032), ("o", 1280, 776)]}


@pytest.mark.parametrize("layout", ["blocked", "plain"])
@pytest.mark.parametrize("kernel,r", [(TC, 8), (TC2, 16), (TF, 8), (TC, 32)])
def test_timeout_mid_launch_leaves_whole_tiles_and_rebase_recovers(kernel, r, layout):
    """A bounded wait that runs out in the middle of a switch: the hook
    stalls each CTA's second tile, so every CTA stores its first tile and
    stops.  Every 128 x 128 tile must then be either untouched or fully
    switched (the oracle's prev -> cur result), with both kinds present; the
    documented recovery, a re-base from the registered pristine weights,
    gives the oracle's W0 + dW(cur) everywhere."""
    shapes = MID_SHAPES[layout]
    cfg = wl.custom("mid", 2, shapes, n_experts=4, rank=r, alpha=2.0 * r, n_tokens=2,
                    d=shapes[0][2])
    m = wl.make_model(cfg, device="cuda", seed=90 + r)
    sw = Bnd.Switcher(m.W, m.A, m.B, cfg.n_layers, len(cfg.targets), cfg.n_experts, cfg.rank,
                      cfg.alpha, device=torch.cuda.current_device())
    sw.set_kernel(kernel)
    assert sw.map_layout == (Bnd.ADAFUSE_MAPS_BLOCKED if layout == "blocked"
                             else Bnd.ADAFUSE_MAPS_PLAIN)
    base = [w.clone() for w in m.W]
    sw.set_base(base)
    W0 = [bits(w) for w in base]
    A_h, B_h = [bits(a) for a in m.A], [bits(b) for b in m.B]
    routes = make_routes(np.array([[0, 2], [3, 1]], np.int32),
                         np.array([[0.7, 0.3], [0.6, 0.4]], np.float32))
    r_np = routes_to_np(routes)
    p = lambda t: Bnd.Switcher.route_ptr(routes, t)
    sw.switch(None, p(0), stream())
    torch.cuda.synchronize()
    assert sw.status(stream()) == 0
    before = [bits(w) for w in m.W]
    Bnd.adafuse_debug_stall_next_switch_at(sw.ctx, 2)
    sw.switch(p(0), p(1), stream())
    assert sw.status(stream()) == Bnd.ADAFUSE_STATUS_TIMEOUT
    n_old = n_new = 0
    for i, w in enumerate(m.W):
        got = bits(w)
        out, inn = got.shape
        rows = np.arange(out, dtype=np.int64)
        want, _ = oracle.switch_rows(before[i], rows, out, A_h[i], B_h[i], cfg.scale,
                                     route_tuple(r_np, 0), route_tuple(r_np, 1), exact=True)
        patched = got.copy()
        for r0 in range(0, out, 128):
            for c0 in range(0, inn, 128):
                t_got = got[r0:r0 + 128, c0:c0 + 128]
                if np.array_equal(t_got, before[i][r0:r0 + 128, c0:c0 + 128]):
                    n_old += 1
                    patched[r0:r0 + 128, c0:c0 + 128] = want[r0:r0 + 128, c0:c0 + 128]
                else:
                    n_new += 1
        # every tile that changed holds the full prev -> cur switch
        check_switch_rows(patched, before[i], rows, out, A_h[i], B_h[i], cfg.scale,
                          route_tuple(r_np, 0), route_tuple(r_np, 1))
    assert n_old > 0 and n_new > 0, (n_old, n_new)
    # recovery: re-base every tile from the pristine weights onto route 1
    sw.rebase(p(1), stream())
    torch.cuda.synchronize()
    assert sw.status(stream()) == 0
    for i, w in enumerate(m.W):
        rows = np.arange(w.shape[0], dtype=np.int64)
        check_switch_rows(bits(w), W0[i], rows, w.shape[0], A_h[i], B_h[i], cfg.scale, None,
                          route_tuple(r_np, 1))


def test_stall_hook_rejects_a_tile_number_below_one():
    cfg, m, sw = _model(TC, seed=23, r=8)
    with pytest.raises(Bnd.AdafuseError):
        Bnd.adafuse_debug_stall_next_switch_at(sw.ctx, 0)


def test_stall_hook_is_refused_by_the_wait_free_kernel():
    cfg, m, sw = _model(MMA, seed=22, r=8)
    with pytest.raises(Bnd.AdafuseError):
        Bnd.adafuse_debug_stall_next_switch(sw.ctx)


@pytest.mark.parametrize("kernel,r", [(TC, 1), (TC, 4), (TC, 7), (TF, 4)])
def test_ranks_below_8_read_a_padded_copy_of_b_refreshed_on_request(kernel, r):
    """Below rank 8 the tensor-core paths read B through the context's
    zero-padded copy.  After the caller changes B, adafuse_refresh_adapters
    brings the copy up to date and the switch matches the oracle on the new B."""
    cfg, m, sw = _model(kernel, seed=30 + r, r=r)
    assert sw.kernel == kernel
    routes = make_routes(np.array([[0, 2], [3, 1]], np.int32),
                         np.array([[0.7, 0.3], [0.6, 0.4]], np.float32))
    _switch_and_check(cfg, m, sw, routes, [(None, 0)])
    with torch.no_grad():
        for b in m.B:
            b.mul_(-1.5)
    Bnd.adafuse_refresh_adapters(sw.ctx, stream())
    _switch_and_check(cfg, m, sw, routes, [(0, 1), (1, None)])


@pytest.mark.parametrize("r", [8, 5])
def test_folded_kernel_reads_a_afresh_on_every_switch(r):
    """The folded kernel rebuilds c_e * A_e from A before every switch, so a
    caller's in-place change of A needs no refresh call."""
    cfg, m, sw = _model(TF, seed=40 + r, r=r)
    routes = make_routes(np.array([[0, 2], [3, 1], [1, 2]], np.int32),
                         np.array([[0.7, 0.3], [0.6, 0.4], [0.5, 0.5]], np.float32))
    _switch_and_check(cfg, m, sw, routes, [(None, 0), (0, 1)])
    with torch.no_grad():
        for a in m.A:
            a.mul_(-0.75)
    _switch_and_check(cfg, m, sw, routes, [(1, 2), (2, None)])
