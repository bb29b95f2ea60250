"""adafuse_switch_noalloc: the switch for callers that cannot allocate.

A caller whose device memory belongs to its own pre-reserved pool, or whose
decode loop must not stall on cudaMalloc, switches the model through
adafuse_switch_noalloc: no context, no allocation, only a fixed 64 KiB
static device scratch.  Its result must match the oracle and the regular
entry point's (adafuse_switch through a context) within the parity tolerance
the other tests use, call after call.  This file is collected last on purpose, so a
run that stops at the first failure has already run every other test; it
also passes on its own in a fresh process (the first call on a device does
the scratch set-up).
"""
import ctypes

import numpy as np
import pytest
import torch

from weight_merge_b200 import binding as Bnd
from weight_merge_b200 import workloads as wl

from .util import bits, check_switch_rows, make_routes, route_tuple, routes_to_np, ulp_dist

SHAPES = [("q", 264, 392), ("o", 392, 264), ("up", 1024, 512), ("tail", 136, 8)]


def _noalloc(desc, prev, cur, status, stream):
    L = Bnd.lib()
    fn = L.adafuse_switch_noalloc
    fn.argtypes = [ctypes.POINTER(Bnd.Desc), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn(ctypes.byref(desc), prev, cur, status, stream)


def _desc_of(model):
    c = model.cfg
    ts = [(c.targets[i % len(c.targets)].name, w.shape[0], w.shape[1], w.data_ptr(),
           a.data_ptr(), b.data_ptr()) for i, (w, a, b) in enumerate(zip(model.W, model.A, model.B))]
    return Bnd.make_desc(c.n_layers, len(c.targets), c.n_experts, c.rank, c.alpha, ts)


@pytest.mark.gpu
@pytest.mark.parametrize("rank", [8, 12])
def test_noalloc_matches_adafuse_switch_two_calls_in_a_row(rank):
    from weight_merge_b200 import build
    build.build()
    cfg = wl.custom("noalloc", 3, SHAPES, n_experts=5, rank=rank, alpha=2.0 * rank,
                    n_tokens=2, d=392)
    ref = wl.make_model(cfg, device="cuda", seed=77 + rank)     # regular entry point
    mine = wl.make_model(cfg, device="cuda", seed=77 + rank)    # allocation-free entry point
    W0 = [bits(w) for w in ref.W]
    for a, b in zip(ref.W, mine.W):
        assert torch.equal(a, b)
    sw = Bnd.Switcher(ref.W, ref.A, ref.B, cfg.n_layers, len(cfg.targets), cfg.n_experts,
                      cfg.rank, cfg.alpha, device=torch.cuda.current_device())
    desc = _desc_of(mine)
    routes = make_routes(np.array([[1, 3], [4, 1]], np.int32),
                         np.array([[0.625, 0.375], [0.8, 0.2]], np.float32))
    r_np = routes_to_np(routes)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    p = lambda t: None if t is None else Bnd.Switcher.route_ptr(routes, t)
    A_h = [bits(a) for a in ref.A]
    B_h = [bits(b) for b in ref.B]
    before = W0
    for prev, cur in [(None, 0), (0, 1)]:
        sw.switch(p(prev), p(cur), stream)
        assert _noalloc(desc, p(prev), p(cur), status.data_ptr(), stream) == Bnd.ADAFUSE_OK
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert sw.status(stream) == 0
        pr = route_tuple(r_np, prev) if prev is not None else None
        cu = route_tuple(r_np, cur)
        for i, (a, b) in enumerate(zip(ref.W, mine.W)):
            got, want = bits(b), bits(a)
            rows = np.arange(got.shape[0], dtype=np.int64)
            # every element of the allocation-free result against the oracle
            # (one bf16 step, or the fp32 accumulation bound where W and dW
            # cancel), and the regular entry point's result the same way
            check_switch_rows(got, before[i], rows, got.shape[0], A_h[i], B_h[i], cfg.scale,
                              pr, cu)
            check_switch_rows(want, before[i], rows, got.shape[0], A_h[i], B_h[i], cfg.scale,
                              pr, cu)
            # the two entry points agree to one step away from cancellation
            d = ulp_dist(got, want)
            assert (d > 1).sum() <= max(2, d.size // 100000), (i, int(d.max()))
        before = [bits(w) for w in mine.W]
        # keep both models on the same pre-switch state for the next call
        for a, b in zip(ref.W, mine.W):
            a.copy_(b)
    sw.close()


@pytest.mark.gpu
def test_noalloc_many_weights_span_several_table_launches():
    # 2 x 70 = 140 weights: the table is written by two argument-carrying
    # launches (96 entries each at most); every weight must be switched with
    # its own W, A and B
    cfg = wl.custom("noalloc", 70, [("a", 136, 264), ("b", 264, 136)], n_experts=3, rank=8,
                    alpha=16.0, n_tokens=1, d=264)
    m = wl.make_model(cfg, device="cuda", seed=11)
    W0 = [bits(w) for w in m.W]
    routes = make_routes(np.array([[2, 0]], np.int32), np.array([[0.7, 0.3]], np.float32))
    r_np = routes_to_np(routes)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert _noalloc(_desc_of(m), None, Bnd.Switcher.route_ptr(routes, 0), status.data_ptr(),
                    stream) == Bnd.ADAFUSE_OK
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for i, w in enumerate(m.W):
        got = bits(w)
        rows = np.arange(i % 5, got.shape[0], 5, dtype=np.int64)
        check_switch_rows(got[rows], W0[i][rows], rows, got.shape[0], bits(m.A[i]),
                          bits(m.B[i]), cfg.scale, None, route_tuple(r_np, 0))


@pytest.mark.gpu
def test_noalloc_bad_route_reports_status_and_writes_nothing():
    cfg = wl.custom("noalloc", 1, SHAPES[:2], n_experts=4, rank=8, alpha=16.0, n_tokens=1,
                    d=392)
    m = wl.make_model(cfg, device="cuda", seed=5)
    W0 = [bits(w) for w in m.W]
    routes = make_routes(np.array([[0, 7]], np.int32), np.array([[0.5, 0.5]], np.float32))
    status = torch.zeros((1,), dtype=torch.int32, device="cuda")
    rc = _noalloc(_desc_of(m), None, Bnd.Switcher.route_ptr(routes, 0), status.data_ptr(),
                  torch.cuda.current_stream().cuda_stream)
    assert rc == Bnd.ADAFUSE_OK
    torch.cuda.synchronize()
    assert int(status.item()) == Bnd.ADAFUSE_STATUS_BAD_EXPERT
    for w, w0 in zip(m.W, W0):
        assert np.array_equal(bits(w), w0)


def test_noalloc_rejects_more_weights_than_its_scratch_holds():
    limit = 1638   # ADAFUSE_NOALLOC_MAX_WEIGHTS: 64 KiB / 40-byte entries
    ts = [("t", 8, 8, 16, 16, 16)] * (limit + 1)
    desc = Bnd.make_desc(limit + 1, 1, 2, 8, 16.0, ts)
    assert _noalloc(desc, None, None, None, None) == Bnd.ADAFUSE_ERR_UNSUPPORTED_SHAPE
