"""GPU parity of the re-base switch: W <- bf16_rne(W0 + s*sum_{e in cur} g B A).

The AdaFuse pages merge in place (gist.science technical summary, section
2-na); the re-base variant writes the same merged weight from a pristine copy
W0 instead, so its oracle is the in-place oracle with prev = none applied to
W0.  Checked for both kernels, ragged shapes and every rank class, with the
same tolerance as the in-place switch.
"""
import numpy as np
import pytest
import torch

import oracle
from weight_merge_b200 import binding as Bnd
from weight_merge_b200 import workloads as wl

from .util import bits, check_switch_rows, make_routes, route_tuple, routes_to_np

pytestmark = pytest.mark.gpu

MMA, TC, TC2, TF = (Bnd.ADAFUSE_KERNEL_MMA_SYNC, Bnd.ADAFUSE_KERNEL_TCGEN05,
                    Bnd.ADAFUSE_KERNEL_TCGEN05_PAIR, Bnd.ADAFUSE_KERNEL_TCGEN05_FOLD)
SHAPES = [("a", 200, 136), ("b", 264, 392), ("c", 128, 256), ("d", 8, 8)]
# every in a multiple of 64 (blocked tensor maps), half-width last tiles
SHAPES_BLOCKED = [("a", 200, 192), ("b", 264, 320), ("c", 128, 256), ("d", 8, 64)]


@pytest.fixture(scope="module", autouse=True)
def built():
    from weight_merge_b200 import build
    build.build()
    oracle.build()


def stream():
    return torch.cuda.current_stream().cuda_stream


def _setup(E, r, kernel, seed=0, shapes=SHAPES, layers=2):
    cfg = wl.custom("rebase", layers, shapes, n_experts=E, rank=r, alpha=2.0 * r, n_tokens=3,
                    d=shapes[0][2])
    m = wl.make_model(cfg, device="cuda", seed=seed)
    sw = Bnd.Switcher(m.W, m.A, m.B, cfg.n_layers, len(cfg.targets), cfg.n_experts, cfg.rank,
                      cfg.alpha, device=torch.cuda.current_device())
    sw.set_kernel(kernel)
    W0 = [w.clone() for w in m.W]
    # make W differ from W0 so a missed tile cannot pass as "unchanged"
    for w in m.W:
        w.add_(1.0)
    sw.set_base(W0)
    return cfg, m, sw, W0


def _check_against_oracle(cfg, m, W0, route, A_h, B_h):
    for i, w in enumerate(m.W):
        rows = np.arange(w.shape[0], dtype=np.int64)
        check_switch_rows(bits(w), bits(W0[i]), rows, w.shape[0], A_h[i], B_h[i], cfg.scale,
                          None, route)


@pytest.mark.parametrize("blocked", [False, True])
@pytest.mark.parametrize("E,r,kernel", [(3, 3, MMA), (4, 8, MMA), (4, 8, TC), (5, 16, TC),
                                        (3, 24, MMA), (4, 32, TC), (6, 64, TC), (5, 16, TC2),
                                        (3, 24, TC2), (4, 32, TC2), (6, 64, TC2), (3, 3, TC),
                                        (4, 4, TC), (4, 8, TF), (3, 3, TF)])
def test_rebase_matches_oracle_and_does_not_accumulate(E, r, kernel, blocked):
    cfg, m, sw, W0 = _setup(E, r, kernel, seed=31 * r + E,
                            shapes=SHAPES_BLOCKED if blocked else SHAPES)
    if kernel != MMA:
        assert sw.map_layout == (Bnd.ADAFUSE_MAPS_BLOCKED if blocked else Bnd.ADAFUSE_MAPS_PLAIN)
    W0_bits = [bits(w) for w in W0]
    A_h = [bits(a) for a in m.A]
    B_h = [bits(b) for b in m.B]
    idx = np.array([[0, 2 % E], [1 % E, -1], [2 % E, 0]], np.int32)
    gate = np.array([[0.7, 0.3], [1.0, 0.0], [0.55, 0.45]], np.float32)
    routes = make_routes(idx, gate)
    r_np = routes_to_np(routes)
    for t in range(3):
        sw.rebase(Bnd.Switcher.route_ptr(routes, t), stream())
        torch.cuda.synchronize()
        assert sw.status(stream()) == 0
        _check_against_oracle(cfg, m, W0, route_tuple(r_np, t), A_h, B_h)
    # an empty route copies the base back
    sw.rebase(None, stream())
    torch.cuda.synchronize()
    for w, w0 in zip(m.W, W0_bits):
        assert np.array_equal(bits(w), w0)
    # the base itself is never written
    for w0, b0 in zip(W0, W0_bits):
        assert np.array_equal(bits(w0), b0)


@pytest.mark.parametrize("kernel,r", [(MMA, 8), (TC, 8), (TF, 8), (TC2, 16)])
def test_rebase_layer_ranges_equal_full(kernel, r):
    cfg, m1, s1, _ = _setup(4, r, kernel, seed=3, layers=3)
    _, m2, s2, _ = _setup(4, r, kernel, seed=3, layers=3)
    routes = make_routes(np.array([[3, 1]], np.int32), np.array([[0.6, 0.4]], np.float32))
    cur = Bnd.Switcher.route_ptr(routes, 0)
    s1.rebase(cur, stream())
    s2.rebase_layers(0, 2, cur, stream())
    s2.rebase_layers(2, 1, cur, stream())
    torch.cuda.synchronize()
    for a, b in zip(m1.W, m2.W):
        assert torch.equal(a, b)


@pytest.mark.parametrize("kernel,r", [(MMA, 8), (TC, 8), (TF, 8), (TC2, 16)])
def test_rebase_bad_route_writes_nothing(kernel, r):
    cfg, m, sw, _ = _setup(4, r, kernel, seed=4)
    before = [bits(w) for w in m.W]
    routes = make_routes(np.array([[0, 9]], np.int32), np.array([[0.5, 0.5]], np.float32))
    sw.rebase(Bnd.Switcher.route_ptr(routes, 0), stream())
    assert sw.status(stream()) == Bnd.ADAFUSE_STATUS_BAD_EXPERT
    for w, b in zip(m.W, before):
        assert np.array_equal(bits(w), b)


def test_rebase_needs_a_base():
    cfg = wl.custom("nb", 1, SHAPES[:1], n_experts=2, rank=8, alpha=16.0, n_tokens=1, d=136)
    m = wl.make_model(cfg, device="cuda")
    sw = Bnd.Switcher(m.W, m.A, m.B, 1, 1, 2, 8, 16.0, device=torch.cuda.current_device())
    with pytest.raises(Bnd.AdafuseError):
        sw.rebase(None, stream())
    with pytest.raises(Bnd.AdafuseError):
        sw.set_base([m.W[0]])        # the base may not alias W


def test_rebase_llama2_7b_shape_sampled():
    cfg = wl.CONFIGS["7b"]
    torch.cuda.empty_cache()
    m = wl.make_model(cfg, device="cuda")
    sw = Bnd.Switcher(m.W, m.A, m.B, cfg.n_layers, len(cfg.targets), cfg.n_experts, cfg.rank,
                      cfg.alpha, device=torch.cuda.current_device())
    assert sw.kernel == TC
    W0 = [w.clone() for w in m.W]
    sw.set_base(W0)
    A_h = [bits(a) for a in m.A]
    B_h = [bits(b) for b in m.B]
    idx, gate = wl.synth_routes(cfg, T=2)
    routes = make_routes(idx, gate)
    r_np = routes_to_np(routes)
    nt = len(cfg.targets)
    for t in range(2):
        sw.rebase(Bnd.Switcher.route_ptr(routes, t), stream())
        torch.cuda.synchronize()
        assert sw.status(stream()) == 0
        for i, w in enumerate(m.W):
            off = ((i // nt) * 7 + (i % nt) * 13) % 97
            rows = np.arange(off, w.shape[0], 97, dtype=np.int64)
            sel = torch.as_tensor(rows, device="cuda")
            check_switch_rows(bits(w[sel]), bits(W0[i][sel]), rows, w.shape[0], A_h[i], B_h[i],
                              cfg.scale, None, route_tuple(r_np, t))
    sw.close()
    del m, W0
    torch.cuda.empty_cache()
