"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Bars (AdaFuse pages, gist.science technical summary sections 2-ga / 2-na,
with the tolerances of the build's contract):
  * expert indices bit-exact (ties to the lower index; a token whose fp64
    order is within the fp32 rounding bound may differ and is counted),
  * gates within 1e-5 relative,
  * every checked W element within 1 bf16 step of the oracle, which starts
    from the GPU's own pre-switch W (lockstep, so rounding drift over many
    switches does not accumulate into the comparison).
"""
import numpy as np
import pytest
import torch

import oracle
from weight_merge_b200 import binding as Bnd
from weight_merge_b200 import workloads as wl

from .util import (bits, check_switch_rows, make_routes, pregate_consistent, route_tuple,
                   routes_to_np, ulp_dist)

pytestmark = pytest.mark.gpu

GATE_RTOL = 1e-5
MAX_ULP = 1


@pytest.fixture(scope="module", autouse=True)
def built():
    from weight_merge_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    oracle.build()


def stream():
    return torch.cuda.current_stream().cuda_stream


MMA, TC, TC2, TF = (Bnd.ADAFUSE_KERNEL_MMA_SYNC, Bnd.ADAFUSE_KERNEL_TCGEN05,
                    Bnd.ADAFUSE_KERNEL_TCGEN05_PAIR, Bnd.ADAFUSE_KERNEL_TCGEN05_FOLD)


def make_switcher(model: wl.Model, kernel: int = Bnd.ADAFUSE_KERNEL_AUTO) -> Bnd.Switcher:
    c = model.cfg
    sw = Bnd.Switcher(model.W, model.A, model.B, c.n_layers, len(c.targets), c.n_experts,
                      c.rank, c.alpha, device=torch.cuda.current_device(),
                      names=[t.name for t in c.targets])
    sw.set_kernel(kernel)
    if kernel != Bnd.ADAFUSE_KERNEL_AUTO:
        assert sw.kernel == kernel
    return sw


def kernels_for(rank):
    if rank <= 8:
        return [MMA, TC, TF]
    return [MMA, TC, TC2] if rank % 8 == 0 else [MMA]


# (kernel, rank) for the small-model tests: each kernel at a rank it takes
KERNEL_RANKS = [(MMA, 8), (TC, 8), (TF, 8), (TF, 3), (TC2, 16)]


def host_ab(model):
    return [bits(a) for a in model.A], [bits(b) for b in model.B]


def check_pregate(sw, h, Wr, E):
    T, d = h.shape
    routes = torch.zeros((T, 4), dtype=torch.int32, device="cuda")
    sw.pregate(h, Wr, routes, stream())
    torch.cuda.synchronize()
    got = routes_to_np(routes)
    h_np, Wr_np = h.cpu().numpy(), Wr.cpu().numpy()
    idx_ref, gate_ref, z = oracle.pregate(h_np, Wr_np, return_logits=True)
    exact, amb = pregate_consistent(got[:, :2], idx_ref, z, h_np, Wr_np)
    match = np.all(got[:, :2] == idx_ref, axis=1)
    g = got[:, 2:].view(np.float32)
    np.testing.assert_allclose(g[match], gate_ref[match], rtol=GATE_RTOL, atol=0)
    return routes, got, amb


def lockstep(sw, model, routes_np, routes_dev, steps, rows_of, A_h, B_h):
    """Run switches (prev_t, cur_t) -- None = no route -- and compare the rows
    rows_of(pair_index, out) of every weight with the oracle after each.
    Returns (worst step distance, cancellation-clause elements, elements checked)."""
    cfg = model.cfg
    nt = len(cfg.targets)
    worst = ncancel = nchecked = 0
    for (p, c) in steps:
        sel = [rows_of(i, w.shape[0]) for i, w in enumerate(model.W)]
        before = [bits(w[torch.as_tensor(r, device="cuda")]) for w, r in zip(model.W, sel)]
        sw.switch(Bnd.Switcher.route_ptr(routes_dev, p), Bnd.Switcher.route_ptr(routes_dev, c),
                  stream())
        torch.cuda.synchronize()
        assert sw.status(stream()) == 0
        prev = route_tuple(routes_np, p) if p is not None else None
        cur = route_tuple(routes_np, c) if c is not None else None
        for i, w in enumerate(model.W):
            after = bits(w[torch.as_tensor(sel[i], device="cuda")])
            try:
                wd, nc = check_switch_rows(after, before[i], sel[i], w.shape[0], A_h[i], B_h[i],
                                           cfg.scale, prev, cur, MAX_ULP)
            except AssertionError as ex:
                raise AssertionError(f"switch {(p, c)} layer {i // nt} target "
                                     f"{cfg.targets[i % nt].name}: {ex}") from None
            worst, ncancel = max(worst, wd), ncancel + nc
            nchecked += after.size
    # the cancellation clause is for rare elements only
    assert ncancel <= max(2, nchecked * 1e-5), (ncancel, nchecked)
    return worst, ncancel, nchecked


def all_rows(i, out):
    return np.arange(out, dtype=np.int64)


# --------------------------------------------------------------------------
# pre-gating

@pytest.mark.parametrize("T,d,E", [(1, 4, 1), (1, 4096, 8), (7, 256, 4), (64, 4096, 8),
                                   (33, 5120, 16), (5, 264, 33), (9, 128, 64), (300, 512, 3),
                                   (4096, 4096, 8),    # the Llama-3-8B-shaped router batch
                                   (512, 1024, 16), (257, 2944, 12)])
def test_pregate_matches_oracle(T, d, E):
    cfg = wl.custom("p", 1, [("q", 8, 8)], n_experts=E, rank=8, alpha=16, n_tokens=T, d=d)
    model = wl.make_model(cfg, device="cuda", seed=11 + E)
    g = torch.Generator(device="cuda").manual_seed(100 + T)
    h = torch.randn((T, d), generator=g, device="cuda")
    Wr = torch.randn((d, E), generator=g, device="cuda") * 0.05
    sw = make_switcher(model)
    _, got, amb = check_pregate(sw, h, Wr, E)
    # tokens whose fp32 pick differs from the fp64 oracle, each checked to lie
    # inside the fp32 rounding bound; none are expected at these sizes
    print(f"ambiguous tokens: {len(amb)} of {T}")
    assert len(amb) <= 1
    if E == 1:
        assert np.all(got[:, 1] == -1)


@pytest.mark.parametrize("T,d,E", [(65, 12, 3), (131, 1028, 5), (1027, 2948, 8), (66, 3072, 8),
                                   (257, 4092, 7), (64, 1024, 2)])
def test_batch_router_matches_the_one_token_router_bit_for_bit(T, d, E):
    """The batch kernel (a warp pair per 4-token group, the odd warp adding
    its four virtual-warp sums on top of the even warp's) against one-token
    launches of the decode kernel, for every token: partial last groups,
    every chunk count 1..4, chunks past d, fewer than 8 experts.  Routes must
    agree bit for bit (indices and gate bits)."""
    cfg = wl.custom("p", 1, [("q", 8, 8)], n_experts=E, rank=8, alpha=16, n_tokens=T, d=d)
    sw = make_switcher(wl.make_model(cfg, device="cuda"))
    g = torch.Generator(device="cuda").manual_seed(T + d + E)
    h = torch.randn((T, d), generator=g, device="cuda")
    Wr = torch.randn((d, E), generator=g, device="cuda") * 0.05
    batch = torch.zeros((T, 4), dtype=torch.int32, device="cuda")
    sw.pregate(h, Wr, batch, stream())
    single = torch.zeros((T, 4), dtype=torch.int32, device="cuda")
    for t in range(T):
        sw.pregate(h[t:t + 1], Wr, single[t:t + 1], stream())
    torch.cuda.synchronize()
    assert torch.equal(batch, single)
    sw.close()


@pytest.mark.parametrize("E", [8, 16])
def test_pregate_route_does_not_depend_on_batch_size(E):
    """A token's route is bitwise the same whether it is gated alone or inside
    a large batch (the batched path stages Wr in shared memory, the small one
    reads it through L1, with the same arithmetic order)."""
    T, d = 1024, 2048
    cfg = wl.custom("p", 1, [("q", 8, 8)], n_experts=E, rank=8, alpha=16, n_tokens=T, d=d)
    sw = make_switcher(wl.make_model(cfg, device="cuda"))
    g = torch.Generator(device="cuda").manual_seed(77)
    h = torch.randn((T, d), generator=g, device="cuda")
    Wr = torch.randn((d, E), generator=g, device="cuda") * 0.05
    batch = torch.zeros((T, 4), dtype=torch.int32, device="cuda")
    sw.pregate(h, Wr, batch, stream())
    single = torch.zeros((T, 4), dtype=torch.int32, device="cuda")
    for t in range(0, T, 97):
        sw.pregate(h[t:t + 1], Wr, single[t:t + 1], stream())
    torch.cuda.synchronize()
    rows = list(range(0, T, 97))
    assert torch.equal(batch[rows], single[rows])


def test_pregate_duplicate_columns_tie_exactly():
    T, d, E = 64, 4096, 8
    cfg = wl.custom("p", 1, [("q", 8, 8)], n_experts=E, rank=8, alpha=16, n_tokens=T, d=d)
    sw = make_switcher(wl.make_model(cfg, device="cuda"))
    g = torch.Generator(device="cuda").manual_seed(5)
    h = torch.randn((T, d), generator=g, device="cuda").abs()
    Wr = torch.randn((d, E), generator=g, device="cuda") * 0.05
    Wr[:, 2] = Wr[:, 2].abs() + 0.5
    Wr[:, 6] = Wr[:, 2]
    routes = torch.zeros((T, 4), dtype=torch.int32, device="cuda")
    sw.pregate(h, Wr, routes, stream())
    got = routes_to_np(routes)
    assert np.all(got[:, 0] == 2) and np.all(got[:, 1] == 6)
    assert np.all(got[:, 2:].view(np.float32) == np.float32(0.5))


# --------------------------------------------------------------------------
# the switch, small sizes, every element

def test_tiny_sequence_lockstep_all_elements():
    cfg = wl.CONFIGS["tiny"]
    model = wl.make_model(cfg, device="cuda")
    sw = make_switcher(model)
    h = wl.make_hidden(cfg, device="cuda")
    routes, routes_np, amb = check_pregate(sw, h, model.Wr, cfg.n_experts)
    assert len(amb) == 0
    A_h, B_h = host_ab(model)
    steps = [(None, 0)] + [(t - 1, t) for t in range(1, cfg.n_tokens)] + [(cfg.n_tokens - 1, None)]
    lockstep(sw, model, routes_np, routes, steps, all_rows, A_h, B_h)


RAGGED = [("a", 200, 136), ("b", 8, 8), ("c", 264, 392), ("d", 128, 256), ("e", 136, 8)]
# every in a multiple of 64, so the context takes blocked tensor maps; in = 192,
# 64 and 320 end on a half-width (64-column) tile
RAGGED_BLOCKED = [("a", 200, 192), ("b", 8, 64), ("c", 264, 320), ("d", 128, 256), ("e", 136, 64)]
SHAPE_SETS = {"plain": (RAGGED, Bnd.ADAFUSE_MAPS_PLAIN),
              "blocked": (RAGGED_BLOCKED, Bnd.ADAFUSE_MAPS_BLOCKED)}


RANKS = [(1, 1), (3, 3), (4, 4), (5, 8), (16, 12), (4, 16), (6, 24), (3, 32), (4, 40), (5, 64)]


@pytest.mark.parametrize("layout", sorted(SHAPE_SETS))
@pytest.mark.parametrize("E,r,kernel", [(E, r, k) for (E, r) in RANKS for k in kernels_for(r)])
def test_ragged_shapes_every_rank_class(E, r, kernel, layout):
    shapes, want_layout = SHAPE_SETS[layout]
    cfg = wl.custom("ragged", 2, shapes, n_experts=E, rank=r, alpha=2.0 * r, n_tokens=6,
                    d=shapes[0][2])
    model = wl.make_model(cfg, device="cuda", seed=1000 + 7 * r + E)
    sw = make_switcher(model, kernel)
    if kernel != MMA:
        assert sw.map_layout == want_layout
    rng = np.random.default_rng(r * 31 + E)
    T = 6
    idx = rng.integers(0, E, size=(T, 2)).astype(np.int32)
    if E > 1:
        idx[2] = [idx[1][0], (idx[1][0] + 1) % E]   # token 2 shares an expert with token 1
    idx[3, 1] = -1                                # an empty slot
    if E > 1:
        idx[4] = [idx[4][0], idx[4][0]]           # the same expert twice
    gate = rng.uniform(0.05, 1.0, size=(T, 2)).astype(np.float32)
    routes = make_routes(idx, gate)
    routes_np = routes_to_np(routes)
    A_h, B_h = host_ab(model)
    steps = [(None, 0), (0, 1), (1, 2), (2, 3), (3, 4), (4, 5), (5, None)]
    lockstep(sw, model, routes_np, routes, steps, all_rows, A_h, B_h)


def _small_model(seed=3, E=4, r=8, L=3):
    cfg = wl.custom("s", L, [("q", 256, 384), ("o", 384, 256)], n_experts=E, rank=r,
                    alpha=2.0 * r, n_tokens=4, d=384)
    return wl.make_model(cfg, device="cuda", seed=seed)


@pytest.mark.parametrize("kernel,r", KERNEL_RANKS)
def test_identity_switches_leave_w_bit_identical(kernel, r):
    model = _small_model(r=r)
    sw = make_switcher(model, kernel)
    W0 = [bits(w) for w in model.W]
    idx = np.array([[1, 2], [2, 1], [0, 3]], dtype=np.int32)
    gate = np.array([[0.8, 0.2], [0.2, 0.8], [0.0, 0.0]], dtype=np.float32)
    routes = make_routes(idx, gate)
    p = lambda t: Bnd.Switcher.route_ptr(routes, t)
    for prev, cur in [(p(0), p(0)), (p(0), p(1)), (None, None), (None, p(2)), (p(2), None)]:
        sw.switch(prev, cur, stream())
    torch.cuda.synchronize()
    assert sw.status(stream()) == 0
    for w, w0 in zip(model.W, W0):
        assert np.array_equal(bits(w), w0)


@pytest.mark.parametrize("kernel,r", KERNEL_RANKS)
def test_merge_then_unmerge_restores_within_rounding(kernel, r):
    model = _small_model(seed=4, r=r)
    sw = make_switcher(model, kernel)
    W0 = [bits(w) for w in model.W]
    routes = make_routes(np.array([[0, 3]], np.int32), np.array([[0.55, 0.45]], np.float32))
    sw.switch(None, Bnd.Switcher.route_ptr(routes, 0), stream())
    W1 = [bits(w) for w in model.W]
    sw.switch(Bnd.Switcher.route_ptr(routes, 0), None, stream())
    torch.cuda.synchronize()
    for w, w0, w1 in zip(model.W, W0, W1):
        w2 = bits(w)
        assert ulp_dist(w1, w0).max() > 0
        # two roundings of at most half a step each (see the oracle pin)
        f = lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        e = lambda b: np.ldexp(1.0, np.where(((b >> 7) & 0xFF) == 0, -133,
                                             ((b.astype(np.int32) >> 7) & 0xFF) - 134))
        assert np.all(np.abs(f(w2) - f(w0)) <= 0.5 * e(w1) + 0.5 * e(w2) + 1e-30)


@pytest.mark.parametrize("kernel,r", KERNEL_RANKS)
def test_layer_ranges_equal_one_full_switch(kernel, r):
    m1, m2 = _small_model(seed=9, r=r), _small_model(seed=9, r=r)
    s1, s2 = make_switcher(m1, kernel), make_switcher(m2, kernel)
    routes = make_routes(np.array([[0, 1], [2, 3]], np.int32),
                         np.array([[0.7, 0.3], [0.6, 0.4]], np.float32))
    p = lambda t: Bnd.Switcher.route_ptr(routes, t)
    s1.switch(p(0), p(1), stream())
    s2.switch_layers(0, 1, p(0), p(1), stream())
    s2.switch_layers(1, 0, p(0), p(1), stream())
    s2.switch_layers(1, 2, p(0), p(1), stream())
    torch.cuda.synchronize()
    for a, b in zip(m1.W, m2.W):
        assert np.array_equal(bits(a), bits(b))
    with pytest.raises(Bnd.AdafuseError):
        s2.switch_layers(2, 2, p(0), p(1), stream())


@pytest.mark.parametrize("kernel,r", [(TC, 8), (TC2, 16), (TF, 8), (MMA, 12)])
def test_pipelined_switch_against_a_forward_equals_one_full_switch(kernel, r):
    """The switch pipelined against a decode forward: a side stream switches
    one layer per launch and records an event; the main stream waits for
    layer l's event and then reads layer l's weights (a stand-in forward,
    one GEMV per weight) while the side stream switches layer l + 1.  Two
    tokens in a row, the second side stream waiting for the first forward.
    W must end bit-identical to one full switch per token, and the forward
    must have read the switched weights."""
    m1 = _small_model(seed=19, r=r, L=4)
    m2 = _small_model(seed=19, r=r, L=4)
    s1, s2 = make_switcher(m1, kernel), make_switcher(m2, kernel)
    cfg = m1.cfg
    L, nt = cfg.n_layers, len(cfg.targets)
    routes = make_routes(np.array([[0, 1], [2, 3], [3, 0]], np.int32),
                         np.array([[0.7, 0.3], [0.6, 0.4], [0.55, 0.45]], np.float32))
    p = lambda t: Bnd.Switcher.route_ptr(routes, t)
    g = torch.Generator(device="cuda").manual_seed(3)
    xs = [torch.randn(w.shape[1], generator=g, device="cuda").to(torch.bfloat16)
          for w in m1.W[:nt]]
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    ev = [torch.cuda.Event() for _ in range(L)]
    ys = []
    for prev, cur in [(None, 0), (0, 1), (1, 2)]:
        s1.switch(p(prev), p(cur), main.cuda_stream)
        side.wait_stream(main)          # the previous forward is done with W
        for layer in range(L):
            s2.switch_layers(layer, 1, p(prev), p(cur), side.cuda_stream)
            ev[layer].record(side)
        y = []
        for layer in range(L):
            main.wait_event(ev[layer])
            y += [torch.mv(m2.W[layer * nt + k], xs[k]) for k in range(nt)]
        ys.append(y)
    torch.cuda.synchronize()
    assert s1.status(stream()) == 0 and s2.status(stream()) == 0
    for a, b in zip(m1.W, m2.W):
        assert np.array_equal(bits(a), bits(b))
    # the last token's forward read the fully switched weights
    for i, y in enumerate(ys[-1]):
        torch.testing.assert_close(y, torch.mv(m1.W[i], xs[i % nt]), rtol=0, atol=0)


@pytest.mark.parametrize("kernel,r,cap", [(TC, 8, 7), (TC, 16, 1), (TC2, 16, 7), (TC2, 64, 2),
                                           (TF, 8, 5), (MMA, 12, 3)])
def test_grid_cap_gives_the_same_w_bit_for_bit(kernel, r, cap):
    """adafuse_set_max_ctas only shrinks the persistent grid: each tile is
    computed the same way whichever CTA takes it, so a capped context and an
    uncapped one end with the same W, bit for bit, over full and layer-range
    switches (both tile schedules of the single-CTA and pair kernels)."""
    m1, m2 = _small_model(seed=23, r=r), _small_model(seed=23, r=r)
    s1, s2 = make_switcher(m1, kernel), make_switcher(m2, kernel)
    s2.set_max_ctas(cap)
    if kernel in (TC, TC2):
        s1.set_schedule(Bnd.ADAFUSE_SCHEDULE_STATIC)
    routes = make_routes(np.array([[0, 1], [2, 3], [1, 2]], np.int32),
                         np.array([[0.7, 0.3], [0.6, 0.4], [0.5, 0.5]], np.float32))
    p = lambda t: Bnd.Switcher.route_ptr(routes, t)
    for sw in (s1, s2):
        sw.switch(None, p(0), stream())
        sw.switch(p(0), p(1), stream())
        sw.switch_layers(1, 2, p(1), p(2), stream())
        sw.switch_layers(0, 1, p(1), p(2), stream())
    torch.cuda.synchronize()
    assert s1.status(stream()) == 0 and s2.status(stream()) == 0
    for a, b in zip(m1.W, m2.W):
        assert np.array_equal(bits(a), bits(b))
    with pytest.raises(Bnd.AdafuseError):
        s2.set_max_ctas(-1)


@pytest.mark.parametrize("kernel,r", [(TC, 8), (TC, 4), (TC, 16), (TC2, 16), (TC2, 32),
                                      (TC2, 64)])
def test_static_and_dynamic_tile_schedules_agree_bitwise(kernel, r):
    """The schedule only decides which CTA (CTA pair) takes a tile, never how
    a tile is computed: a static and a dynamic context give the same W, bit
    for bit, over repeated full and layer-range launches (the dynamic ticket
    counter is back at zero after every launch)."""
    m1, m2 = _small_model(seed=12, r=r), _small_model(seed=12, r=r)
    s1, s2 = make_switcher(m1, kernel), make_switcher(m2, kernel)
    s1.set_schedule(Bnd.ADAFUSE_SCHEDULE_STATIC)
    s2.set_schedule(Bnd.ADAFUSE_SCHEDULE_DYNAMIC)
    routes = make_routes(np.array([[0, 1], [2, 3], [1, 2], [3, 0]], np.int32),
                         np.array([[0.7, 0.3], [0.6, 0.4], [0.5, 0.5], [0.9, 0.1]], np.float32))
    p = lambda t: Bnd.Switcher.route_ptr(routes, t)
    for sw in (s1, s2):
        sw.switch(None, p(0), stream())
        sw.switch(p(0), p(1), stream())
        sw.switch_layers(1, 1, p(1), p(2), stream())
        sw.switch_layers(0, 1, p(1), p(2), stream())
        sw.switch(p(2), p(3), stream())
    torch.cuda.synchronize()
    assert s1.status(stream()) == 0 and s2.status(stream()) == 0
    for a, b in zip(m1.W, m2.W):
        assert torch.equal(a, b)
    with pytest.raises(Bnd.AdafuseError):
        s1.set_schedule(7)


@pytest.mark.parametrize("kernel,r", KERNEL_RANKS)
@pytest.mark.parametrize("bad", ["index_high", "index_low", "gate_nan", "gate_inf"])
def test_bad_route_sets_status_and_writes_nothing(bad, kernel, r):
    model = _small_model(seed=5, r=r)
    sw = make_switcher(model, kernel)
    W0 = [bits(w) for w in model.W]
    idx = np.array([[0, 1], [2, 3]], np.int32)
    gate = np.array([[0.6, 0.4], [0.5, 0.5]], np.float32)
    if bad == "index_high":
        idx[1, 1] = 4
    elif bad == "index_low":
        idx[1, 0] = -2
    elif bad == "gate_nan":
        gate[1, 0] = np.nan
    else:
        gate[1, 1] = np.inf
    routes = make_routes(idx, gate)
    sw.switch(Bnd.Switcher.route_ptr(routes, 0), Bnd.Switcher.route_ptr(routes, 1), stream())
    st = sw.status(stream())
    want = Bnd.ADAFUSE_STATUS_BAD_EXPERT if bad.startswith("index") else Bnd.ADAFUSE_STATUS_BAD_GATE
    assert st == want
    assert sw.status(stream()) == 0          # reading clears it
    for w, w0 in zip(model.W, W0):
        assert np.array_equal(bits(w), w0)


@pytest.mark.parametrize("kernel,r", KERNEL_RANKS)
def test_gate_on_empty_slot_is_ignored(kernel, r):
    model = _small_model(seed=6, r=r)
    sw = make_switcher(model, kernel)
    routes = make_routes(np.array([[1, -1]], np.int32), np.array([[1.0, np.nan]], np.float32))
    W0 = [bits(w) for w in model.W]
    sw.switch(None, Bnd.Switcher.route_ptr(routes, 0), stream())
    assert sw.status(stream()) == 0
    A_h, B_h = host_ab(model)
    for i, w in enumerate(model.W):
        rows = np.arange(w.shape[0], dtype=np.int64)
        check_switch_rows(bits(w), W0[i], rows, w.shape[0], A_h[i], B_h[i], model.cfg.scale,
                          None, (np.array([1, -1], np.int32), np.array([1.0, 0.0], np.float32)))


# --------------------------------------------------------------------------
# full Llama-shaped sizes, the launch the benchmark times, sampled rows

def _sample_rows(cfg, full_layers=()):
    nt = len(cfg.targets)

    def rows_of(i, out):
        layer = i // nt
        if layer in full_layers:
            return np.arange(out, dtype=np.int64)
        off = (layer * 7 + (i % nt) * 13) % 97
        return np.arange(off, out, 97, dtype=np.int64)
    return rows_of


def _full_size_case(name, n_switches, full_first=True, kernel=Bnd.ADAFUSE_KERNEL_AUTO):
    cfg = wl.CONFIGS[name]
    torch.cuda.empty_cache()
    model = wl.make_model(cfg, device="cuda")
    sw = make_switcher(model, kernel)
    assert sw.kernel in (TC, TC2, TF)  # a tensor-core kernel, as the benchmark launches
    A_h, B_h = host_ab(model)
    if cfg.route_mode == "router":
        h = wl.make_hidden(cfg, T=n_switches, device="cuda")
        routes, routes_np, amb = check_pregate(sw, h, model.Wr, cfg.n_experts)
        assert len(amb) <= 1
    else:
        idx, gate = wl.synth_routes(cfg, T=n_switches)
        routes = make_routes(idx, gate)
        routes_np = routes_to_np(routes)
    L = cfg.n_layers
    if full_first:
        lockstep(sw, model, routes_np, routes, [(None, 0)],
                 _sample_rows(cfg, full_layers=(0, L - 1)), A_h, B_h)
    steps = [(t - 1, t) for t in range(1, n_switches)]
    lockstep(sw, model, routes_np, routes, steps, _sample_rows(cfg), A_h, B_h)
    sw.close()
    del model
    torch.cuda.empty_cache()


def test_auto_picks_tensor_cores_when_rank_allows():
    for r, want in [(1, TC), (4, TC), (7, TC), (8, TC), (12, MMA), (16, TC2), (24, TC2), (64, TC2)]:
        cfg = wl.custom("k", 1, [("q", 64, 64)], n_experts=2, rank=r, alpha=2.0 * r, n_tokens=1)
        sw = make_switcher(wl.make_model(cfg, device="cuda"))
        assert sw.kernel == want
        # in-place top-k switches take the folded kernel wherever it runs
        assert sw.topk_kernel == (TF if r <= 8 else want)
        if want == MMA:
            with pytest.raises(Bnd.AdafuseError):
                sw.set_kernel(TC)
        if r <= 8:
            with pytest.raises(Bnd.AdafuseError):
                sw.set_kernel(TC2)
            sw.set_kernel(TF)
        else:
            with pytest.raises(Bnd.AdafuseError):
                sw.set_kernel(TF)


@pytest.mark.parametrize("kernel", [Bnd.ADAFUSE_KERNEL_AUTO, TC, TF])
def test_llama2_7b_shape_sampled(kernel):
    _full_size_case("7b", 3, kernel=kernel)


@pytest.mark.parametrize("kernel", [Bnd.ADAFUSE_KERNEL_AUTO, TC, TC2])
def test_llama2_7b_r64_shape_sampled(kernel):
    _full_size_case("7b-r64", 3, full_first=False, kernel=kernel)


@pytest.mark.parametrize("kernel", [Bnd.ADAFUSE_KERNEL_AUTO, TC2])
def test_llama2_13b_shape_sampled(kernel):
    _full_size_case("13b", 2, full_first=False, kernel=kernel)


def test_llama3_8b_gqa_shape_sampled():
    _full_size_case("l3-8b", 3, full_first=False)
