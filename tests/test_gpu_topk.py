"""GPU parity of top-k routing (k = 1..4) against the fp64 oracle.

The AdaFuse router is top-2 (gist.science technical summary, section 2-ga);
the top-k entry points widen it to k picks by the same rule, and the fused
switch (section 2-na) then un-merges up to k experts and merges up to k, so
one in-place switch touches up to 8 experts: the tensor-core kernels fill
TMEM with batches of at most four accumulators.  Bars as for top-2: expert
indices bit-exact (outside the fp32 ambiguity bound), gates within 1e-5
relative, every W element within 1 bf16 step of the oracle in lockstep.
"""
import numpy as np
import pytest
import torch

import oracle
from weight_merge_b200 import binding as Bnd
from weight_merge_b200 import workloads as wl

from .util import (bits, check_switch_rows, make_routes4, pregate_topk_consistent, route4_tuple,
                   routes4_to_np)

pytestmark = pytest.mark.gpu

MMA, TC, TC2, TF = (Bnd.ADAFUSE_KERNEL_MMA_SYNC, Bnd.ADAFUSE_KERNEL_TCGEN05,
                    Bnd.ADAFUSE_KERNEL_TCGEN05_PAIR, Bnd.ADAFUSE_KERNEL_TCGEN05_FOLD)
GATE_RTOL = 1e-5
# tokens whose fp32 pick may differ from the fp64 oracle (each one checked to
# lie inside the fp32 rounding bound); none are expected at these sizes
AMBIGUOUS_MAX = 1


@pytest.fixture(scope="module", autouse=True)
def built():
    from weight_merge_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    oracle.build()


def stream():
    return torch.cuda.current_stream().cuda_stream


def switcher(model, kernel=Bnd.ADAFUSE_KERNEL_AUTO):
    c = model.cfg
    sw = Bnd.Switcher(model.W, model.A, model.B, c.n_layers, len(c.targets), c.n_experts,
                      c.rank, c.alpha, device=torch.cuda.current_device())
    sw.set_kernel(kernel)
    return sw


def kernels_for(rank):
    if rank <= 8:
        return [MMA, TC, TF]
    return [MMA, TC, TC2] if rank % 8 == 0 else [MMA]


# --------------------------------------------------------------------------
# pre-gating

@pytest.mark.parametrize("T,d,E,k", [(1, 4096, 8, 4), (7, 256, 4, 3), (64, 4096, 16, 4),
                                     (300, 512, 6, 3), (4096, 4096, 8, 4), (33, 5120, 16, 1),
                                     (9, 128, 3, 4), (257, 2944, 12, 2)])
def test_pregate_topk_matches_oracle(T, d, E, k):
    cfg = wl.custom("p", 1, [("q", 8, 8)], n_experts=E, rank=8, alpha=16, n_tokens=T, d=d)
    sw = switcher(wl.make_model(cfg, device="cuda", seed=5 + E))
    g = torch.Generator(device="cuda").manual_seed(200 + T + k)
    h = torch.randn((T, d), generator=g, device="cuda")
    Wr = torch.randn((d, E), generator=g, device="cuda") * 0.05
    routes = torch.zeros((T, 8), dtype=torch.int32, device="cuda")
    sw.pregate_topk(h, Wr, k, routes, stream())
    torch.cuda.synchronize()
    got = routes4_to_np(routes)
    h_np, Wr_np = h.cpu().numpy(), Wr.cpu().numpy()
    idx_ref, gate_ref, z = oracle.pregate_topk(h_np, Wr_np, k, return_logits=True)
    amb = pregate_topk_consistent(got[:, :k], idx_ref, z, h_np, Wr_np)
    print(f"ambiguous tokens: {len(amb)} of {T}")
    assert len(amb) <= AMBIGUOUS_MAX
    match = np.all(got[:, :k] == idx_ref, axis=1)
    gates = got[:, 4:].view(np.float32)
    np.testing.assert_allclose(gates[match, :k], gate_ref[match], rtol=GATE_RTOL, atol=1e-30)
    # slots past k are empty
    assert np.all(got[:, k:4] == -1) and np.all(gates[:, k:] == 0.0)


@pytest.mark.parametrize("E", [2, 8, 16])
def test_pregate_topk_with_k2_is_the_top2_router_bit_for_bit(E):
    T, d = 512, 1024
    cfg = wl.custom("p", 1, [("q", 8, 8)], n_experts=E, rank=8, alpha=16, n_tokens=T, d=d)
    sw = switcher(wl.make_model(cfg, device="cuda"))
    g = torch.Generator(device="cuda").manual_seed(31)
    h = torch.randn((T, d), generator=g, device="cuda")
    Wr = torch.randn((d, E), generator=g, device="cuda") * 0.05
    r2 = torch.zeros((T, 4), dtype=torch.int32, device="cuda")
    rk = torch.zeros((T, 8), dtype=torch.int32, device="cuda")
    sw.pregate(h, Wr, r2, stream())
    sw.pregate_topk(h, Wr, 2, rk, stream())
    torch.cuda.synchronize()
    assert torch.equal(rk[:, 0:2], r2[:, 0:2])
    assert torch.equal(rk[:, 4:6], r2[:, 2:4])


def test_pregate_topk_route_does_not_depend_on_batch_size():
    T, d, E, k = 1024, 2048, 8, 3
    cfg = wl.custom("p", 1, [("q", 8, 8)], n_experts=E, rank=8, alpha=16, n_tokens=T, d=d)
    sw = switcher(wl.make_model(cfg, device="cuda"))
    g = torch.Generator(device="cuda").manual_seed(77)
    h = torch.randn((T, d), generator=g, device="cuda")
    Wr = torch.randn((d, E), generator=g, device="cuda") * 0.05
    batch = torch.zeros((T, 8), dtype=torch.int32, device="cuda")
    sw.pregate_topk(h, Wr, k, batch, stream())
    single = torch.zeros((T, 8), dtype=torch.int32, device="cuda")
    for t in range(0, T, 97):
        sw.pregate_topk(h[t:t + 1], Wr, k, single[t:t + 1], stream())
    torch.cuda.synchronize()
    rows = list(range(0, T, 97))
    assert torch.equal(batch[rows], single[rows])


def test_pregate_topk_rejects_bad_k():
    cfg = wl.custom("p", 1, [("q", 8, 8)], n_experts=4, rank=8, alpha=16, n_tokens=1, d=64)
    m = wl.make_model(cfg, device="cuda")
    sw = switcher(m)
    h = torch.randn((1, 64), device="cuda")
    routes = torch.zeros((1, 8), dtype=torch.int32, device="cuda")
    for k in (0, 5):
        with pytest.raises(Bnd.AdafuseError):
            sw.pregate_topk(h, m.Wr, k, routes, stream())


# --------------------------------------------------------------------------
# the switch with top-k routes

RAGGED = [("a", 200, 136), ("b", 8, 8), ("c", 264, 392), ("d", 128, 256), ("e", 136, 8)]
# blocked tensor maps (every in a multiple of 64), half-width last tiles
RAGGED_BLOCKED = [("a", 200, 192), ("b", 8, 64), ("c", 264, 320), ("d", 128, 256), ("e", 136, 64)]
RANKS = [(9, 4), (9, 8), (9, 16), (9, 24), (10, 64)]


def _lockstep(sw, model, routes, steps, A_h, B_h, rows_of=None):
    cfg = model.cfg
    r_np = routes4_to_np(routes)
    ncancel = nchecked = 0
    for (p, c) in steps:
        sel = [np.arange(w.shape[0], dtype=np.int64) if rows_of is None else rows_of(i, w.shape[0])
               for i, w in enumerate(model.W)]
        before = [bits(w[torch.as_tensor(r, device="cuda")]) for w, r in zip(model.W, sel)]
        sw.switch_topk(Bnd.Switcher.route4_ptr(routes, p), Bnd.Switcher.route4_ptr(routes, c),
                       stream())
        torch.cuda.synchronize()
        assert sw.status(stream()) == 0
        prev = route4_tuple(r_np, p) if p is not None else None
        cur = route4_tuple(r_np, c) if c is not None else None
        for i, w in enumerate(model.W):
            after = bits(w[torch.as_tensor(sel[i], device="cuda")])
            try:
                _, nc = check_switch_rows(after, before[i], sel[i], w.shape[0], A_h[i], B_h[i],
                                          cfg.scale, prev, cur, 1)
            except AssertionError as ex:
                raise AssertionError(f"switch {(p, c)} weight {i}: {ex}") from None
            ncancel += nc
            nchecked += after.size
    assert ncancel <= max(2, nchecked * 1e-5), (ncancel, nchecked)


def _ragged_routes(E, seed):
    rng = np.random.default_rng(seed)
    idx = np.full((7, 4), -1, dtype=np.int32)
    gate = np.zeros((7, 4), dtype=np.float32)
    perm = lambda: rng.permutation(E)
    idx[0] = perm()[:4]                       # top-4
    p = perm()
    idx[1] = [x for x in p if x not in idx[0]][:4]   # disjoint from token 0: 8 experts
    idx[2] = [idx[1][2], idx[1][0]] + [x for x in perm() if x not in idx[1]][:2]  # two shared
    idx[3, :3] = perm()[:3]                   # a top-3 route (slot 3 empty)
    idx[4] = idx[3]                           # same experts, new gates
    idx[4, 3] = -1
    idx[5, :1] = perm()[:1]                   # top-1
    idx[6] = perm()[:4]
    for t in range(7):
        n = int(np.sum(idx[t] >= 0))
        g = np.sort(rng.uniform(0.05, 1.0, size=n))[::-1]
        gate[t, :n] = (g / g.sum()).astype(np.float32)
    gate[3, 3] = np.float32(np.nan)           # gate on an empty slot is ignored
    return idx, gate


@pytest.mark.parametrize("blocked", [False, True])
@pytest.mark.parametrize("E,r,kernel", [(E, r, k) for (E, r) in RANKS for k in kernels_for(r)])
def test_switch_topk_ragged_shapes_every_kernel(E, r, kernel, blocked):
    shapes = RAGGED_BLOCKED if blocked else RAGGED
    cfg = wl.custom("ragged", 2, shapes, n_experts=E, rank=r, alpha=2.0 * r, n_tokens=7,
                    d=shapes[0][2])
    model = wl.make_model(cfg, device="cuda", seed=3000 + 7 * r + E)
    sw = switcher(model, kernel)
    assert sw.kernel == kernel
    assert sw.map_layout == (Bnd.ADAFUSE_MAPS_BLOCKED if blocked else Bnd.ADAFUSE_MAPS_PLAIN)
    idx, gate = _ragged_routes(E, seed=r * 13 + E)
    routes = make_routes4(idx, gate)
    A_h, B_h = [bits(a) for a in model.A], [bits(b) for b in model.B]
    steps = [(None, 0), (0, 1), (1, 2), (2, 3), (3, 4), (4, 5), (5, 6), (6, None)]
    _lockstep(sw, model, routes, steps, A_h, B_h)


def _small(seed=3, E=8, r=16):
    cfg = wl.custom("s", 3, [("q", 256, 384), ("o", 384, 256)], n_experts=E, rank=r,
                    alpha=2.0 * r, n_tokens=4, d=384)
    return wl.make_model(cfg, device="cuda", seed=seed)


KERNEL_RANKS = [(MMA, 8), (TC, 8), (TC, 4), (TF, 8), (TF, 4), (TC, 16), (TC2, 16)]


@pytest.mark.parametrize("kernel,r", KERNEL_RANKS)
def test_switch_topk_identity_and_empty_routes(kernel, r):
    model = _small(r=r)
    sw = switcher(model, kernel)
    W0 = [bits(w) for w in model.W]
    idx = np.array([[1, 2, 5, 7], [7, 5, 2, 1], [-1, -1, -1, -1]], dtype=np.int32)
    gate = np.array([[0.4, 0.3, 0.2, 0.1], [0.4, 0.3, 0.2, 0.1], [0, 0, 0, 0]], np.float32)
    routes = make_routes4(idx, gate)
    p = lambda t: Bnd.Switcher.route4_ptr(routes, t)
    for prev, cur in [(p(0), p(0)), (p(1), p(1)), (None, None), (None, p(2)), (p(2), None)]:
        sw.switch_topk(prev, cur, stream())
    torch.cuda.synchronize()
    assert sw.status(stream()) == 0
    for w, w0 in zip(model.W, W0):
        assert np.array_equal(bits(w), w0)


@pytest.mark.parametrize("kernel,r", KERNEL_RANKS)
@pytest.mark.parametrize("bad", ["index_slot3", "index_low", "gate_nan_slot2"])
def test_switch_topk_bad_route_writes_nothing(bad, kernel, r):
    model = _small(seed=5, r=r)
    sw = switcher(model, kernel)
    W0 = [bits(w) for w in model.W]
    idx = np.array([[0, 1, 2, 3], [4, 5, 6, 7]], np.int32)
    gate = np.array([[0.4, 0.3, 0.2, 0.1], [0.4, 0.3, 0.2, 0.1]], np.float32)
    if bad == "index_slot3":
        idx[1, 3] = 8
    elif bad == "index_low":
        idx[1, 1] = -3
    else:
        gate[1, 2] = np.nan
    routes = make_routes4(idx, gate)
    sw.switch_topk(Bnd.Switcher.route4_ptr(routes, 0), Bnd.Switcher.route4_ptr(routes, 1), stream())
    st = sw.status(stream())
    want = Bnd.ADAFUSE_STATUS_BAD_GATE if bad.startswith("gate") else Bnd.ADAFUSE_STATUS_BAD_EXPERT
    assert st == want
    for w, w0 in zip(model.W, W0):
        assert np.array_equal(bits(w), w0)


@pytest.mark.parametrize("kernel,r", KERNEL_RANKS)
def test_switch_topk_layer_ranges_equal_one_full_switch(kernel, r):
    m1, m2 = _small(seed=9, r=r), _small(seed=9, r=r)
    s1, s2 = switcher(m1, kernel), switcher(m2, kernel)
    routes = make_routes4(np.array([[0, 1, 2, 3], [4, 5, 1, 0]], np.int32),
                          np.array([[0.4, 0.3, 0.2, 0.1], [0.5, 0.2, 0.2, 0.1]], np.float32))
    p = lambda t: Bnd.Switcher.route4_ptr(routes, t)
    s1.switch_topk(p(0), p(1), stream())
    s2.switch_topk_layers(0, 1, p(0), p(1), stream())
    s2.switch_topk_layers(1, 2, p(0), p(1), stream())
    torch.cuda.synchronize()
    for a, b in zip(m1.W, m2.W):
        assert np.array_equal(bits(a), bits(b))


@pytest.mark.parametrize("kernel,r", KERNEL_RANKS + [(TC2, 64)])
def test_rebase_topk_matches_oracle(kernel, r):
    model = _small(seed=11, r=r)
    sw = switcher(model, kernel)
    W0 = [w.clone() for w in model.W]
    for w in model.W:
        w.add_(1.0)
    sw.set_base(W0)
    idx = np.array([[3, 6, 0, 1], [2, -1, -1, -1]], np.int32)
    gate = np.array([[0.4, 0.3, 0.2, 0.1], [1.0, 0, 0, 0]], np.float32)
    routes = make_routes4(idx, gate)
    r_np = routes4_to_np(routes)
    A_h, B_h = [bits(a) for a in model.A], [bits(b) for b in model.B]
    for t in range(2):
        sw.rebase_topk(Bnd.Switcher.route4_ptr(routes, t), stream())
        torch.cuda.synchronize()
        assert sw.status(stream()) == 0
        for i, w in enumerate(model.W):
            rows = np.arange(w.shape[0], dtype=np.int64)
            check_switch_rows(bits(w), bits(W0[i]), rows, w.shape[0], A_h[i], B_h[i],
                              model.cfg.scale, None, route4_tuple(r_np, t))


@pytest.mark.parametrize("kernel,runs", [(Bnd.ADAFUSE_KERNEL_AUTO, TF), (TC, TC)])
def test_switch_topk_llama2_7b_shape_sampled(kernel, runs):
    """The 7B shape (E = 8, r = 8) with top-4 routes from the router: every
    in-place switch touches up to 8 experts.  AUTO sums them in the folded
    kernel's one accumulator (the launch the benchmark times); the
    four-accumulator kernel takes two TMEM batches per tile."""
    cfg = wl.CONFIGS["7b"]
    torch.cuda.empty_cache()
    model = wl.make_model(cfg, device="cuda")
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    sw = switcher(model, kernel)
    created = free0 - torch.cuda.mem_get_info()[0]
    # the context holds its tile table (8 B per 128 x 128 tile), three tensor
    # maps and one descriptor per weight; the folded kernel's operand buffer
    # (437 MB here) waits for the first folded switch
    table = 8 * 395264 + len(model.W) * (3 * 128 + 64)
    assert created < table + (16 << 20), created
    assert sw.topk_kernel == runs
    A_h, B_h = [bits(a) for a in model.A], [bits(b) for b in model.B]
    T, k = 3, 4
    h = wl.make_hidden(cfg, T=T, device="cuda")
    routes = torch.zeros((T, 8), dtype=torch.int32, device="cuda")
    sw.pregate_topk(h, model.Wr, k, routes, stream())
    torch.cuda.synchronize()
    idx_ref, _, z = oracle.pregate_topk(h.cpu().numpy(), model.Wr.cpu().numpy(), k,
                                        return_logits=True)
    assert len(pregate_topk_consistent(routes4_to_np(routes)[:, :k], idx_ref, z,
                                       h.cpu().numpy(), model.Wr.cpu().numpy())) == 0
    nt = len(cfg.targets)

    def rows_of(i, out):
        off = ((i // nt) * 7 + (i % nt) * 13) % 97
        return np.arange(off, out, 97, dtype=np.int64)
    _lockstep(sw, model, routes, [(None, 0), (0, 1), (1, 2)], A_h, B_h, rows_of)
    if runs == TF:
        # the first folded switch allocated the buffer
        assert free0 - torch.cuda.mem_get_info()[0] - created >= 400 << 20
    sw.close()
    del model
    torch.cuda.empty_cache()


def test_first_folded_switch_is_refused_inside_graph_capture():
    """The folded kernel's buffer is allocated by its first use, which may not
    sit inside stream capture: the call returns INVALID_ARG with nothing
    enqueued.  Made eagerly afterwards, the same switch matches the oracle."""
    model = _small(seed=14, r=8)
    sw = switcher(model)
    assert sw.topk_kernel == TF
    routes = make_routes4(np.array([[0, 2, 5, 1]], np.int32),
                          np.array([[0.4, 0.3, 0.2, 0.1]], np.float32))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with pytest.raises(Bnd.AdafuseError) as err:
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                sw.switch_topk(None, Bnd.Switcher.route4_ptr(routes, 0), side.cuda_stream)
    assert err.value.code == Bnd.ADAFUSE_ERR_INVALID_ARG
    del graph
    torch.cuda.synchronize()
    A_h, B_h = [bits(a) for a in model.A], [bits(b) for b in model.B]
    _lockstep(sw, model, routes, [(None, 0)], A_h, B_h)


# --------------------------------------------------------------------------
# limits: the largest expert count, odd sizes, misaligned routes

@pytest.mark.parametrize("kernel", [MMA, TC, TC2])
def test_switch_topk_sixty_four_experts_rank_64(kernel):
    """E = 64 (the largest expert count) at rank 64: the TMA maps span the
    whole stacked adapter tensors; experts come from the far end too."""
    cfg = wl.custom("e64", 1, [("a", 264, 136), ("b", 128, 392)], n_experts=64, rank=64,
                    alpha=128.0, n_tokens=3, d=136)
    model = wl.make_model(cfg, device="cuda", seed=64)
    sw = switcher(model, kernel)
    idx = np.array([[63, 0, 31, 62], [1, 63, 40, 2], [62, 61, -1, -1]], np.int32)
    gate = np.array([[0.4, 0.3, 0.2, 0.1], [0.5, 0.2, 0.2, 0.1], [0.6, 0.4, 0, 0]], np.float32)
    routes = make_routes4(idx, gate)
    A_h, B_h = [bits(a) for a in model.A], [bits(b) for b in model.B]
    _lockstep(sw, model, routes, [(None, 0), (0, 1), (1, 2)], A_h, B_h)


@pytest.mark.parametrize("T,d,E,k", [(5, 4100, 64, 4), (130, 1028, 64, 3), (1, 12, 5, 4)])
def test_pregate_topk_odd_sizes_and_many_experts(T, d, E, k):
    cfg = wl.custom("p", 1, [("q", 8, 8)], n_experts=E, rank=8, alpha=16, n_tokens=T, d=d)
    sw = switcher(wl.make_model(cfg, device="cuda", seed=E))
    g = torch.Generator(device="cuda").manual_seed(300 + d)
    h = torch.randn((T, d), generator=g, device="cuda")
    Wr = torch.randn((d, E), generator=g, device="cuda") * 0.05
    routes = torch.zeros((T, 8), dtype=torch.int32, device="cuda")
    sw.pregate_topk(h, Wr, k, routes, stream())
    torch.cuda.synchronize()
    got = routes4_to_np(routes)
    h_np, Wr_np = h.cpu().numpy(), Wr.cpu().numpy()
    idx_ref, gate_ref, z = oracle.pregate_topk(h_np, Wr_np, k, return_logits=True)
    amb = pregate_topk_consistent(got[:, :k], idx_ref, z, h_np, Wr_np)
    print(f"ambiguous tokens: {len(amb)} of {T}")
    assert len(amb) <= AMBIGUOUS_MAX
    match = np.all(got[:, :k] == idx_ref, axis=1)
    np.testing.assert_allclose(got[match, 4:4 + k].view(np.float32), gate_ref[match],
                               rtol=GATE_RTOL, atol=1e-30)


def test_topk_entry_points_refuse_misaligned_routes():
    model = _small(seed=12, r=8)
    sw = switcher(model)
    buf = torch.zeros((4, 8), dtype=torch.int32, device="cuda")
    bad = buf.data_ptr() + 4          # not 16-byte aligned
    good = buf.data_ptr()
    with pytest.raises(Bnd.AdafuseError):
        sw.switch_topk(bad, good, stream())
    with pytest.raises(Bnd.AdafuseError):
        sw.switch_topk(good, bad, stream())
    h = torch.zeros((1, 384), device="cuda")
    with pytest.raises(Bnd.AdafuseError):
        Bnd.adafuse_pregate_topk(sw.ctx, h.data_ptr(), 1, 384, model.Wr.data_ptr(), 2, bad, stream())
    sw.switch_topk_layers(0, 0, good, good, stream())   # an empty layer range is a no-op
    with pytest.raises(Bnd.AdafuseError):
        sw.switch_topk_layers(2, 2, good, good, stream())
