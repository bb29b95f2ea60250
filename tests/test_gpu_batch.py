"""GPU parity of batch decode: one routing decision for a batch of tokens
that shares one merged weight, against the fp64 oracle.

The pages route token by token (gist.science technical summary, section
2-ga); for a decode batch the reading is the token rule applied to the mean
of the tokens' router logits (oracle.pregate_batch).  Bars as for the token
router: expert indices bit-exact outside the fp32 rounding bound of the mean
logits, gates within 1e-5 relative; the switch that follows is the ordinary
fused switch, checked in lockstep against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from weight_merge_b200 import binding as Bnd
from weight_merge_b200 import workloads as wl

from .util import bits, check_switch_rows, route4_tuple, route_tuple

pytestmark = pytest.mark.gpu

GATE_RTOL = 1e-5


@pytest.fixture(scope="module", autouse=True)
def built():
    from weight_merge_b200 import build
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    oracle.build()


def stream():
    return torch.cuda.current_stream().cuda_stream


def switcher(model):
    c = model.cfg
    return Bnd.Switcher(model.W, model.A, model.B, c.n_layers, len(c.targets), c.n_experts,
                        c.rank, c.alpha, device=torch.cuda.current_device())


def _router(T, d, E, seed):
    cfg = wl.custom("b", 1, [("q", 8, 8)], n_experts=E, rank=8, alpha=16, n_tokens=T, d=d)
    model = wl.make_model(cfg, device="cuda", seed=seed)
    g = torch.Generator(device="cuda").manual_seed(500 + seed)
    h = torch.randn((T, d), generator=g, device="cuda")
    Wr = torch.randn((d, E), generator=g, device="cuda") * 0.05
    return model, h, Wr


def _gpu_batch(sw, h, Wr, k):
    """The batch route through the C ABI: the top-2 entry point for k = 2
    (16-byte record), the top-k one otherwise (32-byte record)."""
    if k == 2:
        r = torch.zeros((1, 4), dtype=torch.int32, device="cuda")
        sw.pregate_batch(h, Wr, r, stream())
        torch.cuda.synchronize()
        row = r.cpu().numpy()[0]
        return row[:2].copy(), row[2:].view(np.float32).copy()
    r = torch.zeros((1, 8), dtype=torch.int32, device="cuda")
    sw.pregate_batch_topk(h, Wr, k, r, stream())
    torch.cuda.synchronize()
    row = r.cpu().numpy()[0]
    return row[:k].copy(), row[4:4 + k].view(np.float32).copy()


def _mean_bound(h, Wr, z_tok):
    """fp32 rounding bound of the GPU's mean logits: each token's logit within
    2*d*2^-24*sum_i|h_i Wr_ie|, then T - 1 fp32 additions and one division."""
    T, d = h.shape
    per = 2.0 * d * 2.0 ** -24 * (np.abs(h.astype(np.float64)) @ np.abs(Wr.astype(np.float64)))
    return (per.sum(axis=0) + (T + 1) * 2.0 ** -24 * np.abs(z_tok).sum(axis=0)) / T


def _consistent(got, want, zbar, bound):
    """Indices equal, or the fp64 order is inside the bound for the picks made."""
    if list(got) == list(want):
        return False
    E = zbar.size
    picks = [int(x) for x in got if x >= 0]
    assert len(set(picks)) == len(picks) and all(0 <= x < E for x in picks), (got, want)
    for j, a in enumerate(picks):
        for e in range(E):
            if e in picks[:j + 1]:
                continue
            assert zbar[a] + bound[a] >= zbar[e] - bound[e], (got, want, zbar)
    return True


@pytest.mark.parametrize("T,d,E,k", [(1, 4096, 8, 2), (8, 4096, 8, 2), (64, 4096, 8, 4),
                                     (256, 5120, 8, 3), (4096, 4096, 8, 2), (33, 264, 16, 3),
                                     (5, 128, 64, 4), (7, 12, 5, 1), (130, 1028, 12, 2),
                                     (100, 4096, 4, 2)])
def test_pregate_batch_matches_oracle(T, d, E, k):
    model, h, Wr = _router(T, d, E, seed=T + E)
    sw = switcher(model)
    idx, gate = _gpu_batch(sw, h, Wr, k)
    h_np, Wr_np = h.cpu().numpy(), Wr.cpu().numpy()
    want_idx, want_gate, zbar = oracle.pregate_batch(h_np, Wr_np, k, return_logits=True)
    _, _, z_tok = oracle.pregate_topk(h_np, Wr_np, 1, return_logits=True)
    ambiguous = _consistent(idx, want_idx, zbar, _mean_bound(h_np, Wr_np, z_tok))
    assert not ambiguous, "no near ties expected in this data"
    np.testing.assert_allclose(gate, want_gate, rtol=GATE_RTOL, atol=1e-30)
    sw.close()


@pytest.mark.parametrize("E,d", [(8, 4096), (16, 4096), (5, 384)])
def test_batch_of_one_token_is_its_token_route_bit_for_bit(E, d):
    """The mean of one token's logits is the logits themselves, so the batch
    record of a one-token batch equals adafuse_pregate's record for it (both
    router kernels: E <= 8 streams h, E = 16 takes the other kernel)."""
    model, h, Wr = _router(6, d, E, seed=40 + E)
    sw = switcher(model)
    tok = torch.zeros((6, 4), dtype=torch.int32, device="cuda")
    sw.pregate(h, Wr, tok, stream())
    tok4 = torch.zeros((6, 8), dtype=torch.int32, device="cuda")
    sw.pregate_topk(h, Wr, 3, tok4, stream())
    one = torch.zeros((6, 4), dtype=torch.int32, device="cuda")
    one4 = torch.zeros((6, 8), dtype=torch.int32, device="cuda")
    for t in range(6):
        sw.pregate_batch(h[t:t + 1], Wr, one[t:t + 1], stream())
        sw.pregate_batch_topk(h[t:t + 1], Wr, 3, one4[t:t + 1], stream())
    torch.cuda.synchronize()
    assert torch.equal(tok, one)
    assert torch.equal(tok4, one4)
    sw.close()


def test_batch_route_drives_the_switch():
    """Two decode steps of a batch of 6 sequences: each step makes one batch
    route, and the switch moves W from the previous batch route to it; every
    W element matches the oracle in lockstep."""
    cfg = wl.custom("bs", 2, [("q", 264, 384), ("o", 384, 264)], n_experts=6, rank=8,
                    alpha=16.0, n_tokens=12, d=384)
    model = wl.make_model(cfg, device="cuda", seed=71)
    sw = switcher(model)
    h = wl.make_hidden(cfg, T=12, device="cuda", seed=72)
    routes = torch.zeros((2, 4), dtype=torch.int32, device="cuda")
    A_h, B_h = [bits(a) for a in model.A], [bits(b) for b in model.B]
    prev = None
    for step in range(2):
        hb = h[6 * step:6 * step + 6]
        sw.pregate_batch(hb, model.Wr, routes[step:step + 1], stream())
        W0 = [bits(w) for w in model.W]
        sw.switch(Bnd.Switcher.route_ptr(routes, prev), Bnd.Switcher.route_ptr(routes, step),
                  stream())
        torch.cuda.synchronize()
        assert sw.status(stream()) == 0
        r_np = routes.cpu().numpy()
        want_idx, want_gate = oracle.pregate_batch(hb.cpu().numpy(), model.Wr.cpu().numpy(), 2)
        assert np.array_equal(r_np[step, :2], want_idx)
        np.testing.assert_allclose(r_np[step, 2:].view(np.float32), want_gate, rtol=GATE_RTOL)
        p = None if prev is None else route_tuple(r_np, prev)
        for i, w in enumerate(model.W):
            rows = np.arange(w.shape[0], dtype=np.int64)
            check_switch_rows(bits(w), W0[i], rows, w.shape[0], A_h[i], B_h[i], cfg.scale, p,
                              route_tuple(r_np, step))
        prev = step
    sw.close()


def test_batch_topk_route_drives_the_topk_switch():
    cfg = wl.custom("bk", 1, [("q", 256, 256)], n_experts=8, rank=8, alpha=16.0, n_tokens=8,
                    d=256)
    model = wl.make_model(cfg, device="cuda", seed=81)
    sw = switcher(model)
    h = wl.make_hidden(cfg, T=8, device="cuda", seed=82)
    routes = torch.zeros((1, 8), dtype=torch.int32, device="cuda")
    sw.pregate_batch_topk(h, model.Wr, 4, routes, stream())
    W0 = [bits(w) for w in model.W]
    sw.switch_topk(None, Bnd.Switcher.route4_ptr(routes, 0), stream())
    torch.cuda.synchronize()
    assert sw.status(stream()) == 0
    r_np = routes.cpu().numpy()
    want_idx, _ = oracle.pregate_batch(h.cpu().numpy(), model.Wr.cpu().numpy(), 4)
    assert np.array_equal(r_np[0, :4], want_idx)
    rows = np.arange(256, dtype=np.int64)
    check_switch_rows(bits(model.W[0]), W0[0], rows, 256, bits(model.A[0]), bits(model.B[0]),
                      cfg.scale, None, route4_tuple(r_np, 0))
    sw.close()


def test_batch_limits():
    model, h, Wr = _router(8, 64, 4, seed=3)
    sw = switcher(model)
    r = torch.full((1, 8), 7, dtype=torch.int32, device="cuda")
    big = torch.zeros((Bnd.ADAFUSE_MAX_BATCH_TOKENS + 1, 64), device="cuda")
    with pytest.raises(Bnd.AdafuseError) as err:
        sw.pregate_batch(big, Wr, r, stream())
    assert err.value.code == Bnd.ADAFUSE_ERR_INVALID_ARG
    with pytest.raises(Bnd.AdafuseError):
        sw.pregate_batch_topk(h, Wr, 5, r, stream())
    sw.pregate_batch(h[:0], Wr, r, stream())        # an empty batch writes nothing
    torch.cuda.synchronize()
    assert torch.all(r == 7)
    sw.close()
