"""Seeded synthetic workloads for the adapter switch.

This module only draws random inputs (shapes, distributions, route sequences);
it holds none of the method's arithmetic.  Both the CUDA path's tests/bench
and the CPU oracle's tests take their inputs from here.

Shapes stand in for the decoders the AdaFuse pages evaluate on (LLaMA2-7B and
Mistral-7B decoding, gist.science technical summary, section 4); the 13B and
Llama-3-8B GQA shapes widen the set.  Weights are random, not trained.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Tuple

import numpy as np
import torch

BASE_SEED = 20260312


@dataclasses.dataclass(frozen=True)
class Target:
    name: str
    out: int
    inn: int


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    n_layers: int
    d: int
    targets: Tuple[Target, ...]
    n_experts: int
    rank: int
    alpha: float
    n_tokens: int
    route_mode: str = "router"      # router | share_one | zipf
    repeat_p: float = 0.0            # probability h[t] := h[t-1]
    share_p: float = 0.0             # share_one: probability one expert is kept
    zipf_a: float = 1.1
    pregate_T: int = 0               # extra router-throughput batch (0 = none)
    w_std: float = 0.02
    b_std: float = 0.01
    wr_std: float = 0.05
    index: int = 0
    shape: str = ""                  # the decoder whose weight shapes these are

    @property
    def scale(self) -> float:
        return self.alpha / self.rank

    @property
    def a_std(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def n_pairs(self) -> int:
        return self.n_layers * len(self.targets)

    def w_elems(self) -> int:
        return self.n_layers * sum(t.out * t.inn for t in self.targets)

    def w_bytes_per_switch(self) -> int:
        """W bytes read + written by one non-identity switch (bf16)."""
        return 4 * self.w_elems()

    def seed(self) -> int:
        return BASE_SEED + self.index


def _llama(d, ffn, kv=None):
    kv = d if kv is None else kv
    return (Target("q_proj", d, d), Target("k_proj", kv, d), Target("v_proj", kv, d),
            Target("o_proj", d, d), Target("gate_proj", ffn, d), Target("up_proj", ffn, d),
            Target("down_proj", d, ffn))


CONFIGS = {
    "tiny": Config("tiny", 2, 256, (Target("q_proj", 256, 256), Target("v_proj", 256, 256)),
                   n_experts=4, rank=4, alpha=8.0, n_tokens=16, index=0, shape="tiny"),
    "7b": Config("7b", 32, 4096, _llama(4096, 11008), n_experts=8, rank=8, alpha=16.0,
                 n_tokens=64, index=1, shape="Llama-2-7B-shaped"),
    "7b-r64": Config("7b-r64", 32, 4096, _llama(4096, 11008), n_experts=16, rank=64,
                     alpha=128.0, n_tokens=64, route_mode="share_one", share_p=0.3, index=2,
                     shape="Llama-2-7B-shaped"),
    "13b": Config("13b", 40, 5120, _llama(5120, 13824), n_experts=8, rank=16, alpha=32.0,
                  n_tokens=128, repeat_p=0.1, index=3, shape="Llama-2-13B-shaped"),
    "l3-8b": Config("l3-8b", 32, 4096, _llama(4096, 14336, kv=1024), n_experts=8, rank=16,
                    alpha=32.0, n_tokens=256, route_mode="zipf", pregate_T=4096, index=4,
                    shape="Llama-3-8B-shaped (GQA)"),
}


def describe_targets(cfg: Config) -> str:
    """'q_proj 4096x4096, ...' with equal shapes grouped: 'q,o 4096x4096; k,v 1024x4096'."""
    groups = {}
    for t in cfg.targets:
        groups.setdefault((t.out, t.inn), []).append(t.name.replace("_proj", ""))
    return "; ".join(f"{','.join(n)} {o}x{i}" for (o, i), n in groups.items())


def scaled(cfg: Config, n_layers: Optional[int] = None, **kw) -> Config:
    """A copy of ``cfg`` with fewer layers (for parity runs at full matrix sizes)."""
    return dataclasses.replace(cfg, n_layers=n_layers or cfg.n_layers, **kw)


def custom(name, n_layers, targets, n_experts, rank, alpha, n_tokens, d=None, **kw) -> Config:
    ts = tuple(Target(*t) if not isinstance(t, Target) else t for t in targets)
    return Config(name, n_layers, d or ts[0].inn, ts, n_experts, rank, alpha, n_tokens, **kw)


# ---------------------------------------------------------------------------
# tensors

@dataclasses.dataclass
class Model:
    cfg: Config
    W: List[torch.Tensor]      # [L*nt] each [out, in] bf16
    A: List[torch.Tensor]      # [L*nt] each [E, r, in] bf16
    B: List[torch.Tensor]      # [L*nt] each [E, out, r] bf16
    Wr: torch.Tensor           # [d, E] fp32


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_model(cfg: Config, device="cpu", seed: Optional[int] = None) -> Model:
    """Random-init weights of the config's shapes (seeded Philox on ``device``)."""
    seed = cfg.seed() if seed is None else seed
    g = _gen(device, seed)
    W, A, B = [], [], []
    E, r = cfg.n_experts, cfg.rank
    for _layer in range(cfg.n_layers):
        for t in cfg.targets:
            w = torch.empty((t.out, t.inn), dtype=torch.float32, device=device)
            w.normal_(0.0, cfg.w_std, generator=g)
            W.append(w.to(torch.bfloat16))
            del w
            a = torch.empty((E, r, t.inn), dtype=torch.float32, device=device)
            a.normal_(0.0, cfg.a_std, generator=g)
            A.append(a.to(torch.bfloat16))
            b = torch.empty((E, t.out, r), dtype=torch.float32, device=device)
            b.normal_(0.0, cfg.b_std, generator=g)
            B.append(b.to(torch.bfloat16))
    Wr = torch.empty((cfg.d, E), dtype=torch.float32, device=device)
    Wr.normal_(0.0, cfg.wr_std, generator=g)
    return Model(cfg, W, A, B, Wr)


def make_hidden(cfg: Config, T: Optional[int] = None, device="cpu",
                seed: Optional[int] = None) -> torch.Tensor:
    """h [T, d] fp32 ~ N(0,1); with ``repeat_p`` some rows copy the previous row."""
    T = cfg.n_tokens if T is None else T
    seed = (cfg.seed() if seed is None else seed) + 7919
    g = _gen(device, seed)
    h = torch.empty((T, cfg.d), dtype=torch.float32, device=device)
    h.normal_(0.0, 1.0, generator=g)
    if cfg.repeat_p > 0 and T > 1:
        rng = np.random.default_rng(seed)
        rep = rng.random(T) < cfg.repeat_p
        for t in range(1, T):
            if rep[t]:
                h[t].copy_(h[t - 1])
    return h


def synth_routes(cfg: Config, T: Optional[int] = None, seed: Optional[int] = None):
    """Route records drawn directly (configs whose switch sequence is synthesised).

    share_one: with probability ``share_p`` exactly one expert of the previous
    token is kept, otherwise the pair is disjoint from it.
    zipf: the C(E,2) unordered pairs are ranked by a seeded permutation and
    drawn with P(rank k) proportional to k^-zipf_a.
    Gates: g0 ~ U(0.5, 1), g1 = 1 - g0; slot 0 holds the larger gate.
    Returns idx [T, 2] int32, gate [T, 2] fp32 (numpy).
    """
    T = cfg.n_tokens if T is None else T
    E = cfg.n_experts
    rng = np.random.default_rng((cfg.seed() if seed is None else seed) + 104729)
    idx = np.zeros((T, 2), dtype=np.int32)
    gate = np.zeros((T, 2), dtype=np.float32)
    pairs = [(a, b) for a in range(E) for b in range(a + 1, E)]
    order = rng.permutation(len(pairs))
    w = np.arange(1, len(pairs) + 1, dtype=np.float64) ** (-cfg.zipf_a)
    w /= w.sum()
    prev = None
    for t in range(T):
        if cfg.route_mode == "zipf":
            a, b = pairs[order[rng.choice(len(pairs), p=w)]]
        else:
            if prev is None:
                a, b = rng.choice(E, size=2, replace=False)
            elif rng.random() < cfg.share_p:
                keep = prev[rng.integers(2)]
                others = [e for e in range(E) if e not in prev]
                a, b = keep, others[rng.integers(len(others))]
            else:
                others = [e for e in range(E) if e not in prev]
                a, b = rng.choice(others, size=2, replace=False)
        g0 = np.float32(rng.uniform(0.5, 1.0))
        g1 = np.float32(1.0) - g0
        if rng.random() < 0.5:
            a, b = b, a
        idx[t] = (a, b)
        gate[t] = (g0, g1)
        prev = (int(a), int(b))
    return idx, gate
