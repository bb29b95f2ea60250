"""Test helpers: bit-pattern conversions and comparisons (no method arithmetic)."""
import numpy as np
import torch


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> uint16 numpy bit patterns."""
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def from_bits(b: np.ndarray, device="cpu") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).to(device)


def ordered(u: np.ndarray) -> np.ndarray:
    u = u.astype(np.int32)
    return np.where(u & 0x8000, -(u & 0x7FFF), u)


def ulp_dist(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in bf16 steps between bit patterns (+0 == -0)."""
    return np.abs(ordered(a) - ordered(b))


def route_tuple(routes_np: np.ndarray, t: int):
    """Row t of an int32 [T, 4] route buffer -> (idx[2], gate[2]) for the oracle."""
    row = routes_np[t]
    return (row[:2].astype(np.int32), row[2:].view(np.float32).copy())


def routes_to_np(routes: torch.Tensor) -> np.ndarray:
    return routes.cpu().numpy().view(np.int32).reshape(-1, 4)


def make_routes(idx: np.ndarray, gate: np.ndarray, device="cuda") -> torch.Tensor:
    """idx [T,2] int32 + gate [T,2] fp32 -> device int32 [T, 4] route buffer."""
    T = idx.shape[0]
    buf = np.zeros((T, 4), dtype=np.int32)
    buf[:, :2] = idx
    buf[:, 2:] = np.ascontiguousarray(gate, dtype=np.float32).view(np.int32)
    return torch.from_numpy(buf).to(device)


def make_routes4(idx: np.ndarray, gate: np.ndarray, device="cuda") -> torch.Tensor:
    """idx [T,k] int32 + gate [T,k] fp32 (k <= 4) -> device int32 [T, 8] top-k
    route buffer (adafuse_route4 records; slots past k empty)."""
    T, k = idx.shape
    buf = np.zeros((T, 8), dtype=np.int32)
    buf[:, :4] = -1
    buf[:, :k] = idx
    g = np.zeros((T, 4), dtype=np.float32)
    g[:, :k] = gate
    buf[:, 4:] = g.view(np.int32)
    return torch.from_numpy(buf).to(device)


def routes4_to_np(routes: torch.Tensor) -> np.ndarray:
    return routes.cpu().numpy().view(np.int32).reshape(-1, 8)


def route4_tuple(routes_np: np.ndarray, t: int):
    """Row t of an int32 [T, 8] top-k route buffer -> (idx[4], gate[4]) for the oracle."""
    row = routes_np[t]
    return (row[:4].astype(np.int32), row[4:].view(np.float32).copy())


def pregate_topk_consistent(idx_gpu, idx_ref, z, h, Wr):
    """Top-k form of pregate_consistent: a token may differ from the fp64
    oracle only where the fp32 rounding bound makes the order ambiguous; the
    GPU's picks must then be an order the bound allows.  Returns the list of
    ambiguous token indices."""
    T, d = h.shape
    E = z.shape[1]
    bound = 2.0 * d * 2.0 ** -24 * (np.abs(h.astype(np.float64)) @ np.abs(Wr.astype(np.float64)))
    ambiguous = []
    for t in range(T):
        got = [int(x) for x in idx_gpu[t]]
        if got == [int(x) for x in idx_ref[t]]:
            continue

        def can_precede(x, y):
            return z[t, x] + bound[t, x] >= z[t, y] - bound[t, y]
        picks = [x for x in got if x >= 0]
        ok = len(set(picks)) == len(picks) and all(0 <= x < E for x in picks)
        for j, a in enumerate(picks):
            ok = ok and all(can_precede(a, e) for e in range(E) if e not in picks[:j + 1])
        assert ok, f"token {t}: gpu picked {got}, oracle {list(idx_ref[t])}, z={z[t]}"
        ambiguous.append(t)
    return ambiguous


def pregate_consistent(idx_gpu, idx_ref, z, h, Wr):
    """Accept a top-2 choice that differs from the fp64 oracle only where the
    fp32 rounding bound 2*d*2^-24*sum|h_i Wr_ie| makes the order ambiguous.
    Returns (number of exact matches, list of ambiguous token indices)."""
    T, d = h.shape
    bound = 2.0 * d * 2.0 ** -24 * (np.abs(h.astype(np.float64)) @ np.abs(Wr.astype(np.float64)))
    exact, ambiguous = 0, []
    for t in range(T):
        a, b = int(idx_gpu[t, 0]), int(idx_gpu[t, 1])
        if a == idx_ref[t, 0] and b == idx_ref[t, 1]:
            exact += 1
            continue
        E = z.shape[1]

        def can_precede(x, y):
            return z[t, x] + bound[t, x] >= z[t, y] - bound[t, y]
        ok = 0 <= a < E and (b == -1 or 0 <= b < E) and a != b
        ok = ok and all(can_precede(a, e) for e in range(E) if e != a)
        if b >= 0:
            ok = ok and all(can_precede(b, e) for e in range(E) if e not in (a, b))
        assert ok, f"token {t}: gpu picked {(a, b)}, oracle {tuple(idx_ref[t])}, z={z[t]}"
        ambiguous.append(t)
    return exact, ambiguous


def bf16_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_step(b: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at the given bit patterns (2^-133 when subnormal)."""
    e = (b.astype(np.int32) >> 7) & 0xFF
    return np.ldexp(1.0, np.where(e == 0, -133, e - 127 - 7))


def fp32_accum_gamma(rank: int, n_experts: int = 4) -> float:
    """Relative error bound of the fp32 path: rank products summed per expert,
    up to n_experts expert terms (at least four counted) and W combined, the
    coefficient rounded once."""
    return (rank + max(4, n_experts) + 4) * 2.0 ** -24


def check_switch_rows(after, before, rows, out, A, B, s, prev, cur, max_ulp=1):
    """Compare GPU rows with the oracle.

    Pass per element if it is within `max_ulp` bf16 steps of the oracle's
    bf16_rne(W + dW), or -- where the result cancels far below the terms it
    is formed from -- within half a step plus the fp32 accumulation bound
    gamma * (|W| + s * sum_e g_e sum_k |B_ek| |A_kj|) of the exact value.
    Returns (worst step distance, number of elements that needed the
    cancellation clause)."""
    import oracle
    want, exact = oracle.switch_rows(before, rows, out, A, B, s, prev, cur, exact=True)
    d = ulp_dist(after, want)
    bad = d > max_ulp
    if not bad.any():
        return int(d.max()) if d.size else 0, 0
    brows = np.unique(np.nonzero(bad)[0])
    M = np.abs(bf16_to_f64(before[brows]))
    Af, Bf = np.abs(bf16_to_f64(A)), np.abs(bf16_to_f64(B))
    for rt in (prev, cur):
        if rt is None:
            continue
        for e, g in zip(rt[0], rt[1]):
            if e < 0:
                continue
            M += s * abs(float(g)) * (Bf[e][rows[brows]] @ Af[e])
    r = A.shape[1]
    n_exp = sum(int(np.sum(np.asarray(rt[0]) >= 0)) for rt in (prev, cur) if rt is not None)
    gpu = bf16_to_f64(after[brows])
    tol = 0.5 * bf16_step(after[brows]) + fp32_accum_gamma(r, n_exp) * M
    sub_bad = bad[brows]
    err = np.abs(gpu - exact[brows])
    ok = err <= tol
    if not np.all(ok[sub_bad]):
        i, j = np.argwhere(sub_bad & ~ok)[0]
        raise AssertionError(
            f"row {rows[brows[i]]} col {j}: gpu {gpu[i, j]!r} exact {exact[brows[i], j]!r} "
            f"err {err[i, j]:.3e} > tol {tol[i, j]:.3e} ({d[brows[i], j]} steps)")
    return int(d[~bad].max()) if (~bad).any() else 0, int(bad.sum())
