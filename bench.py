#!/usr/bin/env python
"""Benchmark of the AdaFuse decode-step hot path on B200.

One step = one token of the decode switch sequence: pre-gate the token's
first-layer hidden state (one top-2 routing decision), then one fused switch
launch that un-merges the previous token's experts and merges this token's
into every LoRA-targeted weight of every layer, in place.

value   = W bytes read + written by the switches / device time (GB/s), summed
          over ranks (each rank is an independent replica: the switch of one
          model has no exchange step).
e2e     = the same through the public API with the step's input (the token's
          hidden state) copied from pinned host memory and the step's result
          (its route record) copied back, inside the timed region.
roofline= the switch kernel's algorithmic W bytes / its CUDA-event duration,
          against the measured HBM copy bandwidth.

`--impl reference` times the fp64 CPU oracle on the host cores instead, on a
bounded row sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "adapter-switch latency & HBM GB/s (W read+write) at Llama-2-7B shape, % of peak"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="7b")
    ap.add_argument("--layers", type=int, default=None,
                    help="override the layer count (small cases for ncu captures)")
    ap.add_argument("--kernel", choices=["auto", "mma", "tc", "tc2", "fold"], default="auto",
                    help="switch kernel: tensor-core (tc), tensor-core on CTA pairs (tc2), "
                         "mma.sync (mma), or auto")
    ap.add_argument("--mode", choices=["switch", "rebase"], default="switch",
                    help="in-place switch (prev -> cur) or re-base from a pristine copy W0")
    ap.add_argument("--top-k", type=int, default=2,
                    help="experts per token: 2 is the top-2 router and route record; 1..4 "
                         "uses the top-k entry points (an in-place switch touches up to 2k)")
    ap.add_argument("--router-tokens", type=int, default=4096,
                    help="also time the pre-gate alone on this many tokens (0 = skip)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-torch-baseline", action="store_true",
                    help="skip the unfused per-weight torch addmm_ context figure")
    ap.add_argument("--schedule", choices=["auto", "dynamic", "static"], default="auto",
                    help="tile schedule of the tensor-core kernels (auto: dynamic for the "
                         "single-CTA kernel, static for the pair kernel)")
    ap.add_argument("--no-layerwise", action="store_true",
                    help="skip the per-layer-launch context figures (graph, per-layer routing)")
    ap.add_argument("--no-pipelined", action="store_true",
                    help="skip the switch pipelined against a stand-in forward")
    ap.add_argument("--configs", default="7b-r64,13b,l3-8b",
                    help="further workloads timed after the headline one (comma list, '' = none)")
    ap.add_argument("--config-steps", type=int, default=12,
                    help="timed switches per further workload (at least 10)")
    return ap.parse_args()


# the sources that define each profiled kernel and its launch (tensor maps,
# grid, shared memory); editing any of them voids that kernel's ncu figures
KERNEL_SOURCES = {
    "switch_tc_kernel": ["common.cuh", "sm100_ptx.cuh", "switch_tc.cuh", "switch_tc_host.cuh"],
    "switch_mma_kernel": ["common.cuh", "switch_mma.cuh"],
    "switch_tc2_kernel": ["common.cuh", "sm100_ptx.cuh", "switch_tc.cuh", "switch_tc2.cuh",
                          "switch_tc_host.cuh"],
    "switch_fold_kernel": ["common.cuh", "sm100_ptx.cuh", "switch_tc.cuh", "switch_fold.cuh",
                           "switch_tc_host.cuh"],
    "pregate_group_kernel": ["common.cuh", "sm100_ptx.cuh", "pregate.cuh"],
}


def kernel_source_hash(kernel_name="switch_tc_kernel"):
    """sha256 over the code of one kernel's sources and the ABI header
    (identifies the code an ncu capture was taken on).  Comments and
    whitespace are left out, so a documentation edit keeps the figures while
    any change to the code voids them."""
    import hashlib
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "weight_merge_b200", "csrc")
    files = [os.path.join(csrc, f) for f in KERNEL_SOURCES[kernel_name]]
    for f in files + [os.path.join(ROOT, "include", "adafuse.h")]:
        with open(f, encoding="utf-8") as fh:
            text = fh.read()
        # strip comments (string literals in these files hold no comment markers)
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        text = " ".join(text.split())
        h.update(os.path.basename(f).encode())
        h.update(text.encode())
    return h.hexdigest()


def profiled_traffic(kernel_name, workload):
    """DRAM bytes (read + write) per full launch from a committed ncu summary
    in profiles/, or None when none matches the current kernel sources."""
    d = os.path.join(ROOT, "profiles")
    if not os.path.isdir(d):
        return None
    want = kernel_source_hash(kernel_name)
    for f in sorted(os.listdir(d)):
        if not f.endswith(".md"):
            continue
        meta = {}
        for line in open(os.path.join(d, f)):
            if line.startswith("- ") and ": " in line:
                k, v = line[2:].strip().split(": ", 1)
                meta[k.strip("`")] = v.strip().strip("`")
        if (meta.get("kernel") == kernel_name and meta.get("workload") == workload
                and meta.get("kernel-source-sha256") == want
                and "dram-bytes-per-full-launch" in meta):
            return int(meta["dram-bytes-per-full-launch"])
    return None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def same_gpu_copy_gbs():
    """Read+write bytes of a 1 GiB bf16 device copy on this GPU, best of 5 (CUDA
    events): context for the roofline, whose denominator stays the driver's
    measured peak.  HBM bandwidth differs by several percent between boards."""
    import torch
    a = torch.empty(1 << 30, dtype=torch.bfloat16, device="cuda")
    b = torch.empty_like(a)
    best = 0.0
    for i in range(7):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        b.copy_(a)
        e1.record()
        torch.cuda.synchronize()
        if i >= 2:
            best = max(best, 4.0 * a.numel() / (e0.elapsed_time(e1) * 1e-3) / 1e9)
    del a, b
    torch.cuda.empty_cache()
    return best


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "timestamp")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None   # wall-clock bounds of the timed region

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9 and parts[1].isdigit():
                    rows.append(parts)
        except Exception:
            pass
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        # keep the samples taken inside the timed region
        window = "timed region"
        if self.t0 is not None and self.t1 is not None:
            import datetime
            inside = []
            for r in rows:
                try:
                    ts = datetime.datetime.strptime(r[9], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                except Exception:
                    continue
                if self.t0 <= ts <= self.t1:
                    inside.append(r)
            if inside:
                rows = inside
            else:
                window = "whole run (no sample fell inside the timed region)"
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [int(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": int(rows[0][2]),
                "reasons": reasons, "samples": len(rows), "window": window,
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())
                if any(r[3].replace(".", "").isdigit() for r in rows) else None}


# --------------------------------------------------------------------------
# CPU oracle timing (the reported baseline; never the product path)

_ORACLE_MODELS = {}


def oracle_rate(cfg, target_s=10.0, seed_layers=1):
    """fp64 oracle switch on a bounded row sample of layer 0 of the workload.
    Returns (W GB/s equivalent, threads, sample description, elapsed s)."""
    import numpy as np
    import torch

    import oracle
    from weight_merge_b200 import workloads as wl

    oracle.build()
    key = (cfg.name, seed_layers)
    if key not in _ORACLE_MODELS:
        _ORACLE_MODELS[key] = wl.make_model(wl.scaled(cfg, n_layers=seed_layers), device="cpu")
    m = _ORACLE_MODELS[key]
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    A = [bits(a) for a in m.A]
    B = [bits(b) for b in m.B]
    E = cfg.n_experts
    prev = (np.array([0, 1], np.int32), np.array([0.6, 0.4], np.float32))
    cur = (np.array([2, 3 % E], np.int32), np.array([0.7, 0.3], np.float32))

    def run(rows_per_target):
        elems = 0
        t0 = time.perf_counter()
        for i, w in enumerate(m.W):
            out = w.shape[0]
            rows = np.arange(min(rows_per_target, out), dtype=np.int64)
            oracle.switch_rows(bits(w[: len(rows)]), rows, out, A[i], B[i], cfg.scale, prev, cur)
            elems += len(rows) * w.shape[1]
        return elems, time.perf_counter() - t0

    e0, t0 = run(8)
    rate = e0 / max(t0, 1e-6)
    per_row = e0 / 8
    rows = int(max(8, min(4096, target_s * rate / per_row)))
    elems, dt = run(rows)
    gbs = elems * 4 / dt / 1e9
    desc = (f"fp64 oracle switch (4 experts: 2 out, 2 in) on the first {rows} rows of each of "
            f"the {len(cfg.targets)} targets of one layer, {elems/1e6:.1f} M W elements; "
            f"W-bytes rate extrapolates to a full switch")
    return gbs, oracle.num_threads(), desc, dt, elems


def workload_label(cfg, n_tokens, top_k=2):
    from weight_merge_b200 import workloads as wl
    return (f"{cfg.name}: {cfg.shape}, {cfg.n_layers} layers x {len(cfg.targets)} targets "
            f"({wl.describe_targets(cfg)}), E={cfg.n_experts}, r={cfg.rank}, "
            f"alpha={cfg.alpha:g}, top-{top_k}, {n_tokens}-token decode switch sequence")


# --------------------------------------------------------------------------
# the reference arm: the oracle, on the host cores

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from weight_merge_b200 import workloads as wl
    cfg = wl.CONFIGS[args.config]
    # each step: a bounded sample (~2 s) of one switch
    times = []
    gbs_all = []
    desc = threads = None
    for k in range(args.warmup + args.steps):
        gbs, threads, desc, dt, elems = oracle_rate(cfg, target_s=2.0)
        if k >= args.warmup:
            times.append(dt)
            gbs_all.append(gbs)
    value = statistics.mean(gbs_all)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1000 * statistics.mean(times), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_label(cfg, cfg.n_tokens),
                   "sample": "each step times a row sample of one layer"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
# our arm

def torch_addmm_baseline(model, cfg, r_np, t_prev, t_cur, stream, reps=5):
    """Median time of one switch done as one torch.addmm_ per weight."""
    import numpy as np
    import torch
    slots = r_np.shape[1] // 2
    coef = {}
    for sign, t in ((-1.0, t_prev), (1.0, t_cur)):
        idx = r_np[t, :slots]
        gate = r_np[t, slots:].copy().view(np.float32)
        for e, g in zip(idx, gate):
            if e >= 0:
                coef[int(e)] = coef.get(int(e), 0.0) + sign * cfg.scale * float(g)
    experts = [e for e, c in coef.items() if c != 0.0]
    if not experts:
        return None
    Bc, Ac = [], []
    for A, B in zip(model.A, model.B):
        Bc.append(torch.cat([B[e] * coef[e] for e in experts], dim=1).contiguous())
        Ac.append(torch.cat([A[e] for e in experts], dim=0).contiguous())
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps + 1)]
    for i, (e0, e1) in enumerate(ev):
        e0.record(stream)
        for W, b, a in zip(model.W, Bc, Ac):
            W.addmm_(b, a)
        e1.record(stream)
    torch.cuda.synchronize()
    ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in ev[1:])
    return {"ms": round(ms, 4), "launches": len(model.W),
            "w_gbs": round(cfg.w_bytes_per_switch() / (ms / 1e3) / 1e9, 1),
            "kind": "torch.addmm_ per weight (cuBLAS bf16 GEMM), coefficient folded into bf16 B; "
                    "context only"}


def layerwise_graph(sw, cfg, routes, r_np, t_from, stream, reps=6):
    """The same switch issued as one launch per layer, the granularity at which
    a decode forward can run layer l while later layers still switch (the
    pages' in-place update pipelined behind the forward pass).  Two CUDA
    graphs, t_from -> x and x -> t_from, are captured once and replayed in
    turn, so W ends on the route it started from.  Context for the cost of
    that granularity against the single launch; the forward itself is not
    part of this library."""
    import numpy as np
    import torch
    from weight_merge_b200 import binding as B

    x = next((t for t in range(routes.shape[0]) if not np.array_equal(r_np[t], r_np[t_from])),
             None)
    if x is None:
        return None
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    graphs = []
    for a, b in ((t_from, x), (x, t_from)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                for layer in range(cfg.n_layers):
                    sw.switch_layers(layer, 1, B.Switcher.route_ptr(routes, a),
                                     B.Switcher.route_ptr(routes, b), side.cuda_stream)
        graphs.append(g)
    stream.wait_stream(side)
    for g in graphs:
        g.replay()
    torch.cuda.synchronize()
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(2 * reps)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(2 * reps)]
    for i in range(2 * reps):
        ev0[i].record(stream)
        graphs[i % 2].replay()
        ev1[i].record(stream)
    torch.cuda.synchronize()
    ms = statistics.median(a.elapsed_time(b) for a, b in zip(ev0, ev1))
    del graphs
    return {"launches_per_switch": cfg.n_layers, "ms": round(ms, 4),
            "hbm_gbs": round(cfg.w_bytes_per_switch() / (ms / 1e3) / 1e9, 1),
            "replays": 2 * reps}


def reduce_over_ranks(total_ms, n_units, world, device="cpu"):
    """Whole-job timing: the slowest rank's device time and the units (real
    switches) all ranks processed.  Every rank takes the same collective
    steps; world == 1 takes none."""
    import torch
    import torch.distributed as dist
    if world <= 1:
        return float(total_ms), float(n_units)
    mx = torch.tensor([float(total_ms)], dtype=torch.float64, device=device)
    sm = torch.tensor([float(n_units)], dtype=torch.float64, device=device)
    dist.all_reduce(mx, op=dist.ReduceOp.MAX)
    dist.all_reduce(sm, op=dist.ReduceOp.SUM)
    return float(mx[0]), float(sm[0])


def moving_steps(r_np, seq, prev_t, rebase=False):
    """For each token t of ``seq`` (the first switch goes prev_t -> seq[0],
    then token to token): True when that switch moves W.  An in-place switch
    between bitwise-equal routes is the identity and moves no W bytes; a
    re-base always writes W.  ``r_np`` must hold the routes the loop used."""
    import numpy as np
    out = []
    p = prev_t
    for t in seq:
        out.append(bool(rebase or p is None or not np.array_equal(r_np[p], r_np[t])))
        p = t
    return out


def e2e_leg(seq, prev_t, run_step, start, stop, read_routes, rebase=False):
    """The end-to-end loop: ``run_step(prev, t)`` issues one step (host->device
    copy of the token's input, pre-gate, switch, device->host copy of its
    route); ``start`` / ``stop`` bracket the loop on the device (``stop``
    synchronises and returns ms).  The routes are read back AFTER the loop, so
    the count of W-moving switches describes the routes this loop computed.
    Returns (ms, moving flags, the token W carries afterwards)."""
    start()
    pe = prev_t
    for t in seq:
        run_step(pe, t)
        pe = t
    ms = stop()
    return ms, moving_steps(read_routes(), seq, prev_t, rebase), pe


def effective_schedule(requested, kind):
    """The tile schedule a launch of kernel `kind` uses under the context's
    setting (ADAFUSE_SCHEDULE_AUTO: dynamic for the single-CTA tensor-core
    kernel, static for the pair kernel; the other kernels are static)."""
    if kind == 2:                      # ADAFUSE_KERNEL_TCGEN05
        return "static" if requested == "static" else "dynamic"
    if kind == 3:                      # ADAFUSE_KERNEL_TCGEN05_PAIR
        return "dynamic" if requested == "dynamic" else "static"
    return "static"


# adafuse_get_tensor_map_layout values (ADAFUSE_MAPS_NONE, _PLAIN, _BLOCKED)
MAP_LAYOUTS = {0: "none", 1: "plain", 2: "blocked"}
KERNEL_NAMES = {1: "switch_mma_kernel", 2: "switch_tc_kernel", 3: "switch_tc2_kernel",
                4: "switch_fold_kernel"}


def route_buffer(cfg, T, topk, device):
    """Route records of a workload whose switch sequence is synthesised
    (``share_one`` / ``zipf``), or None when the router makes them."""
    import numpy as np
    import torch
    from weight_merge_b200 import workloads as wl
    if cfg.route_mode == "router":
        return None
    idx, gate = wl.synth_routes(cfg, T=T)
    width = 8 if topk else 4
    buf = np.zeros((T, width), dtype=np.int32)
    half = width // 2
    if topk:
        buf[:, :half] = -1
    buf[:, :2] = idx
    g = np.zeros((T, half), dtype=np.float32)
    g[:, :2] = gate
    buf[:, half:] = g.view(np.int32)
    return torch.from_numpy(buf).to(device)


def percentile(xs, q):
    s = sorted(xs)
    return s[min(len(s) - 1, int(q * len(s)))]


def config_leg(name, args, dev, stream, peak, peak_kind):
    """One more workload of the set, switch latency only: the model is built,
    its route sequence made (router over its hidden states, or synthesised),
    then 3 warm-up and ``args.config_steps`` timed switches, with CUDA events
    around each launch on the launching stream.  Identity switches (prev ==
    cur bitwise) are timed apart and kept out of the roofline."""
    import numpy as np
    import torch
    from weight_merge_b200 import binding as B
    from weight_merge_b200 import workloads as wl

    cfg = wl.CONFIGS[name]
    sh = stream.cuda_stream
    model = wl.make_model(cfg, device="cuda")
    sw = B.Switcher(model.W, model.A, model.B, cfg.n_layers, len(cfg.targets), cfg.n_experts,
                    cfg.rank, cfg.alpha, device=dev, names=[t.name for t in cfg.targets])
    try:
        kind = sw.kernel
        maps = MAP_LAYOUTS[sw.map_layout]
        T = cfg.n_tokens
        routes = route_buffer(cfg, T, False, "cuda")
        if routes is None:
            h = wl.make_hidden(cfg, T=T, device="cuda")
            routes = torch.zeros((T, 4), dtype=torch.int32, device="cuda")
            sw.pregate(h, model.Wr, routes, sh)     # a token's route does not depend on its batch
            del h
        torch.cuda.synchronize()
        r_np = routes.cpu().numpy()
        warm, n = 3, max(10, args.config_steps)
        # where the sequence repeats a token (an identity switch, timed
        # apart), the timed window is placed so that it holds the first one
        rep = next((t for t in range(1, T) if np.array_equal(r_np[t], r_np[t - 1])), None)
        start = 0 if rep is None else max(0, rep - warm - n // 2)
        seq = [(start + k) % T for k in range(warm + n)]
        flags = moving_steps(r_np, seq, None)
        ptr = B.Switcher.route_ptr
        for k in range(warm):
            sw.switch(ptr(routes, None if k == 0 else seq[k - 1]), ptr(routes, seq[k]), sh)
        torch.cuda.synchronize()
        assert sw.status(sh) == 0
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n)]
        with ClockSampler(dev) as clk:
            torch.cuda.synchronize()
            clk.mark_start()
            for k in range(n):
                i = warm + k
                ev[k][0].record(stream)
                sw.switch(ptr(routes, seq[i - 1]), ptr(routes, seq[i]), sh)
                ev[k][1].record(stream)
            torch.cuda.synchronize()
            clk.mark_end()
        assert sw.status(sh) == 0
        ms = [a.elapsed_time(b) for a, b in ev]
        real = [x for x, f in zip(ms, flags[warm:]) if f]
        ident = [x for x, f in zip(ms, flags[warm:]) if not f]
        w_bytes = cfg.w_bytes_per_switch()
        achieved = w_bytes / (sum(real) / len(real) / 1e3) / 1e9
        kname = KERNEL_NAMES[kind]
        cpu = None
        if not args.no_cpu_baseline:
            gbs, threads, desc, _dt, _el = oracle_rate(cfg, target_s=3.0)
            cpu = {"value": round(gbs, 5), "unit": "GB/s", "cores": threads, "kind": "oracle",
                   "sample": desc}
        return {
            "workload": workload_label(cfg, T),
            "route_source": "router" if cfg.route_mode == "router" else f"synthesised ({cfg.route_mode})",
            "tensor_maps": maps,
            "tile_schedule": effective_schedule("auto", kind),
            "w_bytes_per_switch": w_bytes,
            "timed_switches": n,
            "switch_ms_p50": round(percentile(real, 0.5), 4),
            "switch_ms_p90": round(percentile(real, 0.9), 4),
            "switches_per_s": round(n / (sum(ms) / 1e3), 3),
            "identity_steps": len(ident),
            "identity_switch_ms_p50": round(percentile(ident, 0.5), 5) if ident else None,
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "peak_kind": peak_kind, "traffic": profiled_traffic(kname, cfg.name),
                         "kernel": kname},
            "cpu_baseline": cpu,
            "clocks": clk.summary(),
        }
    finally:
        sw.close()
        del sw, model
        torch.cuda.synchronize()
        torch.cuda.empty_cache()


def layerwise_dynamic(sw, model, cfg, stream, reps=6):
    """Layer-wise dynamic routing built from this library's own kernels, the
    pattern the pages measure AdaFuse against: every layer makes its own
    routing decision (one pre-gate launch per layer, here over a per-layer
    stand-in hidden state) and switches its own adapters (one layer-range
    switch launch per layer, not captured in a graph): 2L launches per token
    against one pre-gate and one fused switch.  Context only; it leaves W on
    other routes than the headline sequence, so it runs after it."""
    import torch
    from weight_merge_b200 import binding as B
    L = cfg.n_layers
    T = reps + 2
    g = torch.Generator(device="cuda").manual_seed(cfg.seed() + 31)
    hl = torch.empty((L, T, cfg.d), dtype=torch.float32, device="cuda").normal_(0.0, 1.0, generator=g)
    rl = torch.zeros((L, T, 4), dtype=torch.int32, device="cuda")
    sh = stream.cuda_stream
    ptr = B.Switcher.route_ptr

    def step(t):
        for layer in range(L):
            sw.pregate(hl[layer, t:t + 1], model.Wr, rl[layer, t:t + 1], sh)
            sw.switch_layers(layer, 1, ptr(rl[layer], t - 1) if t > 0 else None,
                             ptr(rl[layer], t), sh)
    step(0)
    step(1)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    for i in range(reps):
        ev[i][0].record(stream)
        step(2 + i)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    assert sw.status(sh) == 0
    ms = statistics.median(a.elapsed_time(b) for a, b in ev)
    del hl, rl
    return {"launches_per_step": 2 * L, "ms_per_step": round(ms, 4), "steps": reps,
            "kind": "per-layer pre-gate + per-layer switch launch (this library's kernels, "
                    "no graph); context only"}


def pipelined_forward(sw, model, cfg, routes, t_a, t_b, stream, reps=6, caps=(0, 128, 112)):
    """The switch pipelined against a decode forward, layer by layer: a side
    stream switches layer l (one layer-range launch) and records an event;
    the main stream waits for it and runs layer l's forward while the side
    stream switches layer l+1.  The forward here is a stand-in for the
    caller's decoder (one torch GEMV per targeted weight of the layer, bf16,
    cuBLAS), not part of this library.  Timed against the serial order (one
    full switch launch, then the whole forward) and the forward alone.  Each
    repetition switches t_a -> t_b or back, so W ends where it started."""
    import torch
    from weight_merge_b200 import binding as B
    L, nt = cfg.n_layers, len(cfg.targets)
    g = torch.Generator(device="cuda").manual_seed(cfg.seed() + 53)
    xs = [torch.empty(t.inn, dtype=torch.float32, device="cuda").normal_(0.0, 1.0, generator=g)
          .to(torch.bfloat16) for t in cfg.targets]
    ys = [torch.empty(t.out, dtype=torch.bfloat16, device="cuda") for t in cfg.targets]
    side = torch.cuda.Stream()
    ptr = B.Switcher.route_ptr
    pair = [(t_a, t_b), (t_b, t_a)]
    lev = [torch.cuda.Event() for _ in range(L)]

    def forward_layer(layer):
        for k in range(nt):
            torch.mv(model.W[layer * nt + k], xs[k], out=ys[k])

    def serial(i):
        a, b = pair[i % 2]
        sw.switch(ptr(routes, a), ptr(routes, b), stream.cuda_stream)
        for layer in range(L):
            forward_layer(layer)

    def forward_only(i):
        for layer in range(L):
            forward_layer(layer)

    def pipelined(i):
        a, b = pair[i % 2]
        side.wait_stream(stream)           # the previous forward is done with W
        for layer in range(L):
            sw.switch_layers(layer, 1, ptr(routes, a), ptr(routes, b), side.cuda_stream)
            lev[layer].record(side)
        for layer in range(L):
            stream.wait_event(lev[layer])
            forward_layer(layer)

    def timed(fn):
        fn(0)
        fn(1)
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(reps)]
        for i in range(reps):
            ev[i][0].record(stream)
            fn(i)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in ev)

    out = {}
    with torch.cuda.stream(stream):
        out["serial"] = timed(serial)
        out["forward_only"] = timed(forward_only)
        # the pipelined schedule with the switch's grid capped, so that the
        # forward's kernels find free SMs beside it (0 = no cap)
        for cap in caps:
            sw.set_max_ctas(cap)
            out[f"pipelined_cap{cap}"] = timed(pipelined)
        sw.set_max_ctas(0)
    assert sw.status(stream.cuda_stream) == 0
    best_cap = min(caps, key=lambda c: out[f"pipelined_cap{c}"])
    best = out[f"pipelined_cap{best_cap}"]
    hidden = (out["serial"] - best) / out["forward_only"] if out["forward_only"] else None
    return {"serial_ms": round(out["serial"], 4),
            "pipelined_ms": {str(c): round(out[f"pipelined_cap{c}"], 4) for c in caps},
            "best_switch_ctas": best_cap or None,
            "forward_only_ms": round(out["forward_only"], 4),
            "speedup": round(out["serial"] / best, 4),
            "forward_hidden_frac": round(hidden, 4) if hidden is not None else None,
            "switch_launches": L, "forward_gemvs": L * nt, "reps": reps,
            "kind": "side-stream layer-range switches ordered by events against a stand-in "
                    "GEMV forward (torch, the caller's code), switch grid capped at the given "
                    "CTA counts (0 = every SM); context only"}


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    from weight_merge_b200 import binding as B
    from weight_merge_b200 import workloads as wl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.cuda.current_device()

    cfg = wl.CONFIGS[args.config]
    if args.layers:
        cfg = wl.scaled(cfg, n_layers=args.layers)
    model = wl.make_model(cfg, device="cuda")
    sw = B.Switcher(model.W, model.A, model.B, cfg.n_layers, len(cfg.targets), cfg.n_experts,
                    cfg.rank, cfg.alpha, device=dev, names=[t.name for t in cfg.targets])
    sw.set_kernel({"auto": B.ADAFUSE_KERNEL_AUTO, "mma": B.ADAFUSE_KERNEL_MMA_SYNC,
                   "tc": B.ADAFUSE_KERNEL_TCGEN05, "tc2": B.ADAFUSE_KERNEL_TCGEN05_PAIR,
                   "fold": B.ADAFUSE_KERNEL_TCGEN05_FOLD}[args.kernel])
    sw.set_schedule({"auto": B.ADAFUSE_SCHEDULE_AUTO, "dynamic": B.ADAFUSE_SCHEDULE_DYNAMIC,
                     "static": B.ADAFUSE_SCHEDULE_STATIC}[args.schedule])
    # the kernel this run's switches launch (in-place top-k calls have their own choice)
    kind = sw.topk_kernel if (args.top_k != 2 and args.mode != "rebase") else sw.kernel
    maps = MAP_LAYOUTS[sw.map_layout]
    kernel_name = KERNEL_NAMES[kind]
    # the folded kernel's switch is two launches (fold, then switch); the
    # events around a switch cover both
    launches_per_switch = 2 if kind == B.ADAFUSE_KERNEL_TCGEN05_FOLD else 1
    rebase = args.mode == "rebase"
    if rebase:
        sw.set_base([w.clone() for w in model.W])
    T = cfg.n_tokens
    h = wl.make_hidden(cfg, T=T, device="cuda")
    topk = args.top_k != 2
    width = 8 if topk else 4
    # routes: the router's output for router-driven workloads; otherwise the
    # workload's synthesised sequence (the router still runs every step, into
    # its own buffer, so the step costs what a decode step costs)
    synth = route_buffer(cfg, T, topk, "cuda")
    gated = torch.zeros((T, width), dtype=torch.int32, device="cuda")
    routes = gated if synth is None else synth
    rptr = B.Switcher.route4_ptr if topk else B.Switcher.route_ptr

    def pregate(hh, r_rows):
        if topk:
            sw.pregate_topk(hh, model.Wr, args.top_k, r_rows, sh)
        else:
            sw.pregate(hh, model.Wr, r_rows, sh)
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream
    w_bytes = cfg.w_bytes_per_switch()

    def barrier():
        if world > 1:
            dist.barrier()

    def do_switch(prev_t, t):
        if rebase:
            (sw.rebase_topk if topk else sw.rebase)(rptr(routes, t), sh)
        else:
            (sw.switch_topk if topk else sw.switch)(rptr(routes, prev_t), rptr(routes, t), sh)

    def step(k, prev_t):
        t = k % T
        pregate(h[t:t + 1], gated[t:t + 1])
        do_switch(prev_t, t)
        return t

    # warm-up
    prev_t = None
    for k in range(args.warmup):
        prev_t = step(k, prev_t)
    torch.cuda.synchronize()
    assert sw.status(sh) == 0
    first_prev = prev_t

    # timed region: K steps, events around every switch launch for the roofline
    n_ev = args.steps
    sw_start = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    sw_end = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    st_start = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    seq = [(args.warmup + k) % T for k in range(args.steps)]
    with ClockSampler(dev) as clk:
        barrier()
        torch.cuda.synchronize()
        clk.mark_start()
        t_begin.record(stream)
        for k, t in enumerate(seq):
            st_start[k].record(stream)
            pregate(h[t:t + 1], gated[t:t + 1])
            sw_start[k].record(stream)
            do_switch(prev_t, t)
            sw_end[k].record(stream)
            prev_t = t
        t_end.record(stream)
        torch.cuda.synchronize()
        clk.mark_end()
        barrier()
    clocks = clk.summary()
    assert sw.status(sh) == 0
    total_ms = t_begin.elapsed_time(t_end)
    sw_ms = [a.elapsed_time(b) for a, b in zip(sw_start, sw_end)]
    step_ms = [st_start[k].elapsed_time(st_start[k + 1]) for k in range(n_ev - 1)]
    step_ms.append(st_start[-1].elapsed_time(t_end))

    # identity steps (prev == cur bit-identical) move no W bytes; the routes
    # are read after the loop that computed them
    r_np = routes.cpu().numpy()
    real = moving_steps(r_np, seq, first_prev, rebase)
    n_real = sum(real)
    # the roofline averages the switches that move W; identity switches are
    # reported on their own
    sw_real = [x for x, rl in zip(sw_ms, real) if rl] or sw_ms
    sw_ident = [x for x, rl in zip(sw_ms, real) if not rl]

    max_ms, all_real = reduce_over_ranks(total_ms, n_real, world, device="cuda")
    value = all_real * w_bytes / (max_ms / 1000.0) / 1e9

    # e2e through the public API with host buffers: each step copies the
    # token's hidden state from pinned host memory, pre-gates, switches and
    # copies the token's route record back
    e2e = None
    last_t = prev_t                  # the route W currently carries
    if not args.no_e2e:
        h_host = h.cpu().pin_memory()
        r_host = torch.zeros((1, width), dtype=torch.int32).pin_memory()
        h_dev = torch.empty((1, cfg.d), dtype=torch.float32, device="cuda")
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)

        def run_step(pe, t):
            h_dev.copy_(h_host[t:t + 1], non_blocking=True)
            pregate(h_dev, gated[t:t + 1])
            do_switch(pe, t)
            r_host.copy_(routes[t:t + 1], non_blocking=True)

        def start():
            barrier()
            torch.cuda.synchronize()
            ev0.record(stream)

        def stop():
            ev1.record(stream)
            torch.cuda.synchronize()
            barrier()
            return ev0.elapsed_time(ev1)

        e_seq = [(args.warmup + args.steps + k) % T for k in range(args.steps)]
        e_ms, e_flags, last_t = e2e_leg(e_seq, prev_t, run_step, start, stop,
                                        lambda: routes.cpu().numpy(), rebase)
        assert sw.status(sh) == 0
        e_max, e_units = reduce_over_ranks(e_ms, sum(e_flags), world, device="cuda")
        e2e = {"value": round(e_units * w_bytes / (e_max / 1000) / 1e9, 2),
               "unit": "GB/s", "h2d_bytes_per_step": cfg.d * 4,
               "d2h_bytes_per_step": 4 * width, "moving_switches": int(sum(e_flags)),
               "steps": args.steps, "ms_per_step": round(e_max / args.steps, 4)}
        r_np = routes.cpu().numpy()

    # the router alone on a batch of tokens (the Llama-3-8B-shaped router
    # batch: T=4096, d=4096, E=8): an HBM-bound GEMV over h
    router = None
    if args.router_tokens > 0 and rank == 0:
        Tr = args.router_tokens
        hr = torch.empty((Tr, cfg.d), dtype=torch.float32, device="cuda")
        hr.normal_(0.0, 1.0, generator=torch.Generator(device="cuda").manual_seed(cfg.seed() + 17))
        rr = torch.zeros((Tr, 4), dtype=torch.int32, device="cuda")
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")  # > L2 (126 MB)
        for _ in range(3):
            sw.pregate(hr, model.Wr, rr, sh)
        ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(10)]
        ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(10)]
        for i in range(10):
            flush.zero_()                      # evict h from L2 between timed launches
            ev0[i].record(stream)
            sw.pregate(hr, model.Wr, rr, sh)
            ev1[i].record(stream)
        torch.cuda.synchronize()
        rms = [a.elapsed_time(b) for a, b in zip(ev0, ev1)]
        r_ms = statistics.median(rms)
        # one decode token: the launch a decode step makes
        h1 = hr[:1].contiguous()
        d0 = [torch.cuda.Event(enable_timing=True) for _ in range(20)]
        d1 = [torch.cuda.Event(enable_timing=True) for _ in range(20)]
        for i in range(20):
            d0[i].record(stream)
            sw.pregate(h1, model.Wr, rr[:1], sh)
            d1[i].record(stream)
        torch.cuda.synchronize()
        dec_ms = statistics.median(a.elapsed_time(b) for a, b in zip(d0, d1))
        del flush
        r_bytes = Tr * cfg.d * 4 + cfg.d * cfg.n_experts * 4 + Tr * 16
        router = {"tokens": Tr, "d": cfg.d, "experts": cfg.n_experts,
                  "ms_p50": round(r_ms, 5), "tokens_per_s": round(Tr / (r_ms / 1e3)),
                  "hbm_gbs": round(r_bytes / (r_ms / 1e3) / 1e9, 1),
                  "frac_of_peak": round(r_bytes / (r_ms / 1e3) / 1e9 / measured_peaks()[0], 4),
                  "decode_token_ms_p50": round(dec_ms, 5),
                  "kernel": "pregate_group_kernel" if (cfg.n_experts <= 8 and cfg.d <= 4096)
                            else "pregate_kernel",
                  "traffic": profiled_traffic("pregate_group_kernel", f"router-{Tr}x{cfg.d}-E{cfg.n_experts}"),
                  "l2": "flushed (256 MB write) before each timed batch launch"}
        del hr, rr

    # context figures (never the product path), each after the headline
    # sequence because they move W off it
    solo = rank == 0 and world == 1
    layerwise = None
    if solo and not args.no_layerwise and not rebase and not topk:
        layerwise = layerwise_graph(sw, cfg, routes, r_np, last_t if last_t is not None else 0,
                                    stream)
        if layerwise is not None:
            layerwise["launches_per_switch"] *= launches_per_switch
            layerwise["vs_single_launch"] = round(
                statistics.mean(sw_real) / layerwise["ms"], 4)
        assert sw.status(sh) == 0

    pipelined = None
    if solo and not args.no_pipelined and not rebase and not topk and last_t is not None:
        other = next((t for t in range(T) if not np.array_equal(r_np[t], r_np[last_t])), None)
        if other is not None:
            pipelined = pipelined_forward(sw, model, cfg, routes, last_t, other, stream)

    per_layer_routing = None
    if solo and not args.no_layerwise and not rebase and not topk:
        per_layer_routing = layerwise_dynamic(sw, model, cfg, stream)
        fused = statistics.median(step_ms)
        per_layer_routing["fused_step_ms_p50"] = round(fused, 4)
        per_layer_routing["vs_fused_step"] = round(per_layer_routing["ms_per_step"] / fused, 4)

    torch_base = None
    if solo and not args.no_torch_baseline and not rebase and T > 1:
        torch_base = torch_addmm_baseline(model, cfg, r_np, 0, 1, stream)

    peak, peak_kind = measured_peaks()
    sw_avg = statistics.mean(sw_real)
    achieved = w_bytes / (sw_avg / 1000.0) / 1e9
    cpu = None
    if solo and not args.no_cpu_baseline:
        gbs, threads, desc, dt, elems = oracle_rate(cfg, target_s=10.0)
        cpu = {"value": round(gbs, 5), "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": desc}
    copy_gbs = same_gpu_copy_gbs() if rank == 0 else None

    line = None
    if rank == 0:
        sw_sorted = sorted(sw_real)
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(max_ms / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded random weights and hidden states)",
            "config": {
                "workload": workload_label(cfg, T, args.top_k),
                "w_bytes_per_switch": w_bytes,
                "l2": "inputs larger than L2 (W read+write per switch >> 126 MB), no flush",
                "parallelism": f"replicas x{world}",
                "mode": args.mode,
                "route_source": "router" if synth is None else f"synthesised ({cfg.route_mode})",
                "tile_schedule": effective_schedule(args.schedule, kind),
                "tensor_maps": maps,
            },
            "switch_ms_p50": round(sw_sorted[len(sw_sorted) // 2], 4),
            "switch_ms_p90": round(sw_sorted[min(len(sw_sorted) - 1, int(0.9 * len(sw_sorted)))], 4),
            "step_ms_p50": round(sorted(step_ms)[len(step_ms) // 2], 4),
            "switches_per_s": round(world * args.steps / (max_ms / 1000.0), 3),
            "identity_steps": args.steps - n_real,
            "identity_switch_ms_p50": (round(sorted(sw_ident)[len(sw_ident) // 2], 5)
                                       if sw_ident else None),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "peak_kind": peak_kind,
                         "traffic": profiled_traffic(kernel_name, cfg.name),
                         "kernel": kernel_name,
                         "copy_gbs_this_gpu": round(copy_gbs, 1),
                         "frac_of_this_gpu_copy": round(achieved / copy_gbs, 4)},
            "cpu_baseline": cpu,
            "torch_addmm_baseline": torch_base,
            "layerwise_graph": layerwise,
            "per_layer_routing": per_layer_routing,
            "pipelined": pipelined,
            "e2e": e2e,
            "gpu_launches": (1 + launches_per_switch) * args.steps,
            "router": router,
            "clocks": clocks,
        }
    sw.close()
    del sw, model, h, routes, gated, synth
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    # the other workloads of the set, one at a time (replicas run only the
    # headline workload)
    if solo and args.configs:
        extra = {}
        for name in [c for c in args.configs.split(",") if c and c != args.config]:
            extra[name] = config_leg(name, args, dev, stream, peak, peak_kind)
        line["configs"] = extra
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
