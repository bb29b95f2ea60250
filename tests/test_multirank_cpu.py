"""The benchmark's multi-rank plumbing on CPU (gloo, world size 2).

The switch has no exchange step, so N GPUs run N independent replicas; the
only collectives are the timing reductions (slowest rank's time, units summed
over ranks) and barriers.  These tests run that host logic on two gloo ranks.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # rank r pretends to have taken (10 + 5r) ms for (3 + r) real switches
        ms, units = bench.reduce_over_ranks(10.0 + 5 * rank, 3 + rank, world, device="cpu")
        dist.barrier()
        q.put((rank, ms, units))
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, units in got:
        assert ms == 15.0          # the slowest rank's time
        assert units == 7.0        # 3 + 4 switches over both ranks


def test_reduce_single_rank_takes_no_collective():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_over_ranks(12.5, 4, 1) == (12.5, 4.0)


def test_reference_arm_non_zero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
