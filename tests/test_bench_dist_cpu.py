"""Multi-rank logic of bench.py on the CPU: two gloo ranks (127.0.0.1).

The benchmark is weak scaling (every rank runs its own independent heads, no
collective on the data path); the only cross-rank operations are a barrier
and the max of the per-rank times, checked here without a GPU."""
import json
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
        bench.dist_barrier(world)
        per_rank_ms = [12.5, 20.0][rank]
        mx = bench.dist_max(per_rank_ms, world)
        val = bench.weak_scaling_value(world, 10, 16384, mx)
        q.put((rank, mx, val))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, mx, val in res:
        assert mx == 20.0                                    # slowest rank
        assert val == pytest.approx(2 * 10 * 16384 / 0.020)  # units of both ranks / max time


def test_single_rank_helpers():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.dist_max(3.0, 1) == 3.0
    assert bench.weak_scaling_value(1, 4, 100, 2000.0) == pytest.approx(200.0)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                         env=env, timeout=120)
    assert res.returncode == 0 and res.stdout.strip() == ""
