"""Host-side logic of the multi-GPU benchmark path, on CPU with gloo (world size 2).

The attention work units are independent, so ranks share no data; the only
cross-rank steps are the barriers around the timed region and the max-over-
ranks reduction of the timings.  These run here with two gloo ranks.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms_local = 2.0 + 3.0 * rank  # rank 1 is the slow one
        slowest = bench.max_over_ranks(ms_local, world, device="cpu")
        per_s, ms = bench.weak_scaling_value(1e9, ms_local, world, device="cpu")
        bench.barrier(world)
        q.put((rank, slowest, per_s, ms))
    finally:
        dist.destroy_process_group()


def test_weak_scaling_aggregation_two_gloo_ranks():
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
    for rank, slowest, per_s, ms in res:
        assert slowest == 5.0 and ms == 5.0
        # both ranks did 1e9 units; the job took the slowest rank's 5 ms
        assert per_s == pytest.approx(2 * 1e9 / 5e-3)


def test_weak_scaling_single_rank_is_local():
    sys.path.insert(0, ROOT)
    import bench
    per_s, ms = bench.weak_scaling_value(1e9, 4.0, 1)
    assert ms == 4.0 and per_s == pytest.approx(1e9 / 4e-3)


def test_reference_arm_nonzero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
