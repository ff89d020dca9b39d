"""The N > 1 bookkeeping of bench.py on CPU gloo ranks: every rank runs its own replica
(the path has no exchange step), the job's time is the slowest rank's, and the value is
the work of all ranks over that time. The reference arm prints only on rank 0."""
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


def _rank(rank, world, port, q):
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        bench._barrier(world)
        mine = 10.0 + 7.0 * rank  # this rank's elapsed ms
        slowest = bench._max_over_ranks(mine, world, torch.device("cpu"))
        value = bench.job_throughput(world, 5.0, 4, slowest)
        bench._barrier(world)
        q.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_job_time_is_the_slowest_rank_and_value_counts_every_rank(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(world):
            r, slowest, value = q.get(timeout=120)
            got[r] = (slowest, value)
    finally:
        for p in procs:
            p.join(60)
            if p.is_alive():
                p.terminate()
                p.join(10)
    assert all(p.exitcode == 0 for p in procs)
    slowest = 10.0 + 7.0 * (world - 1)
    for r in range(world):
        assert got[r][0] == slowest
        # 5 units per rank and step, 4 steps, every rank, over the slowest rank's time
        assert got[r][1] == pytest.approx(world * 5.0 * 4 / (slowest * 1e-3))


def test_one_rank_needs_no_process_group():
    import bench
    assert bench._max_over_ranks(12.5, 1, torch.device("cpu")) == 12.5
    bench._barrier(1)
    assert bench.job_throughput(1, 2.0, 10, 500.0) == pytest.approx(40.0)


def test_reference_arm_prints_nothing_on_other_ranks():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
