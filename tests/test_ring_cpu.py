"""Ring attention host logic on the CPU: the per-rank schedule, and the shard exchange
run for real over torch.distributed (gloo, world sizes 2 and 3): at every step each
rank must hold the key/value shard its schedule names."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_attention_155_b200.ring import CAUSAL, FULL, SKIP, ring_pass, ring_schedule


@pytest.mark.parametrize("world", [1, 2, 3, 5])
@pytest.mark.parametrize("causal", [False, True])
def test_schedule_visits_every_shard_once(world, causal):
    for rank in range(world):
        sched = ring_schedule(rank, world, causal)
        assert [s for s, _, _ in sched] == list(range(world))
        assert sorted(src for _, src, _ in sched) == list(range(world))
        assert sched[0][1] == rank  # own shard first, nothing to receive yet
        for _, src, mode in sched:
            if not causal:
                assert mode == FULL
            else:
                assert mode == (CAUSAL if src == rank else FULL if src < rank else SKIP)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        buf = torch.full((2, 3, 4), float(rank))
        nxt = torch.empty_like(buf)
        seen = []
        for s, src, _ in ring_schedule(rank, world, causal=False):
            seen.append(int(buf[0, 0, 0].item()))
            assert torch.all(buf == float(src))
            if s + 1 < world:
                for r in ring_pass(buf, nxt, rank, world):
                    r.wait()
                buf, nxt = nxt, buf
        q.put((rank, seen))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ring_exchange_delivers_scheduled_shards(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(world))
    for rank in range(world):
        assert got[rank] == [src for _, src, _ in ring_schedule(rank, world, False)]
