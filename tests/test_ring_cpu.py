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


def _ring_worker(rank, world, port, causal, q):
    """Runs ring_attention_fwd on CPU tensors over gloo with the per-block compute
    replaced by the float64 oracle (a test seam: the product path calls the CUDA
    library), and returns this rank's rows."""
    import numpy as np

    import oracle
    from exact_attention_155_b200 import ring

    def attend_and_merge(qs, ks, vs, mode, scale, o_acc, lse_acc, out, stream=None):
        if mode == ring.SKIP:
            return
        to64 = lambda t: t.double().numpy()
        o, l = oracle.attention_forward(to64(qs), to64(ks), to64(vs), causal=(mode == ring.CAUSAL),
                                        scale=scale)
        acc_o = o_acc.double().numpy()
        acc_l = lse_acc.double().numpy()
        mo, ml = oracle.merge_partials(np.stack([acc_o, o]),
                                       np.stack([acc_l.transpose(0, 2, 1), l.transpose(0, 2, 1)]))
        o_acc.copy_(torch.from_numpy(mo))
        lse_acc.copy_(torch.from_numpy(ml.transpose(0, 2, 1)))

    ring._attend_and_merge = attend_and_merge
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        g = torch.Generator().manual_seed(123)
        B, S, H, d = 1, 6, 2, 4
        full = [torch.randn((B, S * world, H, d), generator=g) for _ in range(3)]
        qs, ks, vs = (t[:, rank * S:(rank + 1) * S].contiguous() for t in full)
        out, lse = ring.ring_attention_fwd(qs, ks, vs, causal=causal, scale=0.5)
        q.put((rank, out.float().numpy(), lse.numpy(), [t.numpy() for t in full]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_attention_driver_over_gloo(world, causal):
    import numpy as np

    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ring_worker, args=(r, world, port, causal, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    got = {}
    for _ in range(world):
        rank, o, l, full = q.get(timeout=10)
        got[rank] = (o, l)
    ref_o, ref_l = oracle.attention_forward(*[f.astype(np.float64) for f in full], causal=causal,
                                            scale=0.5)
    S = ref_o.shape[1] // world
    for rank in range(world):
        o, l = got[rank]
        # The driver's output is bf16; the LSE stays fp32 from the merges.
        np.testing.assert_allclose(o, ref_o[:, rank * S:(rank + 1) * S], atol=2e-2)
        np.testing.assert_allclose(l, ref_l[:, :, rank * S:(rank + 1) * S], atol=1e-6)
