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


def _oracle_attend_and_merge(qs, ks, vs, mode, scale, o_acc, lse_acc, out, stream=None):
    """Stand-in for ring._attend_and_merge on CPU tensors: the float64 oracle's
    attention and merge (a test seam; the product path calls the CUDA library)."""
    import numpy as np

    import oracle
    from exact_attention_155_b200 import ring
    _SEAM_CALLS.append(("fwd", mode, out is not None))
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
    if out is not None:
        out.copy_(o_acc)


def _oracle_pair_terms(qs, ks, vs, out, dout, lse, mode, scale, bufs, stream=None):
    """Stand-in for ring._pair_terms on CPU tensors: the oracle's terms of one shard
    pair (None for a skipped pair)."""
    import oracle
    from exact_attention_155_b200 import ring
    _SEAM_CALLS.append(("terms", mode, False))
    if mode == ring.SKIP:
        return None
    to64 = lambda t: t.double().numpy()
    g = oracle.attention_backward_from_stats(
        to64(qs), to64(ks), to64(vs), to64(out), to64(dout), to64(lse),
        causal=(mode == ring.CAUSAL), scale=scale)
    return tuple(torch.from_numpy(t) for t in g)


def _oracle_add_terms(terms, dq_acc, dk_acc, dv_acc, dq_out, stream=None):
    """Stand-in for ring._add_terms: adds the terms to the running sums."""
    _SEAM_CALLS.append(("bwd", "skip" if terms is None else "pair", dq_out is not None))
    if terms is None:
        return
    tq, tk, tv = terms
    dq_acc += tq.to(dq_acc.dtype)
    dk_acc += tk.to(dk_acc.dtype)
    dv_acc += tv.to(dv_acc.dtype)
    if dq_out is not None:
        dq_out.copy_(dq_acc)


def _oracle_to_bf16(acc, out, stream=None):
    _SEAM_CALLS.append(("convert", None, True))
    out.copy_(acc)


_SEAM_CALLS = []
# The driver keeps its running sums in fp32 (as on the GPU); the seams compute in fp64.
_ATOL = 1e-5


def _use_oracle_seams(ring):
    ring._attend_and_merge = _oracle_attend_and_merge
    ring._pair_terms = _oracle_pair_terms
    ring._add_terms = _oracle_add_terms
    ring._to_bf16 = _oracle_to_bf16


def _full_inputs(world, S=6, B=1, H=2, d=4, seed=123):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn((B, S * world, H, d), generator=g, dtype=torch.float64) for _ in range(4)]


def _ring_worker(rank, world, port, causal, q):
    """Runs ring_attention_fwd on CPU tensors over gloo with the per-block compute
    replaced by the float64 oracle, and returns this rank's rows."""
    from exact_attention_155_b200 import ring

    _use_oracle_seams(ring)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        full = _full_inputs(world)
        S = full[0].shape[1] // world
        qs, ks, vs = (t[:, rank * S:(rank + 1) * S].contiguous() for t in full[:3])
        out, lse = ring.ring_attention_fwd(qs, ks, vs, causal=causal, scale=0.5)
        q.put((rank, out.numpy(), lse.numpy(), [t.numpy() for t in full], list(_SEAM_CALLS)))
    finally:
        dist.destroy_process_group()


def _check_out_written_once(calls, kind):
    # The bf16 result is written by the last merge (or sum) that is not skipped, once.
    writes = [i for i, c in enumerate(calls) if c[0] == kind and c[2]]
    assert len(writes) == 1
    later = [c for c in calls[writes[0] + 1:] if c[0] == kind]
    assert all(c[1] == "skip" for c in later)


def _spawn(target, world, *args):
    """Runs target(rank, world, port, *args, queue) in `world` spawned processes and
    returns {rank: rest of the tuple the rank put on the queue}. A rank that hangs or
    dies fails the test within a few minutes; the children are always reaped."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, *args, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(world):
            item = q.get(timeout=120)
            got[item[0]] = item[1:]
    finally:
        for p in procs:
            p.join(60 if len(got) == world else 1)
            if p.is_alive():
                p.terminate()
                p.join(10)
    for p in procs:
        assert p.exitcode == 0
    return got


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_attention_driver_over_gloo(world, causal):
    import numpy as np

    import oracle
    got = _spawn(_ring_worker, world, causal)
    full = got[0][2]
    ref_o, ref_l = oracle.attention_forward(*full[:3], causal=causal, scale=0.5)
    S = ref_o.shape[1] // world
    for rank in range(world):
        o, l, _, calls = got[rank]
        _check_out_written_once(calls, "fwd")
        np.testing.assert_allclose(o, ref_o[:, rank * S:(rank + 1) * S], atol=_ATOL)
        np.testing.assert_allclose(l, ref_l[:, :, rank * S:(rank + 1) * S], atol=_ATOL)


def _ring_bwd_worker(rank, world, port, causal, q):
    """Runs ring_attention_bwd on CPU tensors over gloo with the per-pair compute
    replaced by the oracle, from the oracle's whole-sequence forward (what the ring
    forward returns); returns this rank's gradients."""
    import oracle
    from exact_attention_155_b200 import ring

    _use_oracle_seams(ring)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        full = _full_inputs(world, seed=321)
        out, lse = oracle.attention_forward(*[t.numpy() for t in full[:3]], causal=causal,
                                            scale=0.5)
        S = out.shape[1] // world
        rows = lambda t: t[:, rank * S:(rank + 1) * S].contiguous()
        qs, ks, vs, dos = (rows(t) for t in full)
        os_ = rows(torch.from_numpy(out))
        ls = torch.from_numpy(lse[:, :, rank * S:(rank + 1) * S]).contiguous()
        dq, dk, dv = ring.ring_attention_bwd(qs, ks, vs, os_, dos, ls, causal=causal, scale=0.5)
        q.put((rank, [g.numpy() for g in (dq, dk, dv)], [t.numpy() for t in full],
               list(_SEAM_CALLS)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_attention_bwd_driver_over_gloo(world, causal):
    """dQ stays home, the dK/dV sums travel a full turn: each rank ends with the
    whole-sequence gradients of its own shards."""
    import numpy as np

    import oracle
    got = _spawn(_ring_bwd_worker, world, causal)
    full = got[0][1]
    refs = oracle.attention_backward(*full, causal=causal, scale=0.5)
    S = refs[0].shape[1] // world
    for rank in range(world):
        grads, _, calls = got[rank]
        _check_out_written_once(calls, "bwd")
        assert [c for c in calls if c[0] == "convert"] == [("convert", None, True)] * 2
        for g, r in zip(grads, refs):
            np.testing.assert_allclose(g, r[:, rank * S:(rank + 1) * S], atol=_ATOL)


@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_emulated_ring_fwd_and_bwd_on_cpu(world, causal, monkeypatch):
    """The one-process emulation's bookkeeping (shard slicing, the per-shard sums, the
    step that writes each result) with the oracle standing in for the kernels."""
    import numpy as np

    import oracle
    from exact_attention_155_b200 import ring
    monkeypatch.setattr(ring, "_attend_and_merge", _oracle_attend_and_merge)
    monkeypatch.setattr(ring, "_pair_terms", _oracle_pair_terms)
    monkeypatch.setattr(ring, "_add_terms", _oracle_add_terms)
    monkeypatch.setattr(ring, "_to_bf16", _oracle_to_bf16)
    full = _full_inputs(world, seed=99 + world)
    q, k, v, do = full
    out, lse = ring.ring_attention_fwd_emulated(q, k, v, world, causal=causal, scale=0.7)
    ref_o, ref_l = oracle.attention_forward(*[t.numpy() for t in full[:3]], causal=causal, scale=0.7)
    np.testing.assert_allclose(out.numpy(), ref_o, atol=_ATOL)
    np.testing.assert_allclose(lse.numpy(), ref_l, atol=_ATOL)
    grads = ring.ring_attention_bwd_emulated(q, k, v, out, do, lse, world, causal=causal, scale=0.7)
    refs = oracle.attention_backward(*[t.numpy() for t in full], causal=causal, scale=0.7)
    for g, r in zip(grads, refs):
        np.testing.assert_allclose(g.numpy(), r, atol=_ATOL)


def _subgroup_worker(rank, world, port, q):
    """Ranks 1 and 3 of four run the ring (forward, then backward) over a process
    subgroup; ranks 0 and 2 only take part in creating it."""
    from exact_attention_155_b200 import ring

    _use_oracle_seams(ring)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        members = [1, 3]
        grp = dist.new_group(members)
        if rank in members:
            gr = members.index(rank)
            full = _full_inputs(2, seed=555)
            S = full[0].shape[1] // 2
            qs, ks, vs, dos = (t[:, gr * S:(gr + 1) * S].contiguous() for t in full)
            out, lse = ring.ring_attention_fwd(qs, ks, vs, causal=True, scale=0.5, group=grp)
            grads = ring.ring_attention_bwd(qs, ks, vs, out, dos, lse, causal=True, scale=0.5,
                                            group=grp)
            q.put((rank, gr, out.numpy(), lse.numpy(), [g.numpy() for g in grads],
                   [t.numpy() for t in full]))
        else:
            q.put((rank, None, None, None, None, None))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_ring_over_a_process_subgroup():
    """Point-to-point peers are global ranks: a ring over ranks {1, 3} must exchange
    between 1 and 3, not between group ranks 0 and 1."""
    import numpy as np

    import oracle
    got = _spawn(_subgroup_worker, 4)
    full = got[1][4]
    ref_o, ref_l = oracle.attention_forward(*full[:3], causal=True, scale=0.5)
    refs = oracle.attention_backward(*full, causal=True, scale=0.5)
    S = ref_o.shape[1] // 2
    for rank in (1, 3):
        gr, o, l, grads, _ = got[rank]
        rows = slice(gr * S, (gr + 1) * S)
        np.testing.assert_allclose(o, ref_o[:, rows], atol=_ATOL)
        np.testing.assert_allclose(l, ref_l[:, :, rows], atol=_ATOL)
        for g, r in zip(grads, refs):
            np.testing.assert_allclose(g, r[:, rows], atol=_ATOL)


class _AbiStandIns:
    """CPU stand-ins for the binding calls the ring driver makes (fwd_ex,
    merge_partials, bwd_ex, bwd_workspace_size, accumulate), each following its C ABI
    contract (outputs written into the buffers passed in) with the oracle's arithmetic,
    so the driver's own buffer handling runs unchanged."""

    def __init__(self):
        self.calls = []

    def fwd_ex(self, q, k, v, causal=False, scale=None, stream=None, **kw):
        import oracle
        self.calls.append("fwd_ex")
        o, l = oracle.attention_forward(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                        causal=causal, scale=scale)
        return torch.from_numpy(o).to(q.dtype), torch.from_numpy(l).float()

    def merge_partials(self, o_acc, lse_acc, o_part, lse_part, out=None, stream=None):
        import numpy as np

        import oracle
        self.calls.append("merge_partials")
        mo, ml = oracle.merge_partials(
            np.stack([o_acc.double().numpy(), o_part.double().numpy()]),
            np.stack([lse_acc.double().numpy().transpose(0, 2, 1),
                      lse_part.double().numpy().transpose(0, 2, 1)]))
        o_acc.copy_(torch.from_numpy(mo))
        lse_acc.copy_(torch.from_numpy(ml.transpose(0, 2, 1)))
        if out is not None:
            out.copy_(o_acc)
        return o_acc, lse_acc

    def bwd_workspace_size(self, B, H, N, d):
        return 256

    def bwd_ex(self, q, k, v, out, dout, lse, causal=False, scale=None, dq=None, dk=None, dv=None,
               workspace=None, stream=None, **kw):
        import oracle
        self.calls.append("bwd_ex")
        assert dq is not None and dk is not None and dv is not None and workspace is not None
        g = oracle.attention_backward_from_stats(*(t.double().numpy() for t in (q, k, v, out, dout, lse)),
                                                 causal=causal, scale=scale)
        for dst, src in zip((dq, dk, dv), g):
            dst.copy_(torch.from_numpy(src))
        return dq, dk, dv

    def accumulate(self, acc, part=None, out=None, stream=None):
        self.calls.append("accumulate")
        assert part is not None or out is not None
        if part is not None:
            assert part.shape == acc.shape
            acc += part.to(acc.dtype)
        if out is not None:
            assert out.shape == acc.shape
            out.copy_(acc)
        return acc


@pytest.mark.parametrize("world", [1, 2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_emulated_ring_through_the_binding_calls(world, causal, monkeypatch):
    """The ring driver's real per-step code (_attend_and_merge, _pair_terms, _add_terms,
    _to_bf16)
    against CPU stand-ins of the binding calls it makes: every result buffer is written
    through those calls and the sums match the oracle over the whole sequence."""
    import numpy as np

    import oracle
    from exact_attention_155_b200 import ring
    fake = _AbiStandIns()
    for name in ("fwd_ex", "merge_partials", "bwd_ex", "bwd_workspace_size", "accumulate"):
        monkeypatch.setattr(ring.ops, name, getattr(fake, name))
    full = _full_inputs(world, seed=700 + world)
    q, k, v, do = full
    out, lse = ring.ring_attention_fwd_emulated(q, k, v, world, causal=causal, scale=0.6)
    ref_o, ref_l = oracle.attention_forward(*[t.numpy() for t in full[:3]], causal=causal, scale=0.6)
    np.testing.assert_allclose(out.numpy(), ref_o, atol=_ATOL)
    np.testing.assert_allclose(lse.numpy(), ref_l, atol=_ATOL)
    grads = ring.ring_attention_bwd_emulated(q, k, v, out, do, lse, world, causal=causal, scale=0.6)
    refs = oracle.attention_backward(*[t.numpy() for t in full], causal=causal, scale=0.6)
    for g, r in zip(grads, refs):
        np.testing.assert_allclose(g.numpy(), r, atol=_ATOL)
    pairs = world * world if not causal else world * (world + 1) // 2
    assert fake.calls.count("bwd_ex") == pairs
    # three sums per visited pair, plus one bf16 copy each of dK and dV per shard
    assert fake.calls.count("accumulate") == 3 * pairs + 2 * world


def _autograd_worker(rank, world, port, q):
    """ring_flash_attn_func forward and autograd backward over gloo with the oracle
    standing in for the kernels; returns this rank's output and input gradients."""
    from exact_attention_155_b200 import ring

    _use_oracle_seams(ring)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        full = _full_inputs(world, seed=808)
        S = full[0].shape[1] // world
        qs, ks, vs, dos = (t[:, rank * S:(rank + 1) * S].contiguous() for t in full)
        for t in (qs, ks, vs):
            t.requires_grad_()
        out = ring.ring_flash_attn_func(qs, ks, vs, causal=True, softmax_scale=0.5)
        out.backward(dos)
        q.put((rank, out.detach().numpy(), [t.grad.numpy() for t in (qs, ks, vs)],
               [t.numpy() for t in full]))
    finally:
        dist.destroy_process_group()


def test_ring_flash_attn_func_autograd_over_gloo():
    import numpy as np

    import oracle
    world = 2
    got = _spawn(_autograd_worker, world)
    full = got[0][2]
    ref_o, _ = oracle.attention_forward(*full[:3], causal=True, scale=0.5)
    refs = oracle.attention_backward(*full, causal=True, scale=0.5)
    S = ref_o.shape[1] // world
    for rank in range(world):
        o, grads, _ = got[rank]
        rows = slice(rank * S, (rank + 1) * S)
        np.testing.assert_allclose(o, ref_o[:, rows], atol=_ATOL)
        for g, r in zip(grads, refs):
            np.testing.assert_allclose(g, r[:, rows], atol=_ATOL)


# ----------------------------------------------------------------- zigzag layout
@pytest.mark.parametrize("world", [1, 2, 3, 4, 5])
@pytest.mark.parametrize("causal", [False, True])
def test_zigzag_plan_covers_every_visible_chunk_pair_once_with_equal_work(world, causal):
    """Brute force over the 2R chunks: the plans of all (rank, step) name each chunk
    pair a query chunk sees exactly once (causal on its own chunk), and every rank does
    the same work at every step (a causal chunk pair counts half)."""
    from exact_attention_155_b200.ring import zigzag_plan
    chunk = lambda r, half: r if half == 0 else 2 * world - 1 - r
    seen = {}
    for rank in range(world):
        for s, src, _ in ring_schedule(rank, world, False):
            work = 0.0
            for a, b, mode in zigzag_plan(rank, src, causal):
                qc, kc = chunk(rank, a), chunk(src, b)
                assert (qc, kc) not in seen
                seen[(qc, kc)] = mode
                work += 0.5 if mode == CAUSAL else 1.0
            assert work == (2.0 if causal else 4.0)
    want = {(qc, kc): (CAUSAL if qc == kc else FULL) for qc in range(2 * world)
            for kc in range(2 * world) if not causal or kc <= qc}
    if not causal:
        want = {key: FULL for key in want}
    assert seen == want


@pytest.mark.parametrize("world", [1, 2, 3])
def test_zigzag_shard_and_unshard_round_trip(world):
    from exact_attention_155_b200.ring import zigzag_shard, zigzag_unshard
    x = torch.arange(2 * 4 * world * 3, dtype=torch.float32).reshape(2, 4 * world, 3)
    shards = [zigzag_shard(x, r, world) for r in range(world)]
    c = 2
    assert torch.equal(shards[0][:, :c], x[:, :c])                      # chunk 0
    assert torch.equal(shards[0][:, c:], x[:, (2 * world - 1) * c:])     # chunk 2R-1
    assert torch.equal(zigzag_unshard(shards), x)
    with pytest.raises(ValueError):
        zigzag_shard(x[:, :3], 0, world + 1)


@pytest.mark.parametrize("world", [1, 2, 3, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_emulated_zigzag_ring_fwd_and_bwd_on_cpu(world, causal, monkeypatch):
    """The zigzag emulation's bookkeeping (chunk halves, per-chunk sums, reassembly in
    sequence order) with the oracle standing in for the kernels."""
    import numpy as np

    import oracle
    from exact_attention_155_b200 import ring
    monkeypatch.setattr(ring, "_attend_and_merge", _oracle_attend_and_merge)
    monkeypatch.setattr(ring, "_pair_terms", _oracle_pair_terms)
    monkeypatch.setattr(ring, "_add_terms", _oracle_add_terms)
    monkeypatch.setattr(ring, "_to_bf16", _oracle_to_bf16)
    full = _full_inputs(world, S=8, seed=199 + world)
    q, k, v, do = full
    out, lse = ring.ring_attention_fwd_emulated(q, k, v, world, causal=causal, scale=0.7,
                                                layout=ring.ZIGZAG)
    ref_o, ref_l = oracle.attention_forward(*[t.numpy() for t in full[:3]], causal=causal, scale=0.7)
    np.testing.assert_allclose(out.numpy(), ref_o, atol=_ATOL)
    np.testing.assert_allclose(lse.numpy(), ref_l, atol=_ATOL)
    grads = ring.ring_attention_bwd_emulated(q, k, v, out, do, lse, world, causal=causal, scale=0.7,
                                             layout=ring.ZIGZAG)
    refs = oracle.attention_backward(*[t.numpy() for t in full], causal=causal, scale=0.7)
    for g, r in zip(grads, refs):
        np.testing.assert_allclose(g.numpy(), r, atol=_ATOL)


def _zigzag_worker(rank, world, port, causal, q):
    """ring_attention_fwd and ring_attention_bwd in the zigzag layout over gloo with the
    oracle standing in for the kernels; returns this rank's shards of the results."""
    import oracle
    from exact_attention_155_b200 import ring

    _use_oracle_seams(ring)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        full = _full_inputs(world, S=8, seed=4242 + world)
        zz = lambda t, dim=1: ring.zigzag_shard(t, rank, world, dim)
        qs, ks, vs, dos = (zz(t).contiguous() for t in full)
        out, lse = ring.ring_attention_fwd(qs, ks, vs, causal=causal, scale=0.5, layout=ring.ZIGZAG)
        # The backward from the oracle's whole-sequence forward, as the ring forward gives it.
        ro, rl = oracle.attention_forward(*[t.numpy() for t in full[:3]], causal=causal, scale=0.5)
        os_ = zz(torch.from_numpy(ro)).contiguous()
        ls = zz(torch.from_numpy(rl), 2).contiguous()
        grads = ring.ring_attention_bwd(qs, ks, vs, os_, dos, ls, causal=causal, scale=0.5,
                                        layout=ring.ZIGZAG)
        q.put((rank, out.numpy(), lse.numpy(), [g.numpy() for g in grads], [t.numpy() for t in full]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_zigzag_ring_driver_over_gloo(world, causal):
    """Each rank's zigzag shards of the output, LSE and gradients equal the oracle's over
    the whole sequence."""
    import numpy as np

    import oracle
    from exact_attention_155_b200.ring import zigzag_shard
    got = _spawn(_zigzag_worker, world, causal)
    full = [torch.from_numpy(t) for t in got[0][3]]
    ref_o, ref_l = oracle.attention_forward(*[t.numpy() for t in full[:3]], causal=causal, scale=0.5)
    refs = oracle.attention_backward(*[t.numpy() for t in full], causal=causal, scale=0.5)
    zz = lambda a, r, dim=1: zigzag_shard(torch.from_numpy(a), r, world, dim).numpy()
    for rank in range(world):
        o, l, grads, _ = got[rank]
        np.testing.assert_allclose(o, zz(ref_o, rank), atol=_ATOL)
        np.testing.assert_allclose(l, zz(ref_l, rank, 2), atol=_ATOL)
        for g, r in zip(grads, refs):
            np.testing.assert_allclose(g, zz(r, rank), atol=_ATOL)
