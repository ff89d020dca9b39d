"""Ring attention: exact attention over a sequence split into shards, one per rank,
built from the library's kernels (the ring sequence-parallel mode of
"Flash-Attention 2/3在ms-swift中的集成与性能提升", section on distributed training: each
device runs attention on its local segment and a ring exchange aggregates the global
context, with no all-to-all).

Two layouts of the sequence over the R ranks:
  * contiguous: rank r holds rows [r*S, (r+1)*S) of q, k and v (S = N / R);
  * zigzag: the sequence is cut into 2R chunks of S/2 rows and rank r holds chunks r
    and 2R-1-r, in that order. Under a causal mask every rank then does the same work
    at every step (two chunk-by-chunk products), where the contiguous layout gives
    rank r work at r+1 of the R steps and leaves the others idle.
At step s rank r holds the key/value shard of rank (r - s) mod R, attends its query
shard to it with fa_fwd_ex (contiguous: causal only on its own shard, shards after its
own skipped when causal; zigzag: per pair of chunks, see zigzag_plan), folds the
partial result into a running fp32 output with fa_merge_partials, and passes the shard
on to rank r + 1 while it computes.

The backward visits the shards in the same order. With the forward's output and LSE of
its query rows fixed, the recomputed backward of one (query shard, key/value shard)
pair (fa_bwd_ex) gives that pair's terms of dQ, dK and dV, and each gradient is the sum
of its terms (fa_accumulate keeps the sums in fp32). dQ stays on its rank; the sums
for dK and dV travel with their key/value shard and reach its owner after a full turn,
each hop overlapping the next pair's backward.

Every arithmetic step runs in the CUDA library; this module only orders calls and
moves buffers (torch.distributed point-to-point, NCCL on GPUs).
"""
from __future__ import annotations

from typing import List, Optional, Tuple

import torch

from . import ops

SKIP, FULL, CAUSAL = "skip", "full", "causal"
CONTIGUOUS, ZIGZAG = "contiguous", "zigzag"


def zigzag_plan(rank: int, src: int, causal: bool) -> List[Tuple[int, int, str]]:
    """The chunk pairs of one step in the zigzag layout: (query half, key/value half,
    mask) for this rank's queries against the key/value shard of rank `src`. Half 0 of
    rank r's shard is chunk r, half 1 is chunk 2R-1-r; a query chunk sees all of an
    earlier key chunk, the causal part of its own chunk and nothing of a later one."""
    if not causal:
        return [(0, 0, FULL), (0, 1, FULL), (1, 0, FULL), (1, 1, FULL)]
    if src == rank:
        return [(0, 0, CAUSAL), (1, 0, FULL), (1, 1, CAUSAL)]
    if src < rank:  # chunk src is before both of ours; chunk 2R-1-src is after both
        return [(0, 0, FULL), (1, 0, FULL)]
    return [(1, 0, FULL), (1, 1, FULL)]  # both chunks of src lie between ours


def zigzag_shard(x: torch.Tensor, rank: int, world: int, dim: int = 1) -> torch.Tensor:
    """Rank `rank`'s zigzag shard of a whole-sequence tensor: chunks rank and
    2*world-1-rank (of 2*world equal chunks along `dim`), concatenated."""
    n = x.shape[dim]
    if n % (2 * world):
        raise ValueError(f"sequence length {n} is not a multiple of 2 * world ({2 * world})")
    c = n // (2 * world)
    return torch.cat([x.narrow(dim, rank * c, c), x.narrow(dim, (2 * world - 1 - rank) * c, c)], dim)


def zigzag_unshard(shards: List[torch.Tensor], dim: int = 1) -> torch.Tensor:
    """The whole-sequence tensor from every rank's zigzag shard, in rank order."""
    world = len(shards)
    c = shards[0].shape[dim] // 2
    chunks = [None] * (2 * world)
    for r, t in enumerate(shards):
        chunks[r] = t.narrow(dim, 0, c)
        chunks[2 * world - 1 - r] = t.narrow(dim, c, c)
    return torch.cat(chunks, dim)


def _halves(t: torch.Tensor, dim: int = 1) -> Tuple[torch.Tensor, torch.Tensor]:
    """The two halves of a shard along `dim`, each contiguous (the kernels index a
    [B, N, H, d] operand from its sizes)."""
    c = t.shape[dim] // 2
    return t.narrow(dim, 0, c).contiguous(), t.narrow(dim, c, c).contiguous()


def ring_schedule(rank: int, world: int, causal: bool) -> List[Tuple[int, int, str]]:
    """(step, source rank of the key/value shard held at that step, mask) for `rank`."""
    out = []
    for s in range(world):
        src = (rank - s) % world
        if not causal:
            mode = FULL
        elif src == rank:
            mode = CAUSAL
        elif src < rank:
            mode = FULL
        else:
            mode = SKIP
        out.append((s, src, mode))
    return out


def ring_pass(send: torch.Tensor, recv: torch.Tensor, rank: int, world: int, group=None):
    """Start sending `send` to rank + 1 and receiving rank - 1's buffer into `recv`
    (ranks within `group`); returns the requests to wait on."""
    import torch.distributed as dist

    def peer(r):  # point-to-point calls take global ranks
        return r if group is None else dist.get_global_rank(group, r)
    ops_ = [dist.P2POp(dist.isend, send, peer((rank + 1) % world), group),
            dist.P2POp(dist.irecv, recv, peer((rank - 1) % world), group)]
    return dist.batch_isend_irecv(ops_)


def last_step(schedule) -> int:
    """The last step of a schedule that is not skipped (a rank always attends its own
    shard, at step 0): the step whose merge or sum also writes the bf16 result."""
    return max(s for s, _, mode in schedule if mode != SKIP)


def _attend_and_merge(q, k, v, mode, scale, o_acc, lse_acc, out, stream=None):
    """Folds the attention of q to one key/value shard into (o_acc, lse_acc); writes
    the merged output as bf16 into `out` when given."""
    if mode == SKIP:
        return
    o_p, lse_p = ops.fwd_ex(q, k, v, causal=(mode == CAUSAL), scale=scale, stream=stream)
    ops.merge_partials(o_acc, lse_acc, o_p, lse_p, out=out, stream=stream)


def _pair_terms(q, k, v, out, dout, lse, mode, scale, bufs, stream=None):
    """The terms of dQ, dK and dV of one (query shard, key/value shard) pair (bf16, in the
    buffers of `bufs`, made on first use with the backward workspace), or None for a
    skipped pair."""
    if mode == SKIP:
        return None
    if not bufs:
        B, S, H, d = q.shape
        bufs["terms"] = tuple(torch.empty_like(q) for _ in range(3))
        bufs["ws"] = torch.empty(max(1, ops.bwd_workspace_size(B, H, S, d)), dtype=torch.uint8,
                                 device=q.device)
    tq, tk, tv = bufs["terms"]
    ops.bwd_ex(q, k, v, out, dout, lse, causal=(mode == CAUSAL), scale=scale, dq=tq, dk=tk, dv=tv,
               workspace=bufs["ws"], stream=stream)
    return bufs["terms"]


def _add_terms(terms, dq_acc, dk_acc, dv_acc, dq_out, stream=None):
    """Adds a pair's terms to the fp32 sums dq_acc, dk_acc, dv_acc (nothing for a skipped
    pair); writes the dQ sum as bf16 into `dq_out` when given."""
    if terms is None:
        return
    tq, tk, tv = terms
    ops.accumulate(dq_acc, tq, out=dq_out, stream=stream)
    ops.accumulate(dk_acc, tk, stream=stream)
    ops.accumulate(dv_acc, tv, stream=stream)


def _to_bf16(acc, out, stream=None):
    """Writes the fp32 sum `acc` as bf16 into `out`."""
    ops.accumulate(acc, None, out=out, stream=stream)


def ring_attention_fwd(q, k, v, causal: bool = False, scale: Optional[float] = None, group=None,
                       layout: str = CONTIGUOUS):
    """Distributed forward. q, k, v: this rank's shards [B, S, H, d] bf16 on its GPU, in
    the given layout; the process group must connect every rank of the ring. Returns
    (out [B, S, H, d] bf16, lse [B, H, S] fp32) for this rank's query rows over the
    whole sequence, in the same layout."""
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    if layout == ZIGZAG:
        return _zigzag_fwd(q, k, v, causal, scale, rank, world, group)
    if layout != CONTIGUOUS:
        raise ValueError(f"unknown layout {layout!r}")
    B, S, H, d = q.shape
    kv = torch.stack([k, v]).contiguous()
    nxt = torch.empty_like(kv)
    o_acc = torch.zeros((B, S, H, d), dtype=torch.float32, device=q.device)
    lse_acc = torch.full((B, H, S), float("-inf"), dtype=torch.float32, device=q.device)
    out = torch.empty_like(q)
    sched = ring_schedule(rank, world, causal)
    last = last_step(sched)
    for s, src, mode in sched:
        reqs = ring_pass(kv, nxt, rank, world, group) if s + 1 < world else []
        _attend_and_merge(q, kv[0], kv[1], mode, scale, o_acc, lse_acc, out if s == last else None)
        for r in reqs:
            r.wait()
        kv, nxt = nxt, kv
    return out, lse_acc


def _zigzag_fwd(q, k, v, causal, scale, rank, world, group):
    """ring_attention_fwd in the zigzag layout: the running outputs of the two query
    chunks are kept apart and every kernel call is one pair of chunks."""
    B, S, H, d = q.shape
    if S % 2:
        raise ValueError("a zigzag shard holds two chunks of equal length")
    c = S // 2
    qh = _halves(q)
    kv = torch.stack([k, v]).contiguous()
    nxt = torch.empty_like(kv)
    o_acc = [torch.zeros((B, c, H, d), dtype=torch.float32, device=q.device) for _ in range(2)]
    lse_acc = [torch.full((B, H, c), float("-inf"), dtype=torch.float32, device=q.device)
               for _ in range(2)]
    for s, src, _ in ring_schedule(rank, world, False):
        reqs = ring_pass(kv, nxt, rank, world, group) if s + 1 < world else []
        kh, vh = _halves(kv[0]), _halves(kv[1])
        for a, b, mode in zigzag_plan(rank, src, causal):
            _attend_and_merge(qh[a], kh[b], vh[b], mode, scale, o_acc[a], lse_acc[a], None)
        for r in reqs:
            r.wait()
        kv, nxt = nxt, kv
    outs = [torch.empty_like(qh[a]) for a in range(2)]
    for a in range(2):
        _to_bf16(o_acc[a], outs[a])
    return torch.cat(outs, dim=1), torch.cat(lse_acc, dim=2)


def ring_attention_fwd_emulated(q, k, v, world: int, causal: bool = False,
                                scale: Optional[float] = None, layout: str = CONTIGUOUS,
                                step_events: Optional[list] = None):
    """The same schedule and kernels for `world` virtual ranks in one process on one GPU
    (the shard exchange becomes indexing); q, k, v are the whole [B, N, H, d] tensors
    in sequence order. Returns (out [B, N, H, d], lse [B, H, N]) in sequence order.
    step_events: if a list is given, (rank, step, start, stop) CUDA events around each
    rank's work at each step are appended to it (for the time of a parallel run:
    the sum over steps of the slowest rank's time)."""
    if layout == ZIGZAG:
        parts = [_zigzag_fwd_rank(q, k, v, world, r, causal, scale, step_events) for r in range(world)]
        return (zigzag_unshard([o for o, _ in parts], dim=1),
                zigzag_unshard([l for _, l in parts], dim=2))
    if layout != CONTIGUOUS:
        raise ValueError(f"unknown layout {layout!r}")
    B, N, H, d = q.shape
    if N % world:
        raise ValueError("N must be a multiple of the number of shards")
    S = N // world
    outs, lses = [], []
    for rank in range(world):
        qs = q[:, rank * S:(rank + 1) * S].contiguous()
        o_acc = torch.zeros((B, S, H, d), dtype=torch.float32, device=q.device)
        lse_acc = torch.full((B, H, S), float("-inf"), dtype=torch.float32, device=q.device)
        out = torch.empty_like(qs)
        sched = ring_schedule(rank, world, causal)
        last = last_step(sched)
        for s, src, mode in sched:
            ks = k[:, src * S:(src + 1) * S].contiguous()
            vs = v[:, src * S:(src + 1) * S].contiguous()
            ev = _step_start(step_events, rank, s)
            _attend_and_merge(qs, ks, vs, mode, scale, o_acc, lse_acc, out if s == last else None)
            _step_stop(ev)
        outs.append(out)
        lses.append(lse_acc)
    return torch.cat(outs, dim=1), torch.cat(lses, dim=2)


def _step_start(step_events, rank, step):
    if step_events is None or not torch.cuda.is_available():
        return None
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    step_events.append((rank, step, a, b))
    return b


def _step_stop(ev):
    if ev is not None:
        ev.record()


def _zigzag_fwd_rank(q, k, v, world, rank, causal, scale, step_events=None):
    """One virtual rank of the emulated zigzag forward: its shard's (out, lse)."""
    zz = lambda t, r, dim=1: zigzag_shard(t, r, world, dim)
    qh = _halves(zz(q, rank))
    B, c, H, d = qh[0].shape
    o_acc = [torch.zeros((B, c, H, d), dtype=torch.float32, device=q.device) for _ in range(2)]
    lse_acc = [torch.full((B, H, c), float("-inf"), dtype=torch.float32, device=q.device)
               for _ in range(2)]
    for s, src, _ in ring_schedule(rank, world, False):
        kh, vh = _halves(zz(k, src)), _halves(zz(v, src))
        ev = _step_start(step_events, rank, s)
        for a, b, mode in zigzag_plan(rank, src, causal):
            _attend_and_merge(qh[a], kh[b], vh[b], mode, scale, o_acc[a], lse_acc[a], None)
        _step_stop(ev)
    outs = [torch.empty_like(qh[a]) for a in range(2)]
    for a in range(2):
        _to_bf16(o_acc[a], outs[a])
    return torch.cat(outs, dim=1), torch.cat(lse_acc, dim=2)


def ring_attention_bwd(q, k, v, out, dout, lse, causal: bool = False,
                       scale: Optional[float] = None, group=None, layout: str = CONTIGUOUS):
    """Distributed backward of ring_attention_fwd. q, k, v, out, dout: this rank's
    shards [B, S, H, d] bf16 (out as ring_attention_fwd returned it); lse: this rank's
    rows of the LSE over the whole sequence [B, H, S] fp32; all in the given layout.
    Returns (dq, dk, dv) of this rank's shards, bf16."""
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    if layout == ZIGZAG:
        return _zigzag_bwd(q, k, v, out, dout, lse, causal, scale, rank, world, group)
    if layout != CONTIGUOUS:
        raise ValueError(f"unknown layout {layout!r}")
    kv = torch.stack([k, v]).contiguous()
    nxt = torch.empty_like(kv)
    dkv = torch.zeros((2, *q.shape), dtype=torch.float32, device=q.device)
    dkv_nxt = torch.empty_like(dkv)
    dq_acc = torch.zeros(q.shape, dtype=torch.float32, device=q.device)
    dq = torch.empty_like(q)
    sched = ring_schedule(rank, world, causal)
    last = last_step(sched)
    bufs = {}
    dreqs = []  # the pass of the dK/dV sums started at the previous step
    for s, src, mode in sched:
        reqs = ring_pass(kv, nxt, rank, world, group) if s + 1 < world else []
        terms = _pair_terms(q, kv[0], kv[1], out, dout, lse, mode, scale, bufs)
        # The sums of the shard held now arrive from rank - 1 while the terms are computed.
        if dreqs:
            for r in dreqs:
                r.wait()
            dkv, dkv_nxt = dkv_nxt, dkv
        _add_terms(terms, dq_acc, dkv[0], dkv[1], dq if s == last else None)
        # They move on with their shard; after the last step this pass brings every rank
        # the sums of its own shard.
        dreqs = ring_pass(dkv, dkv_nxt, rank, world, group) if world > 1 else []
        for r in reqs:
            r.wait()
        kv, nxt = nxt, kv
    for r in dreqs:
        r.wait()
    if dreqs:
        dkv, dkv_nxt = dkv_nxt, dkv
    dk, dv = torch.empty_like(k), torch.empty_like(v)
    _to_bf16(dkv[0], dk)
    _to_bf16(dkv[1], dv)
    return dq, dk, dv


def _zigzag_bwd(q, k, v, out, dout, lse, causal, scale, rank, world, group):
    """ring_attention_bwd in the zigzag layout: every kernel call is one pair of chunks;
    the fp32 dK/dV sums of both chunks of a key/value shard travel together."""
    B, S, H, d = q.shape
    if S % 2:
        raise ValueError("a zigzag shard holds two chunks of equal length")
    c = S // 2
    qh, oh, doh = _halves(q), _halves(out), _halves(dout)
    lh = _halves(lse, dim=2)
    kv = torch.stack([k, v]).contiguous()
    nxt = torch.empty_like(kv)
    dkv = torch.zeros((2, 2, B, c, H, d), dtype=torch.float32, device=q.device)  # [k|v][half]
    dkv_nxt = torch.empty_like(dkv)
    dq_acc = [torch.zeros((B, c, H, d), dtype=torch.float32, device=q.device) for _ in range(2)]
    bufs = {}
    dreqs = []  # the pass of the dK/dV sums started at the previous step
    for s, src, _ in ring_schedule(rank, world, False):
        reqs = ring_pass(kv, nxt, rank, world, group) if s + 1 < world else []
        kh, vh = _halves(kv[0]), _halves(kv[1])
        for i, (a, b, mode) in enumerate(zigzag_plan(rank, src, causal)):
            terms = _pair_terms(qh[a], kh[b], vh[b], oh[a], doh[a], lh[a], mode, scale, bufs)
            # The sums of the shard held now arrive from rank - 1 while the first pair's
            # terms are computed.
            if i == 0 and dreqs:
                for r in dreqs:
                    r.wait()
                dkv, dkv_nxt = dkv_nxt, dkv
            _add_terms(terms, dq_acc[a], dkv[0][b], dkv[1][b], None)
        dreqs = ring_pass(dkv, dkv_nxt, rank, world, group) if world > 1 else []
        for r in reqs:
            r.wait()
        kv, nxt = nxt, kv
    for r in dreqs:
        r.wait()
    if dreqs:
        dkv, dkv_nxt = dkv_nxt, dkv
    grads = []
    for acc in (dq_acc, dkv[0], dkv[1]):
        parts = [torch.empty_like(qh[0]) for _ in range(2)]
        for a in range(2):
            _to_bf16(acc[a], parts[a])
        grads.append(torch.cat(parts, dim=1))
    return tuple(grads)


def ring_attention_bwd_emulated(q, k, v, out, dout, lse, world: int, causal: bool = False,
                                scale: Optional[float] = None, layout: str = CONTIGUOUS):
    """ring_attention_bwd's schedule and kernels for `world` virtual ranks in one
    process on one GPU (the travelling dK/dV sums become one sum per shard); q, k, v,
    out, dout are the whole [B, N, H, d] tensors and lse [B, H, N], in sequence order.
    Returns (dq, dk, dv) [B, N, H, d] in sequence order."""
    if layout == ZIGZAG:
        return _zigzag_bwd_emulated(q, k, v, out, dout, lse, world, causal, scale)
    if layout != CONTIGUOUS:
        raise ValueError(f"unknown layout {layout!r}")
    B, N, H, d = q.shape
    if N % world:
        raise ValueError("N must be a multiple of the number of shards")
    S = N // world
    rows = lambda t, r: t[:, r * S:(r + 1) * S].contiguous()
    ks = [rows(k, r) for r in range(world)]
    vs = [rows(v, r) for r in range(world)]
    dk_acc = [torch.zeros((B, S, H, d), dtype=torch.float32, device=q.device) for _ in range(world)]
    dv_acc = [torch.zeros((B, S, H, d), dtype=torch.float32, device=q.device) for _ in range(world)]
    bufs = {}
    dqs = []
    for rank in range(world):
        qs, os_, dos = rows(q, rank), rows(out, rank), rows(dout, rank)
        ls = lse[:, :, rank * S:(rank + 1) * S].contiguous()
        dq_acc = torch.zeros((B, S, H, d), dtype=torch.float32, device=q.device)
        dq = torch.empty_like(qs)
        sched = ring_schedule(rank, world, causal)
        last = last_step(sched)
        for s, src, mode in sched:
            terms = _pair_terms(qs, ks[src], vs[src], os_, dos, ls, mode, scale, bufs)
            _add_terms(terms, dq_acc, dk_acc[src], dv_acc[src], dq if s == last else None)
        dqs.append(dq)
    dks, dvs = [], []
    for j in range(world):
        dks.append(torch.empty_like(ks[j]))
        dvs.append(torch.empty_like(vs[j]))
        _to_bf16(dk_acc[j], dks[j])
        _to_bf16(dv_acc[j], dvs[j])
    return torch.cat(dqs, dim=1), torch.cat(dks, dim=1), torch.cat(dvs, dim=1)


def _zigzag_bwd_emulated(q, k, v, out, dout, lse, world, causal, scale):
    zz = lambda t, r, dim=1: zigzag_shard(t, r, world, dim)
    B, N, H, d = q.shape
    c = N // (2 * world)
    kh = [_halves(zz(k, r)) for r in range(world)]
    vh = [_halves(zz(v, r)) for r in range(world)]
    new = lambda: torch.zeros((B, c, H, d), dtype=torch.float32, device=q.device)
    dk_acc = [[new(), new()] for _ in range(world)]
    dv_acc = [[new(), new()] for _ in range(world)]
    bufs = {}
    dqs = []
    for rank in range(world):
        qh, oh, doh = _halves(zz(q, rank)), _halves(zz(out, rank)), _halves(zz(dout, rank))
        lh = _halves(zz(lse, rank, 2), dim=2)
        dq_acc = [new(), new()]
        for s, src, _ in ring_schedule(rank, world, False):
            for a, b, mode in zigzag_plan(rank, src, causal):
                terms = _pair_terms(qh[a], kh[src][b], vh[src][b], oh[a], doh[a], lh[a], mode, scale, bufs)
                _add_terms(terms, dq_acc[a], dk_acc[src][b], dv_acc[src][b], None)
        dqs.append(dq_acc)
    results = []
    for accs in (dqs, dk_acc, dv_acc):
        shards = []
        for r in range(world):
            parts = [torch.empty((B, c, H, d), dtype=q.dtype, device=q.device) for _ in range(2)]
            for a in range(2):
                _to_bf16(accs[r][a], parts[a])
            shards.append(torch.cat(parts, dim=1))
        results.append(zigzag_unshard(shards, dim=1))
    return tuple(results)


class _RingAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal, scale, group, layout):
        out, lse = ring_attention_fwd(q, k, v, causal=causal, scale=scale, group=group, layout=layout)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.cfg = (causal, scale, group, layout)
        ctx.mark_non_differentiable(lse)
        return out, lse

    @staticmethod
    def backward(ctx, dout, dlse):
        q, k, v, out, lse = ctx.saved_tensors
        causal, scale, group, layout = ctx.cfg
        dout = dout if dout.is_contiguous() else dout.contiguous()
        dq, dk, dv = ring_attention_bwd(q, k, v, out, dout, lse, causal=causal, scale=scale,
                                        group=group, layout=layout)
        return dq, dk, dv, None, None, None, None


def ring_flash_attn_func(q, k, v, causal: bool = False, softmax_scale: Optional[float] = None,
                         group=None, return_lse: bool = False, layout: str = CONTIGUOUS):
    """Differentiable ring attention: this rank's shards q, k, v [B, S, H, d] (bf16) of a
    sequence split over the ranks of `group`: contiguous (rank r holds rows
    [r*S, (r+1)*S)) or zigzag (rank r holds chunks r and 2R-1-r of 2R, see zigzag_shard;
    balanced work under a causal mask). Returns this rank's rows of the output over the
    whole sequence, or (out, lse); the backward runs ring_attention_bwd (every rank must
    call it)."""
    out, lse = _RingAttention.apply(q, k, v, bool(causal), softmax_scale, group, layout)
    return (out, lse) if return_lse else out
