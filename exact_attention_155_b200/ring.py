"""Ring attention: exact attention over a sequence split into contiguous shards, one
per rank, built from the library's kernels (the ring sequence-parallel mode of
"Flash-Attention 2/3在ms-swift中的集成与性能提升", section on distributed training: each
device runs attention on its local segment and a ring exchange aggregates the global
context, with no all-to-all).

Rank r holds rows [r*S, (r+1)*S) of q, k and v (S = N / world). At step s it holds
the key/value shard of rank (r - s) mod world, attends its query shard to it with
fa_fwd_ex (causal only on its own shard; shards after its own are skipped when
causal), folds the partial result into a running fp32 output with fa_merge_partials,
and passes the shard on to rank r + 1 while it computes.

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


def ring_attention_fwd(q, k, v, causal: bool = False, scale: Optional[float] = None, group=None):
    """Distributed forward. q, k, v: this rank's shards [B, S, H, d] bf16 on its GPU;
    the process group must connect every rank of the ring. Returns (out [B, S, H, d]
    bf16, lse [B, H, S] fp32) for this rank's query rows over the whole sequence."""
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
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


def ring_attention_fwd_emulated(q, k, v, world: int, causal: bool = False,
                                scale: Optional[float] = None):
    """The same schedule and kernels for `world` virtual ranks in one process on one GPU
    (the shard exchange becomes indexing); q, k, v are the whole [B, N, H, d] tensors.
    Returns (out [B, N, H, d], lse [B, H, N])."""
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
            _attend_and_merge(qs, ks, vs, mode, scale, o_acc, lse_acc, out if s == last else None)
        outs.append(out)
        lses.append(lse_acc)
    return torch.cat(outs, dim=1), torch.cat(lses, dim=2)


def ring_attention_bwd(q, k, v, out, dout, lse, causal: bool = False,
                       scale: Optional[float] = None, group=None):
    """Distributed backward of ring_attention_fwd. q, k, v, out, dout: this rank's
    shards [B, S, H, d] bf16 (out as ring_attention_fwd returned it); lse: this rank's
    rows of the LSE over the whole sequence [B, H, S] fp32. Returns (dq, dk, dv) of this
    rank's shards, bf16."""
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
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


def ring_attention_bwd_emulated(q, k, v, out, dout, lse, world: int, causal: bool = False,
                                scale: Optional[float] = None):
    """ring_attention_bwd's schedule and kernels for `world` virtual ranks in one
    process on one GPU (the travelling dK/dV sums become one sum per shard); q, k, v,
    out, dout are the whole [B, N, H, d] tensors and lse [B, H, N]. Returns (dq, dk, dv)
    [B, N, H, d]."""
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


class _RingAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal, scale, group):
        out, lse = ring_attention_fwd(q, k, v, causal=causal, scale=scale, group=group)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.cfg = (causal, scale, group)
        ctx.mark_non_differentiable(lse)
        return out, lse

    @staticmethod
    def backward(ctx, dout, dlse):
        q, k, v, out, lse = ctx.saved_tensors
        causal, scale, group = ctx.cfg
        dout = dout if dout.is_contiguous() else dout.contiguous()
        dq, dk, dv = ring_attention_bwd(q, k, v, out, dout, lse, causal=causal, scale=scale,
                                        group=group)
        return dq, dk, dv, None, None, None


def ring_flash_attn_func(q, k, v, causal: bool = False, softmax_scale: Optional[float] = None,
                         group=None, return_lse: bool = False):
    """Differentiable ring attention: this rank's shards q, k, v [B, S, H, d] (bf16) of a
    sequence split into equal contiguous shards over the ranks of `group` (rank r holds
    rows [r*S, (r+1)*S)). Returns this rank's rows of the output over the whole sequence,
    or (out, lse); the backward runs ring_attention_bwd (every rank must call it)."""
    out, lse = _RingAttention.apply(q, k, v, bool(causal), softmax_scale, group)
    return (out, lse) if return_lse else out
