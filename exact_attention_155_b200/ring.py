"""Ring attention: exact attention over a sequence split into contiguous shards, one
per rank, built from the library's kernels (the ring sequence-parallel mode of
"Flash-Attention 2/3在ms-swift中的集成与性能提升", section on distributed training: each
device runs attention on its local segment and a ring exchange aggregates the global
context, with no all-to-all).

Rank r holds rows [r*S, (r+1)*S) of q, k and v (S = N / world). At step s it holds
the key/value shard of rank (r - s) mod world, attends its query shard to it with
fa_fwd_ex (causal only on its own shard; shards after its own are skipped when
causal), folds the partial result into a running fp32 output with fa_merge_partials,
and passes the shard on to rank r + 1 while it computes. Every arithmetic step runs in
the CUDA library; this module only orders calls and moves buffers (torch.distributed
point-to-point, NCCL on GPUs).
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
    """Start sending `send` to rank + 1 and receiving rank - 1's buffer into `recv`;
    returns the requests to wait on."""
    import torch.distributed as dist
    ops_ = [dist.P2POp(dist.isend, send, (rank + 1) % world, group),
            dist.P2POp(dist.irecv, recv, (rank - 1) % world, group)]
    return dist.batch_isend_irecv(ops_)


def _attend_and_merge(q, k, v, mode, scale, o_acc, lse_acc, out, stream=None):
    if mode == SKIP:
        return
    o_p, lse_p = ops.fwd_ex(q, k, v, causal=(mode == CAUSAL), scale=scale, stream=stream)
    ops.merge_partials(o_acc, lse_acc, o_p, lse_p, out=out, stream=stream)


def _finish(o_acc, out):
    # Rows whose every shard was skipped cannot occur (a rank always attends its own
    # shard); the last merge wrote `out` unless the last steps were skipped, so write
    # it from the accumulator here in every case.
    out.copy_(o_acc.to(torch.bfloat16))
    return out


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
    for s, src, mode in ring_schedule(rank, world, causal):
        reqs = ring_pass(kv, nxt, rank, world, group) if s + 1 < world else []
        _attend_and_merge(q, kv[0], kv[1], mode, scale, o_acc, lse_acc, None)
        for r in reqs:
            r.wait()
        kv, nxt = nxt, kv
    return _finish(o_acc, out), lse_acc


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
        for _, src, mode in ring_schedule(rank, world, causal):
            ks = k[:, src * S:(src + 1) * S].contiguous()
            vs = v[:, src * S:(src + 1) * S].contiguous()
            _attend_and_merge(qs, ks, vs, mode, scale, o_acc, lse_acc, None)
        outs.append(_finish(o_acc, torch.empty_like(qs)))
        lses.append(lse_acc)
    return torch.cat(outs, dim=1), torch.cat(lses, dim=2)
