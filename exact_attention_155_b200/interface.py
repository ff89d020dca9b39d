"""Drop-in entry points with the names and arguments of the flash_attn API the pages use:
flash_attn_func(q, k, v, dropout_p, softmax_scale, causal) ("ms-swift长文本训练优化，
Flash-Attention显存省一半" section 2.3; "突破AI算力瓶颈：FlashAttention与MindSpore 2.0全场景
融合方案" section 核心API与使用示例), flash_attn_qkvpacked_func (same section of the MindSpore
page), flash_attn_varlen_func (long-text page section 4.3) and flash_attn_with_kvcache
(MindSpore page section 推理优化与KV缓存).

The first three are differentiable (torch.autograd.Function): the forward runs the fused
forward kernel and keeps (q, k, v, out, lse); the backward runs the recompute backward
kernel. flash_attn_with_kvcache is the decode step. Argument marshalling only; every
arithmetic step runs in libfa.so. dropout_p must be 0: dropout is not part of this library.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import ops

__all__ = ["flash_attn_func", "flash_attn_qkvpacked_func", "flash_attn_varlen_func",
           "flash_attn_with_kvcache"]


def _no_dropout(dropout_p):
    if dropout_p:
        raise NotImplementedError("dropout_p must be 0: dropout is not part of this library")


def _window(window_size, causal):
    """(left, right) for the library, or None when nothing but the causal mask remains.
    With causal the right edge is 0 (as in flash_attn, where causal overrides it)."""
    wl, wr = (-1, -1) if window_size is None else (int(window_size[0]), int(window_size[1]))
    if causal and wr > 0:
        wr = 0
    if wl < 0 and (wr < 0 or (causal and wr == 0)):
        return None
    return (wl, wr)


def _dense(t):
    """The output gradient as the kernels read it: a contiguous tensor (autograd may hand
    over a broadcast or a strided view)."""
    return t if t.is_contiguous() else t.contiguous()


class _Attention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal, scale, window, cu_seqlens, max_seqlen, deterministic):
        out, lse = ops.fwd_ex(q, k, v, causal=causal, scale=scale, window=window,
                              cu_seqlens=cu_seqlens, max_seqlen=max_seqlen)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.cfg = (causal, scale, window, cu_seqlens, max_seqlen, deterministic)
        ctx.mark_non_differentiable(lse)
        return out, lse

    @staticmethod
    def backward(ctx, dout, dlse):
        # lse is an output for inspection only (not differentiable).
        q, k, v, out, lse = ctx.saved_tensors
        causal, scale, window, cu_seqlens, max_seqlen, deterministic = ctx.cfg
        dq, dk, dv = ops.bwd_ex(q, k, v, out, _dense(dout), lse, causal=causal, scale=scale,
                                window=window, cu_seqlens=cu_seqlens, max_seqlen=max_seqlen,
                                deterministic=deterministic)
        return dq, dk, dv, None, None, None, None, None, None


class _PackedAttention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, qkv, causal, scale, window, deterministic):
        out, lse = ops.fwd_qkvpacked(qkv, causal=causal, scale=scale, window=window)
        ctx.save_for_backward(qkv, out, lse)
        ctx.cfg = (causal, scale, window, deterministic)
        ctx.mark_non_differentiable(lse)
        return out, lse

    @staticmethod
    def backward(ctx, dout, dlse):
        qkv, out, lse = ctx.saved_tensors
        causal, scale, window, deterministic = ctx.cfg
        dqkv = ops.bwd_qkvpacked(qkv, out, _dense(dout), lse, causal=causal, scale=scale,
                                 window=window, deterministic=deterministic)
        return dqkv, None, None, None, None


def flash_attn_func(q, k, v, dropout_p: float = 0.0, softmax_scale: Optional[float] = None,
                    causal: bool = False, window_size: Tuple[int, int] = (-1, -1),
                    deterministic: bool = False, return_attn_probs: bool = False,
                    block_size: Optional[int] = None):
    """Exact attention of q, k, v [batch, seqlen, nheads, headdim] (bf16, CUDA); returns
    out [batch, seqlen, nheads, headdim], or (out, lse [batch, nheads, seqlen]) with
    return_attn_probs=True. softmax_scale=None is 1/sqrt(headdim); window_size=(left,
    right) limits query i to keys [i - left, i + right] (-1: unbounded). block_size (the
    tiling hint of the ms-swift FA2/3 page's custom forward) is accepted and has no effect:
    the kernels' tiles are fixed by the tensor-core shapes, and tiling does not change the
    result of exact attention. deterministic=True (the flag the MindSpore page's
    常见问题与解决方案 sets) makes the backward bitwise repeatable (a slower kernel pair
    that writes every gradient element once); the forward is repeatable either way."""
    _no_dropout(dropout_p)
    if block_size is not None and int(block_size) <= 0:
        raise ValueError("block_size must be positive")
    out, lse = _Attention.apply(q, k, v, bool(causal), softmax_scale, _window(window_size, causal),
                                None, None, bool(deterministic))
    return (out, lse) if return_attn_probs else out


def flash_attn_qkvpacked_func(qkv, dropout_p: float = 0.0, softmax_scale: Optional[float] = None,
                              causal: bool = False, window_size: Tuple[int, int] = (-1, -1),
                              deterministic: bool = False, return_attn_probs: bool = False):
    """flash_attn_func on a packed qkv [batch, seqlen, 3, nheads, headdim], read in place;
    its gradient is packed the same way."""
    _no_dropout(dropout_p)
    out, lse = _PackedAttention.apply(qkv, bool(causal), softmax_scale, _window(window_size, causal),
                                      bool(deterministic))
    return (out, lse) if return_attn_probs else out


def flash_attn_varlen_func(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                           max_seqlen_k: int, dropout_p: float = 0.0,
                           softmax_scale: Optional[float] = None, causal: bool = False,
                           window_size: Tuple[int, int] = (-1, -1),
                           deterministic: bool = False, return_attn_probs: bool = False):
    """Packed variable-length batches: q, k, v [total_tokens, nheads, headdim]; sequence b
    is tokens [cu_seqlens[b], cu_seqlens[b + 1]) (int32 on the device). Queries and keys
    share one packing (self-attention): cu_seqlens_k must hold the same offsets as
    cu_seqlens_q (the same tensor, or an equal copy) and max_seqlen_k must equal
    max_seqlen_q. Returns out [total_tokens, nheads, headdim], or
    (out, lse [nheads, total_tokens])."""
    _no_dropout(dropout_p)
    same = cu_seqlens_k is cu_seqlens_q or (
        isinstance(cu_seqlens_k, torch.Tensor) and isinstance(cu_seqlens_q, torch.Tensor)
        and cu_seqlens_k.shape == cu_seqlens_q.shape and cu_seqlens_k.device == cu_seqlens_q.device
        and bool(torch.equal(cu_seqlens_k, cu_seqlens_q)))
    if not same or int(max_seqlen_k) != int(max_seqlen_q):
        raise NotImplementedError("queries and keys must share one packing (equal cu_seqlens "
                                  "offsets for both, and equal max_seqlen)")
    out, lse = _Attention.apply(q, k, v, bool(causal), softmax_scale, _window(window_size, causal),
                                cu_seqlens_q, int(max_seqlen_q), bool(deterministic))
    return (out, lse) if return_attn_probs else out


def flash_attn_with_kvcache(q, k_cache, v_cache, k=None, v=None, cache_seqlens=None,
                            softmax_scale: Optional[float] = None, causal: bool = False,
                            block_table=None, return_softmax_lse: bool = False):
    """One decode step: q [batch, 1, nheads, headdim]; k_cache, v_cache [batch, capacity,
    nheads, headdim], or pages [num_pages, page_size, nheads, headdim] with block_table
    [batch, max_blocks] (int32). cache_seqlens (int32 [batch] on the device, or an int for
    every sequence) counts the valid rows before this step; k, v ([batch, 1, nheads,
    headdim]) are appended at that row. Returns out [batch, 1, nheads, headdim], or
    (out, lse [batch, nheads])."""
    if cache_seqlens is None:
        raise ValueError("cache_seqlens is required")
    if not isinstance(cache_seqlens, torch.Tensor):
        cache_seqlens = torch.full((q.shape[0],), int(cache_seqlens), dtype=torch.int32,
                                   device=q.device)
    if block_table is None:
        out, lse = ops.decode(q, k_cache, v_cache, cache_seqlens, k_new=k, v_new=v, causal=causal,
                              scale=softmax_scale)
    else:
        out, lse = ops.decode_paged(q, k_cache, v_cache, block_table, cache_seqlens, k_new=k,
                                    v_new=v, causal=causal, scale=softmax_scale)
    return (out, lse) if return_softmax_lse else out
