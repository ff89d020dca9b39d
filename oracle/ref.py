"""Float64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY. This module is the slow, obviously-correct statement of
what the GPU path computes. Only the test suite, the smoke check in
``__graft_entry__`` and the ``cpu_baseline`` / reference arm of ``bench.py`` may
import it. The product path (the CUDA library and its Python binding) never
imports, calls or falls back to anything here, and nothing here imports the
product path.

Sources (web pages on FlashAttention, cited by title and section):

* "Flash-Attention 2/3在ms-swift中的集成与性能提升" (FA2/3 in ms-swift), opening
  formula: Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V, and the statement that
  the full score matrix S is what tiling avoids storing.
* Qwen flash_attn explainer, section 一 "什么是 Attention": the three steps
  (scores Q.K^T, scale by 1/sqrt(d_k) and softmax, weighted sum of V).
* "FlashAttention优化Transformer显存与计算效率", section 2.1 (the naive
  computation over [batch, heads, seq_len, dim]) and section 2.2.2 (blockwise
  softmax: per block a max m and an exp-sum l, combined stably).
* "突破AI算力瓶颈：FlashAttention与MindSpore 2.0全场景融合方案", section
  推理优化与KV缓存 (flash_attn_with_kvcache: append one K/V row per step at
  position cache_seqlens, attend one query row, causal=True).

Readings taken where the pages are silent (each is also listed in the design notes):

* Layout: tensors are [B, N, H, d] (batch, seq_len, heads, head_dim), as in the
  ms-swift long-text page section 1.1.
* scale=None means 1/sqrt(d) (the formula's d_k).
* LSE is the natural-log log-sum-exp of the *scaled* scores of each query row
  over its visible keys, laid out [B, H, Nq].
* Causal with Nq != Nk aligns bottom-right: key j is visible to query i iff
  j <= i + (Nk - Nq). With Nq == Nk this is the usual j <= i.
* A query row with no visible key returns out = 0 and lse = -inf.
* cache_seqlens[b] is the number of valid cache rows before the step's append;
  with k_new given, the new row is written at that index and attention covers
  cache_seqlens[b] + 1 rows; without it, it covers cache_seqlens[b] rows.
* The backward is the analytic gradient of the definition (the pages only say the
  scores are recomputed, not stored).
* Sliding window ("Flash-Attention 2/3在ms-swift中的集成与性能提升", FA3 feature list;
  the page names the mask, not its parameters): with the query's position on the key
  axis i' = i + (Nk - Nq), key j is visible iff i' - window_left <= j <= i' +
  window_right; -1 leaves a side unbounded. It combines with the causal mask by AND.
* Paged KV cache ("突破AI算力瓶颈：FlashAttention与MindSpore 2.0全场景融合方案",
  section 推理优化与KV缓存: the cache is stored in pages to avoid fragmentation): pages
  of page_size rows are [num_pages, page_size, H, d]; row r of sequence b is row
  r % page_size of page block_table[b][r // page_size]. Paging is addressing only:
  the step is the contiguous decode step on the rows the table names.
* Variable-length batches (packing, "ms-swift长文本训练优化，Flash-Attention显存省一半"
  sections 4.2 and 5.1): tokens of B sequences are packed into [total, H, d] and
  sequence b is tokens [cu_seqlens[b], cu_seqlens[b+1]); each sequence is an
  independent attention problem (nothing is attended across sequences); the LSE is
  laid out [H, total].
* Ring attention's backward ("Flash-Attention 2/3在ms-swift中的集成与性能提升", section on
  distributed training, names the ring for training but gives no backward): with each
  query row's LSE and output taken from the whole sequence, the backward's terms for one
  key shard add up over the shards to the gradients (attention_backward_from_stats).

Every array is numpy float64; callers convert the exact bf16 input values first.
Large problems are processed in blocks of query rows; each block's softmax is the
exact row softmax over all keys (no online rescaling), so blocking does not change
the arithmetic beyond floating-point summation order inside BLAS.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "default_scale",
    "visible_mask",
    "window_mask",
    "scores",
    "softmax_rows",
    "attention_forward",
    "attention_backward",
    "attention_backward_from_stats",
    "attention_forward_varlen",
    "attention_backward_varlen",
    "blockwise_forward",
    "merge_partials",
    "decode_step",
    "decode_sequence",
    "decode_step_paged",
]


def default_scale(d: int) -> float:
    """softmax_scale=None -> 1/sqrt(d_k) (the formula of the ms-swift FA2/3 page)."""
    return 1.0 / math.sqrt(d)


def visible_mask(q_pos: np.ndarray, nk: int, causal: bool, nq_total: int) -> np.ndarray:
    """Boolean [len(q_pos), nk] mask of keys each query may attend to.

    Causal uses bottom-right alignment: key j visible to query i iff
    j <= i + (nk - nq_total). Non-causal sees every key.
    """
    j = np.arange(nk)[None, :]
    if not causal:
        return np.ones((len(q_pos), nk), dtype=bool)
    return j <= (np.asarray(q_pos)[:, None] + (nk - nq_total))


def window_mask(q_pos: np.ndarray, nk: int, nq_total: int, window_left: int,
                window_right: int) -> np.ndarray:
    """Boolean [len(q_pos), nk] sliding-window mask: key j visible to query i iff
    i' - window_left <= j <= i' + window_right with i' = i + (nk - nq_total);
    -1 = unbounded side."""
    j = np.arange(nk)[None, :]
    ip = np.asarray(q_pos)[:, None] + (nk - nq_total)
    m = np.ones((len(q_pos), nk), dtype=bool)
    if window_left >= 0:
        m &= j >= ip - window_left
    if window_right >= 0:
        m &= j <= ip + window_right
    return m


def _mask(ridx, nk, causal, nq, window_left, window_right):
    mask = visible_mask(ridx, nk, causal, nq)
    if window_left >= 0 or window_right >= 0:
        mask = mask & window_mask(ridx, nk, nq, window_left, window_right)
    return mask


def scores(qm: np.ndarray, km: np.ndarray, scale: float) -> np.ndarray:
    """S = scale * Q K^T for one (batch, head): [nq, d] x [nk, d] -> [nq, nk]."""
    return scale * (qm @ km.T)


def softmax_rows(s: np.ndarray, mask: np.ndarray):
    """Max-subtracted row softmax with masked entries excluded.

    Returns (P, lse). Rows with no visible entry give P = 0 and lse = -inf.
    """
    s = np.where(mask, s, -np.inf)
    m = np.max(s, axis=1, keepdims=True)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    e = np.where(mask, np.exp(s - m_safe), 0.0)
    l = np.sum(e, axis=1, keepdims=True)
    p = np.where(empty, 0.0, e / np.where(empty, 1.0, l))
    with np.errstate(divide="ignore"):
        lse = np.where(empty, -np.inf, m_safe + np.log(np.where(empty, 1.0, l)))
    return p, lse[:, 0]


def _resolve_scale(scale, d):
    return default_scale(d) if scale is None else float(scale)


def attention_forward(q, k, v, causal=False, scale=None, row_block=1024,
                      heads=None, rows=None, window_left=-1, window_right=-1):
    """Exact attention forward, materialising S per (b, h) in query-row blocks.

    q: [B, Nq, H, d]; k, v: [B, Nk, H, d] (float64).
    Returns out [B, Nq, H, d] and lse [B, H, Nq].

    ``heads`` (list of (b, h)) and ``rows`` (sorted query indices) restrict the
    work to a sample; entries outside the sample are left as NaN.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    sc = _resolve_scale(scale, d)
    out = np.full((B, Nq, H, v.shape[3]), np.nan)
    lse = np.full((B, H, Nq), np.nan)
    head_list = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    row_idx = np.arange(Nq) if rows is None else np.asarray(rows)
    for (b, h) in head_list:
        km = k[b, :, h, :]
        vm = v[b, :, h, :]
        for s0 in range(0, len(row_idx), row_block):
            ridx = row_idx[s0:s0 + row_block]
            qm = q[b, ridx, h, :]
            mask = _mask(ridx, Nk, causal, Nq, window_left, window_right)
            p, l = softmax_rows(scores(qm, km, sc), mask)
            out[b, ridx, h, :] = p @ vm
            lse[b, h, ridx] = l
    return out, lse


def attention_backward(q, k, v, dout, causal=False, scale=None, row_block=1024,
                       heads=None, window_left=-1, window_right=-1):
    """Analytic gradients of out = softmax(scale*Q K^T, mask) V.

    With P the row softmax and dO the output gradient:
      dV = P^T dO,  dP = dO V^T,  dS = P * (dP - rowsum(P * dP)),
      dQ = scale * dS K,  dK = scale * dS^T Q.
    S is rebuilt from Q and K in query-row blocks (recomputation, as the pages
    describe for the backward pass), never stored whole.
    Returns dq, dk, dv with the shapes of q, k, v (NaN outside ``heads``).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    sc = _resolve_scale(scale, d)
    dq = np.full(q.shape, np.nan)
    dk = np.full(k.shape, np.nan)
    dv = np.full(v.shape, np.nan)
    head_list = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for (b, h) in head_list:
        km = k[b, :, h, :]
        vm = v[b, :, h, :]
        dk_acc = np.zeros((Nk, d))
        dv_acc = np.zeros((Nk, v.shape[3]))
        for r0 in range(0, Nq, row_block):
            ridx = np.arange(r0, min(Nq, r0 + row_block))
            qm = q[b, ridx, h, :]
            dom = dout[b, ridx, h, :]
            mask = _mask(ridx, Nk, causal, Nq, window_left, window_right)
            p, _ = softmax_rows(scores(qm, km, sc), mask)
            dv_acc += p.T @ dom
            dp = dom @ vm.T
            rowdot = np.sum(p * dp, axis=1, keepdims=True)
            ds = p * (dp - rowdot)
            dq[b, ridx, h, :] = sc * (ds @ km)
            dk_acc += sc * (ds.T @ qm)
        dk[b, :, h, :] = dk_acc
        dv[b, :, h, :] = dv_acc
    return dq, dk, dv


def attention_backward_from_stats(q, k, v, out, dout, lse, causal=False, scale=None):
    """The backward's terms for one key set, with the softmax statistics of every query
    row given rather than computed over these keys.

    The backward recomputes the probabilities from Q, K and what the forward kept
    (the recomputation of the ms-swift FA2/3 page's key-techniques list and section 1.2
    of "ms-swift长文本训练优化，Flash-Attention显存省一半"): P = exp(scale*Q K^T - lse)
    on visible entries, with lse the row's log-sum-exp over ALL its keys, and the
    row term rowsum(P * dP) of the softmax gradient written as rowsum(dO * O) with O
    the row's full output (the two are equal when the key set is complete). Then
      dV = P^T dO,  dS = P * (dO V^T - rowsum(dO * O)),  dQ = scale dS K,
      dK = scale dS^T Q.
    Over a partition of the keys the terms add up to attention_backward's gradients;
    this is how attention split over sequence shards gets its gradients.

    q, out, dout: [B, Nq, H, d]; k, v: [B, Nk, H, d]; lse: [B, H, Nq]. Returns the
    terms dq [B, Nq, H, d], dk, dv [B, Nk, H, d].
    """
    q, k, v, out, dout, lse = (np.asarray(t, dtype=np.float64) for t in (q, k, v, out, dout, lse))
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    sc = _resolve_scale(scale, d)
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    ridx = np.arange(Nq)
    mask = _mask(ridx, Nk, causal, Nq, -1, -1)
    for b in range(B):
        for h in range(H):
            qm, km, vm = q[b, :, h, :], k[b, :, h, :], v[b, :, h, :]
            dom = dout[b, :, h, :]
            row_lse = lse[b, h, :][:, None]
            fin = np.isfinite(row_lse)  # lse = -inf: the row sees no key at all
            live = mask & fin
            shifted = scores(qm, km, sc) - np.where(fin, row_lse, 0.0)
            p = np.zeros((Nq, Nk))
            p[live] = np.exp(shifted[live])
            dv[b, :, h, :] = p.T @ dom
            dp = dom @ vm.T
            rowdot = np.sum(dom * out[b, :, h, :], axis=1, keepdims=True)
            ds = p * (dp - rowdot)
            dq[b, :, h, :] = sc * (ds @ km)
            dk[b, :, h, :] = sc * (ds.T @ qm)
    return dq, dk, dv


def attention_forward_varlen(q, k, v, cu_seqlens, causal=False, scale=None,
                             window_left=-1, window_right=-1):
    """Packed variable-length forward: q, k, v [total, H, d]; sequence b is tokens
    [cu_seqlens[b], cu_seqlens[b+1]). Returns out [total, H, d] and lse [H, total]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    total, H, d = q.shape
    out = np.full((total, H, v.shape[2]), np.nan)
    lse = np.full((H, total), np.nan)
    cu = [int(x) for x in cu_seqlens]
    for b in range(len(cu) - 1):
        s0, s1 = cu[b], cu[b + 1]
        if s1 == s0:
            continue
        o, l = attention_forward(q[None, s0:s1], k[None, s0:s1], v[None, s0:s1], causal=causal,
                                 scale=scale, window_left=window_left, window_right=window_right)
        out[s0:s1] = o[0]
        lse[:, s0:s1] = l[0]
    return out, lse


def attention_backward_varlen(q, k, v, dout, cu_seqlens, causal=False, scale=None,
                              window_left=-1, window_right=-1):
    """Gradients of attention_forward_varlen; dq, dk, dv [total, H, d]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    dq = np.full(q.shape, np.nan)
    dk = np.full(k.shape, np.nan)
    dv = np.full(v.shape, np.nan)
    cu = [int(x) for x in cu_seqlens]
    for b in range(len(cu) - 1):
        s0, s1 = cu[b], cu[b + 1]
        if s1 == s0:
            continue
        g = attention_backward(q[None, s0:s1], k[None, s0:s1], v[None, s0:s1], dout[None, s0:s1],
                               causal=causal, scale=scale, window_left=window_left,
                               window_right=window_right)
        dq[s0:s1], dk[s0:s1], dv[s0:s1] = g[0][0], g[1][0], g[2][0]
    return dq, dk, dv


def merge_partials(o_parts, lse_parts):
    """Combine partial attention results computed over disjoint key sets.

    Each part s holds o_s (its own normalised output) and lse_s (its own
    log-sum-exp). This is the stable combination of the per-block max m and
    exp-sum l described in section 2.2.2 of "FlashAttention优化Transformer显存与
    计算效率", written in log space: LSE = log sum_s exp(lse_s) and
    O = sum_s exp(lse_s - LSE) o_s. Parts with lse_s = -inf contribute nothing.

    o_parts: [S, ..., d]; lse_parts: [S, ...]. Returns (o, lse).
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = np.max(lse_parts, axis=0)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    w = np.exp(lse_parts - m_safe[None])
    tot = np.sum(w, axis=0)
    with np.errstate(divide="ignore"):
        lse = np.where(empty, -np.inf, m_safe + np.log(np.where(empty, 1.0, tot)))
    coef = np.where(empty[None], 0.0, w / np.where(empty, 1.0, tot)[None])
    o = np.sum(coef[..., None] * o_parts, axis=0)
    return o, lse


def blockwise_forward(q, k, v, causal=False, scale=None, block_q=64, block_k=64):
    """Tiled forward with a running max m and running sum l per query row.

    Restates section 2.2.1/2.2.2 of "FlashAttention优化Transformer显存与计算效率":
    loop over query blocks and, inside, over key blocks; for each key block take
    the block's row max and exp-sum and fold them into the running (m, l, acc)
    with the rescale factor exp(m_old - m_new). The full S is never formed. Used
    only to check the materialising oracle above.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    sc = _resolve_scale(scale, d)
    out = np.zeros((B, Nq, H, v.shape[3]))
    lse = np.zeros((B, H, Nq))
    for b in range(B):
        for h in range(H):
            for i0 in range(0, Nq, block_q):
                ridx = np.arange(i0, min(Nq, i0 + block_q))
                qb = q[b, ridx, h, :]
                m = np.full(len(ridx), -np.inf)
                l = np.zeros(len(ridx))
                acc = np.zeros((len(ridx), v.shape[3]))
                for j0 in range(0, Nk, block_k):
                    cidx = np.arange(j0, min(Nk, j0 + block_k))
                    s = sc * (qb @ k[b, cidx, h, :].T)
                    vis = visible_mask(ridx, Nk, causal, Nq)[:, cidx]
                    s = np.where(vis, s, -np.inf)
                    m_blk = np.max(s, axis=1)
                    m_new = np.maximum(m, m_blk)
                    base = np.where(np.isfinite(m_new), m_new, 0.0)
                    alpha = np.where(np.isfinite(m), np.exp(m - base), 0.0)
                    p = np.where(vis, np.exp(s - base[:, None]), 0.0)
                    l = alpha * l + np.sum(p, axis=1)
                    acc = alpha[:, None] * acc + p @ v[b, cidx, h, :]
                    m = m_new
                empty = l == 0.0
                out[b, ridx, h, :] = np.where(empty[:, None], 0.0,
                                              acc / np.where(empty, 1.0, l)[:, None])
                with np.errstate(divide="ignore"):
                    lse[b, h, ridx] = np.where(empty, -np.inf,
                                               np.where(np.isfinite(m), m, 0.0)
                                               + np.log(np.where(empty, 1.0, l)))
    return out, lse


def decode_step(q, k_cache, v_cache, cache_seqlens, k_new=None, v_new=None,
                scale=None):
    """One incremental decode step (flash_attn_with_kvcache, MindSpore page,
    section 推理优化与KV缓存).

    q: [B, 1, H, d]; caches: [B, Ncap, H, d]; cache_seqlens: int [B] = valid rows
    before this step. With k_new/v_new ([B, 1, H, d]) the new row is written at
    index cache_seqlens[b] of *copies* of the caches and the query attends rows
    [0, cache_seqlens[b] + 1); without them it attends rows [0, cache_seqlens[b]).
    A single query row at the end of the sequence sees every valid key, so the
    causal flag changes nothing here (bottom-right alignment).

    Returns (out [B, 1, H, d], lse [B, H], k_cache', v_cache').
    """
    q = np.asarray(q, dtype=np.float64)
    kc = np.array(k_cache, dtype=np.float64, copy=True)
    vc = np.array(v_cache, dtype=np.float64, copy=True)
    B, _, H, d = q.shape
    Ncap = kc.shape[1]
    sc = _resolve_scale(scale, d)
    out = np.zeros((B, 1, H, vc.shape[3]))
    lse = np.zeros((B, H))
    for b in range(B):
        L = int(cache_seqlens[b])
        if k_new is not None:
            if L + 1 > Ncap:
                raise ValueError("cache full: cache_seqlens[b] + 1 > capacity")
            kc[b, L] = np.asarray(k_new, dtype=np.float64)[b, 0]
            vc[b, L] = np.asarray(v_new, dtype=np.float64)[b, 0]
            L += 1
        if L > Ncap:
            raise ValueError("cache_seqlens[b] > capacity")
        for h in range(H):
            if L == 0:
                out[b, 0, h] = 0.0
                lse[b, h] = -np.inf
                continue
            s = scores(q[b, :, h, :], kc[b, :L, h, :], sc)
            p, l = softmax_rows(s, np.ones_like(s, dtype=bool))
            out[b, 0, h] = (p @ vc[b, :L, h, :])[0]
            lse[b, h] = l[0]
    return out, lse, kc, vc


def decode_step_paged(q, k_pages, v_pages, block_table, cache_seqlens, k_new=None, v_new=None,
                      scale=None):
    """decode_step over a paged cache: gather each sequence's logical rows through its
    block table, run decode_step, and scatter the appended row back into its page.

    k_pages, v_pages: [num_pages, page_size, H, d]; block_table: int [B, max_blocks].
    Returns (out [B, 1, H, d], lse [B, H], k_pages', v_pages') with the pages copied.
    """
    kp = np.array(k_pages, dtype=np.float64, copy=True)
    vp = np.array(v_pages, dtype=np.float64, copy=True)
    bt = np.asarray(block_table)
    B, max_blocks = bt.shape
    P = kp.shape[1]
    rows = np.arange(max_blocks * P)
    page_of, slot_of = rows // P, rows % P
    kc = np.stack([kp[bt[b, page_of], slot_of] for b in range(B)])  # [B, cap, H, d]
    vc = np.stack([vp[bt[b, page_of], slot_of] for b in range(B)])
    out, lse, kc2, vc2 = decode_step(q, kc, vc, cache_seqlens, k_new, v_new, scale=scale)
    if k_new is not None:
        for b in range(B):
            r = int(cache_seqlens[b])
            kp[bt[b, r // P], r % P] = kc2[b, r]
            vp[bt[b, r // P], r % P] = vc2[b, r]
    return out, lse, kp, vp


def decode_sequence(q_steps, k_steps, v_steps, k_cache, v_cache, start_seqlens,
                    scale=None):
    """Replay T decode steps with append (the incremental loop of the MindSpore
    page): step t uses cache_seqlens = start_seqlens + t.

    q_steps, k_steps, v_steps: [T, B, 1, H, d]. Returns outs [T, B, 1, H, d],
    lses [T, B, H] and the final caches.
    """
    kc = np.asarray(k_cache, dtype=np.float64)
    vc = np.asarray(v_cache, dtype=np.float64)
    T = len(q_steps)
    outs, lses = [], []
    seq = np.asarray(start_seqlens, dtype=np.int64)
    for t in range(T):
        o, l, kc, vc = decode_step(q_steps[t], kc, vc, seq + t, k_steps[t], v_steps[t],
                                   scale=scale)
        outs.append(o)
        lses.append(l)
    return np.stack(outs), np.stack(lses), kc, vc
