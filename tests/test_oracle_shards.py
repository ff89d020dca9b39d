"""Pins for oracle.attention_backward_from_stats, the backward's terms for one key set
with the rows' LSE and output given (what the recomputed backward of one pair of
sequence shards computes). It is pinned to the whole-sequence backward, which the
finite-difference tests pin in turn: over a complete key set the terms are the
gradients, and over any partition of the keys (and of the queries, for dK and dV) they
add up to them. Planting the plausible mistake (each shard's own LSE instead of the
row's) must break the sum."""
import numpy as np
import pytest

import oracle


def _inputs(B, N, H, d, seed):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((B, N, H, d)) for _ in range(4)]


@pytest.mark.parametrize("causal", [False, True])
def test_complete_key_set_gives_the_gradients(causal):
    q, k, v, do = _inputs(2, 11, 3, 5, 41 + causal)
    out, lse = oracle.attention_forward(q, k, v, causal=causal, scale=0.6)
    ref = oracle.attention_backward(q, k, v, do, causal=causal, scale=0.6)
    got = oracle.attention_backward_from_stats(q, k, v, out, do, lse, causal=causal, scale=0.6)
    for g, r in zip(got, ref):
        np.testing.assert_allclose(g, r, atol=1e-12, rtol=1e-10)


def _shard_sums(q, k, v, out, do, lse, world, causal, scale, local_lse=False):
    """Sums of the terms over every (query shard, key shard) pair that the ring
    schedule visits: the diagonal pair with the causal mask, pairs below it in full,
    pairs above it skipped (causal) or in full (non-causal)."""
    B, N, H, d = q.shape
    S = N // world
    rows = lambda t, r: t[:, r * S:(r + 1) * S]
    dq, dk, dv = np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape)
    for i in range(world):
        for j in range(world):
            if causal and j > i:
                continue
            pair_causal = causal and j == i
            li = lse[:, :, i * S:(i + 1) * S]
            if local_lse:  # the mistake: each pair's own normaliser
                _, li = oracle.attention_forward(rows(q, i), rows(k, j), rows(v, j),
                                                 causal=pair_causal, scale=scale)
            tq, tk, tv = oracle.attention_backward_from_stats(
                rows(q, i), rows(k, j), rows(v, j), rows(out, i), rows(do, i), li,
                causal=pair_causal, scale=scale)
            dq[:, i * S:(i + 1) * S] += tq
            dk[:, j * S:(j + 1) * S] += tk
            dv[:, j * S:(j + 1) * S] += tv
    return dq, dk, dv


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_terms_over_shards_add_up_to_the_gradients(world, causal):
    q, k, v, do = _inputs(1, 12, 2, 4, 50 + world + 10 * causal)
    out, lse = oracle.attention_forward(q, k, v, causal=causal, scale=0.8)
    ref = oracle.attention_backward(q, k, v, do, causal=causal, scale=0.8)
    got = _shard_sums(q, k, v, out, do, lse, world, causal, 0.8)
    for g, r in zip(got, ref):
        np.testing.assert_allclose(g, r, atol=1e-12, rtol=1e-10)


@pytest.mark.parametrize("causal", [False, True])
def test_shard_local_lse_is_caught(causal):
    q, k, v, do = _inputs(1, 12, 2, 4, 77 + causal)
    out, lse = oracle.attention_forward(q, k, v, causal=causal, scale=0.8)
    ref = oracle.attention_backward(q, k, v, do, causal=causal, scale=0.8)
    bad = _shard_sums(q, k, v, out, do, lse, 3, causal, 0.8, local_lse=True)
    assert max(np.max(np.abs(g - r)) for g, r in zip(bad, ref)) > 1e-2


def test_row_with_no_key_contributes_nothing():
    # lse = -inf marks a row that saw no key: all its terms are exactly zero.
    q, k, v, do = _inputs(1, 4, 1, 3, 5)
    out = np.zeros_like(q)
    lse = np.full((1, 1, 4), -np.inf)
    tq, tk, tv = oracle.attention_backward_from_stats(q, k, v, out, do, lse, causal=True, scale=1.0)
    assert not tq.any() and not tk.any() and not tv.any()
