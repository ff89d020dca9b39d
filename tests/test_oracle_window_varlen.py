"""Pins for the oracle's sliding window and variable-length (packed) batches.

* brute force on tiny inputs: every (query, key) pair decided by explicit loops from
  the window definition, scores and softmax summed term by term with math.exp;
* closed forms and special cases: a window of (0, 0) returns v_i and lse = scale q_i.k_i;
  a left window of at least N with right edge 0 is the causal mask; (-1, -1) is no mask;
* central finite differences of the windowed forward for the backward;
* packing invariants: sequences of a packed batch are independent (perturbing one
  leaves the others bit-identical) and empty sequences are skipped;
* a planted off-by-one in the window mask is caught by the brute-force pin.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import ref


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _brute(q, k, v, causal, scale, wl, wr):
    """Term-by-term attention for [1, Nq, H, d] / [1, Nk, H, d] with a window."""
    _, nq, H, d = q.shape
    nk = k.shape[1]
    out = np.zeros((nq, H, v.shape[3]))
    lse = np.zeros((H, nq))
    for h in range(H):
        for i in range(nq):
            ip = i + (nk - nq)
            vis = []
            for j in range(nk):
                ok = True
                if causal and j > ip:
                    ok = False
                if wl >= 0 and j < ip - wl:
                    ok = False
                if wr >= 0 and j > ip + wr:
                    ok = False
                if ok:
                    vis.append(j)
            if not vis:
                lse[h, i] = -math.inf
                continue
            s = {j: scale * sum(q[0, i, h, c] * k[0, j, h, c] for c in range(d)) for j in vis}
            m = max(s.values())
            e = {j: math.exp(s[j] - m) for j in vis}
            tot = sum(e.values())
            lse[h, i] = m + math.log(tot)
            for c in range(v.shape[3]):
                out[i, h, c] = sum(e[j] / tot * v[0, j, h, c] for j in vis)
    return out, lse


WINDOWS = [(-1, -1), (0, 0), (2, 0), (0, 3), (1, 2), (3, -1), (-1, 1), (6, 6)]


@pytest.mark.parametrize("wl,wr", WINDOWS)
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq", [7, 5])
def test_window_matches_brute_force(wl, wr, causal, nq):
    nk, H, d = 7, 2, 3
    q, k, v = _rand((1, nq, H, d), 1), _rand((1, nk, H, d), 2), _rand((1, nk, H, d), 3)
    out, lse = oracle.attention_forward(q, k, v, causal=causal, scale=0.7, window_left=wl,
                                        window_right=wr)
    bo, bl = _brute(q, k, v, causal, 0.7, wl, wr)
    np.testing.assert_allclose(out[0], bo, atol=1e-12)
    np.testing.assert_allclose(lse[0], bl, atol=1e-12)


def test_window_special_cases():
    N, H, d = 9, 2, 4
    q, k, v = _rand((1, N, H, d), 4), _rand((1, N, H, d), 5), _rand((1, N, H, d), 6)
    sc = 0.5
    # (0, 0): each query sees only its own key.
    out, lse = oracle.attention_forward(q, k, v, scale=sc, window_left=0, window_right=0)
    np.testing.assert_array_equal(out, v)
    np.testing.assert_allclose(lse[0].T, sc * np.sum(q[0] * k[0], axis=-1), atol=1e-14)
    # A left window reaching every earlier key, right edge 0: the causal mask.
    o1, l1 = oracle.attention_forward(q, k, v, scale=sc, window_left=N, window_right=0)
    o2, l2 = oracle.attention_forward(q, k, v, scale=sc, causal=True)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    # Unbounded on both sides: no mask; right edge 0 without causal: causal.
    o3, _ = oracle.attention_forward(q, k, v, scale=sc, window_left=-1, window_right=-1)
    o4, _ = oracle.attention_forward(q, k, v, scale=sc)
    np.testing.assert_array_equal(o3, o4)
    o5, _ = oracle.attention_forward(q, k, v, scale=sc, window_left=-1, window_right=0)
    np.testing.assert_array_equal(o5, o2)


@pytest.mark.parametrize("causal,wl,wr", [(False, 2, 1), (True, 3, 0), (False, -1, 0)])
def test_window_backward_matches_central_differences(causal, wl, wr):
    B, N, H, d = 1, 8, 1, 4
    q, k, v, do = (_rand((B, N, H, d), s) for s in (60, 61, 62, 63))
    sc = 0.5

    def loss(q_, k_, v_):
        o, _ = oracle.attention_forward(q_, k_, v_, causal=causal, scale=sc, window_left=wl,
                                        window_right=wr)
        return float(np.sum(o * do))

    grads = oracle.attention_backward(q, k, v, do, causal=causal, scale=sc, window_left=wl,
                                      window_right=wr)
    eps = 1e-6
    for which, g in enumerate(grads):
        num = np.zeros_like(g)
        for idx in np.ndindex(g.shape):
            args_p, args_m = [q.copy(), k.copy(), v.copy()], [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += eps
            args_m[which][idx] -= eps
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        err = np.max(np.abs(num - g)) / max(1e-12, np.max(np.abs(g)))
        assert err <= 1e-6, (which, err)


def test_varlen_sequences_are_independent():
    lens = [3, 0, 5, 1, 4]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    total, H, d = int(cu[-1]), 2, 4
    q, k, v, do = (_rand((total, H, d), s) for s in (70, 71, 72, 73))
    out, lse = oracle.attention_forward_varlen(q, k, v, cu, causal=True, scale=0.4)
    assert np.isfinite(out).all() and np.isfinite(lse).all()  # every token covered
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    s0, s1 = cu[2], cu[3]  # perturb sequence 2 only
    q2[s0:s1] += 1.0
    k2[s0:s1] -= 2.0
    v2[s0:s1] *= 3.0
    out2, lse2 = oracle.attention_forward_varlen(q2, k2, v2, cu, causal=True, scale=0.4)
    keep = np.ones(total, bool)
    keep[s0:s1] = False
    np.testing.assert_array_equal(out2[keep], out[keep])
    np.testing.assert_array_equal(lse2[:, keep], lse[:, keep])
    assert not np.allclose(out2[~keep], out[~keep])
    # Token 0 of every non-empty causal sequence copies its own value row.
    for b in range(len(lens)):
        if lens[b]:
            np.testing.assert_allclose(out[cu[b]], v[cu[b]], atol=1e-15)
    dq, dk, dv = oracle.attention_backward_varlen(q, k, v, do, cu, causal=True, scale=0.4)
    # Softmax translation invariance per sequence and head: sum over keys of dK is 0.
    for b in range(len(lens)):
        if lens[b]:
            np.testing.assert_allclose(dk[cu[b]:cu[b + 1]].sum(axis=0), 0.0, atol=1e-12)


def test_packing_example_of_the_long_text_page():
    """The packing example of "ms-swift长文本训练优化，Flash-Attention显存省一半" (section on
    --packing): a sample of 1024 tokens and one of 2048 are packed into one 3072-token
    sequence instead of each being padded to max_length. Packed attention must give each
    sample exactly its own attention (nothing crosses the boundary at token 1024), so
    the packed forward equals the two separate forwards computed alone."""
    lens = [1024, 2048]
    cu = np.array([0, 1024, 3072], dtype=np.int64)
    H, d = 1, 4
    q, k, v = (_rand((3072, H, d), s) for s in (90, 91, 92))
    out, lse = oracle.attention_forward_varlen(q, k, v, cu, causal=True, scale=0.5)
    for b in range(2):
        s0, s1 = cu[b], cu[b + 1]
        o_b, l_b = oracle.attention_forward(q[None, s0:s1], k[None, s0:s1], v[None, s0:s1],
                                            causal=True, scale=0.5)
        np.testing.assert_allclose(out[s0:s1], o_b[0], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[:, s0:s1], l_b[0], rtol=0, atol=1e-13)
    assert sum(lens) == 3072  # no padding tokens


def test_window_pin_catches_planted_off_by_one(monkeypatch):
    q, k, v = _rand((1, 7, 1, 3), 80), _rand((1, 7, 1, 3), 81), _rand((1, 7, 1, 3), 82)
    orig = ref.window_mask

    def bad(q_pos, nk, nqt, wl, wr):  # strict inequality on the left edge
        m = orig(q_pos, nk, nqt, wl, wr)
        j = np.arange(nk)[None, :]
        ip = np.asarray(q_pos)[:, None] + (nk - nqt)
        return m & (j > ip - wl) if wl >= 0 else m

    monkeypatch.setattr(ref, "window_mask", bad)
    out, _ = ref.attention_forward(q, k, v, scale=0.7, window_left=2, window_right=0)
    bo, _ = _brute(q, k, v, False, 0.7, 2, 0)
    assert not np.allclose(out[0], bo, atol=1e-6)


# ------------------------------------------------------------------- paged KV cache


def _paged_from_contiguous(kc, P, perm):
    """Split a contiguous [B, cap, H, d] cache into pages placed at `perm` positions."""
    B, cap, H, d = kc.shape
    nb = cap // P
    pages = np.full((B * nb + 3, P, H, d), np.nan)  # spare pages stay NaN: never read
    table = np.zeros((B, nb), dtype=np.int64)
    for b in range(B):
        for j in range(nb):
            pid = perm[b * nb + j]
            pages[pid] = kc[b, j * P:(j + 1) * P]
            table[b, j] = pid
    return pages, table


def test_paged_decode_is_contiguous_decode_under_any_page_placement():
    B, cap, H, d, P = 3, 64, 2, 8, 16
    kc, vc = _rand((B, cap, H, d), 90), _rand((B, cap, H, d), 91)
    q, kn, vn = _rand((B, 1, H, d), 92), _rand((B, 1, H, d), 93), _rand((B, 1, H, d), 94)
    seq = np.array([0, 37, 63])
    ref_o, ref_l, ref_k, _ = oracle.decode_step(q, kc, vc, seq, kn, vn, scale=0.3)
    perm = np.random.default_rng(95).permutation(B * (cap // P) + 3)
    kp, table = _paged_from_contiguous(kc, P, perm)
    vp, _ = _paged_from_contiguous(vc, P, perm)
    o, l, kp2, _ = oracle.decode_step_paged(q, kp, vp, table, seq, kn, vn, scale=0.3)
    np.testing.assert_array_equal(o, ref_o)
    np.testing.assert_array_equal(l, ref_l)
    # The appended row landed in its page, at the slot its position names.
    for b in range(B):
        r = seq[b]
        np.testing.assert_array_equal(kp2[table[b, r // P], r % P], kn[b, 0])
    # Spare pages were neither read (outputs finite) nor written.
    spare = sorted(set(range(kp.shape[0])) - set(table.ravel().tolist()))
    assert np.isnan(kp2[spare]).all()
    assert np.isfinite(o).all()
    # Step 0 of sequence 0 returns the new value row exactly.
    np.testing.assert_array_equal(o[0, 0], vn[0, 0])
