"""Pins for the float64 oracle: checks against facts fixed by the pages and by
mathematics, none of which re-types the oracle's own formulas.

* hand-derived closed forms (tests/golden/closed_form.json);
* the tiled online-softmax restatement of section 2.2.1/2.2.2 of
  "FlashAttention优化Transformer显存与计算效率" (running max m / running sum l);
* invariants: rows of P sum to 1, identical keys average the visible V rows,
  causal row 0 copies V[0], uniform scores give lse = ln(#visible),
  translation invariance of the softmax (sum of dK over keys is 0);
* central finite differences of the forward for the backward;
* an independent library routine (torch's float64 CPU scaled_dot_product_attention
  and autograd);
* mutation checks: plausible mistakes planted in a copy of the oracle are caught.
"""
import json
import math
import os
import re

import numpy as np
import pytest
import torch

import oracle
from oracle import ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_form.json")


def _eval_expr(s: str) -> float:
    """Evaluate a closed-form expression with numbers, + - * / ( ) and ln()."""
    if not re.fullmatch(r"[0-9lnm\(\)\+\-\*/\. ]+", s):
        raise ValueError(f"unexpected token in {s!r}")
    return float(eval(s.replace("ln(", "math.log("), {"__builtins__": {}}, {"math": math}))


def _arr(x):
    return np.array([[_eval_expr(c) for c in row] for row in x], dtype=np.float64)


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ----------------------------------------------------------------------------- golden


@pytest.mark.parametrize("case_idx", [0, 1, 2])
def test_closed_form_cases(case_idx):
    case = json.load(open(GOLDEN))["cases"][case_idx]
    q = _arr(case["q"])[None, :, None, :]
    k = _arr(case["k"])[None, :, None, :]
    v = _arr(case["v"])[None, :, None, :]
    scale = _eval_expr(case["scale"])
    out, lse = oracle.attention_forward(q, k, v, causal=case["causal"], scale=scale)
    np.testing.assert_allclose(out[0, :, 0, :], _arr(case["out"]), rtol=0, atol=1e-12)
    exp_lse = np.array([_eval_expr(x) for x in case["lse"]])
    np.testing.assert_allclose(lse[0, 0], exp_lse, rtol=0, atol=1e-12)
    if "dout" in case:
        do = _arr(case["dout"])[None, :, None, :]
        dq, dk, dv = oracle.attention_backward(q, k, v, do, causal=case["causal"], scale=scale)
        np.testing.assert_allclose(dq[0, :, 0, :], _arr(case["dq"]), atol=1e-12)
        np.testing.assert_allclose(dk[0, :, 0, :], _arr(case["dk"]), atol=1e-12)
        np.testing.assert_allclose(dv[0, :, 0, :], _arr(case["dv"]), atol=1e-12)


# ------------------------------------------------------------------ blockwise restatement


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk,bq,bk", [(37, 37, 8, 5), (16, 16, 16, 16), (9, 23, 4, 7), (1, 50, 1, 8)])
def test_naive_equals_blockwise_online_softmax(causal, nq, nk, bq, bk):
    q = _rand((2, nq, 3, 5), 1) * 2.0
    k = _rand((2, nk, 3, 5), 2)
    v = _rand((2, nk, 3, 5), 3)
    o1, l1 = oracle.attention_forward(q, k, v, causal=causal, scale=0.7, row_block=6)
    o2, l2 = oracle.blockwise_forward(q, k, v, causal=causal, scale=0.7, block_q=bq, block_k=bk)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def test_row_blocking_is_invisible():
    q, k, v = _rand((1, 50, 2, 4), 4), _rand((1, 50, 2, 4), 5), _rand((1, 50, 2, 4), 6)
    do = _rand((1, 50, 2, 4), 7)
    a = oracle.attention_forward(q, k, v, causal=True, row_block=7)
    b = oracle.attention_forward(q, k, v, causal=True, row_block=1024)
    np.testing.assert_allclose(a[0], b[0], atol=1e-13)
    ga = oracle.attention_backward(q, k, v, do, causal=True, row_block=3)
    gb = oracle.attention_backward(q, k, v, do, causal=True, row_block=64)
    for x, y in zip(ga, gb):
        np.testing.assert_allclose(x, y, atol=1e-12)


# ----------------------------------------------------------------------------- invariants


@pytest.mark.parametrize("causal", [False, True])
def test_softmax_rows_sum_to_one(causal):
    s = _rand((20, 20), 8) * 10
    mask = ref.visible_mask(np.arange(20), 20, causal, 20)
    p, _ = ref.softmax_rows(s, mask)
    assert np.all(p >= 0)
    assert np.all(p[~mask] == 0)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys_average_visible_values(causal):
    N, d = 12, 6
    q = _rand((1, N, 1, d), 9)
    krow = _rand((d,), 10)
    k = np.broadcast_to(krow, (1, N, 1, d)).copy()
    v = _rand((1, N, 1, d), 11)
    out, lse = oracle.attention_forward(q, k, v, causal=causal, scale=0.3)
    for i in range(N):
        vis = i + 1 if causal else N
        np.testing.assert_allclose(out[0, i, 0], v[0, :vis, 0].mean(axis=0), atol=1e-13)
        s = 0.3 * q[0, i, 0] @ krow
        np.testing.assert_allclose(lse[0, 0, i], s + math.log(vis), atol=1e-13)


def test_causal_row_zero_copies_first_value():
    q, k, v = _rand((2, 9, 3, 4), 12), _rand((2, 9, 3, 4), 13), _rand((2, 9, 3, 4), 14)
    out, lse = oracle.attention_forward(q, k, v, causal=True)
    np.testing.assert_allclose(out[:, 0], v[:, 0], atol=1e-14)
    np.testing.assert_allclose(lse[:, :, 0], (q[:, 0] * k[:, 0]).sum(-1) / 2.0, atol=1e-14)


def test_constant_values_give_constant_output():
    q, k = _rand((1, 10, 2, 1), 15), _rand((1, 10, 2, 1), 16)
    v = np.full((1, 10, 2, 1), 3.25)
    for causal in (False, True):
        out, _ = oracle.attention_forward(q, k, v, causal=causal)
        np.testing.assert_allclose(out, 3.25, atol=1e-14)


def test_uniform_scores_give_log_count():
    q = np.zeros((1, 7, 1, 3))
    k, v = _rand((1, 7, 1, 3), 17), _rand((1, 7, 1, 3), 18)
    _, lse = oracle.attention_forward(q, k, v, causal=True)
    np.testing.assert_allclose(lse[0, 0], np.log(np.arange(1, 8)), atol=1e-15)
    _, lse = oracle.attention_forward(q, k, v, causal=False)
    np.testing.assert_allclose(lse[0, 0], math.log(7), atol=1e-15)


def test_bottom_right_alignment_for_short_queries():
    # 3 queries over 8 keys: query i sees keys 0 .. i+5.
    q, k, v = _rand((1, 3, 1, 4), 19), _rand((1, 8, 1, 4), 20), _rand((1, 8, 1, 4), 21)
    out, _ = oracle.attention_forward(q, k, v, causal=True)
    for i in range(3):
        o_i, _ = oracle.attention_forward(q[:, i:i + 1], k[:, :i + 6], v[:, :i + 6], causal=False)
        np.testing.assert_allclose(out[0, i], o_i[0, 0], atol=1e-14)


def test_translation_invariance_of_softmax_grad():
    # Adding the same vector to every key shifts a row's scores uniformly, which the
    # softmax ignores, so the gradient summed over keys vanishes (non-causal).
    q, k, v, do = (_rand((1, 11, 2, 5), s) for s in (22, 23, 24, 25))
    _, dk, _ = oracle.attention_backward(q, k, v, do, causal=False)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)


# ----------------------------------------------------------------- finite differences


def _loss(q, k, v, do, causal, scale):
    out, _ = oracle.attention_forward(q, k, v, causal=causal, scale=scale)
    return float(np.sum(out * do))


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_central_differences(causal):
    B, N, H, d = 1, 8, 1, 4
    q, k, v, do = (_rand((B, N, H, d), s) for s in (30, 31, 32, 33))
    scale = 0.5
    dq, dk, dv = oracle.attention_backward(q, k, v, do, causal=causal, scale=scale)
    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": q, "k": k, "v": v}
            args_m = {"q": q, "k": k, "v": v}
            args_p[name], args_m[name] = xp, xm
            num[idx] = (_loss(args_p["q"], args_p["k"], args_p["v"], do, causal, scale)
                        - _loss(args_m["q"], args_m["k"], args_m["v"], do, causal, scale)) / (2 * eps)
        err = np.max(np.abs(num - g)) / max(1e-12, np.max(np.abs(g)))
        assert err <= 1e-6, (name, err)


# --------------------------------------------------- independent library routine (torch)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("nq,nk", [(33, 33), (128, 128)])
def test_matches_torch_sdpa_float64(causal, nq, nk):
    B, H, d = 2, 3, 16
    q, k, v, do = (_rand(s, i) for s, i in (((B, nq, H, d), 40), ((B, nk, H, d), 41),
                                           ((B, nk, H, d), 42), ((B, nq, H, d), 43)))
    scale = 1 / 4
    out, lse = oracle.attention_forward(q, k, v, causal=causal, scale=scale)
    tq, tk, tv = (torch.tensor(x).permute(0, 2, 1, 3).requires_grad_(True) for x in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
    np.testing.assert_allclose(out, to.permute(0, 2, 1, 3).detach().numpy(), atol=1e-12)
    to.backward(torch.tensor(do).permute(0, 2, 1, 3))
    dq, dk, dv = oracle.attention_backward(q, k, v, do, causal=causal, scale=scale)
    for mine, theirs in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(mine, theirs.grad.permute(0, 2, 1, 3).numpy(), atol=1e-11)
    # LSE against torch.logsumexp of the masked scaled scores.
    s = torch.einsum("bhid,bhjd->bhij", tq.detach(), tk.detach()) * scale
    if causal:
        s = s.masked_fill(torch.ones(nq, nk, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), atol=1e-12)


# ------------------------------------------------------------------------ split / merge


@pytest.mark.parametrize("cuts", [[5], [1, 2, 30], [10, 20, 29, 40]])
def test_merge_of_key_splits_equals_full(cuts):
    q, k, v = _rand((2, 1, 3, 8), 50), _rand((2, 41, 3, 8), 51), _rand((2, 41, 3, 8), 52)
    full_o, full_l = oracle.attention_forward(q, k, v, causal=False)
    bounds = [0] + cuts + [41]
    parts = [oracle.attention_forward(q, k[:, a:b], v[:, a:b], causal=False)
             for a, b in zip(bounds[:-1], bounds[1:])]
    # out is [B, Nq, H, d] and lse is [B, H, Nq]: align lse to out's leading dims.
    o, l = oracle.merge_partials([p[0] for p in parts], [p[1].transpose(0, 2, 1) for p in parts])
    np.testing.assert_allclose(o, full_o, atol=1e-13)
    np.testing.assert_allclose(l, full_l.transpose(0, 2, 1), atol=1e-13)


def test_merge_ignores_empty_parts():
    o_parts = np.array([[[1.0, 2.0]], [[0.0, 0.0]]])
    lse_parts = np.array([[0.5], [-np.inf]])
    o, l = oracle.merge_partials(o_parts, lse_parts)
    np.testing.assert_allclose(o, [[1.0, 2.0]])
    np.testing.assert_allclose(l, [0.5])
    o, l = oracle.merge_partials(np.zeros((2, 1, 2)), np.full((2, 1), -np.inf))
    assert np.all(o == 0) and np.all(np.isneginf(l))


# ------------------------------------------------------------------------------ decode


def test_decode_first_step_returns_new_value():
    B, H, d, Ncap = 2, 3, 8, 16
    q, kn, vn = (_rand((B, 1, H, d), s) for s in (60, 61, 62))
    kc, vc = _rand((B, Ncap, H, d), 63), _rand((B, Ncap, H, d), 64)
    out, lse, kc2, vc2 = oracle.decode_step(q, kc, vc, np.zeros(B, int), kn, vn)
    np.testing.assert_allclose(out, vn, atol=1e-15)
    np.testing.assert_allclose(lse, (q[:, 0] * kn[:, 0]).sum(-1) / math.sqrt(d), atol=1e-14)
    np.testing.assert_array_equal(kc2[:, 0], kn[:, 0])
    np.testing.assert_array_equal(kc2[:, 1:], kc[:, 1:])


def test_decode_equals_last_row_of_causal_forward():
    B, H, d, Ncap = 2, 2, 8, 32
    L = np.array([5, 17])
    q, kn, vn = (_rand((B, 1, H, d), s) for s in (70, 71, 72))
    kc, vc = _rand((B, Ncap, H, d), 73), _rand((B, Ncap, H, d), 74)
    out, lse, kc2, vc2 = oracle.decode_step(q, kc, vc, L, kn, vn)
    for b in range(B):
        n = L[b] + 1
        qfull = _rand((1, n, H, d), 75)
        qfull[0, -1] = q[b, 0]
        o, l = oracle.attention_forward(qfull, kc2[b:b + 1, :n], vc2[b:b + 1, :n], causal=True)
        np.testing.assert_allclose(out[b, 0], o[0, -1], atol=1e-13)
        np.testing.assert_allclose(lse[b], l[0, :, -1], atol=1e-13)


def test_decode_ignores_rows_beyond_seqlen_and_handles_empty():
    B, H, d, Ncap = 3, 2, 4, 10
    q = _rand((B, 1, H, d), 80)
    kc, vc = _rand((B, Ncap, H, d), 81), _rand((B, Ncap, H, d), 82)
    L = np.array([0, 4, 10])
    out, lse, _, _ = oracle.decode_step(q, kc, vc, L)
    kc_b, vc_b = kc.copy(), vc.copy()
    kc_b[1, 4:] = 1e3
    vc_b[1, 4:] = -1e3
    out_b, lse_b, _, _ = oracle.decode_step(q, kc_b, vc_b, L)
    np.testing.assert_array_equal(out, out_b)
    np.testing.assert_array_equal(lse, lse_b)
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    with pytest.raises(ValueError):
        oracle.decode_step(q, kc, vc, np.array([0, 0, 10]), q, q)


def test_decode_sequence_replays_steps():
    B, H, d, Ncap, T = 2, 2, 4, 8, 5
    kc, vc = _rand((B, Ncap, H, d), 90), _rand((B, Ncap, H, d), 91)
    qs, ks, vs = (_rand((T, B, 1, H, d), s) for s in (92, 93, 94))
    outs, lses, kc2, vc2 = oracle.decode_sequence(qs, ks, vs, kc, vc, np.zeros(B, int))
    np.testing.assert_array_equal(kc2[:, :T], ks[:, :, 0].transpose(1, 0, 2, 3))
    np.testing.assert_array_equal(kc2[:, T:], kc[:, T:])
    for t in range(T):
        qf = _rand((B, t + 1, H, d), 95)
        qf[:, -1] = qs[t][:, 0]
        o, l = oracle.attention_forward(qf, kc2[:, :t + 1], vc2[:, :t + 1], causal=True)
        np.testing.assert_allclose(outs[t][:, 0], o[:, -1], atol=1e-13)


# ----------------------------------------------------------------------- mutations


def test_pins_catch_planted_mistakes(monkeypatch):
    """Plant plausible mistakes in the oracle (on the CPU) and check a pin fails."""
    q, k, v = _rand((1, 12, 1, 4), 100), _rand((1, 12, 1, 4), 101), _rand((1, 12, 1, 4), 102)

    # 1) off-by-one causal mask (j < i instead of j <= i): the causal row-0 pin fails.
    orig = ref.visible_mask
    monkeypatch.setattr(ref, "visible_mask",
                        lambda qp, nk, c, nqt: (np.arange(nk)[None] < np.asarray(qp)[:, None] + (nk - nqt))
                        if c else orig(qp, nk, c, nqt))
    out, _ = ref.attention_forward(q, k, v, causal=True)
    assert not np.allclose(out[:, 0], v[:, 0])
    monkeypatch.setattr(ref, "visible_mask", orig)

    # 2) scores without the scale: blockwise (unaffected) and naive disagree.
    orig_scores = ref.scores
    monkeypatch.setattr(ref, "scores", lambda qm, km, sc: qm @ km.T)
    o1, _ = ref.attention_forward(q, k, v, causal=False, scale=0.3)
    monkeypatch.setattr(ref, "scores", orig_scores)
    o2, _ = ref.blockwise_forward(q, k, v, causal=False, scale=0.3)
    assert not np.allclose(o1, o2, atol=1e-6)

    # 3) backward with the row-dot term dropped: the translation-invariance pin fails.
    do = _rand((1, 12, 1, 4), 103)
    _, dk_good, _ = ref.attention_backward(q, k, v, do)
    qm, km, vm, dom = q[0, :, 0], k[0, :, 0], v[0, :, 0], do[0, :, 0]
    p, _ = ref.softmax_rows(ref.scores(qm, km, 0.5), np.ones((12, 12), bool))
    dk_bad = 0.5 * (p * (dom @ vm.T)).T @ qm
    assert np.allclose(dk_good.sum(axis=1), 0, atol=1e-12)
    assert not np.allclose(dk_bad.sum(axis=0), 0, atol=1e-6)

    # 4) transposed value operand (P V^T) changes the output: torch pin would fail.
    out_good, _ = ref.attention_forward(q, k, v, causal=False)
    p_full, _ = ref.softmax_rows(ref.scores(qm, km, 0.5), np.ones((12, 12), bool))
    bad = p_full.T @ vm
    assert not np.allclose(out_good[0, :, 0], bad, atol=1e-6)
