"""Parity of the extended entry points (fa_fwd_ex / fa_bwd_ex) against the oracle:
packed QKV read through row strides, packed variable-length batches, sliding windows,
and their combination; device-side rejection of bad cu_seqlens."""
import numpy as np
import pytest
import torch

import exact_attention_155_b200 as fa
import oracle
from exact_attention_155_b200.inputs import bf16_randn, to_f64
from helpers import GRAD_REL, LSE_ATOL, OUT_ATOL, ZERO_GRAD_ATOL, check_fwd, check_grads, \
    default_scale, make_inputs

pytestmark = pytest.mark.gpu


def _cmp_out(out, lse, ref_o, ref_l):
    got_o = out.float().cpu().numpy().astype(np.float64)
    got_l = lse.cpu().numpy().astype(np.float64)
    assert np.isfinite(got_o).all() and np.isfinite(got_l).all()
    assert np.max(np.abs(got_o - ref_o)) <= OUT_ATOL
    assert np.max(np.abs(got_l - ref_l)) <= LSE_ATOL


def _cmp_grads(grads, refs):
    for name, g, r in zip(("dq", "dk", "dv"), grads, refs):
        got = g.float().cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all(), name
        err, rmax = np.max(np.abs(got - r)), np.max(np.abs(r))
        if rmax == 0.0:
            assert err <= ZERO_GRAD_ATOL, name
        else:
            assert err <= GRAD_REL * rmax, f"{name}: {err} > {GRAD_REL * rmax}"


def test_fwd_ex_dense_is_fwd():
    inp = make_inputs(2, 300, 3, 128, 9100, with_dout=False)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    a = fa.fwd(q, k, v, causal=True)
    b = fa.fwd_ex(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_qkvpacked_forward_and_backward(d, causal):
    B, N, H = 2, 333, 3
    inp = make_inputs(B, N, H, d, 9200 + d + int(causal))
    qkv = torch.stack([inp["q"], inp["k"], inp["v"]], dim=2).cuda()  # [B, N, 3, H, d]
    sc = default_scale(d)
    out, lse = fa.fwd_qkvpacked(qkv, causal=causal, scale=sc)
    do = inp["dout"].cuda()
    dqkv = fa.bwd_qkvpacked(qkv, out, do, lse, causal=causal, scale=sc)
    torch.cuda.synchronize()
    check_fwd(out, lse, inp, causal, sc)
    check_grads((dqkv[:, :, 0], dqkv[:, :, 1], dqkv[:, :, 2]), inp, causal, sc)


LENS = [1, 127, 128, 129, 300, 0, 700, 5]
# The packing example of the long-text ms-swift page: samples of 1024 and 2048 tokens
# packed into one 3072-token batch.
PAGE_PACKING = [1024, 2048]


@pytest.mark.parametrize("lens", [LENS, PAGE_PACKING], ids=["ragged", "page_packing_example"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_varlen_forward_and_backward(d, causal, lens):
    H = 2
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    total = int(cu[-1])
    g = torch.Generator().manual_seed(9300 + d + int(causal) + (0 if lens is LENS else 17))
    q, k, v, do = (bf16_randn((total, H, d), g) for _ in range(4))
    sc = default_scale(d)
    cu_t = torch.from_numpy(cu).cuda()
    qc, kc, vc, doc = (t.cuda() for t in (q, k, v, do))
    out, lse = fa.fwd_ex(qc, kc, vc, causal=causal, scale=sc, cu_seqlens=cu_t, max_seqlen=max(lens))
    grads = fa.bwd_ex(qc, kc, vc, out, doc, lse, causal=causal, scale=sc, cu_seqlens=cu_t,
                      max_seqlen=max(lens))
    torch.cuda.synchronize()
    assert fa.device_status()[0] == 0
    ref_o, ref_l = oracle.attention_forward_varlen(to_f64(q), to_f64(k), to_f64(v), cu,
                                                   causal=causal, scale=sc)
    _cmp_out(out, lse, ref_o, ref_l)
    refs = oracle.attention_backward_varlen(to_f64(q), to_f64(k), to_f64(v), to_f64(do), cu,
                                            causal=causal, scale=sc)
    _cmp_grads(grads, refs)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_varlen_many_short_sequences(d, causal):
    """60 sequences of 0-300 tokens and one of 1000: thousands of work units, most of
    them past the end of their (short or empty) sequence, spread over more units than
    SMs, so the persistent kernels skip units and take several each."""
    g = torch.Generator().manual_seed(9400 + d + int(causal))
    lens = [int(x) for x in torch.randint(0, 301, (60,), generator=g)]
    lens[7] = 0
    lens[33] = 0
    lens[20] = 1000
    H = 4
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    total = int(cu[-1])
    q, k, v, do = (bf16_randn((total, H, d), g) for _ in range(4))
    sc = default_scale(d)
    cu_t = torch.from_numpy(cu).cuda()
    qc, kc, vc, doc = (t.cuda() for t in (q, k, v, do))
    out, lse = fa.fwd_ex(qc, kc, vc, causal=causal, scale=sc, cu_seqlens=cu_t, max_seqlen=max(lens))
    grads = fa.bwd_ex(qc, kc, vc, out, doc, lse, causal=causal, scale=sc, cu_seqlens=cu_t,
                      max_seqlen=max(lens))
    torch.cuda.synchronize()
    assert fa.device_status()[0] == 0
    ref_o, ref_l = oracle.attention_forward_varlen(to_f64(q), to_f64(k), to_f64(v), cu,
                                                   causal=causal, scale=sc)
    _cmp_out(out, lse, ref_o, ref_l)
    refs = oracle.attention_backward_varlen(to_f64(q), to_f64(k), to_f64(v), to_f64(do), cu,
                                            causal=causal, scale=sc)
    _cmp_grads(grads, refs)


WINDOW_CASES = [(True, 64, 0), (True, 300, 0), (True, 0, 0), (False, 100, 50), (False, -1, 37),
                (False, 200, -1), (False, 129, 129)]


@pytest.mark.parametrize("causal,wl,wr", WINDOW_CASES)
@pytest.mark.parametrize("d", [64, 128])
def test_sliding_window_forward_and_backward(d, causal, wl, wr):
    B, N, H = 1, 1000, 2
    inp = make_inputs(B, N, H, d, 9400 + d + wl + 3 * wr)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    sc = default_scale(d)
    out, lse = fa.fwd_ex(q, k, v, causal=causal, scale=sc, window=(wl, wr))
    grads = fa.bwd_ex(q, k, v, out, do, lse, causal=causal, scale=sc, window=(wl, wr))
    torch.cuda.synchronize()
    qf, kf, vf, dof = (to_f64(inp[n]) for n in ("q", "k", "v", "dout"))
    ref_o, ref_l = oracle.attention_forward(qf, kf, vf, causal=causal, scale=sc, window_left=wl,
                                            window_right=wr)
    _cmp_out(out, lse, ref_o, ref_l)
    refs = oracle.attention_backward(qf, kf, vf, dof, causal=causal, scale=sc, window_left=wl,
                                     window_right=wr)
    _cmp_grads(grads, refs)


def test_window_varlen_strided_combined():
    """Packed [total, 3, H, d] storage read through strides, variable lengths, a causal
    sliding window, and gradients written into a packed [total, 3, H, d] buffer."""
    H, d, wl = 2, 128, 100
    lens = [260, 3, 513]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    total = int(cu[-1])
    g = torch.Generator().manual_seed(9500)
    qkv = bf16_randn((total, 3, H, d), g)
    do = bf16_randn((total, H, d), g)
    sc = default_scale(d)
    qkv_c, do_c, cu_t = qkv.cuda(), do.cuda(), torch.from_numpy(cu).cuda()
    q, k, v = qkv_c[:, 0], qkv_c[:, 1], qkv_c[:, 2]
    out, lse = fa.fwd_ex(q, k, v, causal=True, scale=sc, window=(wl, 0), cu_seqlens=cu_t,
                         max_seqlen=max(lens))
    dqkv = torch.empty_like(qkv_c)
    fa.bwd_ex(q, k, v, out, do_c, lse, causal=True, scale=sc, window=(wl, 0), cu_seqlens=cu_t,
              max_seqlen=max(lens), dq=dqkv[:, 0], dk=dqkv[:, 1], dv=dqkv[:, 2])
    torch.cuda.synchronize()
    qf, kf, vf = (to_f64(qkv[:, i]) for i in range(3))
    ref_o, ref_l = oracle.attention_forward_varlen(qf, kf, vf, cu, causal=True, scale=sc,
                                                   window_left=wl, window_right=0)
    _cmp_out(out, lse, ref_o, ref_l)
    refs = oracle.attention_backward_varlen(qf, kf, vf, to_f64(do), cu, causal=True, scale=sc,
                                            window_left=wl, window_right=0)
    _cmp_grads((dqkv[:, 0], dqkv[:, 1], dqkv[:, 2]), refs)


def test_bad_cu_seqlens_are_reported_on_the_device():
    """A decreasing offset pair and a sequence longer than max_seqlen: both are
    reported as FA_ERR_DEVICE_INPUT; the valid sequence is still computed."""
    H, d = 2, 64
    g = torch.Generator().manual_seed(9600)
    q, k, v = (bf16_randn((40, H, d), g).cuda() for _ in range(3))
    fa.device_status()  # clear
    for cu in ([0, 10, 5, 40], [0, 10, 40]):
        cu_t = torch.tensor(cu, dtype=torch.int32, device="cuda")
        out = torch.zeros_like(q)
        out, lse = fa.fwd_ex(q, k, v, causal=True, cu_seqlens=cu_t, max_seqlen=16, out=out)
        st, site, info = fa.device_status()
        assert st == 6, (cu, st)
        ref_o, _ = oracle.attention_forward_varlen(to_f64(q.cpu()[:10]), to_f64(k.cpu()[:10]),
                                                   to_f64(v.cpu()[:10]), [0, 10], causal=True,
                                                   scale=default_scale(d))
        got = out[:10].float().cpu().numpy()
        assert np.max(np.abs(got - ref_o)) <= OUT_ATOL


def test_window_bench_size_sampled():
    """The sliding-window workload bench.py times (B=1 H=32 N=16384 d=128, causal,
    window 4096), in the same launch; the oracle recomputes heads 0 and 31 (forward on
    sampled rows, backward on all rows of head 0)."""
    from exact_attention_155_b200.inputs import WINDOW_BENCH as wb
    inp = make_inputs(wb["B"], wb["N"], wb["H"], wb["d"], wb["seed"])
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    sc = default_scale(wb["d"])
    wl, wr = wb["window"]
    out, lse = fa.fwd_ex(q, k, v, causal=True, scale=sc, window=(wl, wr))
    grads = fa.bwd_ex(q, k, v, out, do, lse, causal=True, scale=sc, window=(wl, wr))
    torch.cuda.synchronize()
    rows = sorted(set(list(range(0, wb["N"], 97)) + list(range(wb["N"] - 130, wb["N"]))
                      + list(range(wl - 3, wl + 130))))
    qf, kf, vf, dof = (to_f64(inp[n]) for n in ("q", "k", "v", "dout"))
    ref_o, ref_l = oracle.attention_forward(qf, kf, vf, causal=True, scale=sc, heads=[(0, 0), (0, 31)],
                                            rows=rows, window_left=wl, window_right=wr)
    m = ~np.isnan(ref_o)
    got = out.float().cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got[m] - ref_o[m])) <= OUT_ATOL
    ml = ~np.isnan(ref_l)
    assert np.max(np.abs(lse.cpu().numpy()[ml] - ref_l[ml])) <= LSE_ATOL
    refs = oracle.attention_backward(qf, kf, vf, dof, causal=True, scale=sc, heads=[(0, 0)],
                                     window_left=wl, window_right=wr)
    for name, g, r in zip(("dq", "dk", "dv"), grads, refs):
        mm = ~np.isnan(r)
        gg = g.float().cpu().numpy().astype(np.float64)
        assert np.max(np.abs(gg[mm] - r[mm])) <= GRAD_REL * np.max(np.abs(r[mm])), name


def test_varlen_bench_size_sampled():
    """The packed variable-length workload bench.py times (32768 tokens, H=32, d=128,
    causal), in the same launch; the oracle recomputes heads 0 and 31 of every sequence."""
    from exact_attention_155_b200.inputs import VARLEN_BENCH as vb, packed_lengths
    lens = packed_lengths(vb["total"], vb["lo"], vb["hi"], vb["seed"])
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    g = torch.Generator().manual_seed(vb["seed"])
    q, k, v, do = (bf16_randn((vb["total"], vb["H"], vb["d"]), g) for _ in range(4))
    sc = default_scale(vb["d"])
    cu_t = torch.from_numpy(cu).cuda()
    qc, kc, vc, doc = (t.cuda() for t in (q, k, v, do))
    out, lse = fa.fwd_ex(qc, kc, vc, causal=True, scale=sc, cu_seqlens=cu_t, max_seqlen=max(lens))
    grads = fa.bwd_ex(qc, kc, vc, out, doc, lse, causal=True, scale=sc, cu_seqlens=cu_t,
                      max_seqlen=max(lens))
    torch.cuda.synchronize()
    hs = [0, vb["H"] - 1]
    sub = lambda t: to_f64(t[:, hs])
    ref_o, ref_l = oracle.attention_forward_varlen(sub(q), sub(k), sub(v), cu, causal=True, scale=sc)
    _cmp_out(out[:, hs], lse[hs], ref_o, ref_l)
    refs = oracle.attention_backward_varlen(sub(q), sub(k), sub(v), sub(do), cu, causal=True, scale=sc)
    _cmp_grads(tuple(gr[:, hs] for gr in grads), refs)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_flash_attn_func_autograd(d, causal):
    """The flash_attn-style entry point: out from the forward kernel, gradients from the
    backward kernel through torch.autograd, against the oracle."""
    B, N, H = 1, 300, 2
    inp = make_inputs(B, N, H, d, 9700 + d + int(causal))
    q, k, v = (inp[n].cuda().requires_grad_() for n in ("q", "k", "v"))
    do = inp["dout"].cuda()
    sc = default_scale(d)
    out = fa.flash_attn_func(q, k, v, causal=causal)
    out.backward(do)
    torch.cuda.synchronize()
    qf, kf, vf, dof = (to_f64(inp[n]) for n in ("q", "k", "v", "dout"))
    ref_o, _ = oracle.attention_forward(qf, kf, vf, causal=causal, scale=sc)
    assert np.max(np.abs(out.detach().float().cpu().numpy() - ref_o)) <= OUT_ATOL
    refs = oracle.attention_backward(qf, kf, vf, dof, causal=causal, scale=sc)
    _cmp_grads((q.grad, k.grad, v.grad), refs)
