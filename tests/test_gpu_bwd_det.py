"""The deterministic backward (fa_bwd_ex with deterministic = 1: a dK/dV kernel per key
tile and a dQ kernel per query tile, each gradient element written once) against the
float64 oracle, and its bitwise repeatability."""
import numpy as np
import pytest
import torch

import exact_attention_155_b200 as fa
import oracle
from exact_attention_155_b200.inputs import WORKLOADS, bf16_randn, seed_for, to_f64
from helpers import GRAD_REL, ZERO_GRAD_ATOL, check_grads, default_scale, make_inputs

pytestmark = pytest.mark.gpu


def _run(inp, causal, scale, window=None):
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    out, lse = fa.fwd_ex(q, k, v, causal=causal, scale=scale, window=window)
    grads = fa.bwd_ex(q, k, v, out, do, lse, causal=causal, scale=scale, window=window,
                      deterministic=True)
    torch.cuda.synchronize()
    assert fa.device_status()[0] == 0
    return grads


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 17, 128, 129, 200, 640])
def test_det_bwd_ragged_lengths(N, d, causal):
    inp = make_inputs(1, N, 2, d, 8400 + N + d)
    check_grads(_run(inp, causal, default_scale(d)), inp, causal, default_scale(d))


@pytest.mark.parametrize("name", ["tiny", "tiny_causal"])
def test_det_bwd_tiny(name):
    w = WORKLOADS[name]
    inp = make_inputs(w.B, w.N, w.H, w.d, seed_for(w.config_id))
    check_grads(_run(inp, w.causal, w.scale), inp, w.causal, w.scale)


@pytest.mark.parametrize("window,causal", [((100, 0), True), ((200, 333), False), ((0, 0), False)])
def test_det_bwd_sliding_window(window, causal):
    d, N = 128, 777
    inp = make_inputs(1, N, 2, d, 8500 + window[0])
    q, k, v, do = (to_f64(inp[n]) for n in ("q", "k", "v", "dout"))
    refs = oracle.attention_backward(q, k, v, do, causal=causal, scale=default_scale(d),
                                     window_left=window[0], window_right=window[1])
    grads = _run(inp, causal, default_scale(d), window=window)
    for name, g, r in zip(("dq", "dk", "dv"), grads, refs):
        got = g.float().cpu().numpy().astype(np.float64)
        err, rmax = np.max(np.abs(got - r)), np.max(np.abs(r))
        assert err <= (ZERO_GRAD_ATOL if rmax == 0.0 else GRAD_REL * rmax), name


@pytest.mark.parametrize("causal", [False, True])
def test_det_bwd_varlen(causal):
    lens, H, d = [1, 127, 128, 129, 300, 0, 700, 5], 2, 128
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    total = int(cu[-1])
    g = torch.Generator().manual_seed(8600 + int(causal))
    q, k, v, do = (bf16_randn((total, H, d), g) for _ in range(4))
    sc = default_scale(d)
    cu_t = torch.from_numpy(cu).cuda()
    qc, kc, vc, doc = (t.cuda() for t in (q, k, v, do))
    out, lse = fa.fwd_ex(qc, kc, vc, causal=causal, scale=sc, cu_seqlens=cu_t, max_seqlen=max(lens))
    grads = fa.bwd_ex(qc, kc, vc, out, doc, lse, causal=causal, scale=sc, cu_seqlens=cu_t,
                      max_seqlen=max(lens), deterministic=True)
    torch.cuda.synchronize()
    assert fa.device_status()[0] == 0
    refs = oracle.attention_backward_varlen(*(to_f64(t) for t in (q, k, v, do)), cu, causal=causal,
                                            scale=sc)
    for name, gr, r in zip(("dq", "dk", "dv"), grads, refs):
        got = gr.float().cpu().numpy().astype(np.float64)
        err, rmax = np.max(np.abs(got - r)), np.max(np.abs(r))
        assert err <= GRAD_REL * rmax, name


def test_det_bwd_matches_the_fused_backward_and_repeats_bit_for_bit():
    inp = make_inputs(1, 1000, 4, 128, 8700)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    out, lse = fa.fwd(q, k, v, causal=True)
    a = fa.bwd_ex(q, k, v, out, do, lse, causal=True, deterministic=True)
    b = fa.bwd_ex(q, k, v, out, do, lse, causal=True, deterministic=True)
    fused = fa.bwd(q, k, v, out, do, lse, causal=True)
    torch.cuda.synchronize()
    for x, y, z in zip(a, b, fused):
        assert torch.equal(x, y)
        ref = z.float()
        assert (x.float() - ref).abs().max() <= 1e-2 * ref.abs().max()


def test_det_bwd_train_full_size_sampled():
    """Causal training workload B=1, H=32, N=16384, d=128; the oracle recomputes two
    whole heads."""
    w = WORKLOADS["train"]
    inp = make_inputs(w.B, w.N, w.H, w.d, seed_for(w.config_id))
    grads = _run(inp, w.causal, w.scale)
    check_grads(grads, inp, w.causal, w.scale, heads=[(0, 0), (0, 31)])
