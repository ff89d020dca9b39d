"""Backward parity: recomputation-based gradients against the float64 oracle."""
import numpy as np
import pytest
import torch

import exact_attention_155_b200 as fa
from exact_attention_155_b200.inputs import WORKLOADS, seed_for
from helpers import check_grads, default_scale, make_inputs

pytestmark = pytest.mark.gpu


def _run(inp, causal, scale):
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    out, lse = fa.fwd(q, k, v, causal=causal, scale=scale)
    grads = fa.bwd(q, k, v, out, do, lse, causal=causal, scale=scale)
    torch.cuda.synchronize()
    return grads


@pytest.mark.parametrize("name", ["tiny", "tiny_causal"])
def test_bwd_tiny(name):
    w = WORKLOADS[name]
    inp = make_inputs(w.B, w.N, w.H, w.d, seed_for(w.config_id))
    check_grads(_run(inp, w.causal, w.scale), inp, w.causal, w.scale)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 17, 129, 200, 384])
def test_bwd_ragged_lengths(N, d, causal):
    inp = make_inputs(1, N, 2, d, 8000 + N + d)
    check_grads(_run(inp, causal, default_scale(d)), inp, causal, default_scale(d))


def test_bwd_peaky_and_many_heads():
    inp = make_inputs(2, 512, 80, 64, 8100, q_mult=4.0)
    heads = [(0, 0), (1, 79), (0, 40)]
    check_grads(_run(inp, True, 0.125), inp, True, 0.125, heads=heads)


def test_bwd_train_full_size_sampled():
    """Causal training step B=1, H=32, N=16384, d=128: fwd + bwd in the launch the
    bench times; the oracle recomputes two whole heads."""
    w = WORKLOADS["train"]
    inp = make_inputs(w.B, w.N, w.H, w.d, seed_for(w.config_id))
    grads = _run(inp, w.causal, w.scale)
    check_grads(grads, inp, w.causal, w.scale, heads=[(0, 0), (0, 31)])
    for g in grads:
        assert torch.isfinite(g.float()).all()


def test_bwd_dk_dv_are_deterministic():
    inp = make_inputs(1, 640, 4, 128, 8200)
    a = _run(inp, True, default_scale(128))
    b = _run(inp, True, default_scale(128))
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    # dq is summed with fp32 reductions in an order that is not fixed; it must still agree to rounding.
    assert torch.allclose(a[0].float(), b[0].float(), atol=1e-2, rtol=0)


def test_bwd_ignores_workspace_contents_with_many_units_per_cta():
    """The persistent kernel's unit counter lives in the workspace and is reset by the
    call itself: a workspace full of 0xFF bytes (counter 0xFFFFFFFF, NaN accumulator)
    gives the oracle's gradients. 2 x 8 heads x 20 key tiles = 320 units, more than one
    per SM, so CTAs take units from the counter."""
    B, N, H, d = 2, 2560, 8, 128
    inp = make_inputs(B, N, H, d, 8300)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    sc = default_scale(d)
    out, lse = fa.fwd(q, k, v, causal=True, scale=sc)
    ws = torch.full((fa.bwd_workspace_size(B, H, N, d),), 0xFF, dtype=torch.uint8, device="cuda")
    grads = fa.bwd(q, k, v, out, do, lse, causal=True, scale=sc, workspace=ws)
    torch.cuda.synchronize()
    assert fa.device_status()[0] == 0
    check_grads(grads, inp, True, sc, heads=[(0, 0), (1, 7), (1, 3)])
    # Reusing the workspace (counter left at its final value) gives the same dk, dv bits.
    again = fa.bwd(q, k, v, out, do, lse, causal=True, scale=sc, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(grads[1], again[1]) and torch.equal(grads[2], again[2])
    assert torch.allclose(grads[0].float(), again[0].float(), atol=1e-2, rtol=0)


def test_bwd_on_two_streams_with_own_workspaces():
    """Two backward calls overlapping on two streams, each with its own workspace (and so
    its own unit counter), give the results of the same calls on one stream."""
    B, N, H, d = 1, 4096, 8, 128
    sc = default_scale(d)
    runs = []
    for seed in (8400, 8401):
        inp = make_inputs(B, N, H, d, seed)
        q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
        out, lse = fa.fwd(q, k, v, causal=True, scale=sc)
        runs.append((q, k, v, out, do, lse))
    torch.cuda.synchronize()
    serial = [fa.bwd(*r, causal=True, scale=sc) for r in runs]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    wss = [torch.empty(fa.bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda") for _ in streams]
    for s in streams:
        s.wait_stream(torch.cuda.current_stream())
    overlapped = []
    for r, s, ws in zip(runs, streams, wss):
        with torch.cuda.stream(s):
            overlapped.append(fa.bwd(*r, causal=True, scale=sc, workspace=ws, stream=s))
    torch.cuda.synchronize()
    assert fa.device_status()[0] == 0
    for a, b in zip(serial, overlapped):
        assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
        assert torch.allclose(a[0].float(), b[0].float(), atol=1e-2, rtol=0)
