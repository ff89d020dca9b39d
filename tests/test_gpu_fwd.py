"""Forward parity: the CUDA kernel against the float64 oracle on seeded inputs."""
import math

import numpy as np
import pytest
import torch

import exact_attention_155_b200 as fa
from exact_attention_155_b200.inputs import WORKLOADS, seed_for
from helpers import check_fwd, default_scale, make_inputs

pytestmark = pytest.mark.gpu


def _run(inp, causal, scale):
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    out, lse = fa.fwd(q, k, v, causal=causal, scale=scale)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("name", ["tiny", "tiny_causal", "vit"])
def test_fwd_small_workloads(name):
    w = WORKLOADS[name]
    inp = make_inputs(w.B, w.N, w.H, w.d, seed_for(w.config_id), with_dout=False)
    out, lse = _run(inp, w.causal, w.scale)
    check_fwd(out, lse, inp, w.causal, w.scale)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 17, 127, 129, 200, 256, 1000])
def test_fwd_ragged_lengths(N, d, causal):
    inp = make_inputs(2, N, 3, d, 7000 + N + d, with_dout=False)
    out, lse = _run(inp, causal, default_scale(d))
    check_fwd(out, lse, inp, causal, default_scale(d))


@pytest.mark.parametrize("d", [64, 128])
def test_fwd_peaky_scores_exercise_rescale(d):
    # Scaled-up queries make the running max jump between key tiles.
    inp = make_inputs(1, 1024, 4, d, 7100 + d, q_mult=6.0, with_dout=False)
    for causal in (False, True):
        out, lse = _run(inp, causal, default_scale(d))
        check_fwd(out, lse, inp, causal, default_scale(d))


def test_fwd_many_heads_more_ctas_than_sms():
    inp = make_inputs(3, 384, 64, 64, 7200, with_dout=False)
    out, lse = _run(inp, True, 0.125)
    check_fwd(out, lse, inp, True, 0.125)


def test_fwd_prefill_full_size_sampled():
    """Causal prefill B=1, H=32, N=8192, d=128 in the launch the bench times; the
    oracle checks sampled heads and rows (tile edges, the first and last rows)."""
    w = WORKLOADS["prefill"]
    inp = make_inputs(w.B, w.N, w.H, w.d, seed_for(w.config_id), with_dout=False)
    out, lse = _run(inp, w.causal, w.scale)
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 255, 256, 4095, 4096, 8190, 8191],
                                     rng.choice(w.N, 200, replace=False)]))
    check_fwd(out, lse, inp, w.causal, w.scale, heads=[(0, 0), (0, 13), (0, 31)], rows=rows)
    # Properties that hold everywhere: finite outputs, and lse >= the diagonal score.
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


def test_fwd_is_deterministic():
    inp = make_inputs(1, 1000, 4, 128, 7300, with_dout=False)
    a = _run(inp, True, default_scale(128))
    b = _run(inp, True, default_scale(128))
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_fwd_rejects_bad_inputs():
    q = torch.zeros(1, 128, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        fa.fwd(q.float(), q, q)
    with pytest.raises(fa.FAError, match="UNSUPPORTED"):
        z = torch.zeros(1, 128, 2, 96, dtype=torch.bfloat16, device="cuda")
        fa.fwd(z, z, z)


def test_fwd_on_concurrent_streams_matches_one_stream():
    """The persistent forward takes work units from a per-launch ticket counter; calls
    in flight on different streams use different counters, so overlapping launches
    (many of them, wrapping the counter pool) give the same bits as one at a time."""
    shapes = [(1, 2048, 8, 128, True), (2, 777, 4, 64, False), (1, 4096, 4, 128, True)]
    inputs = [make_inputs(B, N, H, d, 7400 + i, with_dout=False) for i, (B, N, H, d, _) in enumerate(shapes)]
    dev = [tuple(inp[n].cuda() for n in ("q", "k", "v")) for inp in inputs]
    ref = []
    for (q, k, v), (_, _, _, d, causal) in zip(dev, shapes):
        ref.append(fa.fwd(q, k, v, causal=causal, scale=default_scale(d)))
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in shapes]
    outs = [[None] * 30 for _ in shapes]
    for rep in range(30):  # 90 launches: more than the pool of counters
        for i, ((q, k, v), (_, _, _, d, causal), s) in enumerate(zip(dev, shapes, streams)):
            with torch.cuda.stream(s):
                outs[i][rep] = fa.fwd(q, k, v, causal=causal, scale=default_scale(d))
    torch.cuda.synchronize()
    assert fa.device_status()[0] == 0
    for i in range(len(shapes)):
        for o, l in outs[i]:
            assert torch.equal(o, ref[i][0]) and torch.equal(l, ref[i][1])
