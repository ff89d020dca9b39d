"""KV-cache decode parity against the float64 oracle, plus the device-side status
word (out-of-range cache length, forced pipeline timeout)."""
import numpy as np
import pytest
import torch

import exact_attention_155_b200 as fa
import oracle
from exact_attention_155_b200.inputs import DECODE_STEPS, DECODE_SWEEP, decode_inputs, seed_for, to_f64
from helpers import LSE_ATOL, OUT_ATOL

pytestmark = pytest.mark.gpu


def _cmp(out, lse, ref_o, ref_l):
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(o - ref_o)) <= OUT_ATOL
    fin = np.isfinite(ref_l)
    assert np.array_equal(np.isfinite(l), fin)
    if fin.any():
        assert np.max(np.abs(l[fin] - ref_l[fin])) <= LSE_ATOL


def test_decode_incremental_steps():
    c = DECODE_STEPS
    kc0, vc0, qs, ks, vs = decode_inputs(c["B"], c["H"], c["d"], c["Ncap"], c["steps"],
                                         seed_for(c["config_id"]))
    kc, vc = kc0.cuda(), vc0.cuda()
    scale = 1.0 / 8.0
    got = []
    for t in range(c["steps"]):
        seq = torch.full((c["B"],), t, dtype=torch.int32, device="cuda")
        o, l = fa.decode(qs[t].cuda(), kc, vc, seq, ks[t].cuda(), vs[t].cuda(), causal=True,
                         scale=scale)
        got.append((o.cpu(), l.cpu()))
    assert fa.device_status()[0] == 0
    ref_o, ref_l, ref_kc, ref_vc = oracle.decode_sequence(
        to_f64(qs), to_f64(ks), to_f64(vs), to_f64(kc0), to_f64(vc0), np.zeros(c["B"], int),
        scale=scale)
    for t, (o, l) in enumerate(got):
        _cmp(o, l, ref_o[t], ref_l[t])
    # The appended rows are copied bit for bit; the other rows are untouched.
    assert np.array_equal(to_f64(kc.cpu()), ref_kc)
    assert np.array_equal(to_f64(vc.cpu()), ref_vc)
    # Step 0 attends only its own new row: out = v_new exactly (up to bf16 output).
    assert torch.equal(got[0][0], vs[0])


def test_decode_full_cache_sweep():
    c = DECODE_SWEEP
    kc0, vc0, qs, _, _ = decode_inputs(c["B"], c["H"], c["d"], c["Ncap"], 1, seed_for(c["config_id"]))
    seq = torch.full((c["B"],), c["seqlen"], dtype=torch.int32, device="cuda")
    scale = 1.0 / 8.0
    o, l = fa.decode(qs[0].cuda(), kc0.cuda(), vc0.cuda(), seq, scale=scale)
    ref_o, ref_l, _, _ = oracle.decode_step(to_f64(qs[0]), to_f64(kc0), to_f64(vc0),
                                            np.full(c["B"], c["seqlen"]), scale=scale)
    _cmp(o.cpu(), l.cpu(), ref_o, ref_l)


@pytest.mark.parametrize("d", [64, 128])
def test_decode_mixed_lengths_and_edges(d):
    B, H, Ncap = 4, 3, 777
    kc0, vc0, qs, ks, vs = decode_inputs(B, H, d, Ncap, 1, 9100 + d)
    scale = 1.0 / np.sqrt(d)
    # With append: lengths 0 (attend only the new row), 5, Ncap-1 (fills the cache).
    seq_a = np.array([0, 5, Ncap - 1, 300])
    kc, vc = kc0.cuda(), vc0.cuda()
    o, l = fa.decode(qs[0].cuda(), kc, vc, torch.tensor(seq_a, dtype=torch.int32, device="cuda"),
                     ks[0].cuda(), vs[0].cuda(), scale=scale)
    ref_o, ref_l, rkc, rvc = oracle.decode_step(to_f64(qs[0]), to_f64(kc0), to_f64(vc0), seq_a,
                                                to_f64(ks[0]), to_f64(vs[0]), scale=scale)
    _cmp(o.cpu(), l.cpu(), ref_o, ref_l)
    assert np.array_equal(to_f64(kc.cpu()), rkc) and np.array_equal(to_f64(vc.cpu()), rvc)
    # Without append: length 0 gives out = 0 and lse = -inf; Ncap uses every row.
    seq_b = np.array([0, 7, Ncap, 1])
    o, l = fa.decode(qs[0].cuda(), kc0.cuda(), vc0.cuda(),
                     torch.tensor(seq_b, dtype=torch.int32, device="cuda"), scale=scale)
    ref_o, ref_l, _, _ = oracle.decode_step(to_f64(qs[0]), to_f64(kc0), to_f64(vc0), seq_b,
                                            scale=scale)
    _cmp(o.cpu(), l.cpu(), ref_o, ref_l)
    assert torch.all(o[0] == 0) and torch.all(torch.isneginf(l[0]))
    assert fa.device_status()[0] == 0


def test_decode_reports_full_cache_on_device():
    B, H, d, Ncap = 2, 2, 64, 64
    kc0, vc0, qs, ks, vs = decode_inputs(B, H, d, Ncap, 1, 9200)
    seq = torch.tensor([Ncap, 3], dtype=torch.int32, device="cuda")  # entry 0 is full
    kc = kc0.cuda()
    fa.decode(qs[0].cuda(), kc, vc0.cuda(), seq, ks[0].cuda(), vs[0].cuda(), scale=0.125)
    st, site, info = fa.device_status()
    assert st == 6 and info == 0
    assert torch.equal(kc[0].cpu(), kc0[0])  # nothing appended for the bad entry
    assert fa.device_status()[0] == 0        # reading clears the word


def test_bounded_wait_times_out_without_hanging():
    from exact_attention_155_b200 import ops
    ops.debug_timeout_probe(50_000_000)
    st, site, _ = fa.device_status()
    assert st == 5 and site == 0x7FF
    # The context stays usable afterwards.
    q = torch.randn(1, 64, 1, 64, device="cuda").to(torch.bfloat16)
    out, lse = fa.fwd(q, q, q)
    torch.cuda.synchronize()
    assert torch.isfinite(lse).all()
    assert fa.device_status()[0] == 0
