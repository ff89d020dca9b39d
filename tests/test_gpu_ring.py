"""Ring attention pieces on one GPU: the LSE merge kernel against the oracle's merge,
the fp32 sum kernel of the backward, and the full ring schedule (forward and backward)
for 1, 2 and 4 shards emulated in one process (the shard exchange becomes indexing)
against the oracle's attention and gradients over the whole sequence."""
import numpy as np
import pytest
import torch

import exact_attention_155_b200 as fa
import oracle
from exact_attention_155_b200.inputs import bf16_randn, to_f64
from exact_attention_155_b200.ring import ring_attention_bwd_emulated, ring_attention_fwd_emulated
from helpers import LSE_ATOL, OUT_ATOL, check_fwd, check_grads, default_scale, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128])
def test_merge_kernel_matches_oracle_merge(d):
    B, N, H = 2, 77, 3
    g = torch.Generator().manual_seed(9970 + d)
    o1 = torch.randn((B, N, H, d), generator=g, dtype=torch.float32)
    o2 = bf16_randn((B, N, H, d), g)
    l1 = torch.randn((B, H, N), generator=g) * 3
    l2 = torch.randn((B, H, N), generator=g) * 3
    l1[0, 0, :5] = float("-inf")   # nothing merged yet on some rows
    l2[1, 2, 3:9] = float("-inf")  # an empty partial on others
    l1[1, 1, 10] = l2[1, 1, 10] = float("-inf")  # both empty
    # A row with nothing merged yet holds a zero running output, as the ring starts it.
    o1[torch.isneginf(l1).permute(0, 2, 1)] = 0.0
    o_acc, lse_acc = o1.cuda(), l1.cuda()
    out = torch.empty((B, N, H, d), dtype=torch.bfloat16, device="cuda")
    fa.ops.merge_partials(o_acc, lse_acc, o2.cuda(), l2.cuda(), out=out)
    torch.cuda.synchronize()
    # The oracle takes each LSE in the layout of its output rows: [B, N, H].
    ref_o, ref_l = oracle.merge_partials(
        np.stack([o1.numpy().astype(np.float64), to_f64(o2)]),
        np.stack([l1.numpy().transpose(0, 2, 1), l2.numpy().transpose(0, 2, 1)]).astype(np.float64))
    ref_l = ref_l.transpose(0, 2, 1)  # back to [B, H, N]
    got_o = o_acc.cpu().numpy()
    assert np.max(np.abs(got_o - ref_o)) <= 1e-5 * max(1.0, np.max(np.abs(ref_o)))
    got_l = lse_acc.cpu().numpy()
    fin = np.isfinite(ref_l)
    assert np.array_equal(np.isneginf(got_l), np.isneginf(ref_l))
    assert np.max(np.abs(got_l[fin] - ref_l[fin])) <= 1e-5
    assert torch.equal(out, o_acc.to(torch.bfloat16))


@pytest.mark.parametrize("world", [1, 2, 4])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_emulated_ring_matches_whole_sequence(world, causal, d):
    B, N, H = 1, 1024, 2
    inp = make_inputs(B, N, H, d, 9980 + world + d + int(causal), with_dout=False)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    sc = default_scale(d)
    out, lse = ring_attention_fwd_emulated(q, k, v, world, causal=causal, scale=sc)
    torch.cuda.synchronize()
    check_fwd(out, lse, inp, causal, sc)


def test_accumulate_kernel_is_exact():
    """fa_accumulate: one fp32 addition of an exactly converted bf16 term, and a
    round-to-nearest-even bf16 copy; both are fixed to the bit."""
    g = torch.Generator().manual_seed(9990)
    acc = torch.randn((3, 77, 5, 64), generator=g, dtype=torch.float32).cuda()
    part = bf16_randn((3, 77, 5, 64), g).cuda()
    ref = acc + part.float()
    out = torch.empty_like(part)
    fa.ops.accumulate(acc, part, out=out)
    torch.cuda.synchronize()
    assert torch.equal(acc, ref)
    assert torch.equal(out, ref.to(torch.bfloat16))
    out2 = torch.zeros_like(part)
    fa.ops.accumulate(acc, None, out=out2)  # copy only: the sum is unchanged
    torch.cuda.synchronize()
    assert torch.equal(acc, ref) and torch.equal(out2, out)
    with pytest.raises(ValueError):
        fa.ops.accumulate(acc)
    odd = torch.zeros(12, dtype=torch.float32, device="cuda")
    with pytest.raises(fa.FAError):
        fa.ops.accumulate(odd, torch.zeros(12, dtype=torch.bfloat16, device="cuda"))


@pytest.mark.parametrize("world", [1, 2, 4])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_emulated_ring_bwd_matches_whole_sequence(world, causal, d):
    """Ring backward for 1, 2 and 4 shards (the exchange emulated in one process): the
    recomputed backward of every visited shard pair with the whole rows' LSE and
    output, summed in fp32, against the oracle's gradients of the whole sequence."""
    B, N, H = 1, 1024, 2
    inp = make_inputs(B, N, H, d, 9990 + world + d + int(causal))
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    sc = default_scale(d)
    out, lse = ring_attention_fwd_emulated(q, k, v, world, causal=causal, scale=sc)
    grads = ring_attention_bwd_emulated(q, k, v, out, do, lse, world, causal=causal, scale=sc)
    torch.cuda.synchronize()
    check_grads(grads, inp, causal, sc)


@pytest.mark.parametrize("world", [1, 2, 4])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_emulated_zigzag_ring_matches_whole_sequence(world, causal, d):
    """The zigzag layout (rank r holds chunks r and 2R-1-r) for 1, 2 and 4 shards, the
    exchange emulated in one process: forward output and LSE, and the gradients, against
    the oracle over the whole sequence (given and returned in sequence order)."""
    B, N, H = 2, 1024, 2
    inp = make_inputs(B, N, H, d, 9995 + world + d + int(causal))
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    sc = default_scale(d)
    out, lse = ring_attention_fwd_emulated(q, k, v, world, causal=causal, scale=sc, layout="zigzag")
    grads = ring_attention_bwd_emulated(q, k, v, out, do, lse, world, causal=causal, scale=sc,
                                        layout="zigzag")
    torch.cuda.synchronize()
    check_fwd(out, lse, inp, causal, sc)
    check_grads(grads, inp, causal, sc)
