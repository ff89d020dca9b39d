"""Paged KV-cache decode (fa_decode_paged) against the oracle: shuffled pages in a
shared pool, appends landing in the right page, unused pages never touched, bad
block-table entries reported on the device."""
import numpy as np
import pytest
import torch

import exact_attention_155_b200 as fa
import oracle
from exact_attention_155_b200.inputs import bf16_randn, to_f64
from helpers import LSE_ATOL, OUT_ATOL

pytestmark = pytest.mark.gpu


def _pool(B, cap, H, d, P, seed, spare=5):
    """Seeded contiguous caches split into pages of P rows at shuffled pool positions;
    spare pages hold NaN so any read of them would show."""
    g = torch.Generator().manual_seed(seed)
    kc, vc = bf16_randn((B, cap, H, d), g), bf16_randn((B, cap, H, d), g)
    nb = cap // P
    n_pages = B * nb + spare
    perm = torch.randperm(n_pages, generator=g)
    kp = torch.full((n_pages, P, H, d), float("nan"), dtype=torch.bfloat16)
    vp = kp.clone()
    table = torch.empty((B, nb), dtype=torch.int32)
    for b in range(B):
        for j in range(nb):
            pid = int(perm[b * nb + j])
            kp[pid] = kc[b, j * P:(j + 1) * P]
            vp[pid] = vc[b, j * P:(j + 1) * P]
            table[b, j] = pid
    return kc, vc, kp, vp, table


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("P", [16, 64, 256])
def test_paged_decode_with_append(d, P):
    B, cap, H = 4, 1024, 4
    kc, vc, kp, vp, table = _pool(B, cap, H, d, P, 9700 + P + d)
    g = torch.Generator().manual_seed(9800 + P)
    q, kn, vn = (bf16_randn((B, 1, H, d), g) for _ in range(3))
    seq = torch.tensor([0, 1, 500, cap - 1], dtype=torch.int32)
    kp_d, vp_d = kp.cuda(), vp.cuda()
    out, lse = fa.decode_paged(q.cuda(), kp_d, vp_d, table.cuda(), seq.cuda(), kn.cuda(), vn.cuda(),
                               scale=d ** -0.5)
    torch.cuda.synchronize()
    assert fa.device_status()[0] == 0
    ro, rl, rkp, rvp = oracle.decode_step_paged(to_f64(q), to_f64(kp), to_f64(vp), table.numpy(),
                                                seq.numpy(), to_f64(kn), to_f64(vn), scale=d ** -0.5)
    got_o = out.float().cpu().numpy()
    assert np.isfinite(got_o).all()
    assert np.max(np.abs(got_o - ro)) <= OUT_ATOL
    assert np.max(np.abs(lse.cpu().numpy() - rl)) <= LSE_ATOL
    # The pages after the step: appended rows in place, everything else untouched,
    # spare pages still NaN.
    for got, ref in ((kp_d, rkp), (vp_d, rvp)):
        got = got.float().cpu().numpy()
        assert np.array_equal(np.isnan(got), np.isnan(ref))
        m = ~np.isnan(ref)
        assert np.array_equal(got[m], ref[m])


def test_paged_equals_contiguous_decode():
    """Paging is addressing only: same rows, same split, same arithmetic."""
    B, cap, H, d, P = 8, 2048, 16, 64, 64
    kc, vc, kp, vp, table = _pool(B, cap, H, d, P, 9900)
    g = torch.Generator().manual_seed(9901)
    q = bf16_randn((B, 1, H, d), g).cuda()
    seq = torch.tensor([2048, 1, 700, 1500, 0, 2047, 64, 65], dtype=torch.int32).cuda()
    o1, l1 = fa.decode(q, kc.cuda(), vc.cuda(), seq, scale=0.125)
    o2, l2 = fa.decode_paged(q, kp.cuda(), vp.cuda(), table.cuda(), seq, scale=0.125)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bad_block_table_entry_is_reported_not_read():
    B, cap, H, d, P = 2, 256, 2, 64, 16
    kc, vc, kp, vp, table = _pool(B, cap, H, d, P, 9950)
    table[1, 3] = kp.shape[0] + 7  # row 48..63 of sequence 1 point outside the pool
    g = torch.Generator().manual_seed(9951)
    q = bf16_randn((B, 1, H, d), g)
    seq = torch.tensor([100, 100], dtype=torch.int32)
    fa.device_status()
    out, lse = fa.decode_paged(q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), seq.cuda(), scale=0.125)
    st, site, info = fa.device_status()
    assert st == 6 and info == 1
    # Sequence 0 is unaffected.
    good = table.clone()
    good[1, 3] = 0
    ro, rl, _, _ = oracle.decode_step_paged(to_f64(q), to_f64(kp), to_f64(vp), good.numpy(),
                                            seq.numpy(), scale=0.125)
    assert np.max(np.abs(out[0].float().cpu().numpy() - ro[0])) <= OUT_ATOL
    assert np.isfinite(out.float().cpu().numpy()).all()
