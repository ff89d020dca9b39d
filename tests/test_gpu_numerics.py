"""Accuracy of the FMA-pipe exp2 that replaces the MUFU exponential for a share of
the softmax elements, against exact exp2 (float64)."""
import numpy as np
import pytest
import torch

from exact_attention_155_b200 import ops

pytestmark = pytest.mark.gpu


def test_exp2_polynomial_relative_error():
    g = torch.Generator().manual_seed(11)
    x = torch.cat([torch.rand(200000, generator=g) * 108 - 100,   # [-100, 8]
                   torch.linspace(-2, 2, 4001),
                   torch.tensor([0.0, 0.5, -0.5, 1.0, -1.0, 8.0, -0.49999, 0.49999])]).float()
    y = ops.debug_exp2(x.cuda()).cpu().double().numpy()
    ref = np.exp2(x.double().numpy())
    rel = np.abs(y / ref - 1.0)
    # The cubic's own bound is 1.14e-4 (gen_exp2_poly.py); allow fp32 rounding on top.
    assert rel.max() <= 2e-4, rel.max()
    assert y[-8] == 1.0  # 2^0 is exact (constant term pinned to 1)


def test_exp2_polynomial_clamps_far_negative_inputs():
    x = torch.tensor([-126.0, -200.0, -1e30, float("-inf")]).float().cuda()
    y = ops.debug_exp2(x).cpu().numpy()
    assert np.all(y >= 0) and np.all(y <= 2.0 ** -125)
