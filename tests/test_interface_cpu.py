"""The flash_attn-style entry points (exact_attention_155_b200.interface) on the CPU: their
autograd wiring, argument mapping and refusals, with the binding calls they make replaced
by stand-ins that compute with the float64 oracle (a test seam: on a GPU they call the
CUDA library)."""
import numpy as np
import pytest
import torch

import oracle
from exact_attention_155_b200 import interface, ops


class _OracleOps:
    """Stand-ins for the binding calls the interface makes, recording their arguments."""

    def __init__(self):
        self.calls = []

    @staticmethod
    def _np(t):
        return t.detach().double().numpy()

    def fwd_ex(self, q, k, v, causal=False, scale=None, window=None, cu_seqlens=None,
               max_seqlen=None, **kw):
        self.calls.append(("fwd_ex", causal, scale, window, cu_seqlens is not None, max_seqlen))
        wl, wr = (-1, -1) if window is None else window
        if cu_seqlens is None:
            o, l = oracle.attention_forward(self._np(q), self._np(k), self._np(v), causal=causal,
                                            scale=scale, window_left=wl, window_right=wr)
        else:
            o, l = oracle.attention_forward_varlen(self._np(q), self._np(k), self._np(v),
                                                   cu_seqlens.numpy(), causal=causal, scale=scale,
                                                   window_left=wl, window_right=wr)
        return torch.from_numpy(o).to(q.dtype), torch.from_numpy(l).float()

    def bwd_ex(self, q, k, v, out, dout, lse, causal=False, scale=None, window=None,
               cu_seqlens=None, max_seqlen=None, deterministic=False, **kw):
        self.calls.append(("bwd_ex", causal, scale, window, dout.is_contiguous()))
        self.deterministic = deterministic
        assert dout.is_contiguous()
        wl, wr = (-1, -1) if window is None else window
        args = [self._np(t) for t in (q, k, v, dout)]
        if cu_seqlens is None:
            g = oracle.attention_backward(*args, causal=causal, scale=scale, window_left=wl,
                                          window_right=wr)
        else:
            g = oracle.attention_backward_varlen(*args, cu_seqlens.numpy(), causal=causal,
                                                 scale=scale, window_left=wl, window_right=wr)
        return tuple(torch.from_numpy(x).to(q.dtype) for x in g)

    def fwd_qkvpacked(self, qkv, causal=False, scale=None, window=None, **kw):
        self.calls.append(("fwd_qkvpacked", causal, scale, window))
        return self.fwd_ex(qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2], causal=causal, scale=scale,
                           window=window)

    def bwd_qkvpacked(self, qkv, out, dout, lse, causal=False, scale=None, window=None, **kw):
        self.calls.append(("bwd_qkvpacked", causal, scale, window))
        g = self.bwd_ex(qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2], out, dout, lse, causal=causal,
                        scale=scale, window=window)
        return torch.stack(g, dim=2)

    def decode(self, q, k_cache, v_cache, cache_seqlens, k_new=None, v_new=None, causal=True,
               scale=None, **kw):
        self.calls.append(("decode", tuple(cache_seqlens.tolist()), k_new is not None, scale))
        return q.clone(), torch.zeros(q.shape[0], q.shape[2])

    def decode_paged(self, q, k_pages, v_pages, block_table, cache_seqlens, k_new=None, v_new=None,
                     causal=True, scale=None, **kw):
        self.calls.append(("decode_paged", tuple(block_table.shape), scale))
        return q.clone(), torch.zeros(q.shape[0], q.shape[2])


@pytest.fixture
def fake(monkeypatch):
    f = _OracleOps()
    for name in ("fwd_ex", "bwd_ex", "fwd_qkvpacked", "bwd_qkvpacked", "decode", "decode_paged"):
        monkeypatch.setattr(ops, name, getattr(f, name))
    return f


def _qkv(B=1, N=10, H=2, d=4, seed=0):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn((B, N, H, d), generator=g, dtype=torch.float64).requires_grad_() for _ in range(3)]


@pytest.mark.parametrize("causal", [False, True])
def test_flash_attn_func_autograd_matches_the_oracle(fake, causal):
    q, k, v = _qkv(seed=1 + causal)
    out = interface.flash_attn_func(q, k, v, softmax_scale=0.4, causal=causal)
    g = torch.randn(out.shape, generator=torch.Generator().manual_seed(5), dtype=torch.float64)
    out.backward(g)
    ref_o, _ = oracle.attention_forward(*(t.detach().numpy() for t in (q, k, v)), causal=causal, scale=0.4)
    refs = oracle.attention_backward(*(t.detach().numpy() for t in (q, k, v)), g.numpy(),
                                     causal=causal, scale=0.4)
    np.testing.assert_allclose(out.detach().numpy(), ref_o, atol=1e-12)
    for t, r in zip((q, k, v), refs):
        np.testing.assert_allclose(t.grad.numpy(), r, atol=1e-12)
    assert [c[0] for c in fake.calls] == ["fwd_ex", "bwd_ex"]


def test_a_broadcast_output_gradient_reaches_the_kernel_dense(fake):
    q, k, v = _qkv(seed=3)
    out, lse = interface.flash_attn_func(q, k, v, causal=True, return_attn_probs=True)
    assert lse.shape == (1, 2, 10) and not lse.requires_grad
    out.sum().backward()  # autograd hands over an expanded (stride 0) gradient
    assert fake.calls[-1] == ("bwd_ex", True, None, None, True)
    ones = np.ones(out.shape)
    refs = oracle.attention_backward(*(t.detach().numpy() for t in (q, k, v)), ones, causal=True)
    np.testing.assert_allclose(q.grad.numpy(), refs[0], atol=1e-12)


@pytest.mark.parametrize("window_size,causal,expect", [
    ((-1, -1), False, None), ((-1, -1), True, None), ((-1, 0), True, None),
    ((4, 3), True, (4, 0)), ((4, 3), False, (4, 3)), ((-1, 2), False, (-1, 2))])
def test_window_size_maps_to_the_library_window(fake, window_size, causal, expect):
    q, k, v = _qkv(seed=4)
    interface.flash_attn_func(q, k, v, causal=causal, window_size=window_size)
    assert fake.calls[0][3] == expect


def test_packed_qkv_gradient_is_packed_and_matches(fake):
    g = torch.Generator().manual_seed(6)
    qkv = torch.randn((1, 9, 3, 2, 4), generator=g, dtype=torch.float64).requires_grad_()
    out = interface.flash_attn_qkvpacked_func(qkv, causal=True)
    out.backward(torch.ones_like(out))
    parts = [qkv.detach()[:, :, i].numpy() for i in range(3)]
    refs = oracle.attention_backward(*parts, np.ones(out.shape), causal=True)
    assert qkv.grad.shape == qkv.shape
    for i in range(3):
        np.testing.assert_allclose(qkv.grad[:, :, i].numpy(), refs[i], atol=1e-12)


def test_varlen_uses_one_packing(fake):
    cu = torch.tensor([0, 3, 10], dtype=torch.int32)
    g = torch.Generator().manual_seed(7)
    q, k, v = (torch.randn((10, 2, 4), generator=g, dtype=torch.float64).requires_grad_() for _ in range(3))
    out = interface.flash_attn_varlen_func(q, k, v, cu, cu, 7, 7, causal=True)
    out.backward(torch.ones_like(out))
    ref_o, _ = oracle.attention_forward_varlen(*(t.detach().numpy() for t in (q, k, v)), cu.numpy(),
                                               causal=True)
    np.testing.assert_allclose(out.detach().numpy(), ref_o, atol=1e-12)
    assert fake.calls[0] == ("fwd_ex", True, None, None, True, 7)
    # An equal copy of the offsets is the same packing.
    again = interface.flash_attn_varlen_func(q, k, v, cu, cu.clone(), 7, 7, causal=True)
    np.testing.assert_allclose(again.detach().numpy(), ref_o, atol=1e-12)
    with pytest.raises(NotImplementedError):
        interface.flash_attn_varlen_func(q, k, v, cu, torch.tensor([0, 4, 10], dtype=torch.int32), 7, 7)
    with pytest.raises(NotImplementedError):
        interface.flash_attn_varlen_func(q, k, v, cu, cu, 7, 8)


def test_dropout_is_refused_and_deterministic_reaches_the_backward(fake):
    q, k, v = _qkv()
    with pytest.raises(NotImplementedError):
        interface.flash_attn_func(q, k, v, dropout_p=0.1)
    for flag in (False, True):  # False is the pages' setting
        q.grad = None
        out = interface.flash_attn_func(q, k, v, deterministic=flag)
        out.sum().backward()
        assert fake.deterministic is flag
    assert [c[0] for c in fake.calls] == ["fwd_ex", "bwd_ex", "fwd_ex", "bwd_ex"]


def test_kvcache_step_routes_to_decode_and_paged_decode(fake):
    q = torch.zeros((2, 1, 3, 4), dtype=torch.float64)
    cache = torch.zeros((2, 16, 3, 4), dtype=torch.float64)
    out = interface.flash_attn_with_kvcache(q, cache, cache, k=q, v=q, cache_seqlens=5, softmax_scale=0.5)
    assert out.shape == q.shape
    assert fake.calls[-1] == ("decode", (5, 5), True, 0.5)
    out, lse = interface.flash_attn_with_kvcache(q, cache, cache, cache_seqlens=torch.tensor([1, 2], dtype=torch.int32),
                                                 block_table=torch.zeros((2, 4), dtype=torch.int32),
                                                 return_softmax_lse=True)
    assert fake.calls[-1] == ("decode_paged", (2, 4), None) and lse.shape == (2, 3)
    with pytest.raises(ValueError):
        interface.flash_attn_with_kvcache(q, cache, cache)


def test_block_size_hint_is_accepted_and_changes_nothing(fake):
    q, k, v = _qkv(seed=9)
    a = interface.flash_attn_func(q, k, v, causal=True, block_size=128)
    b = interface.flash_attn_func(q, k, v, causal=True)
    assert torch.equal(a, b)
    with pytest.raises(ValueError):
        interface.flash_attn_func(q, k, v, block_size=0)
