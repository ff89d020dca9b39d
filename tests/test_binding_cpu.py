"""Host-side checks of the Python binding, on the CPU: every tensor the kernels will
touch is checked (dtype, contiguity or row layout, exact shape, device) before the
library is called, so a wrong output or workspace shape can never reach a kernel as an
out-of-bounds write; valid calls reach the C ABI with the sizes and strides the header
documents. The library is replaced by a recorder and the device type by "cpu" (a test
seam: the product path calls libfa.so on CUDA tensors)."""
import contextlib

import pytest
import torch

from exact_attention_155_b200 import ops


class _Recorder:
    """Stands in for libfa.so: records every entry point call and returns FA_OK."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if not name.startswith("fa_"):
            raise AttributeError(name)

        def fn(*args):
            self.calls.append((name, args))
            if name == "fa_bwd_workspace_size":
                return 4096
            if name in ("fa_decode_workspace_size",):
                return 0
            if name == "fa_last_error":
                return b""
            return 0
        return fn

    def names(self):
        return [n for n, _ in self.calls if not n.endswith("_size")]


@pytest.fixture
def lib(monkeypatch):
    rec = _Recorder()
    monkeypatch.setattr(ops, "_lib", rec)
    monkeypatch.setattr(ops, "_DEVICE_TYPE", "cpu")
    monkeypatch.setattr(ops, "_device_ctx", lambda dev: contextlib.nullcontext())
    monkeypatch.setattr(ops, "_stream", lambda stream=None: None)
    return rec


def _bf(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def _f32(*shape):
    return torch.zeros(shape, dtype=torch.float32)


def test_fwd_passes_sizes_and_allocates_outputs(lib):
    q = _bf(2, 256, 3, 64)
    out, lse = ops.fwd(q, q.clone(), q.clone(), causal=True)
    assert out.shape == q.shape and lse.shape == (2, 3, 256) and lse.dtype == torch.float32
    (name, args), = lib.calls
    assert name == "fa_fwd" and args[5:10] == (2, 3, 256, 64, 1)
    assert args[10] == pytest.approx(64 ** -0.5)


@pytest.mark.parametrize("bad", ["k_shape", "out_shape", "lse_shape", "lse_dtype", "q_strided", "q_dtype"])
def test_fwd_rejects_before_any_launch(lib, bad):
    B, N, H, d = 1, 128, 2, 64
    q, k, v = _bf(B, N, H, d), _bf(B, N, H, d), _bf(B, N, H, d)
    out, lse = None, None
    if bad == "k_shape":
        k = _bf(B, N - 1, H, d)
    elif bad == "out_shape":
        out = _bf(B, N, H, d // 2)
    elif bad == "lse_shape":
        lse = _f32(B, N, H)  # [B, N, H] instead of [B, H, N]
    elif bad == "lse_dtype":
        lse = torch.zeros((B, H, N), dtype=torch.bfloat16)
    elif bad == "q_strided":
        q = _bf(B, H, N, d).transpose(1, 2)
    else:
        q = q.float()
    with pytest.raises(ValueError):
        ops.fwd(q, k, v, out=out, lse=lse)
    assert lib.names() == []


@pytest.mark.parametrize("bad", ["dq_shape", "dv_dtype", "lse_shape", "dout_shape", "workspace_dtype"])
def test_bwd_rejects_before_any_launch(lib, bad):
    B, N, H, d = 1, 128, 2, 64
    t = {n: _bf(B, N, H, d) for n in ("q", "k", "v", "out", "dout")}
    lse = _f32(B, H, N)
    kw = {}
    if bad == "dq_shape":
        kw["dq"] = _bf(B, N, H, 2 * d)
    elif bad == "dv_dtype":
        kw["dv"] = _f32(B, N, H, d)
    elif bad == "lse_shape":
        lse = _f32(B, H, N + 1)
    elif bad == "dout_shape":
        t["dout"] = _bf(B, N, H + 1, d)
    else:
        kw["workspace"] = _f32(4096)  # sizes are counted in bytes: uint8 only
    with pytest.raises(ValueError):
        ops.bwd(t["q"], t["k"], t["v"], t["out"], t["dout"], lse, **kw)
    assert lib.names() == []


def test_bwd_passes_workspace_bytes(lib):
    B, N, H, d = 1, 128, 2, 64
    t = [_bf(B, N, H, d) for _ in range(5)]
    ws = torch.zeros(5000, dtype=torch.uint8)
    ops.bwd(*t, _f32(B, H, N), workspace=ws)
    (name, args), = [c for c in lib.calls if c[0] == "fa_bwd"]
    assert args[9:14] == (B, H, N, d, 0) and args[16] == 5000


def test_packed_qkv_reaches_the_abi_with_row_strides(lib):
    B, N, H, d = 2, 128, 4, 64
    qkv = _bf(B, N, 3, H, d)
    out, lse = ops.fwd_qkvpacked(qkv, causal=True, window=(64, 0))
    (name, args), = lib.calls
    assert name == "fa_fwd_ex"
    assert args[6:11] == (0, B, H, N, d)
    assert args[11:15] == (3 * H * d, 3 * H * d, 3 * H * d, H * d)  # q, k, v, out
    assert args[15:18] == (1, 64, 0)
    lib.calls.clear()
    dqkv = ops.bwd_qkvpacked(qkv, out, out.clone(), lse, causal=True)
    (name, args), = [c for c in lib.calls if c[0] == "fa_bwd_ex"]
    assert list(args[15]) == [3 * H * d] * 3 + [H * d] * 2 + [3 * H * d] * 3
    assert args[20] == 0  # deterministic off by default
    assert dqkv.shape == qkv.shape
    lib.calls.clear()
    ops.bwd_qkvpacked(qkv, out, out.clone(), lse, causal=True, deterministic=True)
    (name, args), = [c for c in lib.calls if c[0] == "fa_bwd_ex"]
    assert args[20] == 1


def test_packed_qkv_rejects_a_wrong_gradient_buffer(lib):
    qkv = _bf(1, 128, 3, 2, 64)
    out, lse = _bf(1, 128, 2, 64), _f32(1, 2, 128)
    with pytest.raises(ValueError):
        ops.bwd_qkvpacked(qkv, out, out, lse, dqkv=_bf(1, 128, 3, 2, 32))
    assert lib.names() == []


def test_varlen_layout_and_lse_shape(lib):
    total, H, d = 300, 2, 64
    cu = torch.tensor([0, 100, 300], dtype=torch.int32)
    q = _bf(total, H, d)
    out, lse = ops.fwd_ex(q, q.clone(), q.clone(), cu_seqlens=cu, max_seqlen=200, causal=True)
    assert lse.shape == (H, total)
    (name, args), = lib.calls
    assert args[6:11] == (total, 2, H, 200, d)
    with pytest.raises(ValueError):  # the dense LSE layout is wrong for a packed batch
        ops.fwd_ex(q, q, q, cu_seqlens=cu, max_seqlen=200, lse=_f32(2, H, 200))
    with pytest.raises(ValueError):
        ops.fwd_ex(q, q, q, cu_seqlens=cu.view(1, 3), max_seqlen=200)
    with pytest.raises(ValueError):
        ops.fwd_ex(q, q, q, cu_seqlens=cu)  # max_seqlen missing
    with pytest.raises(ValueError):
        ops.bwd_ex(q, q, q, out, out, lse, cu_seqlens=cu, max_seqlen=200, dk=_bf(total - 1, H, d))
    assert lib.names() == ["fa_fwd_ex"]


@pytest.mark.parametrize("bad", ["out", "lse", "k_new", "seqlens", "v_cache"])
def test_decode_rejects_before_any_launch(lib, bad):
    B, H, d, cap = 2, 4, 64, 256
    q = _bf(B, 1, H, d)
    kc, vc = _bf(B, cap, H, d), _bf(B, cap, H, d)
    seq = torch.zeros(B, dtype=torch.int32)
    kw = {}
    if bad == "out":
        kw["out"] = _bf(B, 2, H, d)
    elif bad == "lse":
        kw["lse"] = _f32(H, B)
    elif bad == "k_new":
        kw["k_new"], kw["v_new"] = _bf(B, 1, H, d), _bf(B, 2, H, d)
    elif bad == "seqlens":
        seq = torch.zeros(B + 1, dtype=torch.int32)
    else:
        vc = _bf(B, cap // 2, H, d)
    with pytest.raises(ValueError):
        ops.decode(q, kc, vc, seq, **kw)
    assert lib.names() == []


@pytest.mark.parametrize("bad", ["k_new", "out", "table", "v_pages"])
def test_decode_paged_rejects_before_any_launch(lib, bad):
    B, H, d = 2, 4, 64
    q = _bf(B, 1, H, d)
    kp, vp = _bf(8, 16, H, d), _bf(8, 16, H, d)
    table = torch.zeros((B, 4), dtype=torch.int32)
    seq = torch.zeros(B, dtype=torch.int32)
    kw = {}
    if bad == "k_new":
        kw["k_new"], kw["v_new"] = _bf(B, 1, H, 2 * d), _bf(B, 1, H, 2 * d)
    elif bad == "out":
        kw["out"] = _bf(B, 1, H + 1, d)
    elif bad == "table":
        table = torch.zeros((B + 1, 4), dtype=torch.int32)
    else:
        vp = _bf(8, 8, H, d)
    with pytest.raises(ValueError):
        ops.decode_paged(q, kp, vp, table, seq, **kw)
    assert lib.names() == []


def test_decode_paged_passes_the_page_geometry(lib):
    B, H, d = 2, 4, 64
    q = _bf(B, 1, H, d)
    ops.decode_paged(q, _bf(8, 16, H, d), _bf(8, 16, H, d), torch.zeros((B, 5), dtype=torch.int32),
                     torch.zeros(B, dtype=torch.int32))
    (name, args), = lib.calls
    assert name == "fa_decode_paged" and args[4:7] == (5, 16, 8) and args[12:15] == (B, H, d)


def test_merge_and_accumulate_reject_mismatched_buffers(lib):
    B, N, H, d = 1, 8, 2, 64
    with pytest.raises(ValueError):
        ops.merge_partials(_f32(B, N, H, d), _f32(B, H, N), _bf(B, N, H, d), _f32(B, H, N),
                           out=_bf(B, N, H, d // 2))
    with pytest.raises(ValueError):
        ops.merge_partials(_f32(B, N, H, d), _f32(B, N, H), _bf(B, N, H, d), _f32(B, H, N))
    with pytest.raises(ValueError):
        ops.accumulate(_f32(64), _bf(32))
    with pytest.raises(ValueError):
        ops.accumulate(_f32(64), None, out=_f32(64))
    assert lib.names() == []
    ops.accumulate(_f32(64), _bf(64))
    assert lib.names() == ["fa_accumulate"] and lib.calls[-1][1][3] == 64
