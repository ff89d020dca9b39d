"""C ABI checks that need no GPU: the library builds, loads and exports every entry
point include/fa.h declares; host-side argument validation returns the documented
status before anything touches a device."""
import ctypes
import math
import os
import re

import pytest

from exact_attention_155_b200 import build as fa_build
from exact_attention_155_b200 import ops

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "fa.h")

FA_OK, INVALID, UNSUPPORTED, CUDA, WORKSPACE = 0, 1, 2, 3, 4
P16 = ctypes.c_void_p(0x10000)   # fake, 16-byte aligned: never dereferenced on the host
P_ODD = ctypes.c_void_p(0x10008)  # 8-byte aligned only
NULL = None
S0 = ctypes.c_void_p(0)


def _header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return ops.load_library()


def test_header_and_binding_agree():
    assert _header_functions() == ops.declared_symbols()


def test_library_exports_every_declared_symbol(lib):
    for name in _header_functions():
        assert hasattr(lib, name), name
    assert lib.fa_abi_version() == 2


def test_bwd_workspace_size_is_pure_and_padded(lib):
    # dQ accumulator [B,H,Np,d] fp32 + two [B,H,Np] fp32 vectors, Np = roundup(N, 128),
    # + 256 bytes for the work-unit counter of the persistent kernel.
    for (B, H, N, d) in [(1, 2, 128, 64), (2, 3, 129, 128), (1, 32, 16384, 128)]:
        Np = (N + 127) // 128 * 128
        rows = B * H * Np
        r256 = lambda x: (x + 255) // 256 * 256
        expect = r256(rows * d * 4) + 2 * r256(rows * 4) + 256
        assert lib.fa_bwd_workspace_size(B, H, N, d) == expect
    assert lib.fa_bwd_workspace_size(1, 1, 128, 96) == 0
    assert lib.fa_bwd_workspace_size(0, 1, 128, 64) == 0


def _fwd(lib, q=P16, k=P16, v=P16, o=P16, lse=P16, B=1, H=1, N=128, d=64, causal=0, scale=0.125):
    return lib.fa_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, S0)


def test_fwd_argument_errors(lib):
    assert _fwd(lib, d=96) == UNSUPPORTED
    assert b"head dim" in lib.fa_last_error()
    assert _fwd(lib, N=-1) == INVALID
    assert _fwd(lib, scale=math.inf) == INVALID
    assert _fwd(lib, scale=math.nan) == INVALID
    assert _fwd(lib, q=NULL) == INVALID
    assert _fwd(lib, o=P_ODD) == INVALID
    assert b"aligned" in lib.fa_last_error()
    # Empty problems are a no-op, even with null pointers.
    assert _fwd(lib, q=NULL, k=NULL, v=NULL, o=NULL, lse=NULL, N=0) == FA_OK
    assert _fwd(lib, B=0) == FA_OK


def _bwd(lib, ws=P16, ws_bytes=1 << 40, d=64, N=128, dq=P16, scale=0.125):
    return lib.fa_bwd(P16, P16, P16, P16, P16, P16, dq, P16, P16, 1, 2, N, d, 0, scale, ws,
                      ws_bytes, S0)


def test_bwd_argument_errors(lib):
    assert _bwd(lib, d=32) == UNSUPPORTED
    assert _bwd(lib, dq=NULL) == INVALID
    assert _bwd(lib, dq=P_ODD) == INVALID
    assert _bwd(lib, ws=NULL) == WORKSPACE
    need = lib.fa_bwd_workspace_size(1, 2, 128, 64)
    assert _bwd(lib, ws_bytes=need - 1) == WORKSPACE
    assert b"workspace" in lib.fa_last_error()
    assert _bwd(lib, ws=ctypes.c_void_p(0x10010)) == INVALID  # not 256-byte aligned
    assert _bwd(lib, scale=math.inf) == INVALID


def _fwd_ex(lib, cu=NULL, total=0, B=1, H=2, N=128, d=64, rs=(128, 128, 128, 128), causal=0,
            wl=-1, wr=-1, scale=0.125, q=P16):
    return lib.fa_fwd_ex(q, P16, P16, P16, P16, cu, total, B, H, N, d, *rs, causal, wl, wr, scale,
                         NULL)


def test_fwd_ex_argument_errors(lib):
    # Row strides: a multiple of 8 elements and at least H*d.
    assert _fwd_ex(lib, rs=(128, 128, 120, 128)) == INVALID
    assert b"stride" in lib.fa_last_error()
    assert _fwd_ex(lib, rs=(132, 128, 128, 128)) == INVALID
    # Window edges: >= 0 or -1; causal allows only a right edge of 0 or -1.
    assert _fwd_ex(lib, wl=-2) == INVALID
    assert _fwd_ex(lib, causal=1, wr=5) == INVALID
    assert b"window_right" in lib.fa_last_error()
    assert _fwd_ex(lib, d=80) == UNSUPPORTED
    assert _fwd_ex(lib, q=NULL) == INVALID
    assert _fwd_ex(lib, scale=math.nan) == INVALID
    # A packed batch with no tokens, or no sequences, is a no-op.
    assert _fwd_ex(lib, cu=P16, total=0) == FA_OK
    assert _fwd_ex(lib, B=0) == FA_OK


def test_bwd_ex_argument_errors(lib):
    rs8 = (ctypes.c_longlong * 8)(*([128] * 8))

    def call(rs=rs8, ws=P16, ws_bytes=1 << 30, wr=-1, causal=0, det=0):
        return lib.fa_bwd_ex(P16, P16, P16, P16, P16, P16, P16, P16, P16, NULL, 0, 1, 2, 128, 64,
                             rs, causal, -1, wr, 0.125, det, ws, ws_bytes, NULL)

    for det in (0, 1):  # the deterministic backward takes the same checks
        assert call(rs=None, det=det) == INVALID
        bad = (ctypes.c_longlong * 8)(*([128] * 7 + [100]))
        assert call(rs=bad, det=det) == INVALID
        assert call(causal=1, wr=3, det=det) == INVALID
        assert call(ws=NULL, det=det) == WORKSPACE


def test_decode_paged_argument_errors(lib):
    def call(page_size=64, max_blocks=4, num_pages=8, table=P16, d=64, B=2, kn=NULL, vn=NULL):
        return lib.fa_decode_paged(P16, P16, P16, table, max_blocks, page_size, num_pages, P16, kn, vn,
                                   P16, NULL, B, 2, d, 1, 0.125, NULL)
    assert call(page_size=48) == INVALID  # not a power of two
    assert b"power of two" in lib.fa_last_error()
    assert call(page_size=0) == INVALID
    assert call(max_blocks=0) == INVALID
    assert call(num_pages=0) == INVALID
    assert call(table=NULL) == INVALID
    assert call(kn=P16) == INVALID  # k_new without v_new
    assert call(d=96) == UNSUPPORTED
    assert call(B=0) == FA_OK


def test_merge_partials_argument_errors(lib):
    def call(o=P16, l=P16, op=P16, lp=P16, out=NULL, d=64, N=8):
        return lib.fa_merge_partials(o, l, op, lp, out, 1, N, 2, d, NULL)
    assert call(d=80) == UNSUPPORTED
    assert call(o=NULL) == INVALID
    assert call(out=P_ODD) == INVALID
    assert call(N=0) == FA_OK


def test_accumulate_argument_errors(lib):
    def call(acc=P16, part=P16, out=NULL, n=64):
        return lib.fa_accumulate(acc, part, out, n, NULL)
    assert call(n=-8) == INVALID
    assert call(acc=NULL) == INVALID
    assert call(part=NULL, out=NULL) == INVALID
    assert b"both NULL" in lib.fa_last_error()
    assert call(n=60) == INVALID
    assert b"multiple of 8" in lib.fa_last_error()
    assert call(part=P_ODD) == INVALID
    assert call(out=P_ODD) == INVALID
    assert call(acc=P_ODD, part=NULL, out=P16) == INVALID
    # Nothing to add: a no-op, even with null pointers.
    assert call(acc=NULL, part=NULL, n=0) == FA_OK


def _dec(lib, q=P16, kn=NULL, vn=NULL, seq=P16, Ncap=2048, d=64, B=2):
    return lib.fa_decode(q, P16, P16, seq, kn, vn, P16, NULL, B, 16, Ncap, d, 1, 0.125, NULL, 0, S0)


def test_decode_argument_errors(lib):
    assert _dec(lib, d=80) == UNSUPPORTED
    assert _dec(lib, Ncap=0) == INVALID
    assert _dec(lib, kn=P16, vn=NULL) == INVALID
    assert b"both" in lib.fa_last_error()
    assert _dec(lib, q=P_ODD) == INVALID
    assert _dec(lib, seq=NULL) == INVALID
    assert _dec(lib, B=0) == FA_OK


def test_decode_needs_no_workspace(lib):
    # Split partials are combined inside a thread-block cluster, on chip.
    for args in [(32, 16, 2048, 64), (1, 1, 16, 64), (2, 16, 2048, 128)]:
        assert lib.fa_decode_workspace_size(*args) == 0


def test_calls_without_a_gpu_report_an_error_not_a_crash(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st = _fwd(lib)
    assert st in (CUDA, UNSUPPORTED)
    assert lib.fa_last_error()


def test_binding_raises_when_library_missing(tmp_path):
    saved = ops._lib
    ops._lib = None
    try:
        with pytest.raises(RuntimeError, match="not built"):
            ops.load_library(str(tmp_path / "missing.so"))
    finally:
        ops._lib = saved
