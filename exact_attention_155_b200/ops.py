"""Python binding of libfa.so: argument marshalling only.

Every function here checks torch tensor metadata (device, dtype, contiguity,
shapes), allocates outputs and workspaces with torch (device memory is the only
thing PyTorch provides), and calls the C ABI declared in include/fa.h on the
current CUDA stream. All arithmetic runs in the library's CUDA kernels; there is
no CPU or PyTorch fallback: a missing library or an unsupported device raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

__all__ = ["FAError", "load_library", "fwd", "bwd", "fwd_ex", "bwd_ex", "fwd_qkvpacked",
           "bwd_qkvpacked", "decode", "decode_paged", "merge_partials", "accumulate", "bwd_workspace_size", "decode_workspace_size",
           "device_status", "debug_timeout_probe", "LIB_PATH", "declared_symbols"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa.so")

FA_OK = 0
STATUS_NAMES = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_CUDA",
                4: "FA_ERR_WORKSPACE", 5: "FA_ERR_TIMEOUT", 6: "FA_ERR_DEVICE_INPUT"}

_c_void_p = ctypes.c_void_p
_c_int = ctypes.c_int
_c_float = ctypes.c_float
_c_size_t = ctypes.c_size_t
_c_ll = ctypes.c_longlong

# name -> (restype, argtypes); mirrors include/fa.h
_SIGNATURES = {
    "fa_fwd": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                        _c_int, _c_int, _c_int, _c_int, _c_int, _c_float, _c_void_p]),
    "fa_fwd_ex": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                           _c_void_p, _c_int, _c_int, _c_int, _c_int, _c_int,
                           _c_ll, _c_ll, _c_ll, _c_ll, _c_int, _c_int, _c_int, _c_float,
                           _c_void_p]),
    "fa_bwd_ex": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                           _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_int,
                           _c_int, _c_int, ctypes.POINTER(_c_ll), _c_int, _c_int, _c_int,
                           _c_float, _c_int, _c_void_p, _c_size_t, _c_void_p]),
    "fa_bwd_workspace_size": (_c_size_t, [_c_int, _c_int, _c_int, _c_int]),
    "fa_bwd": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                        _c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int, _c_int,
                        _c_float, _c_void_p, _c_size_t, _c_void_p]),
    "fa_bwd_profiled": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                 _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_int,
                                 _c_int, _c_int, _c_int, _c_float, _c_void_p, _c_size_t,
                                 _c_void_p, _c_void_p, _c_void_p]),
    "fa_bwd_noalloc": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_int,
                                _c_int, _c_int, _c_int, _c_float, _c_void_p]),
    "fa_decode_workspace_size": (_c_size_t, [_c_int, _c_int, _c_int, _c_int]),
    "fa_decode": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                           _c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int, _c_int,
                           _c_float, _c_void_p, _c_size_t, _c_void_p]),
    "fa_decode_paged": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_int,
                                 _c_int, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                 _c_int, _c_int, _c_int, _c_int, _c_float, _c_void_p]),
    "fa_merge_partials": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int,
                                   _c_int, _c_int, _c_int, _c_void_p]),
    "fa_accumulate": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_ll, _c_void_p]),
    "fa_last_error": (ctypes.c_char_p, []),
    "fa_device_status": (_c_int, [_c_void_p, ctypes.POINTER(ctypes.c_uint),
                                  ctypes.POINTER(ctypes.c_uint)]),
    "fa_debug_timeout_probe": (_c_int, [ctypes.c_longlong, _c_void_p]),
    "fa_abi_version": (_c_int, []),
}


def declared_symbols():
    """Names of the C entry points this binding expects (those of include/fa.h)."""
    return sorted(_SIGNATURES)


class FAError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libfa.so (once) and attach the C signatures. Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"CUDA library not built: {path} is missing. Build it with "
            "`python -m exact_attention_155_b200.build` (or __graft_entry__.build()).")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status: int):
    if status != FA_OK:
        msg = load_library().fa_last_error()
        raise FAError(status, msg.decode() if msg else "")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _device_ctx(device):
    """Makes `device` current for the call (the library launches on the current device)."""
    return torch.cuda.device(device)


# Device type every tensor handed to the library must have.
_DEVICE_TYPE = "cuda"


def _on_device_type(t: torch.Tensor) -> bool:
    return t.is_cuda if _DEVICE_TYPE == "cuda" else t.device.type == _DEVICE_TYPE


def _require(t: torch.Tensor, name: str, dtype=torch.bfloat16, shape=None, device=None):
    """Checks a tensor the library will read or write: a contiguous tensor of `dtype` on
    the library's device type, and, when given, exactly `shape` and on `device` (the
    kernels index every buffer from the sizes alone, so a wrong shape or another GPU's
    buffer must never reach them). The passing case is one expression; the messages
    are built only on failure."""
    if (isinstance(t, torch.Tensor) and _on_device_type(t) and t.dtype == dtype and t.is_contiguous()
            and (shape is None or t.shape == shape) and (device is None or t.device == device)):
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not _on_device_type(t):
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} (got {t.dtype}); inputs and outputs share one dtype")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)} (got {tuple(t.shape)})")
    raise ValueError(f"{name} must be on {device} like the other operands (got {t.device})")


def _workspace(workspace, need: int, device):
    """The caller's workspace (uint8, contiguous, on `device`; the library checks its
    size) or a new one of `need` bytes."""
    if workspace is None:
        return torch.empty(max(need, 1), dtype=torch.uint8, device=device)
    _require(workspace, "workspace", torch.uint8, device=device)
    return workspace


def _scale(scale, d):
    return 1.0 / math.sqrt(d) if scale is None else float(scale)


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
        scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
        lse: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Exact attention forward. q, k, v: [B, N, H, d] bf16 CUDA tensors.

    Returns (out [B, N, H, d] bf16, lse [B, H, N] fp32). scale=None -> 1/sqrt(d).
    """
    _require(q, "q")
    if q.dim() != 4:
        raise ValueError(f"q must be [B, N, H, d] (got {tuple(q.shape)})")
    dev = q.device
    for name, t in (("k", k), ("v", v)):
        _require(t, name, shape=q.shape, device=dev)
    B, N, H, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    _require(out, "out", shape=q.shape, device=dev)
    _require(lse, "lse", torch.float32, shape=(B, H, N), device=dev)
    lib = load_library()
    with _device_ctx(dev):
        _check(lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, d,
                          int(bool(causal)), _scale(scale, d), _stream(stream)))
    return out, lse


def bwd_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(load_library().fa_bwd_workspace_size(B, H, N, d))


def bwd(q, k, v, out, dout, lse, causal: bool = False, scale: Optional[float] = None,
        dq=None, dk=None, dv=None, workspace=None, stream=None, main_events=None):
    """Attention backward by recomputation. Returns (dq, dk, dv), bf16 [B, N, H, d].

    main_events: optional (start, stop) torch.cuda.Event pair recorded around the main
    backward kernel (fa_bwd_profiled), for timing that kernel on its own stream.
    """
    _require(q, "q")
    if q.dim() != 4:
        raise ValueError(f"q must be [B, N, H, d] (got {tuple(q.shape)})")
    dev = q.device
    for name, t in (("k", k), ("v", v), ("out", out), ("dout", dout)):
        _require(t, name, shape=q.shape, device=dev)
    B, N, H, d = q.shape
    _require(lse, "lse", torch.float32, shape=(B, H, N), device=dev)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _require(t, name, shape=q.shape, device=dev)
    lib = load_library()
    workspace = _workspace(workspace, int(lib.fa_bwd_workspace_size(B, H, N, d)), dev)
    with _device_ctx(dev):
        if main_events is None:
            _check(lib.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse),
                              _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, int(bool(causal)),
                              _scale(scale, d), _ptr(workspace), workspace.numel(),
                              _stream(stream)))
        else:
            ev0, ev1 = main_events
            for ev in (ev0, ev1):
                if ev.cuda_event == 0:
                    ev.record()  # torch creates the CUDA event handle lazily
            _check(lib.fa_bwd_profiled(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout),
                                       _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d,
                                       int(bool(causal)), _scale(scale, d), _ptr(workspace),
                                       workspace.numel(), _stream(stream),
                                       ctypes.c_void_p(ev0.cuda_event), ctypes.c_void_p(ev1.cuda_event)))
    return dq, dk, dv


def _row_stride(t: torch.Tensor, name: str, varlen: bool, shape, device=None) -> int:
    """Elements between consecutive tokens of a [B, N, H, d] (or [total, H, d]) view
    whose (H, d) block is contiguous; raises for any other layout."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not _on_device_type(t):
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device} like the other operands (got {t.device})")
    if t.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be torch.bfloat16 (got {t.dtype}); inputs and outputs share one dtype")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)} (got {tuple(t.shape)})")
    H, d = shape[-2], shape[-1]
    st = t.stride()
    row = st[-3]
    if st[-1] != 1 or (H > 1 and st[-2] != d):
        raise ValueError(f"{name}: the (heads, head_dim) block of each row must be contiguous")
    if not varlen and shape[0] > 1 and st[0] != shape[1] * row:
        raise ValueError(f"{name}: batches must be N row strides apart")
    return int(row)


def _window(window):
    wl, wr = (-1, -1) if window is None else (int(window[0]), int(window[1]))
    return wl, wr


def _ex_layout(q, cu_seqlens, max_seqlen):
    """(varlen, B, N, H, d, total, shape) of an extended call from q and cu_seqlens."""
    varlen = cu_seqlens is not None
    if varlen:
        _require(cu_seqlens, "cu_seqlens", torch.int32, device=q.device)
        if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
            raise ValueError("cu_seqlens must be int32 [B + 1]")
        if max_seqlen is None:
            raise ValueError("max_seqlen is required with cu_seqlens")
        if q.dim() != 3:
            raise ValueError(f"q must be [total, H, d] with cu_seqlens (got {tuple(q.shape)})")
        total, H, d = q.shape
        B, N = cu_seqlens.numel() - 1, int(max_seqlen)
        return True, B, N, H, d, total, (total, H, d)
    if q.dim() != 4:
        raise ValueError(f"q must be [B, N, H, d] (got {tuple(q.shape)})")
    B, N, H, d = q.shape
    return False, B, N, H, d, 0, (B, N, H, d)


def fwd_ex(q, k, v, causal: bool = False, scale: Optional[float] = None, window=None,
           cu_seqlens: Optional[torch.Tensor] = None, max_seqlen: Optional[int] = None,
           out=None, lse=None, stream=None):
    """Forward with row strides, variable-length batches and a sliding window (fa_fwd_ex).

    Dense: q, k, v are [B, N, H, d] views whose (H, d) block is contiguous (for example
    slices of a packed [B, N, 3, H, d] tensor); lse is [B, H, N].
    Variable length: q, k, v are [total, H, d]; cu_seqlens int32 [B + 1] on the device;
    max_seqlen bounds every sequence length; lse is [H, total].
    window = (left, right): query i sees keys [i - left, i + right], -1 = unbounded;
    causal fixes right = 0. Returns (out, lse); out is contiguous unless given.
    """
    if not isinstance(q, torch.Tensor):
        raise TypeError("q must be a torch.Tensor")
    dev = q.device
    varlen, B, N, H, d, total, shape = _ex_layout(q, cu_seqlens, max_seqlen)
    rs = [_row_stride(t, n, varlen, shape, dev) for n, t in (("q", q), ("k", k), ("v", v))]
    if out is None:
        out = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    rs.append(_row_stride(out, "out", varlen, shape, dev))
    lse_shape = (H, total) if varlen else (B, H, N)
    if lse is None:
        lse = torch.empty(lse_shape, dtype=torch.float32, device=dev)
    _require(lse, "lse", torch.float32, shape=lse_shape, device=dev)
    wl, wr = _window(window)
    lib = load_library()
    with _device_ctx(dev):
        _check(lib.fa_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens),
                             total, B, H, N, d, rs[0], rs[1], rs[2], rs[3], int(bool(causal)),
                             wl, wr, _scale(scale, d), _stream(stream)))
    return out, lse


def bwd_ex(q, k, v, out, dout, lse, causal: bool = False, scale: Optional[float] = None,
           window=None, cu_seqlens: Optional[torch.Tensor] = None,
           max_seqlen: Optional[int] = None, dq=None, dk=None, dv=None, workspace=None,
           stream=None, deterministic: bool = False):
    """Backward of fwd_ex (fa_bwd_ex): same layouts and options. Returns (dq, dk, dv).

    deterministic=True selects the bitwise-repeatable backward (separate dK/dV and dQ
    kernels, no reductions into a shared accumulator); it is slower."""
    if not isinstance(q, torch.Tensor):
        raise TypeError("q must be a torch.Tensor")
    dev = q.device
    varlen, B, N, H, d, total, shape = _ex_layout(q, cu_seqlens, max_seqlen)
    dq = torch.empty(shape, dtype=torch.bfloat16, device=dev) if dq is None else dq
    dk = torch.empty(shape, dtype=torch.bfloat16, device=dev) if dk is None else dk
    dv = torch.empty(shape, dtype=torch.bfloat16, device=dev) if dv is None else dv
    names = (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout), ("dq", dq), ("dk", dk),
             ("dv", dv))
    rs = (_c_ll * 8)(*[_row_stride(t, n, varlen, shape, dev) for n, t in names])
    lse_shape = (H, total) if varlen else (B, H, N)
    _require(lse, "lse", torch.float32, shape=lse_shape, device=dev)
    wl, wr = _window(window)
    lib = load_library()
    workspace = _workspace(workspace, int(lib.fa_bwd_workspace_size(B, H, N, d)), dev)
    with _device_ctx(dev):
        _check(lib.fa_bwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse),
                             _ptr(dq), _ptr(dk), _ptr(dv), _ptr(cu_seqlens), total, B, H, N, d, rs,
                             int(bool(causal)), wl, wr, _scale(scale, d), int(bool(deterministic)),
                             _ptr(workspace), workspace.numel(), _stream(stream)))
    return dq, dk, dv


def fwd_qkvpacked(qkv, causal: bool = False, scale: Optional[float] = None, window=None,
                  stream=None):
    """Forward on a packed [B, N, 3, H, d] tensor (flash_attn_qkvpacked_func layout),
    read in place through row strides. Returns (out [B, N, H, d], lse [B, H, N])."""
    _require(qkv, "qkv")
    if qkv.dim() != 5 or qkv.shape[2] != 3:
        raise ValueError("qkv must be [B, N, 3, H, d]")
    return fwd_ex(qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2], causal=causal, scale=scale,
                  window=window, stream=stream)


def bwd_qkvpacked(qkv, out, dout, lse, causal: bool = False, scale: Optional[float] = None,
                  window=None, dqkv=None, stream=None, deterministic: bool = False):
    """Backward of fwd_qkvpacked; the gradient is written packed, [B, N, 3, H, d]."""
    _require(qkv, "qkv")
    if qkv.dim() != 5 or qkv.shape[2] != 3:
        raise ValueError("qkv must be [B, N, 3, H, d]")
    dqkv = torch.empty_like(qkv) if dqkv is None else dqkv
    _require(dqkv, "dqkv", shape=qkv.shape, device=qkv.device)
    bwd_ex(qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2], out, dout, lse, causal=causal, scale=scale,
           window=window, dq=dqkv[:, :, 0], dk=dqkv[:, :, 1], dv=dqkv[:, :, 2], stream=stream,
           deterministic=deterministic)
    return dqkv


def decode_workspace_size(B: int, H: int, Ncap: int, d: int) -> int:
    return int(load_library().fa_decode_workspace_size(B, H, Ncap, d))


def _decode_step_args(q, cache_seqlens, k_new, v_new, out, lse):
    """Checks shared by the decode calls; returns (B, H, d, out, lse)."""
    _require(q, "q")
    if q.dim() != 4 or q.shape[1] != 1:
        raise ValueError(f"q must be [B, 1, H, d] (got {tuple(q.shape)})")
    dev = q.device
    B, _, H, d = q.shape
    _require(cache_seqlens, "cache_seqlens", torch.int32, shape=(B,), device=dev)
    if (k_new is None) != (v_new is None):
        raise ValueError("k_new and v_new must be given together")
    if k_new is not None:
        _require(k_new, "k_new", shape=q.shape, device=dev)
        _require(v_new, "v_new", shape=q.shape, device=dev)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H), dtype=torch.float32, device=dev) if lse is None else lse
    _require(out, "out", shape=q.shape, device=dev)
    _require(lse, "lse", torch.float32, shape=(B, H), device=dev)
    return B, H, d, out, lse


def decode(q, k_cache, v_cache, cache_seqlens, k_new=None, v_new=None, causal: bool = True,
           scale: Optional[float] = None, out=None, lse=None, workspace=None, stream=None):
    """One KV-cache decode step (flash_attn_with_kvcache semantics).

    q: [B, 1, H, d]; k_cache, v_cache: [B, Ncap, H, d]; cache_seqlens: int32 [B] on the
    device (valid rows before the append). With k_new / v_new ([B, 1, H, d]) the row is
    appended at cache_seqlens[b]. Returns (out [B, 1, H, d] bf16, lse [B, H] fp32).
    """
    B, H, d, out, lse = _decode_step_args(q, cache_seqlens, k_new, v_new, out, lse)
    dev = q.device
    _require(k_cache, "k_cache", device=dev)
    if k_cache.dim() != 4 or k_cache.shape[0] != B or k_cache.shape[2] != H or k_cache.shape[3] != d:
        raise ValueError("q must be [B,1,H,d] and caches [B,Ncap,H,d]")
    _require(v_cache, "v_cache", shape=k_cache.shape, device=dev)
    Ncap = k_cache.shape[1]
    lib = load_library()
    need = int(lib.fa_decode_workspace_size(B, H, Ncap, d))
    if workspace is not None or need > 0:
        workspace = _workspace(workspace, need, dev)
    ws_bytes = 0 if workspace is None else workspace.numel()
    with _device_ctx(dev):
        _check(lib.fa_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_seqlens),
                             _ptr(k_new), _ptr(v_new), _ptr(out), _ptr(lse), B, H, Ncap, d,
                             int(bool(causal)), _scale(scale, d), _ptr(workspace), ws_bytes,
                             _stream(stream)))
    return out, lse


def decode_paged(q, k_pages, v_pages, block_table, cache_seqlens, k_new=None, v_new=None,
                 causal: bool = True, scale: Optional[float] = None, out=None, lse=None,
                 stream=None):
    """One decode step over a paged cache (fa_decode_paged).

    q: [B, 1, H, d]; k_pages, v_pages: [num_pages, page_size, H, d]; block_table: int32
    [B, max_blocks] on the device; cache_seqlens: int32 [B] on the device. Returns
    (out [B, 1, H, d] bf16, lse [B, H] fp32)."""
    B, H, d, out, lse = _decode_step_args(q, cache_seqlens, k_new, v_new, out, lse)
    dev = q.device
    _require(k_pages, "k_pages", device=dev)
    if k_pages.dim() != 4 or k_pages.shape[2] != H or k_pages.shape[3] != d:
        raise ValueError("q must be [B,1,H,d] and pages [num_pages,page_size,H,d]")
    _require(v_pages, "v_pages", shape=k_pages.shape, device=dev)
    _require(block_table, "block_table", torch.int32, device=dev)
    if block_table.dim() != 2 or block_table.shape[0] != B:
        raise ValueError("block_table must be int32 [B, max_blocks]")
    num_pages, page_size = k_pages.shape[0], k_pages.shape[1]
    lib = load_library()
    with _device_ctx(dev):
        _check(lib.fa_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table),
                                   block_table.shape[1], page_size, num_pages, _ptr(cache_seqlens),
                                   _ptr(k_new), _ptr(v_new), _ptr(out), _ptr(lse), B, H, d,
                                   int(bool(causal)), _scale(scale, d), _stream(stream)))
    return out, lse


def merge_partials(o_acc, lse_acc, o_part, lse_part, out=None, stream=None):
    """Fold a partial result (o_part bf16 [B, N, H, d], lse_part [B, H, N]) into the
    running one (o_acc fp32 [B, N, H, d], lse_acc [B, H, N]) in place (fa_merge_partials);
    optionally write the merged output as bf16 into `out`."""
    _require(o_part, "o_part")
    if o_part.dim() != 4:
        raise ValueError("o_part must be [B, N, H, d]")
    dev = o_part.device
    B, N, H, d = o_part.shape
    _require(o_acc, "o_acc", torch.float32, shape=o_part.shape, device=dev)
    _require(lse_acc, "lse_acc", torch.float32, shape=(B, H, N), device=dev)
    _require(lse_part, "lse_part", torch.float32, shape=(B, H, N), device=dev)
    if out is not None:
        _require(out, "out", shape=o_part.shape, device=dev)
    lib = load_library()
    with _device_ctx(dev):
        _check(lib.fa_merge_partials(_ptr(o_acc), _ptr(lse_acc), _ptr(o_part), _ptr(lse_part),
                                     _ptr(out), B, N, H, d, _stream(stream)))
    return o_acc, lse_acc


def accumulate(acc, part=None, out=None, stream=None):
    """acc (fp32) += part (bf16, same shape) in place when part is given, then write the
    sum as bf16 into `out` when given (fa_accumulate). Returns acc."""
    _require(acc, "acc", torch.float32)
    if part is None and out is None:
        raise ValueError("give part, out or both")
    for name, t in (("part", part), ("out", out)):
        if t is not None:
            _require(t, name, shape=acc.shape, device=acc.device)
    lib = load_library()
    with _device_ctx(acc.device):
        _check(lib.fa_accumulate(_ptr(acc), _ptr(part), _ptr(out), acc.numel(), _stream(stream)))
    return acc


def device_status(stream=None):
    """Synchronise the stream and return (status, site, info) from the device status word."""
    lib = load_library()
    site, info = ctypes.c_uint(0), ctypes.c_uint(0)
    st = lib.fa_device_status(_stream(stream), ctypes.byref(site), ctypes.byref(info))
    return st, site.value, info.value


def debug_timeout_probe(limit_cycles: int, stream=None):
    """Launch the diagnostic kernel whose wait must time out (see include/fa.h)."""
    _check(load_library().fa_debug_timeout_probe(int(limit_cycles), _stream(stream)))
