"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory
(for instance a host runtime that reserved all device memory up front, or plugin
code with no access to the application's allocator). It must give the same
gradients as fa_bwd with a caller-provided workspace, call after call, although its
built-in scratch keeps the previous call's contents.

This file is collected last so that, if it fails, a run that stops at the first
failure has already run every other test.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import exact_attention_155_b200 as fa
from exact_attention_155_b200 import ops
from exact_attention_155_b200.inputs import attention_inputs
from helpers import GRAD_REL

pytestmark = pytest.mark.gpu


def _call_noalloc(lib, q, k, v, out, do, lse, causal, scale):
    B, N, H, d = q.shape
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    st = lib.fa_bwd_noalloc(*(ctypes.c_void_p(t.data_ptr()) for t in (q, k, v, out, do, lse, dq, dk, dv)),
                            B, H, N, d, int(causal), scale,
                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, lib.fa_last_error()
    return dq, dk, dv


@pytest.mark.parametrize("d,causal", [(128, True), (64, False)])
def test_noalloc_backward_matches_workspace_backward_twice(d, causal):
    lib = ops.load_library()
    B, N, H = 1, 700, 4
    scale = 1.0 / math.sqrt(d)
    inp = attention_inputs(B, N, H, d, seed=4321 + d)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "dout"))
    out, lse = fa.fwd(q, k, v, causal=causal, scale=scale)
    ref = fa.bwd(q, k, v, out, do, lse, causal=causal, scale=scale)
    for _ in range(2):  # the second call starts from the first call's leftover scratch
        got = _call_noalloc(lib, q, k, v, out, do, lse, causal, scale)
        torch.cuda.synchronize()
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            g64 = g.float().cpu().numpy().astype(np.float64)
            r64 = r.float().cpu().numpy().astype(np.float64)
            bound = GRAD_REL * np.max(np.abs(r64))
            assert np.max(np.abs(g64 - r64)) <= bound, name
        # dk and dv do not depend on reduction order: they match bit for bit.
        assert torch.equal(got[1], ref[1]) and torch.equal(got[2], ref[2])
    assert fa.device_status()[0] == 0


def test_noalloc_rejects_problems_larger_than_its_scratch():
    lib = ops.load_library()
    B, N, H, d = 1, 16384, 32, 128  # needs ~258 MiB of scratch, more than the 32 MiB built in
    assert lib.fa_bwd_workspace_size(B, H, N, d) > 32 * 1024 * 1024
    p = ctypes.c_void_p(0x10000)  # never dereferenced: the size check comes first
    st = lib.fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, B, H, N, d, 1, 0.1, ctypes.c_void_p(0))
    assert st == 4  # FA_ERR_WORKSPACE
    assert b"scratch" in lib.fa_last_error()
