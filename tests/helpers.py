"""Shared helpers for the GPU parity tests: seeded inputs, oracle calls and the
tolerances the tests enforce.

Tolerances (stated for bf16 inputs against the float64 oracle):
  forward  max |out - ref| <= 2e-2 and max |lse - ref| <= 1e-3 (absolute);
  gradients max |g - ref| <= 5e-2 * max |ref|, per tensor; where the oracle's
  gradient is identically zero, max |g| <= 1e-5.
"""
import math

import numpy as np
import torch

import oracle
from exact_attention_155_b200.inputs import attention_inputs, to_f64

OUT_ATOL = 2e-2
LSE_ATOL = 1e-3
GRAD_REL = 5e-2
ZERO_GRAD_ATOL = 1e-5  # for gradients that are exactly zero in the oracle


def make_inputs(B, N, H, d, seed, q_mult=1.0, with_dout=True):
    inp = attention_inputs(B, N, H, d, seed, with_dout=with_dout)
    if q_mult != 1.0:
        inp["q"] = (inp["q"].float() * q_mult).to(torch.bfloat16)
    return inp


def check_fwd(out, lse, inp, causal, scale, heads=None, rows=None):
    """Compare GPU out/lse with the oracle on (optionally sampled) heads and rows."""
    q, k, v = (to_f64(inp[n]) for n in ("q", "k", "v"))
    ref_o, ref_l = oracle.attention_forward(q, k, v, causal=causal, scale=scale, heads=heads,
                                            rows=rows)
    got_o = out.detach().float().cpu().numpy().astype(np.float64)
    got_l = lse.detach().cpu().numpy().astype(np.float64)
    mask_o = ~np.isnan(ref_o)
    mask_l = ~np.isnan(ref_l)
    assert mask_o.any() and mask_l.any()
    err_o = np.max(np.abs(got_o[mask_o] - ref_o[mask_o]))
    err_l = np.max(np.abs(got_l[mask_l] - ref_l[mask_l]))
    assert np.isfinite(got_o[mask_o]).all() and np.isfinite(got_l[mask_l]).all()
    assert err_o <= OUT_ATOL, f"max |dout| = {err_o}"
    assert err_l <= LSE_ATOL, f"max |dlse| = {err_l}"
    return err_o, err_l


def check_grads(grads, inp, causal, scale, heads=None):
    q, k, v, do = (to_f64(inp[n]) for n in ("q", "k", "v", "dout"))
    refs = oracle.attention_backward(q, k, v, do, causal=causal, scale=scale, heads=heads)
    errs = {}
    for name, g, r in zip(("dq", "dk", "dv"), grads, refs):
        got = g.detach().float().cpu().numpy().astype(np.float64)
        m = ~np.isnan(r)
        assert m.any()
        assert np.isfinite(got[m]).all(), name
        err = np.max(np.abs(got[m] - r[m]))
        ref_max = np.max(np.abs(r[m]))
        if ref_max == 0.0:
            # The gradient vanishes identically (e.g. dq with a single visible key:
            # dS = P (dP - D) = 0). The relative bound is then empty; require the
            # cancellation to come out at fp32 rounding level instead.
            assert err <= ZERO_GRAD_ATOL, f"{name}: exact-zero gradient, got max |g| = {err}"
            errs[name] = err
            continue
        bound = GRAD_REL * ref_max
        errs[name] = err / ref_max
        assert err <= bound, f"{name}: max |d| = {err} > {bound}"
    return errs


def default_scale(d):
    return 1.0 / math.sqrt(d)
