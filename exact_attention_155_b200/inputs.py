"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module draws random numbers and nothing else: it holds none of the
attention arithmetic, so both the CUDA path and the float64 oracle can be fed
from it without sharing any computation.

Recipe: a CPU ``torch.Generator`` seeded with ``1000 + config_id`` draws float32
N(0, 1) values in a fixed order (q, k, v, dout for the dense workloads; cache K,
cache V, then per step q, k_new, v_new for decode), rounded to bf16 (round to
nearest even). The oracle sees exactly these bf16 values upcast to float64.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

__all__ = ["Workload", "WORKLOADS", "bf16_randn", "attention_inputs", "decode_inputs",
           "to_f64", "seed_for"]


@dataclass(frozen=True)
class Workload:
    """One named workload: shapes, causality and which passes it exercises."""
    name: str
    config_id: int
    B: int
    H: int
    N: int
    d: int
    causal: bool
    passes: tuple
    scale: float


WORKLOADS = {
    # tiny correctness case, both masks, fwd + bwd
    "tiny": Workload("tiny", 1, 1, 2, 128, 64, False, ("fwd", "bwd"), 1.0 / 8.0),
    "tiny_causal": Workload("tiny_causal", 1, 1, 2, 128, 64, True, ("fwd", "bwd"), 1.0 / 8.0),
    # ViT / packed-QKV shape (batch 2, seq 1024, 16 heads, head dim 64), forward only
    "vit": Workload("vit", 2, 2, 16, 1024, 64, False, ("fwd",), 1.0 / 8.0),
    # Llama-7B-like causal prefill: 32 heads of dim 128 at 8192 tokens
    "prefill": Workload("prefill", 3, 1, 32, 8192, 128, True, ("fwd",), 1.0 / math.sqrt(128)),
    # long-context causal training step: 16384 tokens, forward + backward
    "train": Workload("train", 4, 1, 32, 16384, 128, True, ("fwd", "bwd"), 1.0 / math.sqrt(128)),
}

# KV-cache decode: (B, capacity 2048, 16 heads, dim 64), 100 appending steps,
# then a full-cache sweep at batch 32 without append.
DECODE_STEPS = dict(B=2, H=16, d=64, Ncap=2048, steps=100, config_id=5)
DECODE_SWEEP = dict(B=32, H=16, d=64, Ncap=2048, seqlen=2048, config_id=5)


# Sliding-window workload: long causal sequence, local window of 4096 keys.
WINDOW_BENCH = dict(B=1, H=32, N=16384, d=128, window=(4096, 0), seed=1007)
# Packed variable-length workload: the packing example of the long-text page (samples
# of 1-2K tokens packed instead of padded) stood in for by seeded lengths drawn
# uniformly from [512, 4096] until 32768 tokens are filled (the last one is cut).
VARLEN_BENCH = dict(total=32768, H=32, d=128, lo=512, hi=4096, seed=1006)


def packed_lengths(total: int, lo: int, hi: int, seed: int):
    """Seeded sequence lengths in [lo, hi] summing to exactly `total`."""
    g = torch.Generator().manual_seed(int(seed))
    lens = []
    left = total
    while left > 0:
        n = int(torch.randint(lo, hi + 1, (1,), generator=g))
        n = min(n, left)
        lens.append(n)
        left -= n
    return lens


def seed_for(config_id: int) -> int:
    return 1000 + int(config_id)


def bf16_randn(shape, gen: torch.Generator) -> torch.Tensor:
    """float32 N(0,1) from ``gen`` rounded to bf16 (CPU tensor)."""
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def attention_inputs(B, N, H, d, seed, with_dout=True, Nk=None):
    """q [B,N,H,d], k/v [B,Nk,H,d], dout [B,N,H,d] as contiguous CPU bf16 tensors."""
    g = torch.Generator().manual_seed(int(seed))
    nk = N if Nk is None else Nk
    out = {
        "q": bf16_randn((B, N, H, d), g),
        "k": bf16_randn((B, nk, H, d), g),
        "v": bf16_randn((B, nk, H, d), g),
    }
    if with_dout:
        out["dout"] = bf16_randn((B, N, H, d), g)
    return out


def decode_inputs(B, H, d, Ncap, steps, seed):
    """Cache K/V [B,Ncap,H,d] filled with N(0,1) and per-step q, k_new, v_new
    [steps, B, 1, H, d]; all CPU bf16."""
    g = torch.Generator().manual_seed(int(seed))
    k_cache = bf16_randn((B, Ncap, H, d), g)
    v_cache = bf16_randn((B, Ncap, H, d), g)
    qs, ks, vs = [], [], []
    for _ in range(steps):
        qs.append(bf16_randn((B, 1, H, d), g))
        ks.append(bf16_randn((B, 1, H, d), g))
        vs.append(bf16_randn((B, 1, H, d), g))
    if steps:
        return k_cache, v_cache, torch.stack(qs), torch.stack(ks), torch.stack(vs)
    empty = torch.empty((0, B, 1, H, d), dtype=torch.bfloat16)
    return k_cache, v_cache, empty, empty, empty


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact upcast of a (bf16) tensor to a float64 numpy array."""
    return t.detach().to("cpu").to(torch.float64).numpy()
