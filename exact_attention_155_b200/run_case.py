"""Run one operation of the library on a synthetic workload a few times.

Meant for profilers (ncu) and quick timing: it launches only the library's own
kernels for the chosen op, on seeded N(0,1) bf16 inputs.

  python -m exact_attention_155_b200.run_case --op fwd --B 1 --H 32 --N 8192 --d 128 --causal 1
  python -m exact_attention_155_b200.run_case --op bwd --N 8192
  python -m exact_attention_155_b200.run_case --op decode --B 32 --H 16 --d 64 --N 2048
  python -m exact_attention_155_b200.run_case --op decode --B 32 --H 16 --d 64 --N 2048 --page-size 64
"""
from __future__ import annotations

import argparse
import math
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", choices=["fwd", "bwd", "decode"], required=True)
    ap.add_argument("--B", type=int, default=1)
    ap.add_argument("--H", type=int, default=32)
    ap.add_argument("--N", type=int, default=8192, help="sequence length (decode: cached rows)")
    ap.add_argument("--d", type=int, default=128)
    ap.add_argument("--causal", type=int, default=1)
    ap.add_argument("--reps", type=int, default=2)
    ap.add_argument("--page-size", type=int, default=0,
                    help="decode: >0 runs the paged cache (pages of this many rows at shuffled pool positions)")
    a = ap.parse_args(argv)

    import torch
    import exact_attention_155_b200 as fa
    from exact_attention_155_b200.inputs import attention_inputs, decode_inputs

    dev = torch.device("cuda", 0)
    scale = 1.0 / math.sqrt(a.d)
    if a.op in ("fwd", "bwd"):
        inp = attention_inputs(a.B, a.N, a.H, a.d, seed=4242, with_dout=(a.op == "bwd"))
        q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
        out, lse = fa.fwd(q, k, v, causal=bool(a.causal), scale=scale)
        if a.op == "fwd":
            for _ in range(a.reps - 1):
                fa.fwd(q, k, v, causal=bool(a.causal), scale=scale, out=out, lse=lse)
        else:
            do = inp["dout"].to(dev)
            ws = torch.empty(fa.bwd_workspace_size(a.B, a.H, a.N, a.d), dtype=torch.uint8, device=dev)
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
            for _ in range(a.reps):
                fa.bwd(q, k, v, out, do, lse, causal=bool(a.causal), scale=scale, dq=dq, dk=dk,
                       dv=dv, workspace=ws)
    else:
        kc, vc, qs, _, _ = decode_inputs(a.B, a.H, a.d, a.N, 1, seed=4243)
        kc, vc, q = kc.to(dev), vc.to(dev), qs[0].to(dev)
        seq = torch.full((a.B,), a.N, dtype=torch.int32, device=dev)
        if a.page_size > 0:
            if a.N % a.page_size:
                raise SystemExit("--N must be a multiple of --page-size")
            nb = a.N // a.page_size
            perm = torch.randperm(a.B * nb, generator=torch.Generator().manual_seed(1008)).to(dev)
            table = perm.view(a.B, nb).to(torch.int32)
            shape = (a.B * nb, a.page_size, a.H, a.d)
            kp = torch.empty(shape, dtype=torch.bfloat16, device=dev)
            vp = torch.empty_like(kp)
            kp[perm] = kc.view(shape)
            vp[perm] = vc.view(shape)
            for _ in range(a.reps):
                fa.decode_paged(q, kp, vp, table, seq, scale=scale)
        else:
            for _ in range(a.reps):
                fa.decode(q, kc, vc, seq, scale=scale)
    torch.cuda.synchronize()
    st = fa.device_status()
    if st[0] != 0:
        raise SystemExit(f"device status {st}")
    print("ok", a.op)


if __name__ == "__main__":
    main()
