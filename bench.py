#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200.

One step = the long-context causal training step: fused forward (O and LSE) plus
the recompute backward (dQ, dK, dV) at B=1, H=32, N=16384, d=128, bf16, on
synthetic N(0,1) inputs already resident in HBM. The metric is attention TFLOP/s
with the algorithmic count 4*B*H*N^2*d/2 for the causal forward and 2.5x that for
the backward. The same JSON line also reports, measured in the same run:
  * "roofline": the backward main kernel (the step's dominant kernel) timed with
    CUDA events on its launch stream inside the timed region;
  * "e2e": the step through the public API from pinned host buffers, with the
    host->device copies of q, k, v, dout and the device->host copies of out, lse,
    dq, dk, dv inside the timed region;
  * "parts": the causal prefill forward (B=1, H=32, N=8192, d=128) and the
    KV-cache decode sweep (B=32, H=16, d=64, 2048 cached rows) with their own
    rooflines, and the per-step latency of the 100-step incremental decode;
  * "cpu_baseline": the float64 CPU oracle on a bounded sample of the same step.

Multi-GPU: every rank runs an independent replica (the path has no exchange
step); value is the sum over ranks divided by the slowest rank's time.

--impl reference times the float64 oracle itself (the only reference this
method has) on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import itertools
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention TFLOP/s fwd/bwd (causal, bf16) and decode GB/s; % of B200 roofline"
WORKLOAD = dict(name="train", B=1, H=32, N=16384, d=128, causal=True)
PREFILL = dict(B=1, H=32, N=8192, d=128, causal=True)
SWEEP = dict(B=32, H=16, d=64, Ncap=2048, seqlen=2048)
STEPS5 = dict(B=2, H=16, d=64, Ncap=2048, steps=100)
TINY = dict(B=1, H=2, N=128, d=64)
VIT = dict(B=2, H=16, N=1024, d=64)


# Nominal B200 figures the targets are stated against (dense bf16, HBM3e): reported
# beside the measured-peak fractions.
NOMINAL_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 8000.0

# DRAM bytes per launch of the backward main kernel from an ncu capture of the training
# workload, valid only for the kernel source it was taken on (sha256 of csrc/bwd.cuh);
# null otherwise.
BWD_TRAFFIC = {"src_sha256": "0d3a88e3527275458e9d5b8bd589d935486a2fd3e2fc10c2e700e594ad897658",
               "bytes_per_launch": 837.20e6 + 518.84e6}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def fwd_flops(B, H, N, d, causal):
    f = 4.0 * B * H * N * N * d
    return f / 2 if causal else f


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), tf_burst=float(p["bf16_tflops"]),
                    tf_sustained=float(p["bf16_tflops_sustained"]), source="measured")
    except Exception:
        return dict(hbm=6650.0, tf_burst=1590.0, tf_sustained=1400.0, source="fallback")


def src_sha(rel):
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


# ----------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clock, power and throttle reasons (50 ms period: the
    power cap lowers the SM clock for tens of milliseconds at a time under this load)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.lines = []
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            sel = str(device_index)
        self.cmd = ["nvidia-smi", "-i", sel, f"--query-gpu={self.FIELDS}",
                    "--format=csv,noheader,nounits", "-lms", "50"]

    def start(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                 flags=parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return None
        # Samples under load: power well above idle; fall back to all samples.
        pmax = max(r["power"] for r in rows)
        load = [r for r in rows if r["power"] >= 0.5 * pmax] or rows
        reasons = sorted({self.NAMES[i] for r in load for i, f in enumerate(r["flags"])
                          if f.lower() == "active"})
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_mhz_min": min(r["sm"] for r in load),
                "sm_max_mhz": max(r["smax"] for r in rows), "reasons": reasons,
                "samples": len(load), "power_w_max": pmax}


# ------------------------------------------------------------------ CPU oracle
def oracle_sample(target_s=6.0, max_n=None):
    """Time the float64 oracle on one head of the causal training step, restricted to
    a causal prefix of Ns rows (an independent sub-problem of the same workload).
    Ns grows until one forward+backward takes about target_s seconds."""
    import numpy as np
    import oracle
    from exact_attention_155_b200.inputs import attention_inputs, to_f64
    w = WORKLOAD
    d = w["d"]
    scale = 1.0 / math.sqrt(d)
    inp = attention_inputs(1, w["N"], 1, d, seed=1004)
    full = {n: to_f64(inp[n]) for n in ("q", "k", "v", "dout")}
    ns = 1024
    limit = max_n or w["N"]
    while True:
        sub = {n: full[n][:, :ns] for n in full}
        t0 = time.perf_counter()
        oracle.attention_forward(sub["q"], sub["k"], sub["v"], causal=True, scale=scale)
        oracle.attention_backward(sub["q"], sub["k"], sub["v"], sub["dout"], causal=True, scale=scale)
        dt = time.perf_counter() - t0
        if dt * 4 > target_s or ns * 2 > limit:
            break
        ns *= 2
    flops = 3.5 * fwd_flops(1, 1, ns, d, True)
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        cores = os.cpu_count() or 1

    def run_once():
        sub = {n: full[n][:, :ns] for n in full}
        t0 = time.perf_counter()
        oracle.attention_forward(sub["q"], sub["k"], sub["v"], causal=True, scale=scale)
        oracle.attention_backward(sub["q"], sub["k"], sub["v"], sub["dout"], causal=True, scale=scale)
        return time.perf_counter() - t0

    sample = (f"float64 oracle fwd+bwd of 1 of {w['B'] * w['H']} heads, causal prefix of "
              f"{ns} of {w['N']} rows (d={d})")
    return run_once, flops, int(cores), sample, dt


def run_reference(args, rank):
    if rank != 0:
        return
    run_once, flops, cores, sample, _ = oracle_sample(target_s=4.0)
    for _ in range(max(0, args.warmup)):
        run_once()
    times = [run_once() for _ in range(max(1, args.steps))]
    mean = statistics.mean(times)
    value = flops / mean / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": mean * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(n):
    w = WORKLOAD
    return {"workload": (f"causal training step (fwd+bwd): B={w['B']} H={w['H']} N={w['N']} "
                         f"d={w['d']} bf16"),
            "B": w["B"], "H": w["H"], "N": w["N"], "d": w["d"], "causal": True,
            "global_batch": w["B"] * n, "seq_len": w["N"],
            "l2": "inputs larger than L2 (q, k, v, dout: 4 x 128 MiB per step)",
            "parallelism": f"replicas x{n}"}


# ----------------------------------------------------------------- GPU timing
def timed_events(torch, fn, reps, flush=None):
    """Median device time (ms) of fn over reps, CUDA events on the current stream.
    flush: callable run before every rep (outside the timed interval)."""
    times = []
    for _ in range(reps):
        if flush is not None:
            flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b))
    return statistics.median(times)


def _barrier(world):
    """Barrier over all ranks (no-op for one rank)."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _max_over_ranks(x, world, device):
    """The largest of every rank's x (a device time: the job ends with its slowest rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, units_per_rank_step, steps, elapsed_ms):
    """Whole-job rate: the units every rank processed over `steps` steps, divided by the
    slowest rank's time (per-rank work is fixed as ranks are added: weak scaling)."""
    return world * units_per_rank_step * steps / (elapsed_ms * 1e-3)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import exact_attention_155_b200 as fa
    from exact_attention_155_b200.inputs import (VARLEN_BENCH, WINDOW_BENCH, attention_inputs,
                                                 bf16_randn, decode_inputs, packed_lengths)

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    w = WORKLOAD
    B, H, N, d = w["B"], w["H"], w["N"], w["d"]
    scale = 1.0 / math.sqrt(d)
    f_fwd = fwd_flops(B, H, N, d, True)
    f_bwd = 2.5 * f_fwd
    f_step = f_fwd + f_bwd

    inp = attention_inputs(B, N, H, d, seed=1004 + rank)
    host = {n: inp[n].pin_memory() for n in ("q", "k", "v", "dout")}
    q, k, v, do = (host[n].to(dev) for n in ("q", "k", "v", "dout"))
    out = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)

    def step(ev=None):
        if ev is None:
            fa.fwd(q, k, v, causal=True, scale=scale, out=out, lse=lse)
            fa.bwd(q, k, v, out, do, lse, causal=True, scale=scale, dq=dq, dk=dk, dv=dv, workspace=ws)
        else:
            ev[0].record()
            fa.fwd(q, k, v, causal=True, scale=scale, out=out, lse=lse)
            ev[1].record()
            fa.bwd(q, k, v, out, do, lse, causal=True, scale=scale, dq=dq, dk=dk, dv=dv,
                   workspace=ws, main_events=(ev[2], ev[3]))

    def barrier():
        _barrier(world)

    def max_over_ranks(x):
        return _max_over_ranks(x, world, dev)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    for e in evs:  # create the event handles (torch does so on first record)
        for x in e:
            x.record()
    sampler = ClockSampler(local_rank)
    barrier()
    sampler.start()
    torch.cuda.synchronize()
    barrier()
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for i in range(K):
        step(evs[i])
    t_stop.record()
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_stop))
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_main_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    ms_per_step = elapsed_ms / K
    value = job_throughput(world, f_step, K, elapsed_ms) / 1e12
    status = fa.device_status()[0]
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")

    achieved = f_bwd / (bwd_main_ms * 1e-3) / 1e12
    traffic = None
    if BWD_TRAFFIC["src_sha256"] == src_sha("exact_attention_155_b200/csrc/bwd.cuh"):
        traffic = BWD_TRAFFIC["bytes_per_launch"]
    # The timed region lasts well under a second at the SM clock recorded in `clocks`,
    # so the burst bf16 peak is the denominator; the sustained one (a seconds-long
    # loop at a lower, power-capped clock) is reported beside it.
    roofline = {"kernel": "bwd_kernel<128,causal>", "bound": "tensor", "achieved": achieved,
                "peak": peaks["tf_burst"], "unit": "TFLOP/s",
                "frac": achieved / peaks["tf_burst"],
                "frac_of_sustained": achieved / peaks["tf_sustained"],
                "frac_of_nominal": achieved / NOMINAL_TFLOPS,
                "peak_kind": f"bf16 dense, burst, of {peaks['source']}",
                "sm_mhz_median": clocks["sm_mhz"] if clocks else None,
                "traffic": traffic, "avg_launch_ms": bwd_main_ms,
                "algorithmic_flop_per_launch": f_bwd}

    # ---- end to end through the public API from pinned host buffers
    # Every step copies its own inputs host->device and its results device->host.
    # Steps are pipelined the way a caller streaming batches would run them: two sets
    # of device tensors, one stream each for copy-in, compute and copy-out, so step
    # i's copies overlap the compute of its neighbours.
    e2e = None
    if not args.no_e2e:
        hout = torch.empty_like(out, device="cpu").pin_memory()
        hlse = torch.empty_like(lse, device="cpu").pin_memory()
        hdq, hdk, hdv = (torch.empty_like(x, device="cpu").pin_memory() for x in (dq, dk, dv))
        sets = [dict(q=q, k=k, v=v, dout=do, out=out, lse=lse, dq=dq, dk=dk, dv=dv)]
        sets.append({n: torch.empty_like(t) for n, t in sets[0].items()})
        s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        for e in ev_comp + ev_out:
            e.record()

        def e2e_step(i):
            x = i % 2
            t = sets[x]
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_comp[x])  # step i-2 finished reading these inputs
                for n in ("q", "k", "v", "dout"):
                    t[n].copy_(host[n], non_blocking=True)
                ev_in[x].record()
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_in[x])
                s_comp.wait_event(ev_out[x])  # step i-2's results were copied out
                fa.fwd(t["q"], t["k"], t["v"], causal=True, scale=scale, out=t["out"], lse=t["lse"])
                fa.bwd(t["q"], t["k"], t["v"], t["out"], t["dout"], t["lse"], causal=True, scale=scale,
                       dq=t["dq"], dk=t["dk"], dv=t["dv"], workspace=ws)
                ev_comp[x].record()
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[x])
                for src, dst in ((t["out"], hout), (t["lse"], hlse), (t["dq"], hdq), (t["dk"], hdk),
                                 (t["dv"], hdv)):
                    dst.copy_(src, non_blocking=True)
                ev_out[x].record()

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        Ke = K
        barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s_in):
            a.record()
        for i in range(Ke):
            e2e_step(i)
        with torch.cuda.stream(s_out):
            b.record()
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(a.elapsed_time(b))
        h2d = sum(host[n].numel() * host[n].element_size() for n in host)
        d2h = sum(x.numel() * x.element_size() for x in (out, lse, dq, dk, dv))
        e2e = {"value": job_throughput(world, f_step, Ke, e2e_ms) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_ms / Ke, "steps": Ke,
               "pipelining": "2 device buffer sets; copy-in, compute and copy-out streams"}
        del hout, hlse, hdq, hdk, hdv, sets

    # ---- parts: prefill forward, decode sweep, incremental decode steps
    parts = None
    if not args.no_parts:
        del dq, dk, dv, ws
        torch.cuda.synchronize()
        time.sleep(2.0)  # let clocks recover from the long step loops before short kernels
        p = PREFILL
        pin = attention_inputs(p["B"], p["N"], p["H"], p["d"], seed=1003)
        pq, pk, pv = (pin[n].to(dev) for n in ("q", "k", "v"))
        pout, plse = torch.empty_like(pq), torch.empty((p["B"], p["H"], p["N"]), device=dev)
        for _ in range(3):
            fa.fwd(pq, pk, pv, causal=True, scale=scale, out=pout, lse=plse)
        pms = timed_events(torch, lambda: fa.fwd(pq, pk, pv, causal=True, scale=scale, out=pout,
                                                 lse=plse), 20)
        ptf = fwd_flops(p["B"], p["H"], p["N"], p["d"], True) / (pms * 1e-3) / 1e12
        del pq, pk, pv, pout, plse
        # L2 flush between calls of the short kernels below: write 512 MiB (evicts
        # everything), then read another 256 MiB so the lines left in L2 are clean and
        # the timed kernel does not pay for write-backs of the flush itself.
        flush_w = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
        flush_r = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)

        def flush():
            flush_w.zero_()
            flush_r.max()
        # Tiny correctness workload (B=1 H=2 N=128 d=64): one tile per head, latency.
        t = TINY
        tin = attention_inputs(t["B"], t["N"], t["H"], t["d"], seed=1001)
        tq, tk, tv, tdo = (tin[n].to(dev) for n in ("q", "k", "v", "dout"))
        tiny = {"workload": "B=1 H=2 N=128 d=64, scale 1/8, fwd and bwd (whole call: "
                            "preprocess, main and dq-convert kernels)",
                "unit": "us per call (CUDA events around one call, L2 flushed before each)"}
        for causal_t in (False, True):
            to, tl = fa.fwd(tq, tk, tv, causal=causal_t, scale=0.125)
            tg = [torch.empty_like(tq) for _ in range(3)]
            tws = torch.empty(fa.bwd_workspace_size(t["B"], t["H"], t["N"], t["d"]),
                              dtype=torch.uint8, device=dev)
            ff = lambda: fa.fwd(tq, tk, tv, causal=causal_t, scale=0.125, out=to, lse=tl)
            bf = lambda: fa.bwd(tq, tk, tv, to, tdo, tl, causal=causal_t, scale=0.125, dq=tg[0],
                                dk=tg[1], dv=tg[2], workspace=tws)
            for _ in range(5):
                ff()
                bf()
            tiny["causal" if causal_t else "non_causal"] = {
                "fwd_us": timed_events(torch, ff, 30, flush=flush) * 1e3,
                "bwd_us": timed_events(torch, bf, 30, flush=flush) * 1e3}
        del tq, tk, tv, tdo, to, tl, tg, tws
        # ViT / packed-QKV shape (B=2 H=16 N=1024 d=64, non-causal forward, scale 1/8),
        # read in place from one packed [B, N, 3, H, d] tensor as the qkvpacked call does.
        vt = VIT
        vin = attention_inputs(vt["B"], vt["N"], vt["H"], vt["d"], seed=1002, with_dout=False)
        qkv = torch.stack([vin[n] for n in ("q", "k", "v")], dim=2).to(dev)
        del vin
        vo, vl = fa.fwd_qkvpacked(qkv, causal=False, scale=0.125)
        vit_fn = lambda: fa.fwd_ex(qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2], causal=False,
                                   scale=0.125, out=vo, lse=vl)
        for _ in range(5):
            vit_fn()
        vit_ms = timed_events(torch, vit_fn, 30, flush=flush)
        vit_warm_ms = timed_events(torch, vit_fn, 30)
        vit_fl = fwd_flops(vt["B"], vt["H"], vt["N"], vt["d"], False)
        vit_tf = vit_fl / (vit_ms * 1e-3) / 1e12
        del qkv, vo, vl
        s = SWEEP
        kc, vc, qs, _, _ = decode_inputs(s["B"], s["H"], s["d"], s["Ncap"], 1, seed=1005)
        kc, vc, qd = kc.to(dev), vc.to(dev), qs[0].to(dev)
        seq = torch.full((s["B"],), s["seqlen"], dtype=torch.int32, device=dev)
        dws = torch.empty(max(1, fa.decode_workspace_size(s["B"], s["H"], s["Ncap"], s["d"])),
                          dtype=torch.uint8, device=dev)
        dout_ = torch.empty_like(qd)
        dlse = torch.empty((s["B"], s["H"]), device=dev)
        dec = lambda: fa.decode(qd, kc, vc, seq, scale=1 / 8, out=dout_, lse=dlse, workspace=dws)
        for _ in range(3):
            dec()
        dms = timed_events(torch, dec, 30, flush=flush)
        dbytes = 2 * s["B"] * s["H"] * s["seqlen"] * s["d"] * 2
        dgbs = dbytes / (dms * 1e-3) / 1e9
        # The same sweep over a paged cache: 64-row pages at shuffled pool positions.
        page = 64
        nb = s["Ncap"] // page
        gperm = torch.Generator().manual_seed(1008)
        perm = torch.randperm(s["B"] * nb, generator=gperm).to(dev)
        table = perm.view(s["B"], nb).to(torch.int32)
        kp = torch.empty((s["B"] * nb, page, s["H"], s["d"]), dtype=torch.bfloat16, device=dev)
        vp = torch.empty_like(kp)
        kp[perm] = kc.view(s["B"] * nb, page, s["H"], s["d"])
        vp[perm] = vc.view(s["B"] * nb, page, s["H"], s["d"])
        decp = lambda: fa.decode_paged(qd, kp, vp, table, seq, scale=1 / 8, out=dout_, lse=dlse)
        for _ in range(3):
            decp()
        pdms = timed_events(torch, decp, 30, flush=flush)
        pdgbs = dbytes / (pdms * 1e-3) / 1e9
        del kc, vc, kp, vp, table, flush_w, flush_r
        c5 = STEPS5
        kc, vc, qs, ks, vs = decode_inputs(c5["B"], c5["H"], c5["d"], c5["Ncap"], c5["steps"], seed=1005)
        kc, vc, qs, ks, vs = kc.to(dev), vc.to(dev), qs.to(dev), ks.to(dev), vs.to(dev)
        seqs = [torch.full((c5["B"],), t, dtype=torch.int32, device=dev) for t in range(c5["steps"])]
        o5 = torch.empty_like(qs[0])
        l5 = torch.empty((c5["B"], c5["H"]), device=dev)
        ws5 = torch.empty(max(1, fa.decode_workspace_size(c5["B"], c5["H"], c5["Ncap"], c5["d"])),
                          dtype=torch.uint8, device=dev)

        def steps100():
            for t in range(c5["steps"]):
                fa.decode(qs[t], kc, vc, seqs[t], ks[t], vs[t], scale=1 / 8, out=o5, lse=l5,
                          workspace=ws5)
        steps100()
        sms = timed_events(torch, steps100, 5)
        # The same 100 steps replayed from one CUDA graph: no host launch overhead.
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            steps100()
        torch.cuda.current_stream().wait_stream(side)
        with torch.cuda.graph(graph):
            steps100()
        graph.replay()
        gms = timed_events(torch, graph.replay, 10)
        del graph
        del kc, vc, qs, ks, vs, o5, l5, ws5
        # Sliding-window causal attention (window 4096) on a 16K sequence, fwd and bwd.
        wb = WINDOW_BENCH
        win = attention_inputs(wb["B"], wb["N"], wb["H"], wb["d"], seed=wb["seed"])
        wq, wk, wv, wdo = (win[n].to(dev) for n in ("q", "k", "v", "dout"))
        del win
        wwin = wb["window"]
        wo, wlse = fa.fwd_ex(wq, wk, wv, causal=True, scale=scale, window=wwin)
        wg = [torch.empty_like(wq) for _ in range(3)]
        wws = torch.empty(fa.bwd_workspace_size(wb["B"], wb["H"], wb["N"], wb["d"]),
                          dtype=torch.uint8, device=dev)
        fwd_w = lambda: fa.fwd_ex(wq, wk, wv, causal=True, scale=scale, window=wwin, out=wo, lse=wlse)
        bwd_w = lambda: fa.bwd_ex(wq, wk, wv, wo, wdo, wlse, causal=True, scale=scale, window=wwin,
                                  dq=wg[0], dk=wg[1], dv=wg[2], workspace=wws)
        for _ in range(3):
            fwd_w()
            bwd_w()
        wf_ms = timed_events(torch, fwd_w, 10)
        wb_ms = timed_events(torch, bwd_w, 10)
        w_left = wwin[0]
        pairs = w_left * (w_left + 1) // 2 + (wb["N"] - w_left) * (w_left + 1)  # visible (q, k)
        wf_fl = 4.0 * wb["d"] * wb["B"] * wb["H"] * pairs
        del wq, wk, wv, wdo, wo, wlse, wg, wws
        # Packed variable-length batch (seeded length mix), causal, fwd and bwd.
        vb = VARLEN_BENCH
        lens = packed_lengths(vb["total"], vb["lo"], vb["hi"], vb["seed"])
        cu = torch.tensor([0] + list(itertools.accumulate(lens)), dtype=torch.int32, device=dev)
        gen = torch.Generator().manual_seed(vb["seed"])
        vq, vk, vv, vdo = (bf16_randn((vb["total"], vb["H"], vb["d"]), gen).to(dev) for _ in range(4))
        vo, vlse = fa.fwd_ex(vq, vk, vv, causal=True, scale=scale, cu_seqlens=cu, max_seqlen=max(lens))
        vg = [torch.empty_like(vq) for _ in range(3)]
        vws = torch.empty(fa.bwd_workspace_size(len(lens), vb["H"], max(lens), vb["d"]),
                          dtype=torch.uint8, device=dev)
        fwd_v = lambda: fa.fwd_ex(vq, vk, vv, causal=True, scale=scale, cu_seqlens=cu,
                                  max_seqlen=max(lens), out=vo, lse=vlse)
        bwd_v = lambda: fa.bwd_ex(vq, vk, vv, vo, vdo, vlse, causal=True, scale=scale, cu_seqlens=cu,
                                  max_seqlen=max(lens), dq=vg[0], dk=vg[1], dv=vg[2], workspace=vws)
        for _ in range(3):
            fwd_v()
            bwd_v()
        vf_ms = timed_events(torch, fwd_v, 10)
        vb_ms = timed_events(torch, bwd_v, 10)
        vf_fl = 4.0 * vb["d"] * vb["H"] * sum(n * (n + 1) // 2 for n in lens)
        del vq, vk, vv, vdo, vo, vlse, vg, vws
        # Ring attention, 4 shards emulated on this GPU (exchange = indexing): the compute
        # side of the sequence-parallel forward on the prefill workload.
        from exact_attention_155_b200.ring import ring_attention_fwd_emulated
        p = PREFILL
        pin = attention_inputs(p["B"], p["N"], p["H"], p["d"], seed=1003, with_dout=False)
        rq, rk, rv = (pin[n].to(dev) for n in ("q", "k", "v"))
        del pin
        ring_fn = lambda: ring_attention_fwd_emulated(rq, rk, rv, 4, causal=True, scale=scale)
        for _ in range(2):
            ring_fn()
        rms = timed_events(torch, ring_fn, 5)

        def ring_parallel_ms(xq, xk, xv, layout):
            """Time of a parallel run of the emulated ranks: per step, the slowest rank's
            kernels (CUDA events around each rank's work at each step), summed over steps;
            the exchange (NCCL point-to-point, overlapped with the compute) is not in it."""
            ring_attention_fwd_emulated(xq, xk, xv, 4, causal=True, scale=scale, layout=layout)
            best = None
            for _ in range(3):
                evs = []
                ring_attention_fwd_emulated(xq, xk, xv, 4, causal=True, scale=scale, layout=layout,
                                            step_events=evs)
                torch.cuda.synchronize()
                per_step = {}
                for _r, st, a, b in evs:
                    per_step.setdefault(st, []).append(a.elapsed_time(b))
                ms = sum(max(v) for v in per_step.values())
                best = ms if best is None else min(best, ms)
            return best
        ring_par = {p["N"]: {lay: ring_parallel_ms(rq, rk, rv, lay) for lay in ("contiguous", "zigzag")}}
        del rq, rk, rv
        # The same estimate on a 32768-token sequence (8192 rows per rank), the length where
        # splitting the sequence over GPUs is the point.
        RN = 32768
        rin = attention_inputs(1, RN, p["H"], p["d"], seed=1009, with_dout=False)
        rq, rk, rv = (rin[n].to(dev) for n in ("q", "k", "v"))
        del rin
        ring_par[RN] = {lay: ring_parallel_ms(rq, rk, rv, lay) for lay in ("contiguous", "zigzag")}
        del rq, rk, rv
        parts = {
            "prefill_fwd": {"workload": "causal fwd B=1 H=32 N=8192 d=128", "value": ptf,
                            "unit": "TFLOP/s", "ms": pms, "roofline_bound": "tensor",
                            "frac": ptf / peaks["tf_burst"],
                            "frac_of_nominal": ptf / NOMINAL_TFLOPS,
                            "peak": peaks["tf_burst"],
                            "peak_kind": f"bf16 dense, burst, of {peaks['source']}"},
            "tiny": tiny,
            "vit_fwd": {"workload": "ViT / packed-QKV shape: non-causal fwd B=2 H=16 N=1024 d=64, "
                                    "q, k, v read in place from one [B, N, 3, H, d] tensor",
                        "value": vit_tf, "unit": "TFLOP/s", "us": vit_ms * 1e3,
                        "us_l2_warm": vit_warm_ms * 1e3,
                        "flop_per_call": vit_fl, "roofline_bound": "tensor",
                        "frac": vit_tf / peaks["tf_burst"], "frac_of_nominal": vit_tf / NOMINAL_TFLOPS,
                        "peak": peaks["tf_burst"],
                        "peak_kind": f"bf16 dense, burst, of {peaks['source']}",
                        "l2": "flushed before every call (us_l2_warm: back to back)"},
            "train_fwd_in_step": {"value": f_fwd / (fwd_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                                  "ms": fwd_ms},
            "decode_sweep": {"workload": "decode B=32 H=16 d=64, 2048 cached rows, no append",
                             "value": dgbs, "unit": "GB/s", "us": dms * 1e3,
                             "roofline_bound": "hbm", "frac": dgbs / peaks["hbm"],
                             "frac_of_nominal": dgbs / NOMINAL_HBM_GBS,
                             "peak": peaks["hbm"], "peak_kind": f"HBM copy, of {peaks['source']}",
                             "l2": "flushed before every call (512 MiB write, then 256 MiB read)"},
            "decode_sweep_paged": {"workload": "decode B=32 H=16 d=64, 2048 rows in 64-row pages "
                                               "at shuffled pool positions, no append",
                                   "value": pdgbs, "unit": "GB/s", "us": pdms * 1e3,
                                   "roofline_bound": "hbm", "frac": pdgbs / peaks["hbm"],
                                   "peak": peaks["hbm"],
                                   "peak_kind": f"HBM copy, of {peaks['source']}",
                                   "l2": "flushed before every call"},
            "ring_fwd_emulated": {
                "workload": "causal fwd B=1 H=32 N=8192 d=128 as 4 sequence shards on one GPU "
                            "(ring schedule, partial attention + LSE merge per shard pair)",
                "value": fwd_flops(p["B"], p["H"], p["N"], p["d"], True) / (rms * 1e-3) / 1e12,
                "unit": "TFLOP/s", "ms": rms,
                "parallel_estimate": {
                    f"N={n}": {lay: {"ms": ms, "tflops_per_gpu":
                                     fwd_flops(1, p["H"], n, p["d"], True) / 4 / (ms * 1e-3) / 1e12}
                               for lay, ms in v.items()}
                    for n, v in ring_par.items()},
                "note": "value: all 4 ranks run one after another on this GPU (exchange is "
                        "indexing); parallel_estimate: sum over the 4 steps of the slowest "
                        "rank's kernel time, contiguous shards vs zigzag chunks, at N = 8192 "
                        "and N = 32768"},
            "window_causal": {
                "workload": f"causal sliding window {wwin[0]}, B=1 H=32 N=16384 d=128",
                "fwd_tflops": wf_fl / (wf_ms * 1e-3) / 1e12, "fwd_ms": wf_ms,
                "bwd_tflops": 2.5 * wf_fl / (wb_ms * 1e-3) / 1e12, "bwd_ms": wb_ms,
                "flop_count": "4*d*H per visible (query, key) pair, x2.5 for bwd",
                "bwd_includes": "preprocess, main and dq-convert kernels",
                "roofline_bound": "tensor",
                "fwd_frac": wf_fl / (wf_ms * 1e-3) / 1e12 / peaks["tf_burst"],
                "peak": peaks["tf_burst"], "peak_kind": f"bf16 dense, burst, of {peaks['source']}"},
            "varlen_causal": {
                "workload": f"packed causal batch, {len(lens)} sequences of {min(lens)}-{max(lens)} tokens "
                            f"({vb['total']} tokens), H=32 d=128",
                "fwd_tflops": vf_fl / (vf_ms * 1e-3) / 1e12, "fwd_ms": vf_ms,
                "bwd_tflops": 2.5 * vf_fl / (vb_ms * 1e-3) / 1e12, "bwd_ms": vb_ms,
                "bwd_includes": "preprocess, main and dq-convert kernels",
                "roofline_bound": "tensor",
                "fwd_frac": vf_fl / (vf_ms * 1e-3) / 1e12 / peaks["tf_burst"],
                "peak": peaks["tf_burst"], "peak_kind": f"bf16 dense, burst, of {peaks['source']}"},
            "decode_steps": {"workload": "decode B=2 H=16 d=64 cap 2048, 100 appending steps",
                             "us_per_step": sms * 1e3 / c5["steps"],
                             "us_per_step_cuda_graph": gms * 1e3 / c5["steps"],
                             "gb_s": 8192 * sum(t + 1 for t in range(c5["steps"]))
                             / (sms * 1e-3) / 1e9},
        }

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        run_once, flops, cores, sample, _ = oracle_sample(target_s=12.0)
        dt = min(run_once() for _ in range(1))
        cpu = {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": sample, "seconds": dt}

    launches_per_step = 4  # fwd kernel + bwd preprocess, main and dq-convert kernels
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(world), "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches_per_step * K, "clocks": clocks, "parts": parts,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-parts", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        log("warmup raised to 3 (minimum)")
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
