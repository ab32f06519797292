#!/usr/bin/env python
"""Benchmark of exact tiled attention (forward + backward) on B200.

One step = the whole hot path on one batch of synthetic inputs already in HBM:
fa2_forward, then the three backward stages (preprocess, main, dQ convert),
each launched through the C ABI on the current stream with CUDA events between
them, so every kernel's duration is measured live inside the timed region.

Default workload (one GPU): B=1, H=16, N=16384, d=128, causal, bf16 i.i.d.
N(0,1) Q/K/V/dO from the shared seeded generator: the longest sequence of the
attention benchmark the pages quote (forward, backward and forward+backward
TFLOP/s against sequence length up to 16k, head dimension 64 and 128, with and
without the causal mask: Figures 4-7 of the FlashAttention-2 paper's
reproduction page). ``--workload`` selects the shorter forward+backward
(B=8 H=16 N=2048 d=128 causal) or the forward-only (B=8 H=32 N=2048 d=64)
workload instead. FLOPs: forward 4*B*H*N^2*d, backward 2.5x, causal halved
(value) and unhalved (value_unhalved).

Multi-GPU (torchrun): every rank runs the same per-GPU workload on its own
seeded batch (independent heads; no collective on the data path), timing is
the max over ranks, and value is the whole-job throughput (weak scaling).

``--impl reference`` times the fp64 CPU oracle instead (rank 0 only), on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention TFLOP/s (fwd, bwd, fwd+bwd) and % of B200 dense BF16 peak"
WORKLOADS = {
    "fwd_bwd_b8_h16_n2048_d128_causal": dict(cfg=2, B=8, H=16, N=2048, d=128, causal=True),
    "fwd_b8_h32_n2048_d64": dict(cfg=1, B=8, H=32, N=2048, d=64, causal=False),
    "fwd_bwd_b1_h16_n16384_d128_causal": dict(cfg=3, B=1, H=16, N=16384, d=128, causal=True),
}
DEFAULT_WORKLOAD = "fwd_bwd_b1_h16_n16384_d128_causal"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = {
    "fa2_fwd_kernel": ["fwd_sm100.cuh", "sm100_ptx.cuh", "exp2_poly.cuh"],
    "fa2_bwd_kernel": ["bwd_sm100.cuh", "sm100_ptx.cuh"],
    "fa2_bwd_pre_kernel": ["bwd_sm100.cuh"],
    "fa2_bwd_dq_convert_kernel": ["bwd_sm100.cuh"],
}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_src_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "exact_tiled_attention_30_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current source of that kernel and this workload; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel]
    except Exception:
        return None
    if rec.get("src_hash") != kernel_src_hash(kernel) or rec.get("workload") != workload:
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 20 ms in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: str):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20", "-i", str(device_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    @staticmethod
    def _reasons(samples):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for p in samples:
            for name, val in zip(names, p[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return reasons

    def summary(self, t0: float, t1: float):
        """Median SM clock and the throttle reasons seen by the samples taken inside
        [t0, t1]. With no sample inside, the clock fields are null (a number taken
        outside the timed region would not describe it); the reasons seen by the
        samples within 0.2 s of it are still listed, under ``reasons_nearby``."""
        inside = [p for t, p in self.samples if t0 <= t <= t1]
        if not inside:
            near = [p for t, p in self.samples if t0 - 0.2 <= t <= t1 + 0.2]
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "reasons_nearby": sorted(self._reasons(near)) if near else
                    ["no nvidia-smi samples"]}
        used = inside
        reasons = self._reasons(used)
        mhz = []
        for p in used:
            try:
                mhz.append(float(p[1]))
            except ValueError:
                pass
        try:
            smax = float(used[0][2])
        except ValueError:
            smax = None
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(inside),
                "power_w_max": max(float(p[3]) for p in used if p[3].replace(".", "").isdigit())
                if any(p[3].replace(".", "").isdigit() for p in used) else None}


def flops(w, passes: str, halve_causal: bool = True) -> float:
    f = 4.0 * w["B"] * w["H"] * w["N"] ** 2 * w["d"]
    mult = {"fwd": 1.0, "bwd": 2.5, "fwd+bwd": 3.5}[passes]
    f *= mult
    if w["causal"] and halve_causal:
        f /= 2
    return f


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise maximum of a list of floats over all ranks (identity on one rank).
    Every rank must call it with the same number of values."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return [float(v) for v in values]
    import torch

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def rank_config_index(config_index: int, rank: int) -> int:
    """Seed index of a rank's batch: every rank draws an independent batch."""
    return config_index + 1000 * rank


def make_inputs(w, rank: int):
    import attn_inputs

    return attn_inputs.make_qkvdo(rank_config_index(w["cfg"], rank), w["B"], w["H"], w["N"],
                                  w["d"], with_do=True)


# ------------------------------------------------------------- oracle timing
#: heads whose full N x N backward the oracle holds in memory; above this the
#: oracle runs the whole forward of a head and the gradients of sampled rows
FULL_BACKWARD_MAX_N = 4096
#: query rows (dQ) and key rows (dK, dV) per head in the row-sampled backward
SAMPLED_GRAD_ROWS = 64


def _visible(i, N, causal):
    """Keys that query i sees (self-attention)."""
    return i + 1 if causal else N


def oracle_head(w, host, head: int, threads: int):
    """Runs the oracle on one (b, h) head of the workload and returns
    (seconds, FLOPs of the arithmetic it did, description).

    N <= FULL_BACKWARD_MAX_N: the full forward and backward of the head; FLOPs
    counted like the GPU's (forward 4 N^2 d, backward 2.5x, causal halved).
    Longer heads: the full forward of the head (every O_i, LSE_i, D_i) and the
    gradients of SAMPLED_GRAD_ROWS evenly spaced query rows (dQ) and key rows
    (dK, dV), straight from their definitions. FLOPs counted per visible
    (query, key) pair: 4 d for a forward row (score and weighted sum), 6 d for a
    dQ row (score, dP, weighted sum), 8 d for a dK/dV row (score, dP and both
    weighted sums)."""
    import oracle

    N, d, causal = w["N"], w["d"], w["causal"]
    b, h = divmod(head % (w["B"] * w["H"]), w["H"])
    scale = 1.0 / math.sqrt(d)
    args = (host["q"][b, h], host["k"][b, h], host["v"][b, h], host["do"][b, h], causal, scale)
    if N <= FULL_BACKWARD_MAX_N:
        t0 = time.perf_counter()
        oracle.attention_backward(*args, nthreads=threads)
        secs = time.perf_counter() - t0
        return secs, flops(dict(w, B=1, H=1), "fwd+bwd"), "full forward + backward in fp64"
    rows = [int(x) for x in np.linspace(0, N - 1, SAMPLED_GRAD_ROWS).round()]
    t0 = time.perf_counter()
    oracle.attention_backward_rows(*args, rows, rows, nthreads=threads)
    secs = time.perf_counter() - t0
    fl = 4.0 * d * sum(_visible(i, N, causal) for i in range(N))
    fl += 6.0 * d * sum(_visible(i, N, causal) for i in rows)
    fl += 8.0 * d * sum((N - j) if causal else N for j in rows)
    desc = (f"fp64 forward of all {N} rows + dQ of {len(rows)} query rows and dK, dV of "
            f"{len(rows)} key rows; FLOPs of the arithmetic done")
    return secs, fl, desc


def oracle_sample(w, host, max_seconds: float):
    """Times the fp64 oracle on whole heads of this workload (oracle_head), adding
    heads until about max_seconds of CPU work; returns (TFLOP/s, desc, threads, s)."""
    import oracle

    oracle.build()
    threads = oracle.default_threads()
    done, elapsed, fl, desc = 0, 0.0, 0.0, ""
    total_heads = w["B"] * w["H"]
    while done < total_heads and elapsed < max_seconds:
        secs, f, desc = oracle_head(w, host, done, threads)
        elapsed += secs
        fl += f
        done += 1
    return fl / elapsed / 1e12, f"{done} of {total_heads} heads: {desc}", threads, elapsed


def run_reference(args, w, rank: int):
    """The reference arm: the fp64 oracle as it stands on the host cores, one head
    of the workload per step (oracle_head), rank 0 only."""
    if rank != 0:
        return
    host = make_inputs(w, 0)
    import oracle

    oracle.build()
    threads = oracle.default_threads()
    for i in range(args.warmup):
        oracle_head(w, host, i, threads)
    elapsed, fl, desc = 0.0, 0.0, ""
    for i in range(args.steps):
        secs, f, desc = oracle_head(w, host, args.warmup + i, threads)
        elapsed += secs
        fl += f
    value = fl / elapsed / 1e12
    sample = (f"one ({w['N']}x{w['d']}, causal={w['causal']}) head of the workload per step: "
              f"{desc}")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": elapsed / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args, w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def workload_config(args, w):
    return {
        "workload": args.workload, "batch_per_gpu": w["B"], "global_batch": w["B"] * args.gpus,
        "heads": w["H"], "seq_len": w["N"], "head_dim": w["d"], "causal": w["causal"],
        "parallelism": f"replicas x{args.gpus} (independent heads, no collective)",
        "l2": "inputs larger than L2 (Q, K, V, dO, O, dQ, dK, dV and workspace >> 126 MB)",
        "flops": "fwd 4*B*H*N^2*d, bwd 2.5x, causal halved (value) / unhalved (value_unhalved)",
        "inputs": "bf16 i.i.d. N(0,1), SplitMix64 + Box-Muller, seed 0xFA2+1000*config+tensor",
    }


# ------------------------------------------------------- benchmark-figure grid
def grid_points():
    """The pages' attention benchmark axes: hidden size 2048 (H = 2048 / d),
    d in {64, 128}, N in 512 .. 16k with B = 16384 / N, causal and not; then
    ragged lengths (N = 2000 and 4000 at d = 128, same B and H as 2048 and
    4096), which show what a length that is not a multiple of the 128-row tile
    costs."""
    pts = []
    for d in (64, 128):
        for causal in (False, True):
            for N in (512, 1024, 2048, 4096, 8192, 16384):
                pts.append({"B": 16384 // N, "H": 2048 // d, "N": N, "d": d, "causal": causal})
    for causal in (False, True):
        for N, B in ((2000, 8), (4000, 4)):
            pts.append({"B": B, "H": 16, "N": N, "d": 128, "causal": causal, "ragged": True})
    return pts


def run_grid(args):
    """One JSON line per grid point: forward, backward (three kernels) and their sum
    in TFLOP/s on device-resident random bf16 inputs, CUDA events around enough
    calls for at least ~60 ms of work (and at least 10) after warm-up, with the
    nvidia-smi clocks sampled in that span (not the contract line; the contract
    line is the default run)."""
    import torch

    import exact_tiled_attention_30_b200 as fa2

    fa2.load_library()
    peaks, _ = load_peaks()
    min_reps = max(args.steps // 40, 5)
    visible = [e.strip() for e in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if e.strip()]
    sampler = ClockSampler(visible[0] if visible else "0")
    for w in grid_points():
        if args.grid_filter and not any(f"{k}={w.get(k)}" in args.grid_filter.split(",")
                                        for k in ("d", "N")):
            continue
        B, H, N, d, causal = w["B"], w["H"], w["N"], w["d"], w["causal"]
        scale = 1.0 / math.sqrt(d)
        q = torch.randn(B, H, N, d, device="cuda", dtype=torch.bfloat16)
        k, v, do = torch.randn_like(q), torch.randn_like(q), torch.randn_like(q)
        o = torch.empty_like(q)
        lse = torch.empty(B, H, N, device="cuda", dtype=torch.float32)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
        ws = torch.empty(fa2.fa2_backward_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")

        def fwd():
            fa2.fa2_forward(q, k, v, o, lse, causal, scale)

        def bwd():
            fa2.fa2_backward(q, k, v, o, lse, do, dq, dk, dv, causal, scale, ws)

        res = {}
        t_in = []
        for name, fn in (("fwd", fwd), ("bwd", bwd)):
            for _ in range(args.warmup):
                fn()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            reps = int(min(2000, max(min_reps, math.ceil(60.0 / max(e0.elapsed_time(e1), 1e-3)))))
            t_in.append(time.time())
            e0.record()
            for _ in range(reps):
                fn()
            e1.record()
            torch.cuda.synchronize()
            t_in.append(time.time())
            res[name] = e0.elapsed_time(e1) / reps
        res["fwd+bwd"] = res["fwd"] + res["bwd"]
        line = {"grid": True, **w, "clocks": sampler.summary(t_in[0], t_in[-1])}
        for name, ms in res.items():
            tf = flops(w, name) / (ms * 1e-3) / 1e12
            line[name] = {"ms": round(ms, 4), "tflops": round(tf, 1),
                          "frac": round(tf / peaks["bf16_tflops"], 3)}
        print(json.dumps(line), flush=True)
        del q, k, v, do, o, lse, dq, dk, dv, ws
        torch.cuda.empty_cache()
    sampler.stop()


# --------------------------------------------------------------- GPU timing
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the host-buffer measurement (profiling runs: fewer launches)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--grid", action="store_true",
                    help="time every point of the benchmark-figure grid (1 GPU), one JSON line each")
    ap.add_argument("--grid-filter", default="",
                    help="with --grid: only points matching one of these, e.g. 'd=64,N=2000'")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.grid:
        run_grid(args)
        return
    w = WORKLOADS[args.workload]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, w, rank)
        return

    import torch

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    import exact_tiled_attention_30_b200 as fa2

    fa2.load_library()
    peaks, peaks_kind = load_peaks()
    B, H, N, d, causal = w["B"], w["H"], w["N"], w["d"], w["causal"]
    scale = 1.0 / math.sqrt(d)
    host = make_inputs(w, rank)

    def pinned(bits):
        import numpy as np

        t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
        return t.pin_memory()

    hq, hk, hv, hdo = (pinned(host[n]) for n in ("q", "k", "v", "do"))
    dev = torch.device("cuda", local_rank)
    q, k, v, do = (t.to(dev) for t in (hq, hk, hv, hdo))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa2.fa2_backward_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]

    def step(events=None):
        if events:
            events[0].record(stream)
        fa2.fa2_forward(q, k, v, o, lse, causal, scale, stream)
        if events:
            events[1].record(stream)
        fa2.fa2_backward_preprocess(o, lse, do, ws, stream)
        if events:
            events[2].record(stream)
        fa2.fa2_backward_main(q, k, v, do, dk, dv, causal, scale, ws, stream)
        if events:
            events[3].record(stream)
        fa2.fa2_backward_dq_convert(dq, scale, ws, stream)
        if events:
            events[4].record(stream)

    # nvidia-smi takes the index or UUID this rank's GPU has in CUDA_VISIBLE_DEVICES
    visible = [e.strip() for e in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if e.strip()]
    sampler = ClockSampler(visible[local_rank] if local_rank < len(visible) else str(local_rank))
    for _ in range(args.warmup):
        step()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        step(ev[i])
    end.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if dist:
        dist.barrier()
    sampler.stop()
    st, site = fa2.fa2_get_device_status(stream)
    if st != 0:
        raise RuntimeError(f"device status {fa2.fa2_status_string(st)} at site {site:#x}")

    total_ms = start.elapsed_time(end)
    names = ["fa2_fwd_kernel", "fa2_bwd_pre_kernel", "fa2_bwd_kernel", "fa2_bwd_dq_convert_kernel"]
    kern_ms = {n: sum(e[j].elapsed_time(e[j + 1]) for e in ev) / args.steps
               for j, n in enumerate(names)}
    red = max_over_ranks([total_ms] + [kern_ms[n] for n in names], dist, dev)
    total_ms = red[0]
    kern_ms = {n: red[1 + j] for j, n in enumerate(names)}
    ms_step = total_ms / args.steps

    # e2e through the C ABI's host-buffer entry: pinned host inputs in, every
    # output back to pinned host memory, copies pipelined with the kernels
    e2e_ms = None
    if not args.no_e2e:
        outs_host = [torch.empty_like(x, device="cpu").pin_memory() for x in (o, lse, dq, dk, dv)]
        host_ws = torch.empty(fa2.fa2_forward_backward_host_workspace_size(B, H, N, d, 0),
                              dtype=torch.uint8, device=dev)

        def e2e_step():
            fa2.fa2_forward_backward_host(hq, hk, hv, hdo, *outs_host, causal, scale, host_ws, 0,
                                          stream)

        e2e_step()
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks([e0.elapsed_time(e1) / args.e2e_steps], dist, dev)[0]
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hdo))
        d2h = sum(x.numel() * x.element_size() for x in outs_host)

    clocks = sampler.summary(t_wall0, t_wall1)

    fl_step = flops(w, "fwd+bwd") * world
    value = fl_step / (ms_step * 1e-3) / 1e12
    value_unhalved = flops(w, "fwd+bwd", halve_causal=False) * world / (ms_step * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    fwd_ms = kern_ms["fa2_fwd_kernel"]
    bwd_ms = kern_ms["fa2_bwd_pre_kernel"] + kern_ms["fa2_bwd_kernel"] + \
        kern_ms["fa2_bwd_dq_convert_kernel"]
    fwd_tf = flops(w, "fwd") / (fwd_ms * 1e-3) / 1e12
    bwd_tf = flops(w, "bwd") / (bwd_ms * 1e-3) / 1e12

    # per-kernel algorithmic work per launch
    Np = (N + 127) // 128 * 128
    bh = B * H
    hbm = {
        "fa2_bwd_pre_kernel": 2 * bh * N * d * 2 + bh * N * 4 + bh * Np * (d * 4 + 8),
        "fa2_bwd_dq_convert_kernel": bh * N * d * (4 + 2),
    }
    kernels = {}
    for n in names:
        ms = kern_ms[n]
        if n in hbm:
            ach = hbm[n] / (ms * 1e-3) / 1e9
            kernels[n] = {"ms": ms, "bound": "hbm", "achieved": ach, "unit": "GB/s",
                          "frac": ach / peaks["hbm_gbs"]}
        else:
            f = flops(w, "fwd" if n == "fa2_fwd_kernel" else "bwd")
            ach = f / (ms * 1e-3) / 1e12
            kernels[n] = {"ms": ms, "bound": "tensor", "achieved": ach, "unit": "TFLOP/s",
                          "frac": ach / peak}
    dom = max(names, key=lambda n: kern_ms[n])
    kd = kernels[dom]
    roofline = {"kernel": dom, "bound": kd["bound"], "achieved": kd["achieved"],
                "peak": peak if kd["bound"] == "tensor" else peaks["hbm_gbs"], "unit": kd["unit"],
                "frac": kd["frac"], "traffic": ncu_traffic(dom, args.workload),
                "peak_source": f"{peaks_kind} (MEASURED_PEAKS.json burst bf16 / copy bandwidth)"
                if peaks_kind == "measured" else "fallback (6.65 TB/s, 1.59 PFLOP/s)",
                "algorithmic": "bwd FLOPs 10*B*H*N^2*d (causal halved) per launch"
                if dom == "fa2_bwd_kernel" else "see kernels"}

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": workload_config(args, w),
        "value_unhalved": value_unhalved,
        "frac_of_peak": value / (peak * world),
        "passes": {
            "fwd": {"ms": fwd_ms, "tflops": fwd_tf, "frac": fwd_tf / peak},
            "bwd": {"ms": bwd_ms, "tflops": bwd_tf, "frac": bwd_tf / peak},
            "fwd+bwd": {"ms": fwd_ms + bwd_ms, "tflops": value / world, "frac": value / world / peak},
        },
        "kernels": kernels,
        "roofline": roofline,
        "gpu_launches": 4 * args.steps,
        "clocks": clocks,
        "e2e": None if e2e_ms is None else {
            "value": fl_step / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
            "path": "pinned host Q,K,V,dO -> fa2_forward_backward_host (C ABI; chunks of "
                    "B*H/8 heads, copies in both directions overlapped with the kernels) -> "
                    "O, LSE, dQ, dK, dV in pinned host memory"},
        "peaks": {"kind": peaks_kind, **peaks},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, desc, threads, secs = oracle_sample(w, host, args.cpu_seconds)
        line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                "sample": desc, "seconds": secs}
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))


if __name__ == "__main__":
    main()
