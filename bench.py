#!/usr/bin/env python
"""Benchmark of exact tiled attention (forward + backward) on B200.

One step = the whole hot path on one batch of synthetic inputs already in HBM:
fa2_forward, then the three backward stages (preprocess, main, dQ convert),
each launched through the C ABI on the current stream with CUDA events between
them, so every kernel's duration is measured live inside the timed region.

Default workload (one GPU): B=8, H=16, N=2048, d=128, causal, bf16 i.i.d.
N(0,1) Q/K/V/dO from the shared seeded generator: the forward+backward
configuration the attention benchmark of the pages quotes (forward, backward
and forward+backward TFLOP/s, Figures 4-6 of the FlashAttention-2 paper's
reproduction page). FLOPs: forward 4*B*H*N^2*d, backward 2.5x, causal halved
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention TFLOP/s (fwd, bwd, fwd+bwd) and % of B200 dense BF16 peak"
WORKLOADS = {
    "fwd_bwd_b8_h16_n2048_d128_causal": dict(cfg=2, B=8, H=16, N=2048, d=128, causal=True),
    "fwd_b8_h32_n2048_d64": dict(cfg=1, B=8, H=32, N=2048, d=64, causal=False),
    "fwd_bwd_b1_h16_n16384_d128_causal": dict(cfg=3, B=1, H=16, N=16384, d=128, causal=True),
}
DEFAULT_WORKLOAD = "fwd_bwd_b8_h16_n2048_d128_causal"
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
    """nvidia-smi clocks and throttle reasons, sampled every 50 ms in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: str):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(device_index)],
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

    def summary(self, t0: float, t1: float):
        inside = [p for t, p in self.samples if t0 <= t <= t1]
        used = inside
        if not used:  # timed region shorter than one sample period: nearest samples
            used = [p for t, p in self.samples if t0 - 0.2 <= t <= t1 + 0.2]
        if not used:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"],
                    "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        mhz = []
        for p in used:
            try:
                mhz.append(float(p[1]))
            except ValueError:
                pass
            for name, val in zip(names, p[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
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
def oracle_sample(w, host, max_seconds: float):
    """Times the fp64 oracle (fwd + full bwd) on whole heads of this workload,
    adding heads until about max_seconds of CPU work; returns (TFLOP/s, desc, threads)."""
    import oracle

    oracle.build()
    threads = oracle.default_threads()
    scale = 1.0 / math.sqrt(w["d"])
    per_head = dict(w, B=1, H=1)
    done, elapsed = 0, 0.0
    total_heads = w["B"] * w["H"]
    while done < total_heads and elapsed < max_seconds:
        b, h = divmod(done, w["H"])
        t0 = time.perf_counter()
        if w["N"] <= 4096:
            oracle.attention_backward(host["q"][b, h], host["k"][b, h], host["v"][b, h],
                                      host["do"][b, h], w["causal"], scale, nthreads=threads)
        else:  # forward of the whole head plus dQ/dK/dV of 8 rows (the sampled-row path)
            rows = [0, 1, w["N"] // 2, w["N"] - 1]
            oracle.attention_backward_rows(host["q"][b, h], host["k"][b, h], host["v"][b, h],
                                           host["do"][b, h], w["causal"], scale, rows, rows,
                                           nthreads=threads)
        elapsed += time.perf_counter() - t0
        done += 1
    if w["N"] <= 4096:
        fl = flops(per_head, "fwd+bwd") * done
        desc = f"{done} of {total_heads} heads, full fwd+bwd in fp64"
    else:
        fl = flops(per_head, "fwd") * done
        desc = f"{done} of {total_heads} heads, fp64 forward of every row (+4 gradient rows)"
    return fl / elapsed / 1e12, desc, threads, elapsed


def run_reference(args, w, rank: int):
    if rank != 0:
        return
    host = make_inputs(w, 0)
    import oracle

    oracle.build()
    threads = oracle.default_threads()
    scale = 1.0 / math.sqrt(w["d"])
    per_head = dict(w, B=1, H=1)

    def step(i):
        b, h = divmod(i % (w["B"] * w["H"]), w["H"])
        oracle.attention_backward(host["q"][b, h], host["k"][b, h], host["v"][b, h],
                                  host["do"][b, h], w["causal"], scale, nthreads=threads)

    if w["N"] > 4096:
        print(json.dumps({"impl": "reference", "unavailable":
                          "the fp64 oracle's full backward needs N x N memory per head at this N"}))
        return
    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = time.perf_counter() - t0
    value = flops(per_head, "fwd+bwd") * args.steps / dt / 1e12
    sample = f"one head ({w['N']}x{w['d']}, causal={w['causal']}) of the workload per step, fp64"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
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
    d in {64, 128}, N in 512 .. 16k with B = 16384 / N, causal and not."""
    pts = []
    for d in (64, 128):
        for causal in (False, True):
            for N in (512, 1024, 2048, 4096, 8192, 16384):
                pts.append({"B": 16384 // N, "H": 2048 // d, "N": N, "d": d, "causal": causal})
    return pts


def run_grid(args):
    """One JSON line per grid point: forward, backward (three kernels) and their sum
    in TFLOP/s on device-resident random bf16 inputs, CUDA events around `reps`
    calls after warm-up (not the contract line; the contract line is the default
    run)."""
    import torch

    import exact_tiled_attention_30_b200 as fa2

    fa2.load_library()
    peaks, _ = load_peaks()
    reps = max(args.steps // 40, 5)
    for w in grid_points():
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
        for name, fn in (("fwd", fwd), ("bwd", bwd)):
            for _ in range(args.warmup):
                fn()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                fn()
            e1.record()
            torch.cuda.synchronize()
            res[name] = e0.elapsed_time(e1) / reps
        res["fwd+bwd"] = res["fwd"] + res["bwd"]
        line = {"grid": True, **w}
        for name, ms in res.items():
            tf = flops(w, name) / (ms * 1e-3) / 1e12
            line[name] = {"ms": round(ms, 4), "tflops": round(tf, 1),
                          "frac": round(tf / peaks["bf16_tflops"], 3)}
        print(json.dumps(line), flush=True)
        del q, k, v, do, o, lse, dq, dk, dv, ws
        torch.cuda.empty_cache()


# --------------------------------------------------------------- GPU timing
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--grid", action="store_true",
                    help="time every point of the benchmark-figure grid (1 GPU), one JSON line each")
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
        "e2e": {"value": fl_step / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
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
