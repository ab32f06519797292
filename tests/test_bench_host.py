"""Host-side pieces of bench.py: FLOP counts, peaks, the ncu traffic record, the
per-rank seeds, the max-over-ranks timing reduction (world size 2 over gloo), the
benchmark-figure grid and the reference arm's JSON line."""
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_flop_counts():
    w = dict(B=8, H=16, N=2048, d=128, causal=True)
    fwd = 4.0 * 8 * 16 * 2048 ** 2 * 128
    assert bench.flops(w, "fwd") == fwd / 2
    assert bench.flops(w, "bwd") == 2.5 * fwd / 2
    assert bench.flops(w, "fwd+bwd") == 3.5 * fwd / 2
    assert bench.flops(w, "fwd+bwd", halve_causal=False) == 3.5 * fwd
    assert bench.flops(dict(w, causal=False), "fwd") == fwd


def test_default_workload_is_the_longest_forward_backward():
    """The contract line runs the largest single-GPU forward+backward workload:
    B=1 H=16 N=16384 d=128 causal (the benchmark's longest sequence)."""
    w = bench.WORKLOADS[bench.DEFAULT_WORKLOAD]
    assert (w["B"], w["H"], w["N"], w["d"], w["causal"]) == (1, 16, 16384, 128, True)


def test_clock_summary_is_null_without_samples_inside():
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    row = ["0", "1965", "1965", "300.0", "0x0", "Not Active", "Not Active", "Not Active", "Active"]
    s.samples = [(10.0, row), (10.5, row)]
    out = s.summary(10.1, 10.2)  # no sample inside the timed region
    assert out["sm_mhz"] is None and out["sm_max_mhz"] is None and out["samples"] == 0
    assert out["reasons_nearby"] == ["sw_power_cap"]
    out = s.summary(9.9, 10.6)
    assert out["sm_mhz"] == 1965.0 and out["samples"] == 2 and out["reasons"] == ["sw_power_cap"]


def test_row_sampled_oracle_flop_count(monkeypatch):
    """Heads longer than the full-backward limit: forward of every row (4 d per
    visible pair) + dQ rows (6 d) + dK, dV rows (8 d), counted exactly."""
    import numpy as np

    import attn_inputs

    monkeypatch.setattr(bench, "FULL_BACKWARD_MAX_N", 64)
    monkeypatch.setattr(bench, "SAMPLED_GRAD_ROWS", 4)
    N, d = 200, 64
    w = dict(B=1, H=1, N=N, d=d, causal=True)
    host = attn_inputs.make_qkvdo(9, 1, 1, N, d)
    secs, fl, desc = bench.oracle_head(w, host, 0, 2)
    rows = [int(x) for x in np.linspace(0, N - 1, 4).round()]
    want = 4 * d * N * (N + 1) // 2 + sum(6 * d * (i + 1) for i in rows) + \
        sum(8 * d * (N - j) for j in rows)
    assert fl == want and secs > 0 and "dQ of 4 query rows" in desc


def test_peaks_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, kind = bench.load_peaks()
    assert kind == "fallback" and peaks["bf16_tflops"] == 1590.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}))
    peaks, kind = bench.load_peaks()
    assert kind == "measured" and peaks["bf16_tflops"] == 1600.0


def test_traffic_record_is_dropped_when_the_kernel_changes(tmp_path, monkeypatch):
    real = bench.kernel_src_hash("fa2_bwd_kernel")
    prof = tmp_path / "profiles"
    prof.mkdir()
    rec = {"fa2_bwd_kernel": {"dram_bytes_per_launch": 123, "workload": "w", "src_hash": real}}
    (prof / "ncu_traffic.json").write_text(json.dumps(rec))
    csrc = os.path.join(bench.ROOT, "exact_tiled_attention_30_b200", "csrc")
    os.makedirs(tmp_path / "exact_tiled_attention_30_b200")
    os.symlink(csrc, tmp_path / "exact_tiled_attention_30_b200" / "csrc")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic("fa2_bwd_kernel", "w") == 123
    assert bench.ncu_traffic("fa2_bwd_kernel", "other workload") is None
    rec["fa2_bwd_kernel"]["src_hash"] = "0" * 16
    (prof / "ncu_traffic.json").write_text(json.dumps(rec))
    assert bench.ncu_traffic("fa2_bwd_kernel", "w") is None


def test_ranks_draw_independent_batches():
    seeds = {bench.rank_config_index(2, r) for r in range(8)}
    assert len(seeds) == 8
    w = dict(bench.WORKLOADS[bench.DEFAULT_WORKLOAD], B=1, H=1, N=16, d=64)
    a, b = bench.make_inputs(w, 0), bench.make_inputs(w, 1)
    assert not (a["q"] == b["q"]).all()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 0.5 * rank], dist, "cpu")
        out[rank] = got
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world_size_2():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == [2.0, 10.0, 0.5]


def test_max_over_ranks_single_process():
    assert bench.max_over_ranks([3, 4.5]) == [3.0, 4.5]


def test_grid_points_mirror_the_benchmark_axes():
    import bench

    pts = [p for p in bench.grid_points() if not p.get("ragged")]
    assert len(pts) == 24  # x 3 passes (fwd, bwd, fwd+bwd) = 72 measurements
    assert {p["d"] for p in pts} == {64, 128} and {p["causal"] for p in pts} == {False, True}
    assert sorted({p["N"] for p in pts}) == [512, 1024, 2048, 4096, 8192, 16384]
    for p in pts:
        assert p["B"] * p["N"] == 16384 and p["H"] * p["d"] == 2048
    ragged = [p for p in bench.grid_points() if p.get("ragged")]
    assert {(p["N"], p["causal"]) for p in ragged} == {(2000, False), (2000, True), (4000, False),
                                                       (4000, True)}
    assert all(p["N"] % 128 for p in ragged)


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` runs the oracle on the host and prints one JSON
    line with the contract's keys (no GPU involved)."""
    import json
    import subprocess
    import sys

    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in rec, key
    assert rec["impl"] == "reference" and rec["steps"] == 1 and rec["warmup"] == 3
    assert rec["metric"] == bench.METRIC and rec["unit"] == "TFLOP/s"
    assert rec["value"] > 0 and rec["higher_is_better"] is True
    assert rec["config"]["workload"] == bench.DEFAULT_WORKLOAD
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] >= 1
    assert rec["e2e"]["value"] == rec["value"]
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_under_two_ranks_prints_from_rank_zero_only():
    """Launched like the multi-GPU bench (torch.distributed.run, two ranks), the
    reference arm runs on rank 0 alone; the other rank exits 0 without work."""
    import subprocess
    import sys

    port = _free_port()
    out = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                          "--nproc-per-node", "2", "--master-addr", "127.0.0.1", "--master-port",
                          str(port), os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "fwd_bwd_b8_h16_n2048_d128_causal",
                          "--gpus", "2", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
