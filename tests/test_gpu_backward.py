"""Backward parity of the sm_100a kernels against the fp64 oracle, through the C ABI.

The GPU backward consumes the GPU forward's bf16 O and fp32 LSE (as a user
would); the oracle computes everything in fp64 from the same bf16 inputs.
Tolerance (written here, from the stated bar): relative Frobenius error
||g_gpu - g_ref|| / ||g_ref|| <= 2e-2 for each of dQ, dK, dV. Small shapes are
checked in full; long sequences on sampled heads and rows, which the oracle
computes one by one.
"""
import math

import numpy as np
import pytest

from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa2():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_tiled_attention_30_b200 as m

    m.load_library()
    m.fa2_clear_device_status()
    return m


STRATEGIES = pytest.mark.parametrize("strategy", [1, 2], ids=["reduce", "separate"])


def run_fwd_bwd(fa2, t, causal, scale, strategy=0):
    q, k, v, do = (gh.to_device(t[n]) for n in ("q", "k", "v", "do"))
    o, lse = fa2.attention_forward(q, k, v, causal=causal, scale=scale)
    dq, dk, dv = fa2.attention_backward(q, k, v, o, lse, do, causal=causal, scale=scale,
                                        dq_strategy=strategy)
    st, site = fa2.fa2_get_device_status()
    assert st == 0, f"device status {fa2.fa2_status_string(st)} at site {site:#x}"
    return {"dq": gh.to_host_f64(dq), "dk": gh.to_host_f64(dk), "dv": gh.to_host_f64(dv),
            "o": gh.to_host_f64(o)}


def check_grads(got: dict, ref: dict, where=""):
    for name in ("dq", "dk", "dv"):
        gh.check_grad(name, got[name], ref[name], where)


SMALL = [
    (0, 1, 2, 128, 64, False),   # tiny workload: B=1 H=2 N=128 d=64
    (0, 1, 2, 128, 64, True),
    (0, 1, 2, 128, 128, False),
    (12, 2, 1, 12, 64, True),    # twelve-token walk-through shape
    (13, 1, 2, 127, 128, True),
    (13, 1, 2, 127, 64, False),
    (14, 2, 2, 129, 64, True),
    (14, 2, 2, 129, 128, False),
    (15, 1, 2, 1000, 128, True),
    (15, 1, 2, 1000, 64, False),
    (16, 2, 3, 384, 128, True),
    (16, 2, 3, 384, 64, True),
    (16, 2, 3, 384, 128, False),
    (17, 4, 80, 300, 128, True),  # several items per CTA, ragged N
    (17, 4, 80, 300, 64, False),
]


@STRATEGIES
@pytest.mark.parametrize("cfg,B,H,N,d,causal", SMALL)
def test_backward_small(fa2, oracle_mod, cfg, B, H, N, d, causal, strategy):
    t = gh.inputs(cfg, B, H, N, d, with_do=True)
    scale = 1.0 / math.sqrt(d)
    got = run_fwd_bwd(fa2, t, causal, scale, strategy)
    ref = oracle_mod.attention_backward(t["q"], t["k"], t["v"], t["do"], causal, scale)
    where = f"backward B={B} H={H} N={N} d={d} causal={causal} dq_strategy={strategy}"
    check_grads(got, ref, where)
    # per-head too, so that one wrong head cannot hide in the global norm
    for b in range(B):
        for h in range(H):
            check_grads({n: got[n][b, h] for n in ("dq", "dk", "dv")},
                        {n: ref[n][b, h] for n in ("dq", "dk", "dv")}, f"{where} head ({b},{h})")


@STRATEGIES
@pytest.mark.parametrize("d", [64, 128])
def test_backward_single_token(fa2, d, strategy):
    """N = 1: dV = dO exactly, dQ = dK = 0 up to rounding."""
    t = gh.inputs(11, 2, 2, 1, d, with_do=True)
    got = run_fwd_bwd(fa2, t, True, 1.0 / math.sqrt(d), strategy)
    np.testing.assert_array_equal(got["dv"], gh.to_host_f64(gh.to_device(t["do"])))
    assert np.abs(got["dq"]).max() <= 1e-3 and np.abs(got["dk"]).max() <= 1e-3


@STRATEGIES
def test_backward_scale_zero(fa2, oracle_mod, strategy):
    t = gh.inputs(17, 1, 2, 200, 64, with_do=True)
    got = run_fwd_bwd(fa2, t, True, 0.0, strategy)
    ref = oracle_mod.attention_backward(t["q"], t["k"], t["v"], t["do"], True, 0.0)
    for name in ("dk", "dv"):
        assert np.isfinite(got[name]).all()
    np.testing.assert_array_equal(got["dq"], 0.0)  # scale multiplies dQ and dK
    np.testing.assert_array_equal(got["dk"], 0.0)
    assert gh.rel_fro(got["dv"], ref["dv"]) <= gh.GRAD_RTOL


def test_backward_workspace_reuse(fa2):
    """The workspace content on entry does not matter (it is re-initialised each call)."""
    import torch

    t = gh.inputs(19, 1, 2, 256, 128, with_do=True)
    q, k, v, do = (gh.to_device(t[n]) for n in ("q", "k", "v", "do"))
    o, lse = fa2.attention_forward(q, k, v, causal=True)
    ws = torch.full((fa2.fa2_backward_workspace_size(1, 2, 256, 128),), 0x7F, dtype=torch.uint8,
                    device="cuda")
    a = fa2.attention_backward(q, k, v, o, lse, do, causal=True, workspace=ws)
    b = fa2.attention_backward(q, k, v, o, lse, do, causal=True, workspace=ws)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


LARGE_FULL_HEADS = [
    # forward+backward workload: B=8 H=16 N=2048 d=128 causal; whole sampled heads
    (2, 8, 16, 2048, 128, True),
    # benchmark-grid points (hidden 2048, 16k tokens): d=64 N=2048 B=8 H=32 non-causal
    (4, 8, 32, 2048, 64, False),
]


@STRATEGIES
@pytest.mark.parametrize("cfg,B,H,N,d,causal", LARGE_FULL_HEADS)
def test_backward_large_heads(fa2, oracle_mod, cfg, B, H, N, d, causal, strategy):
    t = gh.inputs(cfg, B, H, N, d, with_do=True)
    scale = 1.0 / math.sqrt(d)
    got = run_fwd_bwd(fa2, t, causal, scale, strategy)
    for b, h in gh.sample_heads(B, H, 2, seed=cfg):
        ref = oracle_mod.attention_backward(t["q"][b, h], t["k"][b, h], t["v"][b, h],
                                            t["do"][b, h], causal, scale)
        check_grads({n: got[n][b, h] for n in ("dq", "dk", "dv")}, ref,
                    f"backward B={B} H={H} N={N} d={d} causal={causal} dq_strategy={strategy} "
                    f"head ({b},{h})")


LONG_ROWS = [
    # long context: B=1 H=16 N=16384 d=128 causal, sampled rows of one head
    (3, 1, 16, 16384, 128, True),
    # benchmark grid: N=8192, d=64, B=2, H=32, non-causal
    (4, 2, 32, 8192, 64, False),
]


@STRATEGIES
@pytest.mark.parametrize("cfg,B,H,N,d,causal", LONG_ROWS)
def test_backward_long_sampled_rows(fa2, oracle_mod, cfg, B, H, N, d, causal, strategy):
    t = gh.inputs(cfg, B, H, N, d, with_do=True)
    scale = 1.0 / math.sqrt(d)
    got = run_fwd_bwd(fa2, t, causal, scale, strategy)
    rows = gh.sample_rows(N, 48, seed=cfg)
    (b, h), = gh.sample_heads(B, H, 1, seed=cfg)[-1:]
    dq, dk, dv = oracle_mod.attention_backward_rows(t["q"][b, h], t["k"][b, h], t["v"][b, h],
                                                    t["do"][b, h], causal, scale, rows, rows)
    check_grads({"dq": got["dq"][b, h, rows], "dk": got["dk"][b, h, rows],
                 "dv": got["dv"][b, h, rows]}, {"dq": dq, "dk": dk, "dv": dv},
                f"backward B={B} H={H} N={N} d={d} causal={causal} dq_strategy={strategy} "
                f"head ({b},{h}) sampled rows")


def test_separate_dq_is_bitwise_repeatable(fa2):
    """The query-parallel dQ kernel has no atomics: repeated runs give identical dQ."""
    import torch

    t = gh.inputs(22, 2, 4, 640, 128, with_do=True)
    q, k, v, do = (gh.to_device(t[n]) for n in ("q", "k", "v", "do"))
    o, lse = fa2.attention_forward(q, k, v, causal=True)
    ref = fa2.attention_backward(q, k, v, o, lse, do, causal=True, dq_strategy=fa2.DQ_SEPARATE)
    for _ in range(5):
        got = fa2.attention_backward(q, k, v, o, lse, do, causal=True, dq_strategy=fa2.DQ_SEPARATE)
        for a, b in zip(got, ref):
            assert torch.equal(a, b)


def test_strategies_agree(fa2):
    """Both dQ strategies produce the same dK, dV bits and dQ within rounding."""
    t = gh.inputs(23, 1, 4, 768, 64, with_do=True)
    q, k, v, do = (gh.to_device(t[n]) for n in ("q", "k", "v", "do"))
    o, lse = fa2.attention_forward(q, k, v, causal=False)
    a = fa2.attention_backward(q, k, v, o, lse, do, dq_strategy=fa2.DQ_REDUCE)
    b = fa2.attention_backward(q, k, v, o, lse, do, dq_strategy=fa2.DQ_SEPARATE)
    import torch

    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert gh.rel_fro(gh.to_host_f64(a[0]), gh.to_host_f64(b[0])) < 5e-3


@pytest.mark.parametrize("N,d,causal", [(3, 64, True), (2, 128, False)])
def test_maximum_head_count(fa2, oracle_mod, N, d, causal):
    """B*H = 65535, the largest the library accepts (one grid dimension of the
    streaming kernels; 65535 work items for each attention kernel): every head is
    computed, checked on sampled heads. Short sequences keep the inputs small."""
    import torch

    B, H = 65535, 1
    t = gh.inputs(47, B, H, N, d, with_do=True)
    scale = 1.0 / math.sqrt(d)
    got = run_fwd_bwd(fa2, t, causal, scale)
    torch.cuda.synchronize()
    for b, h in gh.sample_heads(B, H, 6, seed=N):
        ref = oracle_mod.attention_backward(t["q"][b, h], t["k"][b, h], t["v"][b, h],
                                            t["do"][b, h], causal, scale)
        gh.check_o(got["o"][b, h], ref["o"], f"B*H=65535 N={N} d={d} head ({b},{h})")
        check_grads({n: got[n][b, h] for n in ("dq", "dk", "dv")}, ref,
                    f"B*H=65535 N={N} d={d} causal={causal} head ({b},{h})")
