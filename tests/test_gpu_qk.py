"""Different query and key lengths (Nq != Nk) through the C ABI against the fp64
oracle: forward O/LSE and backward dQ/dK/dV, causal masks aligned to the
bottom-right corner (query i sees keys j <= i + Nk - Nq). Tolerances as in the
other parity tests. With Nq = Nk the _qk entry points must give the bits of the
square ones.
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


def qk_inputs(cfg, B, H, Nq, Nk, d):
    """Seeded q, dO with Nq rows and k, v with Nk rows (same generator as the other tests)."""
    tq = gh.inputs(cfg, B, H, Nq, d, with_do=True)
    tk = gh.inputs(cfg + 500, B, H, Nk, d)
    return {"q": tq["q"], "do": tq["do"], "k": tk["k"], "v": tk["v"]}


CASES = [
    # cfg, B, H, Nq, Nk, d, causal
    (40, 1, 2, 200, 333, 64, True),     # more keys than queries, ragged both
    (41, 2, 1, 129, 128, 128, False),   # more queries than keys (non-causal)
    (42, 1, 2, 256, 1000, 128, True),   # query tiles start deep in the key range
    (43, 1, 3, 384, 127, 64, False),
    (44, 1, 1, 1, 300, 128, True),      # one query: sees every key
    (45, 2, 2, 640, 700, 128, True),
]


@pytest.mark.parametrize("cfg,B,H,Nq,Nk,d,causal", CASES)
def test_qk_forward_backward(fa2, oracle_mod, cfg, B, H, Nq, Nk, d, causal):
    import torch

    t = qk_inputs(cfg, B, H, Nq, Nk, d)
    scale = 1.0 / math.sqrt(d)
    q, k, v, do = (gh.to_device(t[n]) for n in ("q", "k", "v", "do"))
    o, lse = fa2.attention_forward(q, k, v, causal=causal, scale=scale)
    dq, dk, dv = fa2.attention_backward(q, k, v, o, lse, do, causal=causal, scale=scale)
    torch.cuda.synchronize()
    st, site = fa2.fa2_get_device_status()
    assert st == 0, f"device status {fa2.fa2_status_string(st)} at site {site:#x}"
    assert dq.shape == q.shape and dk.shape == k.shape and dv.shape == v.shape
    ref = oracle_mod.attention_backward(t["q"], t["k"], t["v"], t["do"], causal, scale)
    where = f"Nq={Nq} Nk={Nk} B={B} H={H} d={d} causal={causal}"
    gh.check_o(gh.to_host_f64(o), ref["o"], where)
    gh.check_lse(gh.to_host_f64(lse), ref["lse"], where)
    for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
        gh.check_grad(name, gh.to_host_f64(got), ref[name], where)


@pytest.mark.parametrize("causal", [False, True])
def test_qk_equal_lengths_match_square_path(fa2, causal):
    import torch

    B, H, N, d = 1, 2, 300, 128
    t = gh.inputs(46, B, H, N, d, with_do=True)
    q, k, v, do = (gh.to_device(t[n]) for n in ("q", "k", "v", "do"))
    o1, l1 = fa2.attention_forward(q, k, v, causal=causal)
    o2, l2 = torch.empty_like(o1), torch.empty_like(l1)
    fa2.fa2_forward_qk(q, k, v, o2, l2, causal, d ** -0.5)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    g1 = fa2.attention_backward(q, k, v, o1, l1, do, causal=causal)
    g2 = [torch.empty_like(q) for _ in range(3)]
    ws = torch.empty(fa2.fa2_backward_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
    fa2.fa2_backward_qk(q, k, v, o1, l1, do, *g2, causal, d ** -0.5, ws)
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
    assert gh.rel_fro(gh.to_host_f64(g1[0]), gh.to_host_f64(g2[0])) < 1e-4
