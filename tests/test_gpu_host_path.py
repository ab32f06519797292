"""The host-buffer entry point (fa2_forward_backward_host) against the fp64
oracle and against the device-buffer path, through the C ABI.

Chunking by heads must not change any result: O, LSE, dK and dV are compared
bit for bit with fa2_forward / fa2_backward on device copies of the same
inputs (the same kernels run per chunk); dQ, which is accumulated with
floating-point reductions in no fixed order, within 1e-4 relative. Tolerances
against the oracle as in the other parity tests.
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


def host_bf16(bits):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.pin_memory()


CASES = [
    # cfg, B, H, N, d, causal, heads_per_chunk
    (30, 2, 3, 200, 64, True, 0),     # 6 heads, one per chunk
    (30, 2, 3, 200, 64, True, 4),     # ragged last chunk (4 + 2)
    (31, 1, 5, 129, 128, False, 2),   # ragged tail of rows and of chunks
    (32, 1, 4, 384, 128, True, 4),    # one chunk holds every head
]


@pytest.mark.parametrize("cfg,B,H,N,d,causal,hpc", CASES)
def test_host_path_matches_device_path_and_oracle(fa2, oracle_mod, cfg, B, H, N, d, causal, hpc):
    import torch

    t = gh.inputs(cfg, B, H, N, d, with_do=True)
    scale = 1.0 / math.sqrt(d)
    hq, hk, hv, hdo = (host_bf16(t[n]) for n in ("q", "k", "v", "do"))
    o, lse, dq, dk, dv = fa2.attention_forward_backward_host(hq, hk, hv, hdo, causal=causal,
                                                             scale=scale, heads_per_chunk=hpc)
    torch.cuda.current_stream().synchronize()
    st, site = fa2.fa2_get_device_status()
    assert st == 0, f"device status {fa2.fa2_status_string(st)} at site {site:#x}"

    # device path on the same inputs
    q, k, v, do = (x.cuda() for x in (hq, hk, hv, hdo))
    o_d, lse_d = fa2.attention_forward(q, k, v, causal=causal, scale=scale)
    dq_d, dk_d, dv_d = fa2.attention_backward(q, k, v, o_d, lse_d, do, causal=causal, scale=scale)
    assert torch.equal(o, o_d.cpu())
    assert torch.equal(lse, lse_d.cpu())
    assert torch.equal(dk, dk_d.cpu()) and torch.equal(dv, dv_d.cpu())
    assert gh.rel_fro(gh.to_host_f64(dq), gh.to_host_f64(dq_d)) < 1e-4

    # oracle
    ref_o, ref_lse = oracle_mod.attention_forward(t["q"], t["k"], t["v"], causal, scale)
    where = f"host-buffer entry shape={tuple(t['q'].shape)} causal={causal}"
    gh.check_o(gh.to_host_f64(o), ref_o, where)
    gh.check_lse(lse.numpy().astype(np.float64), ref_lse, where)
    ref = oracle_mod.attention_backward(t["q"], t["k"], t["v"], t["do"], causal, scale)
    for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
        gh.check_grad(name, gh.to_host_f64(got), ref[name], where)


def test_host_path_orders_with_the_callers_stream(fa2):
    """Work queued on the caller's stream before the call is seen by it, and the
    outputs are complete once the stream has passed the call."""
    import torch

    B, H, N, d = 1, 4, 256, 64
    t = gh.inputs(33, B, H, N, d, with_do=True)
    hq, hk, hv, hdo = (host_bf16(t[n]) for n in ("q", "k", "v", "do"))
    s = torch.cuda.Stream()
    ws = torch.empty(fa2.fa2_forward_backward_host_workspace_size(B, H, N, d, 1), dtype=torch.uint8,
                     device="cuda")
    with torch.cuda.stream(s):
        ws.fill_(0xFF)  # queued before the call on the same stream
        out = fa2.attention_forward_backward_host(hq, hk, hv, hdo, causal=True, heads_per_chunk=1,
                                                  workspace=ws, stream=s)
    s.synchronize()
    q, k, v, do = (x.cuda() for x in (hq, hk, hv, hdo))
    o_d, lse_d = fa2.attention_forward(q, k, v, causal=True)
    assert torch.equal(out[0], o_d.cpu()) and torch.equal(out[1], lse_d.cpu())
