"""CUDA-graph capture of a forward + backward step through the C ABI.

Once the one-time per-device setup has run (an eager call), a call of
fa2_forward or fa2_backward issues only stream work: a 4-byte memset of the
forward's work counter and the kernel launches. A step captured into a graph
and replayed must therefore give the eager results, read whatever the static
input buffers hold at replay time, and match the fp64 oracle (same tolerances
as the other parity tests: O max-abs 1e-2, LSE 1e-3, gradients 2e-2 relative
Frobenius).
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


def check_against_oracle(oracle_mod, t, got, causal, scale):
    ref = oracle_mod.attention_backward(t["q"], t["k"], t["v"], t["do"], causal, scale)
    where = f"graph replay shape={tuple(t['q'].shape)} causal={causal}"
    gh.check_o(gh.to_host_f64(got["o"]), ref["o"], where)
    gh.check_lse(got["lse"].cpu().numpy().astype(np.float64), ref["lse"], where)
    for name in ("dq", "dk", "dv"):
        gh.check_grad(name, gh.to_host_f64(got[name]), ref[name], where)


@pytest.mark.parametrize("d,causal", [(64, False), (128, True)])
def test_graph_replay_matches_eager_and_oracle(fa2, oracle_mod, d, causal):
    import torch

    B, H, N = 2, 2, 300  # three query and key tiles, ragged last tile
    scale = 1.0 / math.sqrt(d)
    t1 = gh.inputs(19, B, H, N, d, with_do=True)
    t2 = gh.inputs(20, B, H, N, d, with_do=True)
    q, k, v, do = (gh.to_device(t1[n]) for n in ("q", "k", "v", "do"))
    out = {"o": torch.empty_like(q),
           "lse": torch.empty((B, H, N), dtype=torch.float32, device=q.device),
           "dq": torch.empty_like(q), "dk": torch.empty_like(q), "dv": torch.empty_like(q)}
    ws = torch.empty(fa2.fa2_backward_workspace_size(B, H, N, d), dtype=torch.uint8,
                     device=q.device)

    def step():
        fa2.fa2_forward(q, k, v, out["o"], out["lse"], causal, scale)
        fa2.fa2_backward(q, k, v, out["o"], out["lse"], do, out["dq"], out["dk"], out["dv"],
                         causal, scale, ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()  # eager: the one-time device setup happens here, outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    eager = {n: x.clone() for n, x in out.items()}

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for x in out.values():
        x.zero_()
    graph.replay()
    torch.cuda.synchronize()
    st, site = fa2.fa2_get_device_status()
    assert st == 0, f"device status {fa2.fa2_status_string(st)} at site {site:#x}"
    # the forward has no atomics: the same bits as eager; the gradients to well
    # inside their tolerance (dQ is summed by fp32 reductions in varying order)
    for name in ("o", "lse"):
        assert torch.equal(out[name], eager[name]), f"{name} differs from the eager call"
    for name in ("dq", "dk", "dv"):
        e = gh.rel_fro(gh.to_host_f64(out[name]), gh.to_host_f64(eager[name]))
        assert e <= 1e-3, f"{name} differs from the eager call by {e:.3e}"
    check_against_oracle(oracle_mod, t1, out, causal, scale)

    # new contents in the same buffers: the replay reads them
    for x, n in ((q, "q"), (k, "k"), (v, "v"), (do, "do")):
        x.copy_(gh.to_device(t2[n]))
    graph.replay()
    torch.cuda.synchronize()
    check_against_oracle(oracle_mod, t2, out, causal, scale)
    del graph
