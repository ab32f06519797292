"""Guard regions around every buffer the library writes.

compute-sanitizer is not available for these tests, so out-of-bounds writes are
looked for the plain way: each output (O, LSE, dQ, dK, dV) and the backward
workspace is carved out of the middle of a larger buffer whose margins hold a
known byte pattern; after a forward and a backward the margins must be intact,
and the outputs must still match the fp64 oracle. Ragged lengths put the last
tile's padding rows right next to the margin.
"""
import math

import numpy as np
import pytest

from tests import gpu_helpers as gh

pytestmark = pytest.mark.gpu

MARGIN = 64 * 1024  # bytes before and after each buffer (a multiple of 512: alignment kept)
PATTERN = 0xA5


@pytest.fixture(scope="module")
def fa2():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_tiled_attention_30_b200 as m

    m.load_library()
    m.fa2_clear_device_status()
    return m


class Guarded:
    """A tensor of `shape`/`dtype` inside a byte buffer with patterned margins."""

    def __init__(self, shape, dtype):
        import torch

        self.nbytes = math.prod(shape) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((MARGIN + self.nbytes + MARGIN,), PATTERN, dtype=torch.uint8,
                              device="cuda")
        self.t = self.raw[MARGIN:MARGIN + self.nbytes].view(dtype).view(shape)

    def margins_intact(self) -> bool:
        head = self.raw[:MARGIN]
        tail = self.raw[MARGIN + self.nbytes:]
        return bool((head == PATTERN).all().item() and (tail == PATTERN).all().item())


CASES = [
    # cfg, B, H, Nq, Nk, d, causal
    (50, 1, 2, 300, 300, 64, True),
    (51, 2, 1, 129, 129, 128, False),
    (52, 1, 1, 1, 1, 128, True),
    (53, 1, 2, 200, 333, 128, True),   # different lengths, ragged both
    (54, 2, 2, 384, 127, 64, False),
]


@pytest.mark.parametrize("cfg,B,H,Nq,Nk,d,causal", CASES)
def test_writes_stay_inside_their_buffers(fa2, oracle_mod, cfg, B, H, Nq, Nk, d, causal):
    import torch

    tq = gh.inputs(cfg, B, H, Nq, d, with_do=True)
    tk = gh.inputs(cfg + 500, B, H, Nk, d)
    t = {"q": tq["q"], "do": tq["do"], "k": tk["k"], "v": tk["v"]}
    q, k, v, do = (gh.to_device(t[n]) for n in ("q", "k", "v", "do"))
    scale = 1.0 / math.sqrt(d)
    out = {
        "o": Guarded((B, H, Nq, d), torch.bfloat16),
        "lse": Guarded((B, H, Nq), torch.float32),
        "dq": Guarded((B, H, Nq, d), torch.bfloat16),
        "dk": Guarded((B, H, Nk, d), torch.bfloat16),
        "dv": Guarded((B, H, Nk, d), torch.bfloat16),
        "ws": Guarded((fa2.fa2_backward_workspace_size(B, H, Nq, d),), torch.uint8),
    }
    o, lse, dq, dk, dv, ws = (out[n].t for n in ("o", "lse", "dq", "dk", "dv", "ws"))
    if Nq == Nk:
        fa2.fa2_forward(q, k, v, o, lse, causal, scale)
        fa2.fa2_backward(q, k, v, o, lse, do, dq, dk, dv, causal, scale, ws)
    else:
        fa2.fa2_forward_qk(q, k, v, o, lse, causal, scale)
        fa2.fa2_backward_qk(q, k, v, o, lse, do, dq, dk, dv, causal, scale, ws)
    torch.cuda.synchronize()
    st, site = fa2.fa2_get_device_status()
    assert st == 0, f"device status {fa2.fa2_status_string(st)} at site {site:#x}"
    for name, g in out.items():
        assert g.margins_intact(), f"a write landed outside {name}"

    ref = oracle_mod.attention_backward(t["q"], t["k"], t["v"], t["do"], causal, scale)
    where = f"guard regions shape={tuple(t['q'].shape)} keys={tuple(t['k'].shape)} causal={causal}"
    gh.check_o(gh.to_host_f64(o), ref["o"], where)
    gh.check_lse(gh.to_host_f64(lse), ref["lse"], where)
    for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
        gh.check_grad(name, gh.to_host_f64(got), ref[name], where)
