"""Pins the oracle to PyTorch's attention on the CPU, in fp64.

The method's result is that of standard attention ("FlashAttention (v2)"
glossary page, definition and results paragraphs), so a library routine of
standard attention is an independent reference: O from
torch.nn.functional.scaled_dot_product_attention, LSE from torch.logsumexp of
the scaled, masked scores, and dQ, dK, dV from autograd through the same call.
The oracle shares no code with either. Masks use the bottom-right alignment of
the oracle's different-length reading (query i sees keys j <= i + Nk - Nq),
passed to PyTorch as an explicit boolean mask.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import attn_inputs

TOL = 1e-10

CASES = [
    # B, H, Nq, Nk, d, causal
    (1, 2, 7, 7, 8, False),
    (1, 2, 7, 7, 8, True),
    (2, 1, 33, 33, 16, True),
    (1, 1, 1, 1, 4, True),
    (1, 1, 5, 9, 4, True),
    (1, 2, 9, 5, 8, False),
    (1, 1, 130, 130, 64, True),
    (1, 1, 40, 97, 32, True),
]


def inputs(seed, B, H, Nq, Nk, d):
    def f64(bits):
        return attn_inputs.bf16_bits_to_f64(bits)

    return {"q": f64(attn_inputs.normal_bf16(seed, (B, H, Nq, d))),
            "k": f64(attn_inputs.normal_bf16(seed + 1, (B, H, Nk, d))),
            "v": f64(attn_inputs.normal_bf16(seed + 2, (B, H, Nk, d))),
            "do": f64(attn_inputs.normal_bf16(seed + 3, (B, H, Nq, d)))}


def torch_reference(t, causal, scale):
    q, k, v = (torch.tensor(t[n], dtype=torch.float64, requires_grad=True) for n in ("q", "k", "v"))
    Nq, Nk = q.shape[-2], k.shape[-2]
    mask = None
    if causal:
        i = torch.arange(Nq).unsqueeze(1)
        j = torch.arange(Nk).unsqueeze(0)
        mask = j <= i + (Nk - Nq)
    o = F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale)
    scores = scale * (q.detach() @ k.detach().transpose(-1, -2))
    if mask is not None:
        scores = scores.masked_fill(~mask, float("-inf"))
    lse = torch.logsumexp(scores, dim=-1)
    dq, dk, dv = torch.autograd.grad(o, (q, k, v), torch.tensor(t["do"], dtype=torch.float64))
    return {"o": o.detach().numpy(), "lse": lse.numpy(), "dq": dq.numpy(), "dk": dk.numpy(),
            "dv": dv.numpy()}


def close(got, want, what):
    err = np.max(np.abs(got - want))
    assert err <= TOL * max(1.0, np.max(np.abs(want))), f"{what}: {err:.3e}"


def check_case(oracle_mod, B, H, Nq, Nk, d, causal):
    """Every oracle entry point (full forward, forward on chosen rows, full
    backward, backward on chosen rows) against PyTorch on one shape."""
    t = inputs(900 + Nq * 7 + Nk, B, H, Nq, Nk, d)
    scale = 1.0 / math.sqrt(d)
    ref = torch_reference(t, causal, scale)
    o, lse = oracle_mod.attention_forward(t["q"], t["k"], t["v"], causal, scale)
    close(o, ref["o"], "o")
    close(lse, ref["lse"], "lse")
    g = oracle_mod.attention_backward(t["q"], t["k"], t["v"], t["do"], causal, scale)
    for name in ("o", "lse", "dq", "dk", "dv"):
        close(g[name], ref[name], f"backward {name}")
    qrows = np.unique(np.array([0, Nq // 2, Nq - 1]))
    krows = np.unique(np.array([0, Nk // 3, Nk - 1]))
    o_r, lse_r = oracle_mod.attention_forward(t["q"], t["k"], t["v"], causal, scale, rows=qrows)
    close(o_r, ref["o"][..., qrows, :], "o rows")
    close(lse_r, ref["lse"][..., qrows], "lse rows")
    dq_r, dk_r, dv_r = oracle_mod.attention_backward_rows(t["q"], t["k"], t["v"], t["do"], causal,
                                                          scale, qrows, krows)
    close(dq_r, ref["dq"][..., qrows, :], "dq rows")
    close(dk_r, ref["dk"][..., krows, :], "dk rows")
    close(dv_r, ref["dv"][..., krows, :], "dv rows")


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal", CASES)
def test_oracle_matches_pytorch_attention(oracle_mod, B, H, Nq, Nk, d, causal):
    check_case(oracle_mod, B, H, Nq, Nk, d, causal)


def test_scale_other_than_the_default(oracle_mod):
    t = inputs(977, 1, 2, 20, 20, 16)
    for scale in (0.0, 0.05, 1.3):
        ref = torch_reference(t, True, scale)
        g = oracle_mod.attention_backward(t["q"], t["k"], t["v"], t["do"], True, scale)
        for name in ("o", "lse", "dq", "dk", "dv"):
            close(g[name], ref[name], f"{name} at scale {scale}")


def test_random_shapes_match_pytorch(oracle_mod):
    """Seeded random shapes, masks and scales (odd head dims, single rows, more
    queries than keys without the mask), all entry points against PyTorch."""
    rng = np.random.default_rng(20260)
    for trial in range(40):
        B, H = int(rng.integers(1, 3)), int(rng.integers(1, 3))
        Nk = int(rng.integers(1, 41))
        causal = bool(rng.integers(0, 2))
        Nq = int(rng.integers(1, Nk + 1)) if causal else int(rng.integers(1, 41))
        d = int(rng.integers(1, 17))
        scale = float(rng.uniform(0.0, 2.0))
        t = inputs(5000 + 10 * trial, B, H, Nq, Nk, d)
        ref = torch_reference(t, causal, scale)
        where = f"trial {trial}: B={B} H={H} Nq={Nq} Nk={Nk} d={d} causal={causal} scale={scale:.3f}"
        o, lse = oracle_mod.attention_forward(t["q"], t["k"], t["v"], causal, scale)
        close(o, ref["o"], f"o, {where}")
        close(lse, ref["lse"], f"lse, {where}")
        g = oracle_mod.attention_backward(t["q"], t["k"], t["v"], t["do"], causal, scale)
        for name in ("dq", "dk", "dv"):
            close(g[name], ref[name], f"{name}, {where}")
        qrows = np.unique(rng.integers(0, Nq, size=3))
        krows = np.unique(rng.integers(0, Nk, size=3))
        dq_r, dk_r, dv_r = oracle_mod.attention_backward_rows(t["q"], t["k"], t["v"], t["do"],
                                                              causal, scale, qrows, krows)
        close(dq_r, ref["dq"][..., qrows, :], f"dq rows, {where}")
        close(dk_r, ref["dk"][..., krows, :], f"dk rows, {where}")
        close(dv_r, ref["dv"][..., krows, :], f"dv rows, {where}")
