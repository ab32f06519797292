"""Toy end-to-end gradient check through the autograd wrapper: a projection, the
attention op (both passes on the C ABI) and a weighted sum, differentiated by
PyTorch, against the fp64 oracle chained by hand.

x [B, N, C] -> q, k, v = heads(x W_q), heads(x W_k), heads(x W_v) (rounded to
bf16) -> O = attention(q, k, v) -> loss = sum(O * G). The oracle gives O and
dQ, dK, dV for dO = G; then dW_q = sum_b x_b^T merge(dQ)_b, likewise for K, V.
Tolerances as in the other parity tests (relative Frobenius 2e-2 for
gradients, 1e-2 max-abs for O).
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
    return m


def bf16_bits(a: np.ndarray) -> np.ndarray:
    import torch

    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("causal,d", [(True, 64), (False, 128)])
def test_training_step_gradients(fa2, oracle_mod, causal, d):
    import torch

    B, N, H = 2, 200, 2
    C = H * d
    rng = np.random.default_rng(40 + d)
    x = rng.standard_normal((B, N, C)).astype(np.float32) * 0.5
    w = {n: (rng.standard_normal((C, C)) / math.sqrt(C)).astype(np.float32) for n in "qkv"}
    g = rng.standard_normal((B, H, N, d)).astype(np.float32)
    g_bits = bf16_bits(g)  # the upstream gradient O sees is bf16

    dev = torch.device("cuda")
    xt = torch.tensor(x, device=dev)
    wt = {n: torch.tensor(w[n], device=dev, requires_grad=True) for n in "qkv"}

    def heads(t):  # [B, N, C] -> [B, H, N, d], bf16, contiguous
        return t.view(B, N, H, d).transpose(1, 2).contiguous().to(torch.bfloat16)

    q, k, v = (heads(xt @ wt[n]) for n in "qkv")
    for t in (q, k, v):
        t.retain_grad()
    o = fa2.attention(q, k, v, causal=causal)
    gt = torch.from_numpy(g_bits.view(np.int16)).view(torch.bfloat16).to(dev)
    loss = (o.float() * gt.float()).sum()
    loss.backward()

    # oracle on the same bf16 q, k, v
    qb, kb, vb = (t.detach().cpu().view(torch.int16).numpy().view(np.uint16) for t in (q, k, v))
    scale = 1.0 / math.sqrt(d)
    ref_o, _ = oracle_mod.attention_forward(qb, kb, vb, causal, scale)
    ref = oracle_mod.attention_backward(qb, kb, vb, g_bits, causal, scale)
    oo = gh.to_host_f64(o.detach())
    where = f"autograd B={B} H={H} N={N} d={d} causal={causal}"
    gh.check_o(oo, ref_o, where)
    for name, t in (("dq", q), ("dk", k), ("dv", v)):
        gh.check_grad(name, gh.to_host_f64(t.grad), ref[name], where)
    # chain rule through the projections, in fp64 from the oracle's head gradients
    x64 = x.astype(np.float64)
    for n, key in (("q", "dq"), ("k", "dk"), ("v", "dv")):
        merged = ref[key].transpose(0, 2, 1, 3).reshape(B, N, C)
        dw_ref = np.einsum("bnc,bne->ce", x64, merged)
        err = gh.rel_fro(wt[n].grad.double().cpu().numpy(), dw_ref)
        assert err <= gh.GRAD_RTOL, f"dW_{n}: {err:.3e}"
