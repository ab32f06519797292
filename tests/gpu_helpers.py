"""Helpers shared by the GPU parity tests: moving seeded bf16 inputs to the
device, choosing sampled heads/rows, and the tolerances the tests apply."""
from __future__ import annotations

import numpy as np

import attn_inputs

#: forward output, max-abs error against the fp64 oracle
O_ATOL = 1e-2
#: LSE (natural log), max-abs error
LSE_ATOL = 1e-3
#: dQ, dK, dV, relative Frobenius error ||gpu - ref|| / ||ref||
GRAD_RTOL = 2e-2


def to_device(bits: np.ndarray):
    """uint16 bf16 bit patterns -> contiguous torch bf16 CUDA tensor (same bits)."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def to_host_f64(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def o_tolerance(ref: np.ndarray) -> np.ndarray:
    """Per-element bound on |O_gpu - O_ref|: O_ATOL, except where bf16 storage of O
    alone cannot meet it (|O| >= 4, where half a bf16 ulp exceeds 1e-2); there the
    bound is half an ulp plus 2e-3 of arithmetic error."""
    a = np.maximum(np.abs(ref), 2.0 ** -126)
    half_ulp = 2.0 ** (np.floor(np.log2(a)) - 8)
    return np.maximum(O_ATOL, half_ulp + 2e-3)


def rel_fro(x: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-30))


def sample_rows(N: int, count: int, seed: int) -> np.ndarray:
    """Sorted distinct rows: the tile edges and the ragged tail, plus seeded random rows."""
    fixed = {0, 1, 63, 64, 127, 128, 129, 255, 256, N // 2, N - 129, N - 128, N - 2, N - 1}
    rows = {r for r in fixed if 0 <= r < N}
    rng = np.random.default_rng(seed)
    extra = max(0, min(count, N) - len(rows))
    if extra:
        rows |= set(int(x) for x in rng.choice(N, size=min(N, extra + len(rows)), replace=False))
    return np.array(sorted(rows))[: max(count, len(fixed))]


def sample_heads(B: int, H: int, count: int, seed: int):
    """(b, h) pairs: the first and last head plus seeded random ones."""
    rng = np.random.default_rng(seed)
    heads = {(0, 0), (B - 1, H - 1)}
    while len(heads) < min(count, B * H):
        heads.add((int(rng.integers(B)), int(rng.integers(H))))
    return sorted(heads)


def inputs(config_index: int, B: int, H: int, N: int, d: int, with_do: bool = False):
    return attn_inputs.make_qkvdo(config_index, B, H, N, d, with_do=with_do)
