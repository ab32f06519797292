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


def half_ulp_bf16(ref: np.ndarray) -> np.ndarray:
    """Half a bf16 ulp at each value: the largest error that rounding to bf16 alone
    can make there (8 significant bits)."""
    a = np.maximum(np.abs(ref), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 8)


def o_tolerance(ref: np.ndarray) -> np.ndarray:
    """Per-element bound on |O_gpu - O_ref|: O_ATOL, except where bf16 storage of O
    alone cannot meet it (|O| >= 4, where half a bf16 ulp exceeds 1e-2); there the
    bound is half an ulp plus 2e-3 of arithmetic error."""
    return np.maximum(O_ATOL, half_ulp_bf16(ref) + 2e-3)


#: one record per parity check (O, LSE, gradients), printed at the end of the
#: test session and written as JSON lines to $FA2_PARITY_REPORT when it is set
REPORT: list = []


def check_o(o: np.ndarray, ref: np.ndarray, where: str) -> dict:
    """The O check of the parity tests.

    The stated bar is max |O_gpu - O_ref| <= 1e-2. O is stored in bf16, and where
    |O| >= 4 half a bf16 ulp (0.0156) already exceeds that bar, so rounding alone
    can break it. The check therefore (1) counts the elements over the plain bar
    and reports them with the worst plain error, (2) asserts that every such
    element has |O_ref| >= 4, i.e. is one that bf16 storage explains, and stays
    within half an ulp + 2e-3 there, and (3) reports the largest error in excess of
    the output rounding, max(0, |O_gpu - O_ref| - half ulp)."""
    assert o.shape == ref.shape, (o.shape, ref.shape)
    assert np.isfinite(o).all(), f"O not finite {where}"
    err = np.abs(o - ref)
    over = err > O_ATOL
    n_over = int(over.sum())
    excess = np.maximum(0.0, err - half_ulp_bf16(ref))
    rec = {"check": "o", "where": where, "elements": int(err.size), "max_err": float(err.max()),
           "n_over_plain_bar": n_over,
           "min_abs_o_where_over": float(np.abs(ref[over]).min()) if n_over else None,
           "max_excess_over_rounding": float(excess.max())}
    REPORT.append(rec)
    if n_over:
        assert np.abs(ref[over]).min() >= 4.0, (
            f"O error over {O_ATOL} at |O| < 4 ({where}): {rec}")
    tol = o_tolerance(ref)
    worst = np.unravel_index(np.argmax(err - tol), err.shape)
    assert np.all(err <= tol), f"O error {err[worst]:.3e} > {tol[worst]:.3e} at {worst} ({where})"
    return rec


def check_lse(lse: np.ndarray, ref: np.ndarray, where: str) -> dict:
    """LSE max-abs error <= LSE_ATOL (natural log)."""
    assert np.isfinite(lse).all(), f"LSE not finite {where}"
    e = float(np.abs(lse - ref).max())
    rec = {"check": "lse", "where": where, "max_err": e}
    REPORT.append(rec)
    assert e <= LSE_ATOL, f"LSE error {e:.3e} ({where})"
    return rec


def check_grad(name: str, got: np.ndarray, ref: np.ndarray, where: str) -> dict:
    """Relative Frobenius error of one gradient <= GRAD_RTOL."""
    assert np.isfinite(got).all(), f"{name} not finite {where}"
    e = rel_fro(got, ref)
    rec = {"check": name, "where": where, "rel_fro": e}
    REPORT.append(rec)
    assert e <= GRAD_RTOL, f"{name} relative Frobenius error {e:.3e} ({where})"
    return rec


def rel_fro(x: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-30))


def sample_rows(N: int, count: int, seed: int) -> np.ndarray:
    """Sorted distinct rows: every tile edge near the start and the end, the middle
    and the last row, plus seeded random rows up to `count` in all (or all N rows
    when N <= count)."""
    fixed = {0, 1, 63, 64, 127, 128, 129, 255, 256, N // 2, N - 129, N - 128, N - 2, N - 1}
    rows = {r for r in fixed if 0 <= r < N}
    rest = np.array([r for r in range(N) if r not in rows], dtype=np.int64)
    extra = min(max(0, count - len(rows)), rest.size)
    if extra:
        rng = np.random.default_rng(seed)
        rows |= set(int(x) for x in rng.choice(rest, size=extra, replace=False))
    return np.array(sorted(rows), dtype=np.int64)


def sample_heads(B: int, H: int, count: int, seed: int):
    """(b, h) pairs: the first and last head plus seeded random ones."""
    rng = np.random.default_rng(seed)
    heads = {(0, 0), (B - 1, H - 1)}
    while len(heads) < min(count, B * H):
        heads.add((int(rng.integers(B)), int(rng.integers(H))))
    return sorted(heads)


def inputs(config_index: int, B: int, H: int, N: int, d: int, with_do: bool = False):
    return attn_inputs.make_qkvdo(config_index, B, H, N, d, with_do=with_do)
