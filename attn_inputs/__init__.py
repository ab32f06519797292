"""Seeded synthetic inputs for exact attention, shared by the CUDA side and the oracle side.

This module only draws numbers. It holds none of the attention arithmetic: no
scores, no softmax, no products. Both the fp64 CPU oracle (``oracle/``) and the
sm_100a path (``exact_tiled_attention_30_b200``) take their Q, K, V and dO from
here, so the two see bit-identical bf16 inputs.

Generator (written from the published definitions):
  * SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014): output k (k = 1, 2, ...) of stream ``seed`` is the
    64-bit finaliser applied to ``seed + k * 0x9E3779B97F4A7C15`` (mod 2^64).
  * Uniforms: the top 53 bits of an output, times 2^-53, give u in [0, 1);
    Box-Muller uses 1 - u, which lies in (0, 1], so the logarithm is finite.
  * Box-Muller (1958): r = sqrt(-2 ln u1), z0 = r cos(2 pi u2), z1 = r sin(2 pi u2).
  * bf16: the fp64 normal is rounded to fp32 (round to nearest even) and the fp32
    value to bf16 (round to nearest even on the top 16 bits).

The pages benchmark i.i.d. standard-normal bf16 tensors in [B, H, N, d] layout
("FlashAttention-2" paper reproduction page, Figures 4-7; the configurations
follow that benchmark's axes). Seeds follow ``seed_for(config, tensor)``.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "GOLDEN",
    "TENSOR_IDS",
    "seed_for",
    "splitmix64",
    "standard_normal",
    "to_bf16_bits",
    "bf16_bits_to_f64",
    "bf16_bits_to_f32",
    "normal_bf16",
    "make_qkvdo",
]

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

#: tensor ids used in the seed formula
TENSOR_IDS = {"q": 0, "k": 1, "v": 2, "do": 3}


def seed_for(config_index: int, tensor: str | int) -> int:
    """Seed of one tensor of one workload: 0xFA2 + 1000 * config + tensor id."""
    tid = TENSOR_IDS[tensor] if isinstance(tensor, str) else int(tensor)
    return 0xFA2 + 1000 * int(config_index) + tid


def splitmix64(seed: int, n: int, start: int = 0) -> np.ndarray:
    """Outputs start+1 .. start+n of the SplitMix64 stream with the given seed (uint64)."""
    k = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + k * GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def standard_normal(seed: int, n: int) -> np.ndarray:
    """n i.i.d. N(0, 1) doubles by Box-Muller over consecutive SplitMix64 pairs."""
    pairs = (n + 1) // 2
    x = splitmix64(seed, 2 * pairs)
    u = (x >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)
    u1 = 1.0 - u[0::2]
    u2 = u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    t = 2.0 * np.pi * u2
    out = np.empty(2 * pairs, dtype=np.float64)
    out[0::2] = r * np.cos(t)
    out[1::2] = r * np.sin(t)
    return out[:n]


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float values to bf16 (via fp32, nearest even); returns uint16 bit patterns."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    nan = np.isnan(f)
    r = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    r = r.astype(np.uint16)
    if nan.any():
        r[nan] = np.uint16(0x7FC0)
    return r


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp64."""
    return bf16_bits_to_f32(bits).astype(np.float64)


def normal_bf16(seed: int, shape) -> np.ndarray:
    """i.i.d. N(0,1) rounded to bf16, as uint16 bit patterns of the given shape."""
    n = int(np.prod(shape)) if len(shape) else 1
    return to_bf16_bits(standard_normal(seed, n)).reshape(shape)


def make_qkvdo(config_index: int, B: int, H: int, N: int, d: int, with_do: bool = True):
    """Q, K, V (and dO) of one workload as uint16 bf16 bit arrays of shape [B, H, N, d]."""
    shape = (B, H, N, d)
    out = {name: normal_bf16(seed_for(config_index, name), shape) for name in ("q", "k", "v")}
    if with_do:
        out["do"] = normal_bf16(seed_for(config_index, "do"), shape)
    return out
