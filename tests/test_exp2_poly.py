"""Pins for the FMA-pipe exp2 the kernels use for part of their exponentials.

The polynomial table in exp2_poly.cuh must meet its stated minimax error, and
the whole evaluation (rounding trick, f = x - n, Horner with fused multiply-add,
2^n added into the exponent field) is replayed here in float32 and compared with
2^x in float64 over the input range the kernels use.
"""
import importlib.util
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "exact_tiled_attention_30_b200", "csrc")


def coefficients():
    text = open(os.path.join(CSRC, "exp2_poly.cuh")).read()
    vals = dict(re.findall(r"kExp2Poly(\d) = ([-+0-9.eE]+)f;", text))
    return [np.float32(float(vals[str(i)])) for i in range(len(vals))]


def fma32(a, b, c):
    # a * b is exact in float64 for float32 a, b; one rounding to float32 after the add
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly_f32(x):
    c = coefficients()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = fma32(n, np.full_like(n, -1.0), x)
    p = np.full_like(f, c[-1])
    for ck in reversed(c[:-1]):
        p = fma32(p, f, np.full_like(f, ck))
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_table_meets_its_error_bound():
    spec = importlib.util.spec_from_file_location("gen", os.path.join(CSRC, "gen_exp2_poly.py"))
    gen = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(gen)
    c = np.array(coefficients(), dtype=np.float64)
    assert np.max(np.abs(gen.rel_err(c, gen.GRID))) < 3e-6


def test_evaluation_matches_exp2():
    x = np.concatenate([np.linspace(-125.0, 8.0, 1_000_001, dtype=np.float32),
                        np.arange(-125, 9, dtype=np.float32),            # integers (f = 0)
                        np.arange(-125, 8, dtype=np.float32) + 0.5])     # rounding ties
    y = exp2_poly_f32(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 5e-6, (rel.max(), x[np.argmax(rel)])


def test_clamps_far_below():
    y = exp2_poly_f32(np.array([-300.0, -1e30, -127.0], dtype=np.float32))
    assert np.all(np.abs(y) < 2e-38)
