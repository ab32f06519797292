"""Plant plausible mistakes in a copy of the oracle and check that the pins catch each one.

Every mutant is the oracle source with one textual change (a dropped term, a
wrong sign, a transposed index, an off-by-one mask), compiled on the CPU into a
temporary library. The pins of test_oracle.py then run against it and at least
one of them must fail. The committed oracle is never modified.
"""
import math
import os
import subprocess

import numpy as np
import pytest

import oracle
from tests import test_oracle as pins
from tests import test_oracle_library as pins_lib
from tests import test_oracle_qk as pins_qk

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.cpp")

MUTANTS = {
    "ds_sign": ("dsi[j] = pi[j] * (dp[j] - D[(size_t)i]);", "dsi[j] = pi[j] * (dp[j] + D[(size_t)i]);"),
    "dq_drops_scale": ("dqh[i * d + c] *= scale;", "dqh[i * d + c] *= 1.0;"),
    "dk_transposed_ds": ("const double ds = dS[(size_t)(i * Nk + j)];",
                         "const double ds = dS[(size_t)(j * Nk + i)];"),
    "causal_off_by_one": ("return causal ? std::min(Nk, i + 1 + Nk - Nq) : Nk;",
                          "return causal ? std::min(Nk, i + 2 + Nk - Nq) : Nk;"),
    "lse_drops_max": ("return m + std::log(l);", "return std::log(l);"),
    "dv_uses_ds": ("dvj[c] += p * doi[c];", "dvj[c] += ds * doi[c];"),
    "scores_drop_scale": ("for (int64_t j = j0; j < j1; ++j) acc[j - j0] *= scale;", ""),
    "d_from_v": ("D[(size_t)i] = dot(doh + i * d, oh + i * d, d);",
                 "D[(size_t)i] = dot(doh + i * d, vh + i * d, d);"),
    "rows_p_drops_lse": ("ds[j] = std::exp(s[j] - L[(size_t)i]) * (dp[j] - D[(size_t)i]);",
                         "ds[j] = std::exp(s[j]) * (dp[j] - D[(size_t)i]);"),
    "rows_dk_drops_scale": ("      for (int64_t c = 0; c < d; ++c) dkj[c] *= scale;\n    });\n  }\n  return 0;\n}\n\nint oracle_attention_backward_rows(",
                            "    });\n  }\n  return 0;\n}\n\nint oracle_attention_backward_rows("),
    "pv_transposed": ("const double* r = rows + j * d;", "const double* r = rows + j;"),
    "causal_top_left": ("return causal ? std::min(Nk, i + 1 + Nk - Nq) : Nk;",
                        "return causal ? std::min(Nk, i + 1) : Nk;"),
}


def _run_pins():
    """The pins, against whichever oracle library is active. Raises on the first failure."""
    for causal in (False, True):
        for N, d in ((5, 4), (12, 8)):
            pins.test_brute_force(oracle, N, d, causal)
        pins.test_rows_variants_agree(oracle, causal)
        pins.test_gradient_sum_identities(oracle, causal)
        pins.test_uniform_scores_give_mean_of_v(oracle, causal)
    pins.test_causal_row_zero(oracle)
    pins.test_shift_invariance(oracle)
    pins.test_single_token(oracle)
    # different query and key lengths (bottom-right causal alignment)
    pins_qk.test_brute_force(oracle, 3, 7, 4, True)
    pins_qk.test_brute_force(oracle, 7, 3, 4, False)
    pins_qk.test_uniform_scores_bottom_right(oracle)


def test_pins_pass_on_the_committed_oracle():
    _run_pins()


def _run_library_pin():
    """Only the PyTorch pin of test_oracle_library.py, on two shapes."""
    pins_lib.check_case(oracle, 1, 2, 9, 9, 8, True)
    pins_lib.check_case(oracle, 1, 1, 5, 9, 4, True)


def _build_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new, 1)
    path = tmp_path / "mutant.cpp"
    path.write_text(mutated)
    lib = tmp_path / "libmutant.so"
    flags = [f for f in oracle.CXXFLAGS if f != "-O3"] + ["-O1"]
    subprocess.run(["g++", *flags, str(path), "-o", str(lib)], check=True)
    return str(lib)


def test_library_pin_passes_on_the_committed_oracle():
    _run_library_pin()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    with oracle.use_library(_build_mutant(name, tmp_path)):
        with pytest.raises(AssertionError):
            with np.errstate(all="ignore"):
                _run_pins()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_library_pin_alone_catches_mutant(name, tmp_path):
    with oracle.use_library(_build_mutant(name, tmp_path)):
        with pytest.raises(AssertionError):
            with np.errstate(all="ignore"):
                _run_library_pin()
