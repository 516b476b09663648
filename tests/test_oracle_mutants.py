"""The oracle's pins catch plausible mistakes.

Each case copies ``oracle/kda_oracle.c`` to a temporary directory, plants one
mistake there (a dropped term, a wrong sign, a wrong operand or index),
compiles the copy, points the oracle wrapper at it and runs the pin tests.
At least one pin must fail for every mutant. The committed oracle source is
never modified.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")

MUTANTS = {
    "fade dropped": ("S[i * V + j] *= at[i];", "S[i * V + j] *= 1.0;"),
    "fade on the value index": ("S[i * V + j] *= at[i];", "S[i * V + j] *= at[j % K];"),
    "correction sign flipped": ("delta[j] = vt[j] - delta[j];", "delta[j] = delta[j] - vt[j];"),
    "erase term dropped": ("delta[j] = vt[j] - delta[j];", "delta[j] = vt[j];"),
    "write strength dropped": ("+= bt * kt[i] * delta[j];", "+= kt[i] * delta[j];"),
    "read with the key": ("ot[j] += S[i * V + j] * qt[i];", "ot[j] += S[i * V + j] * kt[i];"),
    "initial state ignored": ("if (s0) memcpy(", "if (0) memcpy("),
    "last packed token dropped": ("int64_t t1 = cu_seqlens ? cu_seqlens[n + 1] : T;",
                                  "int64_t t1 = cu_seqlens ? cu_seqlens[n + 1] - (n % 2) : T;"),
    "gate log-scale dropped": ("g_min * oracle_sigmoid(scale * z[idx])", "g_min * oracle_sigmoid(z[idx])"),
    "gate logit sign flipped": ("g_min * oracle_sigmoid(scale * z[idx])", "g_min * oracle_sigmoid(-scale * z[idx])"),
    "gate exp of the wrong sign": ("alpha_out[idx] = exp(g);", "alpha_out[idx] = exp(-g);"),
    "sigmoid branch wrong": ("return e / (1.0 + e);", "return 1.0 / (1.0 + e);"),
}

PIN_CALLS = [
    pins.test_toy_write_overwrite_retain_exact,
    lambda: pins.test_matches_independent_product_form(0),
    lambda: pins.test_matches_independent_product_form(3),
    pins.test_product_form_exact_rationals,
    pins.test_identity_alpha_one_beta_zero,
    pins.test_zero_writes_closed_form,
    pins.test_deltanet_orthonormal_overwrite,
    pins.test_varlen_equals_separate_sequences,
    pins.test_gate_figure3a_points,
    pins.test_gate_against_library_sigmoid_and_range,
    pins.test_gate_log_scale_rescales_logits,
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path, monkeypatch):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name!r} not found exactly once"
    mut_c = tmp_path / "mutant.c"
    mut_c.write_text(src.replace(old, new))
    lib_path = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(lib_path),
                    str(mut_c), "-lm"], check=True)
    real = oracle._load()
    lib = ctypes.CDLL(str(lib_path))
    for fn in ("kda_oracle_bounded_decay", "kda_oracle_scan", "kda_oracle_max_threads"):
        getattr(lib, fn).argtypes = getattr(real, fn).argtypes
        getattr(lib, fn).restype = getattr(real, fn).restype
    monkeypatch.setattr(oracle, "_lib", lib)
    failures = 0
    for call in PIN_CALLS:
        try:
            call()
        except (AssertionError, ValueError):
            failures += 1
    assert failures > 0, f"no pin caught the planted mistake: {name}"
