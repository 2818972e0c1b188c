"""The oracle pins catch plausible mistakes.

Each case plants one mistake into a copy of oracle.c (on the CPU, in a temporary
directory), builds it, and runs the pin suite against the broken build: at least one
pin must fail.  The shipped oracle is untouched.

Not listed: widening the clamp to [-128, 127].  That mutant is equivalent: every |x| is at
most the row's absmax a, and x / fl32(a/127) <= 127 * (1 + 2^-24) rounds to at most 127,
so the clamp in the pages' formula can never bind.
"""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTANTS = {
    "round_half_away": ("float r = nearbyintf(v);", "float r = roundf(v);"),
    "scale_over_128": ("float s = absmax / 127.0f;\n    *scale = s;",
                       "float s = absmax / 128.0f;\n    *scale = s;"),
    "reciprocal_scale": ("round_clamp_127(half_to_float(x[j]) / s)",
                         "round_clamp_127(half_to_float(x[j]) * (127.0f / absmax))"),
    "threshold_not_strict": ("if (fabsf(half_to_float(X[i * K + j])) > t) outlier = 1;",
                             "if (fabsf(half_to_float(X[i * K + j])) >= t) outlier = 1;"),
    "row_max_includes_outliers": ("        if (is_outlier(mask, j)) continue;\n", ""),
    "outlier_term_dropped": ("p += oracle_half_to_double(x[cols[o]]) *",
                             "p += 0.0 * oracle_half_to_double(x[cols[o]]) *"),
    "outlier_wrong_column": ("p += oracle_half_to_double(x[cols[o]]) *",
                             "p += oracle_half_to_double(x[o]) *"),
    "outlier_uses_unscaled_int8": ("float w = (float)Wq[n * K + cols[r]] * w_scale[n];",
                                   "float w = (float)Wq[n * K + cols[r]];"),
    "bias_dropped": ("double b = bias ? oracle_half_to_double(bias[n]) : 0.0;",
                     "double b = 0.0;"),
    "row_scale_dropped": ("(double)a * (double)sx * (double)w_scale[n]",
                          "(double)a * (double)w_scale[n]"),
    "transposed_weight_scale": ("(double)a * (double)sx * (double)w_scale[n]",
                                "(double)a * (double)sx * (double)w_scale[rows[r] % N]"),
    "no_overflow_check": ("if (acc > INT32_MAX || acc < INT32_MIN) return ORACLE_ERANGE;", ""),
    "half_encode_truncates": ("double scaled = nearbyint(2.0 * f * 1024.0);",
                              "double scaled = floor(2.0 * f * 1024.0);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC, encoding="utf-8").read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutated = tmp_path / "oracle_mut.c"
    mutated.write_text(src.replace(old, new), encoding="utf-8")
    lib = tmp_path / "liboracle_mut.so"
    subprocess.check_call(["gcc", "-std=c99", "-O2", "-fPIC", "-shared", "-fopenmp",
                           "-I", os.path.join(ROOT, "oracle"), "-o", str(lib), str(mutated),
                           "-lm"])
    env = dict(os.environ, INT8_ORACLE_LIB=str(lib), OMP_NUM_THREADS="2")
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                          os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode != 0, f"mutant {name} survived every pin:\n{res.stdout[-2000:]}"
