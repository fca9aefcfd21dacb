"""The oracle's pins must catch plausible mistakes.

Each case copies st_oracle.c to a temporary directory, plants one mistake by text substitution
(the committed oracle is never touched), compiles it, and runs the pin suites against that build
through ORACLE_LIB.  A mutation that every pin lets through would mean the pins are too weak.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "st_oracle.c")

MUTATIONS = {
    # local band one key short (the page's "nearest l" prose instead of the set {t..i})
    "band_off_by_one": ("case K_SA1: return j >= (i - l > 0 ? i - l : 0);",
                        "case K_SA1: return j > (i - l > 0 ? i - l : 0);"),
    "stride_wrong_residue": ("case K_SA2: return ((i - j) % l) == 0;",
                             "case K_SA2: return ((i + j + 1) % l) == 0;"),
    # the garbled range {t, ..., l} taken literally: one position too many per block
    "fixed_range_inclusive_l": ("case K_FA2: return (j % l) >= l - c - o && (j % l) <= l - 1 - o;",
                                "case K_FA2: return (j % l) >= l - c - o && (j % l) <= l - o;"),
    "fixed_offset_sign": ("case K_FA2: return (j % l) >= l - c - o && (j % l) <= l - 1 - o;",
                          "case K_FA2: return (j % l) >= l - c + o && (j % l) <= l - 1 + o;"),
    "scale_dropped": ("const double scale = 1.0 / sqrt((double)d);", "const double scale = 1.0;"),
    "softmax_unnormalised": ("const double p = exp(s[a] - m) / z;", "const double p = exp(s[a] - m);"),
    "values_read_from_keys": ("const double *vj = vh + set[a] * e;\n        for (int64_t t = 0; t < e; ++t) orow[t]",
                              "const double *vj = kh + set[a] * e;\n        for (int64_t t = 0; t < e; ++t) orow[t]"),
    # the two widths confused: the score scaled by the value width, value rows stepped by the
    # query-key width, dO rows stepped by the query-key width
    "scale_uses_value_width": ("const double scale = 1.0 / sqrt((double)d);",
                               "const double scale = 1.0 / sqrt((double)e);"),
    "value_rows_at_qk_width": ("const double *vj = vh + set[a] * e;\n        for (int64_t t = 0; t < e; ++t) orow[t]",
                               "const double *vj = vh + set[a] * d;\n        for (int64_t t = 0; t < e; ++t) orow[t]"),
    "dO_rows_at_qk_width": ("const double *qi = qh + i * d, *doi = doh + i * e;",
                            "const double *qi = qh + i * d, *doi = doh + i * d;"),
    "lse_missing_max": ("*lse = m + log(z);", "*lse = log(z);"),
    "dS_sign": ("const double ds = p * (accp - D[i]);", "const double ds = p * (accp + D[i]);"),
    "dK_scale_dropped": ("dkrow[t] += ds * qi[t] * scale;", "dkrow[t] += ds * qi[t];"),
    "dQ_uses_values": ("const double *kj = kh + set[a] * d;\n            for (int64_t t = 0; t < d; ++t) dqrow[t]",
                       "const double *kj = vh + set[a] * d;\n            for (int64_t t = 0; t < d; ++t) dqrow[t]"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_reject_mutation(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {name}"
    mutated = src.replace(old, new)
    c_path = tmp_path / "mut.c"
    so_path = tmp_path / "libmut.so"
    c_path.write_text(mutated)
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", str(c_path),
                           "-o", str(so_path), "-lm"])
    env = dict(os.environ, ORACLE_LIB=str(so_path), OMP_NUM_THREADS="4")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_sets.py"),
                        os.path.join(ROOT, "tests", "test_oracle_math.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode != 0, f"pins let mutation {name!r} through:\n{r.stdout[-2000:]}"
