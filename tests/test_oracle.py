"""CPU tests of the float64 oracle against its pins (no GPU)."""
import os
import shutil
import subprocess
import tempfile

import pytest

import oracle_pins as P
from oracle import oracle as O


@pytest.mark.parametrize("check", P.ALL_CHECKS, ids=lambda c: c.__name__)
def test_oracle_pin(check, oracle_lib):
    check(oracle_lib)


# Plausible mistakes, planted in a private copy of oracle.c. Each must make at
# least one pin fail; this shows the pins constrain every term of the oracle.
MUTANTS = {
    "rotation_sign": ("y[2 * k] = x0 * c - x1 * s;", "y[2 * k] = x0 * c + x1 * s;"),
    "rotation_operands_swapped": ("y[2 * k + 1] = x0 * s + x1 * c;", "y[2 * k + 1] = x1 * s + x0 * c;"),
    "freq_exponent": ("pow(base, -2.0 * (double)k / (double)D)", "pow(base, -1.0 * (double)k / (double)D)"),
    "causal_off_by_one": ("int visible = (j <= i) &&", "int visible = (j < i + 2) &&"),
    "no_document_mask": ("(doc_start[j] == doc_start[i])", "(1)"),
    "gqa_head_map": ("return h / (Hq / Hkv);", "return h % Hkv;"),
    "score_scale": ("const double scale = 1.0 / sqrt((double)D);\n  double m = -INFINITY;",
                    "const double scale = 1.0 / (double)D;\n  double m = -INFINITY;"),
    "value_head": ("const double *vj = vrow + ((int64_t)j * Hkv + g) * D;",
                   "const double *vj = vrow + ((int64_t)j * Hkv + 0) * D;"),
    "decode_query_position": ("rope_rotate_one(q + bh * D, qrot, D, (double)L, freqs);",
                              "rope_rotate_one(q + bh * D, qrot, D, (double)(L - 1), freqs);"),
    "decode_drops_last_key": ("for (int n = 0; n < L; ++n) {\n        double dot",
                              "for (int n = 0; n < L - 1; ++n) {\n        double dot"),
    "decode_scale": ("s[n] = dot * scale;", "s[n] = dot;"),
    "doc_position_not_restarted_inside_row": ("pos[t] = (int32_t)(t - start);",
                                              "pos[t] = (int32_t)(t - start + (t - start) / 2);"),
    "lse_drops_max": ("if (lse) *lse = m + log(sum);", "if (lse) *lse = log(sum);"),
    "lse_base_two": ("if (lse) *lse = m + log(sum);", "if (lse) *lse = m + log2(sum);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name):
    old, new = MUTANTS[name]
    src = open(os.path.join(os.path.dirname(O.__file__), "oracle.c")).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {name}"
    tmp = tempfile.mkdtemp(prefix="oracle_mutant_")
    try:
        cpath = os.path.join(tmp, "mutant.c")
        with open(cpath, "w") as f:
            f.write(src.replace(old, new))
        so = os.path.join(tmp, "libmutant.so")
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", cpath,
                               "-o", so, "-lm"])
        lib = O.load_library(so)
        failed = []
        for check in P.ALL_CHECKS:
            try:
                check(lib)
            except AssertionError:
                failed.append(check.__name__)
        assert failed, f"no pin caught the planted mistake {name}"
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
