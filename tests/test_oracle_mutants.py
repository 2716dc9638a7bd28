"""Pin strength: every planted mistake in the oracle must fail some pin.

Each case copies the oracle's C source, plants one plausible mistake (a wrong
comparison, a rounding mode, a dropped or negated term, a wrong index or
scale), builds it on the CPU and runs the pin suite against that build.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "llmint8_oracle.c")

MUTANTS = {
    "threshold_strict": ("if (a >= (double)tau)", "if (a > (double)tau)"),
    "round_half_even": ("float q = roundf(r);", "float q = rintf(r);"),
    "dequant_one_scale": ("/ 16129.0;", "/ 127.0;"),
    "outlier_term_negated": ("yd[j] += x * oracle_half_to_double(w[j]);",
                             "yd[j] -= x * oracle_half_to_double(w[j]);"),
    "outlier_term_dropped": ("yd[j] += x * oracle_half_to_double(w[j]);",
                             "yd[j] += 0.0 * x * oracle_half_to_double(w[j]);"),
    "row_scale_includes_outliers": ("            if (mask[k])\n                continue;\n            float a = fabsf(half_to_float(X[i * ldx + k]));",
                                    "            float a = fabsf(half_to_float(X[i * ldx + k]));"),
    "outlier_columns_not_zeroed": ("Xq[i * K + k] = mask[k] ? 0 :", "Xq[i * K + k] ="),
    "row_scale_wrong_index": ("(double)rs[i] * (double)cs[j]", "(double)rs[r] * (double)cs[j]"),
    "codec_ties_to_odd": ("fmod(r, 2.0) != 0.0", "fmod(r, 2.0) == 0.0"),
    "dequantized_weight_scale_128": ("(double)Wq[k * N + j] * (double)cs[j] / 127.0",
                                     "(double)Wq[k * N + j] * (double)cs[j] / 128.0"),
    "bias_indexed_by_row": ("yd[j] += oracle_half_to_double(bias[j]);", "yd[j] += oracle_half_to_double(bias[i % N]);"),
    "stats_threshold_strict": ("if ((double)tau <= a) {", "if ((double)tau < a) {"),
    "weight_scale_first_rows_only": ("for (int64_t k = 0; k < K; ++k) {\n            float a = fabsf(half_to_float(W[k * N + j]));",
                                     "for (int64_t k = 0; k < (K + 1) / 2; ++k) {\n            float a = fabsf(half_to_float(W[k * N + j]));"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    mut = tmp_path / "mutant.c"
    mut.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fno-fast-math", "-ffp-contract=off",
                           "-fPIC", "-shared", str(mut), "-o", str(lib), "-lm"])
    env = dict(os.environ, LLMINT8_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} passed every pin:\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout or "error" in r.stdout.lower()
