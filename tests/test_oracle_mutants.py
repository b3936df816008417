"""CPU: the pins are strong enough to catch plausible mistakes.  Each mutant is a copy of
oracle/hstu_oracle.c with one planted mistake (a dropped term, a wrong sign, index or operand),
compiled into a temporary directory; at least one pin must reject it."""
import os
import subprocess

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "hstu_oracle.c")

MUTANTS = {
    "causal_excludes_self": ("if (i < U) return j <= i;", "if (i < U) return j < i;"),
    "candidate_drops_self": ("return j < U || j == i;", "return j < U;"),
    "candidates_see_each_other": ("return j < U || j == i;", "return j <= i;"),
    "history_sees_candidates": ("if (i < U) return j <= i;", "if (i < U) return 1;"),
    "sigmoid_sign": ("return x / (1.0 + exp(-x));", "return x / (1.0 + exp(x));"),
    "gelu_like_instead_of_silu": ("return x / (1.0 + exp(-x));", "return x / (1.0 + exp(-1.702 * x));"),
    "alpha_outside_silu": ("double p = silu(alpha * s);", "double p = alpha * silu(s);"),
    "score_uses_value_rows": ("s += (double)qrow[c] * (double)krow[c];", "s += (double)qrow[c] * (double)vrow[c];"),
    "missing_normaliser": ("res[c] /= N;", "res[c] /= 1.0;"),
    "normaliser_multiplies": ("res[c] /= N;", "res[c] *= N;"),
    "off_by_one_history_length": ("static int64_t one_row(const float* qrow, const float* kseg, const float* vseg, int64_t stride,\n                       int32_t d, int32_t i, int32_t L, int32_t U, double alpha, double N,\n                       double* res) {\n  int64_t macs = 0;",
                                  "static int64_t one_row(const float* qrow, const float* kseg, const float* vseg, int64_t stride,\n                       int32_t d, int32_t i, int32_t L, int32_t U, double alpha, double N,\n                       double* res) {\n  int64_t macs = 0;\n  U = U + 1;"),
    "cached_position_ignores_prefix": ("d, c + r, L, L - T, alpha, N,", "d, r, L, L - T, alpha, N,"),
    "rab_inside_silu": ("double p = silu(alpha * s) + (double)rab_h[rel];",
                        "double p = silu(alpha * s + (double)rab_h[rel]);"),
    "rab_ignores_position": ("int32_t rel = i - j;", "int32_t rel = 0;"),
    "rab_clips_one_early": ("if (rel > R - 1) rel = R - 1;", "if (rel > R - 2) rel = R - 2;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, "mutation anchor not found: %s" % name
    mutated = src.replace(old, new, 1)
    cfile = tmp_path / "mutant.c"
    cfile.write_text(mutated)
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", str(lib), str(cfile), "-lm"],
                   check=True)
    o = oracle.Oracle(str(lib))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(o)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, "no pin rejects mutant %s" % name
