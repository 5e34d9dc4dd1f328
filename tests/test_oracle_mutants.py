"""The pins must catch plausible mistakes in the oracle.

Each case below plants one mistake in a private copy of swa_oracle.c (a dropped
term, an off-by-one window edge, a wrong sign, a transposed head index ...),
builds it, points the oracle wrappers at it and runs the pins: at least one pin
has to fail.  The real oracle is restored afterwards.
"""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "swa_oracle.c")

MUTANTS = {
    "window one key too wide": ("int64_t lo = t - w + 1;", "int64_t lo = t - w;"),
    "sinks dropped": ("int64_t se = s < *lo ? s : *lo;", "int64_t se = 0;"),
    "sinks inside the window counted twice": ("int64_t se = s < *lo ? s : *lo;",
                                              "int64_t se = s;"),
    "query's own key dropped": ("for (int64_t j = lo; j <= t; ++j) key[n++] = j;",
                                "for (int64_t j = lo; j < t; ++j) key[n++] = j;"),
    "GQA heads interleaved": ("const int kvh = h / G;", "const int kvh = h % Hkv;"),
    "max subtracted with the wrong sign": ("const double p = exp(z[i] - m);",
                                           "const double p = exp(m - z[i]);"),
    "scale dropped": ("z[i] = scale * dot;", "z[i] = dot;"),
    "lse without the max": ("lse[(size_t)r * Hq + h] = m + log(l);",
                            "lse[(size_t)r * Hq + h] = log(l);"),
    "not normalised": ("o[c] = acc[c] / l;", "o[c] = acc[c];"),
    "value read from the query head": (
        "const double* vj = v + ((size_t)key[i] * Hkv + kvh) * d;",
        "const double* vj = v + ((size_t)key[i] * Hkv + (h % Hkv)) * d;"),
}

PIN_CASES = [
    lambda: pins.test_brute_force_all_windows_and_sinks(9),
    pins.test_window_covering_sequence_is_full_causal_attention,
    pins.test_window_one_returns_own_value,
    lambda: pins.test_constant_keys_give_mean_of_visible_values(5, 3),
    pins.test_tiny_visible_count_total,
    pins.test_sinks_inside_the_window_are_counted_once,
    lambda: pins.test_golden_hand_examples("hand_sinks_d1.json"),
    lambda: pins.test_golden_hand_examples("hand_gqa_d2.json"),
]


@pytest.fixture(scope="module")
def src_text():
    return open(SRC).read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, src_text, tmp_path):
    old, new = MUTANTS[name]
    assert src_text.count(old) == 1, f"mutation site not unique: {old}"
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src_text.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o",
                           str(lib), str(mutant), "-lm"])
    oracle.use_library(str(lib))
    try:
        failed = 0
        for case in PIN_CASES:
            try:
                case()
            except (AssertionError, ValueError):
                failed += 1
        assert failed > 0, f"no pin caught the planted mistake: {name}"
    finally:
        oracle.use_library(oracle._LIB)
