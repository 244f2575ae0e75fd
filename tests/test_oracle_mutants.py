"""Plant plausible mistakes in a copy of the oracle and check that some pin catches each.

The copy is built in a temporary directory on the CPU; the committed oracle is untouched.
"""
import os
import subprocess

import pytest

import oracle
from tests import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "qsa_oracle.c")

MUTANTS = {
    "mean_divides_by_B_plus_1": ("acc / (double)B;", "acc / (double)(B + 1);"),
    "relu_dropped": ("total += dot > 0.0 ? dot : 0.0;", "total += dot;"),
    "relu_becomes_abs": ("total += dot > 0.0 ? dot : 0.0;", "total += dot > 0.0 ? dot : -dot;"),
    "tie_goes_to_higher_index": ("return (x->idx < y->idx) ? -1 : (x->idx > y->idx);",
                                 "return (x->idx > y->idx) ? -1 : (x->idx < y->idx);"),
    "lowest_scores_selected": ("if (x->score > y->score) return -1;\n    if (x->score < y->score) return 1;",
                               "if (x->score < y->score) return -1;\n    if (x->score > y->score) return 1;"),
    "trailing_drops_query_token": ("for (int64_t u = n_c * B; u <= t; ++u)", "for (int64_t u = n_c * B; u < t; ++u)"),
    "trailing_dropped": ("for (int64_t u = n_c * B; u <= t; ++u) toks[n++] = u;", ""),
    "gqa_modulo_mapping": ("int g = h / G;", "int g = h % Hkv;"),
    "scale_dropped": ("logit[i] = scale * dot;", "logit[i] = dot;"),
    "n_c_off_by_one": ("int64_t n_c = (t + 1) / B;\n            const char", "int64_t n_c = t / B;\n            const char"),
    "qi_transposed": ("orc_load(qi_row, dtype, (size_t)h * di + c)", "orc_load(qi_row, dtype, (size_t)c * Hi + h)"),
    "no_max_subtraction_and_no_norm": ("o_row[(size_t)h * d + c] = n_toks > 0 ? acc / denom : 0.0;",
                                       "o_row[(size_t)h * d + c] = acc;"),
    "selection_keeps_k_minus_1": ("int n_sel = (int)(n_c < k ? n_c : k);", "int n_sel = (int)(n_c < k ? n_c : k - 1);"),
    "rope_adjacent_pairs": ("double a = h[i], b = h[i + half];\n        h[i] = a * c - b * sn;\n        h[i + half] = b * c + a * sn;",
                            "double a = h[2 * i], b = h[2 * i + 1];\n        h[2 * i] = a * c - b * sn;\n        h[2 * i + 1] = b * c + a * sn;"),
    "rope_sin_sign_flipped": ("h[i] = a * c - b * sn;", "h[i] = a * c + b * sn;"),
    "rope_frequency_exponent_halved": ("pow(theta, -2.0 * (double)i / (double)rd)", "pow(theta, -1.0 * (double)i / (double)rd)"),
    "rope_rotates_v_too": ("for (int h = 0; h < Hq + Hkv; ++h)", "for (int h = 0; h < Hq + 2 * Hkv; ++h)"),
    "rope_skips_indexer_key": ("for (int h = 0; h < Hi + 1; ++h)", "for (int h = 0; h < Hi; ++h)"),
    "projection_transposed_weight": ("orc_load(w, dtype, (size_t)o * D + c)", "orc_load(w, dtype, (size_t)c * n_out + o)"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new, 1)
    c = tmp_path / "m.c"
    c.write_text(mutated)
    so = tmp_path / "libm.so"
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fopenmp", "-shared", "-fPIC", "-o", str(so), str(c), "-lm"])
    caught = []
    with oracle.use_library(str(so)):
        for pin in oracle_pins.ALL_PINS:
            try:
                pin(oracle)
            except AssertionError:
                caught.append(pin.__name__)
            except Exception as e:  # a crash in the mutant also counts as caught
                caught.append(f"{pin.__name__}:{type(e).__name__}")
    assert caught, f"no pin caught mutant {name}"
