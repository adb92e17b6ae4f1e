"""The oracle's pins catch plausible mistakes.

Each case copies the oracle to a temporary directory, plants one mistake in the
copied C source (a wrong comparison, sign, index, scale, exponent, count term,
empty-sum reading, decode position or block-selection rule), builds it, and runs the pin tests of
``test_oracle.py`` against the copy: at least one pin must fail.  Mistakes are
only ever planted in these CPU copies.
"""
import importlib.util
import math
import os
import shutil
import sys

import pytest

import test_oracle as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "window_strict_less": ("if ((double)d <= lim[r]) acc +=", "if ((double)d < lim[r]) acc +="),
    "rope_sign": ("y[r] = a * c - b * s;", "y[r] = a * c + b * s;"),
    "pair_index": ("qt[r + H] * kt[r + H];", "qt[r + H] * kt[r];"),
    "missing_scale": ("return acc / sqrt((double)D);", "return acc;"),
    "theta_exponent": ("return pow(base, -2.0 * (double)r / (double)D);",
                       "return pow(base, -1.0 * (double)r / (double)D);"),
    "closed_form_term": ("kp += (W + 1) * (2 * (uint64_t)N - W) / 2;",
                         "kp += (W + 1) * (2 * (uint64_t)N - W + 1) / 2;"),
    "empty_sum_is_minus_inf": ("return acc / sqrt((double)D);",
                               "return acc == 0.0 ? -INFINITY : acc / sqrt((double)D);"),
    "decode_position": ("orc_rope(q + ((size_t)b * Hq + h) * D, D, base, L - 1, qt);",
                        "orc_rope(q + ((size_t)b * Hq + h) * D, D, base, L, qt);"),
    "sparse_diagonal_not_forced": ("return m / tile == n / tile || mask_row[m / tile] != 0;",
                                   "return mask_row[m / tile] != 0;"),
    "sparse_group_index": ("block_mask ? block_mask + ((size_t)g * ntiles",
                           "block_mask ? block_mask + ((size_t)0 * ntiles"),
    "sparse_query_tile": ("+ (size_t)(n / tile)) * (size_t)ntiles : NULL;",
                          "+ (size_t)(n / tile + 1) % ntiles) * (size_t)ntiles : NULL;"),
}

PIN_TESTS = [
    lambda o: pins.test_window_lowest_index_pair_is_two_pi_k(o),
    lambda o: pins.test_window_middle_pair_is_two_pi_sqrt_base(o),
    lambda o: [pins.test_count_closed_equals_bruteforce(o, *c) for c in pins.COUNT_CASES],
    lambda o: pins.test_count_tiny_config_regression(o),
    lambda o: pins.test_pages_printed_pruning_percentages(o),
    lambda o: pins.test_rope_rows_matches_textbook(o),
    lambda o: pins.test_scores_shift_invariant(o),
    lambda o: pins.test_pair_decomposition_equals_full_dot(o),
    lambda o: pins.test_k_inf_is_textbook_causal_attention(o, 64, 16, 1e4, 2, 1),
    lambda o: pins.test_k_zero_closed_form(o),
    lambda o: pins.test_single_pair_window_bruteforce(o),
    lambda o: pins.test_decode_equals_prefill_last_row(o),
    lambda o: [pins.test_sparse_equals_textbook_masked_softmax(o, kw) for kw in (math.inf, 1.0)],
    lambda o: pins.test_sparse_diagonal_and_future_entries_are_ignored(o),
]


def _load_mutant(tmp_path, name, old, new):
    dst = tmp_path / f"oracle_{name}"
    shutil.copytree(os.path.join(ROOT, "oracle"), dst,
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    src = dst / "atflash_oracle.c"
    text = src.read_text()
    assert text.count(old) >= 1, f"mutation site for {name} not found"
    src.write_text(text.replace(old, new, 1))
    modname = f"oracle_mutant_{name}"
    spec = importlib.util.spec_from_file_location(modname, dst / "__init__.py",
                                                  submodule_search_locations=[str(dst)])
    mod = importlib.util.module_from_spec(spec)
    sys.modules[modname] = mod
    spec.loader.exec_module(mod)
    mod.lib()
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    mod = _load_mutant(tmp_path, name, old, new)
    caught = 0
    for t in PIN_TESTS:
        try:
            t(mod)
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin caught mutant {name}"
