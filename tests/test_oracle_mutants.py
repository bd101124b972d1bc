"""The oracle's pins must reject plausible mistakes.

Each case copies hs_oracle.c, plants one mistake in the copy (a dropped key,
a wrong sign, a reversed tie-break, an off-by-one window, a swapped operand,
...), compiles it to a scratch library, and runs the pins of test_oracle.py
against it.  At least one pin has to fail for every mutant; the real oracle
is untouched.
"""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "hs_oracle.c")

MUTANTS = {
    "scale_dropped": ("p->scale * dot(", "dot("),
    "lse_without_log_sum": ("*lse = m + log(l);", "*lse = m;"),
    "value_reads_key": ("kv_row(p, vbase, b, u, keys[x])", "kv_row(p, kbase, b, u, keys[x])"),
    "block_drops_last_key": ("i <= t && i < (c + 1) * B; ++i)\n                    if (prob",
                             "i <= t && i < (c + 1) * B - 1; ++i)\n                    if (prob"),
    "group_uses_first_head": ("if (sh > sbar) sbar = sh;", "if (hh == 0) sbar = sh;"),
    "tie_break_reversed": ("return (x->id > y->id) - (x->id < y->id);",
                           "return (x->id < y->id) - (x->id > y->id);"),
    "score_order_reversed": ("if (x->s > y->s) return -1;", "if (x->s < y->s) return -1;"),
    "window_off_by_one": ("const int lo = t - w + 1; /*", "const int lo = t - w; /*"),
    "budget_short_by_one": ("m = nb < ksel ? nb : ksel;", "m = nb < ksel ? nb : ksel - 1;"),
    "sparse_block_skips_first_key": ("for (int i = id * B; i < (id + 1) * B; ++i)",
                                     "for (int i = id * B + 1; i < (id + 1) * B; ++i)"),
    "sparse_drops_current": ("if (i >= 0 && i <= t) keys[n++] = i;",
                             "if (i >= 0 && i < t) keys[n++] = i;"),
    "local_window_wide": ("const int lo = t - p->window + 1 > 0 ? t - p->window + 1 : 0;",
                          "const int lo = t - p->window > 0 ? t - p->window : 0;"),
    "query_row_transposed": ("((size_t)b * p->hq + h) * p->t_q + j)",
                             "((size_t)h * p->batch + b) * p->t_q + j)"),
    "sink_share_inverted": ("const double fg = s_g ? exp(lse_g[e] - lg) : 1.0;",
                            "const double fg = s_g ? exp(lg - lse_g[e]) : 1.0;"),
    "sink_lse_not_updated": ("const double lg = s_g ? log_add_exp(lse_g[e], s_g[e]) : lse_g[e];",
                             "const double lg = lse_g[e];"),
    "gate_sign_flipped": ("const double gg = z_g ? 1.0 / (1.0 + exp(-z_g[e])) : 1.0;",
                          "const double gg = z_g ? 1.0 / (1.0 + exp(z_g[e])) : 1.0;"),
    "local_gate_reads_global": ("gl = z_l ? 1.0 / (1.0 + exp(-z_l[e])) : 1.0;",
                                "gl = z_l ? 1.0 / (1.0 + exp(-z_g[e])) : 1.0;"),
}

PINS = [
    lambda: pins.test_attention_and_lse_match_library("block", 9, 20),
    lambda: pins.test_attention_and_lse_match_library("token", 0, None),
    lambda: pins.test_block_scores_are_group_max_of_block_max_probability(5),
    lambda: pins.test_block_topk_equals_exhaustive_enumeration(0),
    lambda: pins.test_token_topk_equals_exhaustive_enumeration_with_forced_window(2),
    lambda: pins.test_cardinality_printed_example(),
    lambda: pins.test_token_cardinality_and_window(),
    lambda: pins.test_equal_keys_closed_form_and_lowest_index_tie_break(),
    lambda: pins.test_sparse_equals_dense_when_budget_covers_everything(),
    lambda: pins.test_block_sparse_masks_future_keys_inside_a_selected_block(),
    lambda: pins.test_local_window_branch_matches_banded_library_attention(),
    lambda: pins.test_retained_mass_decomposition_and_bound(),
    lambda: pins.test_sink_is_an_extra_key_with_zero_value(),
    lambda: pins.test_gate_identities(),
    lambda: pins.test_sink_on_an_empty_branch(),
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_mutant(name, tmp_path):
    before, after = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation site for {name} not unique"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(before, after))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o",
                           str(lib), str(mutated), "-lm"])
    caught = []
    with oracle.use_library(str(lib)):
        for pin in PINS:
            try:
                pin()
            except Exception as e:  # any pin failure (assertion or error) counts
                caught.append(type(e).__name__)
                break
    assert caught, f"no pin rejects mutant {name}"
