"""The oracle pins must catch plausible mistakes.

Each case below plants one mistake in a temporary copy of oracle/oracle.c (a dropped term, a wrong
sign or index, a transposed layout, a reversed order), builds it with gcc, routes the oracle module
through that copy, and checks that at least one pin of tests/test_oracle.py fails.  The real oracle
is never modified.  CPU only.
"""
from __future__ import annotations

import os

import pytest

import oracle
from tests import test_oracle as pins
from tests import test_oracle_quest as quest_pins
from tests import test_oracle_stochastic as stochastic_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# (name, exact text in oracle.c, replacement)
MUTANTS = [
    ("drop_softmax_scale", "double scale = 1.0 / sqrt((double)s->d);", "double scale = 1.0;"),
    ("gqa_modulo_mapping", "int kvh = h / G;", "int kvh = h % s->Hkv;"),
    ("ties_to_higher_position", "return (x->pos < y->pos) ? -1 : (x->pos > y->pos);",
     "return (x->pos > y->pos) ? -1 : (x->pos < y->pos);"),
    ("select_smallest", "if (x->s > y->s) return -1;\n    if (x->s < y->s) return 1;",
     "if (x->s < y->s) return -1;\n    if (x->s > y->s) return 1;"),
    ("hnd_instead_of_nhd", "long row = ((long)page * s->P + slot) * s->Hkv + kvh;",
     "long row = ((long)page * s->Hkv + kvh) * s->P + slot;"),
    ("slot_from_wrong_axis", "long slot = p % s->P;", "long slot = (p / s->P) % s->P;"),
    ("drop_first_dim", "for (int j = 0; j < s->d; ++j) acc += bf16_to_double(qh[j]) * bf16_to_double(krow[j]);\n        out[i]",
     "for (int j = 1; j < s->d; ++j) acc += bf16_to_double(qh[j]) * bf16_to_double(krow[j]);\n        out[i]"),
    ("no_normalisation", "for (int j = 0; j < s->d; ++j) out[j] /= den;", ""),
    ("sign_flip_in_exponent", "double e = exp(z[t] - zref)", "double e = exp(zref - z[t])"),
    ("one_row_short", "for (int i = 0; i < take; ++i) idx_row[i] = all[i].pos;",
     "for (int i = 0; i + 1 < take; ++i) idx_row[i] = all[i].pos;"),
    ("unsorted_output", "qsort(idx_row, (size_t)take, sizeof(int32_t), by_pos);", ""),
    # Quest
    ("quest_lower_bound_instead_of_upper", "r += lo > hi ? lo : hi;", "r += lo < hi ? lo : hi;"),
    # (swapping min and max is not a mistake: the relevance is symmetric in them)
    ("quest_max_only", "double lo = qe * mn[e], hi = qe * mx[e];", "double lo = qe * mx[e], hi = qe * mx[e];"),
    ("quest_stale_slots_counted", "    if (p1 > n) p1 = n;\n", ""),
    ("quest_current_page_dropped", "keep[np - 1] = 1;   /* the page of the current position is always kept */", ""),
    ("quest_budget_rounds_down", "long kp = ((long)kb + s->P - 1) / s->P;", "long kp = (long)kb / s->P;"),
    ("quest_current_page_outside_budget", "for (long t = 0; t + 1 < kp; ++t) keep[other[t].pos] = 1;",
     "for (long t = 0; t < kp && t + 1 < np; ++t) keep[other[t].pos] = 1;"),
    # stochastic selection
    ("sample_weight_inverted", "double w = nsamp > 0 ? (double)(n - (nsel - nsamp)) / (double)nsamp : 1.0;",
     "double w = nsamp > 0 ? (double)nsamp / (double)(n - (nsel - nsamp)) : 1.0;"),
    ("sample_weight_numerator_only", "        *den += e;\n", "        *den += exp(z[t] - zref);\n"),
    ("sample_weight_rest_off_by_one", "double w = nsamp > 0 ? (double)(n - (nsel - nsamp)) / (double)nsamp : 1.0;",
     "double w = nsamp > 0 ? (double)(n - 1 - (nsel - nsamp)) / (double)nsamp : 1.0;"),
    ("sample_drawn_from_all_rows", "        if (!in_det[p]) { rest[c].key", "        if (1) { rest[c].key"),
    ("sample_largest_keys", "if (x->key != y->key) return (x->key < y->key) ? -1 : 1;",
     "if (x->key != y->key) return (x->key > y->key) ? -1 : 1;"),
    ("quest_first_dim_dropped", "for (int e = 0; e < s->d && rc == 0; ++e) {\n            double qe",
     "for (int e = 1; e < s->d && rc == 0; ++e) {\n            double qe"),
]

PINS = [
    pins.test_golden_topk_ties,
    pins.test_topk_brute_force_tiny,
    pins.test_topk_brute_force_random_real_scores,
    pins.test_scores_closed_form_paging_and_gqa,
    pins.test_dense_equals_library_sdpa,
    pins.test_any_k_equals_masked_library_sdpa,
    pins.test_k1_returns_argmax_row,
    pins.test_two_rows_logistic_closed_form,
    pins.test_golden_uniform_average,
    quest_pins.test_relevance_is_max_over_box_corners,
    quest_pins.test_relevance_bounds_every_row_of_its_page,
    quest_pins.test_current_page_always_kept,
    quest_pins.test_ties_go_to_lower_page_and_budget_rounds_up,
    quest_pins.test_partial_last_page_and_whole_cache_budget,
    quest_pins.test_selection_is_the_most_relevant_pages,
    stochastic_pins.test_splitmix64_published_outputs,
    stochastic_pins.test_zero_samples_is_exact_topk,
    stochastic_pins.test_sampling_all_the_rest_is_dense_attention,
    stochastic_pins.test_weighted_sums_are_unbiased_over_every_sample,
    stochastic_pins.test_sample_is_distinct_outside_the_deterministic_rows_and_reproducible,
    stochastic_pins.test_each_rest_row_is_drawn_with_probability_m_over_rest,
    stochastic_pins.test_sample_is_the_rows_with_the_smallest_keys,
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new)
    path = tmp_path / "oracle_mut.c"
    path.write_text(mutated)
    lib = oracle.compile_source(str(path), str(tmp_path / "liboracle_mut.so"))
    failed = []
    with oracle.use_library(lib):
        for pin in PINS:
            try:
                pin()
            except (AssertionError, ValueError):
                failed.append(pin.__name__)
    assert failed, f"no pin caught mutant {name}"
