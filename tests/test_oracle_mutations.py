"""The oracle's pins must be sharp: for each plausible mistake, a copy of the
oracle with that mistake planted (compiled on the CPU into a temporary
library) must fail at least one pin of ``test_oracle_pins``."""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "hs2_oracle.c")

# name -> (exact text in hs2_oracle.c, replacement, occurrence to replace: 0 = all)
MUTATIONS = {
    "scale_1_over_D": ("s[j] = acc * scale;", "s[j] = acc * scale * scale;", 0),
    "no_scale_in_sparse": ("s[u] = acc * scale;", "s[u] = acc;", 0),
    "causal_excludes_self": ("const int64_t n_causal = tr + 1;", "const int64_t n_causal = tr > 0 ? tr : 1;", 0),
    "window_off_by_one": ("const int64_t n_cand = tr - window + 1 > 0 ? tr - window + 1 : 0;",
                          "const int64_t n_cand = tr - window + 2 > 0 ? tr - window + 2 : 0;", 0),
    "group_map_modulo": ("const int h = g * G + hh;", "const int h = hh * h_kv + g;", 1),
    "tie_to_higher_index": ("    if (x->j < y->j) return -1;\n    if (x->j > y->j) return 1;",
                            "    if (x->j < y->j) return 1;\n    if (x->j > y->j) return -1;", 0),
    "lse_base_2": ("const double l = m + log(z);", "const double l = m + log2(z);", 0),
    "selection_unsorted": ("qsort(row_idx, (size_t)n_sel, sizeof(int32_t), i32_cmp);", "", 0),
    "pad_with_zero": ("for (int64_t i = n_sel; i < topk; ++i) row_idx[i] = -1;",
                      "for (int64_t i = n_sel; i < topk; ++i) row_idx[i] = 0;", 0),
    "score_max_not_sum": ("for (int64_t j = 0; j < n_cand; ++j) grp[j] += exp(s[j] - l);",
                          "for (int64_t j = 0; j < n_cand; ++j) grp[j] = fmax(grp[j], exp(s[j] - l));", 0),
    "score_unnormalised": ("for (int64_t j = 0; j < n_cand; ++j) grp[j] += exp(s[j] - l);",
                           "for (int64_t j = 0; j < n_cand; ++j) grp[j] += exp(s[j] - m);", 0),
    "sparse_window_short": ("const int64_t w0 = tr - window + 1 > 0 ? tr - window + 1 : 0;",
                            "const int64_t w0 = tr - window + 2 > 0 ? tr - window + 2 : 0;", 0),
    "sparse_wrong_group": ("const int h = g * G + hh;", "const int h = hh * h_kv + g;", 2),
    "branch_window_on_shared_cache": ("attend_rows(qd, k_swa + off, v_swa + off, wset",
                                      "attend_rows(qd, k + off, v_swa + off, wset", 0),
    "branch_selected_attends_the_window": ("attend_rows(qd, k + off, v + off, sset, ns,",
                                           "attend_rows(qd, k + off, v + off, wset, nw,", 0),
    "branch_lse_without_max": ("    *lse = m + log(z);", "    *lse = log(z);", 0),
    "block_partial_window": ("const int64_t n_blk = n_cand / blk;", "const int64_t n_blk = (n_cand + blk - 1) / blk;", 0),
    "block_max_not_sum": ("for (int64_t u = 0; u < blk; ++u) acc += row[bb * blk + u];",
                          "for (int64_t u = 0; u < blk; ++u) acc = fmax(acc, row[bb * blk + u]);", 0),
    "block_budget_one_short": ("const int64_t keep = n_blk < topk / blk ? n_blk : topk / blk;",
                               "const int64_t keep = n_blk < topk / blk ? n_blk : topk / blk - 1;", 0),
    "bridge_k_v_swapped": ("                out_k[r * hd + f] = acc;\n            else\n                out_v[r * hd + (f - hd)] = acc;",
                           "                out_v[r * hd + f] = acc;\n            else\n                out_k[r * hd + (f - hd)] = acc;", 0),
    "bridge_weight_transposed": ("const uint16_t* wf = w + f * (int64_t)d_model;",
                                 "const uint16_t* wf = w + f;", 0),
    "bridge_drops_last_column": ("for (int c = 0; c < d_model; ++c) acc += bf16_to_double(x[c]) * bf16_to_double(wf[c]);",
                                 "for (int c = 0; c + 1 < d_model; ++c) acc += bf16_to_double(x[c]) * bf16_to_double(wf[c]);", 0),
}

FAST_PINS = [
    lambda: pins.test_zero_query_closed_form(2),
    lambda: pins.test_zero_query_closed_form(1),
    pins.test_two_key_scale_and_lse,
    pins.test_identity_values_link_score_to_probabilities,
    pins.test_library_softmax_special_case,
    pins.test_head_to_group_map_is_contiguous,
    pins.test_group_of_identical_heads_scales_score,
    pins.test_dominant_planted_key_is_selected,
    pins.test_selection_invariants_random,
    pins.test_exact_ties_go_to_lower_index,
    pins.test_sparse_with_full_budget_equals_full_attention,
    pins.test_sparse_with_zero_budget_is_sliding_window,
    pins.test_short_context_selects_nothing,
    pins.test_block_of_one_token_is_the_token_selection,
    pins.test_block_ties_take_the_lowest_blocks,
    pins.test_blocks_lie_entirely_before_the_window,
    pins.test_block_with_planted_key_is_kept,
    pins.test_block_scores_sum_the_token_scores,
    pins.test_bridge_identity_weights_copy_the_hidden_state,
    pins.test_bridge_feature_layout_by_permuted_one_hot_rows,
    pins.test_bridge_one_hot_hidden_returns_a_weight_column,
    pins.test_bridge_decimal_brute_force,
    pins.test_branches_merged_by_lse_are_the_union_layer,
    pins.test_window_branch_is_sliding_window_attention_of_its_own_cache,
    pins.test_selected_branch_single_key_closed_form,
    pins.test_selected_branch_without_keys_is_empty,
    pins.test_each_branch_reads_only_its_own_cache,
]


def _mutate(text, old, new, occ):
    assert old in text, old
    if occ == 0:
        return text.replace(old, new)
    parts = text.split(old)
    assert len(parts) > occ
    return old.join(parts[:occ]) + new + old.join(parts[occ:])


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(name, tmp_path, monkeypatch):
    old, new, occ = MUTATIONS[name]
    src = _mutate(open(SRC).read(), old, new, occ)
    c = tmp_path / "mut.c"
    c.write_text(src)
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", str(c), "-o", str(so),
                    "-lm"], check=True)
    monkeypatch.setattr(oracle, "_lib", oracle.open_library(str(so)))
    caught = []
    for pin in FAST_PINS:
        try:
            pin()
        except (AssertionError, RuntimeError, ValueError):
            caught.append(pin)
            break
    assert caught, f"no pin caught the planted mistake {name!r}"
