"""The pins must be sharp: plant a plausible mistake in a copy of the oracle
(on the CPU) and check that at least one pin fails.  Each mutation edits one
line of the oracle's source and loads the result as a separate module; the
real oracle is untouched."""
import importlib.util
import os
import types

import pytest

import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "ssa_oracle.py")

# (original text, planted mistake)
MUTATIONS = {
    "drop_causal_mask": ("causal = s[None, :] <= rows[:, None]",
                         "causal = s[None, :] <= rows[:, None] + 1"),
    "sparse_normalised_over_all": ("h_sparse = o_sel / l_sel[:, None]",
                                   "h_sparse = o_sel / l_all[:, None]"),
    "delta_of_selected_mass": ("\"delta\": l_uns / l_all,", "\"delta\": l_sel / l_all,"),
    "lse_missing_max": ("\"lse_full\": m + np.log(l_all),", "\"lse_full\": np.log(l_all),"),
    "pool_first_half_only": ("return x[: n * block].reshape(n, block, d).sum(axis=1) / float(block)",
                             "return x[: n * block].reshape(n, block, d)[:, : block // 2].sum(axis=1) / float(block)"),
    "scores_transposed": ("return pool_blocks(q, block) @ pool_blocks(k, block).T",
                          "return pool_blocks(k, block) @ pool_blocks(q, block).T"),
    "ties_to_higher_index": ("ranked = sorted(cand, key=lambda j: (-s[i, j], j))",
                             "ranked = sorted(cand, key=lambda j: (-s[i, j], -j))"),
    "margin_always_zero": ("margin[b, h, i] = s[i, ranked[r - 1]] - s[i, ranked[r]]",
                           "margin[b, h, i] = 0.0"),
    "margin_from_the_top_block": ("margin[b, h, i] = s[i, ranked[r - 1]] - s[i, ranked[r]]",
                                  "margin[b, h, i] = s[i, ranked[0]] - s[i, ranked[r]]"),
    "diagonal_outside_budget": ("r = max(topk - len(forced), 0)",
                                "r = max(topk - len(forced) + 1, 0)"),
    "commit_gradient_sign": ("g_sparse = f64(dh_sparse) + w_c * (2.0 / n_total) * (hs - hf)",
                             "g_sparse = f64(dh_sparse) + w_c * (2.0 / n_total) * (hf - hs)"),
    "bwd_missing_scale": ("dk += sm_scale * dx.T @ q[t]", "dk += dx.T @ q[t]"),
    "bwd_dv_sparse_dropped": ("dv += p_full.T @ g_full[t] + p_sparse.T @ g_sparse[t]",
                              "dv += p_full.T @ g_full[t]"),
    "sparsity_gradient_to_wrong_stream": ("g_full = f64(dh_full) + w_s * (2.0 / n_total) * (hf - hs)",
                                          "g_full = f64(dh_full) + w_s * (2.0 / n_total) * (hs - hf)"),
    "bwd_sparse_jacobian_row_term_dropped": (
        "dx += p_sparse * (dp_sparse - (p_sparse * dp_sparse).sum(axis=1, keepdims=True))",
        "dx += p_sparse * dp_sparse"),
    "bwd_dq_unscaled": ("dq[t] = sm_scale * dx @ k", "dq[t] = dx @ k"),
    "bwd_sparse_stream_over_all_causal_keys": (
        "sel = causal & blocksel[t // block][:, s // block]", "sel = causal"),
    "loss_sum_not_mean": ("L = float(np.mean((hf - hs) ** 2))", "L = float(np.sum((hf - hs) ** 2))"),
    "sparse_only_no_causal_mask": ("x = np.where(keys[None, :] <= ts[:, None], x, -np.inf)",
                                   "x = np.where(keys[None, :] <= ts[:, None] + block, x, -np.inf)"),
    "sparse_only_lse_missing_max": ("lse_out[b, h, sel] = m[:, 0] + np.log(l)",
                                    "lse_out[b, h, sel] = np.log(l)"),
    "sparse_only_first_listed_block_dropped": ("blocks = np.sort(idx[b, h, i, :cnt[b, h, i]])",
                                               "blocks = np.sort(idx[b, h, i, 1:cnt[b, h, i]])"),
    "sink_mass_strict_causality": ("w = np.where(keys[None, :] <= np.arange(T)[:, None], np.exp(x - lse[b, h][:, None]), 0.0)",
                                   "w = np.where(keys[None, :] < np.arange(T)[:, None], np.exp(x - lse[b, h][:, None]), 0.0)"),
    "sink_mass_half_block": ("keys = np.arange(min(block, T))", "keys = np.arange(min(block, T) // 2)"),
    "decode_current_block_outside_budget": ("sel = sorted(forced + ranked[: max(topk - len(forced), 0)])",
                                            "sel = sorted(forced + ranked[: max(topk - len(forced) + 1, 0)])"),
    "decode_ties_to_higher_index": ("ranked = sorted(cand, key=lambda j: (-score[j], j))",
                                    "ranked = sorted(cand, key=lambda j: (-score[j], -j))"),
    "sqdiff_mean_not_sum": ("\"sqdiff\": ((h_full - h_sparse) ** 2).sum(axis=1),",
                            "\"sqdiff\": ((h_full - h_sparse) ** 2).mean(axis=1),"),
    "decode_pool_sum_not_mean": (".reshape(B, H, n_done, block, d).mean(axis=3)",
                                 ".reshape(B, H, n_done, block, d).sum(axis=3)"),
    "decode_lse_missing_max": ("lse_out[b, h] = m + np.log(e.sum())",
                               "lse_out[b, h] = np.log(e.sum())"),
    "decode_future_keys_of_current_block": ("keys = np.concatenate([np.arange(j * block, min((j + 1) * block, t + 1)) for j in sel])",
                                            "keys = np.concatenate([np.arange(j * block, (j + 1) * block) for j in sel])"),
}

PIN_TESTS = [
    lambda: pins.test_worked_example_closed_form(),
    lambda: pins.test_worked_example_sink_flag(),
    lambda: pins.test_pooling_closed_forms(),
    lambda: pins.test_scores_are_mean_of_per_query_scores(),
    lambda: pins.test_topk_ties_go_to_lower_block_index(),
    lambda: pins.test_selection_margin_is_zero_exactly_where_the_best_set_is_not_unique(),
    lambda: pins.test_mask_words_beyond_32_blocks(),
    lambda: pins.test_full_budget_reduces_to_causal_attention(),
    lambda: pins.test_streams_match_library_attention_with_masks(),
    lambda: pins.test_lse_against_library_logsumexp(),
    lambda: pins.test_align_loss_is_library_mse(),
    lambda: pins.test_bwd_central_finite_differences(40.0, 25.0),
    lambda: pins.test_bwd_matches_library_autograd(),
    lambda: pins.test_sparse_only_matches_library_attention_on_selected_keys(),
    lambda: pins.test_sparse_only_diagonal_budget_is_blockwise_causal_attention(),
    lambda: pins.test_sparse_only_brute_force_tiny(),
    lambda: pins.test_sink_mass_is_library_softmax_on_block_zero(),
    lambda: pins.test_sqdiff_rows_from_library_attention(),
    lambda: pins.test_decode_pool_is_block_mean(),
    lambda: pins.test_decode_full_budget_is_causal_attention_row(),
    lambda: pins.test_decode_selection_brute_force(),
    lambda: pins.test_decode_ties_sink_and_first_block(),
]


def _mutant(name):
    before, after = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation anchor not unique/present: {name}"
    mod = types.ModuleType(f"ssa_oracle_mutant_{name}")
    exec(compile(src.replace(before, after), SRC, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    monkeypatch.setattr(pins, "O", _mutant(name))
    caught = 0
    for t in PIN_TESTS:
        try:
            t()
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught > 0, f"no pin detects the planted mistake {name!r}"
