"""The pins must catch plausible mistakes: each case plants one mistake in a copy of oracle.c,
builds it on the CPU, points the oracle wrapper at it, and checks that at least one pin fails.
"""
import os
import subprocess
import tempfile

import pytest

import oracle
from oracle import oracle as oracle_mod
from oracle.build_oracle import SRC

import tests.test_oracle_accept as t_acc
import tests.test_oracle_attention as t_att
import tests.test_oracle_fp8 as t_fp8
import tests.test_oracle_ring as t_ring
import tests.test_oracle_stochastic as t_sto
import tests.test_oracle_tree as t_tree
import tests.test_oracle_window as t_win

# (name, original text, mutated text)
MUTATIONS = [
    ("dropped_scale", "s_buf[j] = sm_scale * dot;", "s_buf[j] = dot;"),
    ("value_is_key", "o[d] += w * bf16_to_double(vbase[", "o[d] += w * bf16_to_double(kbase["),
    ("gqa_modulo", "int hk = h / G;", "int hk = h % Hkv;"),
    ("window_off_by_one", "(j >= L_tot - (long long)window)", "(j > L_tot - (long long)window)"),
    ("sink_off_by_one", "(j < (long long)n_sink)", "(j <= (long long)n_sink)"),
    ("softmax_sign", "double w = exp(s_buf[j] - m);", "double w = exp(m - s_buf[j]);"),
    ("lse_dropped_max", "*l_out = m + log(l);", "*l_out = log(l);"),
    ("causal_cut_dropped", "if (j < 0 || j > p_i || j >= L_tot) return 0;",
     "if (j < 0 || j >= L_tot) return 0;"),
    ("ring_no_sink_offset", "(p - n_sink) % (long long)(capacity - n_sink)",
     "p % (long long)(capacity - n_sink)"),
    ("tree_as_chain", "cur = parent[cur];", "cur = cur - 1;"),
    ("accept_wrong_index", "tok[a + 1] == t[a]", "tok[a + 1] == t[a + 1]"),
    ("argmax_last_tie", "if (row[x] > bv)", "if (row[x] >= bv)"),
    ("tree_highest_child", "if (par[c] == cur && tok[c] == t[cur]) { next = c; break; }",
     "if (par[c] == cur && tok[c] == t[cur]) { next = c; }"),
    ("stoch_residual_is_target", "const float d = pr[v] - qr[v];", "const float d = pr[v];"),
    ("stoch_ratio_inverted", "if (u * qx < px * 16777216.0)", "if (u * px < qx * 16777216.0)"),
    ("stoch_bonus_first_row", "y = draw_fixed(p + ((size_t)b * n_q + (n_q - 1)) * (size_t)V",
     "y = draw_fixed(p + ((size_t)b * n_q + 0) * (size_t)V"),
    ("stoch_rows_shifted", "const float* pr = p + ((size_t)b * n_q + (i - 1)) * (size_t)V;",
     "const float* pr = p + ((size_t)b * n_q + i) * (size_t)V;"),
    ("stoch_draw_off_by_one", "if (c > t) return v;", "if (c >= t) return v;"),
    ("e4m3_bias_8", "else mag = ldexp(1.0 + (double)m / 8.0, (int)e - 7);",
     "else mag = ldexp(1.0 + (double)m / 8.0, (int)e - 8);"),
    ("e4m3_subnormal_scale", "if (e == 0u) mag = ldexp((double)m / 8.0, -6);",
     "if (e == 0u) mag = ldexp((double)m / 8.0, -7);"),
    ("e4m3_no_nan", "if (e == 15u && m == 7u) return NAN;", "if (e == 16u && m == 7u) return NAN;"),
]

PINS = [
    t_ring.test_slot_mapping_hand_worked,
    lambda: t_ring.test_ring_matches_linear_layout_through_wraparound(4, 20, [3, 7, 1, 30, 2]),
    lambda: t_ring.test_ring_holds_exactly_the_window(4, 12, 40),
    lambda: t_win.test_window_set_brute_force(40),
    t_win.test_window_key_visible_is_causal_per_query,
    lambda: t_win.test_window_equals_full_attention_on_kept_subsequence(40, 4, 8),
    t_att.test_two_keys_hand_worked,
    t_att.test_single_key_returns_its_value_exactly,
    t_att.test_matches_dense_textbook_softmax_attention,
    t_att.test_causal_query_equals_prefix_attention,
    lambda: t_tree.test_tree_node_equals_chain_along_root_path(3),
    lambda: t_tree.test_tree_visibility_brute_force(1),
    t_acc.test_hand_worked_chain_examples,
    t_acc.test_ties_take_lowest_index,
    lambda: t_acc.test_chain_brute_force_all_drafts(2),
    lambda: t_acc.test_lossless_tree("random", 3),
    t_acc.test_tree_brute_force_small_vocab,
    lambda: t_sto.test_emitted_token_is_distributed_as_the_target(0),
    lambda: t_sto.test_emitted_token_is_distributed_as_the_target(3),
    t_sto.test_second_position_uses_the_second_rows,
    t_sto.test_disjoint_supports_reject_and_resample_from_the_target,
    t_sto.test_acceptance_threshold_is_p_over_q,
    t_fp8.test_published_e4m3_values,
    t_fp8.test_e4m3_codes_are_ordered_and_finite_except_nan,
]


@pytest.mark.parametrize("name,orig,mut", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(name, orig, mut):
    with open(SRC) as f:
        src = f.read()
    assert src.count(orig) == 1, f"mutation anchor not unique: {orig!r}"
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "mut.c")
        lib = os.path.join(d, "libmut.so")
        with open(c, "w") as f:
            f.write(src.replace(orig, mut))
        subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o", lib, c,
                        "-lm"], check=True)
        oracle_mod.use_library(lib)
        try:
            caught = []
            for pin in PINS:
                try:
                    pin()
                except (AssertionError, ValueError):
                    caught.append(pin)
            assert caught, f"no pin caught mutation {name}"
        finally:
            oracle_mod.use_library(None)
    assert oracle.ring_slot(6, 2, 6) == 2     # default library restored
