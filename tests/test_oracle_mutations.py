"""Planted mistakes in the oracle must fail at least one pin.

Each case copies the oracle's C source, plants one plausible mistake (a
dropped term, a wrong sign, a transposed operand, an off-by-one index),
compiles the copy, runs the pins of ``test_oracle_pins`` through it and
expects at least one of them to fail.  Nothing here touches a GPU.
"""
import pytest

import oracle
import test_oracle_backward_pins as bwd
import test_oracle_pins as pins

# (name, text to replace, replacement, pins expected to catch it)
MUTATIONS = [
    ("drop count weighting of low-res terms",
     "double w = cnt_row[c] * exp(", "double w = exp(",
     ["block_constant", "probe"]),
    ("drop 1/sqrt(D) on the low-res map",
     "logit[(size_t)r * nbr + c] = s * scale;", "logit[(size_t)r * nbr + c] = s;",
     ["logits", "block_constant"]),
    ("transposed low-res operands",
     "s += qhat[(size_t)r * D + d] * khat[(size_t)c * D + d];",
     "s += qhat[(size_t)c * D + d] * khat[(size_t)r * D + d];",
     ["logits", "block_constant"]),
    ("wrong sign of the first-n prior",
     "if (first_n > 0 && (r < first_n || c < first_n)) v += ORACLE_PRIOR_BIAS;",
     "if (first_n > 0 && (r < first_n || c < first_n)) v -= ORACLE_PRIOR_BIAS;",
     ["keys", "priors"]),
    ("reversed tie rule",
     "return (a->idx > b->idx) - (a->idx < b->idx);",
     "return (a->idx < b->idx) - (a->idx > b->idx);",
     ["brute", "ties"]),
    ("mask ignored in pooling",
     "double m = mask_row ? mask_row[t] : 1.0;", "double m = 1.0;",
     ["pool", "block_constant"]),
    ("padded keys kept in the high-resolution part",
     "if (mask_row && !(mask_row[j] > 0.0)) continue;", "",
     ["dense"]),
    ("row max over empty columns too",
     "if (!(cnt_row[c] > 0.0)) continue;\n            double v = logit",
     "double v = logit",
     ["keys"]),
    ("diagonal band one diagonal too wide",
     "int hi = (g + 1) / 2 - 1;", "int hi = (g + 1) / 2;",
     ["band", "keys"]),
    ("empty-row penalty dropped",
     "if (!(cnt_row[r] > 0.0)) v -= ORACLE_EMPTY_PENALTY;", "",
     ["keys"]),
    ("softmax over high-res scores without the exponent",
     "double w = exp(s[j] - mx);", "double w = s[j] - mx;",
     ["dense", "sum_to_one"]),
    ("num_block without the cap at the full block count",
     "return budget < all ? budget : all;", "return budget;",
     ["num_block"]),
    ("backward: score gradient without the output term",
     "double ds = p * (dot - delta);", "double ds = p * dot;",
     ["bwd_dense", "bwd_fd"]),
    ("backward: low-resolution logit gradient dropped",
     "dl[(size_t)r * nbr + c] += p * (dot - delta);", "",
     ["bwd_dense_full"]),
    ("backward: block-mean gradient not divided by the count",
     "dq[(size_t)t * D + d] += dqh[(size_t)b * D + d] / cnt_row[b];",
     "dq[(size_t)t * D + d] += dqh[(size_t)b * D + d];",
     ["bwd_dense_full"]),
    ("backward: key gradient without 1/sqrt(D)",
     "dk[(size_t)j * D + d] += ds * scale * qi[d];", "dk[(size_t)j * D + d] += ds * qi[d];",
     ["bwd_dense", "bwd_saturated"]),
]

PINS = {
    "num_block": lambda: pins.test_num_block_matches_page_example(),
    "pool": lambda: pins.test_block_counts_and_pool_closed_form(),
    "logits": lambda: pins.test_lowres_logits_closed_form(),
    "keys": lambda: pins.test_row_max_penalties_and_priors_closed_form(),
    "band": lambda: pins.test_diagonal_band_widths(),
    "brute": lambda: pins.test_select_matches_brute_force(8, 16, 2),
    "ties": lambda: pins.test_tie_rule_on_all_zero_queries(),
    "priors": lambda: pins.test_priors_present_when_they_fit(),
    "dense": lambda: pins.test_saturated_budget_equals_dense(0, [0, 45]),
    "block_constant": lambda: pins.test_block_constant_qk_full_mode_equals_dense(1, 0, 0, [0, 45]),
    "sum_to_one": lambda: pins.test_rows_sum_to_one(1),
    "probe": lambda: pins.test_one_hot_value_probe_measures_block_mass(),
    "bwd_dense": lambda: bwd.test_backward_equals_autograd_of_dense_restatement(1, [20, 0], 2, 1, 1),
    "bwd_dense_full": lambda: bwd.test_backward_equals_autograd_of_dense_restatement(0, [64, 40], 3, 2, 3),
    "bwd_saturated": lambda: bwd.test_saturated_budget_backward_equals_dense_attention_autograd([0, 45]),
    "bwd_fd": lambda: bwd.test_backward_matches_finite_differences(0),
}


@pytest.mark.parametrize("name,old,new,catchers", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_fails_a_pin(tmp_path, name, old, new, catchers):
    src = oracle.source_text()
    assert old in src, f"mutation anchor not found: {name}"
    lib = oracle.compile_variant(src.replace(old, new), str(tmp_path))
    caught = []
    with oracle.use_variant(lib):
        for pin in catchers:
            try:
                PINS[pin]()
            except (AssertionError, ValueError):
                caught.append(pin)
    assert caught, f"no pin caught the planted mistake: {name}"


def test_unmutated_source_passes_the_same_pins(tmp_path):
    lib = oracle.compile_variant(oracle.source_text(), str(tmp_path))
    with oracle.use_variant(lib):
        for fn in PINS.values():
            fn()
