"""Planted mistakes in the oracle's Python functions (the BigBird pattern and
the layer) must fail at least one of their pins.

Each case takes the function's source, plants one plausible mistake (a
narrower window, one global block instead of two, the full-attention
threshold off by one, the random blocks dropped, the heads split in the
wrong order, the bias dropped, the heads merged in the wrong order), builds
the mutated function in the oracle's namespace, swaps it in, and runs the
pins of test_oracle_bigbird_pins / test_oracle_layer_pins, expecting one to
fail.  Nothing here touches a GPU.
"""
import inspect
import textwrap

import numpy as np
import pytest

import oracle
import test_oracle_bigbird_pins as bb
import test_oracle_layer_pins as lp


def _mutant(fn, old, new):
    src = textwrap.dedent(inspect.getsource(fn))
    assert old in src, f"mutation anchor not found: {old!r}"
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new, 1), f"<mutant of {fn.__name__}>", "exec"), ns)
    return ns[fn.__name__]


def _fails(checks):
    for check in checks:
        try:
            check()
        except (AssertionError, ValueError, IndexError):
            return True
    return False


BIGBIRD_MUTATIONS = [
    ("window of two blocks", "sel[i, max(0, i - 1):min(nb, i + 2)] = True", "sel[i, max(0, i - 1):min(nb, i + 1)] = True"),
    ("one global block", "sel[i, [0, nb - 1]] = True", "sel[i, [0]] = True"),
    ("full-attention threshold off by one", "full = nb <= 5 + 2 * r", "full = nb < 5 + 2 * r"),
    ("random blocks dropped", "sel[i, rand_blocks[i]] = True", "pass"),
    ("global rows not attending to everything", "if full or i == 0 or i == nb - 1:", "if full:"),
]


@pytest.mark.parametrize("name,old,new", BIGBIRD_MUTATIONS, ids=[m[0] for m in BIGBIRD_MUTATIONS])
def test_bigbird_mutation_fails_a_pin(monkeypatch, name, old, new):
    monkeypatch.setattr(oracle, "bigbird_blocks", _mutant(oracle.bigbird_blocks, old, new))
    checks = [lambda: bb.test_pattern_rows_by_definition(2048, 64, 3),
              lambda: bb.test_short_sequences_use_full_attention()]
    checks += [lambda row=row: bb.test_keys_per_query_match_the_pages_count(*row) for row in bb._golden_counts()]
    assert _fails(checks), name


LAYER_MUTATIONS = [
    ("heads split in the wrong order", ".reshape(B, N, H, d).transpose(0, 2, 1, 3)", ".reshape(B, N, d, H).transpose(0, 3, 1, 2)"),
    ("bias dropped", "proj = proj + np.asarray(b_qkv, dtype=np.float64)", "proj = proj"),
    ("heads merged in the wrong order", "out.transpose(0, 2, 1, 3).reshape(B, N, hidden)", "out.transpose(0, 2, 3, 1).reshape(B, N, hidden)"),
    ("key and value weights swapped", "for j in range(3)]", "for j in (0, 2, 1)]"),
]


@pytest.mark.parametrize("name,old,new", LAYER_MUTATIONS, ids=[m[0] for m in LAYER_MUTATIONS])
def test_layer_mutation_fails_a_pin(monkeypatch, name, old, new):
    monkeypatch.setattr(oracle, "self_attention", _mutant(oracle.self_attention, old, new))
    checks = [lambda: lp.test_saturated_layer_equals_torch_multihead_attention(2, 64, 128, 2, [10, 0]),
              lambda: lp.test_saturated_layer_equals_torch_multihead_attention(1, 96, 96, 2, None),
              lambda: lp.test_one_identity_head_is_the_forward_pass(),
              lambda: lp.test_head_permutation_permutes_the_output()]
    assert _fails(checks), name


def test_unmutated_python_functions_pass_the_same_pins():
    assert not _fails([lambda: bb.test_pattern_rows_by_definition(2048, 64, 3),
                       lambda: bb.test_short_sequences_use_full_attention(),
                       lambda: lp.test_saturated_layer_equals_torch_multihead_attention(2, 64, 128, 2, [10, 0]),
                       lambda: lp.test_one_identity_head_is_the_forward_pass(),
                       lambda: lp.test_head_permutation_permutes_the_output()])
