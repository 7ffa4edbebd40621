"""Plant plausible mistakes in a copy of the lightning-indexer oracle (on the CPU) and
check that the pins reject every one of them."""

import os
import types

import pytest

import indexer_pins

SRC = os.path.join(os.path.dirname(__file__), os.pardir, "oracle", "indexer.py")

# (name, text in the oracle, replacement)
MUTANTS = [
    ("relu_dropped", "relu = np.maximum(dots, 0.0)", "relu = dots"),
    ("relu_wrong_side", "relu = np.maximum(dots, 0.0)", "relu = np.minimum(dots, 0.0)"),
    ("relu_after_weighting", "relu = np.maximum(dots, 0.0)        # negative correlations count as zero\n    return relu @ w",
     "relu = dots\n    return np.maximum(relu @ w, 0.0)"),
    ("head_weights_ignored", "return relu @ w                     # head-weighted sum",
     "return relu.sum(axis=1)"),
    ("head_weights_reversed", "return relu @ w                     # head-weighted sum",
     "return relu @ w[::-1]"),
    ("keys_reversed", "dots = K @ q.T", "dots = (K @ q.T)[::-1]"),
    ("key_dims_reversed", "dots = K @ q.T", "dots = K[:, ::-1] @ q.T"),
    ("candidate_window_shift", "indexer_scores_row(q[t], w[t], K[s0:s0 + nv])",
     "indexer_scores_row(q[t], w[t], K[s0 + 1:s0 + nv + 1])"),
    ("no_range_check", "if s0 < 0 or nv < 0 or s0 + nv > len(K):", "if False:"),
    ("ties_to_larger_index", "key=lambda i: (-s[i], i)", "key=lambda i: (-s[i], -i)"),
    ("ascending_order", "key=lambda i: (-s[i], i)", "key=lambda i: (s[i], i)"),
    ("one_short", ")[:k]\n", ")[:max(k - 1, 0)]\n"),
    ("pad_with_zero", "idx = np.full(k, -1, dtype=np.int64)", "idx = np.full(k, 0, dtype=np.int64)"),
]


def _mutant_module(old, new):
    src = open(SRC, encoding="utf-8").read()
    assert src.count(old) == 1, f"mutation anchor not unique/present: {old!r}"
    mod = types.ModuleType("indexer_mutant")
    exec(compile(src.replace(old, new), "indexer_mutant", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_mutant(name, old, new):
    mod = _mutant_module(old, new)
    failed = []
    for pin in indexer_pins.ALL_PINS:
        try:
            pin(mod)
        except Exception:  # noqa: BLE001 - any failure counts as a rejection
            failed.append(pin.__name__)
    assert failed, f"no pin rejects mutant {name}"
