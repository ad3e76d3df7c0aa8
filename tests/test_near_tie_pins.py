"""The oracle's near-tie helpers pinned to hand-built rows (CPU only), and
planted mistakes in copies of them that the pins must catch."""
import os
import types

import pytest

from oracle.oracle import inner_gap, topk_gap
from tests.near_tie_pins import check_near_tie_helpers

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "oracle.py")

# (name, exact source text, replacement): plausible slips in the helpers.
MUTANTS = [
    ("topk_gap_off_by_one", "return s[:, k - 1] - s[:, k]\n", "return s[:, k] - s[:, k + 1]\n"),
    ("topk_gap_ascending_sort", "s = -np.sort(-probs, axis=1)\n    return s[:, k - 1]",
     "s = np.sort(probs, axis=1)\n    return s[:, k - 1]"),
    ("topk_gap_no_inf_at_k_equals_E", "if k >= E:\n        return np.full(T, np.inf)",
     "if k > E:\n        return np.full(T, np.inf)"),
    ("inner_gap_includes_boundary", "s = -np.sort(-probs, axis=1)[:, :k]", "s = -np.sort(-probs, axis=1)[:, :k + 1]"),
    ("inner_gap_ascending_sort", "s = -np.sort(-probs, axis=1)[:, :k]", "s = np.sort(probs, axis=1)[:, :k]"),
    ("inner_gap_max_not_min", "return np.min(s[:, :-1] - s[:, 1:], axis=1)",
     "return np.max(s[:, :-1] - s[:, 1:], axis=1)"),
    ("inner_gap_k1_not_inf", "if k < 2:\n        return np.full(T, np.inf)",
     "if k < 2:\n        return np.zeros(T)"),
]


def test_near_tie_helpers_pinned():
    check_near_tie_helpers(topk_gap, inner_gap)


def _load_mutant(old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site not found exactly once: {old!r}"
    mod = types.ModuleType("oracle_mutant")
    mod.__file__ = SRC
    exec(compile(src.replace(old, new), "oracle_mutant.py", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_near_tie_pins_catch_mutant(name, old, new):
    mod = _load_mutant(old, new)
    # a slip may show as a wrong value or as an indexing error; either is caught
    with pytest.raises((AssertionError, IndexError)):
        check_near_tie_helpers(mod.topk_gap, mod.inner_gap)
