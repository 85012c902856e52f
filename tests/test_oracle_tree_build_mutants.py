"""The tree-builder oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of oracle/tree_build.py by text
substitution (a reversed tie-break, a score that is not summed along the
path, the wrong log-prob row, a dropped chain seed, a wrong parent, ...),
loads the copy as a module, points test_oracle_tree_build at it, and checks
that at least one of its pins fails.
"""
import types

import pytest

from oracle import tree_build
from tests import test_oracle_tree_build as pins

SRC = tree_build.__file__

MUTANTS = {
    "score_order_reversed": ("heapq.heappush(heap, (-float(s), d + 1, r, counter, node, s))",
                             "heapq.heappush(heap, (float(s), d + 1, r, counter, node, s))"),
    "deeper_first_on_ties": ("heapq.heappush(heap, (-float(s), d + 1, r, counter, node, s))",
                             "heapq.heappush(heap, (-float(s), -(d + 1), r, counter, node, s))"),
    "higher_rank_first_on_ties": ("heapq.heappush(heap, (-float(s), d + 1, r, counter, node, s))",
                                  "heapq.heappush(heap, (-float(s), d + 1, -r, counter, node, s))"),
    "later_insertion_first_on_ties": ("heapq.heappush(heap, (-float(s), d + 1, r, counter, node, s))",
                                      "heapq.heappush(heap, (-float(s), d + 1, r, -counter, node, s))"),
    "score_not_summed_along_path": ("s = np.float32(score[node] + lp[d][r])", "s = np.float32(lp[d][r])"),
    "wrong_log_prob_row": ("s = np.float32(score[node] + lp[d][r])",
                           "s = np.float32(score[node] + lp[max(d - 1, 0)][r])"),
    "chain_seed_ignored": ("    if chain_seed:\n", "    if False:\n"),
    "one_level_short": ("        if d >= max_depth:\n", "        if d >= max_depth - 1:\n"),
    "parent_is_previous_node": ("parent.append(c[4])", "parent.append(len(parent) - 1)"),
    "rank_recorded_wrong": ("rank.append(c[2])", "rank.append(0)"),
}

PINS = [
    pins.test_hand_worked_example,
    pins.test_ties_break_by_depth_then_rank_then_insertion,
    pins.test_chain_seed_takes_the_greedy_chain_first,
    *[(lambda s=s: pins.test_best_first_equals_brute_force_top_budget(s)) for s in range(8)],
    pins.test_invariants_on_random_trees,
    pins.test_scores_are_float32_sums_along_the_path,
    pins.test_build_trees_stacks_sequences,
    *[(lambda s=s: pins.test_heap_order_equals_scan_of_all_open_children(s)) for s in range(6)],
]


def _mutant(old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("tree_build_mutant")
    exec(compile(src.replace(old, new), "tree_build_mutant.py", "exec"), mod.__dict__)
    return mod


def test_unmutated_oracle_passes_every_pin():
    for pin in PINS:
        pin()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_tree_build_mutant(name, monkeypatch):
    monkeypatch.setattr(pins, "tb", _mutant(*MUTANTS[name]))
    caught = 0
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError, StopIteration, IndexError, KeyError):
            caught += 1
    assert caught, f"no pin caught mutant {name}"
