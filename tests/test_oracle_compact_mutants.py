"""The compaction oracle's pins catch plausible mistakes.

Each case plants one mistake in the source of oracle.compact (the sequence's
node offset ignored, the path check dropped, the last path row skipped, the
varlen offsets replaced by uniform ones), compiles it in the oracle
module's namespace, swaps it in, and checks that a pin of
test_oracle_compact fails.
"""
import inspect

import pytest

import oracle
from tests import test_oracle_compact as pins

MUTANTS = {
    "node_offset_ignored": ("dst[b, i] = rows[n0 + int(accept_path[b, i])]",
                            "dst[b, i] = rows[int(accept_path[b, i])]"),
    "path_unchecked": ("if check_path(parent[n0:n1], accept_path[b], int(accept_len[b])) != OK:",
                       "if False:"),
    "last_row_skipped": ("for i in range(int(accept_len[b])):", "for i in range(int(accept_len[b]) - 1):"),
    "varlen_offsets_uniform": ("cu = np.asarray(cu_nodes, dtype=np.int64)",
                               "cu = np.arange(B + 1, dtype=np.int64) * (parent.shape[0] // B)"),
}

PINS = [pins.test_hand_worked_example, pins.test_bad_paths_write_nothing_for_their_sequence,
        pins.test_varlen_offsets, pins.test_last_compacted_state_is_the_committed_state]


def _mutant(old, new):
    src = inspect.getsource(oracle.compact)
    assert src.count(old) == 1, old
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), "compact_mutant.py", "exec"), ns)
    return ns["compact"]


def test_unmutated_compact_passes_every_pin():
    for pin in PINS:
        pin()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_compact_mutant(name, monkeypatch):
    monkeypatch.setattr(oracle, "compact", _mutant(*MUTANTS[name]))
    caught = 0
    for pin in PINS:
        try:
            pin()
        except (AssertionError, IndexError, ValueError):
            caught += 1
    assert caught, f"no pin caught mutant {name}"
