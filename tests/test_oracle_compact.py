"""Pins of the oracle's accept-time compaction (oracle.compact)."""
import numpy as np

import oracle
from gdn_inputs import make_problem


def test_hand_worked_example():
    # two trees of 4 nodes: 0 -> 1 -> 3 and 0 -> 2
    parent = np.array([-1, 0, 0, 1, -1, 0, 1, 1], np.int32)
    rows = np.arange(8 * 3, dtype=np.float32).reshape(8, 3)
    path = np.array([[0, 1, 3], [0, 1, 2]], np.int32)
    length = np.array([3, 2], np.int32)
    dst, written = oracle.compact(rows, parent, path, length)
    assert dst[0].tolist() == [[0, 1, 2], [3, 4, 5], [9, 10, 11]]
    assert dst[1, :2].tolist() == [[12, 13, 14], [15, 16, 17]]
    assert written.tolist() == [[True, True, True], [True, True, False]]


def test_bad_paths_write_nothing_for_their_sequence():
    parent = np.array([-1, 0, 0, 1, -1, 0, 1, 1], np.int32)
    rows = np.ones((8, 2), np.float32)
    for bad in ([1, 1, 3], [0, 2, 3], [0, 4, 0]):      # not from the root; 3's parent is 1; out of range
        path = np.array([bad, [0, 1, 3]], np.int32)
        dst, written = oracle.compact(rows, parent, path, np.array([3, 3], np.int32))
        assert not written[0].any() and written[1].all()
    dst, written = oracle.compact(rows, parent, np.zeros((2, 3), np.int32), np.array([0, 4], np.int32))
    assert not written.any()                            # lengths 0 and > max_path_len


def test_varlen_offsets():
    parent = np.array([-1, 0, -1, 0, 1, 2], np.int32)   # trees of 2 and 4 nodes
    rows = np.arange(6, dtype=np.int64)[:, None] * 10
    cu = np.array([0, 2, 6])
    path = np.array([[0, 1, 0], [0, 1, 2]], np.int32)
    dst, written = oracle.compact(rows, parent, path, np.array([2, 3], np.int32), cu_nodes=cu)
    assert dst[0, :2, 0].tolist() == [0, 10] and dst[1, :, 0].tolist() == [20, 30, 40]


def test_last_compacted_state_is_the_committed_state():
    # compacting the persisted states along the path and taking the last row
    # is what commit writes
    prob = make_problem(batch=2, n_nodes=8, n_k_heads=2, n_v_heads=4, d_k=32, d_v=32, tree="random",
                        seed=4, qkv_dtype="f32", accept="leaf")
    _, states, _ = oracle.verify_problem(prob, state_dtype="f32")
    committed = oracle.commit(states, prob.parent, prob.accept_path, prob.accept_len)
    B, N = states.shape[:2]
    dst, written = oracle.compact(states.reshape(B * N, *states.shape[2:]), prob.parent.numpy().reshape(-1),
                                  prob.accept_path, prob.accept_len)
    for b in range(B):
        last = int(prob.accept_len[b]) - 1
        assert written[b, last]
        assert np.array_equal(dst[b, last], committed[b])
