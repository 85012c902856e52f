"""Pins of the draft-tree construction oracle (oracle/tree_build.py) against
a hand-worked example, brute-force enumeration and the invariants the
construction fixes."""
import itertools

import numpy as np
import pytest

from oracle import tree_build as tb


def test_hand_worked_example():
    # depth 1: ranks (-0.1, -1.0); depth 2: ranks (-0.2, -0.5); budget 4.
    # scores: a=(0)->-0.1, b=(1)->-1.0, a0=-0.3, a1=-0.6, b0=-1.2, b1=-1.5
    # best first: a (-0.1), a0 (-0.3), a1 (-0.6), b (-1.0)
    lp = np.array([[-0.1, -1.0], [-0.2, -0.5]])
    par, dep, rk, _ = tb.build_tree(lp, 4)
    assert par.tolist() == [-1, 0, 1, 1, 0]
    assert dep.tolist() == [0, 1, 2, 2, 1]
    assert rk.tolist() == [0, 0, 0, 1, 1]


def test_ties_break_by_depth_then_rank_then_insertion():
    lp = np.array([[0.0, 0.0], [0.0, 0.0]])     # every score is 0
    par, dep, rk, _ = tb.build_tree(lp, 6)
    # depth 1 first (ranks 0, 1), then depth 2 in insertion order:
    # children of node 1 (ranks 0, 1) were pushed before those of node 2
    assert dep.tolist() == [0, 1, 1, 2, 2, 2, 2]
    assert rk.tolist() == [0, 0, 1, 0, 0, 1, 1]
    assert par.tolist() == [-1, 0, 0, 1, 2, 1, 2]


def test_chain_seed_takes_the_greedy_chain_first():
    # siblings at depth 1 score well, the deeper greedy chain poorly: without
    # the seed the first picks are depth-1 siblings, with it the chain
    lp = np.array([[-0.1, -0.11, -0.12]] + [[-2.0, -2.5, -3.0]] * 5)
    par, dep, rk, _ = tb.build_tree(lp, 10, chain_seed=True)
    assert par[:7].tolist() == [-1, 0, 1, 2, 3, 4, 5]
    assert rk[1:7].tolist() == [0] * 6 and dep[1:7].tolist() == [1, 2, 3, 4, 5, 6]
    # after the chain, best-first: the depth-1 siblings of node 1
    assert par[7:9].tolist() == [0, 0] and rk[7:9].tolist() == [1, 2]
    par0, dep0, _, _ = tb.build_tree(lp, 10)
    assert dep0[1:4].tolist() == [1, 1, 1]
    # a short budget seeds only that much of the chain
    par2, _, _, _ = tb.build_tree(lp, 3, chain_seed=True)
    assert par2.tolist() == [-1, 0, 1, 2]


@pytest.mark.parametrize("seed", range(8))
def test_best_first_equals_brute_force_top_budget(seed):
    # with log-probs <= 0 scores never grow along a path, so best-first takes
    # exactly the budget highest-scoring rank sequences (prefix-closed)
    rng = np.random.default_rng(seed)
    D, K = 4, 3
    lp = np.sort(-rng.exponential(size=(D, K)).astype(np.float32), axis=1)[:, ::-1].copy()
    budget = int(rng.integers(1, 30))
    par, dep, rk, _ = tb.build_tree(lp, budget)
    # the rank path of every taken node
    paths = {0: ()}
    for n in range(1, len(par)):
        paths[n] = paths[par[n]] + (int(rk[n]),)
    taken = sorted(paths[n] for n in range(1, len(par)))
    # brute force over all sequences, scores in float32 from the root
    allseq = []
    for d in range(1, D + 1):
        for seq in itertools.product(range(K), repeat=d):
            s = np.float32(0.0)
            for i, r in enumerate(seq):
                s = np.float32(s + lp[i][r])
            allseq.append((-float(s), d, seq))
    allseq.sort()
    top = sorted(x[2] for x in allseq[:budget])
    # equal scores at the cut could pick a different member; check only when
    # the cut is strict
    if budget == len(allseq) or allseq[budget - 1][0] != allseq[budget][0]:
        assert taken == top


def test_invariants_on_random_trees():
    rng = np.random.default_rng(7)
    for _ in range(20):
        D, K = int(rng.integers(1, 9)), int(rng.integers(1, 5))
        lp = np.sort(rng.normal(size=(D, K)).astype(np.float32), axis=1)[:, ::-1].copy()
        budget = int(rng.integers(0, min(60, tb.reachable(D, K)) + 1))
        par, dep, rk, _ = tb.build_tree(lp, budget, chain_seed=bool(rng.integers(2)))
        assert len(par) == budget + 1 and par[0] == -1
        for n in range(1, len(par)):
            assert 0 <= par[n] < n
            assert dep[n] == dep[par[n]] + 1 <= D
            assert 0 <= rk[n] < K
        # no two siblings share a rank
        pairs = [(par[n], rk[n]) for n in range(1, len(par))]
        assert len(set(pairs)) == len(pairs)


def test_budget_beyond_the_candidate_tree_is_refused():
    with pytest.raises(ValueError):
        tb.build_tree(np.zeros((2, 1)), 3)   # a chain of 2 holds 2 drafts
    assert tb.reachable(2, 1) == 2 and tb.reachable(3, 2) == 14


def test_scores_are_float32_sums_along_the_path():
    rng = np.random.default_rng(3)
    lp = np.sort(rng.normal(size=(5, 4)).astype(np.float32), axis=1)[:, ::-1].copy()
    par, dep, rk, sc = tb.build_tree(lp, 40)
    for n in range(1, 41):
        path = []
        m = n
        while m:
            path.append(m)
            m = par[m]
        s = np.float32(0.0)
        for node in reversed(path):
            s = np.float32(s + lp[dep[node] - 1][rk[node]])
        assert sc[n] == s


def test_build_trees_stacks_sequences():
    lp = np.stack([np.array([[-0.1, -1.0], [-0.2, -0.5]]), np.array([[-1.0, -1.0], [-0.2, -0.5]])])
    par, dep, rk, sc = tb.build_trees(lp, 4)
    assert par.shape == (2, 5) and par[0].tolist() == [-1, 0, 1, 1, 0]
    # second: ties at depth 1 -> both depth-1 nodes (-1.0) then their rank-0 children (-1.2)
    assert par[1].tolist() == [-1, 0, 0, 1, 2]


@pytest.mark.parametrize("seed", range(6))
def test_heap_order_equals_scan_of_all_open_children(seed):
    # independent statement of the rule: at every step, among all children of
    # taken nodes not yet taken, take the one with the highest float32 score,
    # then lower depth, lower rank, lower parent index.  Quantised log-probs
    # make exact ties common, so every tie-break level is exercised.
    rng = np.random.default_rng(100 + seed)
    D, K = int(rng.integers(1, 5)), int(rng.integers(1, 4))
    lp = np.sort(-0.25 * rng.integers(0, 4, size=(D, K)), axis=1)[:, ::-1].astype(np.float32)
    budget = int(rng.integers(0, min(40, tb.reachable(D, K)) + 1))
    seed_chain = bool(seed % 2)
    par, dep, rk, sc = tb.build_tree(lp, budget, chain_seed=seed_chain)
    t_par, t_dep, t_rk, t_sc = [-1], [0], [0], [np.float32(0.0)]
    taken = {(-1, 0)}
    chain = min(D, budget) if seed_chain else 0
    while len(t_par) < budget + 1:
        n = len(t_par)
        if n <= chain:
            best = (n - 1, 0)
        else:
            best, bkey = None, None
            for p in range(n):
                if t_dep[p] >= D:
                    continue
                for r in range(K):
                    if (p, r) in taken:
                        continue
                    s = np.float32(t_sc[p] + lp[t_dep[p]][r])
                    key = (-float(s), t_dep[p] + 1, r, p)
                    if bkey is None or key < bkey:
                        best, bkey = (p, r), key
        p, r = best
        taken.add(best)
        t_par.append(p)
        t_dep.append(t_dep[p] + 1)
        t_rk.append(r)
        t_sc.append(np.float32(t_sc[p] + lp[t_dep[p]][r]))
    assert par.tolist() == t_par and dep.tolist() == t_dep and rk.tolist() == t_rk
    assert np.array_equal(sc, np.asarray(t_sc, np.float32))
