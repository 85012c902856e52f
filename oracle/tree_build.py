"""Oracle for draft-tree construction (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this module; the CUDA library never does.

What it computes: the best-first draft tree of DDTree-style speculative
decoding (the GreenGames post, "From autoregressive to DDTree": the tree is
built by ``build_ddtree`` from the drafter's per-position top-k candidates,
optionally pre-seeded with the greedy chain; "Key wins": candidates are
ordered best first, rank 0 at the root side).  The pages give no formula;
the reading taken here is:

* ``logp[d][r]`` is the log-probability of the rank-r candidate at draft
  position d + 1 (r = 0 the best, each row non-increasing).
* A node is a sequence of ranks (r_1 .. r_depth); its score is the sum of
  ``logp[i - 1][r_i]`` along its root path, accumulated in float32 from the
  root (score(child) = float32(score(parent) + logp[depth - 1][r])), so the
  order of near-equal candidates is decided in the kernel's precision.
* The root (node 0, depth 0, score 0) starts with its ``top_k`` children as
  candidates.  With the chain pre-seed, the rank-0 chain of depth
  min(max_depth, budget) is taken first, in depth order.  Then, until
  ``budget`` drafts are taken, the best candidate is taken: highest score,
  then lower depth, then lower rank, then earlier insertion.  A taken node
  gets the next index and, below ``max_depth``, its ``top_k`` children
  become candidates (in rank order).

Returns parent[budget + 1] (parent[0] = -1, parent[n] < n) and, per node,
depth, rank and score.
"""
from __future__ import annotations

import heapq
from typing import List

import numpy as np


def reachable(max_depth: int, top_k: int) -> int:
    """Number of non-root nodes of the full candidate tree (capped at 2^31)."""
    total, layer = 0, 1
    for _ in range(max_depth):
        layer *= top_k
        total += layer
        if total >= 2 ** 31:
            return 2 ** 31
    return total


def build_tree(logp, budget: int, chain_seed: bool = False):
    """Best-first tree for one sequence.  logp: [max_depth][top_k].

    Returns (parent, depth, rank, score), each of length budget + 1.  The
    candidates sit in a binary heap (heapq) ordered by (-score, depth, rank,
    insertion counter); every taken node pushes all of its top_k children.
    """
    lp = np.asarray(logp, dtype=np.float32)
    max_depth, top_k = lp.shape
    if budget > reachable(max_depth, top_k):
        raise ValueError("budget exceeds the candidate tree")
    parent: List[int] = [-1]
    depth: List[int] = [0]
    rank: List[int] = [0]
    score: List[np.float32] = [np.float32(0.0)]
    heap: list = []          # (-score, depth, rank, counter, parent, score)
    removed = set()          # counters taken out of turn (the chain seed)
    counter = 0

    def push_children(node: int):
        nonlocal counter
        d = depth[node]
        if d >= max_depth:
            return
        for r in range(top_k):
            s = np.float32(score[node] + lp[d][r])  # float32 add, round to nearest
            heapq.heappush(heap, (-float(s), d + 1, r, counter, node, s))
            counter += 1

    def take(c):
        parent.append(c[4])
        depth.append(c[1])
        rank.append(c[2])
        score.append(c[5])
        push_children(len(parent) - 1)

    push_children(0)
    if chain_seed:
        for d in range(1, min(max_depth, budget) + 1):
            prev = len(parent) - 1
            c = next(c for c in heap if c[1] == d and c[2] == 0 and c[4] == prev)
            removed.add(c[3])
            take(c)
    while len(parent) < budget + 1:
        c = heapq.heappop(heap)
        if c[3] in removed:
            continue
        take(c)
    return (np.asarray(parent, np.int32), np.asarray(depth, np.int32), np.asarray(rank, np.int32),
            np.asarray(score, np.float32))


def build_trees(logp, budget: int, chain_seed: bool = False):
    """build_tree for each sequence of logp [B][max_depth][top_k]; returns
    parent, depth, rank, score, each [B][budget + 1]."""
    lp = np.asarray(logp, dtype=np.float32)
    outs = [build_tree(lp[b], budget, chain_seed) for b in range(lp.shape[0])]
    return tuple(np.stack([o[i] for o in outs]) for i in range(4))
