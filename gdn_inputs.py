"""Seeded synthetic inputs for the gated-delta-rule tree-verify path.

This module is shared by the tests, the benchmark and the smoke check. It holds
none of the method's arithmetic: it only draws random tensors, builds draft
trees and picks accept paths.  Both the CUDA library and the CPU oracle consume
what it returns; neither is imported here.

Workload shapes follow the pages:

* DDTree-style draft trees (DDTree budget 22, block 16, depth <= 16): the
  GreenGames post, "From autoregressive to DDTree" and "Key wins"
  (``build_ddtree`` with per-depth top-k candidates, rank 0 = best candidate,
  ``budget + 1`` verified positions).
* DFlash chains of 16 (block size 16): the GreenGames post, "Prefill".
* Qwen3.5/3.6-27B GDN geometry, 48 GDN layers of 64: the GreenGames post,
  "Why the experiment exists", and the magik.net essay, "The Broader Context".

Value recipe (per node and head): q, k ~ N(0,1) then L2-normalised over d_k with
no epsilon; v ~ N(0,1); g = -softplus(N(0,1)) (or g = ln U(0.5, 1) for the long
chain); beta = sigmoid(N(0,1)); state_in ~ N(0, 0.1^2).  q/k/v are then rounded
to the requested input dtype (bf16 or f32); the rounded values are what both
sides see.  Draw order from one ``torch.Generator``: tree, q, k, v, g, beta,
state_in, accept path.  With ``raw_gates`` the g and beta draws are returned
as drawn (the N(0,1) pre-activations), for callers that apply the gate maps
themselves.
"""
from __future__ import annotations

import dataclasses
import heapq
import math
from typing import List, Optional, Sequence

import numpy as np
import torch

# ---------------------------------------------------------------------------
# Trees
# ---------------------------------------------------------------------------


def chain_tree(n_nodes: int) -> np.ndarray:
    """parent[i] = i - 1 (a width-1 tree, i.e. a DFlash chain)."""
    p = np.arange(-1, n_nodes - 1, dtype=np.int32)
    return p


def random_tree(n_nodes: int, gen: torch.Generator) -> np.ndarray:
    """parent[0] = -1 and parent[i] uniform over 0..i-1."""
    p = np.empty(n_nodes, dtype=np.int32)
    p[0] = -1
    for i in range(1, n_nodes):
        p[i] = int(torch.randint(0, i, (1,), generator=gen).item())
    return p


def ddtree_like_tree(budget: int, gen: torch.Generator, top_k: int = 4,
                     max_depth: int = 16) -> np.ndarray:
    """Best-first draft tree over per-depth top-k candidates.

    Synthetic stand-in for the drafter's per-position top-k (the GreenGames
    post, "From autoregressive to DDTree" and "Key wins"): lp[d][r] ~ N(0,1)
    for depth d = 1..max_depth and rank r = 0..top_k-1, each row sorted in
    descending order so rank 0 is the best candidate.  A node at depth d
    reached through ranks (r_1..r_d) scores sum_i lp[i][r_i].  Starting from
    the root's children, the best-scoring frontier node is popped, given the
    next node index, and its children are pushed (while depth < max_depth),
    until ``budget`` drafts are taken.  Ties break by lower depth, then lower
    rank, then earlier insertion.  Node 0 is the root; parent[n] < n holds by
    construction.  Returns an int32 array of length budget + 1.
    """
    lp = torch.randn(max_depth + 1, top_k, generator=gen, dtype=torch.float64)
    lp, _ = torch.sort(lp, dim=1, descending=True)
    lp = lp.numpy()
    parent = [-1]
    heap: list = []
    counter = 0
    for r in range(top_k):
        # heapq is a min-heap: negate the score.
        heapq.heappush(heap, (-lp[1][r], 1, r, counter, 0))
        counter += 1
    while len(parent) < budget + 1 and heap:
        neg_score, depth, rank, _, par = heapq.heappop(heap)
        idx = len(parent)
        parent.append(par)
        if depth < max_depth:
            for r in range(top_k):
                heapq.heappush(heap, (neg_score - lp[depth + 1][r], depth + 1, r, counter, idx))
                counter += 1
    return np.asarray(parent, dtype=np.int32)


def draft_logprobs(batch: int, max_depth: int, top_k: int, gen: torch.Generator,
                   quantum: float = 0.0) -> np.ndarray:
    """Synthetic drafter output for the tree builder: [batch][max_depth][top_k]
    float32 log-probabilities, each row non-increasing (rank 0 best).

    Per position: logits z ~ N(0, 2^2) for the top_k candidates and one more
    entry r ~ N(0, 1) standing for the rest of the vocabulary; the row is
    log_softmax([z, r]) restricted to the candidates, sorted descending.  With
    quantum > 0 the values are rounded down to multiples of it, which makes
    exact ties common.
    """
    z = torch.randn(batch, max_depth, top_k, generator=gen, dtype=torch.float64) * 2.0
    r = torch.randn(batch, max_depth, 1, generator=gen, dtype=torch.float64)
    lp = torch.log_softmax(torch.cat([z, r], dim=2), dim=2)[:, :, :top_k]
    lp, _ = torch.sort(lp, dim=2, descending=True)
    lp = lp.numpy()
    if quantum > 0:
        lp = np.floor(lp / quantum) * quantum
    return np.ascontiguousarray(lp, dtype=np.float32)


def tree_depths(parent: Sequence[int]) -> np.ndarray:
    d = np.zeros(len(parent), dtype=np.int32)
    for n in range(1, len(parent)):
        d[n] = d[parent[n]] + 1
    return d


def tree_leaves(parent: Sequence[int]) -> List[int]:
    has_child = np.zeros(len(parent), dtype=bool)
    for n in range(1, len(parent)):
        has_child[parent[n]] = True
    return [n for n in range(len(parent)) if not has_child[n]]


def root_path(parent: Sequence[int], node: int) -> List[int]:
    """Node indices from the root (0) to ``node`` inclusive."""
    path = []
    n = int(node)
    while n >= 0:
        path.append(n)
        n = int(parent[n])
    return path[::-1]


# ---------------------------------------------------------------------------
# Problems
# ---------------------------------------------------------------------------


@dataclasses.dataclass
class Problem:
    """One layer's worth of tree-verify inputs, on the host.

    Layouts (row-major, last index contiguous):
      q, k      [B][N][H_k][d_k]   torch bf16 or f32
      v         [B][N][H_v][d_v]   torch bf16 or f32
      g, beta   [B][N][H_v]        torch f32
      parent    [B][N]             torch int32 (parent[b][0] = -1)
      state_in  [B][H_v][d_v][d_k] torch f32
      accept_path [B][P]           torch int32, -1 padded
      accept_len  [B]              torch int32
    """
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor
    beta: torch.Tensor
    parent: torch.Tensor
    state_in: torch.Tensor
    accept_path: torch.Tensor
    accept_len: torch.Tensor
    scale: float

    @property
    def batch(self) -> int:
        return self.q.shape[0]

    @property
    def n_nodes(self) -> int:
        return self.q.shape[1]

    @property
    def n_k_heads(self) -> int:
        return self.q.shape[2]

    @property
    def n_v_heads(self) -> int:
        return self.v.shape[2]

    @property
    def d_k(self) -> int:
        return self.q.shape[3]

    @property
    def d_v(self) -> int:
        return self.v.shape[3]


_DTYPES = {"bf16": torch.bfloat16, "f32": torch.float32}


def _l2n(x: torch.Tensor) -> torch.Tensor:
    # Input preparation (q/k normalisation happens before the call; epsilon 0).
    return x / torch.linalg.vector_norm(x, dim=-1, keepdim=True)


def make_problem(*, batch: int, n_nodes: int, n_k_heads: int, n_v_heads: int,
                 d_k: int, d_v: int, tree: str, seed: int, qkv_dtype: str = "bf16",
                 gate: str = "softplus", scale: Optional[float] = None,
                 accept: str = "leaf", top_k: int = 4, max_depth: int = 16,
                 parents: Optional[np.ndarray] = None, raw_gates: bool = False) -> Problem:
    """Draw one seeded problem.

    tree: "chain" | "random" | "ddtree" | "given" (then ``parents`` [B][N]).
      For "ddtree" and "random" each sequence b gets its own tree from its own
      generator seeded with seed + b; the remaining tensors come from one
      generator seeded with ``seed`` (drawn after the trees).
    gate: "softplus" -> g = -softplus(N(0,1)); "uniform_a" -> g = ln U(0.5, 1).
    raw_gates (with gate "softplus"): g and beta hold the N(0,1) draws
      themselves, untransformed (the same draws as without it).
    accept: "leaf" -> root to a uniformly chosen leaf; "prefix" -> root to a
      uniformly chosen node on the chain (chains); "node" -> root to a
      uniformly chosen node; "root" -> the root alone (no tree walk, so it
      also works for malformed trees).
    """
    gen = torch.Generator().manual_seed(seed)
    if tree == "given":
        assert parents is not None
        par = np.asarray(parents, dtype=np.int32).reshape(batch, n_nodes)
    else:
        rows = []
        for b in range(batch):
            if tree == "chain":
                rows.append(chain_tree(n_nodes))
            elif tree == "random":
                rows.append(random_tree(n_nodes, torch.Generator().manual_seed(seed + b)))
            elif tree == "ddtree":
                rows.append(ddtree_like_tree(n_nodes - 1, torch.Generator().manual_seed(seed + b),
                                             top_k=top_k, max_depth=max_depth))
            else:
                raise ValueError(tree)
        par = np.stack(rows).astype(np.int32)
    dt = _DTYPES[qkv_dtype]
    q = _l2n(torch.randn(batch, n_nodes, n_k_heads, d_k, generator=gen)).to(dt)
    k = _l2n(torch.randn(batch, n_nodes, n_k_heads, d_k, generator=gen)).to(dt)
    v = torch.randn(batch, n_nodes, n_v_heads, d_v, generator=gen).to(dt)
    if raw_gates and gate != "softplus":
        raise ValueError("raw_gates needs gate='softplus'")
    if gate == "softplus":
        g = torch.randn(batch, n_nodes, n_v_heads, generator=gen)
        if not raw_gates:
            g = -torch.nn.functional.softplus(g)
    elif gate == "uniform_a":
        a = 0.5 + 0.5 * torch.rand(batch, n_nodes, n_v_heads, generator=gen)
        g = torch.log(a)
    else:
        raise ValueError(gate)
    beta = torch.randn(batch, n_nodes, n_v_heads, generator=gen)
    if not raw_gates:
        beta = torch.sigmoid(beta)
    state_in = 0.1 * torch.randn(batch, n_v_heads, d_v, d_k, generator=gen)
    paths = []
    for b in range(batch):
        if accept == "root":
            paths.append([0])
            continue
        if accept == "leaf":
            cands = tree_leaves(par[b])
        elif accept in ("prefix", "node"):
            cands = list(range(n_nodes))
        else:
            raise ValueError(accept)
        pick = cands[int(torch.randint(0, len(cands), (1,), generator=gen).item())]
        paths.append(root_path(par[b], pick))
    plen = max(len(p) for p in paths)
    ap = torch.full((batch, plen), -1, dtype=torch.int32)
    for b, p in enumerate(paths):
        ap[b, :len(p)] = torch.tensor(p, dtype=torch.int32)
    al = torch.tensor([len(p) for p in paths], dtype=torch.int32)
    return Problem(q=q.contiguous(), k=k.contiguous(), v=v.contiguous(),
                   g=g.float().contiguous(), beta=beta.float().contiguous(),
                   parent=torch.from_numpy(par).contiguous(), state_in=state_in.float().contiguous(),
                   accept_path=ap.contiguous(), accept_len=al.contiguous(),
                   scale=(1.0 / math.sqrt(d_k)) if scale is None else float(scale))


def make_device_inputs(*, parent: np.ndarray, n_k_heads: int, n_v_heads: int, d_k: int, d_v: int,
                       seed: int, device, qkv_dtype: str = "bf16") -> dict:
    """One layer's q, k, v, g, beta and state_in for the trees in ``parent``
    ([B][N] int32), drawn on ``device`` with a seeded device generator.

    The value recipe is make_problem's (q, k ~ N(0,1) L2-normalised over d_k,
    v ~ N(0,1), g = -softplus(N(0,1)), beta = sigmoid(N(0,1)), state_in ~
    N(0, 0.1^2), q/k/v rounded to the input dtype); only the generator
    differs, so large timing workloads need not be drawn on the host.
    Returns device tensors keyed q, k, v, g, beta, state_in, parent.
    """
    par = torch.from_numpy(np.ascontiguousarray(parent, dtype=np.int32))
    B, N = par.shape
    gen = torch.Generator(device=device).manual_seed(seed)
    dt = _DTYPES[qkv_dtype]

    def randn(*shape):
        return torch.randn(*shape, generator=gen, device=device)

    q = _l2n(randn(B, N, n_k_heads, d_k)).to(dt)
    k = _l2n(randn(B, N, n_k_heads, d_k)).to(dt)
    v = randn(B, N, n_v_heads, d_v).to(dt)
    g = -torch.nn.functional.softplus(randn(B, N, n_v_heads))
    beta = torch.sigmoid(randn(B, N, n_v_heads))
    state_in = 0.1 * randn(B, n_v_heads, d_v, d_k)
    return dict(q=q.contiguous(), k=k.contiguous(), v=v.contiguous(), g=g.contiguous(),
                beta=beta.contiguous(), state_in=state_in.contiguous(), parent=par.to(device))


# The five workloads.  Sizes are per layer; ``layers`` is how many GDN layers a
# step stacks (each layer with its own buffers).
WORKLOADS = {
    "tiny_tree8_d32": dict(batch=1, n_nodes=8, n_k_heads=2, n_v_heads=4, d_k=32, d_v=32,
                           tree="random", qkv_dtype="f32", accept="leaf", layers=1),
    "dflash_chain16": dict(batch=1, n_nodes=16, n_k_heads=16, n_v_heads=48, d_k=128, d_v=128,
                           tree="chain", qkv_dtype="bf16", accept="prefix", layers=48),
    "ddtree_budget22": dict(batch=1, n_nodes=23, n_k_heads=16, n_v_heads=48, d_k=128, d_v=128,
                            tree="ddtree", qkv_dtype="bf16", accept="leaf", layers=48),
    "batched_budget64": dict(batch=32, n_nodes=65, n_k_heads=16, n_v_heads=48, d_k=128, d_v=128,
                             tree="ddtree", qkv_dtype="bf16", accept="leaf", layers=48),
    "long_chain4096": dict(batch=8, n_nodes=4096, n_k_heads=16, n_v_heads=48, d_k=128, d_v=128,
                           tree="chain", qkv_dtype="bf16", gate="uniform_a", accept="prefix",
                           layers=1),
}


def make_workload(name: str, seed: int = 0, **override) -> Problem:
    kw = dict(WORKLOADS[name])
    kw.pop("layers")
    kw.update(override)
    return make_problem(seed=seed, **kw)
