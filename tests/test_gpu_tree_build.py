"""gdn_build_tree against the oracle (oracle/tree_build.py): parent, depth,
rank, token and score of every node are compared exactly -- the pops are
integer decisions taken on float32 scores that both sides sum in the same
order and rounding."""
import numpy as np
import pytest
import torch

import gated_deltanet_tree_verify_b200 as gdn
from gdn_inputs import draft_logprobs
from oracle import tree_build as tb

pytestmark = pytest.mark.gpu


def _build(lp, budget, flags=0, ids=None, status=None, fill=None):
    B, D, K = lp.shape
    dev = torch.device("cuda")
    N = budget + 1
    lp_d = torch.from_numpy(np.ascontiguousarray(lp, dtype=np.float32)).to(dev)
    ids_d = torch.from_numpy(ids).to(dev) if ids is not None else None
    v = -7 if fill is None else fill
    par = torch.full((B, N), v, dtype=torch.int32, device=dev)
    dep = torch.full((B, N), v, dtype=torch.int32, device=dev)
    rk = torch.full((B, N), v, dtype=torch.int32, device=dev)
    tok = torch.full((B, N), v, dtype=torch.int32, device=dev) if ids is not None else None
    sc = torch.full((B, N), float(v), dtype=torch.float32, device=dev)
    desc = gdn.make_build_desc(batch=B, max_depth=D, top_k=K, budget=budget, flags=flags, status=status)
    gdn.gdn_build_tree(desc, lp_d, par, topk_ids=ids_d, node_depth=dep, node_rank=rk, node_token=tok,
                       node_score=sc)
    torch.cuda.synchronize()
    out = dict(parent=par.cpu().numpy(), depth=dep.cpu().numpy(), rank=rk.cpu().numpy(), score=sc.cpu().numpy())
    if tok is not None:
        out["token"] = tok.cpu().numpy()
    return out


def _check(lp, budget, chain_seed=False, ids=None):
    flags = gdn.GDN_BUILD_CHAIN_SEED if chain_seed else 0
    got = _build(lp, budget, flags, ids=ids)
    par, dep, rk, sc = tb.build_trees(lp, budget, chain_seed)
    np.testing.assert_array_equal(got["parent"], par)
    np.testing.assert_array_equal(got["depth"], dep)
    np.testing.assert_array_equal(got["rank"], rk)
    np.testing.assert_array_equal(got["score"].view(np.uint32), sc.view(np.uint32))  # bit-exact
    if ids is not None:
        B = lp.shape[0]
        want = np.full(par.shape, -1, np.int32)
        for b in range(B):
            for n in range(1, par.shape[1]):
                want[b, n] = ids[b, dep[b, n] - 1, rk[b, n]]
        np.testing.assert_array_equal(got["token"], want)


@pytest.mark.parametrize("B,D,K,budget", [
    (1, 16, 4, 22),       # the DDTree budget-22 workload shape
    (8, 16, 8, 22),
    (5, 16, 8, 64),       # B not a multiple of the trees per CTA
    (3, 16, 8, 128),
    (2, 4, 2, 30),        # the whole candidate tree (2 + 4 + 8 + 16)
    (4, 1, 16, 16),       # depth 1: every candidate is a child of the root
    (2, 40, 1, 40),       # top-1: a chain
    (3, 7, 3, 0),         # budget 0: the root alone
])
@pytest.mark.parametrize("chain_seed", [False, True])
def test_build_tree_matches_oracle(B, D, K, budget, chain_seed):
    gen = torch.Generator().manual_seed(1000 + B * 31 + D * 7 + K + budget)
    lp = draft_logprobs(B, D, K, gen)
    _check(lp, budget, chain_seed)


@pytest.mark.parametrize("quantum", [0.25, 1.0])
def test_build_tree_ties(quantum):
    # quantised log-probs: many exact score ties across depth, rank and parent
    gen = torch.Generator().manual_seed(77)
    lp = draft_logprobs(16, 8, 4, gen, quantum=quantum)
    _check(lp, 100)
    _check(lp, 100, chain_seed=True)


def test_build_tree_all_equal_and_minus_inf():
    lp = np.zeros((4, 5, 3), np.float32)
    _check(lp, 50)
    lp2 = np.zeros((3, 6, 4), np.float32)
    lp2[:, :, 2:] = -np.inf          # ranks 2 and 3 impossible: taken last, in key order
    lp2[1, 3, 1:] = -np.inf
    _check(lp2, 200)


def test_build_tree_max_size_sampled():
    # the largest budget at the largest D * K: B trees, all checked
    gen = torch.Generator().manual_seed(5)
    lp = draft_logprobs(6, 64, 64, gen)
    _check(lp, gdn.GDN_MAX_TREE_NODES - 1)
    _check(lp, gdn.GDN_MAX_TREE_NODES - 1, chain_seed=True)


def test_build_tree_tokens():
    gen = torch.Generator().manual_seed(9)
    lp = draft_logprobs(5, 16, 8, gen)
    ids = torch.randint(0, 150000, (5, 16, 8), generator=gen, dtype=torch.int32).numpy()
    _check(lp, 40, ids=ids)


def test_build_tree_feeds_verify_layout():
    # the output is a valid verify tree: parent[0] = -1, parent[n] in [0, n)
    gen = torch.Generator().manual_seed(11)
    lp = draft_logprobs(32, 16, 8, gen)
    got = _build(lp, 96)
    par = got["parent"]
    assert (par[:, 0] == -1).all()
    n = np.arange(1, 97)
    assert ((par[:, 1:] >= 0) & (par[:, 1:] < n)).all()
    assert (got["depth"][:, 1:] == got["depth"][np.arange(32)[:, None], par[:, 1:]] + 1).all()


def test_build_tree_validate_reports_bad_rows():
    gen = torch.Generator().manual_seed(13)
    lp = draft_logprobs(6, 8, 4, gen)
    lp[2, 3, [1, 2]] = lp[2, 3, [2, 1]]     # an unsorted row in sequence 2
    lp[4, 0, 0] = np.nan                     # NaN in sequence 4
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = _build(lp, 20, flags=gdn.GDN_BUILD_VALIDATE, status=status)
    assert int(status.item()) == gdn.GDN_ERR_BAD_INPUT
    for b in (2, 4):
        assert (got["parent"][b] == -7).all() and (got["depth"][b] == -7).all()
    good = [0, 1, 3, 5]
    par, dep, rk, sc = tb.build_trees(lp[good], 20)
    np.testing.assert_array_equal(got["parent"][good], par)
    np.testing.assert_array_equal(got["rank"][good], rk)
    # valid rows: no status
    status.zero_()
    _build(lp[good], 20, flags=gdn.GDN_BUILD_VALIDATE, status=status)
    assert int(status.item()) == 0


def test_build_tree_twice_same_result():
    gen = torch.Generator().manual_seed(17)
    lp = draft_logprobs(64, 16, 8, gen)
    a = _build(lp, 22)
    b = _build(lp, 22, fill=5)
    for key in a:
        np.testing.assert_array_equal(a[key], b[key])
