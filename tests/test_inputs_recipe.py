"""The seeded input generator holds to the stated recipe: each named
workload's shapes and dtypes; q and k unit rows, v ~ N(0, 1), g =
-softplus(N(0, 1)) (or ln U(0.5, 1) for the long chain), beta =
sigmoid(N(0, 1)), state_in ~ N(0, 0.1^2); trees with parent[0] = -1 and
parent[n] < n; accept paths that start at the root and follow parent links;
the same seed giving the same draws."""
import numpy as np
import pytest
import torch

from gdn_inputs import WORKLOADS, make_problem, make_workload, tree_depths


def _small(name):
    # the long chain at full size is 8 x 4096 tokens: the recipe is the same
    # on a slice of it
    return make_workload(name, seed=3, batch=2, n_nodes=300) if name == "long_chain4096" \
        else make_workload(name, seed=3)


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_workload_shapes_and_dtypes(name):
    w = WORKLOADS[name]
    p = _small(name)
    B = 2 if name == "long_chain4096" else w["batch"]
    N = 300 if name == "long_chain4096" else w["n_nodes"]
    dt = torch.float32 if w["qkv_dtype"] == "f32" else torch.bfloat16
    assert p.q.shape == (B, N, w["n_k_heads"], w["d_k"]) and p.q.dtype == dt
    assert p.k.shape == (B, N, w["n_k_heads"], w["d_k"]) and p.k.dtype == dt
    assert p.v.shape == (B, N, w["n_v_heads"], w["d_v"]) and p.v.dtype == dt
    assert p.g.shape == p.beta.shape == (B, N, w["n_v_heads"])
    assert p.g.dtype == p.beta.dtype == torch.float32
    assert p.parent.shape == (B, N) and p.parent.dtype == torch.int32
    assert p.state_in.shape == (B, w["n_v_heads"], w["d_v"], w["d_k"]) and p.state_in.dtype == torch.float32
    assert p.scale == pytest.approx(w["d_k"] ** -0.5)


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_trees_and_accept_paths(name):
    w = WORKLOADS[name]
    p = _small(name)
    par = p.parent.numpy()
    for b in range(par.shape[0]):
        assert par[b, 0] == -1
        assert (par[b, 1:] >= 0).all() and (par[b, 1:] < np.arange(1, par.shape[1])).all()
        if w["tree"] == "chain":
            assert (par[b, 1:] == np.arange(par.shape[1] - 1)).all()
        if w["tree"] == "ddtree":
            assert tree_depths(par[b]).max() <= 16
            assert np.bincount(par[b, 1:], minlength=par.shape[1]).max() <= 4  # top-4 children
        L = int(p.accept_len[b])
        path = p.accept_path[b, :L].numpy()
        assert L >= 1 and path[0] == 0
        assert (p.accept_path[b, L:] == -1).all()
        assert all(par[b, path[i]] == path[i - 1] for i in range(1, L))
        if w["accept"] == "leaf":
            assert path[-1] not in set(par[b].tolist())   # a leaf: nobody's parent


def test_value_distributions():
    p = make_workload("ddtree_budget22", seed=5, batch=4)
    for x in (p.q, p.k):
        n = torch.linalg.vector_norm(x.float(), dim=-1)
        assert (n - 1).abs().max() < 1e-2                 # unit rows, up to bf16 rounding
    v = p.v.float()
    assert abs(v.mean().item()) < 0.02 and abs(v.std().item() - 1) < 0.02
    a = torch.exp(p.g)
    assert (p.g <= 0).all() and abs(a.mean().item() - 0.5) < 0.02   # a = sigmoid(-z), z ~ N(0, 1)
    assert ((p.beta > 0) & (p.beta < 1)).all() and abs(p.beta.mean().item() - 0.5) < 0.02
    assert abs(p.state_in.std().item() - 0.1) < 0.001 and abs(p.state_in.mean().item()) < 0.001


def test_long_chain_gate_spans_half_to_one():
    p = _small("long_chain4096")
    a = torch.exp(p.g)
    assert a.min() >= 0.5 - 1e-6 and a.max() <= 1.0
    assert abs(a.mean().item() - 0.75) < 0.01


def test_tiny_case_is_f32_random_tree():
    p = make_workload("tiny_tree8_d32", seed=0)
    assert p.q.dtype == torch.float32 and p.n_nodes == 8 and p.n_v_heads == 4 and p.n_k_heads == 2


def test_raw_gates_are_the_same_draws():
    kw = dict(batch=1, n_nodes=20, n_k_heads=2, n_v_heads=4, d_k=32, d_v=32, tree="random", seed=9)
    p = make_problem(**kw)
    r = make_problem(raw_gates=True, **kw)
    assert torch.allclose(p.g, -torch.nn.functional.softplus(r.g))
    assert torch.allclose(p.beta, torch.sigmoid(r.beta))
    assert torch.equal(p.q, r.q) and torch.equal(p.v, r.v) and torch.equal(p.state_in, r.state_in)


def test_seeding_is_deterministic():
    a = make_workload("ddtree_budget22", seed=11)
    b = make_workload("ddtree_budget22", seed=11)
    c = make_workload("ddtree_budget22", seed=12)
    for key in ("q", "k", "v", "g", "beta", "parent", "state_in", "accept_path"):
        assert torch.equal(getattr(a, key), getattr(b, key)), key
    assert not torch.equal(a.q, c.q) and not torch.equal(a.state_in, c.state_in)
