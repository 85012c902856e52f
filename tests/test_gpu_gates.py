"""GDN_FLAG_GATES: g and beta given as raw pre-activations x, y; the kernels
apply g = -softplus(x) and beta = sigmoid(y) (the workloads' gate recipe)
once per node.  The oracle applies the same maps in double first
(oracle.verify(raw_gates=True))."""
import numpy as np
import pytest
import torch

import gated_deltanet_tree_verify_b200 as gdn
import oracle
from gdn_inputs import make_problem
from tests.gpu_util import assert_out_close, assert_states_close, run

pytestmark = pytest.mark.gpu

GATES = gdn.GDN_FLAG_GATES


def _problem(**kw):
    return make_problem(qkv_dtype="bf16", raw_gates=True, **kw)


def _scale_qk(prob, seed=0):
    """Raw, non-unit q and k rows (as the q/k normalisation tests use)."""
    g = torch.Generator().manual_seed(seed)
    for key in ("q", "k"):
        x = getattr(prob, key)
        f = torch.empty(x.shape[:3] + (1,)).uniform_(0.25, 4.0, generator=g)
        setattr(prob, key, (x.float() * f).to(x.dtype).contiguous())
    return prob


def _check(prob, sd, flags=0, pairs=None, workspace=False):
    norm = bool(flags & gdn.GDN_FLAG_QK_L2NORM)
    last = bool(flags & gdn.GDN_FLAG_PERSIST_LAST)
    res = run(prob, sd, flags=flags | GATES, workspace=workspace, commit=not last)
    assert res["status"] == 0
    if pairs is None:
        out, _, ex = oracle.verify_problem(prob, state_dtype=sd, want_exact=True, nthreads=8, qk_l2norm=norm,
                                           raw_gates=True)
        assert_out_close(res["out"], out)
        assert_states_close(res["node_states"][:, 0] if last else res["node_states"], ex[:, -1] if last else ex,
                            sd)
        return res
    G = prob.n_v_heads // prob.n_k_heads
    for b, h in pairs:
        hk = h // G
        out, _, ex = oracle.verify(prob.q[b:b + 1, :, hk:hk + 1], prob.k[b:b + 1, :, hk:hk + 1],
                                   prob.v[b:b + 1, :, h:h + 1], prob.g[b:b + 1, :, h:h + 1],
                                   prob.beta[b:b + 1, :, h:h + 1], prob.parent[b:b + 1],
                                   prob.state_in[b:b + 1, h:h + 1], prob.scale, state_dtype=sd,
                                   want_exact=True, qk_l2norm=norm, raw_gates=True)
        assert_out_close(res["out"][b:b + 1, :, h:h + 1], out)
        assert_states_close(res["node_states"][b:b + 1, :, h:h + 1], ex, sd)
    return res


@pytest.mark.parametrize("sd", ["f32", "f16"])
def test_gates_ddtree_budget22(sd):
    prob = _problem(batch=2, n_nodes=23, n_k_heads=16, n_v_heads=48, d_k=128, d_v=128, tree="ddtree", seed=71)
    _check(prob, sd, pairs=[(0, 0), (1, 47), (1, 20)])


def test_gates_large_grid_wide_kernel():
    # batch 8, 65 nodes, f16: two rows per lane, 8-warp CTAs, shared-memory slots
    prob = _problem(batch=8, n_nodes=65, n_k_heads=16, n_v_heads=48, d_k=128, d_v=128, tree="ddtree", seed=72)
    _check(prob, "f16", pairs=[(0, 0), (7, 47), (3, 13)])


@pytest.mark.parametrize("sd", ["f32", "f16"])
def test_gates_chain_and_persist_last(sd):
    prob = _problem(batch=2, n_nodes=16, n_k_heads=2, n_v_heads=6, d_k=64, d_v=64, tree="chain", seed=73)
    _check(prob, sd, flags=gdn.GDN_FLAG_CHAIN)
    _check(prob, sd)
    long = _problem(batch=1, n_nodes=300, n_k_heads=1, n_v_heads=2, d_k=128, d_v=128, tree="chain", seed=74,
                    accept="prefix")
    _check(long, sd, flags=gdn.GDN_FLAG_CHAIN | gdn.GDN_FLAG_PERSIST_LAST)


def test_gates_recompute_workspace_and_ring_paths():
    # a complete binary tree exceeds the f16 stack slots (recomputation reads
    # the gates again); 129 nodes of budget 128 go through the ring kernel
    par = np.array([-1] + [(i - 1) // 2 for i in range(1, 127)], np.int32)
    prob = _problem(batch=1, n_nodes=127, n_k_heads=1, n_v_heads=3, d_k=128, d_v=128, tree="given",
                    parents=par[None], seed=75)
    _check(prob, "f16")
    _check(prob, "f16", workspace=True)
    big = _problem(batch=1, n_nodes=129, n_k_heads=16, n_v_heads=48, d_k=128, d_v=128, tree="ddtree", seed=76)
    _check(big, "f16", pairs=[(0, 0), (0, 31)])
    _check(big, "f32", pairs=[(0, 5)])


def test_gates_with_qk_normalisation():
    prob = _scale_qk(_problem(batch=2, n_nodes=33, n_k_heads=2, n_v_heads=6, d_k=128, d_v=128, tree="ddtree",
                              seed=77))
    _check(prob, "f32", flags=gdn.GDN_FLAG_QK_L2NORM)
    _check(prob, "f16", flags=gdn.GDN_FLAG_QK_L2NORM)


def test_gates_reset_at_positive_infinity():
    # x = +inf: a = 1 / (1 + e^x) = 0, the node's state forgets its parent
    prob = _problem(batch=1, n_nodes=12, n_k_heads=1, n_v_heads=2, d_k=32, d_v=32, tree="random", seed=78)
    prob.g[0, 5] = float("inf")
    prob.g[0, 9] = float("inf")
    res = _check(prob, "f32")
    st = res["node_states"].double().numpy()
    ex_k = prob.k[0, 5, 0].double().numpy()
    be = 1.0 / (1.0 + np.exp(-prob.beta[0, 5, 0].double().item()))
    v = prob.v[0, 5, 0].double().numpy()
    np.testing.assert_allclose(st[0, 5, 0], be * np.outer(v, ex_k), rtol=0, atol=1e-6)


def test_gates_flag_changes_results():
    prob = _problem(batch=1, n_nodes=8, n_k_heads=1, n_v_heads=2, d_k=32, d_v=32, tree="random", seed=79)
    a = run(prob, "f32", flags=GATES)
    b = run(prob, "f32")
    assert (a["out"] - b["out"]).abs().max() > 1e-3


@pytest.mark.parametrize("sd", ["f32", "f16"])
def test_gates_varlen(sd):
    # packed trees of different sizes: each sequence against the oracle alone
    from tests.test_gpu_varlen import _run_varlen
    sizes, trees = [1, 9, 23, 40], ["chain", "random", "ddtree", "ddtree"]
    seqs = [_problem(batch=1, n_nodes=n, n_k_heads=4, n_v_heads=12, d_k=128, d_v=128, tree=t, seed=90 + i)
            for i, (n, t) in enumerate(zip(sizes, trees))]
    vr = _run_varlen(seqs, sd, flags=GATES, commit=False)
    assert vr["status"] == 0
    for i, s in enumerate(seqs):
        a, b = int(vr["cu"][i]), int(vr["cu"][i + 1])
        out, _, ex = oracle.verify_problem(s, state_dtype=sd, want_exact=True, nthreads=8, raw_gates=True)
        assert_out_close(vr["out"][a:b][None], out)
        assert_states_close(vr["node_states"][a:b][None], ex, sd)
