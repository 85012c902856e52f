"""Inputs at the library's maximum sizes.  Trees of GDN_MAX_TREE_NODES =
1024 nodes (random) and a caterpillar 511 levels deep, in both persisted
dtypes, checked node by node against the oracle (outputs, every persisted
state, and the commit of an accepted root-to-leaf path); one node more is
refused before any launch.  A chain of 65535 tokens (the most a desc
allows) by both chain paths.  These take the kernels' large-N routes (records
streamed through the ring, stack slots or parent re-reads) that the
budget-sized workloads never reach."""
import numpy as np
import pytest
import torch

import gated_deltanet_tree_verify_b200 as gdn
import oracle
from gdn_inputs import make_problem
from tests.gpu_util import assert_out_close, assert_states_close, run

pytestmark = pytest.mark.gpu


def _check(prob, sd):
    res = run(prob, sd)
    assert res["status"] == 0
    out, st, ex = oracle.verify_problem(prob, state_dtype=sd, want_exact=True, nthreads=8)
    assert_out_close(res["out"], out)
    assert_states_close(res["node_states"], ex, sd)
    so = oracle.commit(st, prob.parent, prob.accept_path, prob.accept_len)
    assert_states_close(res["state_out"], so, sd)


@pytest.mark.parametrize("sd", ["f32", "f16"])
def test_largest_random_tree(sd):
    prob = make_problem(batch=2, n_nodes=gdn.GDN_MAX_TREE_NODES, n_k_heads=1, n_v_heads=2, d_k=128, d_v=128,
                        tree="random", seed=701, qkv_dtype="bf16")
    _check(prob, sd)


def test_one_node_above_the_maximum_is_refused():
    N = gdn.GDN_MAX_TREE_NODES + 1
    prob = make_problem(batch=1, n_nodes=N, n_k_heads=1, n_v_heads=1, d_k=128, d_v=128, tree="random",
                        seed=702, qkv_dtype="bf16", accept="root")
    d = {k: getattr(prob, k).cuda() for k in ("q", "k", "v", "g", "beta", "parent", "state_in")}
    desc = gdn.make_desc(batch=1, n_nodes=N, n_k_heads=1, n_v_heads=1, d_k=128, d_v=128, scale=prob.scale)
    out = torch.full((1, N, 1, 128), float("nan"), device="cuda")
    ns = torch.full((1, N, 1, 128, 128), float("nan"), device="cuda")
    rc = gdn.gdn_tree_verify(desc, d["q"], d["k"], d["v"], d["g"], d["beta"], d["parent"], d["state_in"], out, ns,
                             check=False)
    torch.cuda.synchronize()
    assert rc == gdn.GDN_ERR_UNSUPPORTED
    assert torch.isnan(out).all() and torch.isnan(ns).all()


@pytest.mark.parametrize("sd", ["f32", "f16"])
def test_deep_caterpillar(sd):
    # a spine 511 nodes deep with one leaf off every spine node: 1023 nodes
    par, cur = [-1], 0
    for _ in range(511):
        par += [cur, cur]
        cur = len(par) - 1
    par = np.asarray(par, np.int32)
    prob = make_problem(batch=1, n_nodes=par.shape[0], n_k_heads=1, n_v_heads=3, d_k=128, d_v=128,
                        tree="given", parents=par[None], seed=811, qkv_dtype="bf16")
    _check(prob, sd)


@pytest.mark.parametrize("chunked", [False, True])
def test_longest_chain_last_state(chunked):
    """A chain of 65535 tokens, the most a desc allows, last state only, by
    the token-by-token walk and by the chunked tensor-core form: every
    output and the last state of 8 rows at each end of d_v against the
    oracle (rows of S evolve independently given k)."""
    N = 0xFFFF
    prob = make_problem(batch=1, n_nodes=N, n_k_heads=1, n_v_heads=1, d_k=128, d_v=128, tree="chain",
                        seed=703, qkv_dtype="bf16", gate="uniform_a", accept="root")
    prob.accept_path = torch.arange(N, dtype=torch.int32)[None].contiguous()
    prob.accept_len = torch.full((1,), N, dtype=torch.int32)
    flags = gdn.GDN_FLAG_CHAIN | gdn.GDN_FLAG_PERSIST_LAST | (gdn.GDN_FLAG_CHUNKED if chunked else 0)
    res = run(prob, "f32", flags=flags)
    assert res["status"] == 0
    for rows in (slice(0, 8), slice(120, 128)):
        out, _, ex = oracle.verify(prob.q, prob.k, prob.v[..., rows], prob.g, prob.beta, prob.parent,
                                   prob.state_in[:, :, rows], prob.scale, want_exact=True)
        assert_out_close(res["out"][..., rows], out)
        assert_states_close(res["node_states"][:, 0, :, rows], ex[:, -1], "f32")
        del out, ex
