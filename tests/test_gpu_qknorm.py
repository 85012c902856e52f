"""GDN_FLAG_QK_L2NORM: q and k given raw, L2-normalised per (node, k-head)
inside the kernels (folded into per-node scalars).  The oracle normalises the
same raw bf16 values in double first (oracle.verify(qk_l2norm=True))."""
import numpy as np
import pytest
import torch

import gated_deltanet_tree_verify_b200 as gdn
import oracle
from gdn_inputs import make_problem
from tests.gpu_util import assert_out_close, assert_states_close, run

pytestmark = pytest.mark.gpu

NORM = gdn.GDN_FLAG_QK_L2NORM


def _raw(prob, seed=0):
    """Scale every (node, head) row of q and k by a factor in [0.25, 4] and
    round to the input dtype: raw, non-unit rows."""
    g = torch.Generator().manual_seed(seed)
    for key in ("q", "k"):
        x = getattr(prob, key)
        f = torch.empty(x.shape[:3] + (1,)).uniform_(0.25, 4.0, generator=g)
        setattr(prob, key, (x.float() * f).to(x.dtype).contiguous())
    return prob


def _check(prob, sd, flags=0, pairs=None, workspace=False):
    res = run(prob, sd, flags=flags | NORM, workspace=workspace)
    assert res["status"] == 0
    if pairs is None:
        out, st, ex = oracle.verify_problem(prob, state_dtype=sd, want_exact=True, nthreads=8, qk_l2norm=True)
        assert_out_close(res["out"], out)
        if flags & gdn.GDN_FLAG_PERSIST_LAST:
            assert_states_close(res["node_states"][:, 0], ex[:, -1], sd)
        else:
            assert_states_close(res["node_states"], ex, sd)
        return res
    G = prob.n_v_heads // prob.n_k_heads
    for b, h in pairs:
        hk = h // G
        out, _, ex = oracle.verify(prob.q[b:b + 1, :, hk:hk + 1], prob.k[b:b + 1, :, hk:hk + 1],
                                   prob.v[b:b + 1, :, h:h + 1], prob.g[b:b + 1, :, h:h + 1],
                                   prob.beta[b:b + 1, :, h:h + 1], prob.parent[b:b + 1],
                                   prob.state_in[b:b + 1, h:h + 1], prob.scale, state_dtype=sd,
                                   want_exact=True, qk_l2norm=True)
        assert_out_close(res["out"][b:b + 1, :, h:h + 1], out)
        assert_states_close(res["node_states"][b:b + 1, :, h:h + 1], ex, sd)
    return res


@pytest.mark.parametrize("sd", ["f32", "f16"])
def test_qknorm_ddtree_budget22(sd):
    prob = _raw(make_problem(batch=2, n_nodes=23, n_k_heads=16, n_v_heads=48, d_k=128, d_v=128, tree="ddtree",
                             seed=61, qkv_dtype="bf16"))
    _check(prob, sd, pairs=[(0, 0), (1, 47), (1, 20)])


@pytest.mark.parametrize("sd", ["f32", "f16"])
def test_qknorm_chain_and_small_heads(sd):
    prob = _raw(make_problem(batch=2, n_nodes=16, n_k_heads=2, n_v_heads=6, d_k=64, d_v=64, tree="chain",
                             seed=62, qkv_dtype="bf16"))
    _check(prob, sd, flags=gdn.GDN_FLAG_CHAIN)
    _check(prob, sd)


def test_qknorm_recompute_and_ring_paths():
    # complete binary trees force recomputation (f16 stack slots exceeded);
    # 129 nodes of budget 128 go through the ring kernel
    par = np.array([-1] + [(i - 1) // 2 for i in range(1, 127)], np.int32)
    prob = _raw(make_problem(batch=1, n_nodes=127, n_k_heads=1, n_v_heads=3, d_k=128, d_v=128, tree="given",
                             parents=par[None], seed=63, qkv_dtype="bf16"))
    _check(prob, "f16")
    _check(prob, "f16", workspace=True)
    big = _raw(make_problem(batch=1, n_nodes=129, n_k_heads=16, n_v_heads=48, d_k=128, d_v=128, tree="ddtree",
                            seed=64, qkv_dtype="bf16"))
    _check(big, "f16", pairs=[(0, 0), (0, 31)])
    _check(big, "f32", pairs=[(0, 5)])


def test_qknorm_without_flag_changes_results():
    prob = _raw(make_problem(batch=1, n_nodes=8, n_k_heads=1, n_v_heads=2, d_k=32, d_v=32, tree="random",
                             seed=65, qkv_dtype="bf16"))
    a = run(prob, "f32", flags=NORM)
    b = run(prob, "f32")
    assert (a["out"] - b["out"]).abs().max() > 1e-3
