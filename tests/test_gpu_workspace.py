"""gdn_tree_verify_ws: the walk's branch states in a global-memory workspace
instead of shared memory.  Results must be bit-identical to gdn_tree_verify
(same walk, same arithmetic) and hence within the oracle tolerances."""
import numpy as np
import pytest
import torch

import gated_deltanet_tree_verify_b200 as gdn
import oracle
from gdn_inputs import make_problem, make_workload
from tests.gpu_util import assert_out_close, assert_states_close, run

pytestmark = pytest.mark.gpu


def _same(a, b):
    for key in ("out", "node_states", "state_out"):
        assert torch.equal(a[key], b[key]), key
    assert a["status"] == b["status"] == 0


def _tree(par, B=2, dk=128, dv=128, Hk=2, Hv=6, seed=31):
    par = np.asarray(par, np.int32)
    return make_problem(batch=B, n_nodes=par.shape[-1], n_k_heads=Hk, n_v_heads=Hv, d_k=dk, d_v=dv,
                        tree="given", parents=np.stack([par] * B), seed=seed, qkv_dtype="bf16")


@pytest.mark.parametrize("budget,batch", [(22, 2), (32, 2), (64, 2), (128, 1)])
def test_ddtree_workspace_bitwise_and_parity(budget, batch):
    prob = make_problem(batch=batch, n_nodes=budget + 1, n_k_heads=16, n_v_heads=48, d_k=128, d_v=128,
                        tree="ddtree", seed=300 + budget, qkv_dtype="bf16")
    ref = run(prob, "f16")
    ws = run(prob, "f16", workspace=True)
    _same(ref, ws)
    for b, h in [(0, 0), (batch - 1, 47)]:
        out, _, ex = oracle.verify_pair(prob, b, h, state_dtype="f16", want_exact=True)
        assert_out_close(ws["out"][b:b + 1, :, h:h + 1], out)
        assert_states_close(ws["node_states"][b:b + 1, :, h:h + 1], ex, "f16")


@pytest.mark.parametrize("N", [63, 127, 255])
def test_complete_binary_needs_more_slots_than_the_workspace_keeps(N):
    # floor(log2 N) >= 5 branch levels: beyond the 4 workspace slots, so the
    # exact recompute path runs too.
    par = np.array([-1] + [(i - 1) // 2 for i in range(1, N)], np.int32)
    prob = _tree(par, B=1)
    ref, ws = run(prob, "f16"), run(prob, "f16", workspace=True)
    _same(ref, ws)
    out, _, ex = oracle.verify(prob.q, prob.k, prob.v, prob.g, prob.beta, prob.parent, prob.state_in,
                               prob.scale, state_dtype="f16", want_exact=True)
    assert_out_close(ws["out"], out)
    assert_states_close(ws["node_states"], ex, "f16")


@pytest.mark.parametrize("shape", ["caterpillar", "star", "random"])
def test_tree_shapes_workspace_bitwise(shape):
    if shape == "caterpillar":
        par, cur = [-1], 0
        for _ in range(20):
            par += [cur, cur]
            cur = len(par) - 1
    elif shape == "star":
        par = [-1] + [0] * 40
    else:
        rng = np.random.default_rng(5)
        par = [-1] + [int(rng.integers(i)) for i in range(1, 90)]
    prob = _tree(par)
    _same(run(prob, "f16"), run(prob, "f16", workspace=True))


def test_persist_last_f32_tree_uses_the_workspace():
    # f32 persistence of the last node only keeps branch states (no node_states
    # to re-read them from)
    prob = make_problem(batch=2, n_nodes=40, n_k_heads=2, n_v_heads=6, d_k=128, d_v=128, tree="random",
                        seed=41, qkv_dtype="bf16", accept="root")
    flags = gdn.GDN_FLAG_PERSIST_LAST
    desc = gdn.make_desc(batch=2, n_nodes=40, n_k_heads=2, n_v_heads=6, d_k=128, d_v=128, scale=prob.scale,
                         state_dtype=gdn.GDN_F32, flags=flags)
    assert gdn.gdn_tree_verify_workspace_bytes(desc) > 0
    ref = run(prob, "f32", flags=flags, commit=False)
    ws = run(prob, "f32", flags=flags, commit=False, workspace=True)
    for key in ("out", "node_states"):
        assert torch.equal(ref[key], ws[key]), key


def test_workspace_too_small_is_rejected_before_launch():
    prob = make_workload("ddtree_budget22", seed=2)
    d = {k: getattr(prob, k).cuda() for k in ("q", "k", "v", "g", "beta", "parent", "state_in")}
    desc = gdn.make_desc(batch=1, n_nodes=23, n_k_heads=16, n_v_heads=48, d_k=128, d_v=128, scale=prob.scale,
                         state_dtype=gdn.GDN_F16)
    need = gdn.gdn_tree_verify_workspace_bytes(desc)
    out = torch.full((1, 23, 48, 128), float("nan"), device="cuda")
    ns = torch.full((1, 23, 48, 128, 128), float("nan"), device="cuda", dtype=torch.float16)
    ws = torch.empty(need // 4, device="cuda")
    rc = gdn.gdn_tree_verify_ws(desc, d["q"], d["k"], d["v"], d["g"], d["beta"], d["parent"], d["state_in"],
                                out, ns, ws, need - 4, check=False)
    assert rc == gdn.GDN_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.isnan(out).all()
