"""gdn_tree_plan + gdn_tree_verify_planned: bit-identical to gdn_tree_verify
(which the parity tests hold to the oracle) for every walk kind that builds
a walk, with malformed trees and mismatched plans reported."""
import pytest
import torch

import gated_deltanet_tree_verify_b200 as gdn
from gdn_inputs import make_problem

pytestmark = pytest.mark.gpu


def _setup(B, N, sd, seed, tree="ddtree", Hk=4, Hv=12):
    prob = make_problem(batch=B, n_nodes=N, n_k_heads=Hk, n_v_heads=Hv, d_k=128, d_v=128, tree=tree, seed=seed,
                        qkv_dtype="bf16", accept="root")
    dev = torch.device("cuda")
    d = {k: getattr(prob, k).to(dev) for k in ("q", "k", "v", "g", "beta", "parent", "state_in")}
    tdt = torch.float16 if sd == "f16" else torch.float32
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    desc = gdn.make_desc(batch=B, n_nodes=N, n_k_heads=Hk, n_v_heads=Hv, d_k=128, d_v=128, scale=prob.scale,
                         qkv_dtype=gdn.GDN_BF16, state_dtype=gdn.GDN_F16 if sd == "f16" else gdn.GDN_F32,
                         status=status)
    return prob, d, tdt, desc, status


def _outputs(B, N, Hv, tdt, fill=float("nan")):
    dev = torch.device("cuda")
    return (torch.full((B, N, Hv, 128), fill, device=dev),
            torch.full((B, N, Hv, 128, 128), fill, device=dev, dtype=tdt))


@pytest.mark.parametrize("B,N,sd,Hv", [
    (32, 23, "f16", 48),    # large grid, warp-built walk, one stack slot
    (8, 65, "f16", 48),     # large grid, 8-warp CTAs, mask-built walk
    (16, 200, "f16", 48),   # serial walk builder (> 128 nodes)
    (8, 129, "f16", 48),    # ring kernel reading the plan
])
def test_planned_equals_unplanned(B, N, sd, Hv):
    prob, d, tdt, desc, status = _setup(B, N, sd, seed=N + B, Hk=Hv // 3, Hv=Hv)
    need = gdn.gdn_tree_plan_bytes(desc)
    assert need > 0
    plan = torch.empty(need // 4, dtype=torch.int32, device="cuda")
    gdn.gdn_tree_plan(desc, d["parent"], plan)
    o1, s1 = _outputs(B, N, Hv, tdt)
    o2, s2 = _outputs(B, N, Hv, tdt)
    gdn.gdn_tree_verify(desc, d["q"], d["k"], d["v"], d["g"], d["beta"], d["parent"], d["state_in"], o1, s1)
    for _ in range(2):  # a plan serves any number of layers
        gdn.gdn_tree_verify_planned(desc, plan, d["q"], d["k"], d["v"], d["g"], d["beta"], d["parent"],
                                    d["state_in"], o2, s2)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(o1, o2)
    assert torch.equal(s1.view(torch.int16) if tdt == torch.float16 else s1.view(torch.int32),
                       s2.view(torch.int16) if tdt == torch.float16 else s2.view(torch.int32))


@pytest.mark.parametrize("B,N", [(1, 23), (2, 65)])
def test_small_grids_need_no_plan(B, N):
    # one row per lane: the walk is built while the previous layer runs
    prob, d, tdt, desc, status = _setup(B, N, "f16", seed=5)
    assert gdn.gdn_tree_plan_bytes(desc) == 0
    o1, s1 = _outputs(B, N, 12, tdt)
    o2, s2 = _outputs(B, N, 12, tdt)
    gdn.gdn_tree_verify(desc, d["q"], d["k"], d["v"], d["g"], d["beta"], d["parent"], d["state_in"], o1, s1)
    gdn.gdn_tree_verify_planned(desc, None, d["q"], d["k"], d["v"], d["g"], d["beta"], d["parent"],
                                d["state_in"], o2, s2, plan_bytes=0)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1.view(torch.int16), s2.view(torch.int16))


def test_plan_not_needed_for_f32_trees():
    prob, d, tdt, desc, status = _setup(2, 23, "f32", seed=3)
    assert gdn.gdn_tree_plan_bytes(desc) == 0
    o1, s1 = _outputs(2, 23, 12, tdt)
    o2, s2 = _outputs(2, 23, 12, tdt)
    gdn.gdn_tree_verify(desc, d["q"], d["k"], d["v"], d["g"], d["beta"], d["parent"], d["state_in"], o1, s1)
    gdn.gdn_tree_verify_planned(desc, None, d["q"], d["k"], d["v"], d["g"], d["beta"], d["parent"],
                                d["state_in"], o2, s2, plan_bytes=0)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


@pytest.mark.parametrize("N", [23, 65])
def test_plan_of_a_malformed_tree(N):
    prob, d, tdt, desc, status = _setup(8, N, "f16", seed=7, Hk=16, Hv=48)
    par = d["parent"].clone()
    par[1, N - 1] = N - 1                     # sequence 1: a node that is its own parent
    plan = torch.empty(gdn.gdn_tree_plan_bytes(desc) // 4, dtype=torch.int32, device="cuda")
    gdn.gdn_tree_plan(desc, par, plan)
    torch.cuda.synchronize()
    assert int(status.item()) == gdn.GDN_ERR_BAD_TREE
    status.zero_()
    o, s = _outputs(8, N, 48, tdt)
    gdn.gdn_tree_verify_planned(desc, plan, d["q"], d["k"], d["v"], d["g"], d["beta"], par, d["state_in"], o, s)
    o_ref, s_ref = _outputs(8, N, 48, tdt)
    gdn.gdn_tree_verify(desc, d["q"], d["k"], d["v"], d["g"], d["beta"], par, d["state_in"], o_ref, s_ref)
    torch.cuda.synchronize()
    assert int(status.item()) == gdn.GDN_ERR_BAD_TREE
    assert torch.isnan(o[1]).all()            # nothing written for the bad sequence
    for b in (0, 2, 7):
        assert torch.equal(o[b], o_ref[b])


def test_plan_for_another_shape_is_rejected():
    # a plan built for 65-node trees read by a 64-node call: the plan is
    # large enough, its walks are not for these trees -> GDN_ERR_BAD_INPUT
    _, d65, tdt, desc65, _ = _setup(8, 65, "f16", seed=9, Hk=16, Hv=48)
    plan = torch.empty(gdn.gdn_tree_plan_bytes(desc65) // 4, dtype=torch.int32, device="cuda")
    gdn.gdn_tree_plan(desc65, d65["parent"], plan)
    prob, d, tdt, desc64, status = _setup(8, 64, "f16", seed=9, Hk=16, Hv=48)
    assert 0 < gdn.gdn_tree_plan_bytes(desc64) <= plan.numel() * 4
    o, s = _outputs(8, 64, 48, tdt)
    gdn.gdn_tree_verify_planned(desc64, plan, d["q"], d["k"], d["v"], d["g"], d["beta"], d["parent"],
                                d["state_in"], o, s)
    torch.cuda.synchronize()
    assert int(status.item()) == gdn.GDN_ERR_BAD_INPUT
    assert torch.isnan(o).all()
