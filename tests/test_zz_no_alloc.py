"""gdn_tree_verify_static_ws: the workspace path on the library's static
device buffer (no allocation per call).  It must give exactly the results of
gdn_tree_verify, call after call, and run descs that need more workspace
than the buffer holds as gdn_tree_verify does.  Kept in the last-collected file: the buffer is
process-wide state."""
import pytest
import torch

import gated_deltanet_tree_verify_b200 as gdn
from gdn_inputs import make_problem

pytestmark = pytest.mark.gpu


def _buffers(prob, sd):
    B, N, Hk, dk = prob.q.shape
    Hv, dv = prob.v.shape[2], prob.v.shape[3]
    tdt = torch.float32 if sd == gdn.GDN_F32 else torch.float16
    out = torch.full((B, N, Hv, dv), float("nan"), device="cuda")
    ns = torch.full((B, N, Hv, dv, dk), float("nan"), device="cuda", dtype=tdt)
    desc = gdn.make_desc(batch=B, n_nodes=N, n_k_heads=Hk, n_v_heads=Hv, d_k=dk, d_v=dv, scale=prob.scale,
                         qkv_dtype=gdn.GDN_BF16, state_dtype=sd)
    return desc, out, ns


def _call(fn, prob, sd):
    d = {k: getattr(prob, k).cuda() for k in ("q", "k", "v", "g", "beta", "parent", "state_in")}
    desc, out, ns = _buffers(prob, sd)
    rc = fn(desc, d["q"], d["k"], d["v"], d["g"], d["beta"], d["parent"], d["state_in"], out, ns, check=False)
    torch.cuda.synchronize()
    return rc, out.cpu(), ns.cpu()


@pytest.mark.parametrize("budget", [22, 64, 128])
def test_static_workspace_matches_verify_over_two_calls(budget):
    # f16 trees at batch 1 keep their branch states in a workspace of
    # 48 heads x 128 x 128 x 4 B x 4 slots = 12 MiB: every case here runs on
    # the static buffer, not the fall-through to gdn_tree_verify.
    sd = gdn.GDN_F16
    probs = [make_problem(batch=1, n_nodes=budget + 1, n_k_heads=16, n_v_heads=48, d_k=128, d_v=128,
                          tree="ddtree", seed=700 + 10 * budget + i, qkv_dtype="bf16") for i in range(2)]
    desc, _, _ = _buffers(probs[0], sd)
    assert 0 < gdn.gdn_tree_verify_workspace_bytes(desc) <= gdn.gdn_static_workspace_capacity()
    for prob in probs:  # the second call reuses the buffer the first one left behind
        rc0, out0, ns0 = _call(gdn.gdn_tree_verify, prob, sd)
        rc1, out1, ns1 = _call(gdn.gdn_tree_verify_static_ws, prob, sd)
        assert rc0 == rc1 == gdn.GDN_OK
        assert torch.equal(out0, out1)
        assert torch.equal(ns0, ns1)


def test_static_workspace_f32_needs_no_buffer():
    # An f32 tree at batch 1 re-reads branch states from node_states, so the
    # desc needs no workspace and the call is gdn_tree_verify itself (f32
    # walks that do keep branch states run on grids whose workspace exceeds
    # the static buffer).
    prob = make_problem(batch=1, n_nodes=23, n_k_heads=16, n_v_heads=48, d_k=128, d_v=128, tree="ddtree",
                        seed=731, qkv_dtype="bf16")
    desc, _, _ = _buffers(prob, gdn.GDN_F32)
    assert gdn.gdn_tree_verify_workspace_bytes(desc) == 0
    rc0, out0, ns0 = _call(gdn.gdn_tree_verify, prob, gdn.GDN_F32)
    rc1, out1, ns1 = _call(gdn.gdn_tree_verify_static_ws, prob, gdn.GDN_F32)
    assert rc0 == rc1 == gdn.GDN_OK
    assert torch.equal(out0, out1) and torch.equal(ns0, ns1)


def test_static_workspace_oversize_runs_without_it():
    """A desc whose walk would need more than the buffer: the call runs it as
    gdn_tree_verify does (shared-memory slots), with the same results."""
    prob = make_problem(batch=8, n_nodes=23, n_k_heads=16, n_v_heads=48, d_k=128, d_v=128, tree="ddtree",
                        seed=9, qkv_dtype="bf16")
    desc, _, _ = _buffers(prob, gdn.GDN_F16)
    assert gdn.gdn_tree_verify_workspace_bytes(desc) > gdn.gdn_static_workspace_capacity()
    rc0, out0, ns0 = _call(gdn.gdn_tree_verify, prob, gdn.GDN_F16)
    rc1, out1, ns1 = _call(gdn.gdn_tree_verify_static_ws, prob, gdn.GDN_F16)
    assert rc0 == rc1 == gdn.GDN_OK
    assert torch.equal(out0, out1) and torch.equal(ns0, ns1)
