"""gdn_tree_verify_varlen / gdn_tree_commit_varlen: trees of different sizes
packed along the node dimension.  Each sequence's results must be
bit-identical to gdn_tree_verify / gdn_tree_commit on that sequence alone
(which the parity tests hold to the oracle), and bad offsets must be
reported without touching other sequences."""
import numpy as np
import pytest
import torch

import gated_deltanet_tree_verify_b200 as gdn
import oracle
from gdn_inputs import make_problem
from tests.gpu_util import assert_out_close, assert_states_close, run

pytestmark = pytest.mark.gpu

SD = {"f32": (gdn.GDN_F32, torch.float32), "f16": (gdn.GDN_F16, torch.float16)}


def _seqs(sizes, trees, Hk=4, Hv=12, d=128, seed=50):
    return [make_problem(batch=1, n_nodes=n, n_k_heads=Hk, n_v_heads=Hv, d_k=d, d_v=d, tree=t, seed=seed + i,
                         qkv_dtype="bf16", accept="leaf") for i, (n, t) in enumerate(zip(sizes, trees))]


def _pack(seqs):
    cat = lambda key: torch.cat([getattr(s, key)[0] for s in seqs]).contiguous()  # noqa: E731
    sizes = [s.n_nodes for s in seqs]
    cu = torch.tensor([0] + list(np.cumsum(sizes)), dtype=torch.int32)
    P = max(s.accept_path.shape[1] for s in seqs)
    path = torch.full((len(seqs), P), -1, dtype=torch.int32)
    for i, s in enumerate(seqs):
        path[i, :s.accept_path.shape[1]] = s.accept_path[0]
    return dict(q=cat("q"), k=cat("k"), v=cat("v"), g=cat("g"), beta=cat("beta"), parent=cat("parent"),
                state_in=torch.cat([s.state_in for s in seqs]).contiguous(), cu=cu, accept_path=path,
                accept_len=torch.cat([s.accept_len for s in seqs]).contiguous(), sizes=sizes)


def _run_varlen(seqs, sd, flags=0, workspace=False, cu=None, commit=True):
    pk = _pack(seqs)
    if cu is not None:
        pk["cu"] = cu
    s0 = seqs[0]
    B, T, Nmax = len(seqs), int(sum(pk["sizes"])), max(pk["sizes"])
    Hk, dk = s0.q.shape[2], s0.q.shape[3]
    Hv, dv = s0.v.shape[2], s0.v.shape[3]
    code, tdt = SD[sd]
    dev = {k: v.cuda() for k, v in pk.items() if isinstance(v, torch.Tensor)}
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    desc = gdn.make_desc(batch=B, n_nodes=Nmax, n_k_heads=Hk, n_v_heads=Hv, d_k=dk, d_v=dv, scale=s0.scale,
                         qkv_dtype=gdn.GDN_BF16, state_dtype=code, flags=flags, status=status)
    NS = B if flags & gdn.GDN_FLAG_PERSIST_LAST else T
    out = torch.full((T, Hv, dv), float("nan"), device="cuda")
    ns = torch.full((NS, Hv, dv, dk), float("nan"), device="cuda", dtype=tdt)
    so = torch.full((B, Hv, dv, dk), float("nan"), device="cuda")
    ws = None
    if workspace:
        nb = gdn.gdn_tree_verify_workspace_bytes(desc)
        ws = torch.full((max(nb, 16) // 4,), float("nan"), device="cuda")
    par = None if flags & gdn.GDN_FLAG_CHAIN else dev["parent"]
    gdn.gdn_tree_verify_varlen(desc, dev["cu"], T, dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], par,
                               dev["state_in"], out, ns, ws)
    if commit:
        gdn.gdn_tree_commit_varlen(desc, dev["cu"], T, [ns], par, dev["accept_path"], dev["accept_len"],
                                   dev["accept_path"].shape[1], [so])
    torch.cuda.synchronize()
    return dict(out=out.cpu(), node_states=ns.cpu(), state_out=so.cpu(), status=int(status.item()),
                cu=pk["cu"], sizes=pk["sizes"])


@pytest.mark.parametrize("sd", ["f32", "f16"])
@pytest.mark.parametrize("workspace", [False, True])
def test_varlen_equals_each_sequence_alone(sd, workspace):
    sizes = [1, 7, 23, 40, 12, 33]
    trees = ["chain", "random", "ddtree", "ddtree", "chain", "random"]
    seqs = _seqs(sizes, trees)
    vr = _run_varlen(seqs, sd, workspace=workspace)
    assert vr["status"] == 0
    for i, s in enumerate(seqs):
        a, b = int(vr["cu"][i]), int(vr["cu"][i + 1])
        ref = run(s, sd)
        assert torch.equal(vr["out"][a:b], ref["out"][0]), i
        assert torch.equal(vr["node_states"][a:b], ref["node_states"][0]), i
        assert torch.equal(vr["state_out"][i], ref["state_out"][0]), i
    # and one sequence against the oracle directly
    s = seqs[2]
    out, _, ex = oracle.verify_problem(s, state_dtype=sd, want_exact=True, nthreads=8)
    a, b = int(vr["cu"][2]), int(vr["cu"][3])
    assert_out_close(vr["out"][a:b][None], out)
    assert_states_close(vr["node_states"][a:b][None], ex, sd)


@pytest.mark.parametrize("sd", ["f32", "f16"])
def test_varlen_48_heads_equals_each_sequence_alone(sd):
    # Eight packed trees on 48 v-heads: the grid of the batched workloads,
    # where f16 trees above 32 nodes take the wide kernel (stack slots in
    # tensor memory).  Bit-identical to each sequence alone (a small grid,
    # another lane shape), and sampled (sequence, head) pairs against the oracle.
    sizes = [9, 65, 23, 16, 33, 23, 49, 9]
    seqs = _seqs(sizes, ["ddtree"] * 8, Hk=16, Hv=48, seed=70)
    vr = _run_varlen(seqs, sd)
    assert vr["status"] == 0
    for i, s in enumerate(seqs):
        a, b = int(vr["cu"][i]), int(vr["cu"][i + 1])
        ref = run(s, sd)
        assert torch.equal(vr["out"][a:b], ref["out"][0]), i
        assert torch.equal(vr["node_states"][a:b], ref["node_states"][0]), i
        assert torch.equal(vr["state_out"][i], ref["state_out"][0]), i
    for i, h in [(1, 0), (6, 47), (4, 20)]:
        a, b = int(vr["cu"][i]), int(vr["cu"][i + 1])
        out, _, ex = oracle.verify_pair(seqs[i], 0, h, state_dtype=sd, want_exact=True)
        assert_out_close(vr["out"][a:b, h:h + 1][None], out)
        assert_states_close(vr["node_states"][a:b, h:h + 1][None], ex, sd)


def test_varlen_chains_with_persist_last():
    sizes = [5, 64, 17]
    seqs = _seqs(sizes, ["chain"] * 3)
    for s in seqs:
        s.accept_path = torch.arange(s.n_nodes, dtype=torch.int32)[None]
        s.accept_len = torch.tensor([s.n_nodes], dtype=torch.int32)
    flags = gdn.GDN_FLAG_CHAIN | gdn.GDN_FLAG_PERSIST_LAST
    vr = _run_varlen(seqs, "f32", flags=flags)
    assert vr["status"] == 0
    for i, s in enumerate(seqs):
        a, b = int(vr["cu"][i]), int(vr["cu"][i + 1])
        ref = run(s, "f32", flags=flags)
        assert torch.equal(vr["out"][a:b], ref["out"][0]), i
        assert torch.equal(vr["node_states"][i], ref["node_states"][0, 0]), i
        assert torch.equal(vr["state_out"][i], ref["state_out"][0]), i


@pytest.mark.parametrize("bad", ["decreasing", "too_long", "past_total"])
def test_bad_offsets_report_and_spare_other_sequences(bad):
    sizes = [9, 9, 5] if bad == "past_total" else [9, 9, 9]
    seqs = _seqs(sizes, ["random"] * 3, Hk=2, Hv=4)
    if bad == "decreasing":
        cu = torch.tensor([0, 9, 5, 27], dtype=torch.int32)     # sequence 1 has -4 nodes
    elif bad == "too_long":
        cu = torch.tensor([0, 9, 27, 27], dtype=torch.int32)    # 18 > N_max = 9, then an empty one
    else:
        cu = torch.tensor([0, 9, 18, 27], dtype=torch.int32)    # sequence 2 runs past the 23 nodes
    vr = _run_varlen(seqs, "f32", cu=cu)
    assert vr["status"] == gdn.GDN_ERR_BAD_TREE
    ref = run(seqs[0], "f32")
    assert torch.equal(vr["out"][0:9], ref["out"][0])
    assert torch.equal(vr["state_out"][0], ref["state_out"][0])
    last = {"decreasing": 1, "too_long": 1, "past_total": 2}[bad]
    assert torch.isnan(vr["state_out"][last]).all()
