"""gdn_tree_compact against the oracle (oracle.compact): every written byte
equal, unwritten rows untouched, bad paths and bad offsets reported."""
import numpy as np
import pytest
import torch

import gated_deltanet_tree_verify_b200 as gdn
import oracle
from gdn_inputs import make_problem, tree_leaves

pytestmark = pytest.mark.gpu


def _trees(B, N, seed, tree="ddtree"):
    prob = make_problem(batch=B, n_nodes=N, n_k_heads=1, n_v_heads=1, d_k=32, d_v=32, tree=tree, seed=seed,
                        qkv_dtype="f32", accept="leaf")
    return prob.parent.numpy().astype(np.int32), prob.accept_path.numpy(), prob.accept_len.numpy()


def _run(rows, parent, path, length, B, N, cu=None, total=0, fill=0x5A):
    dev = torch.device("cuda")
    src = torch.from_numpy(rows).to(dev)
    P = path.shape[1]
    dst = torch.full((B, P) + rows.shape[1:], 0, dtype=src.dtype, device=dev)
    dst.view(torch.uint8).fill_(fill)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    gdn.gdn_tree_compact(src, torch.from_numpy(parent).to(dev), torch.from_numpy(path).to(dev),
                         torch.from_numpy(length).to(dev), dst, batch=B, n_nodes=N,
                         cu_nodes=torch.from_numpy(cu).to(dev) if cu is not None else None, total_nodes=total,
                         status=status)
    torch.cuda.synchronize()
    return dst.cpu().numpy(), int(status.item())


def _check(got, want, written, fill=0x5A):
    B, P = written.shape
    for b in range(B):
        for i in range(P):
            if written[b, i]:
                assert got[b, i].tobytes() == want[b, i].tobytes(), (b, i)
            else:
                assert set(got[b, i].view(np.uint8).ravel().tolist()) == {fill}, (b, i)


@pytest.mark.parametrize("B,N,row", [(1, 23, 48 * 128), (8, 65, 48 * 128), (3, 16, 4), (5, 129, 1000)])
def test_compact_matches_oracle(B, N, row):
    parent, path, length = _trees(B, N, seed=B * 10 + N)
    rng = np.random.default_rng(N)
    rows = rng.standard_normal((B * N, row)).astype(np.float32)
    got, st = _run(rows, parent.reshape(-1), path, length, B, N)
    want, written = oracle.compact(rows, parent.reshape(-1), path, length)
    assert st == 0
    _check(got, want, written)


def test_compact_rows_larger_than_a_piece():
    # node states as rows (64 KB pieces: several CTAs per row)
    B, N = 2, 8
    parent, path, length = _trees(B, N, seed=3, tree="random")
    rows = np.random.default_rng(1).integers(0, 2**31, size=(B * N, 48 * 1024), dtype=np.int32)
    got, st = _run(rows, parent.reshape(-1), path, length, B, N)
    want, written = oracle.compact(rows, parent.reshape(-1), path, length)
    assert st == 0
    _check(got, want, written)


def test_compact_varlen():
    sizes = [23, 9, 65, 1, 33]
    parents, paths, lens = [], [], []
    for i, n in enumerate(sizes):
        p, a, l_ = _trees(1, n, seed=40 + i)
        parents.append(p[0])
        paths.append(a[0])
        lens.append(l_[0])
    P = max(len(a) for a in paths)
    path = np.zeros((len(sizes), P), np.int32)
    for i, a in enumerate(paths):
        path[i, :len(a)] = a
    parent = np.concatenate(parents).astype(np.int32)
    cu = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    rows = np.random.default_rng(2).standard_normal((cu[-1], 24)).astype(np.float32)
    length = np.array(lens, np.int32)
    got, st = _run(rows, parent, path, length, len(sizes), max(sizes), cu=cu, total=int(cu[-1]))
    want, written = oracle.compact(rows, parent, path, length, cu_nodes=cu)
    assert st == 0
    _check(got, want, written)


def test_compact_bad_paths_and_offsets():
    B, N = 4, 12
    parent, path, length = _trees(B, N, seed=5)
    path = path.copy()
    length = length.copy()
    path[1, 0] = 1                      # not from the root
    length[2] = path.shape[1] + 1       # longer than max_path_len
    rows = np.random.default_rng(3).standard_normal((B * N, 8)).astype(np.float32)
    got, st = _run(rows, parent.reshape(-1), path, length, B, N)
    want, written = oracle.compact(rows, parent.reshape(-1), path, length)
    assert st == gdn.GDN_ERR_BAD_PATH
    assert not written[1].any() and not written[2].any() and written[0].any() and written[3].any()
    _check(got, want, written)
    # varlen: a sequence whose offsets run past the packed total
    cu = np.array([0, 12, 24, 36, 48], np.int32)
    cu_bad = cu.copy()
    cu_bad[3] = 47                      # sequence 3 has one node, sequence 2 thirteen (> n_nodes)
    p2, a2, l2 = _trees(B, N, seed=6)
    got, st = _run(rows, p2.reshape(-1), a2, l2, B, N, cu=cu_bad, total=48)
    assert st in (gdn.GDN_ERR_BAD_TREE, gdn.GDN_ERR_BAD_PATH)
    want, written = oracle.compact(rows, p2.reshape(-1), a2, l2, cu_nodes=cu)
    # sequences 0 and 1 are unaffected by the bad offsets
    for b in (0, 1):
        for i in range(a2.shape[1]):
            if written[b, i]:
                assert got[b, i].tobytes() == want[b, i].tobytes()
    assert set(got[2].view(np.uint8).ravel().tolist()) == {0x5A}


def test_compact_outputs_of_a_verify():
    # the accepted path's outputs, in path order, equal gathering verify's
    # outputs by hand
    prob = make_problem(batch=3, n_nodes=23, n_k_heads=2, n_v_heads=6, d_k=128, d_v=128, tree="ddtree", seed=8,
                        qkv_dtype="bf16", accept="leaf")
    dev = torch.device("cuda")
    d = {k: getattr(prob, k).to(dev) for k in ("q", "k", "v", "g", "beta", "parent", "state_in",
                                                "accept_path", "accept_len")}
    out = torch.empty(3, 23, 6, 128, device=dev)
    ns = torch.empty(3, 23, 6, 128, 128, device=dev)
    desc = gdn.make_desc(batch=3, n_nodes=23, n_k_heads=2, n_v_heads=6, d_k=128, d_v=128, scale=prob.scale)
    gdn.gdn_tree_verify(desc, d["q"], d["k"], d["v"], d["g"], d["beta"], d["parent"], d["state_in"], out, ns)
    P = d["accept_path"].shape[1]
    dst = torch.zeros(3, P, 6, 128, device=dev)
    gdn.gdn_tree_compact(out, d["parent"], d["accept_path"], d["accept_len"], dst, batch=3, n_nodes=23)
    torch.cuda.synchronize()
    for b in range(3):
        for i in range(int(prob.accept_len[b])):
            assert torch.equal(dst[b, i], out[b, int(prob.accept_path[b, i])])
    assert all(int(prob.accept_path[b, int(prob.accept_len[b]) - 1]) in tree_leaves(prob.parent[b].numpy())
               for b in range(3))
