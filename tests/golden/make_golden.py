"""Write tests/golden/tiny_tree8_d32.txt from the oracle alone.

Workload: 1 sequence, 8-node tree (parent[i] uniform over earlier nodes, seed
0), 4 v-heads over 2 k-heads, d_k = d_v = 32, f32 inputs, accept path = root to
a random leaf.  Stored: the tree, the accept path, every output o (f64), each
node-head state's Frobenius norm, and the committed state's row sums for f32
and f16 persistence.  Run:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from gdn_inputs import make_workload  # noqa: E402


def compute():
    prob = make_workload("tiny_tree8_d32", seed=0)
    res = {"parent": prob.parent[0].numpy().astype(np.int64),
           "accept_path": prob.accept_path[0, :int(prob.accept_len[0])].numpy().astype(np.int64)}
    for sd in ("f32", "f16"):
        out, st, ex = oracle.verify_problem(prob, state_dtype=sd, want_exact=True)
        so = oracle.commit(st, prob.parent, prob.accept_path, prob.accept_len)
        if sd == "f32":
            res["out"] = out.reshape(-1)
            res["state_fro"] = np.sqrt((ex ** 2).sum(axis=(3, 4))).reshape(-1)
        res[f"state_out_rowsum_{sd}"] = so.sum(axis=3).reshape(-1)
    return res


def main():
    res = compute()
    path = os.path.join(HERE, "tiny_tree8_d32.txt")
    with open(path, "w") as f:
        f.write("# written by tests/golden/make_golden.py from the oracle only\n")
        for key, arr in res.items():
            f.write(f"{key} {' '.join(repr(x.item()) for x in arr)}\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
