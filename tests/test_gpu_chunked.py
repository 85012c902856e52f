"""GDN_FLAG_CHUNKED: chains in chunks of 64 tokens on the tensor cores.  The
oracle (token by token, f64) fixes the answer; the chunked form must match it
within the stated tolerances, for chain lengths around the chunk size, both
state dtypes and gates that reset the state.  It is not bit-identical to the
token-by-token path (different summation order), only close to it."""
import numpy as np
import pytest
import torch

import gated_deltanet_tree_verify_b200 as gdn
import oracle
from gdn_inputs import make_problem, make_workload
from tests.gpu_util import assert_out_close, assert_states_close, rel_fro, run

pytestmark = pytest.mark.gpu

FLAGS = gdn.GDN_FLAG_CHAIN | gdn.GDN_FLAG_PERSIST_LAST


def _chain(N, B=2, Hk=2, Hv=6, dv=128, seed=3, gate="softplus"):
    prob = make_problem(batch=B, n_nodes=N, n_k_heads=Hk, n_v_heads=Hv, d_k=128, d_v=dv, tree="chain",
                        seed=seed, qkv_dtype="bf16", gate=gate, accept="prefix")
    prob.accept_path = torch.arange(N, dtype=torch.int32).repeat(B, 1).contiguous()
    prob.accept_len = torch.full((B,), N, dtype=torch.int32)
    return prob


@pytest.mark.parametrize("N", [1, 5, 63, 64, 65, 100, 130, 257])
@pytest.mark.parametrize("sd", ["f32", "f16"])
def test_chunked_chain_matches_oracle(N, sd):
    prob = _chain(N, gate="uniform_a" if N % 2 else "softplus")
    res = run(prob, sd, flags=FLAGS | gdn.GDN_FLAG_CHUNKED)
    assert res["status"] == 0
    out, _, ex = oracle.verify_problem(prob, state_dtype=sd, want_exact=True, nthreads=8)
    assert_out_close(res["out"], out)
    assert_states_close(res["node_states"][:, 0], ex[:, -1], sd)
    assert torch.equal(res["state_out"], res["node_states"][:, 0].float())
    # close to the token-by-token kernel (not bitwise: different summation order)
    ref = run(prob, sd, flags=FLAGS)
    assert (res["out"] - ref["out"]).abs().max() <= 1e-4
    r = rel_fro(res["node_states"][:, 0].double().numpy(), ref["node_states"][:, 0].double().numpy(),
                axes=(-2, -1))
    assert r.max() <= (1e-5 if sd == "f32" else 2e-3)


@pytest.mark.parametrize("sd", ["f32", "f16"])
def test_chunked_partial_row_tile(sd):
    """A CTA holds 128 state rows: d_v = 64 leaves half of its one tile
    empty; rows past d_v are neither read nor written."""
    prob = _chain(100, dv=64, gate="uniform_a")
    res = run(prob, sd, flags=FLAGS | gdn.GDN_FLAG_CHUNKED)
    assert res["status"] == 0
    out, _, ex = oracle.verify_problem(prob, state_dtype=sd, want_exact=True, nthreads=8)
    assert_out_close(res["out"], out)
    assert_states_close(res["node_states"][:, 0], ex[:, -1], sd)


def test_chunked_one_v_head_per_k_head():
    """G = 1: each v-head reads its own k-head (the grid's y index is the
    v-head, the k/q tensor maps take h / G)."""
    prob = _chain(130, B=3, Hk=4, Hv=4, seed=9)
    res = run(prob, "f32", flags=FLAGS | gdn.GDN_FLAG_CHUNKED)
    assert res["status"] == 0
    out, _, ex = oracle.verify_problem(prob, state_dtype="f32", want_exact=True, nthreads=8)
    assert_out_close(res["out"], out)
    assert_states_close(res["node_states"][:, 0], ex[:, -1], "f32")


@pytest.mark.parametrize("sd", ["f32", "f16"])
def test_chunked_raw_gates(sd):
    """GDN_FLAG_GATES: g and beta given as the pre-activations x, y; the
    chunked form applies a = 1 / (1 + e^x), beta = sigmoid(y) per token, x =
    +inf resets, and tokens past the end stay a = 1, beta = 0."""
    prob = make_problem(batch=2, n_nodes=150, n_k_heads=2, n_v_heads=6, d_k=128, d_v=128, tree="chain",
                        seed=21, qkv_dtype="bf16", raw_gates=True, accept="prefix")
    prob.g[:, 77] = float("inf")  # a = 0: the state restarts at token 77
    prob.accept_path = torch.arange(150, dtype=torch.int32).repeat(2, 1).contiguous()
    prob.accept_len = torch.full((2,), 150, dtype=torch.int32)
    res = run(prob, sd, flags=FLAGS | gdn.GDN_FLAG_CHUNKED | gdn.GDN_FLAG_GATES)
    assert res["status"] == 0
    out, _, ex = oracle.verify_problem(prob, state_dtype=sd, want_exact=True, nthreads=8, raw_gates=True)
    assert_out_close(res["out"], out)
    assert_states_close(res["node_states"][:, 0], ex[:, -1], sd)
    ref = run(prob, sd, flags=FLAGS | gdn.GDN_FLAG_GATES)
    assert (res["out"] - ref["out"]).abs().max() <= 1e-4


@pytest.mark.parametrize("sd", ["f32", "f16"])
def test_chunked_fused_normalisation_and_gates(sd):
    """GDN_FLAG_QK_L2NORM (+ GATES): q and k given raw, each token's rows
    normalised inside, folded into per-token scalars (1 / |k_t| into the
    decays and K K^T, 1 / |q_t| into Q K^T and the outputs)."""
    prob = make_problem(batch=2, n_nodes=150, n_k_heads=2, n_v_heads=6, d_k=128, d_v=128, tree="chain",
                        seed=23, qkv_dtype="bf16", raw_gates=True, accept="prefix")
    gen = torch.Generator().manual_seed(24)
    prob.q = (prob.q.float() * (0.5 + 3 * torch.rand(prob.q.shape[:3] + (1,), generator=gen))).to(torch.bfloat16)
    prob.k = (prob.k.float() * (0.5 + 3 * torch.rand(prob.k.shape[:3] + (1,), generator=gen))).to(torch.bfloat16)
    prob.accept_path = torch.arange(150, dtype=torch.int32).repeat(2, 1).contiguous()
    prob.accept_len = torch.full((2,), 150, dtype=torch.int32)
    flags = FLAGS | gdn.GDN_FLAG_QK_L2NORM | gdn.GDN_FLAG_GATES
    res = run(prob, sd, flags=flags | gdn.GDN_FLAG_CHUNKED)
    assert res["status"] == 0
    out, _, ex = oracle.verify_problem(prob, state_dtype=sd, want_exact=True, nthreads=8, qk_l2norm=True,
                                       raw_gates=True)
    assert_out_close(res["out"], out)
    assert_states_close(res["node_states"][:, 0], ex[:, -1], sd)
    ref = run(prob, sd, flags=flags)
    assert (res["out"] - ref["out"]).abs().max() <= 1e-4


def test_chunked_chain_reset_and_zero_beta():
    prob = _chain(150)
    prob.g[:, 70] = float("-inf")   # a = 0: the state restarts at token 70
    prob.beta[:, 10:20] = 0.0       # no writes for 10 tokens
    res = run(prob, "f32", flags=FLAGS | gdn.GDN_FLAG_CHUNKED)
    assert res["status"] == 0
    out, _, ex = oracle.verify_problem(prob, state_dtype="f32", want_exact=True, nthreads=8)
    assert_out_close(res["out"], out)
    assert_states_close(res["node_states"][:, 0], ex[:, -1], "f32")


def test_chunked_long_chain4096_sampled():
    prob = make_workload("long_chain4096", seed=4)
    N = prob.n_nodes
    prob.accept_path = torch.arange(N, dtype=torch.int32).repeat(prob.batch, 1).contiguous()
    prob.accept_len = torch.full((prob.batch,), N, dtype=torch.int32)
    res = run(prob, "f32", flags=FLAGS | gdn.GDN_FLAG_CHUNKED)
    assert res["status"] == 0
    rows = slice(40, 48)  # rows of S evolve independently given k
    for b, h in [(0, 0), (3, 17), (7, 47)]:
        hk = h // 3
        out, st, ex = oracle.verify(prob.q[b:b + 1, :, hk:hk + 1], prob.k[b:b + 1, :, hk:hk + 1],
                                    prob.v[b:b + 1, :, h:h + 1, rows], prob.g[b:b + 1, :, h:h + 1],
                                    prob.beta[b:b + 1, :, h:h + 1], prob.parent[b:b + 1],
                                    prob.state_in[b:b + 1, h:h + 1, rows], prob.scale, want_exact=True)
        assert_out_close(res["out"][b:b + 1, :, h:h + 1, rows], out)
        r = rel_fro(res["node_states"][b, 0, h, rows].double().numpy(), ex[0, -1, 0], axes=(-2, -1))
        assert r <= 1e-3
    assert np.isfinite(res["out"].numpy()).all()
    assert torch.equal(res["state_out"], res["node_states"][:, 0])


def test_chunked_long_chain4096_rows_of_every_tile():
    from tests.test_gpu_parity import CHAIN_PAIRS, CHAIN_ROWS, _chain_rows_parity
    prob = make_workload("long_chain4096", seed=4)
    N = prob.n_nodes
    prob.accept_path = torch.arange(N, dtype=torch.int32).repeat(prob.batch, 1).contiguous()
    prob.accept_len = torch.full((prob.batch,), N, dtype=torch.int32)
    res = run(prob, "f32", flags=FLAGS | gdn.GDN_FLAG_CHUNKED)
    assert res["status"] == 0
    _chain_rows_parity(prob, res, CHAIN_PAIRS, CHAIN_ROWS)


def test_chunked_is_refused_outside_its_shapes():
    prob = _chain(70, dv=32)
    d = {k: getattr(prob, k).cuda() for k in ("q", "k", "v", "g", "beta", "parent", "state_in")}
    desc = gdn.make_desc(batch=2, n_nodes=70, n_k_heads=2, n_v_heads=6, d_k=128, d_v=32, scale=prob.scale,
                         flags=FLAGS | gdn.GDN_FLAG_CHUNKED)
    out = torch.empty(2, 70, 6, 32, device="cuda")
    ns = torch.empty(2, 1, 6, 32, 128, device="cuda")
    rc = gdn.gdn_tree_verify(desc, d["q"], d["k"], d["v"], d["g"], d["beta"], None, d["state_in"], out, ns,
                             check=False)
    assert rc == gdn.GDN_ERR_UNSUPPORTED
