"""Pins for the CPU oracle: closed forms, invariants, brute force, library routines.

None of these re-types the oracle's formula.  Each checks a property that the
gated delta rule (Gated DeltaNet recurrence; named as ggml_gated_delta_net in
the GreenGames post, "TL;DR") and the tree/commit contract (DDTree row of the
dflash-caddtree-integrations README, "What's in here": a width-1 tree equals
the chain exactly, branch states are kept consistent; GreenGames "Key wins":
states written by the kernel that computes them, in f16 or f32) fix,
chosen so that a dropped term, a wrong sign or index, or a transposed operand
fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gdn_inputs import make_problem, root_path, random_tree, ddtree_like_tree


def _rand_case(rng, N=1, dk=6, dv=5, Hk=1, Hv=1, parent=None, unit_k=True):
    q = rng.standard_normal((1, N, Hk, dk))
    k = rng.standard_normal((1, N, Hk, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((1, N, Hv, dv))
    g = -np.log1p(np.exp(rng.standard_normal((1, N, Hv))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((1, N, Hv))))
    s0 = 0.1 * rng.standard_normal((1, Hv, dv, dk))
    if parent is None:
        parent = np.arange(-1, N - 1, dtype=np.int32)[None]
    return dict(q=q, k=k, v=v, g=g, beta=beta, parent=np.asarray(parent, np.int32).reshape(1, N),
                state_in=s0, scale=1.0 / math.sqrt(dk))


def _run(c, state_dtype="f32"):
    return oracle.verify(c["q"], c["k"], c["v"], c["g"], c["beta"], c["parent"], c["state_in"],
                         c["scale"], state_dtype=state_dtype, want_exact=True)


# --------------------------------------------------------------------------
# Persisted-dtype rounding against numpy's own conversions (library routines)
# --------------------------------------------------------------------------

def test_round_f16_matches_numpy():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(20000),
        rng.standard_normal(2000) * 1e-6,          # subnormal range of f16
        rng.standard_normal(2000) * 3e4,           # near f16 max / overflow
        np.array([0.0, -0.0, 65504.0, 65520.0, 65519.99, 6e-8, 2.0 ** -25, 3 * 2.0 ** -26]),
        # exact ties between neighbouring f16 values: round to even
        1.0 + (2 * np.arange(64) + 1) * 2.0 ** -11,
    ])
    got = oracle.round_to("f16", x)
    want = x.astype(np.float16).astype(np.float64)
    np.testing.assert_array_equal(got, want)
    assert oracle.round_to("f16", np.array([1.0 + 2.0 ** -11]))[0] == 1.0       # tie -> even
    assert oracle.round_to("f16", np.array([1.0 + 3 * 2.0 ** -11]))[0] == 1.0 + 2.0 ** -9


def test_round_f32_matches_numpy():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.standard_normal(20000), rng.standard_normal(100) * 1e-40,
                        1.0 + (2 * np.arange(64) + 1) * 2.0 ** -24])
    np.testing.assert_array_equal(oracle.round_to("f32", x), x.astype(np.float32).astype(np.float64))


# --------------------------------------------------------------------------
# Single-node closed forms
# --------------------------------------------------------------------------

def test_identity_beta0_g0_leaves_state_unchanged():
    rng = np.random.default_rng(3)
    c = _rand_case(rng, N=4)
    c["g"][:] = 0.0
    c["beta"][:] = 0.0
    out, _, ex = _run(c)
    for n in range(4):
        np.testing.assert_array_equal(ex[0, n, 0], c["state_in"][0, 0])
        want = c["scale"] * c["state_in"][0, 0] @ c["q"][0, n, 0]
        np.testing.assert_allclose(out[0, n, 0], want, rtol=0, atol=1e-14)


def test_decay_only_is_exp_of_g():
    # beta = 0: S_n = exp(g_n) * S_p (math.exp, not the oracle's, gives a).
    rng = np.random.default_rng(4)
    c = _rand_case(rng, N=1)
    c["beta"][:] = 0.0
    c["g"][:] = -0.7
    _, _, ex = _run(c)
    np.testing.assert_array_equal(ex[0, 0, 0], math.exp(-0.7) * c["state_in"][0, 0])


def test_reset_g_minus_inf():
    # a = 0: S_n = beta v k^T, whatever S_p was.
    rng = np.random.default_rng(5)
    c = _rand_case(rng, N=1)
    c["g"][:] = -np.inf
    _, _, ex1 = _run(c)
    c2 = dict(c)
    c2["state_in"] = 7.0 * rng.standard_normal(c["state_in"].shape)
    _, _, ex2 = _run(c2)
    want = np.outer(c["beta"][0, 0, 0] * c["v"][0, 0, 0], c["k"][0, 0, 0])
    np.testing.assert_array_equal(ex1[0, 0, 0], want)
    np.testing.assert_array_equal(ex2[0, 0, 0], want)


@pytest.mark.parametrize("beta", [1.0, 0.3, 0.0])
def test_delta_rule_write(beta):
    # ||k|| = 1  =>  S_n k_n = (1 - beta) a S_p k_n + beta v_n.  beta = 1 writes v exactly.
    rng = np.random.default_rng(6)
    for trial in range(5):
        c = _rand_case(rng, N=1, dk=7, dv=9)
        c["beta"][:] = beta
        _, _, ex = _run(c)
        a = math.exp(c["g"][0, 0, 0])
        k = c["k"][0, 0, 0]
        want = (1 - beta) * a * (c["state_in"][0, 0] @ k) + beta * c["v"][0, 0, 0]
        np.testing.assert_allclose(ex[0, 0, 0] @ k, want, rtol=0, atol=1e-13)


def test_state_is_dv_by_dk_not_transposed():
    # With d_k != d_v a transposed state cannot even be shaped; with d_k = d_v a
    # non-symmetric S_p distinguishes S k from S^T k through the write identity.
    rng = np.random.default_rng(7)
    c = _rand_case(rng, N=1, dk=5, dv=5)
    c["beta"][:] = 1.0
    c["state_in"][0, 0] = np.triu(rng.standard_normal((5, 5)) + 3.0)
    _, _, ex = _run(c)
    np.testing.assert_allclose(ex[0, 0, 0] @ c["k"][0, 0, 0], c["v"][0, 0, 0], atol=1e-13)


def test_output_uses_updated_state_and_scale():
    # q = k, beta = 1 -> o = scale * S_n k = scale * v (not scale * a S_p k).
    rng = np.random.default_rng(8)
    c = _rand_case(rng, N=1, dk=8, dv=3)
    c["beta"][:] = 1.0
    c["q"] = c["k"].copy()
    c["scale"] = 0.37
    out, _, _ = _run(c)
    np.testing.assert_allclose(out[0, 0, 0], 0.37 * c["v"][0, 0, 0], atol=1e-13)


def test_output_general_matches_state_times_q():
    rng = np.random.default_rng(9)
    c = _rand_case(rng, N=3, dk=6, dv=4)
    out, _, ex = _run(c)
    for n in range(3):
        np.testing.assert_allclose(out[0, n, 0], c["scale"] * ex[0, n, 0] @ c["q"][0, n, 0],
                                   atol=1e-14)


def test_affine_in_parent_state():
    # S_n(alpha S_p) - S_n(0) = alpha (S_n(S_p) - S_n(0)), along a 4-node chain too.
    rng = np.random.default_rng(10)
    c = _rand_case(rng, N=4)
    _, _, e1 = _run(c)
    c0 = dict(c, state_in=np.zeros_like(c["state_in"]))
    _, _, e0 = _run(c0)
    ca = dict(c, state_in=2.5 * c["state_in"])
    _, _, ea = _run(ca)
    np.testing.assert_allclose(ea - e0, 2.5 * (e1 - e0), atol=1e-13)


# --------------------------------------------------------------------------
# Head grouping
# --------------------------------------------------------------------------

def test_gqa_contiguous_grouping():
    # H_v = 4 over H_k = 2 equals H_k = 4 with k/q expanded as [k0, k0, k1, k1].
    rng = np.random.default_rng(11)
    c = _rand_case(rng, N=3, Hk=2, Hv=4)
    out, _, ex = _run(c)
    idx = [0, 0, 1, 1]
    ce = dict(c, q=c["q"][:, :, idx], k=c["k"][:, :, idx])
    out_e, _, ex_e = _run(ce)
    np.testing.assert_array_equal(out, out_e)
    np.testing.assert_array_equal(ex, ex_e)
    # the interleaved reading gives different numbers: the test discriminates
    ci = dict(c, q=c["q"][:, :, [0, 1, 0, 1]], k=c["k"][:, :, [0, 1, 0, 1]])
    out_i, _, _ = _run(ci)
    assert np.abs(out_i - out).max() > 1e-3


# --------------------------------------------------------------------------
# Chains and trees: composition of single-node steps (brute force)
# --------------------------------------------------------------------------

def _single_step(c, n, hv, state):
    """One node run alone as a 1-node tree with state_in = ``state``."""
    G = c["v"].shape[2] // c["q"].shape[2]
    hk = hv // G
    sub = dict(q=c["q"][:, n:n + 1, hk:hk + 1], k=c["k"][:, n:n + 1, hk:hk + 1],
               v=c["v"][:, n:n + 1, hv:hv + 1], g=c["g"][:, n:n + 1, hv:hv + 1],
               beta=c["beta"][:, n:n + 1, hv:hv + 1], parent=np.array([[-1]], np.int32),
               state_in=state[None, None], scale=c["scale"])
    out, _, ex = _run(sub)
    return out[0, 0, 0], ex[0, 0, 0]


def test_chain_equals_sequential_recurrence():
    rng = np.random.default_rng(12)
    N = 6
    c = _rand_case(rng, N=N, Hk=2, Hv=4)
    out, _, ex = _run(c)
    for h in range(4):
        S = c["state_in"][0, h]
        for n in range(N):
            o1, S = _single_step(c, n, h, S)
            np.testing.assert_array_equal(out[0, n, h], o1)
            np.testing.assert_array_equal(ex[0, n, h], S)


@pytest.mark.parametrize("kind", ["random", "ddtree"])
def test_every_node_equals_its_root_path(kind):
    rng = np.random.default_rng(13)
    N = 12
    gen = torch.Generator().manual_seed(3)
    par = random_tree(N, gen) if kind == "random" else ddtree_like_tree(N - 1, gen, max_depth=5)
    c = _rand_case(rng, N=N, Hk=1, Hv=2, parent=par)
    out, _, ex = _run(c)
    for h in range(2):
        for n in range(N):
            S = c["state_in"][0, h]
            for m in root_path(par, n):
                o1, S = _single_step(c, m, h, S)
            np.testing.assert_array_equal(out[0, n, h], o1)
            np.testing.assert_array_equal(ex[0, n, h], S)


def test_sibling_independence_and_relabeling():
    # Tree A: 0 -> {1, 2}, 1 -> 3.  Tree B adds branches and renumbers:
    # 0 -> {1 (=A2), 2 (new), 3 (=A1)}, 3 -> {4 (new), 5 (=A3)}.
    rng = np.random.default_rng(14)
    ca = _rand_case(rng, N=4, parent=[-1, 0, 0, 1])
    extra = _rand_case(rng, N=2)
    mapB = {1: ("A", 2), 2: ("X", 0), 3: ("A", 1), 4: ("X", 1), 5: ("A", 3), 0: ("A", 0)}
    cb = {key: None for key in ca}
    for key in ("q", "k", "v", "g", "beta"):
        rows = []
        for n in range(6):
            src, i = mapB[n]
            rows.append((ca if src == "A" else extra)[key][:, i:i + 1])
        cb[key] = np.concatenate(rows, axis=1)
    cb["parent"] = np.array([[-1, 0, 0, 0, 3, 3]], np.int32)
    cb["state_in"], cb["scale"] = ca["state_in"], ca["scale"]
    oa, _, ea = _run(ca)
    ob, _, eb = _run(cb)
    for nb, (src, ia) in mapB.items():
        if src == "A":
            np.testing.assert_array_equal(ob[0, nb], oa[0, ia])
            np.testing.assert_array_equal(eb[0, nb], ea[0, ia])


# --------------------------------------------------------------------------
# Persistence and commit
# --------------------------------------------------------------------------

@pytest.mark.parametrize("sd", ["f32", "f16"])
def test_persisted_states_are_rounded_exact_states(sd):
    rng = np.random.default_rng(15)
    c = _rand_case(rng, N=5, parent=[-1, 0, 1, 1, 0])
    _, st, ex = _run(c, state_dtype=sd)
    np_dt = np.float16 if sd == "f16" else np.float32
    np.testing.assert_array_equal(st, ex.astype(np_dt).astype(np.float64))


def test_recurrence_continues_from_unrounded_state():
    # Children see the exact parent state, never the f16 copy: the f16 run's
    # exact states equal the f32 run's exact states bit for bit.
    rng = np.random.default_rng(16)
    c = _rand_case(rng, N=5, parent=[-1, 0, 1, 1, 0])
    o32, _, e32 = _run(c, "f32")
    o16, _, e16 = _run(c, "f16")
    np.testing.assert_array_equal(e32, e16)
    np.testing.assert_array_equal(o32, o16)


@pytest.mark.parametrize("sd", ["f32", "f16"])
def test_commit_equals_rerunning_accepted_path(sd):
    prob = make_problem(batch=3, n_nodes=10, n_k_heads=1, n_v_heads=2, d_k=8, d_v=8,
                        tree="random", seed=5, qkv_dtype="f32", accept="node")
    out, st, _ = oracle.verify_problem(prob, state_dtype=sd)
    so = oracle.commit(st, prob.parent, prob.accept_path, prob.accept_len)
    c = dict(q=prob.q.double().numpy(), k=prob.k.double().numpy(), v=prob.v.double().numpy(),
             g=prob.g.double().numpy(), beta=prob.beta.double().numpy(), scale=prob.scale)
    for b in range(3):
        path = prob.accept_path[b, :int(prob.accept_len[b])].tolist()
        cb = {key: c[key][b:b + 1] if key != "scale" else c[key] for key in c}
        for h in range(2):
            S = prob.state_in[b, h].double().numpy()
            for m in path:
                _, S = _single_step(cb, m, h, S)
            np.testing.assert_array_equal(so[b, h], oracle.round_to(sd, S))


def test_bad_trees_rejected():
    good = np.array([-1, 0, 0, 2], np.int32)
    assert oracle.check_tree(good) == oracle.OK
    for bad in ([0, 0, 0, 2], [-1, 1, 0, 2], [-1, 0, 3, 2], [-1, 0, -1, 2], [-1, 0, 0, 7],
                [5]):
        assert oracle.check_tree(np.array(bad, np.int32)) == oracle.ERR_BAD_TREE
    rng = np.random.default_rng(17)
    c = _rand_case(rng, N=4, parent=[-1, 0, 2, 1])
    with pytest.raises(oracle.OracleError) as e:
        _run(c)
    assert e.value.code == oracle.ERR_BAD_TREE


def test_bad_paths_rejected():
    par = np.array([-1, 0, 0, 1, 3], np.int32)
    ok = [([0, 1, 3, 4], 4), ([0], 1), ([0, 2, -1, -1], 2)]
    for p, L in ok:
        assert oracle.check_path(par, np.array(p, np.int32), L) == oracle.OK
    bad = [([1, 3, 4, 0], 3), ([0, 2, 3, 0], 3), ([0, 1, 3, 4], 0), ([0, 1, 3, 4], 5),
           ([0, 0, 0, 0], 2), ([0, 1, 9, 0], 3), ([0, 1, -3, 0], 3)]
    for p, L in bad:
        assert oracle.check_path(par, np.array(p, np.int32), L) == oracle.ERR_BAD_PATH, (p, L)


# --------------------------------------------------------------------------
# A hand-worked example (d_k = d_v = 2), exact values derived on paper
# --------------------------------------------------------------------------

def test_hand_worked_example_d2():
    """Tree 0 -> {1, 2}, 1 -> 3; S_in = [[1, 0], [0, 2]]; scale = 1/sqrt(2).

    node 0: k=(1,0) q=(0,1) v=(3,4) a=1 beta=1/2
        w = S_in k = (1,0); u = (1,2); S0 = [[2,0],[2,2]]; o0 = (0, 2)/sqrt(2)
    node 1 (of 0): k=(.6,.8) q=(1,0) v=(1,-1) a=1/2 beta=1
        S' = [[1,0],[1,1]]; w = (.6, 1.4); u = (.4, -2.4)
        S1 = [[1.24, .32], [-.44, -.92]]; o1 = (1.24, -.44)/sqrt(2)
    node 2 (of 0): k=(0,1) q=(.6,.8) v=(2,-4) a=1/4 beta=1/2
        S' = [[.5,0],[.5,.5]]; w = (0, .5); u = (1, -2.25)
        S2 = [[.5, 1], [.5, -1.75]]; o2 = (1.1, -1.1)/sqrt(2)
    node 3 (of 1): k=(1,0) q=(1,0) v=(5,5) a=1 beta=1
        w = (1.24, -.44); u = (3.76, 5.44); S3 = [[5, .32], [5, -.92]]; o3 = (5, 5)/sqrt(2)
    commit path [0, 1, 3] -> S3.
    """
    r2 = math.sqrt(2.0)
    q = np.array([[0, 1], [1, 0], [.6, .8], [1, 0]], float)[None, :, None]
    k = np.array([[1, 0], [.6, .8], [0, 1], [1, 0]], float)[None, :, None]
    v = np.array([[3, 4], [1, -1], [2, -4], [5, 5]], float)[None, :, None]
    g = np.log(np.array([1.0, 0.5, 0.25, 1.0]))[None, :, None]
    beta = np.array([0.5, 1.0, 0.5, 1.0])[None, :, None]
    par = np.array([[-1, 0, 0, 1]], np.int32)
    s0 = np.array([[1.0, 0.0], [0.0, 2.0]])[None, None]
    out, st, ex = oracle.verify(q, k, v, g, beta, par, s0, 1 / r2, want_exact=True)
    S = {0: [[2, 0], [2, 2]], 1: [[1.24, .32], [-.44, -.92]], 2: [[.5, 1], [.5, -1.75]],
         3: [[5, .32], [5, -.92]]}
    O = {0: [0, 2], 1: [1.24, -.44], 2: [1.1, -1.1], 3: [5, 5]}
    for n in range(4):
        np.testing.assert_allclose(ex[0, n, 0], np.array(S[n]), atol=1e-14)
        np.testing.assert_allclose(out[0, n, 0], np.array(O[n]) / r2, atol=1e-14)
    so = oracle.commit(st, par, np.array([[0, 1, 3]], np.int32), np.array([3], np.int32))
    np.testing.assert_allclose(so[0, 0], np.float32(np.array(S[3])), atol=0)


# ----------------------------------------------------------------------------
# q/k L2 normalisation (the workloads' input preparation, fused by the
# library's GDN_FLAG_QK_L2NORM)
# ----------------------------------------------------------------------------

def test_l2norm_worked_example():
    # 3-4-5 and 1-2-2-4 (norm 5) triangles, by hand
    x = np.array([[3.0, 4.0, 0.0, 0.0], [1.0, 2.0, 2.0, 4.0]])
    y = oracle.l2norm_rows(x)
    np.testing.assert_array_equal(y[0], [0.6, 0.8, 0.0, 0.0])
    np.testing.assert_allclose(y[1], [0.2, 0.4, 0.4, 0.8], rtol=0, atol=1e-15)


def test_l2norm_invariants():
    rng = np.random.default_rng(3)
    x = rng.normal(size=(5, 7, 32))
    y = oracle.l2norm_rows(x)
    np.testing.assert_allclose(np.sqrt((y ** 2).sum(-1)), 1.0, rtol=0, atol=1e-14)
    # direction kept: y is a positive multiple of x
    ratio = y / x
    np.testing.assert_allclose(ratio, np.broadcast_to(ratio[..., :1], ratio.shape), rtol=1e-12)
    assert (ratio > 0).all()
    # scale invariance and idempotence
    np.testing.assert_allclose(oracle.l2norm_rows(3.5 * x), y, rtol=0, atol=1e-15)
    np.testing.assert_allclose(oracle.l2norm_rows(y), y, rtol=0, atol=1e-15)
    # epsilon 0: a zero row is NaN, not silently zero
    z = oracle.l2norm_rows(np.zeros((1, 4)))
    assert np.isnan(z).all()


def test_verify_with_l2norm_equals_verify_on_normalised_inputs():
    prob = make_problem(batch=1, n_nodes=6, n_k_heads=1, n_v_heads=2, d_k=8, d_v=4, tree="random", seed=5,
                        qkv_dtype="f32")
    rng = np.random.default_rng(9)
    qr = prob.q.double().numpy() * rng.uniform(0.2, 5.0, size=prob.q.shape[:3] + (1,))
    kr = prob.k.double().numpy() * rng.uniform(0.2, 5.0, size=prob.k.shape[:3] + (1,))
    a = oracle.verify(qr, kr, prob.v, prob.g, prob.beta, prob.parent, prob.state_in, prob.scale,
                      want_exact=True, qk_l2norm=True)
    b = oracle.verify(oracle.l2norm_rows(qr), oracle.l2norm_rows(kr), prob.v, prob.g, prob.beta, prob.parent,
                      prob.state_in, prob.scale, want_exact=True)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    # and the raw inputs were not unit (the normalisation did something)
    assert abs(np.linalg.norm(kr[0, 0, 0]) - 1.0) > 1e-3
