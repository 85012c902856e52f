"""Pins of the oracle's gate maps (oracle.gates: g = -softplus(x),
beta = sigmoid(y), the workloads' input recipe) and of their wiring into
oracle.verify(raw_gates=True).  Closed forms, symmetries and limits; the
wiring against an independent numpy formulation."""
import math

import numpy as np
import pytest
import torch

import oracle
from gdn_inputs import make_problem


def test_gate_values_at_closed_forms():
    # softplus(0) = ln 2, softplus(ln 3) = ln 4; sigmoid(0) = 1/2, sigmoid(ln 3) = 3/4
    g, b = oracle.gates([0.0, math.log(3.0), -math.log(3.0)], [0.0, math.log(3.0), -math.log(3.0)])
    assert abs(g[0] + math.log(2.0)) < 1e-15
    assert abs(g[1] + math.log(4.0)) < 1e-15
    assert abs(g[2] + math.log(4.0 / 3.0)) < 1e-15
    assert abs(math.exp(g[1]) - 0.25) < 1e-15          # a = 1 / (1 + e^x)
    assert abs(b[0] - 0.5) < 1e-16
    assert abs(b[1] - 0.75) < 1e-15 and abs(b[2] - 0.25) < 1e-15


def test_gate_symmetries():
    x = np.linspace(-40.0, 40.0, 801)
    g, b = oracle.gates(x, x)
    gm, bm = oracle.gates(-x, -x)
    # softplus(x) - softplus(-x) = x;  sigmoid(y) + sigmoid(-y) = 1
    np.testing.assert_allclose(-g + gm, x, rtol=0, atol=1e-13)
    np.testing.assert_allclose(b + bm, 1.0, rtol=0, atol=1e-15)
    # a = exp(-softplus(x)) = sigmoid(-x)
    np.testing.assert_allclose(np.exp(g), bm, rtol=1e-14, atol=0)
    # both monotone (sigmoid saturates to 1 in double beyond y ~ 37)
    assert np.all(np.diff(g) < 0) and np.all(np.diff(b) >= 0) and np.all(np.diff(b[200:601]) > 0)


def test_gate_limits():
    x = np.array([np.inf, -np.inf, 1000.0, -1000.0, np.nan])
    g, b = oracle.gates(x, x)
    assert g[0] == -np.inf and math.exp(g[0]) == 0.0           # a = 0: a reset
    assert g[1] == 0.0 and math.exp(g[1]) == 1.0
    assert g[2] == -1000.0 and g[3] == 0.0                     # no overflow, no cancellation
    assert np.isnan(g[4]) and np.isnan(b[4])
    assert b[0] == 1.0 and b[1] == 0.0 and b[2] == 1.0 and b[3] == 0.0


def _raw_problem(seed=3):
    prob = make_problem(batch=2, n_nodes=9, n_k_heads=1, n_v_heads=2, d_k=32, d_v=32, tree="random",
                        seed=seed, qkv_dtype="f32", raw_gates=True)
    prob.beta = (prob.beta + 1.5).contiguous()     # x and y from different distributions
    return prob


def test_verify_raw_gates_wiring():
    prob = _raw_problem()
    x, y = prob.g.double().numpy(), prob.beta.double().numpy()
    g_np = -np.logaddexp(0.0, x)
    b_np = 1.0 / (1.0 + np.exp(-y))
    out_r, st_r, _ = oracle.verify(prob.q, prob.k, prob.v, prob.g, prob.beta, prob.parent, prob.state_in,
                                   prob.scale, raw_gates=True)
    out_n, st_n, _ = oracle.verify(prob.q, prob.k, prob.v, g_np, b_np, prob.parent, prob.state_in, prob.scale)
    np.testing.assert_allclose(out_r, out_n, rtol=0, atol=1e-12)
    np.testing.assert_allclose(st_r, st_n, rtol=0, atol=1e-12)
    # the wiring test sees a swap of x and y
    out_s, _, _ = oracle.verify(prob.q, prob.k, prob.v, -np.logaddexp(0.0, y), 1.0 / (1.0 + np.exp(-x)),
                                prob.parent, prob.state_in, prob.scale)
    assert np.abs(out_s - out_r).max() > 1e-3


def test_generator_raw_draws_are_the_default_draws():
    raw = make_problem(batch=1, n_nodes=12, n_k_heads=2, n_v_heads=4, d_k=32, d_v=32, tree="random", seed=8,
                       qkv_dtype="bf16", raw_gates=True)
    dflt = make_problem(batch=1, n_nodes=12, n_k_heads=2, n_v_heads=4, d_k=32, d_v=32, tree="random", seed=8,
                        qkv_dtype="bf16")
    g, b = oracle.gates(raw.g, raw.beta)
    np.testing.assert_allclose(g, dflt.g.double().numpy(), rtol=0, atol=1e-6)
    np.testing.assert_allclose(b, dflt.beta.double().numpy(), rtol=0, atol=1e-6)
    for key in ("q", "k", "v", "state_in", "parent", "accept_path"):
        assert torch.equal(getattr(raw, key), getattr(dflt, key))
    with pytest.raises(ValueError):
        make_problem(batch=1, n_nodes=4, n_k_heads=1, n_v_heads=1, d_k=32, d_v=32, tree="chain", seed=1,
                     gate="uniform_a", raw_gates=True)
