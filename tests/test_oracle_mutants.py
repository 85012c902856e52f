"""The oracle's pins catch plausible mistakes.

Each case copies gdn_oracle.c to a temporary directory, plants one mistake by
text substitution (a dropped term, a wrong sign or index, a transposed operand,
a wrong head group, ...), compiles the copy, swaps it in for the real oracle
library, and checks that at least one pin in test_oracle_pins fails.  Every
planted mistake keeps all memory accesses in bounds.
"""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_gates as gate_pins
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")

MUTANTS = {
    "sign_of_correction": ("u[i] = be * (vn[i] - w[i]);", "u[i] = be * (vn[i] + w[i]);"),
    "beta_dropped": ("u[i] = be * (vn[i] - w[i]);", "u[i] = (vn[i] - w[i]);"),
    "decay_missing_in_read": ("acc += Sp_scaled[(size_t)i * dk + j] * kn[j];",
                              "acc += Sp[(size_t)i * dk + j] * kn[j];"),
    "state_transposed_in_read": ("acc += Sp_scaled[(size_t)i * dk + j] * kn[j];",
                                 "acc += Sp_scaled[(size_t)(j % dv) * dk + (i % dk)] * kn[j];"),
    "decay_missing_in_write": ("Sn[(size_t)i * dk + j] = Sp_scaled[(size_t)i * dk + j] + u[i] * kn[j];",
                               "Sn[(size_t)i * dk + j] = Sp[(size_t)i * dk + j] + u[i] * kn[j];"),
    "q_in_rank1_write": ("+ u[i] * kn[j];", "+ u[i] * qn[j];"),
    "gate_not_exp_g": ("exp(J->g[((size_t)b * N + n) * Hv + h])",
                       "exp(0.5 * J->g[((size_t)b * N + n) * Hv + h])"),
    "output_from_parent_state": ("acc += Sn[(size_t)i * dk + j] * qn[j];",
                                 "acc += Sp_scaled[(size_t)i * dk + j] * qn[j];"),
    "output_uses_k": ("acc += Sn[(size_t)i * dk + j] * qn[j];", "acc += Sn[(size_t)i * dk + j] * kn[j];"),
    "scale_dropped": ("= J->scale * acc;", "= acc;"),
    "gqa_interleaved": ("const int hk = h / G;", "const int hk = h % Hk;"),
    "previous_node_not_parent": ("S + (size_t)p * SS;", "S + (size_t)(n - 1) * SS;"),
    "root_wrong_head": ("J->state_in + ((size_t)b * Hv + h) * SS", "J->state_in + ((size_t)b * Hv + 0) * SS"),
    "f16_not_rounded": ("return (double)(_Float16)x;", "return (double)(float)x;"),
    "recurrence_from_rounded": ("dst[e] = gdn_oracle_round(J->state_dtype, Sn[e]);",
                                "dst[e] = Sn[e] = gdn_oracle_round(J->state_dtype, Sn[e]);"),
    "commit_wrong_node": ("accept_path[(size_t)b * max_path_len + accept_len[b] - 1]",
                          "accept_path[(size_t)b * max_path_len + (accept_len[b] > 1 ? accept_len[b] - 2 : 0)]"),
    "path_link_unchecked": ("if (parent[path[i]] != path[i - 1])", "if (0)"),
    "tree_order_unchecked": ("if (parent[n] < 0 || parent[n] >= n)", "if (parent[n] < 0 || parent[n] >= n_nodes)"),
    # the q/k L2 normalisation
    "l2norm_without_sqrt": ("const double nrm = sqrt(ss);", "const double nrm = ss;"),
    "l2norm_sums_magnitudes": ("ss += row[j] * row[j];", "ss += fabs(row[j]);"),
    # the gate maps g = -softplus(x), beta = sigmoid(y)
    "softplus_sign": ("g[i] = isnan(xi) ? xi : -(fmax(xi, 0.0) + log1p(exp(-fabs(xi))));",
                      "g[i] = isnan(xi) ? xi : (fmax(xi, 0.0) + log1p(exp(-fabs(xi))));"),
    "softplus_max_term_dropped": ("-(fmax(xi, 0.0) + log1p(exp(-fabs(xi))))", "-(log1p(exp(-fabs(xi))))"),
    "sigmoid_sign_positive_branch": ("beta[i] = 1.0 / (1.0 + exp(-yi));", "beta[i] = 1.0 / (1.0 + exp(yi));"),
    "sigmoid_negative_branch_flipped": ("beta[i] = exp(yi) / (1.0 + exp(yi));", "beta[i] = 1.0 / (1.0 + exp(yi));"),
    "gate_inputs_swapped": ("const double xi = x[i], yi = y[i];", "const double xi = y[i], yi = x[i];"),
}

PINS = [
    pins.test_identity_beta0_g0_leaves_state_unchanged,
    pins.test_decay_only_is_exp_of_g,
    pins.test_reset_g_minus_inf,
    lambda: pins.test_delta_rule_write(1.0),
    lambda: pins.test_delta_rule_write(0.3),
    pins.test_state_is_dv_by_dk_not_transposed,
    pins.test_output_uses_updated_state_and_scale,
    pins.test_affine_in_parent_state,
    pins.test_gqa_contiguous_grouping,
    pins.test_chain_equals_sequential_recurrence,
    lambda: pins.test_every_node_equals_its_root_path("random"),
    lambda: pins.test_persisted_states_are_rounded_exact_states("f16"),
    pins.test_recurrence_continues_from_unrounded_state,
    lambda: pins.test_commit_equals_rerunning_accepted_path("f16"),
    pins.test_bad_trees_rejected,
    pins.test_bad_paths_rejected,
    pins.test_hand_worked_example_d2,
    pins.test_l2norm_worked_example,
    pins.test_l2norm_invariants,
    gate_pins.test_gate_values_at_closed_forms,
    gate_pins.test_gate_symmetries,
    gate_pins.test_gate_limits,
    gate_pins.test_verify_raw_gates_wiring,
]


def _build_mutant(tmp_path, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, old
    src = src.replace(old, new)
    path = tmp_path / "mut.c"
    path.write_text(src)
    lib = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", str(path),
                    "-o", str(lib), "-lm", "-lpthread"], check=True)
    return str(lib)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path, monkeypatch):
    import ctypes
    lib_path = _build_mutant(tmp_path, *MUTANTS[name])
    real = oracle._load()
    mut = ctypes.CDLL(lib_path)
    for fn in ("gdn_oracle_verify", "gdn_oracle_commit", "gdn_oracle_round", "gdn_oracle_round_array",
               "gdn_oracle_check_tree", "gdn_oracle_check_path", "gdn_oracle_gates", "gdn_oracle_l2norm_rows"):
        getattr(mut, fn).argtypes = getattr(real, fn).argtypes
        getattr(mut, fn).restype = getattr(real, fn).restype
    monkeypatch.setattr(oracle, "_lib", mut)
    caught = []
    for pin in PINS:
        try:
            pin()
        except (AssertionError, oracle.OracleError, pytest.fail.Exception):
            caught.append(pin)
    assert caught, f"no pin caught mutant {name}"
