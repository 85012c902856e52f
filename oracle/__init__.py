"""CPU oracle for gated-delta-rule tree verification (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its
binding) never imports it.  The arithmetic lives in ``gdn_oracle.c`` (plain C,
double precision); this module only compiles it with gcc and marshals numpy
arrays to it.  See the C file's header for the definition and its citations.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "libgdnoracle.so")

OK, ERR_INVALID_ARG, ERR_BAD_TREE, ERR_BAD_PATH = 0, 1, 3, 4
STATE_F32, STATE_F16 = 0, 1
_STATE = {"f32": STATE_F32, "f16": STATE_F16}

_lib = None


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into libgdnoracle.so next to it (gcc, -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall", "-Wextra",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", _LIB + ".tmp", "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        c_int, c_double, c_i64 = ctypes.c_int, ctypes.c_double, ctypes.c_int64
        lib.gdn_oracle_verify.argtypes = [c_int] * 6 + [c_double, c_int] + [dp] * 5 + [ip, dp, dp, dp, dp, c_int]
        lib.gdn_oracle_verify.restype = c_int
        lib.gdn_oracle_commit.argtypes = [c_int] * 5 + [dp, ip, ip, ip, c_int, dp]
        lib.gdn_oracle_commit.restype = c_int
        lib.gdn_oracle_round.argtypes = [c_int, c_double]
        lib.gdn_oracle_round.restype = c_double
        lib.gdn_oracle_round_array.argtypes = [c_int, dp, dp, c_i64]
        lib.gdn_oracle_round_array.restype = None
        lib.gdn_oracle_l2norm_rows.argtypes = [dp, c_i64, c_int]
        lib.gdn_oracle_l2norm_rows.restype = None
        lib.gdn_oracle_gates.argtypes = [dp, dp, dp, dp, c_i64]
        lib.gdn_oracle_gates.restype = None
        lib.gdn_oracle_check_tree.argtypes = [c_int, ip]
        lib.gdn_oracle_check_tree.restype = c_int
        lib.gdn_oracle_check_path.argtypes = [c_int, ip, ip, c_int, c_int]
        lib.gdn_oracle_check_path.restype = c_int
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor: widen exactly (bf16/f32 -> f64)
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _dp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _ip(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


class OracleError(RuntimeError):
    def __init__(self, code: int):
        super().__init__(f"oracle returned {code}")
        self.code = code


def l2norm_rows(x) -> np.ndarray:
    """x / |x| over the last axis, in double (gdn_oracle_l2norm_rows)."""
    y = _f64(x).copy()
    _load().gdn_oracle_l2norm_rows(_dp(y), y.size // y.shape[-1], y.shape[-1])
    return y


def gates(x, y) -> Tuple[np.ndarray, np.ndarray]:
    """(g, beta) = (-softplus(x), sigmoid(y)) elementwise, in double
    (gdn_oracle_gates)."""
    x, y = _f64(x), _f64(y)
    assert x.shape == y.shape
    g, beta = np.empty_like(x), np.empty_like(y)
    _load().gdn_oracle_gates(_dp(x), _dp(y), _dp(g), _dp(beta), x.size)
    return g, beta


def verify(q, k, v, g, beta, parent, state_in, scale: float, state_dtype: str = "f32",
           want_exact: bool = False, nthreads: int = 1, qk_l2norm: bool = False,
           raw_gates: bool = False) -> Tuple[np.ndarray, np.ndarray, Optional[np.ndarray]]:
    """Run the tree recurrence.  Returns (out, persisted_states, exact_states).

    Shapes as in gdn_oracle.c.  ``persisted_states`` holds each node's state
    rounded to ``state_dtype`` (as float64 values); ``exact_states`` (only if
    ``want_exact``) holds the unrounded float64 states.  With ``qk_l2norm``
    q and k are L2-normalised per (node, head) first (the preparation the
    library's GDN_FLAG_QK_L2NORM fuses).  With ``raw_gates`` g and beta hold
    the pre-activations x and y, and the recurrence runs on g = -softplus(x),
    beta = sigmoid(y) (``gates``; the library's GDN_FLAG_GATES).  Raises
    OracleError on a bad tree or bad arguments.
    """
    lib = _load()
    if qk_l2norm:
        q, k = l2norm_rows(q), l2norm_rows(k)
    if raw_gates:
        g, beta = gates(g, beta)
    q, k, v, g, beta, state_in = map(_f64, (q, k, v, g, beta, state_in))
    parent = _i32(parent)
    B, N, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    assert k.shape == q.shape and v.shape[:2] == (B, N)
    assert g.shape == (B, N, Hv) and beta.shape == (B, N, Hv)
    assert parent.shape == (B, N) and state_in.shape == (B, Hv, dv, dk)
    out = np.zeros((B, N, Hv, dv))
    states = np.zeros((B, N, Hv, dv, dk))
    exact = np.zeros((B, N, Hv, dv, dk)) if want_exact else None
    rc = lib.gdn_oracle_verify(B, N, Hk, Hv, dk, dv, float(scale), _STATE[state_dtype],
                               _dp(q), _dp(k), _dp(v), _dp(g), _dp(beta), _ip(parent),
                               _dp(state_in), _dp(out), _dp(states),
                               _dp(exact) if exact is not None else None, int(nthreads))
    if rc != OK:
        raise OracleError(rc)
    return out, states, exact


def commit(states, parent, accept_path, accept_len) -> np.ndarray:
    """state_out[b] = states[b][path_b[len_b - 1]] after checking every path."""
    lib = _load()
    states = _f64(states)
    parent, accept_path, accept_len = map(_i32, (parent, accept_path, accept_len))
    B, N, Hv, dv, dk = states.shape
    P = accept_path.shape[1]
    out = np.zeros((B, Hv, dv, dk))
    rc = lib.gdn_oracle_commit(B, N, Hv, dk, dv, _dp(states), _ip(parent), _ip(accept_path),
                               _ip(accept_len), P, _dp(out))
    if rc != OK:
        raise OracleError(rc)
    return out


def compact(rows, parent, accept_path, accept_len, cu_nodes=None):
    """Accept-time compaction of per-node rows into path order.

    After verification only the accepted root-to-leaf path's per-node data
    is carried forward (the GreenGames post, "Key wins": the target features
    are compacted after a sibling branch is accepted).  For each sequence b
    whose path checks against its tree (as ``commit`` checks it):
    dst[b][i] = rows[n0_b + path_b[i]] for i < len_b.

    rows: [T, ...] per-node rows in the packed node layout (T = B * N, or
    the varlen total with cu_nodes [B + 1] offsets); parent: [T] int32 local
    indices.  Returns (dst [B, P, ...] with unwritten rows zero, written
    [B, P] bool).  A bad path writes nothing for its sequence.
    """
    rows = np.asarray(rows)
    parent, accept_path, accept_len = map(_i32, (parent, accept_path, accept_len))
    B, P = accept_path.shape
    if cu_nodes is None:
        N = parent.shape[0] // B if B else 0
        cu = np.arange(B + 1, dtype=np.int64) * N
    else:
        cu = np.asarray(cu_nodes, dtype=np.int64)
    dst = np.zeros((B, P) + rows.shape[1:], dtype=rows.dtype)
    written = np.zeros((B, P), dtype=bool)
    for b in range(B):
        n0, n1 = int(cu[b]), int(cu[b + 1])
        if check_path(parent[n0:n1], accept_path[b], int(accept_len[b])) != OK:
            continue
        for i in range(int(accept_len[b])):
            dst[b, i] = rows[n0 + int(accept_path[b, i])]
            written[b, i] = True
    return dst, written


def round_to(state_dtype: str, x) -> np.ndarray:
    """Round float64 values to the persisted dtype and back (RNE)."""
    lib = _load()
    x = _f64(x)
    y = np.empty_like(x)
    lib.gdn_oracle_round_array(_STATE[state_dtype], _dp(x), _dp(y), x.size)
    return y


def check_tree(parent_row) -> int:
    p = _i32(parent_row)
    return _load().gdn_oracle_check_tree(len(p), _ip(p))


def check_path(parent_row, path_row, length: int) -> int:
    p, a = _i32(parent_row), _i32(path_row)
    return _load().gdn_oracle_check_path(len(p), _ip(p), _ip(a), int(length), len(a))


def verify_problem(prob, state_dtype: str = "f32", want_exact: bool = False, nthreads: int = 1,
                   qk_l2norm: bool = False, raw_gates: bool = False):
    """Convenience: run ``verify`` on a gdn_inputs.Problem."""
    return verify(prob.q, prob.k, prob.v, prob.g, prob.beta, prob.parent, prob.state_in,
                  prob.scale, state_dtype=state_dtype, want_exact=want_exact, nthreads=nthreads,
                  qk_l2norm=qk_l2norm, raw_gates=raw_gates)


def verify_pair(prob, b: int, h: int, state_dtype: str = "f32", want_exact: bool = False):
    """Oracle for one (sequence b, v-head h) of a problem: slices the inputs to
    B = 1, H_k = H_v = 1 (v-head h reads k-head h // G) and runs ``verify``."""
    G = prob.n_v_heads // prob.n_k_heads
    hk = h // G
    return verify(prob.q[b:b + 1, :, hk:hk + 1], prob.k[b:b + 1, :, hk:hk + 1],
                  prob.v[b:b + 1, :, h:h + 1], prob.g[b:b + 1, :, h:h + 1],
                  prob.beta[b:b + 1, :, h:h + 1], prob.parent[b:b + 1],
                  prob.state_in[b:b + 1, h:h + 1], prob.scale, state_dtype=state_dtype,
                  want_exact=want_exact)
