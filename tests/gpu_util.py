"""Helpers for the GPU tests: run the CUDA library on a gdn_inputs.Problem and
compare with the oracle at the stated tolerances.

Tolerances (f32 accumulation against the exact f64 oracle on identical inputs):
  outputs o:           max |o_gpu - o_oracle| <= 2e-3
  persisted states:    ||S_gpu - S_oracle||_F / ||S_oracle||_F <= 1e-3 (f32), 5e-3 (f16),
                       per (sequence, node, v-head)
  tree / path indices: bit-exact (status codes, which nodes get written)
"""
from __future__ import annotations

import numpy as np
import torch

import gated_deltanet_tree_verify_b200 as gdn

OUT_ATOL = 2e-3
STATE_RTOL = {"f32": 1e-3, "f16": 5e-3}
_SD = {"f32": (gdn.GDN_F32, torch.float32), "f16": (gdn.GDN_F16, torch.float16)}


def to_dev(prob):
    return {name: getattr(prob, name).cuda() for name in
            ("q", "k", "v", "g", "beta", "parent", "state_in", "accept_path", "accept_len")}


def run(prob, state_dtype="f32", flags=0, parent=True, commit=True, dev=None, stream=None, workspace=False):
    """Verify (+ commit) on the GPU.  Unwritten outputs stay NaN.  With
    ``workspace``, through gdn_tree_verify_ws with a NaN-filled workspace of
    exactly gdn_tree_verify_workspace_bytes."""
    d = dev or to_dev(prob)
    B, N, Hk, dk = prob.q.shape
    Hv, dv = prob.v.shape[2], prob.v.shape[3]
    sd, tdt = _SD[state_dtype]
    NS = 1 if flags & gdn.GDN_FLAG_PERSIST_LAST else N
    out = torch.full((B, N, Hv, dv), float("nan"), device="cuda")
    ns = torch.full((B, NS, Hv, dv, dk), float("nan"), device="cuda", dtype=tdt)
    so = torch.full((B, Hv, dv, dk), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    desc = gdn.make_desc(batch=B, n_nodes=N, n_k_heads=Hk, n_v_heads=Hv, d_k=dk, d_v=dv,
                         scale=prob.scale, qkv_dtype=prob.q.dtype, state_dtype=sd, flags=flags,
                         status=status)
    par = d["parent"] if parent else None
    if workspace:
        nbytes = gdn.gdn_tree_verify_workspace_bytes(desc)
        ws = torch.full((max(nbytes, 16) // 4,), float("nan"), device="cuda")
        gdn.gdn_tree_verify_ws(desc, d["q"], d["k"], d["v"], d["g"], d["beta"], par, d["state_in"], out, ns,
                               ws, nbytes, stream=stream)
    else:
        gdn.gdn_tree_verify(desc, d["q"], d["k"], d["v"], d["g"], d["beta"], par, d["state_in"], out, ns,
                            stream=stream)
    if commit:
        gdn.gdn_tree_commit(desc, ns, par, d["accept_path"], d["accept_len"], d["accept_path"].shape[1],
                            so, stream=stream)
    torch.cuda.synchronize()
    return dict(out=out.cpu(), node_states=ns.cpu(), state_out=so.cpu(), status=int(status.item()))


def rel_fro(a: np.ndarray, b: np.ndarray, axes) -> np.ndarray:
    num = np.sqrt(((a - b) ** 2).sum(axis=axes))
    den = np.sqrt((b ** 2).sum(axis=axes))
    return num / np.maximum(den, 1e-30)


def assert_out_close(gpu_out, ora_out):
    g = gpu_out.double().numpy() if isinstance(gpu_out, torch.Tensor) else gpu_out
    assert np.isfinite(g).all(), "unwritten or non-finite outputs"
    err = np.abs(g - ora_out).max()
    assert err <= OUT_ATOL, f"out max-abs {err:.3e} > {OUT_ATOL}"
    return err


def assert_states_close(gpu_states, ora_states, state_dtype):
    g = gpu_states.double().numpy() if isinstance(gpu_states, torch.Tensor) else gpu_states
    assert np.isfinite(g).all(), "unwritten or non-finite states"
    r = rel_fro(g, ora_states, axes=(-2, -1))
    tol = STATE_RTOL[state_dtype]
    assert r.max() <= tol, f"state rel-Frobenius {r.max():.3e} > {tol}"
    return r.max()
