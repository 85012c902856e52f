"""Python binding of libgdntree (argument marshalling only).

Same names as the C ABI in include/gdntree.h.  Tensors are torch CUDA tensors
(their device pointers are passed through); every step of the computation runs
in the library's CUDA kernels.  There is no fallback: if the shared library is
missing or a tensor is not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Union

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libgdntree.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "gdntree.h")

# gdn_dtype
GDN_F32, GDN_F16, GDN_BF16 = 0, 1, 2
# gdn_status
GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_BAD_TREE, GDN_ERR_BAD_PATH, \
    GDN_ERR_CUDA, GDN_ERR_TIMEOUT, GDN_ERR_BAD_INPUT = range(8)
# flags
GDN_FLAG_CHAIN, GDN_FLAG_PERSIST_LAST, GDN_FLAG_VALIDATE, GDN_FLAG_EARLY_TREE, GDN_FLAG_CHUNKED = 1, 2, 4, 8, 16
GDN_FLAG_QK_L2NORM = 32
GDN_FLAG_GATES = 64
GDN_MAX_TREE_NODES = 1024
# gdn_build_desc.flags
GDN_BUILD_CHAIN_SEED, GDN_BUILD_VALIDATE = 1, 2

_TORCH_DTYPE = {GDN_F32: torch.float32, GDN_F16: torch.float16, GDN_BF16: torch.bfloat16}
_GDN_DTYPE = {torch.float32: GDN_F32, torch.float16: GDN_F16, torch.bfloat16: GDN_BF16}


class GdnTreeDesc(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("n_nodes", ctypes.c_int32),
        ("n_k_heads", ctypes.c_int32),
        ("n_v_heads", ctypes.c_int32),
        ("d_k", ctypes.c_int32),
        ("d_v", ctypes.c_int32),
        ("scale", ctypes.c_float),
        ("qkv_dtype", ctypes.c_int32),
        ("state_dtype", ctypes.c_int32),
        ("flags", ctypes.c_uint32),
        ("status", ctypes.c_void_p),
    ]


class GdnBuildDesc(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("max_depth", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("budget", ctypes.c_int32),
        ("flags", ctypes.c_uint32),
        ("status", ctypes.c_void_p),
    ]


class GdnError(RuntimeError):
    def __init__(self, status: int, detail: str = ""):
        self.status = status
        super().__init__(f"{gdn_status_str(status)}: {detail}" if detail else gdn_status_str(status))


class GdnLibraryMissing(ImportError):
    pass


_lib = None


def load_library() -> ctypes.CDLL:
    """Load lib/libgdntree.so (built by gated_deltanet_tree_verify_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise GdnLibraryMissing(
            f"{LIB_PATH} is missing: build it with `python -m gated_deltanet_tree_verify_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    dp = ctypes.POINTER(GdnTreeDesc)
    lib.gdn_tree_verify.argtypes = [dp] + [vp] * 10
    lib.gdn_tree_verify.restype = ctypes.c_int
    lib.gdn_tree_verify_ws.argtypes = [dp] + [vp] * 10 + [ctypes.c_size_t, vp]
    lib.gdn_tree_verify_ws.restype = ctypes.c_int
    lib.gdn_tree_verify_workspace_bytes.argtypes = [dp]
    lib.gdn_tree_verify_workspace_bytes.restype = ctypes.c_size_t
    lib.gdn_tree_verify_static_ws.argtypes = [dp] + [vp] * 10
    lib.gdn_tree_verify_static_ws.restype = ctypes.c_int
    lib.gdn_static_workspace_capacity.argtypes = []
    lib.gdn_static_workspace_capacity.restype = ctypes.c_size_t
    lib.gdn_tree_verify_varlen.argtypes = [dp, vp, i32] + [vp] * 10 + [ctypes.c_size_t, vp]
    lib.gdn_tree_verify_varlen.restype = ctypes.c_int
    lib.gdn_tree_commit_varlen.argtypes = [dp, vp, i32, i32, ctypes.POINTER(vp), vp, vp, vp, i32,
                                           ctypes.POINTER(vp), vp]
    lib.gdn_tree_commit_varlen.restype = ctypes.c_int
    lib.gdn_tree_commit.argtypes = [dp, vp, vp, vp, vp, i32, vp, vp]
    lib.gdn_tree_commit.restype = ctypes.c_int
    lib.gdn_tree_commit_layers.argtypes = [dp, i32, ctypes.POINTER(vp), vp, vp, vp, i32,
                                           ctypes.POINTER(vp), vp]
    lib.gdn_tree_commit_layers.restype = ctypes.c_int
    lib.gdn_build_tree.argtypes = [ctypes.POINTER(GdnBuildDesc)] + [vp] * 8
    lib.gdn_build_tree.restype = ctypes.c_int
    lib.gdn_tree_compact.argtypes = [i32, i32, vp, i32, ctypes.c_size_t, vp, vp, vp, vp, i32, vp, vp, vp]
    lib.gdn_tree_compact.restype = ctypes.c_int
    lib.gdn_tree_plan_bytes.argtypes = [dp]
    lib.gdn_tree_plan_bytes.restype = ctypes.c_size_t
    lib.gdn_tree_plan.argtypes = [dp, vp, vp, ctypes.c_size_t, vp]
    lib.gdn_tree_plan.restype = ctypes.c_int
    lib.gdn_tree_verify_planned.argtypes = [dp, vp, ctypes.c_size_t] + [vp] * 10
    lib.gdn_tree_verify_planned.restype = ctypes.c_int
    lib.gdn_status_str.argtypes = [ctypes.c_int]
    lib.gdn_status_str.restype = ctypes.c_char_p
    lib.gdn_last_error_detail.argtypes = []
    lib.gdn_last_error_detail.restype = ctypes.c_char_p
    lib.gdn_node_states_bytes.argtypes = [dp]
    lib.gdn_node_states_bytes.restype = ctypes.c_size_t
    lib.gdn_version.argtypes = []
    lib.gdn_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def header_functions() -> list:
    """Names of the functions include/gdntree.h declares."""
    src = open(HEADER_PATH).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_\w+)\s*\(", src)))


def make_desc(*, batch: int, n_nodes: int, n_k_heads: int, n_v_heads: int, d_k: int, d_v: int,
              scale: float, qkv_dtype: Union[int, torch.dtype] = GDN_BF16,
              state_dtype: Union[int, torch.dtype] = GDN_F32, flags: int = 0,
              status: Optional[torch.Tensor] = None) -> GdnTreeDesc:
    if isinstance(qkv_dtype, torch.dtype):
        qkv_dtype = _GDN_DTYPE[qkv_dtype]
    if isinstance(state_dtype, torch.dtype):
        state_dtype = _GDN_DTYPE[state_dtype]
    d = GdnTreeDesc()
    d.batch, d.n_nodes, d.n_k_heads, d.n_v_heads = batch, n_nodes, n_k_heads, n_v_heads
    d.d_k, d.d_v, d.scale = d_k, d_v, float(scale)
    d.qkv_dtype, d.state_dtype, d.flags = int(qkv_dtype), int(state_dtype), int(flags)
    d.status = _ptr(status, "status") if status is not None else None
    return d


def make_build_desc(*, batch: int, max_depth: int, top_k: int, budget: int, flags: int = 0,
                    status: Optional[torch.Tensor] = None) -> GdnBuildDesc:
    d = GdnBuildDesc()
    d.batch, d.max_depth, d.top_k, d.budget, d.flags = batch, max_depth, top_k, budget, int(flags)
    d.status = _ptr(status, "status") if status is not None else None
    return d


def _ptr(x, name: str):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, torch.Tensor):
        if not x.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor (got device {x.device})")
        if not x.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        return x.data_ptr()
    raise TypeError(f"{name}: expected a CUDA tensor, an int device pointer or None")


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, check: bool) -> int:
    if check and rc != GDN_OK:
        raise GdnError(rc, load_library().gdn_last_error_detail().decode())
    return rc


def gdn_status_str(status: int) -> str:
    return load_library().gdn_status_str(int(status)).decode()


def gdn_version() -> str:
    return load_library().gdn_version().decode()


def gdn_node_states_bytes(desc: GdnTreeDesc) -> int:
    return int(load_library().gdn_node_states_bytes(ctypes.byref(desc)))


def gdn_tree_verify(desc: GdnTreeDesc, q, k, v, g, beta, parent_idx, state_in, out, node_states,
                    stream=None, check: bool = True) -> int:
    """Calls gdn_tree_verify (see include/gdntree.h).  Raises GdnError on a
    non-OK host status when ``check``; device-detected errors go to desc.status."""
    lib = load_library()
    rc = lib.gdn_tree_verify(ctypes.byref(desc), _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"),
                             _ptr(g, "g"), _ptr(beta, "beta"), _ptr(parent_idx, "parent_idx"),
                             _ptr(state_in, "state_in"), _ptr(out, "out"),
                             _ptr(node_states, "node_states"), _stream(stream))
    return _check(rc, check)


def gdn_tree_verify_workspace_bytes(desc: GdnTreeDesc) -> int:
    return int(load_library().gdn_tree_verify_workspace_bytes(ctypes.byref(desc)))


def gdn_tree_verify_ws(desc: GdnTreeDesc, q, k, v, g, beta, parent_idx, state_in, out, node_states,
                       workspace, workspace_bytes: Optional[int] = None, stream=None, check: bool = True) -> int:
    """Calls gdn_tree_verify_ws (see include/gdntree.h).  ``workspace_bytes``
    defaults to the tensor's size in bytes."""
    lib = load_library()
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size() if isinstance(workspace, torch.Tensor) else 0
    rc = lib.gdn_tree_verify_ws(ctypes.byref(desc), _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"),
                                _ptr(g, "g"), _ptr(beta, "beta"), _ptr(parent_idx, "parent_idx"),
                                _ptr(state_in, "state_in"), _ptr(out, "out"),
                                _ptr(node_states, "node_states"), _ptr(workspace, "workspace"),
                                int(workspace_bytes), _stream(stream))
    return _check(rc, check)


def gdn_static_workspace_capacity() -> int:
    return int(load_library().gdn_static_workspace_capacity())


def gdn_tree_verify_static_ws(desc: GdnTreeDesc, q, k, v, g, beta, parent_idx, state_in, out, node_states,
                              stream=None, check: bool = True) -> int:
    """Calls gdn_tree_verify_static_ws (see include/gdntree.h): the library's
    static device workspace, shared by every call on the device."""
    lib = load_library()
    rc = lib.gdn_tree_verify_static_ws(ctypes.byref(desc), _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"),
                                       _ptr(g, "g"), _ptr(beta, "beta"), _ptr(parent_idx, "parent_idx"),
                                       _ptr(state_in, "state_in"), _ptr(out, "out"),
                                       _ptr(node_states, "node_states"), _stream(stream))
    return _check(rc, check)


def gdn_tree_commit(desc: GdnTreeDesc, node_states, parent_idx, accept_path, accept_len,
                    max_path_len: int, state_out, stream=None, check: bool = True) -> int:
    """Calls gdn_tree_commit (see include/gdntree.h)."""
    lib = load_library()
    rc = lib.gdn_tree_commit(ctypes.byref(desc), _ptr(node_states, "node_states"),
                             _ptr(parent_idx, "parent_idx"), _ptr(accept_path, "accept_path"),
                             _ptr(accept_len, "accept_len"), int(max_path_len),
                             _ptr(state_out, "state_out"), _stream(stream))
    return _check(rc, check)


def gdn_tree_commit_layers(desc: GdnTreeDesc, node_states, parent_idx, accept_path, accept_len,
                           max_path_len: int, state_out, stream=None, check: bool = True) -> int:
    """Calls gdn_tree_commit_layers (see include/gdntree.h): ``node_states`` and
    ``state_out`` are equal-length sequences of per-layer CUDA tensors (or int
    device pointers)."""
    lib = load_library()
    if len(node_states) != len(state_out):
        raise ValueError("node_states and state_out must have one entry per layer")
    n = len(node_states)
    ns = (ctypes.c_void_p * max(n, 1))(*[_ptr(t, "node_states") for t in node_states])
    so = (ctypes.c_void_p * max(n, 1))(*[_ptr(t, "state_out") for t in state_out])
    rc = lib.gdn_tree_commit_layers(ctypes.byref(desc), n, ns, _ptr(parent_idx, "parent_idx"),
                                    _ptr(accept_path, "accept_path"), _ptr(accept_len, "accept_len"),
                                    int(max_path_len), so, _stream(stream))
    return _check(rc, check)


def gdn_tree_verify_varlen(desc: GdnTreeDesc, cu_nodes, total_nodes: int, q, k, v, g, beta, parent_idx, state_in,
                           out, node_states, workspace=None, workspace_bytes: Optional[int] = None, stream=None,
                           check: bool = True) -> int:
    """Calls gdn_tree_verify_varlen (see include/gdntree.h): trees of
    different sizes packed along the node dimension."""
    lib = load_library()
    if workspace_bytes is None:
        workspace_bytes = workspace.numel() * workspace.element_size() if isinstance(workspace, torch.Tensor) else 0
    rc = lib.gdn_tree_verify_varlen(ctypes.byref(desc), _ptr(cu_nodes, "cu_nodes"), int(total_nodes),
                                    _ptr(q, "q"), _ptr(k, "k"), _ptr(v, "v"), _ptr(g, "g"), _ptr(beta, "beta"),
                                    _ptr(parent_idx, "parent_idx"), _ptr(state_in, "state_in"), _ptr(out, "out"),
                                    _ptr(node_states, "node_states"), _ptr(workspace, "workspace"),
                                    int(workspace_bytes), _stream(stream))
    return _check(rc, check)


def gdn_tree_commit_varlen(desc: GdnTreeDesc, cu_nodes, total_nodes: int, node_states, parent_idx, accept_path,
                           accept_len, max_path_len: int, state_out, stream=None, check: bool = True) -> int:
    """Calls gdn_tree_commit_varlen: ``node_states`` and ``state_out`` are
    equal-length sequences of per-layer CUDA tensors (or int pointers)."""
    lib = load_library()
    if len(node_states) != len(state_out):
        raise ValueError("node_states and state_out must have one entry per layer")
    n = len(node_states)
    ns = (ctypes.c_void_p * max(n, 1))(*[_ptr(t, "node_states") for t in node_states])
    so = (ctypes.c_void_p * max(n, 1))(*[_ptr(t, "state_out") for t in state_out])
    rc = lib.gdn_tree_commit_varlen(ctypes.byref(desc), _ptr(cu_nodes, "cu_nodes"), int(total_nodes), n, ns,
                                    _ptr(parent_idx, "parent_idx"), _ptr(accept_path, "accept_path"),
                                    _ptr(accept_len, "accept_len"), int(max_path_len), so, _stream(stream))
    return _check(rc, check)


def gdn_build_tree(desc: GdnBuildDesc, logp, parent_idx, topk_ids=None, node_depth=None, node_rank=None,
                   node_token=None, node_score=None, stream=None, check: bool = True) -> int:
    """Calls gdn_build_tree (see include/gdntree.h)."""
    lib = load_library()
    rc = lib.gdn_build_tree(ctypes.byref(desc), _ptr(logp, "logp"), _ptr(topk_ids, "topk_ids"),
                            _ptr(parent_idx, "parent_idx"), _ptr(node_depth, "node_depth"),
                            _ptr(node_rank, "node_rank"), _ptr(node_token, "node_token"),
                            _ptr(node_score, "node_score"), _stream(stream))
    return _check(rc, check)


def gdn_tree_compact(src, parent_idx, accept_path, accept_len, dst, *, batch: int, n_nodes: int,
                     row_bytes: Optional[int] = None, max_path_len: Optional[int] = None, cu_nodes=None,
                     total_nodes: int = 0, status=None, stream=None, check: bool = True) -> int:
    """Calls gdn_tree_compact (see include/gdntree.h).  ``row_bytes``
    defaults to dst's bytes per (sequence, path position), ``max_path_len``
    to accept_path's second dimension."""
    lib = load_library()
    if row_bytes is None:
        row_bytes = dst[0, 0].numel() * dst.element_size()
    if max_path_len is None:
        max_path_len = accept_path.shape[1]
    rc = lib.gdn_tree_compact(int(batch), int(n_nodes), _ptr(cu_nodes, "cu_nodes"), int(total_nodes),
                              int(row_bytes), _ptr(src, "src"), _ptr(parent_idx, "parent_idx"),
                              _ptr(accept_path, "accept_path"), _ptr(accept_len, "accept_len"),
                              int(max_path_len), _ptr(dst, "dst"), _ptr(status, "status"), _stream(stream))
    return _check(rc, check)


def gdn_tree_plan_bytes(desc: GdnTreeDesc) -> int:
    return int(load_library().gdn_tree_plan_bytes(ctypes.byref(desc)))


def _nbytes(t, given):
    if given is not None:
        return int(given)
    return t.numel() * t.element_size() if isinstance(t, torch.Tensor) else 0


def gdn_tree_plan(desc: GdnTreeDesc, parent_idx, plan, plan_bytes: Optional[int] = None, stream=None,
                  check: bool = True) -> int:
    """Calls gdn_tree_plan (see include/gdntree.h)."""
    rc = load_library().gdn_tree_plan(ctypes.byref(desc), _ptr(parent_idx, "parent_idx"), _ptr(plan, "plan"),
                                      _nbytes(plan, plan_bytes), _stream(stream))
    return _check(rc, check)


def gdn_tree_verify_planned(desc: GdnTreeDesc, plan, q, k, v, g, beta, parent_idx, state_in, out, node_states,
                            plan_bytes: Optional[int] = None, stream=None, check: bool = True) -> int:
    """Calls gdn_tree_verify_planned (see include/gdntree.h)."""
    rc = load_library().gdn_tree_verify_planned(
        ctypes.byref(desc), _ptr(plan, "plan"), _nbytes(plan, plan_bytes), _ptr(q, "q"), _ptr(k, "k"),
        _ptr(v, "v"), _ptr(g, "g"), _ptr(beta, "beta"), _ptr(parent_idx, "parent_idx"),
        _ptr(state_in, "state_in"), _ptr(out, "out"), _ptr(node_states, "node_states"), _stream(stream))
    return _check(rc, check)
