"""libgdntree for NVIDIA B200 (sm_100a): gated-delta-rule state updates over a
speculative-decoding draft tree, with per-node state persistence and commit.

The compute lives in the CUDA library lib/libgdntree.so (C ABI in
include/gdntree.h); this package is its thin ctypes binding.
"""
from .gdntree import (  # noqa: F401
    GDN_BF16, GDN_BUILD_CHAIN_SEED, GDN_BUILD_VALIDATE, GDN_ERR_BAD_INPUT, GDN_ERR_BAD_PATH, GDN_ERR_BAD_TREE, GDN_ERR_CUDA, GDN_ERR_INVALID_ARG,
    GDN_ERR_TIMEOUT, GDN_ERR_UNSUPPORTED, GDN_F16, GDN_F32, GDN_FLAG_CHAIN, GDN_FLAG_CHUNKED, GDN_FLAG_GATES, GDN_FLAG_QK_L2NORM,
    GDN_FLAG_EARLY_TREE, GDN_FLAG_PERSIST_LAST, GDN_FLAG_VALIDATE, GDN_MAX_TREE_NODES, GDN_OK, GdnError,
    GdnBuildDesc, GdnLibraryMissing, GdnTreeDesc, gdn_build_tree, make_build_desc, gdn_node_states_bytes, gdn_tree_commit_varlen, gdn_tree_verify_varlen, gdn_static_workspace_capacity, gdn_status_str, gdn_tree_commit, gdn_tree_commit_layers, gdn_tree_compact, gdn_tree_plan, gdn_tree_plan_bytes, gdn_tree_verify_planned,
    gdn_tree_verify, gdn_tree_verify_static_ws, gdn_tree_verify_workspace_bytes, gdn_tree_verify_ws, gdn_version, load_library, make_desc,
)
