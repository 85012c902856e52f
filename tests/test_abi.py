"""The C-ABI library loads, exports what include/gdntree.h declares, and its
host-side checks reject bad calls before launching anything (no GPU needed:
every call here fails validation or has batch 0, so no kernel is launched)."""
import ctypes

import pytest

import gated_deltanet_tree_verify_b200 as gdn
from gated_deltanet_tree_verify_b200.build import build
from gated_deltanet_tree_verify_b200.gdntree import header_functions


@pytest.fixture(scope="module")
def lib():
    build()
    return gdn.load_library()


def test_exports_every_declared_function(lib):
    names = header_functions()
    assert {"gdn_tree_verify", "gdn_tree_commit", "gdn_status_str"} <= set(names)
    for name in names:
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in [(0, "GDN_OK"), (1, "GDN_ERR_INVALID_ARG"), (2, "GDN_ERR_UNSUPPORTED"),
                       (3, "GDN_ERR_BAD_TREE"), (4, "GDN_ERR_BAD_PATH"), (5, "GDN_ERR_CUDA"),
                       (6, "GDN_ERR_TIMEOUT"), (7, "GDN_ERR_BAD_INPUT")]:
        assert gdn.gdn_status_str(code) == name
    assert gdn.gdn_status_str(99) == "GDN_ERR_UNKNOWN"


def test_desc_struct_layout():
    # int32 x 6, float, int32 x 2, uint32, pointer
    assert ctypes.sizeof(gdn.GdnTreeDesc) == 48
    assert gdn.GdnTreeDesc.status.offset == 40


def _desc(**kw):
    base = dict(batch=1, n_nodes=23, n_k_heads=16, n_v_heads=48, d_k=128, d_v=128, scale=0.0884,
                qkv_dtype=gdn.GDN_BF16, state_dtype=gdn.GDN_F32, flags=0)
    base.update(kw)
    return gdn.make_desc(**base)


def test_node_states_bytes(lib):
    assert gdn.gdn_node_states_bytes(_desc()) == 23 * 48 * 128 * 128 * 4
    assert gdn.gdn_node_states_bytes(_desc(state_dtype=gdn.GDN_F16, batch=3)) == 3 * 23 * 48 * 128 * 128 * 2
    assert gdn.gdn_node_states_bytes(_desc(flags=gdn.GDN_FLAG_PERSIST_LAST | gdn.GDN_FLAG_CHAIN,
                                           n_nodes=4096, batch=8)) == 8 * 48 * 128 * 128 * 4
    assert gdn.gdn_node_states_bytes(_desc(d_k=48)) == 0


# Fake, well-separated, aligned device addresses: validation runs on the host and
# these calls never reach a launch.
BASE = 1 << 40
MB = 1 << 30


def _ptrs(n=10):
    return [BASE + i * MB for i in range(n)]


def _verify(desc, ptrs=None):
    q, k, v, g, beta, par, sin, out, ns = (ptrs or _ptrs())[:9]
    return gdn.gdn_tree_verify(desc, q, k, v, g, beta, par, sin, out, ns, stream=0, check=False)


def test_verify_batch_zero_is_a_noop(lib):
    assert _verify(_desc(batch=0)) == gdn.GDN_OK


@pytest.mark.parametrize("kw,code", [
    (dict(d_k=48), gdn.GDN_ERR_UNSUPPORTED),
    (dict(d_v=256), gdn.GDN_ERR_UNSUPPORTED),
    (dict(n_v_heads=40), gdn.GDN_ERR_INVALID_ARG),
    (dict(n_nodes=0), gdn.GDN_ERR_INVALID_ARG),
    (dict(batch=-1), gdn.GDN_ERR_INVALID_ARG),
    (dict(n_nodes=gdn.GDN_MAX_TREE_NODES + 1), gdn.GDN_ERR_UNSUPPORTED),
    (dict(qkv_dtype=gdn.GDN_F16), gdn.GDN_ERR_UNSUPPORTED),
    (dict(state_dtype=gdn.GDN_BF16), gdn.GDN_ERR_UNSUPPORTED),
    (dict(flags=128), gdn.GDN_ERR_INVALID_ARG),     # no such flag
    (dict(flags=16 | 2 | 32 | 64), gdn.GDN_ERR_UNSUPPORTED),  # chunked with the fused steps, no CHAIN
    (dict(flags=16), gdn.GDN_ERR_UNSUPPORTED),      # chunked needs CHAIN + PERSIST_LAST
    (dict(flags=16 | 1 | 2, d_v=32), gdn.GDN_ERR_UNSUPPORTED),
    (dict(scale=float("nan")), gdn.GDN_ERR_INVALID_ARG),
])
def test_verify_rejects_bad_desc(lib, kw, code):
    assert _verify(_desc(**kw)) == code


def test_fused_gates_flag_passes_the_host_checks(lib):
    assert gdn.GDN_FLAG_GATES == 64
    for f in (gdn.GDN_FLAG_GATES, gdn.GDN_FLAG_GATES | gdn.GDN_FLAG_QK_L2NORM,
              gdn.GDN_FLAG_GATES | gdn.GDN_FLAG_CHAIN | gdn.GDN_FLAG_PERSIST_LAST):
        assert _verify(_desc(batch=0, flags=f)) == gdn.GDN_OK


def test_verify_rejects_null_desc(lib):
    p = _ptrs()
    rc = lib.gdn_tree_verify(None, *p[:9], None)
    assert rc == gdn.GDN_ERR_INVALID_ARG


def test_verify_null_and_misaligned_pointers(lib):
    for i in range(9):
        p = _ptrs()
        if i == 5:  # parent_idx may be NULL only in chain mode
            p[i] = None
            assert _verify(_desc(), p) == gdn.GDN_ERR_INVALID_ARG
            continue
        p[i] = None
        assert _verify(_desc(), p) == gdn.GDN_ERR_INVALID_ARG, i
    for i, align in [(0, 16), (1, 16), (2, 16), (6, 32), (7, 16), (8, 32), (3, 4), (4, 4), (5, 4)]:
        p = _ptrs()
        p[i] += align // 2
        assert _verify(_desc(), p) == gdn.GDN_ERR_INVALID_ARG, i
    assert "misaligned" in lib.gdn_last_error_detail().decode()


def test_verify_rejects_overlapping_outputs(lib):
    p = _ptrs()
    p[7] = p[8] + 64  # out inside node_states
    assert _verify(_desc(), p) == gdn.GDN_ERR_INVALID_ARG
    p = _ptrs()
    p[8] = p[6]  # node_states on top of state_in
    assert _verify(_desc(), p) == gdn.GDN_ERR_INVALID_ARG
    assert "state_in" in lib.gdn_last_error_detail().decode()


def test_chain_mode_parent_may_be_null_but_not_with_validate(lib):
    p = _ptrs()
    p[5] = None
    # passes every host check, so use batch 0 to stay off the GPU
    assert _verify(_desc(batch=0, flags=gdn.GDN_FLAG_CHAIN), p) == gdn.GDN_OK
    assert _verify(_desc(flags=gdn.GDN_FLAG_CHAIN | gdn.GDN_FLAG_VALIDATE), p) == gdn.GDN_ERR_INVALID_ARG


def _commit(desc, ptrs=None, max_path_len=17):
    ns, par, ap, al, so = (ptrs or _ptrs(5))[:5]
    return gdn.gdn_tree_commit(desc, ns, par, ap, al, max_path_len, so, stream=0, check=False)


def test_commit_host_checks(lib):
    assert _commit(_desc(batch=0)) == gdn.GDN_OK
    assert _commit(_desc(), max_path_len=0) == gdn.GDN_ERR_INVALID_ARG
    assert _commit(_desc(d_k=16)) == gdn.GDN_ERR_UNSUPPORTED
    p = _ptrs(5)
    p[1] = None
    assert _commit(_desc(), p) == gdn.GDN_ERR_INVALID_ARG
    p = _ptrs(5)
    p[4] = p[0] + 256  # state_out inside node_states
    assert _commit(_desc(), p) == gdn.GDN_ERR_INVALID_ARG
    p = _ptrs(5)
    p[4] += 8
    assert _commit(_desc(), p) == gdn.GDN_ERR_INVALID_ARG


def test_binding_refuses_host_tensors(lib):
    import torch
    t = torch.zeros(16)
    with pytest.raises(ValueError):
        gdn.gdn_tree_verify(_desc(), t, t, t, t, t, t, t, t, t, stream=0)


def _commit_layers(desc, ns, so, max_path_len=17, par=BASE + 60 * MB, ap=BASE + 61 * MB, al=BASE + 62 * MB):
    return gdn.gdn_tree_commit_layers(desc, ns, par, ap, al, max_path_len, so, stream=0, check=False)


def test_commit_layers_host_checks(lib):
    ns = [BASE + i * MB for i in range(3)]
    so = [BASE + (10 + i) * MB for i in range(3)]
    assert _commit_layers(_desc(batch=0), ns, so) == gdn.GDN_OK
    assert _commit_layers(_desc(), [], []) == gdn.GDN_OK          # no layers: nothing to do
    assert lib.gdn_tree_commit_layers(ctypes.byref(_desc()), -1, None, BASE, BASE, BASE, 4, None,
                                      None) == gdn.GDN_ERR_INVALID_ARG
    assert _commit_layers(_desc(), ns, [so[0], 0, so[2]]) == gdn.GDN_ERR_INVALID_ARG
    assert _commit_layers(_desc(), ns, [so[0], so[1] + 8, so[2]]) == gdn.GDN_ERR_INVALID_ARG
    assert _commit_layers(_desc(), ns, [so[0], so[0] + 1024, so[2]]) == gdn.GDN_ERR_INVALID_ARG
    assert "overlap" in lib.gdn_last_error_detail().decode()
    assert _commit_layers(_desc(), ns, [so[0], ns[2] + 4096, so[2]]) == gdn.GDN_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        gdn.gdn_tree_commit_layers(_desc(), ns, 0, 0, 0, 4, so[:2], stream=0)


def test_verify_workspace_bytes(lib):
    # f16 tree: B * Hv * dv * dk * 4 bytes per stack slot, floor(log2 N) slots capped at 4
    d = _desc(state_dtype=gdn.GDN_F16)                      # N = 23: 4 slots
    assert gdn.gdn_tree_verify_workspace_bytes(d) == 48 * 128 * 128 * 4 * 4
    assert gdn.gdn_tree_verify_workspace_bytes(_desc(state_dtype=gdn.GDN_F16, n_nodes=3)) == 48 * 128 * 128 * 4
    assert gdn.gdn_tree_verify_workspace_bytes(_desc(state_dtype=gdn.GDN_F16, batch=3, n_nodes=129)) == \
        3 * 48 * 128 * 128 * 4 * 4
    # f32 trees re-read branch states from node_states, except trees above 32
    # nodes on large grids (two rows per lane), which keep slots; chains keep none
    assert gdn.gdn_tree_verify_workspace_bytes(_desc()) == 0
    assert gdn.gdn_tree_verify_workspace_bytes(_desc(batch=8, n_nodes=32)) == 0
    assert gdn.gdn_tree_verify_workspace_bytes(_desc(batch=1, n_nodes=65)) == 0
    assert gdn.gdn_tree_verify_workspace_bytes(_desc(batch=8, n_nodes=65)) == 8 * 48 * 128 * 128 * 4 * 4
    assert gdn.gdn_tree_verify_workspace_bytes(_desc(state_dtype=gdn.GDN_F16, flags=gdn.GDN_FLAG_CHAIN)) == 0
    assert gdn.gdn_tree_verify_workspace_bytes(_desc(flags=gdn.GDN_FLAG_PERSIST_LAST)) > 0
    assert gdn.gdn_tree_verify_workspace_bytes(_desc(d_k=48)) == 0


def _verify_ws(desc, ws, nbytes, ptrs=None):
    q, k, v, g, beta, par, sin, out, ns = (ptrs or _ptrs())[:9]
    return gdn.gdn_tree_verify_ws(desc, q, k, v, g, beta, par, sin, out, ns, ws, nbytes, stream=0, check=False)


def test_verify_ws_host_checks(lib):
    d = _desc(state_dtype=gdn.GDN_F16)
    need = gdn.gdn_tree_verify_workspace_bytes(d)
    ws = BASE + 20 * MB
    assert _verify_ws(d, ws, need - 1) == gdn.GDN_ERR_INVALID_ARG
    assert "workspace" in lib.gdn_last_error_detail().decode()
    assert _verify_ws(d, ws + 8, need) == gdn.GDN_ERR_INVALID_ARG      # misaligned
    assert _verify_ws(_desc(batch=0, state_dtype=gdn.GDN_F16), ws, 0) == gdn.GDN_OK
    p = _ptrs()
    assert _verify_ws(d, p[8] + 64, need, p) == gdn.GDN_ERR_INVALID_ARG  # inside node_states
    assert _verify_ws(d, p[0], need, p) == gdn.GDN_ERR_INVALID_ARG       # on top of q


def test_varlen_host_checks(lib):
    d = _desc(batch=3)
    q, k, v, g, beta, par, sin, out, ns = _ptrs(9)
    cu = BASE + 30 * MB

    def call(desc, cu_ptr, total):
        return gdn.gdn_tree_verify_varlen(desc, cu_ptr, total, q, k, v, g, beta, par, sin, out, ns, None, 0,
                                          stream=0, check=False)
    assert call(d, None, 10) == gdn.GDN_ERR_INVALID_ARG          # no offsets
    assert call(d, cu + 2, 10) == gdn.GDN_ERR_INVALID_ARG        # misaligned
    assert call(d, cu, 2) == gdn.GDN_ERR_INVALID_ARG             # fewer nodes than sequences
    assert call(d, cu, 3 * 23 + 1) == gdn.GDN_ERR_INVALID_ARG    # more than batch * n_nodes
    assert call(_desc(batch=0), cu, 0) == gdn.GDN_OK
    rc = gdn.gdn_tree_commit_varlen(d, None, 10, [ns], par, BASE + 31 * MB, BASE + 32 * MB, 4, [out],
                                    stream=0, check=False)
    assert rc == gdn.GDN_ERR_INVALID_ARG


def test_build_desc_struct_layout():
    # int32 x 4, uint32, padding, pointer
    assert ctypes.sizeof(gdn.GdnBuildDesc) == 32
    assert gdn.GdnBuildDesc.status.offset == 24


def test_build_tree_host_checks(lib):
    lp, ids, par, dep, rk, tok, sc = (BASE + i * MB for i in range(7))

    def call(check_lp=lp, check_par=par, ids_=None, tok_=None, dep_=None, **kw):
        base = dict(batch=2, max_depth=16, top_k=8, budget=22, flags=0)
        base.update(kw)
        d = gdn.make_build_desc(**base)
        return gdn.gdn_build_tree(d, check_lp, check_par, topk_ids=ids_, node_depth=dep_, node_token=tok_,
                                  stream=0, check=False)
    assert call(batch=0) == gdn.GDN_OK
    assert call(batch=0, budget=23, max_depth=2, top_k=2) == gdn.GDN_ERR_INVALID_ARG   # 2 + 4 = 6 candidates
    assert call(batch=0, budget=6, max_depth=2, top_k=2) == gdn.GDN_OK
    assert call(flags=4) == gdn.GDN_ERR_INVALID_ARG
    assert call(max_depth=0) == gdn.GDN_ERR_INVALID_ARG
    assert call(budget=-1) == gdn.GDN_ERR_INVALID_ARG
    assert call(max_depth=256) == gdn.GDN_ERR_UNSUPPORTED
    assert call(max_depth=128, top_k=64) == gdn.GDN_ERR_UNSUPPORTED              # D * K above 4096
    assert call(budget=1024) == gdn.GDN_ERR_UNSUPPORTED
    assert call(check_lp=None) == gdn.GDN_ERR_INVALID_ARG
    assert call(check_par=None) == gdn.GDN_ERR_INVALID_ARG
    assert call(tok_=tok) == gdn.GDN_ERR_INVALID_ARG                             # tokens need topk_ids
    assert call(check_par=par + 2) == gdn.GDN_ERR_INVALID_ARG                     # misaligned
    assert call(dep_=par + 4) == gdn.GDN_ERR_INVALID_ARG                          # outputs overlap
    assert call(check_par=lp + 64) == gdn.GDN_ERR_INVALID_ARG                     # output inside logp
    assert call(ids_=ids, tok_=ids + 4) == gdn.GDN_ERR_INVALID_ARG                # output inside topk_ids


def test_compact_host_checks(lib):
    src, par, path, ln, dst, cu = (BASE + i * MB for i in range(6))

    def call(**kw):
        base = dict(batch=2, n_nodes=23, row_bytes=24576, max_path_len=17)
        args = dict(src=src, par=par, path=path, ln=ln, dst=dst)
        for k in list(kw):
            if k in args:
                args[k] = kw.pop(k)
        base.update(kw)
        return gdn.gdn_tree_compact(args["src"], args["par"], args["path"], args["ln"], args["dst"], stream=0,
                                    check=False, **base)
    assert call(batch=0) == gdn.GDN_OK
    assert call(batch=-1) == gdn.GDN_ERR_INVALID_ARG
    assert call(row_bytes=24) == gdn.GDN_ERR_INVALID_ARG          # not a multiple of 16
    assert call(max_path_len=0) == gdn.GDN_ERR_INVALID_ARG
    assert call(src=None) == gdn.GDN_ERR_INVALID_ARG
    assert call(dst=dst + 8) == gdn.GDN_ERR_INVALID_ARG          # misaligned
    assert call(ln=ln + 2) == gdn.GDN_ERR_INVALID_ARG
    assert call(dst=src + 4096) == gdn.GDN_ERR_INVALID_ARG       # overlaps src
    assert call(cu_nodes=cu, total_nodes=1) == gdn.GDN_ERR_INVALID_ARG  # fewer nodes than sequences
    assert call(cu_nodes=cu, total_nodes=47) == gdn.GDN_ERR_INVALID_ARG  # above batch * n_nodes


def test_plan_bytes_and_host_checks(lib):
    f16 = _desc(state_dtype=gdn.GDN_F16, batch=8, n_nodes=65)
    need = gdn.gdn_tree_plan_bytes(f16)
    assert need > 0 and need % 16 == 0
    assert gdn.gdn_tree_plan_bytes(_desc(batch=8, n_nodes=23)) == 0            # f32 trees re-read parents
    assert gdn.gdn_tree_plan_bytes(_desc(batch=8, n_nodes=65)) > 0             # ... except large ones on large grids
    assert gdn.gdn_tree_plan_bytes(_desc(flags=gdn.GDN_FLAG_CHAIN, state_dtype=gdn.GDN_F16)) == 0
    assert gdn.gdn_tree_plan_bytes(_desc(d_k=48)) == 0
    par, plan = BASE, BASE + 4 * MB
    assert gdn.gdn_tree_plan(f16, par, plan, need - 16, stream=0, check=False) == gdn.GDN_ERR_INVALID_ARG
    assert gdn.gdn_tree_plan(f16, par, plan + 8, need, stream=0, check=False) == gdn.GDN_ERR_INVALID_ARG
    assert gdn.gdn_tree_plan(f16, None, plan, need, stream=0, check=False) == gdn.GDN_ERR_INVALID_ARG
    assert gdn.gdn_tree_plan(f16, par, par, need, stream=0, check=False) == gdn.GDN_ERR_INVALID_ARG  # overlap
    # nothing to build: fine with no buffer at all
    assert gdn.gdn_tree_plan(_desc(batch=8, n_nodes=23), par, None, 0, stream=0, check=False) == gdn.GDN_OK
    q, k, v, g, beta, p_, sin, out, ns = _ptrs(9)
    rc = gdn.gdn_tree_verify_planned(f16, plan, q, k, v, g, beta, p_, sin, out, ns, plan_bytes=need - 16,
                                     stream=0, check=False)
    assert rc == gdn.GDN_ERR_INVALID_ARG
