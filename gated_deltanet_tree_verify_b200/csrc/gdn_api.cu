// gdn_api.cu -- the extern "C" entry points of libgdntree: host-side argument
// checks, then one kernel launch on the caller's stream.  See include/gdntree.h
// for the contract of each call.

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda_runtime.h>

#include "gdn_compact.h"
#include "gdn_internal.h"
#include "gdntree.h"

namespace {

thread_local char g_detail[256] = "";

gdn_status fail(gdn_status s, const char* fmt, const char* what = "")
{
    std::snprintf(g_detail, sizeof(g_detail), fmt, what);
    return s;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Range {
    const void* p;
    size_t bytes;
    const char* name;
};

bool overlap(const Range& x, const Range& y)
{
    if (x.p == nullptr || y.p == nullptr || x.bytes == 0 || y.bytes == 0)
        return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(x.p), a1 = a0 + x.bytes;
    const uintptr_t b0 = reinterpret_cast<uintptr_t>(y.p), b1 = b0 + y.bytes;
    return a0 < b1 && b0 < a1;
}

size_t elem_size(int dt) { return dt == GDN_F32 ? 4 : 2; }

// Shape/dtype checks shared by verify and commit.
gdn_status check_desc(const gdn_tree_desc* d, bool need_qkv)
{
    if (d == nullptr)
        return fail(GDN_ERR_INVALID_ARG, "desc is NULL%s");
    if (d->batch < 0 || d->n_nodes < 1 || d->n_k_heads < 1 || d->n_v_heads < 1)
        return fail(GDN_ERR_INVALID_ARG, "batch, n_nodes or head counts out of range%s");
    if (d->n_v_heads % d->n_k_heads != 0)
        return fail(GDN_ERR_INVALID_ARG, "n_v_heads is not a multiple of n_k_heads%s");
    if ((d->flags & ~127u) != 0)
        return fail(GDN_ERR_INVALID_ARG, "unknown flag bits%s");
    const bool dk_ok = d->d_k == 32 || d->d_k == 64 || d->d_k == 128;
    const bool dv_ok = d->d_v == 32 || d->d_v == 64 || d->d_v == 128;
    if (!dk_ok || !dv_ok)
        return fail(GDN_ERR_UNSUPPORTED, "d_k and d_v must each be 32, 64 or 128%s");
    if (d->state_dtype != GDN_F32 && d->state_dtype != GDN_F16)
        return fail(GDN_ERR_UNSUPPORTED, "state_dtype must be GDN_F32 or GDN_F16%s");
    if (need_qkv) {
        if (d->qkv_dtype != GDN_BF16 && d->qkv_dtype != GDN_F32)
            return fail(GDN_ERR_UNSUPPORTED, "qkv_dtype must be GDN_BF16 or GDN_F32%s");
        if (!std::isfinite(d->scale))
            return fail(GDN_ERR_INVALID_ARG, "scale is not finite%s");
    }
    if (!(d->flags & GDN_FLAG_CHAIN) && d->n_nodes > GDN_MAX_TREE_NODES)
        return fail(GDN_ERR_UNSUPPORTED, "tree has more than GDN_MAX_TREE_NODES nodes%s");
    if (d->n_nodes > 0xffff)
        return fail(GDN_ERR_UNSUPPORTED, "n_nodes above 65535%s");
    return GDN_OK;
}

size_t node_states_bytes(const gdn_tree_desc* d)
{
    const size_t ns = (d->flags & GDN_FLAG_PERSIST_LAST) ? 1 : (size_t)d->n_nodes;
    return (size_t)d->batch * ns * d->n_v_heads * d->d_v * d->d_k * elem_size(d->state_dtype);
}

// Nodes of the node dimension: B N, or the varlen total.
size_t total_nodes(const gdn_tree_desc& d, const int32_t* cu, int32_t total)
{
    return cu ? (size_t)total : (size_t)d.batch * d.n_nodes;
}

// node_states bytes for a fixed or varlen layout.
size_t node_states_bytes_v(const gdn_tree_desc& d, const int32_t* cu, int32_t total)
{
    const size_t ns = (d.flags & GDN_FLAG_PERSIST_LAST) ? (size_t)d.batch : total_nodes(d, cu, total);
    return ns * d.n_v_heads * d.d_v * d.d_k * elem_size(d.state_dtype);
}

// Host checks of the varlen arguments (cu_nodes itself is device memory;
// the kernels check its entries).
gdn_status check_varlen(const gdn_tree_desc& d, const int32_t* cu, int32_t total)
{
    if (!cu)
        return fail(GDN_ERR_INVALID_ARG, "cu_nodes is NULL%s");
    if (!aligned(cu, 4))
        return fail(GDN_ERR_INVALID_ARG, "cu_nodes is misaligned%s");
    if (total < d.batch || (long long)total > (long long)d.batch * d.n_nodes)
        return fail(GDN_ERR_INVALID_ARG, "total_nodes outside [batch, batch * n_nodes]%s");
    return GDN_OK;
}

}  // namespace

extern "C" {

const char* gdn_version(void) { return "0.1.0"; }

const char* gdn_last_error_detail(void) { return g_detail; }

const char* gdn_status_str(gdn_status s)
{
    switch (s) {
        case GDN_OK: return "GDN_OK";
        case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
        case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
        case GDN_ERR_BAD_TREE: return "GDN_ERR_BAD_TREE";
        case GDN_ERR_BAD_PATH: return "GDN_ERR_BAD_PATH";
        case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
        case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
        case GDN_ERR_BAD_INPUT: return "GDN_ERR_BAD_INPUT";
    }
    return "GDN_ERR_UNKNOWN";
}

size_t gdn_node_states_bytes(const gdn_tree_desc* desc)
{
    if (check_desc(desc, false) != GDN_OK)
        return 0;
    return node_states_bytes(desc);
}

}  // extern "C"

namespace {

// VerifyArgs for a desc and buffers (no checks).
gdn::VerifyArgs verify_args(const gdn_tree_desc& d)
{
    gdn::VerifyArgs a{};
    a.status = d.status;
    a.batch = d.batch;
    a.n_nodes = d.n_nodes;
    a.n_k_heads = d.n_k_heads;
    a.n_v_heads = d.n_v_heads;
    a.d_k = d.d_k;
    a.d_v = d.d_v;
    a.scale = d.scale;
    a.qkv_dtype = d.qkv_dtype;
    a.state_dtype = d.state_dtype;
    a.flags = d.flags;
    return a;
}

gdn_status verify_impl(const gdn_tree_desc* desc, const int32_t* cu, int32_t total, const void* q,
                       const void* k, const void* v, const float* g, const float* beta,
                       const int32_t* parent_idx, const float* state_in, float* out, void* node_states,
                       void* workspace, size_t workspace_bytes, cudaStream_t stream, bool varlen,
                       const void* plan = nullptr, size_t plan_bytes = 0)
{
    g_detail[0] = '\0';
    gdn_status st = check_desc(desc, true);
    if (st != GDN_OK)
        return st;
    const gdn_tree_desc& d = *desc;
    if (varlen && (st = check_varlen(d, cu, total)) != GDN_OK)
        return st;
    const bool chain = (d.flags & GDN_FLAG_CHAIN) != 0;
    const bool need_parent = !chain || (d.flags & GDN_FLAG_VALIDATE);
    if (!q || !k || !v || !g || !beta || !state_in || !out || !node_states || (need_parent && !parent_idx))
        return fail(GDN_ERR_INVALID_ARG, "a required pointer is NULL%s");
    const struct { const void* p; size_t a; const char* n; } al[] = {
        {q, 16, "q"}, {k, 16, "k"}, {v, 16, "v"}, {state_in, 32, "state_in"}, {out, 16, "out"},
        {node_states, 32, "node_states"}, {g, 4, "g"}, {beta, 4, "beta"}, {parent_idx, 4, "parent_idx"},
        {d.status, 4, "status"}, {workspace, 16, "workspace"}};
    for (const auto& x : al)
        if (x.p && !aligned(x.p, x.a))
            return fail(GDN_ERR_INVALID_ARG, "%s is misaligned", x.n);
    if (d.batch == 0)
        return GDN_OK;
    gdn::VerifyArgs a = verify_args(d);
    a.q = q;
    a.k = k;
    a.v = v;
    a.g = g;
    a.beta = beta;
    a.parent = parent_idx;
    a.state_in = state_in;
    a.out = out;
    a.node_states = node_states;
    a.workspace = static_cast<float*>(workspace);
    a.cu_nodes = varlen ? cu : nullptr;
    a.total_nodes = varlen ? total : 0;
    if (d.flags & GDN_FLAG_CHUNKED) {
        if (varlen || workspace != nullptr || !gdn::chunked_supported(a))
            return fail(GDN_ERR_UNSUPPORTED,
                        "GDN_FLAG_CHUNKED needs CHAIN + PERSIST_LAST, bf16 q/k/v, d_k = 128, d_v %% 64 == 0%s");
        const size_t B = d.batch, N = d.n_nodes, Hk = d.n_k_heads, Hv = d.n_v_heads, dk = d.d_k, dv = d.d_v;
        const Range ins[] = {{q, B * N * Hk * dk * 2, "q"}, {k, B * N * Hk * dk * 2, "k"},
                             {v, B * N * Hv * dv * 2, "v"}, {g, B * N * Hv * 4, "g"},
                             {beta, B * N * Hv * 4, "beta"}, {state_in, B * Hv * dv * dk * 4, "state_in"}};
        const Range outs[] = {{out, B * N * Hv * dv * 4, "out"}, {node_states, node_states_bytes(&d), "node_states"}};
        if (overlap(outs[0], outs[1]))
            return fail(GDN_ERR_INVALID_ARG, "out overlaps node_states%s");
        for (const auto& o : outs)
            for (const auto& i : ins)
                if (overlap(o, i))
                    return fail(GDN_ERR_INVALID_ARG, "an output overlaps input %s", i.name);
        if (d.n_v_heads > 65535 || d.batch > 65535)
            return fail(GDN_ERR_UNSUPPORTED, "batch or n_v_heads above the grid limit%s");
        const cudaError_t e = gdn::launch_chunked(a, stream);
        if (e != cudaSuccess)
            return fail(GDN_ERR_CUDA, "verify launch failed: %s", cudaGetErrorString(e));
        return GDN_OK;
    }
    const gdn::VerifyGeom geom = gdn::verify_geometry(a, workspace != nullptr);
    if (geom.tiles <= 0 || geom.smem > 227 * 1024)
        return fail(GDN_ERR_UNSUPPORTED, "no launch geometry for this shape%s");
    size_t plan_need = 0;
    if (plan != nullptr) {
        const gdn::PlanGeom pg = gdn::plan_geometry(a);
        if (pg.needed) {
            plan_need = (size_t)d.batch * pg.stride * 4;
            if (!aligned(plan, 16) || plan_bytes < plan_need)
                return fail(GDN_ERR_INVALID_ARG, "plan misaligned or smaller than gdn_tree_plan_bytes()%s");
            a.plan = static_cast<const int32_t*>(plan);
        }
    }
    if (d.n_v_heads > 65535 || d.batch > 65535)
        return fail(GDN_ERR_UNSUPPORTED, "batch or n_v_heads above the grid limit%s");
    if (geom.gslots && workspace_bytes < geom.ws_bytes)
        return fail(GDN_ERR_INVALID_ARG, "workspace smaller than gdn_tree_verify_workspace_bytes()%s");

    const size_t B = d.batch, T = total_nodes(d, a.cu_nodes, total), Hk = d.n_k_heads, Hv = d.n_v_heads,
                 dk = d.d_k, dv = d.d_v;
    const size_t es = elem_size(d.qkv_dtype);
    const Range ins[] = {{q, T * Hk * dk * es, "q"},     {k, T * Hk * dk * es, "k"},
                         {v, T * Hv * dv * es, "v"},     {g, T * Hv * 4, "g"},
                         {beta, T * Hv * 4, "beta"},     {parent_idx, T * 4, "parent_idx"},
                         {state_in, B * Hv * dv * dk * 4, "state_in"},
                         {d.status, 4, "status"},       {a.cu_nodes, (B + 1) * 4, "cu_nodes"},
                         {a.plan, plan_need, "plan"}};
    const Range outs[] = {{out, T * Hv * dv * 4, "out"},
                          {node_states, node_states_bytes_v(d, a.cu_nodes, total), "node_states"},
                          {geom.gslots ? workspace : nullptr, geom.ws_bytes, "workspace"}};
    for (int i = 0; i < 3; ++i)
        for (int j = i + 1; j < 3; ++j)
            if (overlap(outs[i], outs[j]))
                return fail(GDN_ERR_INVALID_ARG, "%s overlaps another output", outs[j].name);
    for (const auto& o : outs)
        for (const auto& i : ins)
            if (overlap(o, i))
                return fail(GDN_ERR_INVALID_ARG, "an output overlaps input %s", i.name);
    const cudaError_t e = gdn::launch_verify(a, geom, stream);
    if (e != cudaSuccess)
        return fail(GDN_ERR_CUDA, "verify launch failed: %s", cudaGetErrorString(e));
    return GDN_OK;
}

}  // namespace

extern "C" {

gdn_status gdn_tree_verify(const gdn_tree_desc* desc, const void* q, const void* k, const void* v,
                           const float* g, const float* beta, const int32_t* parent_idx,
                           const float* state_in, float* out, void* node_states,
                           cudaStream_t stream)
{
    return verify_impl(desc, nullptr, 0, q, k, v, g, beta, parent_idx, state_in, out, node_states, nullptr, 0, stream,
                       false);
}

gdn_status gdn_tree_verify_ws(const gdn_tree_desc* desc, const void* q, const void* k, const void* v,
                              const float* g, const float* beta, const int32_t* parent_idx,
                              const float* state_in, float* out, void* node_states, void* workspace,
                              size_t workspace_bytes, cudaStream_t stream)
{
    return verify_impl(desc, nullptr, 0, q, k, v, g, beta, parent_idx, state_in, out, node_states, workspace,
                       workspace_bytes, stream, false);
}

gdn_status gdn_tree_verify_varlen(const gdn_tree_desc* desc, const int32_t* cu_nodes, int32_t total_nodes,
                                  const void* q, const void* k, const void* v, const float* g,
                                  const float* beta, const int32_t* parent_idx, const float* state_in,
                                  float* out, void* node_states, void* workspace, size_t workspace_bytes,
                                  cudaStream_t stream)
{
    return verify_impl(desc, cu_nodes, total_nodes, q, k, v, g, beta, parent_idx, state_in, out, node_states,
                       workspace, workspace_bytes, stream, true);
}

size_t gdn_tree_verify_workspace_bytes(const gdn_tree_desc* desc)
{
    if (check_desc(desc, true) != GDN_OK)
        return 0;
    const gdn::VerifyGeom geom = gdn::verify_geometry(verify_args(*desc), true);
    return geom.tiles > 0 ? geom.ws_bytes : 0;
}

}  // extern "C"

namespace {

gdn_status commit_impl(const gdn_tree_desc* desc, const int32_t* cu, int32_t total, int32_t n_layers,
                       const void* const* node_states, const int32_t* parent_idx, const int32_t* accept_path,
                       const int32_t* accept_len, int32_t max_path_len, float* const* state_out,
                       cudaStream_t stream, bool varlen)
{
    g_detail[0] = '\0';
    gdn_status st = check_desc(desc, false);
    if (st != GDN_OK)
        return st;
    const gdn_tree_desc& d = *desc;
    if (varlen && (st = check_varlen(d, cu, total)) != GDN_OK)
        return st;
    if (!varlen)
        cu = nullptr;
    const bool chain = (d.flags & GDN_FLAG_CHAIN) != 0;
    if (n_layers < 0)
        return fail(GDN_ERR_INVALID_ARG, "n_layers < 0%s");
    if (n_layers > 0 && (!node_states || !state_out))
        return fail(GDN_ERR_INVALID_ARG, "node_states or state_out array is NULL%s");
    if (!accept_path || !accept_len || (!chain && !parent_idx))
        return fail(GDN_ERR_INVALID_ARG, "a required pointer is NULL%s");
    if (max_path_len < 1)
        return fail(GDN_ERR_INVALID_ARG, "max_path_len < 1%s");
    const struct { const void* p; size_t a; const char* n; } al[] = {
        {parent_idx, 4, "parent_idx"}, {accept_path, 4, "accept_path"}, {accept_len, 4, "accept_len"},
        {d.status, 4, "status"}};
    for (const auto& x : al)
        if (x.p && !aligned(x.p, x.a))
            return fail(GDN_ERR_INVALID_ARG, "%s is misaligned", x.n);
    for (int l = 0; l < n_layers; ++l) {
        if (!node_states[l] || !state_out[l])
            return fail(GDN_ERR_INVALID_ARG, "a per-layer pointer is NULL%s");
        if (!aligned(node_states[l], 16) || !aligned(state_out[l], 16))
            return fail(GDN_ERR_INVALID_ARG, "a per-layer pointer is misaligned%s");
    }
    if (d.batch == 0 || n_layers == 0)
        return GDN_OK;
    const size_t B = d.batch;
    const size_t so_bytes = B * d.n_v_heads * d.d_v * d.d_k * 4;
    const Range shared_in[] = {{parent_idx, total_nodes(d, cu, total) * 4, "parent_idx"},
                               {accept_path, B * (size_t)max_path_len * 4, "accept_path"},
                               {accept_len, B * 4, "accept_len"},
                               {d.status, 4, "status"},
                               {cu, (B + 1) * 4, "cu_nodes"}};
    for (int l = 0; l < n_layers; ++l) {
        const Range so{state_out[l], so_bytes, "state_out"};
        for (const auto& i : shared_in)
            if (overlap(so, i))
                return fail(GDN_ERR_INVALID_ARG, "state_out overlaps input %s", i.name);
        for (int m = 0; m < n_layers; ++m) {
            const Range ns{node_states[m], node_states_bytes_v(d, cu, total), "node_states"};
            if (overlap(so, ns))
                return fail(GDN_ERR_INVALID_ARG, "state_out overlaps node_states%s");
            if (m != l && overlap(so, Range{state_out[m], so_bytes, "state_out"}))
                return fail(GDN_ERR_INVALID_ARG, "two layers' state_out overlap%s");
        }
    }
    if (d.batch > 65535)
        return fail(GDN_ERR_UNSUPPORTED, "batch above the grid limit%s");

    gdn::CommitArgs a{};
    a.n_layers = n_layers;
    a.node_states = node_states;
    a.state_out = state_out;
    a.parent = parent_idx;
    a.accept_path = accept_path;
    a.accept_len = accept_len;
    a.status = d.status;
    a.batch = d.batch;
    a.n_nodes = d.n_nodes;
    a.n_v_heads = d.n_v_heads;
    a.d_k = d.d_k;
    a.d_v = d.d_v;
    a.max_path_len = max_path_len;
    a.state_dtype = d.state_dtype;
    a.flags = d.flags;
    a.cu_nodes = cu;
    a.total_nodes = varlen ? total : 0;
    const cudaError_t e = gdn::launch_commit(a, stream);
    if (e != cudaSuccess)
        return fail(GDN_ERR_CUDA, "commit launch failed: %s", cudaGetErrorString(e));
    return GDN_OK;
}

}  // namespace

extern "C" {

gdn_status gdn_tree_commit_layers(const gdn_tree_desc* desc, int32_t n_layers,
                                  const void* const* node_states, const int32_t* parent_idx,
                                  const int32_t* accept_path, const int32_t* accept_len,
                                  int32_t max_path_len, float* const* state_out, cudaStream_t stream)
{
    return commit_impl(desc, nullptr, 0, n_layers, node_states, parent_idx, accept_path, accept_len, max_path_len,
                       state_out, stream, false);
}

gdn_status gdn_tree_commit_varlen(const gdn_tree_desc* desc, const int32_t* cu_nodes, int32_t total_nodes,
                                  int32_t n_layers, const void* const* node_states, const int32_t* parent_idx,
                                  const int32_t* accept_path, const int32_t* accept_len, int32_t max_path_len,
                                  float* const* state_out, cudaStream_t stream)
{
    return commit_impl(desc, cu_nodes, total_nodes, n_layers, node_states, parent_idx, accept_path, accept_len,
                       max_path_len, state_out, stream, true);
}

gdn_status gdn_tree_commit(const gdn_tree_desc* desc, const void* node_states,
                           const int32_t* parent_idx, const int32_t* accept_path,
                           const int32_t* accept_len, int32_t max_path_len, float* state_out,
                           cudaStream_t stream)
{
    if (!node_states || !state_out) {
        g_detail[0] = '\0';
        const gdn_status st = check_desc(desc, false);
        if (st != GDN_OK)
            return st;
        return fail(GDN_ERR_INVALID_ARG, "a required pointer is NULL%s");
    }
    return gdn_tree_commit_layers(desc, 1, &node_states, parent_idx, accept_path, accept_len,
                                  max_path_len, &state_out, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// gdn_tree_verify_static_ws: the workspace path with a library-owned static
// device buffer, for callers that allocate nothing per call.
// ---------------------------------------------------------------------------

namespace {

constexpr size_t kStaticWorkspaceBytes = size_t(32) << 20;
constexpr int kMaxStaticDevices = 64;

// One buffer per device context, shared by every call in the process.
__device__ __align__(256) unsigned char g_static_ws[kStaticWorkspaceBytes];

// The device address of g_static_ws belongs to the context the module was
// loaded in: a cudaDeviceReset, or another context made current through the
// driver API, gives a new context with its own copy of the array.  So the
// address is cached per device together with the unique id of the context it
// was looked up in (cuCtxGetId ids are never reused within a process), and
// looked up again whenever the current context differs.  The two driver
// calls are resolved once through the runtime, so the library does not link
// libcuda itself; without them the address is looked up on every call.
using CtxGetCurrentFn = int (*)(void**);
using CtxGetIdFn = int (*)(void*, unsigned long long*);

struct StaticWsCache {
    unsigned long long ctx_id;
    void* addr;
};

std::mutex g_static_ws_lock;
StaticWsCache g_static_ws_cache[kMaxStaticDevices];
std::once_flag g_ctx_fn_once;
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

void resolve_ctx_fns()
{
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa = cudaDriverEntryPointSymbolNotFound, qb = qa;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess && qb == cudaDriverEntryPointSuccess && a && b) {
        g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(a);
        g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(b);
    }
    cudaGetLastError();  // a failed lookup leaves no sticky error behind
}

// Id of the context current on this thread; false when there is none yet or
// the driver calls are unavailable.
bool current_ctx_id(unsigned long long* id)
{
    std::call_once(g_ctx_fn_once, resolve_ctx_fns);
    if (g_ctx_get_current == nullptr)
        return false;
    void* ctx = nullptr;
    if (g_ctx_get_current(&ctx) != 0 || ctx == nullptr)
        return false;
    return g_ctx_get_id(ctx, id) == 0;
}

gdn_status static_ws_address(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return fail(GDN_ERR_CUDA, "cudaGetDevice failed: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxStaticDevices)
        return fail(GDN_ERR_UNSUPPORTED, "device ordinal above the static workspace table%s");
    unsigned long long id = 0;
    const bool have_id = current_ctx_id(&id);
    std::lock_guard<std::mutex> guard(g_static_ws_lock);
    StaticWsCache& c = g_static_ws_cache[dev];
    if (have_id && c.addr != nullptr && c.ctx_id == id) {
        *out = c.addr;
        return GDN_OK;
    }
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_ws);
    if (e != cudaSuccess)
        return fail(GDN_ERR_CUDA, "cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
    // the lookup above made the runtime's context current if none was
    if (have_id || current_ctx_id(&id)) {
        c.ctx_id = id;
        c.addr = p;
    }
    *out = p;
    return GDN_OK;
}

}  // namespace

extern "C" {

size_t gdn_static_workspace_capacity(void) { return kStaticWorkspaceBytes; }

gdn_status gdn_tree_verify_static_ws(const gdn_tree_desc* desc, const void* q, const void* k,
                                     const void* v, const float* g, const float* beta,
                                     const int32_t* parent_idx, const float* state_in, float* out,
                                     void* node_states, cudaStream_t stream)
{
    g_detail[0] = '\0';
    gdn_status st = check_desc(desc, true);
    if (st != GDN_OK)
        return st;
    // Descs whose walk needs no workspace, or more than the buffer holds, run
    // as gdn_tree_verify does (stack slots in shared memory, or parent
    // re-reads), which allocates nothing either.
    const size_t need = gdn_tree_verify_workspace_bytes(desc);
    if (need == 0 || need > kStaticWorkspaceBytes || desc->batch == 0)
        return verify_impl(desc, nullptr, 0, q, k, v, g, beta, parent_idx, state_in, out, node_states, nullptr, 0,
                           stream, false);
    void* ws = nullptr;
    st = static_ws_address(&ws);
    if (st != GDN_OK)
        return st;
    return verify_impl(desc, nullptr, 0, q, k, v, g, beta, parent_idx, state_in, out, node_states, ws,
                       kStaticWorkspaceBytes, stream, false);
}

}  // extern "C"

// ---- gdn_build_tree --------------------------------------------------------

namespace {

// K + K^2 + .. + K^D, saturated at 2^31.
long long candidate_nodes(int D, int K)
{
    long long total = 0, layer = 1;
    for (int d = 0; d < D; ++d) {
        layer *= K;
        total += layer;
        if (total >= (1ll << 31))
            return 1ll << 31;
    }
    return total;
}

}  // namespace

extern "C" {

gdn_status gdn_build_tree(const gdn_build_desc* desc, const float* logp, const int32_t* topk_ids,
                          int32_t* parent_idx, int32_t* node_depth, int32_t* node_rank, int32_t* node_token,
                          float* node_score, cudaStream_t stream)
{
    g_detail[0] = '\0';
    if (desc == nullptr)
        return fail(GDN_ERR_INVALID_ARG, "desc is NULL%s");
    const gdn_build_desc& d = *desc;
    if ((d.flags & ~3u) != 0)
        return fail(GDN_ERR_INVALID_ARG, "unknown flag bits%s");
    if (d.batch < 0 || d.max_depth < 1 || d.top_k < 1 || d.budget < 0)
        return fail(GDN_ERR_INVALID_ARG, "batch, max_depth, top_k or budget out of range%s");
    if (d.max_depth > 255 || d.top_k > 255 || d.max_depth * d.top_k > 4096)
        return fail(GDN_ERR_UNSUPPORTED, "max_depth or top_k above 255, or max_depth * top_k above 4096%s");
    if (d.budget > GDN_MAX_TREE_NODES - 1)
        return fail(GDN_ERR_UNSUPPORTED, "budget above GDN_MAX_TREE_NODES - 1%s");
    if (d.budget > candidate_nodes(d.max_depth, d.top_k))
        return fail(GDN_ERR_INVALID_ARG, "budget exceeds the nodes the candidates span%s");
    if (!logp || !parent_idx)
        return fail(GDN_ERR_INVALID_ARG, "logp or parent_idx is NULL%s");
    if (node_token && !topk_ids)
        return fail(GDN_ERR_INVALID_ARG, "node_token needs topk_ids%s");
    const struct { const void* p; const char* n; } al[] = {
        {logp, "logp"}, {topk_ids, "topk_ids"}, {parent_idx, "parent_idx"}, {node_depth, "node_depth"},
        {node_rank, "node_rank"}, {node_token, "node_token"}, {node_score, "node_score"}, {d.status, "status"}};
    for (const auto& x : al)
        if (x.p && !aligned(x.p, 4))
            return fail(GDN_ERR_INVALID_ARG, "%s is misaligned", x.n);
    if (d.batch == 0)
        return GDN_OK;
    const size_t B = d.batch, N = (size_t)d.budget + 1, cand = B * d.max_depth * d.top_k * 4;
    const Range outs[] = {{parent_idx, B * N * 4, "parent_idx"}, {node_depth, B * N * 4, "node_depth"},
                          {node_rank, B * N * 4, "node_rank"},   {node_token, B * N * 4, "node_token"},
                          {node_score, B * N * 4, "node_score"}};
    const Range ins[] = {{logp, cand, "logp"}, {topk_ids, node_token ? cand : 0, "topk_ids"}, {d.status, 4, "status"}};
    for (size_t i = 0; i < sizeof(outs) / sizeof(outs[0]); ++i) {
        for (const auto& x : ins)
            if (overlap(outs[i], x))
                return fail(GDN_ERR_INVALID_ARG, "an output overlaps input %s", x.name);
        for (size_t j = i + 1; j < sizeof(outs) / sizeof(outs[0]); ++j)
            if (overlap(outs[i], outs[j]))
                return fail(GDN_ERR_INVALID_ARG, "outputs overlap (%s)", outs[j].name);
    }

    gdn::BuildArgs a{};
    a.logp = logp;
    a.topk_ids = node_token ? topk_ids : nullptr;
    a.parent = parent_idx;
    a.depth = node_depth;
    a.rank = node_rank;
    a.token = node_token;
    a.score = node_score;
    a.status = d.status;
    a.batch = d.batch;
    a.max_depth = d.max_depth;
    a.top_k = d.top_k;
    a.budget = d.budget;
    a.flags = d.flags;
    const cudaError_t e = gdn::launch_build_tree(a, stream);
    if (e != cudaSuccess)
        return fail(GDN_ERR_CUDA, "build_tree launch failed: %s", cudaGetErrorString(e));
    return GDN_OK;
}

}  // extern "C"

// ---- gdn_tree_compact ------------------------------------------------------

extern "C" {

gdn_status gdn_tree_compact(int32_t batch, int32_t n_nodes, const int32_t* cu_nodes, int32_t total_nodes,
                            size_t row_bytes, const void* src, const int32_t* parent_idx,
                            const int32_t* accept_path, const int32_t* accept_len, int32_t max_path_len,
                            void* dst, int32_t* status, cudaStream_t stream)
{
    g_detail[0] = '\0';
    if (batch < 0 || n_nodes < 1 || max_path_len < 1)
        return fail(GDN_ERR_INVALID_ARG, "batch, n_nodes or max_path_len out of range%s");
    if (row_bytes == 0 || row_bytes % 16 != 0)
        return fail(GDN_ERR_INVALID_ARG, "row_bytes is not a positive multiple of 16%s");
    if (cu_nodes && (total_nodes < batch || (long long)total_nodes > (long long)batch * n_nodes))
        return fail(GDN_ERR_INVALID_ARG, "total_nodes outside [batch, batch * n_nodes]%s");
    if (!src || !dst || !parent_idx || !accept_path || !accept_len)
        return fail(GDN_ERR_INVALID_ARG, "a required pointer is NULL%s");
    if (!aligned(src, 16) || !aligned(dst, 16))
        return fail(GDN_ERR_INVALID_ARG, "src or dst is not 16-byte aligned%s");
    const struct { const void* p; const char* n; } al[] = {
        {cu_nodes, "cu_nodes"}, {parent_idx, "parent_idx"}, {accept_path, "accept_path"},
        {accept_len, "accept_len"}, {status, "status"}};
    for (const auto& x : al)
        if (x.p && !aligned(x.p, 4))
            return fail(GDN_ERR_INVALID_ARG, "%s is misaligned", x.n);
    if (batch == 0)
        return GDN_OK;
    if (batch > 65535)
        return fail(GDN_ERR_UNSUPPORTED, "batch above the grid limit%s");
    const size_t B = batch, T = cu_nodes ? (size_t)total_nodes : B * n_nodes;
    const size_t pieces = (row_bytes + 65535) / 65536;
    if (pieces > 65535)
        return fail(GDN_ERR_UNSUPPORTED, "row_bytes above 4 GiB%s");
    const Range out{dst, B * (size_t)max_path_len * row_bytes, "dst"};
    const Range ins[] = {{src, T * row_bytes, "src"}, {parent_idx, T * 4, "parent_idx"},
                         {accept_path, B * (size_t)max_path_len * 4, "accept_path"},
                         {accept_len, B * 4, "accept_len"}, {cu_nodes, (B + 1) * 4, "cu_nodes"},
                         {status, 4, "status"}};
    for (const auto& x : ins)
        if (overlap(out, x))
            return fail(GDN_ERR_INVALID_ARG, "dst overlaps input %s", x.name);

    gdn::CompactArgs a{};
    a.src = src;
    a.dst = dst;
    a.parent = parent_idx;
    a.accept_path = accept_path;
    a.accept_len = accept_len;
    a.cu_nodes = cu_nodes;
    a.status = status;
    a.batch = batch;
    a.n_nodes = n_nodes;
    a.total_nodes = cu_nodes ? total_nodes : batch * n_nodes;
    a.max_path_len = max_path_len;
    a.row_bytes = row_bytes;
    const cudaError_t e = gdn::launch_compact(a, stream);
    if (e != cudaSuccess)
        return fail(GDN_ERR_CUDA, "compact launch failed: %s", cudaGetErrorString(e));
    return GDN_OK;
}

}  // extern "C"

// ---- tree plans ----------------------------------------------------------

extern "C" {

size_t gdn_tree_plan_bytes(const gdn_tree_desc* desc)
{
    if (check_desc(desc, true) != GDN_OK || (desc->flags & GDN_FLAG_CHUNKED))
        return 0;
    const gdn::PlanGeom pg = gdn::plan_geometry(verify_args(*desc));
    return pg.needed ? (size_t)desc->batch * pg.stride * 4 : 0;
}

gdn_status gdn_tree_plan(const gdn_tree_desc* desc, const int32_t* parent_idx, void* plan, size_t plan_bytes,
                         cudaStream_t stream)
{
    g_detail[0] = '\0';
    gdn_status st = check_desc(desc, true);
    if (st != GDN_OK)
        return st;
    const gdn_tree_desc& d = *desc;
    if (d.flags & GDN_FLAG_CHUNKED)
        return fail(GDN_ERR_UNSUPPORTED, "chunked chains have no tree plan%s");
    const gdn::VerifyArgs a0 = verify_args(d);
    const gdn::PlanGeom pg = gdn::plan_geometry(a0);
    if (!pg.needed || d.batch == 0)
        return GDN_OK;  // this walk kind builds nothing: the plan is not read
    const size_t need = (size_t)d.batch * pg.stride * 4;
    if (!parent_idx || !plan)
        return fail(GDN_ERR_INVALID_ARG, "parent_idx or plan is NULL%s");
    if (!aligned(parent_idx, 4) || !aligned(plan, 16) || (d.status && !aligned(d.status, 4)))
        return fail(GDN_ERR_INVALID_ARG, "a pointer is misaligned%s");
    if (plan_bytes < need)
        return fail(GDN_ERR_INVALID_ARG, "plan smaller than gdn_tree_plan_bytes()%s");
    const Range pr{plan, need, "plan"};
    if (overlap(pr, Range{parent_idx, (size_t)d.batch * d.n_nodes * 4, "parent_idx"}) ||
        overlap(pr, Range{d.status, 4, "status"}))
        return fail(GDN_ERR_INVALID_ARG, "plan overlaps an input%s");
    if (d.batch > (1 << 30))
        return fail(GDN_ERR_UNSUPPORTED, "batch above the grid limit%s");
    gdn::VerifyArgs a = a0;
    a.parent = parent_idx;
    a.status = d.status;
    const cudaError_t e = gdn::launch_plan(a, pg, static_cast<int32_t*>(plan), stream);
    if (e != cudaSuccess)
        return fail(GDN_ERR_CUDA, "plan launch failed: %s", cudaGetErrorString(e));
    return GDN_OK;
}

gdn_status gdn_tree_verify_planned(const gdn_tree_desc* desc, const void* plan, size_t plan_bytes, const void* q,
                                   const void* k, const void* v, const float* g, const float* beta,
                                   const int32_t* parent_idx, const float* state_in, float* out,
                                   void* node_states, cudaStream_t stream)
{
    if (desc && (desc->flags & GDN_FLAG_CHUNKED))
        return fail(GDN_ERR_UNSUPPORTED, "chunked chains have no tree plan%s");
    return verify_impl(desc, nullptr, 0, q, k, v, g, beta, parent_idx, state_in, out, node_states, nullptr, 0,
                       stream, false, plan, plan_bytes);
}

}  // extern "C"
