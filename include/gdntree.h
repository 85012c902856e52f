/*
 * gdntree.h -- C ABI of libgdntree: gated-delta-rule (Gated DeltaNet) state
 * updates over a speculative-decoding draft tree, for NVIDIA B200 (sm_100a).
 *
 * The operation.  A draft tree of N nodes (node 0 is the root, i.e. the last
 * committed token re-fed through the target; nodes 1..N-1 are the drafts, so
 * N = budget + 1 as in the GreenGames post, "Key wins", where verify reads
 * budget + 1 positions) is verified in one pass.  Each node n with parent p
 * runs the gated delta rule from p's state:
 *
 *     a_n = exp(g_n)
 *     S_n = a_n * S_p + beta_n * (v_n - a_n * S_p k_n) k_n^T      (d_v x d_k)
 *     o_n = scale * S_n q_n                                          (d_v)
 *
 * (the Gated DeltaNet recurrence run by ggml_gated_delta_net, named in the
 * GreenGames post, "TL;DR" and "Why the experiment exists"; applied per tree
 * node as in the DDTree row of the dflash-caddtree-integrations README, "What's
 * in here").  The root takes S_p = state_in.  Every node's state is persisted
 * from inside the verify kernel (the GreenGames post, "Key wins": the kernel
 * that computes a state also writes it) in fp32 or f16 (the post's f16 cache
 * of intermediate states), so that the
 * accepted root-to-leaf path is committed by a copy, without re-running it.
 *
 * Conventions shared by every entry point:
 *   - Every data pointer is a caller-owned DEVICE pointer (cudaMalloc'd, or a
 *     framework tensor's storage).  The library allocates nothing, keeps no
 *     data between calls and never synchronises the stream.  It does remember,
 *     per device for the life of the process, that it has raised a kernel's
 *     dynamic shared-memory limit (once per kernel and device): after a
 *     cudaDeviceReset in the same process, a launch that needs more than the
 *     default 48 KB of shared memory returns GDN_ERR_CUDA instead of running
 *     (nothing is written); a new process starts afresh.
 *   - Layouts are row-major with the last index contiguous.  B = batch
 *     (independent sequences), N = n_nodes, H_k / H_v = k-heads / v-heads with
 *     G = H_v / H_k; v-head h reads k-head h / G (contiguous groups).
 *   - Calls are asynchronous on `stream`.  The returned status reports only
 *     what the host can check (arguments, shapes, alignment, overlap of
 *     outputs with inputs, launch errors).  Errors in device data (a bad tree,
 *     a bad accept path) are reported through desc->status, see below.
 *   - Pointers passed for q, k, v, out and state_out must be 16-byte
 *     aligned; state_in and node_states 32-byte aligned for gdn_tree_verify
 *     (states move in 32-byte accesses) and 16-byte aligned for the commit
 *     calls; g, beta, parent_idx, accept_path and accept_len 4-byte aligned.
 */
#ifndef GDNTREE_H
#define GDNTREE_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element types. */
typedef enum {
    GDN_F32 = 0,
    GDN_F16 = 1,
    GDN_BF16 = 2
} gdn_dtype;

/* Status codes (host return values and device-side desc->status words). */
typedef enum {
    GDN_OK = 0,
    GDN_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned or overlapping buffers */
    GDN_ERR_UNSUPPORTED = 2,  /* a shape or dtype the library has no kernel for */
    GDN_ERR_BAD_TREE = 3,     /* device-detected: parent[0] != -1 or parent[n] not in [0, n) */
    GDN_ERR_BAD_PATH = 4,     /* device-detected: accept path/length violates the tree */
    GDN_ERR_CUDA = 5,         /* a CUDA call failed; gdn_last_error_detail() says which */
    GDN_ERR_TIMEOUT = 6,      /* device-detected internal error: a bounded wait on an
                                 on-chip barrier ran out and the kernel stopped early */
    GDN_ERR_BAD_INPUT = 7     /* device-detected: input values break the call's contract
                                 (gdn_build_tree with GDN_BUILD_VALIDATE) */
} gdn_status;

/* desc->flags bits. */
enum {
    /* The caller asserts parent[n] = n - 1 (a DFlash chain).  Same numerics as
     * the tree path; skips the tree walk.  parent_idx may then be NULL. */
    GDN_FLAG_CHAIN = 1,
    /* Persist only the state of the LAST node (n = N - 1); node_states then
     * holds one state per sequence, [B][1][H_v][d_v][d_k].  Meant for long
     * chains (prefill-style).  Commit then accepts only paths that end at
     * node N - 1. */
    GDN_FLAG_PERSIST_LAST = 2,
    /* In chain mode, check parent[n] = n - 1 on the device (needs parent_idx).
     * The tree path always checks its tree. */
    GDN_FLAG_VALIDATE = 4,
    /* Verify only.  The caller asserts that parent_idx and state_in were
     * written before the kernel that precedes this call in the stream was
     * launched (e.g. the draft tree is built once per step, the recurrent
     * state by the previous step's commit, and this is any layer but the
     * first of a layer stack).  The kernels are launched with programmatic
     * dependent launch; with this flag they read parent_idx and state_in and
     * build the tree walk while the preceding kernel may still run, and wait
     * for it only before reading q, k, v, g, beta.  Without the flag every
     * global read waits for the preceding kernel to complete. */
    GDN_FLAG_EARLY_TREE = 8,
    /* Chains only (with GDN_FLAG_CHAIN and GDN_FLAG_PERSIST_LAST, bf16 q/k/v,
     * d_k = 128, d_v a multiple of 64, no varlen or workspace): run the chain
     * in chunks of 64 tokens with tensor-core products (the chunked "WY" form
     * of the delta rule), for long prefill-style chains.  Results agree with
     * the token-by-token path to within a few times its f32 rounding error
     * (products of bf16 parts accumulated in f32), not bit-identically.  q, k, v and out are read and
     * written through TMA tensor maps (the 16-byte alignment required above
     * suffices).  Unsupported shapes: GDN_ERR_UNSUPPORTED. */
    GDN_FLAG_CHUNKED = 16,
    /* q and k are given raw; the kernel L2-normalises each (node, k-head)
     * row, x / |x| with no epsilon (a zero row gives inf/NaN), as the
     * workloads' input preparation does.  Folded into per-node scalars, so
     * the node loop does the same work.  Also with GDN_FLAG_CHUNKED. */
    GDN_FLAG_QK_L2NORM = 32,
    /* g and beta are given raw: they hold the pre-activations x and y of the
     * gates g = -softplus(x) = -log(1 + e^x) and beta = sigmoid(y), the
     * workloads' gate recipe, and the kernels apply both (as
     * a = exp(g) = 1 / (1 + e^x) and beta = 1 / (1 + e^-y), in f32, once per
     * node).  x = +inf gives a = 0 (a reset).  Also with GDN_FLAG_CHUNKED. */
    GDN_FLAG_GATES = 64
};

/* Problem description, shared by verify and commit. */
typedef struct gdn_tree_desc {
    int32_t batch;       /* B >= 0 sequences (0: the call does nothing) */
    int32_t n_nodes;     /* N >= 1 tree nodes per sequence, root included */
    int32_t n_k_heads;   /* H_k >= 1 */
    int32_t n_v_heads;   /* H_v >= 1, a multiple of H_k */
    int32_t d_k;         /* key/query head dim: 32, 64 or 128 */
    int32_t d_v;         /* value head dim: 32, 64 or 128 */
    float scale;         /* output scale, usually 1/sqrt(d_k) */
    int32_t qkv_dtype;   /* gdn_dtype of q, k, v: GDN_BF16 or GDN_F32 */
    int32_t state_dtype; /* gdn_dtype of node_states: GDN_F32 or GDN_F16 */
    uint32_t flags;      /* GDN_FLAG_* bits */
    int32_t* status;     /* optional DEVICE int32.  A kernel that finds an error
                            in device data stores its gdn_status here with an
                            atomic compare-and-swap from 0 (the first error
                            sticks; the library never clears it) and writes
                            nothing for the affected sequence.  NULL: such
                            sequences are skipped silently. */
} gdn_tree_desc;

/*
 * gdn_tree_verify -- run every tree node from its parent's state, emit o_n and
 * persist S_n.
 *
 *   q, k        [B][N][H_k][d_k]    qkv_dtype (bf16 or f32), read-only
 *   v           [B][N][H_v][d_v]    qkv_dtype, read-only
 *   g, beta     [B][N][H_v]         f32, read-only; a_n = exp(g_n), g = -inf resets
 *                                   (with GDN_FLAG_GATES the raw x, y of
 *                                   g = -softplus(x), beta = sigmoid(y))
 *   parent_idx  [B][N]              int32, parent[b][0] = -1 and
 *                                   0 <= parent[b][n] < n; may be NULL only
 *                                   with GDN_FLAG_CHAIN and without VALIDATE
 *   state_in    [B][H_v][d_v][d_k]  f32, read-only; the root's parent state
 *   out         [B][N][H_v][d_v]    f32, written: o_n
 *   node_states [B][N][H_v][d_v][d_k] in state_dtype, written: S_n rounded to
 *               nearest even (f16 or exact f32).  With GDN_FLAG_PERSIST_LAST:
 *               [B][1][H_v][d_v][d_k], node N - 1 only.
 *
 * Children always continue from their parent's unrounded fp32 state, never
 * from the f16 copy.  Trees: N <= GDN_MAX_TREE_NODES unless GDN_FLAG_CHAIN;
 * any depth.  Results for a node depend only on its own root path: they do
 * not change when other branches are added, removed or renumbered.
 *
 * Buffers: out and node_states must not overlap each other or any input.
 * Errors: GDN_ERR_INVALID_ARG / GDN_ERR_UNSUPPORTED / GDN_ERR_CUDA from the
 * host (nothing launched); GDN_ERR_BAD_TREE through desc->status.
 */
gdn_status gdn_tree_verify(const gdn_tree_desc* desc, const void* q, const void* k,
                           const void* v, const float* g, const float* beta,
                           const int32_t* parent_idx, const float* state_in, float* out,
                           void* node_states, cudaStream_t stream);

/*
 * gdn_tree_verify_ws -- gdn_tree_verify with a caller-owned device workspace
 * for the walk's stack of branch states.
 *
 * A tree walk keeps the f32 states of branching nodes until their later
 * children run: with state_dtype f16, with GDN_FLAG_PERSIST_LAST, and with
 * f32 trees above 32 nodes on large grids, not packed (elsewhere an f32 walk
 * re-reads parent states from node_states and needs no workspace).  Without a
 * workspace they live in shared memory, which caps the resident CTAs per SM
 * for trees above ~32 nodes; with one they live in global memory (mostly
 * L2), each loaded one node ahead of its use.  Results are bit-identical
 * either way (the walk order and arithmetic do not change).
 *
 *   workspace        DEVICE buffer, 16-byte aligned, or NULL (then exactly
 *                    gdn_tree_verify); contents on entry are ignored and on
 *                    return undefined; it must not overlap any other buffer
 *                    of the call, and a call in flight owns it
 *   workspace_bytes  its size; at least gdn_tree_verify_workspace_bytes(desc)
 *                    when that is nonzero (else GDN_ERR_INVALID_ARG)
 *
 * The other arguments, layouts and errors are those of gdn_tree_verify.
 * The pages define no workspace: it is this library's placement of the
 * walk's branch states, not part of the method.
 */
gdn_status gdn_tree_verify_ws(const gdn_tree_desc* desc, const void* q, const void* k,
                              const void* v, const float* g, const float* beta,
                              const int32_t* parent_idx, const float* state_in, float* out,
                              void* node_states, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream);

/*
 * gdn_tree_verify_varlen -- gdn_tree_verify(_ws) for B trees of different
 * sizes, packed along the node dimension.
 *
 *   desc->n_nodes  the most nodes any sequence has (N_max); desc->batch = B
 *   cu_nodes       DEVICE [B + 1] int32: sequence b owns packed nodes
 *                  cu_nodes[b] .. cu_nodes[b + 1] - 1, with cu_nodes[0] = 0,
 *                  1 <= cu_nodes[b + 1] - cu_nodes[b] <= N_max and
 *                  cu_nodes[B] = total_nodes (a sequence whose entries break
 *                  this gets GDN_ERR_BAD_TREE through desc->status and
 *                  nothing written)
 *   total_nodes    T, B <= T <= B * N_max (host-checked)
 *   q, k           [T][H_k][d_k];  v [T][H_v][d_v];  g, beta [T][H_v]
 *   parent_idx     [T] int32, each sequence's parents as local indices
 *                  (-1 for its root, 0 <= parent < n within the sequence)
 *   out            [T][H_v][d_v]
 *   node_states    [T][H_v][d_v][d_k] (PERSIST_LAST: [B][H_v][d_v][d_k])
 *   state_in       [B][H_v][d_v][d_k], as for gdn_tree_verify
 *   workspace      optional, as for gdn_tree_verify_ws (size from
 *                  gdn_tree_verify_workspace_bytes with the same desc)
 *
 * Results for each sequence are bit-identical to gdn_tree_verify on that
 * sequence alone.  With GDN_FLAG_EARLY_TREE, cu_nodes counts as tree data.
 */
gdn_status gdn_tree_verify_varlen(const gdn_tree_desc* desc, const int32_t* cu_nodes, int32_t total_nodes,
                                  const void* q, const void* k, const void* v, const float* g,
                                  const float* beta, const int32_t* parent_idx, const float* state_in,
                                  float* out, void* node_states, void* workspace, size_t workspace_bytes,
                                  cudaStream_t stream);

/* Workspace bytes gdn_tree_verify_ws needs for a desc: B * H_v * d_v * d_k *
 * 4 * (stack slots, at most 4) for walks that keep branch states, 0 for
 * chains, f32 trees whose walk re-reads branch states from node_states (32
 * nodes or fewer, or small grids) and invalid descs.  Computed from the desc
 * alone, so for packed trees (whose f32 walks always re-read) it can ask for
 * a workspace the call then leaves unused.  Independent of the buffers'
 * addresses. */
size_t gdn_tree_verify_workspace_bytes(const gdn_tree_desc* desc);

/*
 * gdn_tree_verify_static_ws -- gdn_tree_verify_ws without a caller
 * workspace: the library keeps one static device buffer of
 * gdn_static_workspace_capacity() bytes per device (a __device__ array,
 * resolved with cudaGetSymbolAddress on first use on each device) and
 * allocates nothing per call.  The source pages describe no counterpart; it
 * exists for callers that cannot allocate on the hot path.
 *
 * Same arguments, layouts and results as gdn_tree_verify.  When the desc
 * needs no workspace (gdn_tree_verify_workspace_bytes(desc) == 0), or more
 * than the capacity, this is gdn_tree_verify (which allocates nothing either:
 * its walks keep their branch states in shared memory or re-read parents).
 *
 * Races: the buffer is shared by every call in the process on that device.
 * Calls on one device must be ordered (one stream, or events between
 * streams); two calls in flight at once on different streams or host
 * threads overwrite each other's branch states and give wrong results.
 *
 * Memory: every CUDA context that loads the library holds the buffer's
 * 32 MiB on its device until the context ends, whether or not this entry
 * point is ever called.  The buffer's address belongs to the context: the
 * library looks it up with cudaGetSymbolAddress the first time it runs in a
 * context (identified by its driver context id), and again after the current
 * context changes (a cudaDeviceReset, or another context made current through
 * the driver API).  Make the first call on each device before capturing it
 * into a CUDA graph.
 */
gdn_status gdn_tree_verify_static_ws(const gdn_tree_desc* desc, const void* q, const void* k,
                                     const void* v, const float* g, const float* beta,
                                     const int32_t* parent_idx, const float* state_in, float* out,
                                     void* node_states, cudaStream_t stream);

/* Bytes of the static workspace behind gdn_tree_verify_static_ws. */
size_t gdn_static_workspace_capacity(void);

/*
 * gdn_tree_commit -- write the accepted path's state back as the new
 * recurrent state, without re-running the path.
 *
 *   node_states  as written by gdn_tree_verify with the same desc (state_dtype,
 *                GDN_FLAG_PERSIST_LAST)
 *   parent_idx   [B][N] int32, the tree verify ran on (may be NULL only with
 *                GDN_FLAG_CHAIN: the path is then checked against the chain)
 *   accept_path  [B][max_path_len] int32: node ids from the root, path[0] = 0
 *                and parent[path[i]] = path[i - 1]; entries past the length
 *                are ignored
 *   accept_len   [B] int32, 1 <= len <= min(N, max_path_len)
 *   state_out    [B][H_v][d_v][d_k] f32, written: the persisted state of node
 *                path[len - 1], widened to f32.  It may alias state_in of the
 *                verify call (commit reads only node_states), but must not
 *                overlap node_states.
 *
 * Errors: host-side as for verify.  Through desc->status: GDN_ERR_BAD_TREE
 * when sequence b's parent_idx is not a tree (parent[0] = -1 and
 * 0 <= parent[n] < n for every node, checked before the path), else
 * GDN_ERR_BAD_PATH when its path breaks the rules above; state_out[b] is then
 * left untouched.
 */
gdn_status gdn_tree_commit(const gdn_tree_desc* desc, const void* node_states,
                           const int32_t* parent_idx, const int32_t* accept_path,
                           const int32_t* accept_len, int32_t max_path_len, float* state_out,
                           cudaStream_t stream);

/*
 * gdn_tree_commit_layers -- gdn_tree_commit for n_layers layers in one launch
 * (an engine commits the accepted path of every GDN layer at once, after the
 * verification forward pass).  The tree, accept paths and desc are shared by
 * all layers; each layer has its own node_states and state_out.
 *
 *   n_layers     >= 0 (0: nothing to do)
 *   node_states  HOST array [n_layers] of DEVICE pointers, each as for
 *                gdn_tree_commit
 *   state_out    HOST array [n_layers] of DEVICE pointers, each as for
 *                gdn_tree_commit; no two may overlap, and none may overlap
 *                any layer's node_states
 *
 * The host arrays are read during the call only.  Errors as for
 * gdn_tree_commit (a bad path leaves every layer's state_out[b] untouched).
 */
gdn_status gdn_tree_commit_layers(const gdn_tree_desc* desc, int32_t n_layers,
                                  const void* const* node_states, const int32_t* parent_idx,
                                  const int32_t* accept_path, const int32_t* accept_len,
                                  int32_t max_path_len, float* const* state_out,
                                  cudaStream_t stream);

/*
 * gdn_tree_commit_varlen -- gdn_tree_commit_layers for the packed layout of
 * gdn_tree_verify_varlen: node_states[l] as written there, parent_idx [T]
 * local, accept_path [B][max_path_len] local node ids, the same cu_nodes and
 * total_nodes.  A sequence with bad offsets gets GDN_ERR_BAD_TREE and its
 * state_out is left untouched.
 */
gdn_status gdn_tree_commit_varlen(const gdn_tree_desc* desc, const int32_t* cu_nodes, int32_t total_nodes,
                                  int32_t n_layers, const void* const* node_states, const int32_t* parent_idx,
                                  const int32_t* accept_path, const int32_t* accept_len, int32_t max_path_len,
                                  float* const* state_out, cudaStream_t stream);

/*
 * gdn_tree_compact -- accept-time compaction: carry only the accepted path's
 * per-node rows forward, in path order (the target-feature compaction after
 * a sibling accept, the GreenGames post, "Key wins").  For every sequence b
 * whose path checks against its tree (path[0] = 0, parent[path[i]] =
 * path[i-1], 1 <= accept_len[b] <= min(max_path_len, N_b)):
 *
 *     dst[b][i] = src[n0_b + accept_path[b][i]]      for i < accept_len[b]
 *
 *   src          [T][row_bytes] per-node rows (outputs, features, states...;
 *                the bytes are copied as they are), T = B * n_nodes, or the
 *                packed varlen total.  Read-only.
 *   cu_nodes     NULL (every sequence has n_nodes nodes), or [B + 1] device
 *                int32 offsets as for gdn_tree_verify_varlen (n_nodes is then
 *                the most per sequence, total_nodes = cu_nodes[B])
 *   parent_idx   [T] int32, each sequence's parents as local indices
 *   accept_path  [B][max_path_len] int32, accept_len [B] int32
 *   dst          [B][max_path_len][row_bytes]; rows at i >= accept_len[b]
 *                are left untouched
 *   status       optional device int32: GDN_ERR_BAD_PATH (or
 *                GDN_ERR_BAD_TREE for bad offsets); that sequence's dst rows
 *                are left untouched
 * row_bytes a positive multiple of 16; src and dst 16-byte aligned, the int32
 * arrays 4-byte aligned; dst must not overlap any input.  Errors:
 * GDN_ERR_INVALID_ARG / GDN_ERR_UNSUPPORTED / GDN_ERR_CUDA from the host.
 */
gdn_status gdn_tree_compact(int32_t batch, int32_t n_nodes, const int32_t* cu_nodes, int32_t total_nodes,
                            size_t row_bytes, const void* src, const int32_t* parent_idx,
                            const int32_t* accept_path, const int32_t* accept_len, int32_t max_path_len,
                            void* dst, int32_t* status, cudaStream_t stream);

/*
 * Tree plans.  Every layer of a model verifies the same tree, and the walk
 * the kernels take through it (a depth-first order, which nodes keep their
 * state for later siblings, which re-derive it) depends only on the tree and
 * the launch shape.  gdn_tree_plan builds it once per step (one CTA per
 * sequence) into a caller-owned device buffer; gdn_tree_verify_planned then
 * copies it instead of building it in every CTA of every layer.  A
 * data-layout convenience of this library: the source pages describe no
 * counterpart.
 *
 * gdn_tree_plan_bytes(desc): bytes of the plan for desc (the same desc as
 *   the verify calls; B sequences x a stride that depends on N and the walk
 *   kind), or 0 when the call does not read one: chains and f32 trees of
 *   at most 32 nodes (which re-read branch parents in index order, as f32
 *   trees do on small grids) build no walk, and small grids
 *   (batch x heads too small for two rows per lane) build it while the
 *   previous layer still runs (GDN_FLAG_EARLY_TREE), where it costs nothing.
 * gdn_tree_plan(desc, parent_idx, plan, plan_bytes, stream): parent_idx as
 *   for gdn_tree_verify; plan 16-byte aligned, plan_bytes >= the above.  A
 *   malformed tree gets GDN_ERR_BAD_TREE through desc->status and is marked
 *   so in the plan (the planned verify then writes nothing for it).
 * gdn_tree_verify_planned(desc, plan, plan_bytes, ...): gdn_tree_verify's
 *   arguments and results, with the walks taken from the plan, which must
 *   come from gdn_tree_plan with the same desc, parent_idx and batch (a plan
 *   built for another shape is reported as GDN_ERR_BAD_INPUT through
 *   desc->status and nothing is written).  Bit-identical to gdn_tree_verify.
 *   Not with GDN_FLAG_CHUNKED or varlen layouts.
 */
size_t gdn_tree_plan_bytes(const gdn_tree_desc* desc);
gdn_status gdn_tree_plan(const gdn_tree_desc* desc, const int32_t* parent_idx, void* plan, size_t plan_bytes,
                         cudaStream_t stream);
gdn_status gdn_tree_verify_planned(const gdn_tree_desc* desc, const void* plan, size_t plan_bytes, const void* q,
                                   const void* k, const void* v, const float* g, const float* beta,
                                   const int32_t* parent_idx, const float* state_in, float* out,
                                   void* node_states, cudaStream_t stream);

/* Largest N the tree (non-chain) path takes. */
#define GDN_MAX_TREE_NODES 1024

/* gdn_build_desc.flags bits. */
enum {
    /* Take the greedy chain (rank 0 at every position, min(max_depth, budget)
     * nodes) first, then fill the rest of the budget best-first (the chain
     * pre-seed of build_ddtree, the GreenGames post, "From autoregressive to
     * DDTree"). */
    GDN_BUILD_CHAIN_SEED = 1,
    /* Check on the device that every logp row is non-increasing and holds no
     * NaN or +inf; a sequence that fails gets GDN_ERR_BAD_INPUT through
     * status and none of its outputs are written. */
    GDN_BUILD_VALIDATE = 2
};

/* Problem description of gdn_build_tree. */
typedef struct gdn_build_desc {
    int32_t batch;      /* B >= 0 sequences (0: the call does nothing) */
    int32_t max_depth;  /* D, draft positions: 1..255 */
    int32_t top_k;      /* K, candidates per position: 1..255; D * K <= 4096 */
    int32_t budget;     /* drafts per tree, 0..GDN_MAX_TREE_NODES - 1 and at most
                           the K + K^2 + .. + K^D nodes the candidates span;
                           the tree has N = budget + 1 nodes */
    uint32_t flags;     /* GDN_BUILD_* bits */
    int32_t* status;    /* optional DEVICE int32, as gdn_tree_desc.status */
} gdn_build_desc;

/*
 * gdn_build_tree -- best-first draft tree from the drafter's top-k candidates
 * (build_ddtree, the GreenGames post, "From autoregressive to DDTree"; rank 0
 * is each position's best candidate, "Key wins").
 *
 * A node is a sequence of ranks (r_1 .. r_d), d <= D; node 0 is the root
 * (d = 0, score 0).  Its score is the float32 sum, accumulated from the root
 * (score(child) = score(parent) + logp[d - 1][r_d], rounded to nearest), and
 * the budget nodes taken are picked one at a time among the children of the
 * nodes taken so far: highest score first, then lower depth, lower rank,
 * lower parent index.  Each taken node gets the next index, so the output is
 * a tree in the layout gdn_tree_verify reads (parent[0] = -1, parent[n] < n).
 *
 *   logp        [B][D][K] f32, each row non-increasing (rank 0 best), no NaN;
 *               -inf allowed.  Read-only.
 *   topk_ids    [B][D][K] int32 token ids of the candidates, or NULL
 *   parent_idx  [B][N] int32 out
 *   node_depth  [B][N] int32 out, d (0 for the root), or NULL
 *   node_rank   [B][N] int32 out, r_d (0 for the root), or NULL
 *   node_token  [B][N] int32 out, topk_ids[b][d - 1][r_d] (-1 for the root),
 *               or NULL; needs topk_ids
 *   node_score  [B][N] f32 out, the node's score, or NULL
 *
 * One warp per tree; all pointers 4-byte aligned device memory; outputs must
 * not overlap each other or the inputs.  Errors: GDN_ERR_INVALID_ARG /
 * GDN_ERR_UNSUPPORTED / GDN_ERR_CUDA from the host (nothing launched);
 * GDN_ERR_BAD_INPUT through desc->status (GDN_BUILD_VALIDATE).  Rows that are
 * not non-increasing without GDN_BUILD_VALIDATE give a valid tree that may
 * differ from the rule above.
 */
gdn_status gdn_build_tree(const gdn_build_desc* desc, const float* logp, const int32_t* topk_ids,
                          int32_t* parent_idx, int32_t* node_depth, int32_t* node_rank, int32_t* node_token,
                          float* node_score, cudaStream_t stream);

/* Bytes of node_states for a desc (B * N * H_v * d_v * d_k * element size, or
 * N replaced by 1 with GDN_FLAG_PERSIST_LAST); 0 for an invalid desc. */
size_t gdn_node_states_bytes(const gdn_tree_desc* desc);

/* Static, human-readable name of a status code. */
const char* gdn_status_str(gdn_status s);

/* Detail of the last GDN_ERR_* returned on this host thread (static or
 * thread-local storage; valid until the next call on the same thread). */
const char* gdn_last_error_detail(void);

/* Library version, e.g. "0.1.0". */
const char* gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDNTREE_H */
