// Internal declarations shared by the host entry points and the kernels of
// libgdntree.  Not part of the public ABI (see include/gdntree.h).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "gdntree.h"

namespace gdn {

// Device-side status written when a bounded wait on a shared-memory barrier
// runs out (an internal error: the kernel then stops early).
constexpr int32_t kStatusTimeout = 6;

// Launch geometry of the verify kernels, chosen by the host.
struct VerifyGeom {
    bool staged;          // whole-tree staging kernel (else the producer/ring kernel)
    bool warp_tree;       // staged tree walked from warp registers (N <= 32)
    bool reload;          // branch parents re-read from f32 node_states (no stack)
    bool gslots;          // stack slots in the caller's workspace (global memory)
    bool tslots;          // stack slots in tensor memory (the wide kernel)
    int tmem_cols;        // tslots: tensor-memory columns allocated per CTA
    int tmem_slot_cols;   // tslots: columns from one slot to the next
    size_t ws_bytes;      // workspace the launch needs (gslots), else 0
    int chunks;           // lane shape: chunks of 8 state columns per lane and row (1 or 2)
    int rows_per_lane;    // lane shape: rows per lane (1 or 2)
    int warps;            // compute warps per CTA (the ring kernel adds a producer warp)
    int rows;             // d_v rows per CTA
    int tiles;            // d_v / rows
    int slots;            // f32 parent-state stack slots
    uint32_t raw_bytes;   // one node's record: k row | q row | v slice, input type
    uint32_t off_raw, off_desc, off_ab, off_slots, off_tree;  // shared-memory layout
    size_t smem;          // dynamic shared memory bytes
};

struct VerifyArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* g;
    const float* beta;
    const int32_t* parent;
    const float* state_in;
    float* out;
    void* node_states;
    int32_t* status;
    int batch, n_nodes, n_k_heads, n_v_heads, d_k, d_v;
    float scale;
    int qkv_dtype, state_dtype;
    uint32_t flags;
    float* workspace;  // optional: stack slots in global memory
    const int32_t* cu_nodes;  // optional (varlen): [batch + 1] node offsets; n_nodes = the most per sequence
    int total_nodes;          // varlen: cu_nodes[batch]
    const int32_t* plan;      // optional: walks from gdn_tree_plan
};

// Layout of a tree plan (gdn_tree_plan) for a verify call's geometry: whether
// the call's walk kind uses one (trees walked with stack slots), the int32
// per sequence, and the signature each sequence's header carries.
struct PlanGeom {
    bool needed;
    bool warp_kind;  // MaskTree (<= 32 nodes, staged) else TreeView arrays
    int slots, n_nodes, stride, sig;
};
PlanGeom plan_geometry(const VerifyArgs& a);
cudaError_t launch_plan(const VerifyArgs& a, const PlanGeom& pg, int32_t* plan, cudaStream_t stream);

// Layers one commit launch covers (more are split over several launches).
constexpr int kMaxCommitLayers = 64;

struct CommitArgs {
    int n_layers;
    const void* const* node_states;  // host array [n_layers] of device pointers
    float* const* state_out;         // host array [n_layers] of device pointers
    const int32_t* parent;
    const int32_t* accept_path;
    const int32_t* accept_len;
    int32_t* status;
    int batch, n_nodes, n_v_heads, d_k, d_v, max_path_len;
    int state_dtype;
    uint32_t flags;
    const int32_t* cu_nodes;  // optional (varlen), as in VerifyArgs
    int total_nodes;
};

// Launches kernel(args...) with programmatic stream serialization allowed (see
// pdl_wait_then_release in gdn_device.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Pick the launch geometry for a verify call (host only, no CUDA calls).
// With use_workspace, walks that keep stack slots keep them in global memory
// (VerifyGeom::gslots, ws_bytes).
VerifyGeom verify_geometry(const VerifyArgs& a, bool use_workspace);

// Launch the verify / commit kernels.  Return cudaSuccess or the launch error.
cudaError_t launch_verify(const VerifyArgs& a, const VerifyGeom& geom, cudaStream_t stream);
cudaError_t launch_commit(const CommitArgs& a, cudaStream_t stream);

// Chains in chunks on the tensor cores (GDN_FLAG_CHUNKED): whether a call's
// shapes are supported, and the launch.
bool chunked_supported(const VerifyArgs& a);
cudaError_t launch_chunked(const VerifyArgs& a, cudaStream_t stream);

// Best-first draft-tree construction (gdn_build_tree), checked by the host.
struct BuildArgs {
    const float* logp;
    const int32_t* topk_ids;
    int32_t* parent;
    int32_t* depth;
    int32_t* rank;
    int32_t* token;
    float* score;
    int32_t* status;
    int batch, max_depth, top_k, budget;
    uint32_t flags;
};

cudaError_t launch_build_tree(const BuildArgs& a, cudaStream_t stream);

}  // namespace gdn
