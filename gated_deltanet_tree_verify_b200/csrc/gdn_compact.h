// Accept-time compaction (gdn_tree_compact): the launch the host entry point
// calls after checking its arguments.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

namespace gdn {

struct CompactArgs {
    const void* src;
    void* dst;
    const int32_t* parent;
    const int32_t* accept_path;
    const int32_t* accept_len;
    const int32_t* cu_nodes;  // NULL: n_nodes per sequence
    int32_t* status;
    int batch, n_nodes, total_nodes, max_path_len;
    size_t row_bytes;
};

cudaError_t launch_compact(const CompactArgs& a, cudaStream_t stream);

}  // namespace gdn
