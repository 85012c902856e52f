// gdn_compact.cu -- accept-time compaction of per-node rows (sm_100a).
//
// After a verify step only the accepted root-to-leaf path's per-node data
// is carried forward (the GreenGames post, "Key wins": the target features
// are compacted after a sibling branch is accepted).  For every sequence
// whose accept path checks against its tree, row path[i] of the sequence
// moves to position i of the output: dst[b][i] = src[n0_b + path_b[i]].
//
// Grid (path position, sequence, 64 KB piece of the row).  Warp 0 of every
// CTA checks the sequence's node range and path (a few loads; the same
// checks as the commit kernel) while the other threads wait at a barrier;
// then the CTA copies its piece of one row with 16-byte loads and stores.

#include <cstdint>

#include <cuda_runtime.h>

#include "gdn_compact.h"
#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kCompactThreads = 128;
constexpr size_t kCompactPiece = 64 * 1024;  // bytes of a row per CTA

struct XParams {
    const uint4* src;
    uint4* dst;
    const int32_t* parent;
    const int32_t* accept_path;
    const int32_t* accept_len;
    const int32_t* cu;
    int32_t* status;
    int N, total, P;
    size_t row_vec;  // 16-byte vectors per row
};

__global__ void __launch_bounds__(kCompactThreads) gdn_compact_kernel(XParams p)
{
    __shared__ int s_ok, s_n0, s_node;
    pdl_wait_then_release();
    const int i = blockIdx.x, b = blockIdx.y;
    const int tid = threadIdx.x;
    if (tid < 32) {
        // node range of the sequence
        int n0 = b * p.N, nb = p.N;
        bool ok = true;
        if (p.cu != nullptr) {
            n0 = __ldg(p.cu + b);
            nb = __ldg(p.cu + b + 1) - n0;
            ok = n0 >= 0 && nb >= 1 && nb <= p.N && n0 <= p.total - nb;
        }
        const int len = __ldg(p.accept_len + b);
        ok = ok && len >= 1 && len <= p.P && len <= nb;
        const int32_t* path = p.accept_path + (size_t)b * p.P;
        bool bad = false;
        if (ok) {
            for (int j = tid; j < len; j += 32) {
                const int x = __ldg(path + j);
                if (j == 0)
                    bad |= x != 0;
                else
                    bad |= x < 1 || x >= nb || __ldg(p.parent + (size_t)n0 + x) != __ldg(path + j - 1);
            }
        }
        ok = ok && !__any_sync(0xffffffffu, bad);
        if (tid == 0) {
            s_ok = ok ? (i < len ? 1 : 2) : 0;
            s_n0 = n0;
            s_node = (ok && i < len) ? __ldg(path + i) : 0;
            if (!ok && i == 0 && blockIdx.z == 0)
                report_status(p.status, p.cu != nullptr && !(n0 >= 0 && nb >= 1 && nb <= p.N && n0 <= p.total - nb)
                                            ? GDN_ERR_BAD_TREE
                                            : GDN_ERR_BAD_PATH);
        }
    }
    __syncthreads();
    if (s_ok != 1)
        return;  // a bad path (nothing written for the sequence), or past its end
    const size_t piece = kCompactPiece / 16;
    const size_t v0 = (size_t)blockIdx.z * piece;
    const size_t v1 = min(v0 + piece, p.row_vec);
    const uint4* src = p.src + ((size_t)s_n0 + s_node) * p.row_vec;
    uint4* dst = p.dst + ((size_t)b * p.P + i) * p.row_vec;
    for (size_t v = v0 + tid; v < v1; v += kCompactThreads)
        dst[v] = __ldg(src + v);
}

}  // namespace

cudaError_t launch_compact(const CompactArgs& a, cudaStream_t stream)
{
    XParams p{};
    p.src = static_cast<const uint4*>(a.src);
    p.dst = static_cast<uint4*>(a.dst);
    p.parent = a.parent;
    p.accept_path = a.accept_path;
    p.accept_len = a.accept_len;
    p.cu = a.cu_nodes;
    p.status = a.status;
    p.N = a.n_nodes;
    p.total = a.total_nodes;
    p.P = a.max_path_len;
    p.row_vec = a.row_bytes / 16;
    const unsigned pieces = (unsigned)((a.row_bytes + kCompactPiece - 1) / kCompactPiece);
    const dim3 grid(a.max_path_len, a.batch, pieces);
    return launch_pdl(gdn_compact_kernel, grid, dim3(kCompactThreads), 0, stream, p);
}

}  // namespace gdn
