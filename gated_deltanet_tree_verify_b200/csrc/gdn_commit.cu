// gdn_commit.cu -- commit of the accepted path (sm_100a).
//
// After verification, the accepted root-to-leaf path's last node already has
// its state persisted by the verify kernel (the GreenGames post, "Key wins":
// the persist-write kernel, so no state copy or re-run is needed at verify
// time).  Committing is therefore a bandwidth copy of one node's state per
// sequence and layer into the recurrent state buffer, widened from f16 when
// the persisted dtype is f16.  One launch covers up to kMaxCommitLayers
// layers (an engine commits every GDN layer of the model after the forward
// pass).
//
// Each CTA copies 4096 elements of one (layer, sequence).  Its threads load
// the path's last node id and start loading their part of that node's state
// right away (from a clamped, always in-bounds address), while warp 0 checks
// the tree (parent[0] = -1, 0 <= parent[n] < n) and the whole path against it
// (path[0] = 0, parent[path[i]] = path[i-1]); the stores happen only for a
// valid tree and path.

#include <cstdint>

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kCommitThreads = 256;
constexpr int kCommitElems = 4096;  // elements per CTA (16 KB of f32 output)
constexpr int kPerThread = kCommitElems / (4 * kCommitThreads);

struct CParams {
    const void* node_states[kMaxCommitLayers];
    float* state_out[kMaxCommitLayers];
    const int32_t* parent;
    const int32_t* accept_path;
    const int32_t* accept_len;
    int32_t* status;
    const int32_t* cu;  // varlen node offsets, or NULL
    int total;
    int N, P;
    int persist_last;
    size_t per_seq;  // H_v * d_v * d_k
};

template <typename ST>
struct Load4;

template <>
struct Load4<float> {
    __device__ __forceinline__ static float4 load(const float* p)
    {
        return __ldg(reinterpret_cast<const float4*>(p));
    }
};

template <>
struct Load4<__half> {
    __device__ __forceinline__ static float4 load(const __half* p)
    {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
        const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
        return make_float4(a.x, a.y, b.x, b.y);
    }
};

template <typename ST>
__global__ void __launch_bounds__(kCommitThreads) gdn_commit_kernel(const CParams p)
{
    __shared__ int s_ok;
    const int b = blockIdx.y, layer = blockIdx.z;
    const int tid = threadIdx.x;
    const int32_t* path = p.accept_path + (size_t)b * p.P;
    pdl_wait_then_release();
    // the sequence's nodes: n0 .. n0 + N - 1 (varlen offsets checked)
    int n0 = b * p.N, N = p.N;
    bool seq_ok = true;
    if (p.cu != nullptr) {
        n0 = __ldg(p.cu + b);
        N = __ldg(p.cu + b + 1) - n0;
        seq_ok = n0 >= 0 && N >= 1 && N <= p.N && n0 <= p.total - N;
        if (!seq_ok) {
            n0 = 0;
            N = 1;
        }
    }
    const int len = __ldg(p.accept_len + b);
    const bool len_ok = seq_ok && len >= 1 && len <= N && len <= p.P;

    // speculative: the state of the path's last node (clamped in bounds)
    int last = len_ok ? __ldg(path + len - 1) : 0;
    last = last < 0 ? 0 : (last >= N ? N - 1 : last);
    const ST* src = static_cast<const ST*>(p.node_states[layer]) +
                    (p.persist_last ? (size_t)b : (size_t)n0 + last) * p.per_seq;
    const size_t e0 = (size_t)blockIdx.x * kCommitElems;
    float4 x[kPerThread];
#pragma unroll
    for (int it = 0; it < kPerThread; ++it) {
        const size_t e = e0 + (size_t)(it * kCommitThreads + tid) * 4;
        if (e < p.per_seq)
            x[it] = Load4<ST>::load(src + e);
    }

    if (tid < 32) {
        // the tree itself: parent[0] = -1 and 0 <= parent[n] < n (a path can
        // only be checked against a well-formed tree)
        bool tree_ok = seq_ok;
        if (tree_ok && p.parent) {
            for (int n = tid; n < N; n += 32) {
                const int pn = __ldg(p.parent + (size_t)n0 + n);
                tree_ok &= (n == 0) ? (pn == -1) : (pn >= 0 && pn < n);
            }
        }
        tree_ok = __all_sync(0xffffffffu, tree_ok);
        bool ok = len_ok && tree_ok;
        if (ok) {
            for (int i = tid; i < len; i += 32) {
                const int xi = __ldg(path + i);
                if (i == 0) {
                    ok &= (xi == 0);
                } else {
                    const int prev = __ldg(path + i - 1);
                    const bool in_range = xi > prev && xi < N;
                    const int px = (in_range && p.parent) ? __ldg(p.parent + (size_t)n0 + xi) : xi - 1;
                    ok &= in_range && px == prev;
                }
            }
        }
        ok = __all_sync(0xffffffffu, ok);
        if (ok && p.persist_last && __ldg(path + len - 1) != N - 1)
            ok = false;
        if (tid == 0)
            s_ok = ok ? 1 : (tree_ok ? 0 : -1);
    }
    __syncthreads();
    if (s_ok != 1) {
        if (blockIdx.x == 0 && layer == 0 && tid == 0)
            report_status(p.status, s_ok == 0 ? GDN_ERR_BAD_PATH : GDN_ERR_BAD_TREE);
        return;
    }
    float* dst = p.state_out[layer] + (size_t)b * p.per_seq;
#pragma unroll
    for (int it = 0; it < kPerThread; ++it) {
        const size_t e = e0 + (size_t)(it * kCommitThreads + tid) * 4;
        if (e < p.per_seq)
            *reinterpret_cast<float4*>(dst + e) = x[it];
    }
}

}  // namespace

cudaError_t launch_commit(const CommitArgs& a, cudaStream_t stream)
{
    CParams p{};
    p.parent = a.parent;
    p.accept_path = a.accept_path;
    p.accept_len = a.accept_len;
    p.status = a.status;
    p.N = a.n_nodes;
    p.P = a.max_path_len;
    p.persist_last = (a.flags & GDN_FLAG_PERSIST_LAST) ? 1 : 0;
    p.cu = a.cu_nodes;
    p.total = a.total_nodes;
    p.per_seq = (size_t)a.n_v_heads * a.d_v * a.d_k;
    const unsigned chunks = (unsigned)((p.per_seq + kCommitElems - 1) / kCommitElems);
    for (int l0 = 0; l0 < a.n_layers; l0 += kMaxCommitLayers) {
        const int nl = a.n_layers - l0 < kMaxCommitLayers ? a.n_layers - l0 : kMaxCommitLayers;
        for (int l = 0; l < nl; ++l) {
            p.node_states[l] = a.node_states[l0 + l];
            p.state_out[l] = a.state_out[l0 + l];
        }
        dim3 grid(chunks, a.batch, nl);
        const cudaError_t e =
            a.state_dtype == GDN_F16
                ? launch_pdl(gdn_commit_kernel<__half>, grid, dim3(kCommitThreads), 0, stream, p)
                : launch_pdl(gdn_commit_kernel<float>, grid, dim3(kCommitThreads), 0, stream, p);
        if (e != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

}  // namespace gdn
