// gdn_commit.cu -- commit of the accepted path (sm_100a).
//
// After verification, the accepted root-to-leaf path's last node already has
// its state persisted by the verify kernel (the GreenGames post, "Key wins":
// the persist-write kernel, so no state copy or re-run is needed at verify
// time).  Committing is therefore a bandwidth copy of one node's state per
// sequence into the recurrent state buffer, widened from f16 when the
// persisted dtype is f16.  Each CTA first checks the sequence's accept path
// against the tree (path[0] = 0, parent[path[i]] = path[i-1]) and copies
// nothing for a bad path.

#include <cstdint>

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kCommitThreads = 256;
constexpr int kCommitElems = 4096;  // elements per CTA (16 KB of f32 output)

struct CParams {
    const void* node_states;
    const int32_t* parent;
    const int32_t* accept_path;
    const int32_t* accept_len;
    float* state_out;
    int32_t* status;
    int N, P, NS;
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
    __shared__ int s_ok, s_last;
    const int b = blockIdx.y;
    const int tid = threadIdx.x;
    if (tid < 32) {
        const int len = __ldg(p.accept_len + b);
        const int32_t* path = p.accept_path + (size_t)b * p.P;
        bool ok = len >= 1 && len <= p.N && len <= p.P;
        if (ok) {
            for (int i = tid; i < len; i += 32) {
                const int x = __ldg(path + i);
                if (i == 0) {
                    ok &= (x == 0);
                } else {
                    const int prev = __ldg(path + i - 1);
                    const bool in_range = x > prev && x < p.N;
                    const int px = (in_range && p.parent) ? __ldg(p.parent + (size_t)b * p.N + x) : x - 1;
                    ok &= in_range && px == prev;
                }
            }
        }
        ok = __all_sync(0xffffffffu, ok);
        int last = 0;
        if (ok) {
            last = __ldg(path + len - 1);
            if (p.persist_last && last != p.N - 1)
                ok = false;
        }
        if (tid == 0) {
            s_ok = ok ? 1 : 0;
            s_last = last;
        }
    }
    __syncthreads();
    if (!s_ok) {
        if (blockIdx.x == 0 && tid == 0)
            report_status(p.status, GDN_ERR_BAD_PATH);
        return;
    }
    const ST* src = static_cast<const ST*>(p.node_states) +
                    ((size_t)b * p.NS + (p.persist_last ? 0 : s_last)) * p.per_seq;
    float* dst = p.state_out + (size_t)b * p.per_seq;
    const size_t e0 = (size_t)blockIdx.x * kCommitElems;
#pragma unroll
    for (int it = 0; it < kCommitElems / (4 * kCommitThreads); ++it) {
        const size_t e = e0 + (size_t)(it * kCommitThreads + tid) * 4;
        if (e < p.per_seq)
            *reinterpret_cast<float4*>(dst + e) = Load4<ST>::load(src + e);
    }
}

}  // namespace

cudaError_t launch_commit(const CommitArgs& a, cudaStream_t stream)
{
    CParams p{};
    p.node_states = a.node_states;
    p.parent = a.parent;
    p.accept_path = a.accept_path;
    p.accept_len = a.accept_len;
    p.state_out = a.state_out;
    p.status = a.status;
    p.N = a.n_nodes;
    p.P = a.max_path_len;
    p.persist_last = (a.flags & GDN_FLAG_PERSIST_LAST) ? 1 : 0;
    p.NS = p.persist_last ? 1 : a.n_nodes;
    p.per_seq = (size_t)a.n_v_heads * a.d_v * a.d_k;
    dim3 grid((unsigned)((p.per_seq + kCommitElems - 1) / kCommitElems), a.batch);
    if (a.state_dtype == GDN_F16)
        gdn_commit_kernel<__half><<<grid, kCommitThreads, 0, stream>>>(p);
    else
        gdn_commit_kernel<float><<<grid, kCommitThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace gdn
