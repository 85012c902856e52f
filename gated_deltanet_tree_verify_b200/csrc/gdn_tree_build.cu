// gdn_tree_build.cu -- best-first draft-tree construction (sm_100a).
//
// Builds a DDTree-style draft tree from the drafter's per-position top-k
// log-probabilities (the GreenGames post, "From autoregressive to DDTree":
// the tree built by build_ddtree, optionally pre-seeded with the greedy
// chain; "Key wins": each position's candidates come best first).  A node is
// a sequence of ranks (r_1 .. r_d); its score is the float32 sum, taken from
// the root down, of logp[i - 1][r_i].  The `budget` best candidates are taken
// one at a time -- highest score, then lower depth, lower rank, lower parent
// index -- and each taken node gets the next index, so parent[n] < n.
//
// One warp builds one tree.  A candidate is a 64-bit key that orders exactly
// as that rule: the score's order-preserving bits, then 255 - depth,
// 255 - rank and 0xffff - parent, so a pop is a warp max-reduction and the
// key alone encodes the node.  Frontier slot s belongs to lane s % 32, which
// alone reads and writes it and caches the largest key it holds; after a pop
// only the lane that held the winner rescans its slots.
//
// Each row of logp is non-increasing, so a sibling (p, r + 1) is never taken
// before (p, r): its float32 score is not larger (rounding is monotonic) and
// ties go to the lower rank.  The frontier is therefore filled lazily --
// taking (p, r) inserts (p, r + 1) and the taken node's own rank-0 child --
// which pops the same sequence as inserting all K children of a node at once.
// The first new candidate goes into the slot just emptied, so each pop adds
// at most one slot: budget + 1 slots in all.

#include <cstdint>

#include <cuda_runtime.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kBuildWarps = 4;  // trees per CTA

struct BParams {
    const float* logp;
    const int32_t* topk_ids;
    int32_t* parent;
    int32_t* depth;
    int32_t* rank;
    int32_t* token;
    float* score;
    int32_t* status;
    int B, D, K, budget, chain, validate;
    uint32_t warp_bytes, off_lp, off_ns, off_info;
};

// Order-preserving map of a non-NaN float to uint32 (x < y <=> ord(x) < ord(y);
// -0 and +0 differ, but scores summed from +0 never become -0).
__device__ __forceinline__ uint32_t score_order(float s)
{
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float order_score(uint32_t o)
{
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

// Never 0: score_order(-inf) = 0x007fffff, so 0 marks an empty slot.
__device__ __forceinline__ uint64_t cand_key(float s, int d, int r, int p)
{
    return (uint64_t(score_order(s)) << 32) | (uint32_t(255 - d) << 24) | (uint32_t(255 - r) << 16) |
           uint32_t(0xffff - p);
}

// Largest key over the warp: the high words first, then the low words of the
// lanes that hold the largest high word.
__device__ __forceinline__ uint64_t warp_max(uint64_t v)
{
    const uint32_t hi = __reduce_max_sync(0xffffffffu, uint32_t(v >> 32));
    const uint32_t lo = __reduce_max_sync(0xffffffffu, uint32_t(v >> 32) == hi ? uint32_t(v) : 0u);
    return (uint64_t(hi) << 32) | lo;
}

__global__ void __launch_bounds__(kBuildWarps * 32) gdn_build_tree_kernel(BParams p)
{
    extern __shared__ __align__(16) unsigned char smem[];
    pdl_wait_then_release();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x * kBuildWarps + warp;
    if (b >= p.B)
        return;
    unsigned char* base = smem + (size_t)warp * p.warp_bytes;
    uint64_t* fr = reinterpret_cast<uint64_t*>(base);            // [budget + 1] frontier keys
    float* lp = reinterpret_cast<float*>(base + p.off_lp);       // [D][K] log-probs
    float* ns = reinterpret_cast<float*>(base + p.off_ns);       // [N] node scores
    uint32_t* info = reinterpret_cast<uint32_t*>(base + p.off_info);  // [N] parent << 16 | depth << 8 | rank

    const int K = p.K, DK = p.D * p.K;
    const float* src = p.logp + (size_t)b * DK;
    for (int i = lane; i < DK; i += 32)
        lp[i] = src[i];
    const int slots = p.budget + 1;
    for (int i = lane; i < slots; i += 32)
        fr[i] = 0;
    __syncwarp();
    if (p.validate) {
        bool bad = false;
        for (int i = lane; i < DK; i += 32) {
            const float x = lp[i];
            bad |= !(x < __int_as_float(0x7f800000));  // NaN or +inf
            if (i % K != 0)
                bad |= lp[i - 1] < x;                    // row not non-increasing
        }
        if (__any_sync(0xffffffffu, bad)) {
            if (lane == 0)
                report_status(p.status, GDN_ERR_BAD_INPUT);
            return;
        }
    }

    uint64_t m = 0;  // largest key in this lane's slots
    int next = 0;    // slots used so far (the same in every lane)
    auto append = [&](uint64_t key) {
        if ((next & 31) == lane) {
            fr[next] = key;
            m = key > m ? key : m;
        }
        ++next;
    };
    if (lane == 0) {
        ns[0] = 0.f;
        info[0] = 0;
    }
    if (p.budget > 0)
        append(cand_key(__fadd_rn(0.f, lp[0]), 1, 0, 0));
    const int chain = p.chain ? min(p.D, p.budget) : 0;
    float s_prev = 0.f;  // score of node n - 1
    int n = 1;
    for (; n <= p.budget; ++n) {
        const bool forced = n <= chain;  // the greedy chain: node n = (n - 1, rank 0)
        const uint64_t best = forced ? cand_key(__fadd_rn(s_prev, lp[(n - 1) * K]), n, 0, n - 1) : warp_max(m);
        if (best == 0)
            break;  // empty frontier: excluded by the host's budget check (reported below)
        // The lane holding `best` takes it out (its slot becomes the hole the
        // first new candidate fills) and finds its next-largest key.
        int hole = -1;
        if (forced || m == best) {
            uint64_t mm = 0;
#pragma unroll 4
            for (int s = lane; s < next; s += 32) {
                const uint64_t v = fr[s];
                if (v == best)
                    hole = s;
                else
                    mm = v > mm ? v : mm;
            }
            if (hole >= 0)
                m = mm;
        }
        if (__ballot_sync(0xffffffffu, hole >= 0) == 0)
            break;  // not reached: `best` is always in some lane's slots
        const int d = 255 - int((best >> 24) & 255);
        const int r = 255 - int((best >> 16) & 255);
        const int par = 0xffff - int(best & 0xffff);
        const float s = order_score(uint32_t(best >> 32));
        if (lane == 0) {
            ns[n] = s;
            info[n] = (uint32_t(par) << 16) | (uint32_t(d) << 8) | uint32_t(r);
        }
        __syncwarp();
        // New candidates: the next sibling and the first child.
        const bool sib = r + 1 < K, child = d < p.D;
        const uint64_t k_sib = sib ? cand_key(__fadd_rn(ns[par], lp[(d - 1) * K + r + 1]), d, r + 1, par) : 0;
        const uint64_t k_child = child ? cand_key(__fadd_rn(s, lp[d * K]), d + 1, 0, n) : 0;
        const uint64_t first = sib ? k_sib : k_child;
        if (hole >= 0) {
            fr[hole] = first;
            m = first > m ? first : m;
        }
        if (sib && child)
            append(k_child);
        s_prev = s;
    }
    if (n <= p.budget) {
        if (lane == 0)
            report_status(p.status, GDN_ERR_BAD_INPUT);
        return;
    }
    __syncwarp();
    const int N = p.budget + 1;
    for (int i = lane; i < N; i += 32) {
        const uint32_t x = info[i];
        const int d = (x >> 8) & 255, r = x & 255;
        const size_t o = (size_t)b * N + i;
        p.parent[o] = i == 0 ? -1 : int(x >> 16);
        if (p.depth)
            p.depth[o] = d;
        if (p.rank)
            p.rank[o] = r;
        if (p.score)
            p.score[o] = ns[i];
        if (p.token)
            p.token[o] = i == 0 ? -1 : __ldg(p.topk_ids + ((size_t)b * p.D + d - 1) * K + r);
    }
}

uint32_t round16(size_t x) { return uint32_t((x + 15) & ~size_t(15)); }

}  // namespace

cudaError_t launch_build_tree(const BuildArgs& a, cudaStream_t stream)
{
    BParams p{};
    p.logp = a.logp;
    p.topk_ids = a.topk_ids;
    p.parent = a.parent;
    p.depth = a.depth;
    p.rank = a.rank;
    p.token = a.token;
    p.score = a.score;
    p.status = a.status;
    p.B = a.batch;
    p.D = a.max_depth;
    p.K = a.top_k;
    p.budget = a.budget;
    p.chain = (a.flags & GDN_BUILD_CHAIN_SEED) != 0;
    p.validate = (a.flags & GDN_BUILD_VALIDATE) != 0;
    const size_t N = (size_t)a.budget + 1;
    p.off_lp = round16(8 * N);
    p.off_ns = p.off_lp + round16(4 * (size_t)a.max_depth * a.top_k);
    p.off_info = p.off_ns + round16(4 * N);
    p.warp_bytes = p.off_info + round16(4 * N);
    const size_t smem = (size_t)kBuildWarps * p.warp_bytes;
    if (smem > 48 * 1024) {
        const cudaError_t e =
            cudaFuncSetAttribute(gdn_build_tree_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
    }
    const dim3 grid((a.batch + kBuildWarps - 1) / kBuildWarps);
    return launch_pdl(gdn_build_tree_kernel, grid, dim3(kBuildWarps * 32), smem, stream, p);
}

}  // namespace gdn
