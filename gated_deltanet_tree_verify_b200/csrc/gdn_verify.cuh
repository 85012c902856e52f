// gdn_verify.cuh -- the tree-verify kernels of libgdntree (sm_100a), as
// templates; gdn_verify_d{32,64,128}.cu instantiate them per head dim.
//
// One CTA per (sequence b, v-head h, tile of d_v rows).  The CTA walks the
// tree's nodes in depth-first preorder, a topological order, visiting each
// node's children by increasing subtree size (ties by index) so that the
// largest child subtree comes last, and for each node applies the gated
// delta rule (Gated DeltaNet; the ggml_gated_delta_net recurrence named in
// the GreenGames post, "TL;DR"):
//
//     a = exp(g_n);  w = a * S_p k_n;  u = beta_n * (v_n - w)
//     S_n = a * S_p + u k_n^T;         o_n = scale * S_n q_n
//
// and persists S_n from inside the kernel (the GreenGames post, "Key wins":
// persist-write kernel, f16 intermediate cache).
//
// Compute layout: LR = d_k / 16 lanes share a state row, each holding 16
// columns (4 chunks of 4 at columns 4 * (c + m * LR)); a lane holds RL rows
// (RL = 1 or 2), so a warp owns RL * 32 / LR rows (4 or 8 at d_k = 128).
// S k is a packed-fp32 (FFMA2) partial dot plus an xor-butterfly over the
// row's LR lanes; the rank-1 update is packed fp32.  The partial S q dots of
// four consecutive nodes are reduced together by a transpose-reduce and
// stored as one vector.  Each node's state leaves as 16-byte (f32) or 8-byte
// (f16) stores that cover whole 128-byte lines of a row.  Which rows a lane
// holds (RL, warps per CTA) never changes a row's arithmetic.
//
// Inputs are widened to f32 once per CTA into shared-memory records
// (k_n | q_n | the CTA's slice of v_n).  Two kernels:
//   * gdn_verify_staged: trees and chains small enough to stage whole.  All
//     threads issue 16-byte asynchronous copies (cp.async) of every node's
//     raw rows at kernel start, so they overlap the tree walk and the
//     state_in load; all threads then widen them; all warps compute.  Trees
//     of up to 32 nodes are walked from warp registers (each warp builds the
//     walk with shuffles and ballots, no shared memory, no block barrier).
//   * gdn_verify_ring: anything larger (long chains).  A producer warp loads,
//     widens and streams chunks of walk positions through a ring of
//     mbarrier-guarded slots.
//
// Parents that are not the previous node of the walk: with exact f32
// persistence the parent's state is re-read from node_states (written by the
// same thread, bit-exact).  Otherwise a node with two or more children saves
// its f32 state in a shared-memory stack slot, and a later child reloads it.
// The slot index is the number of edges on the node's root path that enter a
// child other than the last one visited; since every such child's subtree
// holds at most half of its parent's, floor(log2 N) slots always suffice.  If
// fewer slots are configured and a tree needs more, the parent's state is
// recomputed (same instruction sequence, so the same bits) from the deepest
// saved ancestor.  Children therefore always continue from the exact f32
// state; the visiting order of siblings does not change any result.
//
// Every arithmetic step uses explicit round-to-nearest intrinsics in a fixed
// order, so a node's results depend only on its root path: the chain fast
// path, a chain walked as a tree, a reloaded and a recomputed parent give
// identical bits.

#pragma once

#include <atomic>
#include <cstdint>
#include <type_traits>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace verify {

constexpr int kColsPerLane = 16;  // 4 chunks of 4 consecutive columns
constexpr int kMaxWarps = 4;      // compute warps per CTA
constexpr int kChunk = 8;         // walk positions per ring slot
constexpr int kRing = 3;          // ring slots
constexpr int kMaxDevices = 64;
constexpr int kStagedMaxSmem = 100 * 1024;

// Per-position walk metadata (tree mode), packed in one int32:
//   bits 0..15 node id, 16..18 source of the parent state,
//   bits 19..23 save slot + 1 (0: do not save), 24..28 load slot.
enum : int { kSrcCont = 0, kSrcSlot = 1, kSrcRecompute = 2, kSrcRoot = 3, kSrcReload = 4 };

__device__ __forceinline__ int meta_node(int m) { return m & 0xffff; }
__device__ __forceinline__ int meta_src(int m) { return (m >> 16) & 7; }
__device__ __forceinline__ int meta_save(int m) { return ((m >> 19) & 31) - 1; }
__device__ __forceinline__ int meta_load(int m) { return (m >> 24) & 31; }

// The decay gate a = exp(g), compiled once so that every caller gets
// identical bits.
static __device__ __noinline__ float gdn_gate(float g) { return expf(g); }

struct KParams {
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
    int N, Hk, Hv, dv, G;
    float scale;
    int rows, warps, slots;
    int persist_last, validate, reload, early_tree;
    uint32_t raw_bytes;   // one node's raw record (k | q | v slice) in bytes
    uint32_t rec_floats;  // one node's widened record in floats
    uint32_t off_raw, off_rec, off_ab, off_slots, off_tree;
};

// ---------------------------------------------------------------------------
// Lane geometry and per-node arithmetic
// ---------------------------------------------------------------------------

template <int DK, int RL>
struct LaneMap {
    static constexpr int LR = DK / kColsPerLane;  // lanes per row
    static constexpr int RG = 32 / LR;            // row groups per warp
    static constexpr int RPW = RL * RG;           // rows per warp
    int cl;
    int rloc[RL];
    __device__ __forceinline__ LaneMap(int warp, int lane)
    {
        cl = lane % LR;
#pragma unroll
        for (int r = 0; r < RL; ++r)
            rloc[r] = warp * RPW + lane / LR + r * RG;
    }
    __device__ __forceinline__ int col(int m) const { return 4 * (cl + m * LR); }
};

template <int RL>
struct StateT {
    float2 s[RL][8];
};

// One node's state update on a lane's RL rows x 16 columns.  Shared by the
// walk and the recompute path; explicit intrinsics keep both bit-identical.
// With WITH_Q it also reduces this node's output read of the pre-update state,
// pq = S_p q, in the same butterfly as S_p k, and returns u: the output is
// then o = scale * (a * pq + u * (k . q)) = scale * S_n q (S_n = a S_p + u k^T).
template <int LR, int RL, bool WITH_Q>
__device__ __forceinline__ void gdn_step(StateT<RL>& S, const float2 (&k2)[8], const float2 (&q2)[8],
                                         const float (&vr)[RL], float a, float beta, float (&pq)[RL],
                                         float (&uo)[RL])
{
    float w[RL];
#pragma unroll
    for (int r = 0; r < RL; ++r) {
        float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int t = 0; t < 8; t += 2) {
            acc0 = __ffma2_rn(S.s[r][t], k2[t], acc0);
            acc1 = __ffma2_rn(S.s[r][t + 1], k2[t + 1], acc1);
        }
        w[r] = __fadd_rn(__fadd_rn(acc0.x, acc0.y), __fadd_rn(acc1.x, acc1.y));
        if constexpr (WITH_Q) {
            float2 b0 = make_float2(0.f, 0.f), b1 = make_float2(0.f, 0.f);
#pragma unroll
            for (int t = 0; t < 8; t += 2) {
                b0 = __ffma2_rn(S.s[r][t], q2[t], b0);
                b1 = __ffma2_rn(S.s[r][t + 1], q2[t + 1], b1);
            }
            pq[r] = __fadd_rn(__fadd_rn(b0.x, b0.y), __fadd_rn(b1.x, b1.y));
        }
    }
#pragma unroll
    for (int off = 1; off < LR; off <<= 1) {
#pragma unroll
        for (int r = 0; r < RL; ++r) {
            w[r] = __fadd_rn(w[r], __shfl_xor_sync(0xffffffffu, w[r], off));
            if constexpr (WITH_Q)
                pq[r] = __fadd_rn(pq[r], __shfl_xor_sync(0xffffffffu, pq[r], off));
        }
    }
    const float2 a2 = make_float2(a, a);
#pragma unroll
    for (int r = 0; r < RL; ++r) {
        const float u = __fmul_rn(beta, __fsub_rn(vr[r], __fmul_rn(a, w[r])));
        uo[r] = u;
        const float2 u2 = make_float2(u, u);
#pragma unroll
        for (int t = 0; t < 8; ++t)
            S.s[r][t] = __ffma2_rn(u2, k2[t], __fmul2_rn(a2, S.s[r][t]));
    }
}

// State update only (recompute path): the same instructions on S.
template <int LR, int RL>
__device__ __forceinline__ void gdn_update(StateT<RL>& S, const float2 (&k2)[8], const float (&vr)[RL],
                                           float a, float beta)
{
    float pq[RL], uo[RL];
    gdn_step<LR, RL, false>(S, k2, k2, vr, a, beta, pq, uo);
}

// k . q of one node's record, the same reduction wherever it is computed.
template <int DK, typename RT>
__device__ __forceinline__ float node_kq(const RT* rec, int lane)
{
    float acc = 0.f;
#pragma unroll
    for (int j = lane; j < DK; j += 32)
        acc = __fmaf_rn(Widen<RT>::lds1(rec + j), Widen<RT>::lds1(rec + DK + j), acc);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
        acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
    return acc;
}

template <typename ST>
struct Persist;

template <>
struct Persist<float> {
    __device__ __forceinline__ static void store(float* dst, float2 lo, float2 hi)
    {
        *reinterpret_cast<float4*>(dst) = make_float4(lo.x, lo.y, hi.x, hi.y);
    }
};

template <>
struct Persist<__half> {
    __device__ __forceinline__ static void store(__half* dst, float2 lo, float2 hi)
    {
        const __half2 a = __float22half2_rn(lo);
        const __half2 b = __float22half2_rn(hi);
        uint2 u;
        u.x = *reinterpret_cast<const uint32_t*>(&a);
        u.y = *reinterpret_cast<const uint32_t*>(&b);
        *reinterpret_cast<uint2*>(dst) = u;
    }
};

// S <- this lane's part of a [rows][DK] f32 matrix (plain loads, so a state
// this thread stored earlier in the kernel is seen).
template <int DK, int RL>
__device__ __forceinline__ void load_state(StateT<RL>& S, const float* base, const LaneMap<DK, RL>& L)
{
#pragma unroll
    for (int r = 0; r < RL; ++r) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float4 x = *reinterpret_cast<const float4*>(base + (size_t)L.rloc[r] * DK + L.col(m));
            S.s[r][2 * m] = make_float2(x.x, x.y);
            S.s[r][2 * m + 1] = make_float2(x.z, x.w);
        }
    }
}

template <int DK, int RL>
__device__ __forceinline__ void save_state(const StateT<RL>& S, float* base, const LaneMap<DK, RL>& L)
{
#pragma unroll
    for (int r = 0; r < RL; ++r) {
#pragma unroll
        for (int m = 0; m < 4; ++m)
            *reinterpret_cast<float4*>(base + (size_t)L.rloc[r] * DK + L.col(m)) =
                make_float4(S.s[r][2 * m].x, S.s[r][2 * m].y, S.s[r][2 * m + 1].x,
                            S.s[r][2 * m + 1].y);
    }
}

// k and the v slice of one node from its shared-memory record [k | q | v
// slice], stored either widened (RT = float) or raw (RT = bf16: widened here).
template <int DK, int RL, typename RT>
__device__ __forceinline__ void load_k(const RT* rec, const LaneMap<DK, RL>& L, float2 (&k2)[8],
                                       float (&vr)[RL])
{
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const float4 x = Widen<RT>::lds4(rec + L.col(m));
        k2[2 * m] = make_float2(x.x, x.y);
        k2[2 * m + 1] = make_float2(x.z, x.w);
    }
#pragma unroll
    for (int r = 0; r < RL; ++r)
        vr[r] = Widen<RT>::lds1(rec + 2 * DK + L.rloc[r]);
}

template <int DK, int RL, typename RT>
__device__ __forceinline__ void load_q(const RT* rec, const LaneMap<DK, RL>& L, float2 (&q2)[8])
{
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const float4 y = Widen<RT>::lds4(rec + DK + L.col(m));
        q2[2 * m] = make_float2(y.x, y.y);
        q2[2 * m + 1] = make_float2(y.z, y.w);
    }
}

// Shared-memory tree arrays (tree mode), each [N] int:
//   par | ord | meta | rstart | nch | sz | lt | off | last | path scratch [warps][N]
constexpr int kTreeArrays = 9;
struct TreeView {
    int *par, *ord, *meta, *rstart, *nch, *sz, *lt, *off, *last, *path;
    __device__ __forceinline__ TreeView(int* t, int N)
        : par(t), ord(t + N), meta(t + 2 * N), rstart(t + 3 * N), nch(t + 4 * N), sz(t + 5 * N),
          lt(t + 6 * N), off(t + 7 * N), last(t + 8 * N), path(t + 9 * N)
    {
    }
};

// Builds the depth-first walk of one tree with all threads of the CTA (per
// node: O(depth) to walk up its root path, O(N) to rank it among its
// siblings).  Siblings are visited by increasing (subtree size, index).
// Returns false on every thread if the tree is malformed.  K: shared-memory
// stack slots; reload: parents come from node_states instead of slots.
static __device__ bool build_walk(const int32_t* prow, int N, int K, bool reload, const TreeView& T)
{
    const int tid = threadIdx.x, nthr = blockDim.x;
    bool bad = false;
    for (int n = tid; n < N; n += nthr) {
        const int pn = __ldg(prow + n);
        T.par[n] = pn;
        T.nch[n] = 0;
        T.sz[n] = 1;
        bad |= (n == 0) ? (pn != -1) : (pn < 0 || pn >= n);
    }
    if (__syncthreads_or(bad))
        return false;
    // child counts and subtree sizes
    for (int n = 1 + tid; n < N; n += nthr) {
        atomicAdd(&T.nch[T.par[n]], 1);
        for (int x = T.par[n]; x >= 0; x = T.par[x])
            atomicAdd(&T.sz[x], 1);
    }
    __syncthreads();
    // offset of each node inside its parent's block (1 + sizes of the siblings
    // visited before it) and whether it is its parent's last-visited child
    for (int n = tid; n < N; n += nthr) {
        int o = 0, is_last = 1;
        if (n > 0) {
            const int p = T.par[n], zn = T.sz[n];
            o = 1;
            for (int s = p + 1; s < N; ++s) {
                if (s == n || T.par[s] != p)
                    continue;
                const int zs = T.sz[s];
                if (zs < zn || (zs == zn && s < n))
                    o += zs;
                else
                    is_last = 0;
            }
        }
        T.off[n] = o;
        T.last[n] = is_last;
    }
    __syncthreads();
    // preorder position (sum of offsets along the root path) and stack slot
    // (number of path edges entering a child that is not visited last)
    for (int n = tid; n < N; n += nthr) {
        int pos = 0, l = 0;
        for (int x = n; x > 0; x = T.par[x]) {
            pos += T.off[x];
            l += T.last[x] ? 0 : 1;
        }
        T.ord[pos] = n;
        T.lt[n] = l;
    }
    __syncthreads();
    for (int pos = tid; pos < N; pos += nthr) {
        const int n = T.ord[pos];
        const int pp = T.par[n];
        int src, ld = 0, start = -1, save = 0;
        if (pos == 0) {
            src = kSrcRoot;
        } else if (pp == T.ord[pos - 1]) {
            src = kSrcCont;
        } else if (reload) {
            src = kSrcReload;
        } else if (T.lt[pp] < K) {
            src = kSrcSlot;
            ld = T.lt[pp];
        } else {
            src = kSrcRecompute;
            // deepest saved ancestor of pp: the deepest branching ancestor in
            // slot K - 1 (none when K == 0: start from state_in)
            int x = T.par[pp];
            while (x >= 0 && !(T.nch[x] >= 2 && T.lt[x] == K - 1))
                x = T.par[x];
            start = x;
        }
        if (!reload && T.nch[n] >= 2 && T.lt[n] < K)
            save = T.lt[n] + 1;
        T.meta[pos] = n | (src << 16) | (save << 19) | (ld << 24);
        T.rstart[pos] = start;
    }
    __syncthreads();
    return true;
}

// Tree metadata held in shared memory (any N).
struct SmemTree {
    static constexpr bool kIndex = false;
    TreeView T;
    int N, warp;
    __device__ __forceinline__ int meta(int pos) const { return T.meta[pos]; }
    __device__ __forceinline__ int rstart(int pos) const { return T.rstart[pos]; }
    __device__ __forceinline__ int parent(int n) const { return T.par[n]; }
    // Calls f(y) for the nodes y after `start` (exclusive; -1: the root's
    // parent) down to pp (inclusive), root side first.
    template <class F>
    __device__ __forceinline__ void for_path(int pp, int start, F&& f) const
    {
        int* path = T.path + warp * N;
        int len = 0;
        for (int x = pp; x != start; x = T.par[x])
            path[len++] = x;  // every lane writes the same values
        __syncwarp();
        for (int e = len - 1; e >= 0; --e)
            f(path[e]);
        __syncwarp();
    }
};

// Walk of a tree of N <= 32 nodes as built in one warp's registers: lane n
// holds node n's parent and ancestor-or-self bitmask, lane p walk position
// p's metadata.
struct WarpTree {
    int par_l, meta_l, rstart_l;
    unsigned mask_l;
};

// The same walk published in shared memory for every warp of the CTA:
// [meta | rstart | par | mask] x 32.
struct MaskTree {
    static constexpr bool kIndex = false;
    const int* a;
    __device__ __forceinline__ int meta(int pos) const { return a[pos]; }
    __device__ __forceinline__ int rstart(int pos) const { return a[32 + pos]; }
    __device__ __forceinline__ int parent(int n) const { return a[64 + n]; }
    template <class F>
    __device__ __forceinline__ void for_path(int pp, int start, F&& f) const
    {
        // node indices grow along every root path, so ascending bits are the
        // path in root-to-leaf order
        unsigned bits = static_cast<unsigned>(a[96 + pp]);
        if (start >= 0)
            bits &= ~static_cast<unsigned>(a[96 + start]);
        while (bits) {
            const int y = __ffs(bits) - 1;
            bits &= bits - 1;
            f(y);
        }
    }
};

// Index-order walk (f32 persistence): position p is node p; a parent that is
// not the previous node is re-read from node_states, prefetched one node
// ahead.  par: the tree's parent array in shared memory.
struct IndexTree {
    static constexpr bool kIndex = true;
    const int* par;
    __device__ __forceinline__ int meta(int pos) const
    {
        const int src = pos == 0 ? kSrcRoot : (par[pos] == pos - 1 ? kSrcCont : kSrcReload);
        return pos | (src << 16);
    }
    __device__ __forceinline__ int rstart(int) const { return -1; }
    __device__ __forceinline__ int parent(int n) const { return par[n]; }
    template <class F>
    __device__ __forceinline__ void for_path(int, int, F&&) const
    {
    }
};

// Builds the walk of a tree of N <= 32 nodes in the registers of the calling
// warp (same order and metadata as build_walk, no shared memory, no block
// barrier).  Returns false if the tree is malformed (the same on every lane).
static __device__ bool build_warp_walk(const int32_t* prow, int N, int K, bool reload, WarpTree& W)
{
    const unsigned full = 0xffffffffu;
    const int lane = threadIdx.x & 31;
    const bool valid = lane < N;
    const int par = valid ? __ldg(prow + lane) : -1;
    const bool bad = valid && ((lane == 0) ? par != -1 : (par < 0 || par >= lane));
    if (__any_sync(full, bad))
        return false;
    // ancestor-or-self bitmask by pointer jumping (depth < 32)
    unsigned mask = valid ? (1u << lane) : 0u;
    int jump = valid ? par : -1;
#pragma unroll
    for (int it = 0; it < 5; ++it) {
        const unsigned pm = __shfl_sync(full, mask, jump & 31);
        const int pj = __shfl_sync(full, jump, jump & 31);
        if (jump >= 0) {
            mask |= pm;
            jump = pj;
        }
    }
    // child counts and subtree sizes
    int nch = 0, sz = 0;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const unsigned bp = __ballot_sync(full, valid && par == k);
        const unsigned bm = __ballot_sync(full, (mask >> k) & 1u);
        if (lane == k) {
            nch = __popc(bp);
            sz = __popc(bm);
        }
    }
    // offset among siblings visited by increasing (subtree size, index), and
    // whether the node is its parent's last-visited child
    int off = (valid && lane > 0) ? 1 : 0, last = 1;
#pragma unroll
    for (int s = 0; s < 32; ++s) {
        const int ps = __shfl_sync(full, par, s);
        const int zs = __shfl_sync(full, sz, s);
        if (valid && lane > 0 && s < N && s != lane && ps == par) {
            if (zs < sz || (zs == sz && s < lane))
                off += zs;
            else
                last = 0;
        }
    }
    // preorder position and stack slot: sums along the root path
    int pos = 0, lt = 0;
#pragma unroll
    for (int x = 1; x < 32; ++x) {
        const int ox = __shfl_sync(full, off, x);
        const int lx = __shfl_sync(full, last, x);
        if ((mask >> x) & 1u) {
            pos += ox;
            lt += lx ? 0 : 1;
        }
    }
    // lane p: the node at walk position p
    int ord = 0;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const unsigned bb = __ballot_sync(full, valid && pos == k);
        if (lane == k && bb)
            ord = __ffs(bb) - 1;
    }
    const int pp = __shfl_sync(full, par, ord);
    const int prev = __shfl_sync(full, ord, (lane + 31) & 31);
    const int lt_pp = __shfl_sync(full, lt, pp & 31);
    const int lt_n = __shfl_sync(full, lt, ord);
    const int nch_n = __shfl_sync(full, nch, ord);
    const unsigned mask_pp = __shfl_sync(full, mask, pp & 31);
    const unsigned cand_all = __ballot_sync(full, valid && nch >= 2 && lt == K - 1);
    int src, ld = 0, start = -1, save = 0;
    if (lane == 0) {
        src = kSrcRoot;
    } else if (pp == prev) {
        src = kSrcCont;
    } else if (reload) {
        src = kSrcReload;
    } else if (lt_pp < K) {
        src = kSrcSlot;
        ld = lt_pp;
    } else {
        // deepest saved ancestor of pp: the deepest (largest index) branching
        // proper ancestor in slot K - 1
        src = kSrcRecompute;
        const unsigned cand = cand_all & mask_pp & ~(1u << (pp & 31));
        start = cand ? 31 - __clz(cand) : -1;
    }
    if (!reload && nch_n >= 2 && lt_n < K)
        save = lt_n + 1;
    W.par_l = par;
    W.mask_l = mask;
    W.meta_l = ord | (src << 16) | (save << 19) | (ld << 24);
    W.rstart_l = start;
    return true;
}

// Makes S the exact f32 state of node pp, the parent of the node at a walk
// position whose metadata says the state is not already in registers.
// fetch(y, k2, vr, a, beta) supplies node y's inputs for the recompute path.
template <int DK, int RL, class Tree, class Fetch>
__device__ __forceinline__ void source_parent(StateT<RL>& S, int m, int pp, int start, const KParams& p,
                                              const Tree& tree, const float* slotbuf,
                                              const float* sin_head, int b, int h, int row0,
                                              const LaneMap<DK, RL>& L, Fetch fetch)
{
    constexpr int LR = LaneMap<DK, RL>::LR;
    const int src = meta_src(m);
    if (src == kSrcReload) {
        const float* ns = static_cast<const float*>(p.node_states) +
                          (((size_t)b * p.N + pp) * p.Hv + h) * p.dv * DK + (size_t)row0 * DK;
        load_state<DK, RL>(S, ns, L);
    } else if (src == kSrcSlot) {
        load_state<DK, RL>(S, slotbuf + (size_t)meta_load(m) * p.rows * DK, L);
    } else if (src == kSrcRecompute) {
        if (start >= 0)
            load_state<DK, RL>(S, slotbuf + (size_t)(p.slots - 1) * p.rows * DK, L);
        else
            load_state<DK, RL>(S, sin_head, L);
        tree.for_path(pp, start, [&](int y) {
            float2 k2[8];
            float vr[RL];
            float a, be;
            fetch(y, k2, vr, a, be);
            gdn_update<LR, RL>(S, k2, vr, a, be);
        });
    }
}

// Where this lane's rows of node n's state and output live: one 64-bit base
// per node plus per-lane 32-bit offsets computed once.
template <int DK, int RL, typename ST>
struct OutPtrs {
    ST* ns_head;          // node_states of (b, h) at node 0
    size_t ns_stride;     // elements between consecutive nodes' states
    float* out_head;      // out of (b, h) at node 0, row row0
    size_t out_stride;    // elements between consecutive nodes' outputs
    uint32_t ns_off[RL];  // (row0 + row) * DK + 4 * cl
    uint32_t out_off[RL];
    __device__ __forceinline__ OutPtrs(const KParams& p, int b, int h, int row0, const LaneMap<DK, RL>& L)
    {
        const int NS = p.persist_last ? 1 : p.N;
        ns_stride = (size_t)p.Hv * p.dv * DK;
        ns_head = static_cast<ST*>(p.node_states) + (size_t)b * NS * ns_stride + (size_t)h * p.dv * DK;
        out_stride = (size_t)p.Hv * p.dv;
        out_head = p.out + (size_t)b * p.N * out_stride + (size_t)h * p.dv + row0;
#pragma unroll
        for (int r = 0; r < RL; ++r) {
            ns_off[r] = (uint32_t)((row0 + L.rloc[r]) * DK + 4 * L.cl);
            out_off[r] = (uint32_t)L.rloc[r];
        }
    }
};

template <int DK, int RL, typename ST>
__device__ __forceinline__ void persist(const StateT<RL>& S, int n, int pos, const KParams& p,
                                        const OutPtrs<DK, RL, ST>& P)
{
    constexpr int LR = DK / kColsPerLane;
    if (p.persist_last && pos != p.N - 1)
        return;
    ST* node = P.ns_head + (size_t)(p.persist_last ? 0 : n) * P.ns_stride;
#pragma unroll
    for (int r = 0; r < RL; ++r) {
        ST* row = node + P.ns_off[r];
#pragma unroll
        for (int m = 0; m < 4; ++m)
            Persist<ST>::store(row + 4 * m * LR, S.s[r][2 * m], S.s[r][2 * m + 1]);
    }
}

// The walk over positions [0, N): per position, find the parent state,
// update, persist, and batch the outputs.  The context supplies each
// position's widened record, gate and decay (ctx.rec, ctx.ab), the walk's
// input fetcher for recomputation, and the ring handshakes (ctx.begin /
// ctx.end; trivial when everything is staged).
template <int DK, int RL, typename ST, bool CHAIN, class Tree, class Ctx>
__device__ __forceinline__ void walk(StateT<RL>& S, const KParams& p, const Tree& tree,
                                     float* slotbuf, const float* sin_head, int b, int h, int row0,
                                     const LaneMap<DK, RL>& L, Ctx& ctx)
{
    constexpr int LR = LaneMap<DK, RL>::LR;
    const int N = p.N;
    const OutPtrs<DK, RL, ST> P(p, b, h, row0, L);
    StateT<RL> Sn;  // index order: the next position's parent state, prefetched
    const float* nsf = static_cast<const float*>(p.node_states) +
                       ((size_t)b * p.N * p.Hv + h) * p.dv * DK + (size_t)row0 * DK;
    const size_t node_stride = (size_t)p.Hv * p.dv * DK;
    for (int pos = 0; pos < N; ++pos) {
        if (!ctx.begin(pos))
            return;
        int n = pos, save = -1;
        bool next_reload = false;
        if constexpr (Tree::kIndex) {
            // issue the loads of the next position's parent state now; it was
            // persisted by this thread at an earlier position
            if (pos + 1 < N) {
                const int pn = tree.parent(pos + 1);
                next_reload = pn != pos;
                if (next_reload)
                    load_state<DK, RL>(Sn, nsf + (size_t)pn * node_stride, L);
            }
        } else if constexpr (!CHAIN) {
            const int m = tree.meta(pos);
            n = meta_node(m);
            save = meta_save(m);
            const int rs = tree.rstart(pos);
            const int pp = tree.parent(n);
            if (meta_src(m) != kSrcCont && meta_src(m) != kSrcRoot)
                source_parent<DK, RL>(S, m, pp, rs, p, tree, slotbuf, sin_head, b, h, row0, L,
                                      ctx.fetcher());
        }
        const auto* rec = ctx.rec(pos, n);
        float2 k2[8], q2[8];
        float vr[RL];
        load_k<DK, RL>(rec, L, k2, vr);
        load_q<DK, RL>(rec, L, q2);
        float a, be, kq;
        ctx.ab(pos, n, a, be, kq);
        float pq[RL], u[RL];
        gdn_step<LR, RL, true>(S, k2, q2, vr, a, be, pq, u);
        if (L.cl == 0) {
            float* o = P.out_head + (size_t)n * P.out_stride;
#pragma unroll
            for (int r = 0; r < RL; ++r)
                o[P.out_off[r]] = __fmul_rn(p.scale, __fmaf_rn(u[r], kq, __fmul_rn(a, pq[r])));
        }
        persist<DK, RL, ST>(S, n, pos, p, P);
        if (save >= 0)
            save_state<DK, RL>(S, slotbuf + (size_t)save * p.rows * DK, L);
        if constexpr (Tree::kIndex) {
            if (next_reload)
                S = Sn;
        }
        ctx.end(pos);
    }
}

// ---------------------------------------------------------------------------
// Staged kernel: every node's inputs copied into shared memory at start
// ---------------------------------------------------------------------------

// Staged records: RT = float (widened once) or the raw input type.
template <int DK, int RL, typename RT>
struct StagedFetch {
    const RT* recs;
    const float* ab;
    uint32_t rec_elems;
    int N;
    LaneMap<DK, RL> L;
    __device__ __forceinline__ void operator()(int y, float2 (&k2)[8], float (&vr)[RL], float& a,
                                               float& be) const
    {
        load_k<DK, RL>(recs + (size_t)y * rec_elems, L, k2, vr);
        a = ab[y];
        be = ab[N + y];
    }
};

template <int DK, int RL, typename RT>
struct StagedCtx {
    const RT* recs;
    const float* ab_;
    uint32_t rec_elems;
    int N;
    LaneMap<DK, RL> L;
    __device__ __forceinline__ bool begin(int) { return true; }
    __device__ __forceinline__ void end(int) {}
    __device__ __forceinline__ const RT* rec(int, int n) const
    {
        return recs + (size_t)n * rec_elems;
    }
    __device__ __forceinline__ void ab(int, int n, float& a, float& be, float& kq) const
    {
        a = ab_[n];
        be = ab_[N + n];
        kq = ab_[2 * N + n];
    }
    __device__ __forceinline__ StagedFetch<DK, RL, RT> fetcher() const
    {
        return StagedFetch<DK, RL, RT>{recs, ab_, rec_elems, N, L};
    }
};

// Tree policy of the staged kernel: chain, walk in warp registers (N <= 32)
// or walk in shared memory.
enum : int { kTreeChain = 0, kTreeWarp = 1, kTreeSmem = 2, kTreeIndex = 3 };

struct NoTree {
    static constexpr bool kIndex = false;
    __device__ __forceinline__ int meta(int pos) const { return pos; }
    __device__ __forceinline__ int rstart(int) const { return -1; }
    __device__ __forceinline__ int parent(int n) const { return n - 1; }
    template <class F>
    __device__ __forceinline__ void for_path(int, int, F&&) const
    {
    }
};

__device__ __forceinline__ void cp_async16(void* dst_smem, const void* src_gmem)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst_smem)), "l"(src_gmem)
                 : "memory");
}

template <int DK, int RL, typename QT, typename ST, int TREE>
__global__ void __launch_bounds__(kMaxWarps * 32) gdn_verify_staged(const KParams p)
{
    constexpr int EPC = 16 / sizeof(QT);  // elements per 16-byte chunk
    constexpr int QKCH = DK / EPC;        // chunks per k (or q) row
    extern __shared__ __align__(16) unsigned char smem[];
    unsigned char* raw = smem + p.off_raw;
    float* recs = reinterpret_cast<float*>(smem + p.off_rec);
    float* ab = reinterpret_cast<float*>(smem + p.off_ab);
    float* slotbuf = reinterpret_cast<float*>(smem + p.off_slots);
    int* tsm = reinterpret_cast<int*>(smem + p.off_tree);

    const int N = p.N;
    const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int hk = h / p.G;
    const int row0 = tile * p.rows;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int nwarps = blockDim.x >> 5;
    const int32_t* prow = p.parent + (size_t)b * N;
    // Everything that reads q, k, v, g, beta waits for the preceding kernel;
    // with GDN_FLAG_EARLY_TREE the tree and the root's parent state are read
    // before that (they were written before the preceding kernel started).
    if (!p.early_tree)
        pdl_wait_then_release();

    // 1. the parent array (index order keeps it in shared memory; chain
    //    validation only checks it)
    bool bad = false;
    if constexpr (TREE == kTreeIndex) {
        for (int n = tid; n < N; n += blockDim.x) {
            const int pn = __ldg(prow + n);
            tsm[n] = pn;
            bad |= (n == 0) ? (pn != -1) : (pn < 0 || pn >= n);
        }
    } else if constexpr (TREE == kTreeChain) {
        if (p.validate) {
            for (int n = tid; n < N; n += blockDim.x)
                bad |= __ldg(prow + n) != n - 1;
        }
    }
    // 2. the root's parent state
    const LaneMap<DK, RL> L(warp, lane);
    const float* sin_head = p.state_in + ((size_t)b * p.Hv + h) * p.dv * DK + (size_t)row0 * DK;
    StateT<RL> S;
    load_state<DK, RL>(S, sin_head, L);
    // 3. the walk: warp 0 builds it for trees of <= 32 nodes (the other warps
    //    go on to the copies); all threads for larger trees
    const TreeView tv(tsm, N);
    if constexpr (TREE == kTreeWarp) {
        if (warp == 0) {
            WarpTree wt{};
            if (build_warp_walk(prow, N, p.slots, p.reload != 0, wt)) {
                tsm[lane] = wt.meta_l;
                tsm[32 + lane] = wt.rstart_l;
                tsm[64 + lane] = wt.par_l;
                tsm[96 + lane] = static_cast<int>(wt.mask_l);
            } else {
                bad = true;
            }
        }
    } else if constexpr (TREE == kTreeSmem) {
        bad = !build_walk(prow, N, p.slots, p.reload != 0, tv);
    }
    if (p.early_tree)
        pdl_wait_then_release();
    // 4. every node's raw k row, q row and v slice -> shared memory (async);
    //    warp w copies nodes w, w + warps, ...
    const int per_node = p.raw_bytes / 16;  // 16-byte chunks per node
    {
        const QT* kg = static_cast<const QT*>(p.k);
        const QT* qg = static_cast<const QT*>(p.q);
        const QT* vg = static_cast<const QT*>(p.v);
        for (int n = warp; n < N; n += nwarps) {
            const size_t node = (size_t)b * N + n;
            const QT* krow = kg + (node * p.Hk + hk) * DK;
            const QT* qrow = qg + (node * p.Hk + hk) * DK;
            const QT* vrow = vg + (node * p.Hv + h) * p.dv + row0;
            unsigned char* dst = raw + (size_t)n * p.raw_bytes;
            for (int c = lane; c < per_node; c += 32) {
                const QT* src = c < QKCH ? krow + c * EPC
                                         : (c < 2 * QKCH ? qrow + (c - QKCH) * EPC
                                                         : vrow + (c - 2 * QKCH) * EPC);
                cp_async16(dst + 16 * c, src);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    // 5. gates
    for (int n = tid; n < N; n += blockDim.x) {
        const size_t gi = ((size_t)b * N + n) * p.Hv + h;
        ab[n] = gdn_gate(__ldg(p.g + gi));
        ab[N + n] = __ldg(p.beta + gi);
    }
    // 6. the copies target this CTA's shared memory: wait for them even when
    //    the tree is rejected
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (__syncthreads_or(bad)) {
        if (tid == 0)
            report_status(p.status, GDN_ERR_BAD_TREE);
        return;
    }
    // 7. widen the raw records to f32 once (bf16 inputs, two rows per lane);
    //    with one row per lane the node loop widens its own k, q, v instead
    //    (small grids: the loop is store-bound and the prologue is not)
    constexpr bool kWiden = sizeof(QT) == 2 && RL == 2;
    using RT = typename std::conditional<kWiden, float, QT>::type;
    if constexpr (kWiden) {
        for (int n = warp; n < N; n += nwarps) {
            const unsigned char* src = raw + (size_t)n * p.raw_bytes;
            float* dst = recs + (size_t)n * p.rec_floats;
            for (int c = lane; c < per_node; c += 32)
                Widen<QT>::store(dst + 8 * c, *reinterpret_cast<const uint4*>(src + 16 * c));
        }
        __syncthreads();
    }
    const RT* rt = kWiden ? reinterpret_cast<const RT*>(recs) : reinterpret_cast<const RT*>(raw);
    const uint32_t rt_elems = kWiden ? p.rec_floats : p.raw_bytes / (uint32_t)sizeof(QT);
    // 8. k . q of every node (outputs read the pre-update state)
    for (int n = warp; n < N; n += nwarps) {
        const float kq = node_kq<DK, RT>(rt + (size_t)n * rt_elems, lane);
        if (lane == 0)
            ab[2 * N + n] = kq;
    }
    __syncthreads();

    StagedCtx<DK, RL, RT> ctx{rt, ab, rt_elems, N, L};
    if constexpr (TREE == kTreeChain)
        walk<DK, RL, ST, true>(S, p, NoTree{}, slotbuf, sin_head, b, h, row0, L, ctx);
    else if constexpr (TREE == kTreeIndex)
        walk<DK, RL, ST, false>(S, p, IndexTree{tsm}, slotbuf, sin_head, b, h, row0, L, ctx);
    else if constexpr (TREE == kTreeWarp)
        walk<DK, RL, ST, false>(S, p, MaskTree{tsm}, slotbuf, sin_head, b, h, row0, L, ctx);
    else
        walk<DK, RL, ST, false>(S, p, SmemTree{tv, N, warp}, slotbuf, sin_head, b, h, row0, L, ctx);
}

// ---------------------------------------------------------------------------
// Ring kernel: a producer warp streams chunks of walk positions
// ---------------------------------------------------------------------------

template <int DK, int RL, typename QT>
struct GlobalFetch {
    const QT* kg;
    const QT* vg;
    const float* g;
    const float* beta;
    size_t bN;  // b * N
    int Hk, Hv, dv, hk, h, row0;
    LaneMap<DK, RL> L;
    __device__ __forceinline__ void operator()(int y, float2 (&k2)[8], float (&vr)[RL], float& a,
                                               float& be) const
    {
        const size_t node = bN + y;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float4 x = Widen<QT>::load4(kg + (node * Hk + hk) * DK + L.col(m));
            k2[2 * m] = make_float2(x.x, x.y);
            k2[2 * m + 1] = make_float2(x.z, x.w);
        }
#pragma unroll
        for (int r = 0; r < RL; ++r)
            vr[r] = Widen<QT>::load1(vg + (node * Hv + h) * dv + row0 + L.rloc[r]);
        const size_t gi = node * Hv + h;
        a = gdn_gate(__ldg(g + gi));
        be = __ldg(beta + gi);
    }
};

template <int DK, int RL, typename QT>
struct RingCtx {
    uint64_t* full;
    uint64_t* empty;
    const float* ring;  // kRing slots of [kChunk records | a | beta | k.q, kChunk each]
    uint32_t rec_floats;
    uint32_t slot_floats;
    int32_t* status;
    int lane;
    GlobalFetch<DK, RL, QT> gf;
    __device__ __forceinline__ const float* slot(int pos) const
    {
        return ring + (size_t)((pos / kChunk) % kRing) * slot_floats;
    }
    __device__ __forceinline__ bool begin(int pos)
    {
        if (pos % kChunk == 0) {
            const int c = pos / kChunk;
            if (!mbar_wait(&full[c % kRing], (c / kRing) & 1)) {
                report_status(status, kStatusTimeout);
                return false;
            }
        }
        return true;
    }
    // Releases a slot after its last position (the walk's final, partial
    // chunk is never refilled, so it needs no release).
    __device__ __forceinline__ void end(int pos)
    {
        if (pos % kChunk == kChunk - 1) {
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[(pos / kChunk) % kRing]);
        }
    }
    __device__ __forceinline__ const float* rec(int pos, int) const
    {
        return slot(pos) + (size_t)(pos % kChunk) * rec_floats;
    }
    __device__ __forceinline__ void ab(int pos, int, float& a, float& be, float& kq) const
    {
        const float* s = slot(pos) + (size_t)kChunk * rec_floats;
        a = s[pos % kChunk];
        be = s[kChunk + pos % kChunk];
        kq = s[2 * kChunk + pos % kChunk];
    }
    __device__ __forceinline__ GlobalFetch<DK, RL, QT> fetcher() const { return gf; }
};

template <int DK, int RL, typename QT, typename ST, int TREE>
__global__ void __launch_bounds__((kMaxWarps + 1) * 32) gdn_verify_ring(const KParams p)
{
    constexpr bool CHAIN = TREE == kTreeChain;
    constexpr bool INDEX = TREE == kTreeIndex;
    constexpr int EPC = 16 / sizeof(QT);            // elements per 16-byte chunk
    constexpr int QKCH = DK / EPC;                  // chunks per k (or q) row
    constexpr int RPW = LaneMap<DK, RL>::RPW;
    constexpr int VCH_MAX = kMaxWarps * RPW / EPC;  // chunks per v slice, upper bound
    constexpr int MAXT = (kChunk * (2 * QKCH + VCH_MAX) + 31) / 32;

    extern __shared__ __align__(16) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kRing;
    float* ring = reinterpret_cast<float*>(smem + p.off_rec);
    const uint32_t slot_floats = kChunk * p.rec_floats + 3 * kChunk;
    float* slotbuf = reinterpret_cast<float*>(smem + p.off_slots);
    const TreeView T(reinterpret_cast<int*>(smem + p.off_tree), p.N);

    const int N = p.N;
    const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int hk = h / p.G;
    const int row0 = tile * p.rows;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const QT* kg = static_cast<const QT*>(p.k);
    const QT* qg = static_cast<const QT*>(p.q);
    const QT* vg = static_cast<const QT*>(p.v);
    if (!p.early_tree)
        pdl_wait_then_release();

    if (tid == 0) {
        for (int i = 0; i < kRing; ++i) {
            mbar_init(&full[i], 32);
            mbar_init(&empty[i], p.warps);
        }
        mbar_init_fence();
    }
    bool ok = true;
    if constexpr (CHAIN || INDEX) {
        bool bad = false;
        if (INDEX || p.validate) {
            for (int n = tid; n < N; n += blockDim.x) {
                const int pn = __ldg(p.parent + (size_t)b * N + n);
                if (INDEX) {
                    T.par[n] = pn;
                    bad |= (n == 0) ? (pn != -1) : (pn < 0 || pn >= n);
                } else {
                    bad |= pn != n - 1;
                }
            }
        }
        ok = !__syncthreads_or(bad);
    } else {
        __syncthreads();
        ok = build_walk(p.parent + (size_t)b * N, N, p.slots, p.reload != 0, T);
    }
    if (p.early_tree)
        pdl_wait_then_release();
    if (!ok) {
        if (tid == 0)
            report_status(p.status, GDN_ERR_BAD_TREE);
        return;
    }
    const int n_chunks = (N + kChunk - 1) / kChunk;

    if (warp == p.warps) {
        // ------------------------------------------------------------ producer
        const int vch = p.rows / EPC;
        const int per_pos = 2 * QKCH + vch;
        for (int c = 0; c < n_chunks; ++c) {
            const int s = c % kRing, use = c / kRing;
            if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1)) {
                report_status(p.status, kStatusTimeout);
                return;
            }
            float* base = ring + (size_t)s * slot_floats;
            const int p0 = c * kChunk;
            const int cnt = min(kChunk, N - p0);
            const int total = cnt * per_pos;
            uint4 regs[MAXT];
#pragma unroll
            for (int t = 0; t < MAXT; ++t) {
                const int idx = lane + 32 * t;
                if (idx < total) {
                    const int i = idx / per_pos, j = idx - i * per_pos;
                    const int pos = p0 + i;
                    const int n = (CHAIN || INDEX) ? pos : meta_node(T.meta[pos]);
                    const size_t node = (size_t)b * N + n;
                    const QT* src;
                    if (j < QKCH)
                        src = kg + (node * p.Hk + hk) * DK + j * EPC;
                    else if (j < 2 * QKCH)
                        src = qg + (node * p.Hk + hk) * DK + (j - QKCH) * EPC;
                    else
                        src = vg + (node * p.Hv + h) * p.dv + row0 + (j - 2 * QKCH) * EPC;
                    regs[t] = __ldg(reinterpret_cast<const uint4*>(src));
                }
            }
            if (lane < cnt) {
                const int pos = p0 + lane;
                const int n = (CHAIN || INDEX) ? pos : meta_node(T.meta[pos]);
                const size_t gi = ((size_t)b * N + n) * p.Hv + h;
                base[kChunk * p.rec_floats + lane] = gdn_gate(__ldg(p.g + gi));
                base[kChunk * p.rec_floats + kChunk + lane] = __ldg(p.beta + gi);
            }
#pragma unroll
            for (int t = 0; t < MAXT; ++t) {
                const int idx = lane + 32 * t;
                if (idx < total) {
                    const int i = idx / per_pos, j = idx - i * per_pos;
                    Widen<QT>::store(base + (size_t)i * p.rec_floats + j * EPC, regs[t]);
                }
            }
            __syncwarp();
            for (int i = 0; i < cnt; ++i) {
                const float kq = node_kq<DK, float>(base + (size_t)i * p.rec_floats, lane);
                if (lane == 0)
                    base[kChunk * p.rec_floats + 2 * kChunk + i] = kq;
            }
            mbar_arrive(&full[s]);
        }
        return;
    }

    // ---------------------------------------------------------------- compute
    const LaneMap<DK, RL> L(warp, lane);
    const float* sin_head = p.state_in + ((size_t)b * p.Hv + h) * p.dv * DK + (size_t)row0 * DK;
    StateT<RL> S;
    load_state<DK, RL>(S, sin_head, L);
    const GlobalFetch<DK, RL, QT> gf{kg, vg, p.g, p.beta, (size_t)b * N, p.Hk, p.Hv, p.dv, hk, h, row0, L};
    RingCtx<DK, RL, QT> ctx{full, empty, ring, p.rec_floats, slot_floats, p.status, lane, gf};
    if constexpr (CHAIN)
        walk<DK, RL, ST, true>(S, p, NoTree{}, slotbuf, sin_head, b, h, row0, L, ctx);
    else if constexpr (INDEX)
        walk<DK, RL, ST, false>(S, p, IndexTree{T.par}, slotbuf, sin_head, b, h, row0, L, ctx);
    else
        walk<DK, RL, ST, false>(S, p, SmemTree{T, N, warp}, slotbuf, sin_head, b, h, row0, L, ctx);
}

// ---------------------------------------------------------------------------
// Host-side launch
// ---------------------------------------------------------------------------

// Opts kernel Kern in to more than 48 KB of dynamic shared memory, once per
// device for the largest size requested so far (one cache per kernel).
template <auto Kern>
cudaError_t grant_smem(size_t smem)
{
    if (smem <= 48 * 1024)
        return cudaSuccess;
    static std::atomic<int> granted[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev >= 0 && dev < kMaxDevices && granted[dev].load() >= (int)smem)
        return cudaSuccess;
    e = cudaFuncSetAttribute(Kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return e;
    if (dev >= 0 && dev < kMaxDevices) {
        int cur = granted[dev].load();
        while (cur < (int)smem && !granted[dev].compare_exchange_weak(cur, (int)smem)) {
        }
    }
    return cudaSuccess;
}

template <int DK, int RL, typename QT, typename ST, int TREE>
cudaError_t launch_staged(const KParams& kp, const VerifyArgs& a, const VerifyGeom& geom,
                          cudaStream_t stream)
{
    dim3 grid(geom.tiles, a.n_v_heads, a.batch);
    cudaError_t e = grant_smem<gdn_verify_staged<DK, RL, QT, ST, TREE>>(geom.smem);
    if (e != cudaSuccess)
        return e;
    return launch_pdl(gdn_verify_staged<DK, RL, QT, ST, TREE>, grid, dim3(geom.warps * 32), geom.smem,
                      stream, kp);
}

template <int DK, int RL, typename QT, typename ST, int TREE>
cudaError_t launch_ring(const KParams& kp, const VerifyArgs& a, const VerifyGeom& geom,
                        cudaStream_t stream)
{
    dim3 grid(geom.tiles, a.n_v_heads, a.batch);
    cudaError_t e = grant_smem<gdn_verify_ring<DK, RL, QT, ST, TREE>>(geom.smem);
    if (e != cudaSuccess)
        return e;
    return launch_pdl(gdn_verify_ring<DK, RL, QT, ST, TREE>, grid, dim3((geom.warps + 1) * 32),
                      geom.smem, stream, kp);
}

template <int DK, int RL, typename QT, typename ST, bool CHAIN>
cudaError_t launch_one(const KParams& kp, const VerifyArgs& a, const VerifyGeom& geom,
                       cudaStream_t stream)
{
    if (geom.staged) {
        if (CHAIN)
            return launch_staged<DK, RL, QT, ST, kTreeChain>(kp, a, geom, stream);
        if (geom.reload)
            return launch_staged<DK, RL, QT, ST, kTreeIndex>(kp, a, geom, stream);
        if (geom.warp_tree)
            return launch_staged<DK, RL, QT, ST, kTreeWarp>(kp, a, geom, stream);
        return launch_staged<DK, RL, QT, ST, kTreeSmem>(kp, a, geom, stream);
    }
    if (CHAIN)
        return launch_ring<DK, RL, QT, ST, kTreeChain>(kp, a, geom, stream);
    if (geom.reload)
        return launch_ring<DK, RL, QT, ST, kTreeIndex>(kp, a, geom, stream);
    return launch_ring<DK, RL, QT, ST, kTreeSmem>(kp, a, geom, stream);
}

template <int DK, int RL, typename QT, typename ST>
cudaError_t launch_mode(const KParams& kp, const VerifyArgs& a, const VerifyGeom& g, cudaStream_t s)
{
    if (a.flags & GDN_FLAG_CHAIN)
        return launch_one<DK, RL, QT, ST, true>(kp, a, g, s);
    return launch_one<DK, RL, QT, ST, false>(kp, a, g, s);
}

template <int DK, int RL, typename QT>
cudaError_t launch_state(const KParams& kp, const VerifyArgs& a, const VerifyGeom& g, cudaStream_t s)
{
    if (a.state_dtype == GDN_F16)
        return launch_mode<DK, RL, QT, __half>(kp, a, g, s);
    return launch_mode<DK, RL, QT, float>(kp, a, g, s);
}

template <int DK, int RL>
cudaError_t launch_qkv(const KParams& kp, const VerifyArgs& a, const VerifyGeom& g, cudaStream_t s)
{
    if (a.qkv_dtype == GDN_BF16)
        return launch_state<DK, RL, __nv_bfloat16>(kp, a, g, s);
    return launch_state<DK, RL, float>(kp, a, g, s);
}

// Launches the verify kernel for head dim DK (instantiated once per DK, in
// gdn_verify_d{32,64,128}.cu).
template <int DK>
cudaError_t launch_dk(const KParams& kp, const VerifyArgs& a, const VerifyGeom& g, cudaStream_t s)
{
    if (g.rows_per_lane == 1)
        return launch_qkv<DK, 1>(kp, a, g, s);
    return launch_qkv<DK, 2>(kp, a, g, s);
}


}  // namespace verify
}  // namespace gdn
