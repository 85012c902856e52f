// gdn_verify.cuh -- the tree-verify kernels of libgdntree (sm_100a), as
// templates; gdn_verify_d{32,64,128}.cu instantiate them per head dim.
//
// One CTA per (sequence b, v-head h, tile of d_v rows).  The CTA walks the
// tree's nodes in a topological order and for each node applies the gated
// delta rule (Gated DeltaNet; the ggml_gated_delta_net recurrence named in
// the GreenGames post, "TL;DR"):
//
//     a = exp(g_n);  w = a * S_p k_n;  u = beta_n * (v_n - w)
//     S_n = a * S_p + u k_n^T;         o_n = scale * S_n q_n
//
// and persists S_n from inside the kernel (the GreenGames post, "Key wins":
// persist-write kernel, f16 intermediate cache).  The output is formed from
// the parent state, o_n = scale * (a * (S_p q_n) + u * (k_n . q_n)), so S_p q
// is reduced together with S_p k.
//
// Compute layout.  A state row of d_k columns is split into chunks of 8
// consecutive columns; a lane holds C chunks of each of its RL rows (C = 1 or
// 2, RL = 1 or 2), so LR = d_k / (8 C) lanes share a row and a warp owns
// RL * 32 / LR rows.  The shape is picked per launch from the size of the
// grid: (C, RL) = (2, 2) for large batches, (2, 1) for small ones (twice the
// warps to hide the per-node dependency chain); the templates also take
// C = 1, which is not instantiated.  A row's arithmetic is the same in every
// shape:
// each chunk's partial dot product is a chain of four packed-fp32 (FFMA2)
// steps, chunks c and c + d_k / 16 are added next, then an xor butterfly
// adds the rest in a fixed order.  So results never depend on the shape.
//
// Node inputs stay in their storage type in shared memory: each node's
// record is its k row, its q row and the CTA's slice of v, copied with
// 16-byte cp.async; the node loop widens each lane's 16-byte chunks (exact
// for bf16).  Two kernels:
//   * gdn_verify_staged: trees and chains small enough to stage whole.  The
//     copies of every node's record are issued at kernel start and overlap
//     the tree work and the state_in load; a prologue pass then writes one
//     32-byte descriptor per walk position (node, tree metadata, a, beta,
//     k . q).  Trees of up to 32 nodes have their walk built by one warp
//     (build_warp_walk), larger ones by the whole CTA (build_walk).
//   * gdn_verify_ring: anything larger (long chains, large trees).  A
//     producer warp streams records and descriptors of chunks of walk
//     positions through a ring of mbarrier-guarded slots.
//
// Parents that are not the previous node of the walk: with exact f32
// persistence the walk goes in index order and the parent's state is re-read
// from node_states (written by the same thread, bit-exact), prefetched one
// node ahead.  Otherwise the walk is a depth-first preorder visiting each
// node's children by increasing subtree size (ties by index), so the largest
// child subtree comes last; a node with two or more children saves its f32
// state in a shared-memory stack slot, and a later child reloads it.  The
// slot index is the number of edges on the node's root path that enter a
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

constexpr int kMaxWarps = 8;    // compute warps per CTA, at most
constexpr int kSmallWarps = 4;  // compute warps per CTA, usually
constexpr int kChunk = 8;     // walk positions per ring slot
constexpr int kRing = 3;      // ring slots
constexpr int kMaxDevices = 64;
constexpr int kStagedMaxSmem = 112 * 1024;

// Per-position walk metadata (tree mode), packed in one int32:
//   bits 0..15 node id, 16..18 source of the parent state,
//   bits 19..23 save slot + 1 (0: do not save), 24..28 load slot.
enum : int { kSrcCont = 0, kSrcSlot = 1, kSrcRecompute = 2, kSrcRoot = 3, kSrcReload = 4 };

__device__ __forceinline__ int meta_node(int m) { return m & 0xffff; }
__device__ __forceinline__ int meta_src(int m) { return (m >> 16) & 7; }
__device__ __forceinline__ int meta_save(int m) { return ((m >> 19) & 31) - 1; }
__device__ __forceinline__ int meta_load(int m) { return (m >> 24) & 31; }

// A node's decay a and write strength beta from its g and beta inputs,
// compiled once so that every caller gets identical bits: a = exp(g).  With
// raw gates (GDN_FLAG_GATES) g and beta hold x and y with g = -softplus(x)
// and beta = sigmoid(y), so a = exp(-softplus(x)) = 1 / (1 + e^x) and
// beta = 1 / (1 + e^-y) (x = +inf gives a = 0, a reset).
static __device__ __noinline__ float2 gdn_gates(float g, float beta, int raw)
{
    if (raw)
        return make_float2(__fdiv_rn(1.f, __fadd_rn(1.f, expf(g))), __fdiv_rn(1.f, __fadd_rn(1.f, expf(-beta))));
    return make_float2(expf(g), beta);
}

__device__ __forceinline__ void gate_scalars(float g, float beta, int raw, float& a, float& be)
{
    const float2 r = gdn_gates(g, beta, raw);
    a = r.x;
    be = r.y;
}

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
    int persist_last, validate, early_tree;
    int prefetch;        // early_tree on a small layer: L2 prefetch of the records before the wait
    int qk_norm;         // GDN_FLAG_QK_L2NORM: k and q normalised per node inside the kernel
    int gates;           // GDN_FLAG_GATES: g and beta are raw (gate_scalars)
    float* ws;           // global stack slots (kTreeGlobal kinds): slots x rows x d_k per CTA
    int tmem_cols;       // tensor-memory stack slots (kTreeTmem kinds): columns allocated per CTA
    int tmem_slot_cols;  // ... and columns from one slot to the next
    const int32_t* cu;   // varlen: [B + 1] node offsets of the packed layout (N: the most per sequence)
    int total;           // varlen: nodes in the packed layout
    uint32_t raw_bytes;  // one node's record (k row | q row | v slice) in bytes
    uint32_t off_raw, off_desc, off_ab, off_slots, off_tree;
    const int32_t* plan;  // optional: walks built by gdn_tree_plan (see kPlanHeader), else NULL
    int plan_stride;      // int32 per sequence in the plan
    int plan_sig;         // the signature the plan must carry
};

// A tree plan holds, per sequence, a header [signature, ok, N, 0] and then
// the walk as the staged kernels keep it in shared memory: for trees of <= 32
// nodes MaskTree's 128 ints, else TreeView's par | ord | meta | rstart.
constexpr int kPlanHeader = 4;

// The nodes of sequence b: n0 .. n0 + N - 1 of the node dimension (N = p.N
// and n0 = b N, or from the varlen offsets).
struct Seq {
    int n0, N;
};

// Reads sequence b's node range; false (on every thread) if the varlen
// offsets are out of range.
__device__ __forceinline__ bool seq_of(const KParams& p, int b, Seq& q)
{
    if (p.cu == nullptr) {
        q.n0 = b * p.N;
        q.N = p.N;
        return true;
    }
    q.n0 = __ldg(p.cu + b);
    q.N = __ldg(p.cu + b + 1) - q.n0;
    return q.n0 >= 0 && q.N >= 1 && q.N <= p.N && q.n0 <= p.total - q.N;
}

// One walk position: its node and tree metadata, and the node's scalars.
// With qk_norm, each position (ring) or node (staged) also has an output
// coefficient scale / |q|, kept beside the descriptors so that they stay 32
// bytes.
struct PosDesc {
    int4 i;    // node, metadata, recomputation start, parent
    float4 f;  // a = exp(g), beta', k . q, a' (see node_scalars)
};

// A node's scalars for the state step.  With q and k normalised inside the
// kernel (qk_norm; rk = 1 / |k|, rq = 1 / |q|) the step runs on the raw
// k, q: with S k^ = rk (S k) and u = beta (v - a S_p k^),
//     u' = rk u = (beta rk) (v - (a rk) (S_p k)),   S_n = a S_p + u' k^T,
//     o = scale S_n q^ = (scale rq) (a (S_p q) + u' (k . q)),
// so beta' = beta rk, a' = a rk and the output coefficient scale rq.
// Without it rk = rq = 1: beta' = beta, a' = a (bit for bit).
__device__ __forceinline__ void node_scalars(float a, float beta, float rk, float& beta_p, float& a_p)
{
    beta_p = __fmul_rn(beta, rk);
    a_p = __fmul_rn(a, rk);
}

// 1 / |x| from the sum of squares (epsilon 0: a zero vector gives inf).
__device__ __forceinline__ float inv_norm(float ss) { return __fdiv_rn(1.f, __fsqrt_rn(ss)); }

// ---------------------------------------------------------------------------
// Lane geometry and per-node arithmetic
// ---------------------------------------------------------------------------

template <int DK, int C, int RL>
struct LaneMap {
    static constexpr int E = 8 * C;     // state columns per lane and row
    static constexpr int LR = DK / E;   // lanes per row
    static constexpr int RG = 32 / LR;  // row groups per warp
    static constexpr int RPW = RL * RG; // rows per warp
    int cl;                             // lane within its row: chunks cl, cl + LR
    int row;                            // the lane's first row in the tile; then every RG rows
    __device__ __forceinline__ LaneMap(int warp, int lane) : cl(lane % LR), row(warp * RPW + lane / LR)
    {
    }
    // first column of chunk c of this lane
    __device__ __forceinline__ int col(int c) const { return 8 * (cl + c * LR); }
    // offset of this lane's first element in a [rows][DK] row-major tile
    __device__ __forceinline__ int tile_offset() const { return row * DK + 8 * cl; }
    // f32 records (see swz_pos): where the low and high 16-byte halves of
    // this lane's chunks sit, relative to the chunk start of chunk cl
    __device__ __forceinline__ int swz_lo() const { return 8 * cl + 4 * ((cl >> 2) & 1); }
    __device__ __forceinline__ int swz_hi() const { return 8 * cl + 4 * (((cl >> 2) & 1) ^ 1); }
};

// f32 records in shared memory: chunk j (8 floats) of a k or q row has its
// two 16-byte halves swapped when bit 2 of (j mod LR) is set, so the 8 lanes
// of a quarter warp, which read chunks cl = 0..7 of a row, hit 8 distinct
// 4-bank groups.  Position of element e of a row:
template <int LR>
__device__ __forceinline__ int swz_pos(int e)
{
    const int j = e >> 3, w = e & 7;
    return 8 * j + ((((w >> 2) ^ (((j % LR) >> 2) & 1))) << 2) + (w & 3);
}

template <int C, int RL>
struct StateT {
    float2 s[RL][4 * C];
};

// Sum of one chunk's 8 products x * y (pairs t = 0..3): a chain of packed
// FMAs, then the two halves.
__device__ __forceinline__ float chunk_dot(const float2* x, const float2* y)
{
    float2 acc = __fmul2_rn(x[0], y[0]);
    acc = __ffma2_rn(x[1], y[1], acc);
    acc = __ffma2_rn(x[2], y[2], acc);
    acc = __ffma2_rn(x[3], y[3], acc);
    return __fadd_rn(acc.x, acc.y);
}

// Adds up the chunk sums of a row across its LR lanes.  C = 2: the lane's two
// chunks (cl, cl + LR) first, then lanes xor 1, 2, .. LR / 2.  C = 1: lanes
// xor LR / 2 first (chunks c and c + LR / 2, the same pair), then 1, 2, ...
// LR / 4.  Both orders add the same operands in the same sequence.
template <int LR, int C>
__device__ __forceinline__ float row_sum_first(const float (&cs)[C])
{
    if constexpr (C == 2)
        return __fadd_rn(cs[0], cs[1]);
    else
        return __fadd_rn(cs[0], __shfl_xor_sync(0xffffffffu, cs[0], LR / 2));
}

// One node's state update on a lane's RL rows x 8C columns.  Shared by the
// walk and the recompute path; explicit intrinsics keep both bit-identical.
// With WITH_Q it also returns pq = S_p q (reduced in the same butterfly as
// S_p k) and u: the output is then o = scale * (a * pq + u * (k . q)) =
// scale * S_n q, with S_n = a S_p + u k^T.
template <int LR, int C, int RL, bool WITH_Q>
__device__ __forceinline__ void gdn_step(StateT<C, RL>& S, const float2 (&k2)[4 * C],
                                         const float2 (&q2)[4 * C], const float (&vr)[RL], float a,
                                         float a_read, float beta, float (&pq)[RL], float (&uo)[RL])
{
    float w[RL];
#pragma unroll
    for (int r = 0; r < RL; ++r) {
        float cw[C], cq[C];
#pragma unroll
        for (int c = 0; c < C; ++c) {
            cw[c] = chunk_dot(&S.s[r][4 * c], &k2[4 * c]);
            if constexpr (WITH_Q)
                cq[c] = chunk_dot(&S.s[r][4 * c], &q2[4 * c]);
        }
        w[r] = row_sum_first<LR, C>(cw);
        if constexpr (WITH_Q)
            pq[r] = row_sum_first<LR, C>(cq);
    }
    constexpr int BL = C == 2 ? LR : LR / 2;  // lanes still to be added after the first step
#pragma unroll
    for (int off = 1; off < BL; off <<= 1) {
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
        const float u = __fmul_rn(beta, __fsub_rn(vr[r], __fmul_rn(a_read, w[r])));
        uo[r] = u;
        const float2 u2 = make_float2(u, u);
#pragma unroll
        for (int t = 0; t < 4 * C; ++t)
            S.s[r][t] = __ffma2_rn(u2, k2[t], __fmul2_rn(a2, S.s[r][t]));
    }
}

// State update only (recompute path): the same instructions on S.
template <int LR, int C, int RL>
__device__ __forceinline__ void gdn_update(StateT<C, RL>& S, const float2 (&k2)[4 * C],
                                           const float (&vr)[RL], float a, float a_read, float beta)
{
    float pq[RL], uo[RL];
    gdn_step<LR, C, RL, false>(S, k2, k2, vr, a, a_read, beta, pq, uo);
}

// Element e of the k (part 0) or q (part DK) row of a shared-memory record:
// raw bf16 rows are plain, f32 rows swizzled (swz_pos).
template <int DK, int LR>
__device__ __forceinline__ float rec_elem(const __nv_bfloat16* rec, int part, int e)
{
    return Widen<__nv_bfloat16>::lds1(rec + part + e);
}
template <int DK, int LR>
__device__ __forceinline__ float rec_elem(const float* rec, int part, int e)
{
    return rec[part + swz_pos<LR>(e)];
}

// k . q of one node's record, reduced by a group of 8 lanes (sub = lane % 8;
// a warp handles four nodes at once; every lane of the warp must call it).
// The same reduction wherever it is computed.
template <int DK, int LR, typename RT>
__device__ __forceinline__ float node_kq8(const RT* rec, int sub);

// bf16 records: lane sub of the group takes the DK / 8 consecutive elements
// [DK / 8 * sub, DK / 8 * (sub + 1)) of a row, in 16-byte loads (8-byte at
// DK = 32), widened to pairs.
template <int DK>
__device__ __forceinline__ void row_part8(const __nv_bfloat16* rec, int part, int sub, float2 (&x)[DK / 16])
{
    constexpr int E = DK / 8;
    const __nv_bfloat16* base = rec + part + E * sub;
    if constexpr (E >= 8) {
#pragma unroll
        for (int c = 0; c < E / 8; ++c) {
            float2 y[4];
            Widen<__nv_bfloat16>::lds8(base + 8 * c, y);
#pragma unroll
            for (int t = 0; t < 4; ++t)
                x[4 * c + t] = y[t];
        }
    } else {
        const uint2 u = *reinterpret_cast<const uint2*>(base);
        x[0] = bf16x2_to_float2(u.x);
        x[1] = bf16x2_to_float2(u.y);
    }
}

// x . y over a group of 8 lanes holding row_part8 pieces: the lane's pairs
// in order with packed FMAs, its two halves, then the xor butterfly.
template <int NP>
__device__ __forceinline__ float group_dot8(const float2 (&x)[NP], const float2 (&y)[NP])
{
    float2 acc = __fmul2_rn(x[0], y[0]);
#pragma unroll
    for (int t = 1; t < NP; ++t)
        acc = __ffma2_rn(x[t], y[t], acc);
    float s = __fadd_rn(acc.x, acc.y);
#pragma unroll
    for (int off = 4; off >= 1; off >>= 1)
        s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, off));
    return s;
}

// x . y of two rows of one node's record (part 0: k, part DK: q), reduced
// by a group of 8 lanes like node_kq8.
template <int DK, int LR, typename RT>
__device__ __forceinline__ float node_dot8(const RT* rec, int sub, int pa, int pb)
{
    if constexpr (sizeof(RT) == 2) {
        float2 x[DK / 16], y[DK / 16];
        row_part8<DK>(rec, pa, sub, x);
        row_part8<DK>(rec, pb, sub, y);
        return group_dot8(x, y);
    }
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int j = sub; j < DK; j += 16) {
        acc0 = __fmaf_rn(rec_elem<DK, LR>(rec, pa, j), rec_elem<DK, LR>(rec, pb, j), acc0);
        acc1 = __fmaf_rn(rec_elem<DK, LR>(rec, pa, j + 8), rec_elem<DK, LR>(rec, pb, j + 8), acc1);
    }
    float acc = __fadd_rn(acc0, acc1);
#pragma unroll
    for (int off = 4; off >= 1; off >>= 1)
        acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
    return acc;
}

// k . q, k . k and q . q of one node's record in one pass, each summed in
// exactly node_kq8's order (so kq is bit-identical to it).  Not unrolled: it
// runs in prologues only with GDN_FLAG_QK_L2NORM, and unrolled it would set
// the register count of the whole kernel.
template <int DK, int LR, typename RT>
__device__ __forceinline__ void node_dots8(const RT* rec, int sub, float& kq, float& kk, float& qq)
{
    if constexpr (sizeof(RT) == 2) {
        float2 x[DK / 16], y[DK / 16];
        row_part8<DK>(rec, 0, sub, x);
        row_part8<DK>(rec, DK, sub, y);
        kq = group_dot8(x, y);
        kk = group_dot8(x, x);
        qq = group_dot8(y, y);
        return;
    }
    float q0 = 0.f, q1 = 0.f, k0 = 0.f, k1 = 0.f, s0 = 0.f, s1 = 0.f;
#pragma unroll 1
    for (int j = sub; j < DK; j += 16) {
        const float ka = rec_elem<DK, LR>(rec, 0, j), qa = rec_elem<DK, LR>(rec, DK, j);
        const float kb = rec_elem<DK, LR>(rec, 0, j + 8), qb = rec_elem<DK, LR>(rec, DK, j + 8);
        q0 = __fmaf_rn(ka, qa, q0);
        q1 = __fmaf_rn(kb, qb, q1);
        k0 = __fmaf_rn(ka, ka, k0);
        k1 = __fmaf_rn(kb, kb, k1);
        s0 = __fmaf_rn(qa, qa, s0);
        s1 = __fmaf_rn(qb, qb, s1);
    }
    kq = __fadd_rn(q0, q1);
    kk = __fadd_rn(k0, k1);
    qq = __fadd_rn(s0, s1);
#pragma unroll
    for (int off = 4; off >= 1; off >>= 1) {
        kq = __fadd_rn(kq, __shfl_xor_sync(0xffffffffu, kq, off));
        kk = __fadd_rn(kk, __shfl_xor_sync(0xffffffffu, kk, off));
        qq = __fadd_rn(qq, __shfl_xor_sync(0xffffffffu, qq, off));
    }
}

template <int DK, int LR, typename RT>
__device__ __forceinline__ float node_kq8(const RT* rec, int sub)
{
    if constexpr (sizeof(RT) == 2)
        return node_dot8<DK, LR>(rec, sub, 0, DK);
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int j = sub; j < DK; j += 16) {
        acc0 = __fmaf_rn(rec_elem<DK, LR>(rec, 0, j), rec_elem<DK, LR>(rec, DK, j), acc0);
        acc1 = __fmaf_rn(rec_elem<DK, LR>(rec, 0, j + 8), rec_elem<DK, LR>(rec, DK, j + 8), acc1);
    }
    float acc = __fadd_rn(acc0, acc1);
#pragma unroll
    for (int off = 4; off >= 1; off >>= 1)
        acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
    return acc;
}

// ---------------------------------------------------------------------------
// State and record access.  Row-layout accesses take a pointer already at
// the lane's first element (LaneMap::tile_offset), so every other offset is
// a compile-time constant.
// ---------------------------------------------------------------------------

// S <- this lane's part of a row-major f32 tile in global memory (32-byte
// aligned): one 32-byte plain load per chunk, so a state this thread stored
// earlier in the kernel is seen.
template <int DK, int C, int RL>
__device__ __forceinline__ void load_rows(StateT<C, RL>& S, const float* lane_ptr)
{
    using LM = LaneMap<DK, C, RL>;
#pragma unroll
    for (int r = 0; r < RL; ++r) {
#pragma unroll
        for (int c = 0; c < C; ++c) {
            float4 x, y;
            ld_global_v8(lane_ptr + r * LM::RG * DK + c * 8 * LM::LR, x, y);
            S.s[r][4 * c + 0] = make_float2(x.x, x.y);
            S.s[r][4 * c + 1] = make_float2(x.z, x.w);
            S.s[r][4 * c + 2] = make_float2(y.x, y.y);
            S.s[r][4 * c + 3] = make_float2(y.z, y.w);
        }
    }
}

// Persisted-state stores of one chunk (8 values) in f32 (one 32-byte store)
// or f16 (RNE, one 16-byte store): the lanes of a row cover whole sectors.
template <typename ST>
struct Persist;

template <>
struct Persist<float> {
    __device__ __forceinline__ static void store8(float* dst, const float2* x)
    {
        st_global_v8(dst, make_float4(x[0].x, x[0].y, x[1].x, x[1].y), make_float4(x[2].x, x[2].y, x[3].x, x[3].y));
    }
};

template <>
struct Persist<__half> {
    __device__ __forceinline__ static void store8(__half* dst, const float2* x)
    {
        uint4 u;
        __half2 h;
        h = __float22half2_rn(x[0]);
        u.x = *reinterpret_cast<const uint32_t*>(&h);
        h = __float22half2_rn(x[1]);
        u.y = *reinterpret_cast<const uint32_t*>(&h);
        h = __float22half2_rn(x[2]);
        u.z = *reinterpret_cast<const uint32_t*>(&h);
        h = __float22half2_rn(x[3]);
        u.w = *reinterpret_cast<const uint32_t*>(&h);
        *reinterpret_cast<uint4*>(dst) = u;
    }
};

template <int DK, int C, int RL, typename ST>
__device__ __forceinline__ void persist(const StateT<C, RL>& S, ST* lane_ptr)
{
    using LM = LaneMap<DK, C, RL>;
#pragma unroll
    for (int r = 0; r < RL; ++r) {
#pragma unroll
        for (int c = 0; c < C; ++c)
            Persist<ST>::store8(lane_ptr + r * LM::RG * DK + c * 8 * LM::LR, &S.s[r][4 * c]);
    }
}

// Stack slots in shared memory are private to each lane: its 2 C RL float4
// lie `stride` floats apart (the CTA's thread count x 4), consecutive lanes
// in consecutive 16-byte words.
template <int C, int RL>
__device__ __forceinline__ void save_slot(const StateT<C, RL>& S, float* lane_slot, int stride)
{
#pragma unroll
    for (int r = 0; r < RL; ++r) {
#pragma unroll
        for (int j = 0; j < 2 * C; ++j)
            *reinterpret_cast<float4*>(lane_slot + (r * 2 * C + j) * stride) =
                make_float4(S.s[r][2 * j].x, S.s[r][2 * j].y, S.s[r][2 * j + 1].x, S.s[r][2 * j + 1].y);
    }
}

template <int C, int RL>
__device__ __forceinline__ void load_slot(StateT<C, RL>& S, const float* lane_slot, int stride)
{
#pragma unroll
    for (int r = 0; r < RL; ++r) {
#pragma unroll
        for (int j = 0; j < 2 * C; ++j) {
            const float4 x = *reinterpret_cast<const float4*>(lane_slot + (r * 2 * C + j) * stride);
            S.s[r][2 * j] = make_float2(x.x, x.y);
            S.s[r][2 * j + 1] = make_float2(x.z, x.w);
        }
    }
}

// Stack slots in tensor memory: a lane's 8 C RL floats are the 32-bit
// columns taddr .. taddr + 8 C RL - 1 of its TMEM lane (one warp-wide store
// or load of 32 columns).
template <int C, int RL>
__device__ __forceinline__ void tmem_save_slot(const StateT<C, RL>& S, uint32_t taddr)
{
    static_assert(8 * C * RL == 32, "tensor-memory slots hold 32 floats per lane");
    uint32_t r[32];
#pragma unroll
    for (int i = 0; i < RL; ++i) {
#pragma unroll
        for (int t = 0; t < 4 * C; ++t) {
            r[(i * 4 * C + t) * 2] = __float_as_uint(S.s[i][t].x);
            r[(i * 4 * C + t) * 2 + 1] = __float_as_uint(S.s[i][t].y);
        }
    }
    tmem_st32(taddr, r);
}

template <int C, int RL>
__device__ __forceinline__ void tmem_load_slot(StateT<C, RL>& S, uint32_t taddr)
{
    static_assert(8 * C * RL == 32, "tensor-memory slots hold 32 floats per lane");
    uint32_t r[32];
    tmem_ld32(taddr, r);
#pragma unroll
    for (int i = 0; i < RL; ++i) {
#pragma unroll
        for (int t = 0; t < 4 * C; ++t)
            S.s[i][t] = make_float2(__uint_as_float(r[(i * 4 * C + t) * 2]), __uint_as_float(r[(i * 4 * C + t) * 2 + 1]));
    }
}

// This lane's chunks of the k (part 0) or q (part DK) row of a shared-memory
// record: raw bf16 (widened here) or swizzled f32.
template <int DK, int C, int RL>
__device__ __forceinline__ void load_row8(const __nv_bfloat16* rec, int part, const LaneMap<DK, C, RL>& L,
                                          float2 (&x2)[4 * C])
{
#pragma unroll
    for (int c = 0; c < C; ++c) {
        float2 x[4];
        Widen<__nv_bfloat16>::lds8(rec + part + L.col(c), x);
#pragma unroll
        for (int t = 0; t < 4; ++t)
            x2[4 * c + t] = x[t];
    }
}

template <int DK, int C, int RL>
__device__ __forceinline__ void load_row8(const float* rec, int part, const LaneMap<DK, C, RL>& L,
                                          float2 (&x2)[4 * C])
{
    using LM = LaneMap<DK, C, RL>;
    const float* lo = rec + part + L.swz_lo();
    const float* hi = rec + part + L.swz_hi();
#pragma unroll
    for (int c = 0; c < C; ++c) {
        const float4 a = *reinterpret_cast<const float4*>(lo + c * 8 * LM::LR);
        const float4 b = *reinterpret_cast<const float4*>(hi + c * 8 * LM::LR);
        x2[4 * c + 0] = make_float2(a.x, a.y);
        x2[4 * c + 1] = make_float2(a.z, a.w);
        x2[4 * c + 2] = make_float2(b.x, b.y);
        x2[4 * c + 3] = make_float2(b.z, b.w);
    }
}

// One node's inputs for this lane as loaded from its shared-memory record,
// before widening: k and q chunks and the v values of the lane's rows.
template <typename RT, int C, int RL>
struct RawRec;

template <int C, int RL>
struct RawRec<__nv_bfloat16, C, RL> {
    uint4 k[C], q[C];
    uint32_t v[RL];
};

template <int C, int RL>
struct RawRec<float, C, RL> {
    float4 k[2 * C], q[2 * C];
    float v[RL];
};

template <int DK, int C, int RL>
__device__ __forceinline__ void fetch_raw(const __nv_bfloat16* rec, const LaneMap<DK, C, RL>& L,
                                          RawRec<__nv_bfloat16, C, RL>& R)
{
    using LM = LaneMap<DK, C, RL>;
#pragma unroll
    for (int c = 0; c < C; ++c) {
        R.k[c] = *reinterpret_cast<const uint4*>(rec + L.col(c));
        R.q[c] = *reinterpret_cast<const uint4*>(rec + DK + L.col(c));
    }
#pragma unroll
    for (int r = 0; r < RL; ++r)
        R.v[r] = *reinterpret_cast<const unsigned short*>(rec + 2 * DK + L.row + r * LM::RG);
}

template <int DK, int C, int RL>
__device__ __forceinline__ void fetch_raw(const float* rec, const LaneMap<DK, C, RL>& L,
                                          RawRec<float, C, RL>& R)
{
    using LM = LaneMap<DK, C, RL>;
    const float* lo = rec + L.swz_lo();
    const float* hi = rec + L.swz_hi();
#pragma unroll
    for (int c = 0; c < C; ++c) {
        R.k[2 * c] = *reinterpret_cast<const float4*>(lo + c * 8 * LM::LR);
        R.k[2 * c + 1] = *reinterpret_cast<const float4*>(hi + c * 8 * LM::LR);
        R.q[2 * c] = *reinterpret_cast<const float4*>(lo + DK + c * 8 * LM::LR);
        R.q[2 * c + 1] = *reinterpret_cast<const float4*>(hi + DK + c * 8 * LM::LR);
    }
#pragma unroll
    for (int r = 0; r < RL; ++r)
        R.v[r] = rec[2 * DK + L.row + r * LM::RG];
}

template <int C, int RL>
__device__ __forceinline__ void widen_raw(const RawRec<__nv_bfloat16, C, RL>& R, float2 (&k2)[4 * C],
                                          float2 (&q2)[4 * C], float (&vr)[RL])
{
#pragma unroll
    for (int c = 0; c < C; ++c) {
        float2 x[4], y[4];
        Widen<__nv_bfloat16>::pairs(R.k[c], x);
        Widen<__nv_bfloat16>::pairs(R.q[c], y);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            k2[4 * c + t] = x[t];
            q2[4 * c + t] = y[t];
        }
    }
#pragma unroll
    for (int r = 0; r < RL; ++r)
        vr[r] = __uint_as_float(R.v[r] << 16);
}

template <int C, int RL>
__device__ __forceinline__ void widen_raw(const RawRec<float, C, RL>& R, float2 (&k2)[4 * C],
                                          float2 (&q2)[4 * C], float (&vr)[RL])
{
#pragma unroll
    for (int c = 0; c < 2 * C; ++c) {
        k2[2 * c] = make_float2(R.k[c].x, R.k[c].y);
        k2[2 * c + 1] = make_float2(R.k[c].z, R.k[c].w);
        q2[2 * c] = make_float2(R.q[c].x, R.q[c].y);
        q2[2 * c + 1] = make_float2(R.q[c].z, R.q[c].w);
    }
#pragma unroll
    for (int r = 0; r < RL; ++r)
        vr[r] = R.v[r];
}

// k and the v slice of one node from its shared-memory record
// [k | q | v slice] (RT: raw bf16 or swizzled f32).
template <int DK, int C, int RL, typename RT>
__device__ __forceinline__ void load_k(const RT* rec, const LaneMap<DK, C, RL>& L, float2 (&k2)[4 * C],
                                       float (&vr)[RL])
{
    using LM = LaneMap<DK, C, RL>;
    load_row8<DK, C, RL>(rec, 0, L, k2);
#pragma unroll
    for (int r = 0; r < RL; ++r)
        vr[r] = Widen<RT>::lds1(rec + 2 * DK + L.row + r * LM::RG);
}


// ---------------------------------------------------------------------------
// Tree walks
// ---------------------------------------------------------------------------

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
// stack slots.
static __device__ bool build_walk(const int32_t* prow, int N, int K, const TreeView& T)
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
        if (T.nch[n] >= 2 && T.lt[n] < K)
            save = T.lt[n] + 1;
        T.meta[pos] = n | (src << 16) | (save << 19) | (ld << 24);
        T.rstart[pos] = start;
    }
    __syncthreads();
    return true;
}

// Trees of up to kMaskNodes nodes: the same walk as build_walk, built from
// per-node bit masks in O(log depth) barrier rounds instead of O(depth)
// serial chains.  Needs one thread per node and kMaskScratch ints per node
// of scratch (T.path, which the walk only uses afterwards).
constexpr int kMaskNodes = 128;
constexpr int kMaskWords = kMaskNodes / 32;
constexpr int kMaskScratch = 2 * kMaskWords;
static __device__ bool build_walk_masked(const int32_t* prow, int N, int K, const TreeView& T)
{
    const int tid = threadIdx.x;
    const bool own = tid < N;
    unsigned* const anc = reinterpret_cast<unsigned*>(T.path);  // [N][4] ancestor-or-self masks
    unsigned* const kids = anc + kMaskWords * N;                // [N][4] child masks
    int pn = -1;
    bool bad = false;
    if (own) {
        pn = __ldg(prow + tid);
        T.par[tid] = pn;
        bad = (tid == 0) ? (pn != -1) : (pn < 0 || pn >= tid);
#pragma unroll
        for (int w = 0; w < kMaskWords; ++w) {
            kids[kMaskWords * tid + w] = 0u;
            anc[kMaskWords * tid + w] = (w == (tid >> 5)) ? (1u << (tid & 31)) : 0u;
        }
        T.ord[tid] = pn;  // pointer-jumping target, until ord is written
    }
    if (__syncthreads_or(bad))
        return false;
    if (own && tid > 0)
        atomicOr(&kids[kMaskWords * pn + (tid >> 5)], 1u << (tid & 31));
    // ancestor masks: after round r, anc covers the 2^r nearest ancestors
    unsigned m[kMaskWords];
#pragma unroll
    for (int w = 0; w < kMaskWords; ++w)
        m[w] = own ? anc[kMaskWords * tid + w] : 0u;
    int jump = pn;
    while (__syncthreads_or(jump >= 0)) {
        int nj = -1;
        if (jump >= 0) {
#pragma unroll
            for (int w = 0; w < kMaskWords; ++w)
                m[w] |= anc[kMaskWords * jump + w];
            nj = T.ord[jump];
        }
        __syncthreads();
        if (own) {
#pragma unroll
            for (int w = 0; w < kMaskWords; ++w)
                anc[kMaskWords * tid + w] = m[w];
            T.ord[tid] = nj;
        }
        jump = nj;
    }
    // subtree sizes (nodes whose masks hold this one) and child counts
    int sz = 0;
    if (own) {
        const int w = tid >> 5;
        const unsigned bit = 1u << (tid & 31);
        for (int x = 0; x < N; ++x)
            sz += (anc[kMaskWords * x + w] & bit) ? 1 : 0;
        T.sz[tid] = sz;
        int nch = 0;
#pragma unroll
        for (int w2 = 0; w2 < kMaskWords; ++w2)
            nch += __popc(kids[kMaskWords * tid + w2]);
        T.nch[tid] = nch;
    }
    __syncthreads();
    // offset among the siblings (visited by increasing (subtree size,
    // index)) and whether the node is its parent's last-visited child
    if (own) {
        int o = 0, is_last = 1;
        if (tid > 0) {
            o = 1;
#pragma unroll
            for (int w = 0; w < kMaskWords; ++w) {
                unsigned bits = kids[kMaskWords * pn + w];
                if (w == (tid >> 5))
                    bits &= ~(1u << (tid & 31));
                while (bits) {
                    const int t = 32 * w + __ffs(bits) - 1;
                    bits &= bits - 1;
                    const int zt = T.sz[t];
                    if (zt < sz || (zt == sz && t < tid))
                        o += zt;
                    else
                        is_last = 0;
                }
            }
        }
        T.off[tid] = o;
        T.last[tid] = is_last;
    }
    __syncthreads();
    // preorder position and stack slot: sums of off and not-last over the
    // root path
    if (own) {
        int pos = 0, l = 0;
#pragma unroll
        for (int w = 0; w < kMaskWords; ++w) {
            unsigned bits = m[w];
            while (bits) {
                const int x = 32 * w + __ffs(bits) - 1;
                bits &= bits - 1;
                pos += T.off[x];
                l += T.last[x] ? 0 : 1;
            }
        }
        T.ord[pos] = tid;
        T.lt[tid] = l;
    }
    __syncthreads();
    if (own) {
        const int pos = tid;
        const int n = T.ord[pos];
        const int pp = T.par[n];
        int src, ld = 0, start = -1, save = 0;
        if (pos == 0) {
            src = kSrcRoot;
        } else if (pp == T.ord[pos - 1]) {
            src = kSrcCont;
        } else if (T.lt[pp] < K) {
            src = kSrcSlot;
            ld = T.lt[pp];
        } else {
            src = kSrcRecompute;
            // deepest saved ancestor of pp (strictly above it): the highest
            // index among pp's ancestors that branches and sits in slot K - 1
            for (int w = kMaskWords - 1; w >= 0 && start < 0; --w) {
                unsigned bits = anc[kMaskWords * pp + w];
                if (w == (pp >> 5))
                    bits &= ~(1u << (pp & 31));
                while (bits) {
                    const int x = 32 * w + 31 - __clz(bits);
                    bits &= ~(1u << (x & 31));
                    if (T.nch[x] >= 2 && T.lt[x] == K - 1) {
                        start = x;
                        break;
                    }
                }
            }
        }
        if (T.nch[n] >= 2 && T.lt[n] < K)
            save = T.lt[n] + 1;
        T.meta[pos] = n | (src << 16) | (save << 19) | (ld << 24);
        T.rstart[pos] = start;
    }
    __syncthreads();
    return true;
}

// Tree metadata held in shared memory (any N).
struct SmemTree {
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

// Walk of a tree of N <= 32 nodes as built by one warp (build_warp_walk) in
// shared memory: [meta | rstart | par | mask] x 32, followed by the
// builder's scratch.
constexpr int kWarpTreeInts = 10 * 32;
struct MaskTree {
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

// Builds the walk of a tree of N <= 32 nodes with the calling warp, lane j
// standing for node j, into ws[kWarpTreeInts] (same order and metadata as
// build_walk).  Ancestor masks and path sums use pointer jumping (5 rounds
// cover depth < 32), descendant masks a transpose of the 32 x 32 bit matrix
// of ancestor masks, siblings __match_any_sync; per-node values are exchanged
// through ws.  Returns false if the tree is malformed (the same on every
// lane).
static __device__ bool build_warp_walk(const int32_t* prow, int N, int K, int* ws)
{
    const unsigned full = 0xffffffffu;
    const int lane = threadIdx.x & 31;
    int* const w_meta = ws;
    int* const w_rstart = ws + 32;
    int* const w_par = ws + 64;
    int* const w_mask = ws + 96;
    int* const w_sz = ws + 128;
    int* const w_ord = ws + 160;
    int* const w_lt = ws + 192;
    int* const w_nch = ws + 224;
    int* const w_kids = ws + 256;
    const bool valid = lane < N;
    const int par = valid ? __ldg(prow + lane) : -1;
    const bool bad = valid && ((lane == 0) ? par != -1 : (par < 0 || par >= lane));
    if (__any_sync(full, bad))
        return false;
    w_par[lane] = par;
    w_kids[lane] = 0;
    w_ord[lane] = 0;
    // ancestor-or-self mask
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
    // descendant-or-self mask (column `lane` of the mask matrix) and subtree
    // size: swap the off-diagonal blocks at widths 16, 8, 4, 2, 1
    unsigned desc = mask;
#pragma unroll
    for (int sh = 16, k = 0; sh >= 1; sh >>= 1, ++k) {
        const unsigned lo = k == 0 ? 0x0000ffffu
                          : k == 1 ? 0x00ff00ffu
                          : k == 2 ? 0x0f0f0f0fu
                          : k == 3 ? 0x33333333u
                                   : 0x55555555u;
        const unsigned y = __shfl_xor_sync(full, desc, sh);
        desc = (lane & sh) ? ((desc & ~lo) | ((y & ~lo) >> sh)) : ((desc & lo) | ((y & lo) << sh));
    }
    const int sz = __popc(desc);
    w_mask[lane] = static_cast<int>(mask);
    w_sz[lane] = sz;
    // siblings (lanes with the same parent) and child sets
    const unsigned sib = __match_any_sync(full, valid ? par : 64 + lane);
    __syncwarp();
    if (valid && lane > 0)
        w_kids[par] = static_cast<int>(sib);  // every child writes the same set
    // offset among the siblings visited by increasing (subtree size, index),
    // and whether the node is its parent's last-visited child
    int off = 0, last = 1;
    if (valid && lane > 0) {
        off = 1;
        unsigned bits = sib & ~(1u << lane);
        while (bits) {
            const int t = __ffs(bits) - 1;
            bits &= bits - 1;
            const int zt = w_sz[t];
            if (zt < sz || (zt == sz && t < lane))
                off += zt;
            else
                last = 0;
        }
    }
    __syncwarp();
    const int nch = __popc(static_cast<unsigned>(w_kids[lane]));
    // preorder position and stack slot: sums of (off, not-last) along the
    // root path, packed in one int
    int acc = (valid && lane > 0) ? (off | ((last ? 0 : 1) << 16)) : 0;
    jump = valid ? par : -1;
#pragma unroll
    for (int it = 0; it < 5; ++it) {
        const int pa = __shfl_sync(full, acc, jump & 31);
        const int pj = __shfl_sync(full, jump, jump & 31);
        if (jump >= 0) {
            acc += pa;
            jump = pj;
        }
    }
    const int pos = acc & 0xffff, lt = acc >> 16;
    __syncwarp();
    if (valid)
        w_ord[pos] = lane;  // a permutation of [0, N) for a valid tree
    w_lt[lane] = lt;
    w_nch[lane] = nch;
    const unsigned cand_all = __ballot_sync(full, valid && nch >= 2 && lt == K - 1);
    __syncwarp();
    // lane p: the metadata of walk position p
    const int ord = w_ord[lane];
    const int pp = w_par[ord];
    const int prev = lane > 0 ? w_ord[lane - 1] : -1;
    const int lt_pp = pp >= 0 ? w_lt[pp] : 0;
    const int lt_n = w_lt[ord];
    const int nch_n = w_nch[ord];
    const unsigned mask_pp = pp >= 0 ? static_cast<unsigned>(w_mask[pp]) : 0u;
    int src, ld = 0, start = -1, save = 0;
    if (lane == 0) {
        src = kSrcRoot;
    } else if (pp == prev) {
        src = kSrcCont;
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
    if (nch_n >= 2 && lt_n < K)
        save = lt_n + 1;
    w_meta[lane] = ord | (src << 16) | (save << 19) | (ld << 24);
    w_rstart[lane] = start;
    return true;
}

// Makes S the exact f32 state of node pp, the parent of the node at a walk
// position whose metadata says the state is not already in registers: a
// stack slot, or recomputation from the deepest saved ancestor (start; -1:
// from state_in).  fetch(y, k2, vr, a, beta) supplies node y's inputs.
template <int DK, int C, int RL, class Tree, class SlotLoad, class Fetch>
__device__ __forceinline__ void source_parent(StateT<C, RL>& S, int m, int pp, int start, const KParams& p,
                                              const Tree& tree, SlotLoad slot_load, const float* sin_lane,
                                              Fetch fetch)
{
    constexpr int LR = LaneMap<DK, C, RL>::LR;
    const int src = meta_src(m);
    if (src == kSrcSlot) {
        slot_load(S, meta_load(m));
    } else if (src == kSrcRecompute) {
        if (start >= 0)
            slot_load(S, p.slots - 1);
        else
            load_rows<DK, C, RL>(S, sin_lane);
        tree.for_path(pp, start, [&](int y) {
            float2 k2[4 * C];
            float vr[RL];
            float a, ar, be;
            fetch(y, k2, vr, a, ar, be);
            gdn_update<LR, C, RL>(S, k2, vr, a, ar, be);
        });
    }
}

// Walk kinds (bits 0-1) and where a walk's stack slots live (bits 2-3).
// kTreeGlobal added to kTreeWarp or kTreeSmem: the stack slots live in a
// caller workspace in global memory (L2) instead of shared memory, and a
// slot the next position needs is loaded one node ahead.  kTreeTmem added to
// kTreeSmem: they live in the CTA's tensor memory (the wide kernel only).
enum : int { kTreeChain = 0, kTreeWarp = 1, kTreeSmem = 2, kTreeIndex = 3, kTreeGlobal = 4, kTreeTmem = 8 };

// The walk over positions [0, N): per position, find the parent state,
// update, write the output and persist.  The context supplies each
// position's descriptor and record (ctx.desc, ctx.rec), the input fetcher
// for recomputation, and the ring handshakes (ctx.begin / ctx.end; trivial
// when everything is staged).
template <int DK, int C, int RL, typename RT, typename ST, int TREE, class Tree, class Ctx>
__device__ __forceinline__ void walk(StateT<C, RL>& S, const KParams& p, const Seq& sq, const Tree& tree,
                                     float* lane_slot, uint32_t tslot, const float* sin_lane, int b, int h,
                                     int row0, const LaneMap<DK, C, RL>& L, Ctx& ctx)
{
    using LM = LaneMap<DK, C, RL>;
    constexpr bool CHAIN = TREE == kTreeChain;
    constexpr bool INDEX = TREE == kTreeIndex;
    constexpr bool GSLOT = (TREE & kTreeGlobal) != 0;
    constexpr bool TSLOT = (TREE & kTreeTmem) != 0;
    // tensor-memory walks are never launched with last-only persistence or
    // in-kernel q/k normalisation (the host geometry), so for them both are
    // compile-time off and the node loop carries neither test
    const bool persist_last = !TSLOT && p.persist_last;
    const bool qk_norm = !TSLOT && p.qk_norm;
    const int N = sq.N;
    const size_t ns_stride = (size_t)p.Hv * p.dv * DK;  // elements between nodes' states
    ST* const ns_lane = static_cast<ST*>(p.node_states) + (size_t)(persist_last ? b : sq.n0) * ns_stride +
                        (size_t)h * p.dv * DK + (size_t)row0 * DK + L.tile_offset();
    const size_t out_stride = (size_t)p.Hv * p.dv;
    float* const out_lane = p.out + (size_t)sq.n0 * out_stride + (size_t)h * p.dv + row0 + L.row;
    const int slot_floats = p.rows * DK;
    const int stride = p.warps * 32 * 4;
    auto slot_load = [&](StateT<C, RL>& X, int s) {
        if constexpr (TSLOT)
            tmem_load_slot<C, RL>(X, tslot + (uint32_t)(s * p.tmem_slot_cols));
        else
            load_slot<C, RL>(X, lane_slot + (size_t)s * slot_floats, stride);
    };
    // Index order and workspace slots: the next position's parent state,
    // loaded one node ahead.  (Asking for it in L1 instead, with prefetch
    // hints and a load where it is needed, saves ~40 registers but was
    // measured slower.)
    StateT<C, RL> Sn;
    bool have_next = false;
    // (Loading the next position's record a node ahead as well costs ~30
    // registers per thread; on small grids that keeps the next layer's CTAs
    // from becoming resident early, which costs more than it saves.)
    for (int pos = 0; pos < N; ++pos) {
        if (!ctx.begin(pos))
            return;
        const PosDesc d = ctx.desc(pos);
        const int n = CHAIN ? pos : d.i.x;
        RawRec<RT, C, RL> R;
        fetch_raw<DK, C, RL>(ctx.rec(pos, n), L, R);
        if constexpr (INDEX) {
            // the next position's parent state, persisted by this thread at
            // an earlier position, unless it is this position's
            have_next = false;
            if (pos + 1 < N) {
                const int pn = tree.parent(pos + 1);
                if (pn != pos) {
                    load_rows<DK, C, RL>(Sn, reinterpret_cast<const float*>(ns_lane) + (size_t)pn * ns_stride);
                    have_next = true;
                }
            }
        } else if constexpr (!CHAIN) {
            const int src = meta_src(d.i.y);
            if (GSLOT && have_next)
                S = Sn;  // this position's slot, loaded at the previous one
            else if (src != kSrcCont && src != kSrcRoot)
                source_parent<DK, C, RL>(S, d.i.y, d.i.w, d.i.z, p, tree, slot_load, sin_lane, ctx.fetcher());
            if constexpr (GSLOT) {
                // the next position's slot.  A node whose successor in the
                // walk reloads a slot is a leaf, so this position saves
                // nothing into it.
                have_next = false;
                if (pos + 1 < N && ctx.ahead(pos + 1)) {
                    const int mn = ctx.desc(pos + 1).i.y;
                    if (meta_src(mn) == kSrcSlot) {
                        load_slot<C, RL>(Sn, lane_slot + (size_t)meta_load(mn) * slot_floats, stride);
                        have_next = true;
                    }
                }
            }
        }
        float2 k2[4 * C], q2[4 * C];
        float vr[RL];
        widen_raw<C, RL>(R, k2, q2, vr);
        const float a = d.f.x;
        float pq[RL], u[RL];
        gdn_step<LM::LR, C, RL, true>(S, k2, q2, vr, a, d.f.w, d.f.y, pq, u);
        if (L.cl == 0) {
            const float oc = qk_norm ? ctx.out_coef(pos, n) : p.scale;
            float* o = out_lane + (size_t)n * out_stride;
#pragma unroll
            for (int r = 0; r < RL; ++r)
                o[r * LM::RG] = __fmul_rn(oc, __fmaf_rn(u[r], d.f.z, __fmul_rn(a, pq[r])));
        }
        if (!persist_last || pos == N - 1)
            persist<DK, C, RL, ST>(S, ns_lane + (size_t)(persist_last ? 0 : n) * ns_stride);
        if constexpr (!CHAIN && !INDEX) {
            const int save = meta_save(d.i.y);
            if (save >= 0) {
                if constexpr (TSLOT)
                    tmem_save_slot<C, RL>(S, tslot + (uint32_t)(save * p.tmem_slot_cols));
                else
                    save_slot<C, RL>(S, lane_slot + (size_t)save * slot_floats, stride);
            }
        }
        if constexpr (INDEX) {
            if (have_next)
                S = Sn;
        }
        ctx.end(pos);
    }
}

// Chain mode: position p is node p.
struct NoTree {
    __device__ __forceinline__ int meta(int pos) const { return pos | ((pos == 0 ? kSrcRoot : kSrcCont) << 16); }
    __device__ __forceinline__ int rstart(int) const { return -1; }
    __device__ __forceinline__ int parent(int n) const { return n - 1; }
    template <class F>
    __device__ __forceinline__ void for_path(int, int, F&&) const
    {
    }
};

// ---------------------------------------------------------------------------
// Staged kernel: every node's record copied into shared memory at start
// ---------------------------------------------------------------------------

template <int DK, int C, int RL, typename RT>
struct StagedFetch {
    const RT* recs;
    const float* ab;  // a | beta' (| a' | output coefficient with qk_norm), by node
    uint32_t rec_elems;
    int N;
    int qk_norm;
    LaneMap<DK, C, RL> L;
    __device__ __forceinline__ void operator()(int y, float2 (&k2)[4 * C], float (&vr)[RL], float& a,
                                               float& ar, float& be) const
    {
        load_k<DK, C, RL, RT>(recs + (size_t)y * rec_elems, L, k2, vr);
        a = ab[y];
        be = ab[N + y];
        ar = qk_norm ? ab[2 * N + y] : a;
    }
};

template <int DK, int C, int RL, typename RT>
struct StagedCtx {
    const RT* recs;
    const PosDesc* desc_;
    const float* ab;
    uint32_t rec_elems;
    int N;
    int qk_norm;
    LaneMap<DK, C, RL> L;
    __device__ __forceinline__ bool begin(int) { return true; }
    __device__ __forceinline__ void end(int) {}
    // whether position pos's descriptor may be read before begin(pos)
    __device__ __forceinline__ bool ahead(int) const { return true; }
    __device__ __forceinline__ PosDesc desc(int pos) const { return desc_[pos]; }
    __device__ __forceinline__ float out_coef(int, int n) const { return ab[3 * N + n]; }
    __device__ __forceinline__ const RT* rec(int, int n) const { return recs + (size_t)n * rec_elems; }
    __device__ __forceinline__ StagedFetch<DK, C, RL, RT> fetcher() const
    {
        return StagedFetch<DK, C, RL, RT>{recs, ab, rec_elems, N, qk_norm, L};
    }
};

__device__ __forceinline__ void cp_async16(void* dst_smem, const void* src_gmem)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst_smem)), "l"(src_gmem)
                 : "memory");
}

__device__ __forceinline__ void cp_async4(void* dst_smem, const void* src_gmem)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst_smem)), "l"(src_gmem)
                 : "memory");
}

// This CTA's stack slots: shared memory, or its region of the workspace.
template <int DK, int TREE>
__device__ __forceinline__ float* cta_slots(const KParams& p, float* slotbuf)
{
    if constexpr ((TREE & kTreeGlobal) != 0) {
        const size_t cta = ((size_t)blockIdx.z * p.Hv + blockIdx.y) * gridDim.x + blockIdx.x;
        return p.ws + cta * (size_t)p.slots * p.rows * DK;
    } else {
        return slotbuf;
    }
}

// Prologue pass of the staged kernel over walk positions, four per warp and
// pass (8 lanes each): turns ab (g | beta, by node) into a | beta'
// (node_scalars; with qk_norm also a' and the output coefficient, by node)
// and writes each position's descriptor with k . q of its node.
template <int DK, int LR, typename QT, class Tree>
__device__ __forceinline__ void write_descs(const Tree& tree, const unsigned char* raw, uint32_t raw_bytes,
                                            float* ab, PosDesc* desc, int N, int qk_norm, int gates,
                                            float scale)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const int sub = lane & 7;
    for (int p0 = 4 * warp; p0 < N; p0 += 4 * nwarps) {
        const int pos = min(p0 + (lane >> 3), N - 1);
        const int m = tree.meta(pos);
        const int n = meta_node(m);
        const QT* rrec = reinterpret_cast<const QT*>(raw + (size_t)n * raw_bytes);
        const bool valid = p0 + (lane >> 3) < N;
        const float kq = node_kq8<DK, LR>(rrec, sub);
        float rk = 1.f, rq = 1.f;
        if (qk_norm) {
            rk = inv_norm(node_dot8<DK, LR>(rrec, sub, 0, 0));
            rq = inv_norm(node_dot8<DK, LR>(rrec, sub, DK, DK));
        }
        if (sub == 0 && valid) {
            float a, be, bp, ap;
            gate_scalars(ab[n], ab[N + n], gates, a, be);
            node_scalars(a, be, rk, bp, ap);
            ab[n] = a;
            ab[N + n] = bp;
            if (qk_norm) {
                ab[2 * N + n] = ap;
                ab[3 * N + n] = __fmul_rn(scale, rq);
            }
            PosDesc d;
            d.i = make_int4(n, m, tree.rstart(pos), tree.parent(n));
            d.f = make_float4(a, bp, kq, ap);
            desc[pos] = d;
        }
    }
}

template <int DK, int C, int RL, typename QT, typename ST, int TREE, class Tree>
__device__ __forceinline__ void staged_finish(StateT<C, RL>& S, const KParams& p, const Seq& sq, const Tree& tree,
                                              const unsigned char* raw, float* ab, PosDesc* desc, float* slotbuf,
                                              uint32_t tbase, const float* sin_lane, int b, int h, int row0,
                                              const LaneMap<DK, C, RL>& L)
{
    constexpr int LR = LaneMap<DK, C, RL>::LR;
    write_descs<DK, LR, QT>(tree, raw, p.raw_bytes, ab, desc, sq.N, p.qk_norm, p.gates, p.scale);
    __syncthreads();
    const uint32_t rec_elems = p.raw_bytes / (uint32_t)sizeof(QT);
    StagedCtx<DK, C, RL, QT> ctx{reinterpret_cast<const QT*>(raw), desc, ab, rec_elems, sq.N, p.qk_norm, L};
    float* lane_slot = cta_slots<DK, TREE>(p, slotbuf) + 4 * threadIdx.x;
    // tensor-memory slots: warp w's lanes are TMEM lanes 32 (w mod 4) ..; the
    // warps that share a lane quarter use columns 32 apart
    const int warp = threadIdx.x >> 5;
    const uint32_t tslot = tbase + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(32 * (warp >> 2));
    walk<DK, C, RL, QT, ST, TREE>(S, p, sq, tree, lane_slot, tslot, sin_lane, b, h, row0, L, ctx);
}

template <int DK, int C, int RL, typename QT, typename ST, int TREE>
__device__ __forceinline__ void staged_body(const KParams& p, uint32_t tbase)
{
    constexpr int EPC = 16 / sizeof(QT);  // elements per 16-byte chunk
    constexpr int QKCH = DK / EPC;        // chunks per k (or q) row
    extern __shared__ __align__(16) unsigned char smem[];
    unsigned char* raw = smem + p.off_raw;
    PosDesc* desc = reinterpret_cast<PosDesc*>(smem + p.off_desc);
    float* ab = reinterpret_cast<float*>(smem + p.off_ab);
    float* slotbuf = reinterpret_cast<float*>(smem + p.off_slots);
    int* tsm = reinterpret_cast<int*>(smem + p.off_tree);

    constexpr int TK = TREE & 3;  // walk kind without the slot placement
    const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int hk = h / p.G;
    const int row0 = tile * p.rows;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int nwarps = blockDim.x >> 5;
    // Everything that reads q, k, v, g, beta waits for the preceding kernel;
    // with GDN_FLAG_EARLY_TREE the tree (varlen offsets included) and the
    // root's parent state are read before that (they were written before the
    // preceding kernel started).  Every node's raw k row, q row and v slice,
    // and its g and beta, are copied to shared memory asynchronously (warp w
    // copies nodes w, w + warps, ...); the tree work overlaps the copies
    // unless it already ran before the wait.
    if (!p.early_tree)
        pdl_wait_then_release();
    Seq sq;
    if (!seq_of(p, b, sq)) {
        if (tid == 0)
            report_status(p.status, GDN_ERR_BAD_TREE);
        return;
    }
    const int N = sq.N;
    const int32_t* prow = p.parent + sq.n0;
    const int per_node = p.raw_bytes / 16;  // 16-byte chunks per node
    constexpr int LR = LaneMap<DK, C, RL>::LR;
    if (p.prefetch) {
        // Ahead of the wait, bring this CTA's records into L2 so that the
        // copies after it start from there (small layers, where the first
        // records' latency is exposed; on large ones the prefetched lines
        // would compete for L2 with the running layer's states).  Only a
        // hint: global writes land in L2, so a line the preceding kernel
        // rewrites is read new after the wait.
        const char* kg = static_cast<const char*>(p.k);
        const char* qg = static_cast<const char*>(p.q);
        const char* vg = static_cast<const char*>(p.v);
        constexpr int kRowBytes = DK * (int)sizeof(QT);
        for (int n = tid; n < N; n += blockDim.x) {
            const size_t node = (size_t)sq.n0 + n;
            const size_t kq = (node * p.Hk + hk) * kRowBytes;
#pragma unroll
            for (int off = 0; off < kRowBytes; off += 128) {
                prefetch_l2(kg + kq + off);
                prefetch_l2(qg + kq + off);
            }
            prefetch_l2(vg + ((node * p.Hv + h) * p.dv + row0) * sizeof(QT));
            prefetch_l2(p.g + node * p.Hv + h);
            prefetch_l2(p.beta + node * p.Hv + h);
        }
    }
    auto stage = [&]() {
        const QT* kg = static_cast<const QT*>(p.k);
        const QT* qg = static_cast<const QT*>(p.q);
        const QT* vg = static_cast<const QT*>(p.v);
        if constexpr (sizeof(QT) == 2) {
            // k and q rows: 2 QKCH chunks per node over all threads (a warp
            // per node at d_k = 128), then the v slices
            constexpr int KQ = 2 * QKCH;
            for (int idx = tid; idx < N * KQ; idx += blockDim.x) {
                const int n = idx / KQ, c = idx % KQ;
                const size_t node = (size_t)sq.n0 + n;
                const QT* src = (c < QKCH ? kg : qg) + (node * p.Hk + hk) * DK + (c % QKCH) * EPC;
                cp_async16(raw + (size_t)n * p.raw_bytes + 16 * c, src);
            }
            const int vch = per_node - KQ;  // rows / 8
            for (int idx = tid; idx < N * vch; idx += blockDim.x) {
                const int n = idx / vch, c = idx - n * vch;
                const size_t node = (size_t)sq.n0 + n;
                cp_async16(raw + (size_t)n * p.raw_bytes + 16 * (KQ + c),
                           vg + (node * p.Hv + h) * p.dv + row0 + c * EPC);
            }
        }
        for (int n = warp; n < N && sizeof(QT) == 4; n += nwarps) {
            const size_t node = (size_t)sq.n0 + n;
            const QT* krow = kg + (node * p.Hk + hk) * DK;
            const QT* qrow = qg + (node * p.Hk + hk) * DK;
            const QT* vrow = vg + (node * p.Hv + h) * p.dv + row0;
            unsigned char* dst = raw + (size_t)n * p.raw_bytes;
            for (int c = lane; c < per_node; c += 32) {
                const QT* src = c < QKCH ? krow + c * EPC
                                         : (c < 2 * QKCH ? qrow + (c - QKCH) * EPC
                                                         : vrow + (c - 2 * QKCH) * EPC);
                int off = 16 * c;
                if constexpr (sizeof(QT) == 4) {
                    // f32 k and q rows land swizzled (swz_pos): 16-byte half
                    // h of 8-column chunk j
                    if (c < 2 * QKCH) {
                        const int part = c < QKCH ? 0 : QKCH;
                        const int j = (c - part) >> 1, hh = (c - part) & 1;
                        off = 16 * part + 32 * j + 16 * (hh ^ (((j % LR) >> 2) & 1));
                    }
                }
                cp_async16(dst + off, src);
            }
        }
        for (int n = tid; n < N; n += blockDim.x) {
            const size_t gi = ((size_t)sq.n0 + n) * p.Hv + h;
            cp_async4(ab + n, p.g + gi);
            cp_async4(ab + N + n, p.beta + gi);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    if (!p.early_tree)
        stage();

    // 1. the parent array (index order keeps it in shared memory; chain
    //    validation only checks it)
    bool bad = false;
    if constexpr (TK == kTreeIndex) {
        for (int n = tid; n < N; n += blockDim.x) {
            const int pn = __ldg(prow + n);
            tsm[n] = pn;
            bad |= (n == 0) ? (pn != -1) : (pn < 0 || pn >= n);
        }
    } else if constexpr (TK == kTreeChain) {
        if (p.validate) {
            for (int n = tid; n < N; n += blockDim.x)
                bad |= __ldg(prow + n) != n - 1;
        }
    }
    // 2. the root's parent state
    const LaneMap<DK, C, RL> L(warp, lane);
    const float* sin_lane =
        p.state_in + ((size_t)b * p.Hv + h) * p.dv * DK + (size_t)row0 * DK + L.tile_offset();
    StateT<C, RL> S;
    load_rows<DK, C, RL>(S, sin_lane);
    // 3. the walk: warp 0 builds it for trees of <= 32 nodes; all threads for
    //    larger trees
    const TreeView tv(tsm, N);
    if ((TK == kTreeWarp || TK == kTreeSmem) && p.plan != nullptr) {
        // the walk was built once for all layers: copy it (written before
        // the preceding kernel started when the tree is read early)
        const int32_t* pl = p.plan + (size_t)b * p.plan_stride;
        const int cnt = TK == kTreeWarp ? 128 : 4 * N;
        for (int i = 4 * tid; i < cnt; i += 4 * blockDim.x)
            cp_async16(tsm + i, pl + kPlanHeader + i);
        asm volatile("cp.async.commit_group;" ::: "memory");
        const int sig = __ldg(pl), ok = __ldg(pl + 1), pn = __ldg(pl + 2);
        if (sig != p.plan_sig || pn != N) {
            bad = true;
            if (tid == 0)
                report_status(p.status, GDN_ERR_BAD_INPUT);
        } else if (ok != 1) {
            bad = true;
        }
    } else if constexpr (TK == kTreeWarp) {
        if (warp == 0 && !build_warp_walk(prow, N, p.slots, tsm))
            bad = true;
    } else if constexpr (TK == kTreeSmem) {
        bad = (N <= kMaskNodes && N <= (int)blockDim.x) ? !build_walk_masked(prow, N, p.slots, tv)
                                                        : !build_walk(prow, N, p.slots, tv);
    }
    if (p.early_tree) {
        pdl_wait_then_release();
        stage();
    }
    // 4. the copies target this CTA's shared memory: wait for them even when
    //    the tree is rejected
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (__syncthreads_or(bad)) {
        if (tid == 0)
            report_status(p.status, GDN_ERR_BAD_TREE);
        return;
    }
    // 5. descriptors, then the walk
    if constexpr (TK == kTreeChain)
        staged_finish<DK, C, RL, QT, ST, TREE>(S, p, sq, NoTree{}, raw, ab, desc, slotbuf, tbase, sin_lane, b, h,
                                               row0, L);
    else if constexpr (TK == kTreeIndex)
        staged_finish<DK, C, RL, QT, ST, TREE>(S, p, sq, IndexTree{tsm}, raw, ab, desc, slotbuf, tbase, sin_lane, b,
                                               h, row0, L);
    else if constexpr (TK == kTreeWarp)
        staged_finish<DK, C, RL, QT, ST, TREE>(S, p, sq, MaskTree{tsm}, raw, ab, desc, slotbuf, tbase, sin_lane, b,
                                               h, row0, L);
    else
        staged_finish<DK, C, RL, QT, ST, TREE>(S, p, sq, SmemTree{tv, N, warp}, raw, ab, desc, slotbuf, tbase,
                                               sin_lane, b, h, row0, L);
}

template <int DK, int C, int RL, typename QT, typename ST, int TREE>
__global__ void __launch_bounds__(kSmallWarps * 32) gdn_verify_staged(const KParams p)
{
    staged_body<DK, C, RL, QT, ST, TREE>(p, 0u);
}

// Trees of more than 32 nodes with shared-memory slots on large grids:
// kMaxWarps warps share one copy of the node records.
// With kTreeTmem the stack slots live in tensor memory: warp 0 allocates
// p.tmem_cols columns before anything else and frees them after every path
// through the body (its early exits are CTA-wide, so all threads get back
// here).
template <int DK, int C, int RL, typename QT, typename ST, int TREE>
__global__ void __launch_bounds__(kMaxWarps * 32) gdn_verify_staged_wide(const KParams p)
{
    if constexpr ((TREE & kTreeTmem) != 0) {
        __shared__ uint32_t tbase;
        if (threadIdx.x < 32)
            tmem_alloc(&tbase, (uint32_t)p.tmem_cols);
        tmem_fence_before_sync();
        __syncthreads();
        tmem_fence_after_sync();
        staged_body<DK, C, RL, QT, ST, TREE>(p, tbase);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");  // this thread's slot stores are done
        tmem_fence_before_sync();
        __syncthreads();
        if (threadIdx.x < 32) {
            tmem_fence_after_sync();
            tmem_free(tbase, (uint32_t)p.tmem_cols);
        }
    } else {
        staged_body<DK, C, RL, QT, ST, TREE>(p, 0u);
    }
}

// Small trees walked from warp registers with one row per lane (small
// grids), bf16 inputs: at most 80 registers, so that six CTAs fit on an SM
// and the next layer's CTAs become resident while this layer's still run.
template <int DK, int C, int RL, typename QT, typename ST, int TREE>
__global__ void __launch_bounds__(kSmallWarps * 32, 6) gdn_verify_staged_dense(const KParams p)
{
    staged_body<DK, C, RL, QT, ST, TREE>(p, 0u);
}

// ---------------------------------------------------------------------------
// Ring kernel: a producer warp streams chunks of walk positions
// ---------------------------------------------------------------------------

template <int DK, int C, int RL, typename QT>
struct GlobalFetch {
    const QT* kg;
    const QT* vg;
    const float* g;
    const float* beta;
    size_t bN;         // the sequence's first node
    const float* rkn;  // qk_norm: 1 / |k| per node (written by the producer), else NULL
    int Hk, Hv, dv, hk, h, row0;
    LaneMap<DK, C, RL> L;
    int gates;
    __device__ __forceinline__ void operator()(int y, float2 (&k2)[4 * C], float (&vr)[RL], float& a,
                                               float& ar, float& be) const
    {
        using LM = LaneMap<DK, C, RL>;
        const size_t node = bN + y;
#pragma unroll
        for (int c = 0; c < C; ++c) {
            float2 x[4];
            Widen<QT>::ldg8(kg + (node * Hk + hk) * DK + L.col(c), x);
#pragma unroll
            for (int t = 0; t < 4; ++t)
                k2[4 * c + t] = x[t];
        }
#pragma unroll
        for (int r = 0; r < RL; ++r)
            vr[r] = Widen<QT>::load1(vg + (node * Hv + h) * dv + row0 + L.row + r * LM::RG);
        const size_t gi = node * Hv + h;
        float bt;
        gate_scalars(__ldg(g + gi), __ldg(beta + gi), gates, a, bt);
        node_scalars(a, bt, rkn != nullptr ? rkn[y] : 1.f, be, ar);
    }
};

// A ring slot: kChunk records (raw_bytes each) then kChunk descriptors.
template <int DK, int C, int RL, typename QT>
struct RingCtx {
    uint64_t* full;
    uint64_t* empty;
    const unsigned char* ring;
    uint32_t raw_bytes;
    uint32_t slot_bytes;
    uint32_t desc_off;  // offset of the descriptors inside a slot
    int32_t* status;
    int lane;
    GlobalFetch<DK, C, RL, QT> gf;
    const unsigned char* cur = nullptr;  // the slot of the current chunk
    __device__ __forceinline__ const unsigned char* slot(int) const { return cur; }
    __device__ __forceinline__ bool begin(int pos)
    {
        if (pos % kChunk == 0) {
            const int c = pos / kChunk;
            if (!mbar_wait(&full[c % kRing], (c / kRing) & 1)) {
                report_status(status, kStatusTimeout);
                return false;
            }
            cur = ring + (size_t)(c % kRing) * slot_bytes;
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
    __device__ __forceinline__ PosDesc desc(int pos) const
    {
        return reinterpret_cast<const PosDesc*>(slot(pos) + desc_off)[pos % kChunk];
    }
    // only within the chunk already waited for
    __device__ __forceinline__ bool ahead(int pos) const { return pos % kChunk != 0; }
    __device__ __forceinline__ float out_coef(int pos, int) const
    {
        return reinterpret_cast<const float*>(slot(pos) + desc_off + kChunk * sizeof(PosDesc))[pos % kChunk];
    }
    __device__ __forceinline__ const QT* rec(int pos, int) const
    {
        return reinterpret_cast<const QT*>(slot(pos) + (size_t)(pos % kChunk) * raw_bytes);
    }
    __device__ __forceinline__ GlobalFetch<DK, C, RL, QT> fetcher() const { return gf; }
};

template <int DK, int C, int RL, typename QT, typename ST, int TREE>
__global__ void __launch_bounds__((kSmallWarps + 1) * 32) gdn_verify_ring(const KParams p)
{
    constexpr bool CHAIN = TREE == kTreeChain;
    constexpr bool INDEX = TREE == kTreeIndex;
    constexpr int EPC = 16 / sizeof(QT);  // elements per 16-byte chunk
    constexpr int QKCH = DK / EPC;        // chunks per k (or q) row
    using LM = LaneMap<DK, C, RL>;
    constexpr int VCH_MAX = (kSmallWarps * LM::RPW + EPC - 1) / EPC;  // chunks per v slice, upper bound
    constexpr int MAXT = (kChunk * (2 * QKCH + VCH_MAX) + 31) / 32;

    extern __shared__ __align__(16) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kRing;
    unsigned char* ring = smem + p.off_raw;
    const uint32_t desc_off = (kChunk * p.raw_bytes + 15u) & ~15u;
    const uint32_t slot_bytes = desc_off + kChunk * (uint32_t)(sizeof(PosDesc) + 4);
    float* slotbuf = reinterpret_cast<float*>(smem + p.off_slots);
    const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int hk = h / p.G;
    const int row0 = tile * p.rows;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const QT* kg = static_cast<const QT*>(p.k);
    const QT* qg = static_cast<const QT*>(p.q);
    const QT* vg = static_cast<const QT*>(p.v);
    if (!p.early_tree)
        pdl_wait_then_release();
    Seq sq;
    if (!seq_of(p, b, sq)) {
        if (tid == 0)
            report_status(p.status, GDN_ERR_BAD_TREE);
        return;
    }
    const int N = sq.N;
    const TreeView T(reinterpret_cast<int*>(smem + p.off_tree), N);
    // qk_norm on trees: 1 / |k| per node, for recomputations (chains never recompute)
    float* rkn = (p.qk_norm && !CHAIN && !INDEX) ? reinterpret_cast<float*>(smem + p.off_ab) : nullptr;

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
                const int pn = __ldg(p.parent + (size_t)sq.n0 + n);
                if (INDEX) {
                    T.par[n] = pn;
                    bad |= (n == 0) ? (pn != -1) : (pn < 0 || pn >= n);
                } else {
                    bad |= pn != n - 1;
                }
            }
        }
        ok = !__syncthreads_or(bad);
    } else if (p.plan != nullptr) {
        // the walk from the plan (see the staged kernel)
        const int32_t* pl = p.plan + (size_t)b * p.plan_stride;
        for (int i = 4 * tid; i < 4 * N; i += 4 * blockDim.x)
            cp_async16(T.par + i, pl + kPlanHeader + i);
        asm volatile("cp.async.commit_group;" ::: "memory");
        const int sig = __ldg(pl), pok = __ldg(pl + 1), pn = __ldg(pl + 2);
        if (sig != p.plan_sig || pn != N) {
            if (tid == 0)
                report_status(p.status, GDN_ERR_BAD_INPUT);
            ok = false;
        } else {
            ok = pok == 1;
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncthreads();
    } else {
        __syncthreads();
        ok = (N <= kMaskNodes && N <= (int)blockDim.x) ? build_walk_masked(p.parent + (size_t)sq.n0, N, p.slots, T)
                                                       : build_walk(p.parent + (size_t)sq.n0, N, p.slots, T);
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
            unsigned char* base = ring + (size_t)s * slot_bytes;
            PosDesc* sdesc = reinterpret_cast<PosDesc*>(base + desc_off);
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
                    const size_t node = (size_t)sq.n0 + n;
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
            // lane i < cnt: position p0 + i's node, metadata and scalars
            int dn = 0, dm = 0, drs = -1, dpp = -1;
            float da = 0.f, dbe = 0.f;  // g and beta here; a and beta once the records are stored
            if (lane < cnt) {
                const int pos = p0 + lane;
                if constexpr (CHAIN) {
                    dm = NoTree{}.meta(pos);
                } else if constexpr (INDEX) {
                    dm = IndexTree{T.par}.meta(pos);
                } else {
                    dm = T.meta[pos];
                    drs = T.rstart[pos];
                }
                dn = meta_node(dm);
                dpp = CHAIN ? dn - 1 : T.par[dn];
                const size_t gi = ((size_t)sq.n0 + dn) * p.Hv + h;
                da = __ldg(p.g + gi);
                dbe = __ldg(p.beta + gi);
            }
#pragma unroll
            for (int t = 0; t < MAXT; ++t) {
                const int idx = lane + 32 * t;
                if (idx < total) {
                    const int i = idx / per_pos, j = idx - i * per_pos;
                    int off = 16 * j;
                    if constexpr (sizeof(QT) == 4) {
                        // f32 k and q rows land swizzled (swz_pos)
                        if (j < 2 * QKCH) {
                            const int part = j < QKCH ? 0 : QKCH;
                            const int jj = (j - part) >> 1, hh = (j - part) & 1;
                            off = 16 * part + 32 * jj + 16 * (hh ^ (((jj % LM::LR) >> 2) & 1));
                        }
                    }
                    *reinterpret_cast<uint4*>(base + (size_t)i * p.raw_bytes + off) = regs[t];
                }
            }
            // (the gate call comes after the record registers are dead)
            if (lane < cnt)
                gate_scalars(da, dbe, p.gates, da, dbe);
            __syncwarp();
            for (int i0 = 0; i0 < cnt; i0 += 4) {
                const int gi = i0 + (lane >> 3);
                const int i = min(gi, cnt - 1);
                const QT* rrec = reinterpret_cast<const QT*>(base + (size_t)i * p.raw_bytes);
                float kq, rk = 1.f, rq = 1.f;
                if (p.qk_norm) {
                    float kk, qq;
                    node_dots8<DK, LM::LR>(rrec, lane & 7, kq, kk, qq);
                    rk = inv_norm(kk);
                    rq = inv_norm(qq);
                } else {
                    kq = node_kq8<DK, LM::LR>(rrec, lane & 7);
                }
                const int src_lane = i;
                const int n = __shfl_sync(0xffffffffu, dn, src_lane);
                const int m = __shfl_sync(0xffffffffu, dm, src_lane);
                const int rs = __shfl_sync(0xffffffffu, drs, src_lane);
                const int pp = __shfl_sync(0xffffffffu, dpp, src_lane);
                const float a = __shfl_sync(0xffffffffu, da, src_lane);
                const float be = __shfl_sync(0xffffffffu, dbe, src_lane);
                if ((lane & 7) == 0 && gi < cnt) {
                    float bp, ap;
                    node_scalars(a, be, rk, bp, ap);
                    PosDesc d;
                    d.i = make_int4(n, m, rs, pp);
                    d.f = make_float4(a, bp, kq, ap);
                    sdesc[i] = d;
                    reinterpret_cast<float*>(sdesc + kChunk)[i] = __fmul_rn(p.scale, rq);
                    if (rkn != nullptr)
                        rkn[n] = rk;  // for recomputation of this node's subtree
                }
            }
            mbar_arrive(&full[s]);
        }
        return;
    }

    // ---------------------------------------------------------------- compute
    const LM L(warp, lane);
    const float* sin_lane =
        p.state_in + ((size_t)b * p.Hv + h) * p.dv * DK + (size_t)row0 * DK + L.tile_offset();
    StateT<C, RL> S;
    load_rows<DK, C, RL>(S, sin_lane);
    const GlobalFetch<DK, C, RL, QT> gf{kg, vg, p.g, p.beta, (size_t)sq.n0, rkn, p.Hk, p.Hv, p.dv, hk, h, row0, L,
                                        p.gates};
    RingCtx<DK, C, RL, QT> ctx{full, empty, ring, p.raw_bytes, slot_bytes, desc_off, p.status, lane, gf};
    float* lane_slot = cta_slots<DK, TREE>(p, slotbuf) + 4 * threadIdx.x;
    if constexpr (CHAIN)
        walk<DK, C, RL, QT, ST, TREE>(S, p, sq, NoTree{}, lane_slot, 0u, sin_lane, b, h, row0, L, ctx);
    else if constexpr (INDEX)
        walk<DK, C, RL, QT, ST, TREE>(S, p, sq, IndexTree{T.par}, lane_slot, 0u, sin_lane, b, h, row0, L, ctx);
    else
        walk<DK, C, RL, QT, ST, TREE>(S, p, sq, SmemTree{T, N, warp}, lane_slot, 0u, sin_lane, b, h, row0, L, ctx);
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

template <auto KERNEL>
cudaError_t launch_granted(const KParams& kp, dim3 grid, const VerifyGeom& geom, cudaStream_t stream)
{
    cudaError_t e = grant_smem<KERNEL>(geom.smem);
    if (e != cudaSuccess)
        return e;
    return launch_pdl(KERNEL, grid, dim3(geom.warps * 32), geom.smem, stream, kp);
}

template <int DK, int C, int RL, typename QT, typename ST, int TREE>
cudaError_t launch_staged(const KParams& kp, const VerifyArgs& a, const VerifyGeom& geom,
                          cudaStream_t stream)
{
    dim3 grid(geom.tiles, a.n_v_heads, a.batch);
    if constexpr (TREE == kTreeWarp && RL == 1 && sizeof(QT) == 2)
        return launch_granted<gdn_verify_staged_dense<DK, C, RL, QT, ST, TREE>>(kp, grid, geom, stream);
    if constexpr ((TREE == kTreeSmem || TREE == kTreeSmem + kTreeTmem || TREE == kTreeWarp + kTreeTmem) && RL == 2) {
        if (geom.warps > kSmallWarps)
            return launch_granted<gdn_verify_staged_wide<DK, C, RL, QT, ST, TREE>>(kp, grid, geom, stream);
    }
    if constexpr ((TREE & kTreeTmem) != 0)
        return cudaErrorInvalidConfiguration;  // not reached: tensor-memory slots only with the wide kernel
    if (geom.warps > kSmallWarps)
        return cudaErrorInvalidConfiguration;  // not reached: the geometry only widens the kinds above
    return launch_granted<gdn_verify_staged<DK, C, RL, QT, ST, TREE>>(kp, grid, geom, stream);
}

template <int DK, int C, int RL, typename QT, typename ST, int TREE>
cudaError_t launch_ring(const KParams& kp, const VerifyArgs& a, const VerifyGeom& geom,
                        cudaStream_t stream)
{
    dim3 grid(geom.tiles, a.n_v_heads, a.batch);
    cudaError_t e = grant_smem<gdn_verify_ring<DK, C, RL, QT, ST, TREE>>(geom.smem);
    if (e != cudaSuccess)
        return e;
    return launch_pdl(gdn_verify_ring<DK, C, RL, QT, ST, TREE>, grid, dim3((geom.warps + 1) * 32),
                      geom.smem, stream, kp);
}

template <int DK, int C, int RL, typename QT, typename ST, bool CHAIN>
cudaError_t launch_one(const KParams& kp, const VerifyArgs& a, const VerifyGeom& geom,
                       cudaStream_t stream)
{
    if (geom.staged) {
        if (CHAIN)
            return launch_staged<DK, C, RL, QT, ST, kTreeChain>(kp, a, geom, stream);
        if (geom.reload)
            return launch_staged<DK, C, RL, QT, ST, kTreeIndex>(kp, a, geom, stream);
        if (geom.warp_tree) {
            if constexpr (RL == 2 && C * RL * 8 == 32) {
                if (geom.tslots)
                    return launch_staged<DK, C, RL, QT, ST, kTreeWarp + kTreeTmem>(kp, a, geom, stream);
            }
            return geom.gslots ? launch_staged<DK, C, RL, QT, ST, kTreeWarp + kTreeGlobal>(kp, a, geom, stream)
                               : launch_staged<DK, C, RL, QT, ST, kTreeWarp>(kp, a, geom, stream);
        }
        if constexpr (RL == 2 && C * RL * 8 == 32) {
            if (geom.tslots)
                return launch_staged<DK, C, RL, QT, ST, kTreeSmem + kTreeTmem>(kp, a, geom, stream);
        }
        return geom.gslots ? launch_staged<DK, C, RL, QT, ST, kTreeSmem + kTreeGlobal>(kp, a, geom, stream)
                           : launch_staged<DK, C, RL, QT, ST, kTreeSmem>(kp, a, geom, stream);
    }
    if (CHAIN)
        return launch_ring<DK, C, RL, QT, ST, kTreeChain>(kp, a, geom, stream);
    if (geom.reload)
        return launch_ring<DK, C, RL, QT, ST, kTreeIndex>(kp, a, geom, stream);
    return geom.gslots ? launch_ring<DK, C, RL, QT, ST, kTreeSmem + kTreeGlobal>(kp, a, geom, stream)
                       : launch_ring<DK, C, RL, QT, ST, kTreeSmem>(kp, a, geom, stream);
}

template <int DK, int C, int RL, typename QT, typename ST>
cudaError_t launch_mode(const KParams& kp, const VerifyArgs& a, const VerifyGeom& g, cudaStream_t s)
{
    if (a.flags & GDN_FLAG_CHAIN)
        return launch_one<DK, C, RL, QT, ST, true>(kp, a, g, s);
    return launch_one<DK, C, RL, QT, ST, false>(kp, a, g, s);
}

template <int DK, int C, int RL, typename QT>
cudaError_t launch_state(const KParams& kp, const VerifyArgs& a, const VerifyGeom& g, cudaStream_t s)
{
    if (a.state_dtype == GDN_F16)
        return launch_mode<DK, C, RL, QT, __half>(kp, a, g, s);
    return launch_mode<DK, C, RL, QT, float>(kp, a, g, s);
}

template <int DK, int C, int RL>
cudaError_t launch_shape(const KParams& kp, const VerifyArgs& a, const VerifyGeom& g, cudaStream_t s)
{
    if (a.qkv_dtype == GDN_BF16)
        return launch_state<DK, C, RL, __nv_bfloat16>(kp, a, g, s);
    return launch_state<DK, C, RL, float>(kp, a, g, s);
}

// Launches the verify kernel for head dim DK and lane shape (C, RL); each
// shape is instantiated in its own translation unit.
template <int DK, int C, int RL>
cudaError_t launch_dk(const KParams& kp, const VerifyArgs& a, const VerifyGeom& g, cudaStream_t s)
{
    return launch_shape<DK, C, RL>(kp, a, g, s);
}

}  // namespace verify
}  // namespace gdn
