// gdn_verify.cu -- the tree-verify kernel of libgdntree (sm_100a).
//
// One CTA per (sequence b, v-head h, tile of d_v rows).  The CTA walks the
// tree's nodes in depth-first preorder (children in increasing index order),
// which is a topological order, and for each node applies the gated delta
// rule (Gated DeltaNet; the ggml_gated_delta_net recurrence named in the
// GreenGames post, "TL;DR"):
//
//     a = exp(g_n);  w = a * S_p k_n;  u = beta_n * (v_n - w)
//     S_n = a * S_p + u k_n^T;         o_n = scale * S_n q_n
//
// and persists S_n from inside the kernel (the GreenGames post, "Key wins":
// persist-write kernel, f16 intermediate cache).
//
// Work split inside a CTA (warp specialisation):
//   * one producer warp stages, chunk by chunk in walk order, each node's
//     k and q rows (widened to fp32 once), the CTA's slice of v, a = exp(g)
//     and beta into a shared-memory ring guarded by mbarriers;
//   * `warps` compute warps each own 8 (d_k = 128) state rows in registers:
//     lane (row group rg, column lane c) holds 2 rows x 16 columns, with
//     LR = d_k / 16 lanes per row.  S k and S q are 16-term packed-fp32
//     partial dots plus an xor-butterfly over the LR lanes of a row; the
//     rank-1 update is packed fp32 (FFMA2).  Each node's state leaves as
//     16-byte (fp32) or 8-byte (f16) coalesced stores.
//
// Parents that are not the previous node in the walk: a node with two or
// more children saves its fp32 state in a shared-memory stack slot indexed
// by its number of branching ancestors; a later child reloads it.  When a
// tree nests branch points deeper than the stack, the parent's state is
// recomputed exactly (same instruction sequence) from the deepest saved
// ancestor.  The recurrence therefore always continues from the exact fp32
// state, whatever the persisted dtype.
//
// Every arithmetic step uses explicit round-to-nearest intrinsics, so a
// node's results depend only on its root path: a chain run through the tree
// walk, the chain fast path and a recomputed path give identical bits.

#include <atomic>
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int kRowsPerLane = 2;      // RL
constexpr int kColsPerLane = 16;     // 4 chunks of 4 consecutive columns
constexpr int kMaxWarps = 4;         // compute warps per CTA
constexpr int kChunkMax = 8;         // walk positions per ring slot
constexpr int kMaxThreads = (kMaxWarps + 1) * 32;
constexpr int kMaxDevices = 64;

// Per-position walk metadata (tree mode), packed in one int32:
//   bits  0..15 node id, 16..17 source of the parent state,
//   bits 18..22 save slot + 1 (0: do not save), 24..28 load slot.
enum : int { kSrcCont = 0, kSrcSlot = 1, kSrcRecompute = 2, kSrcRoot = 3 };

__device__ __forceinline__ int meta_node(int m) { return m & 0xffff; }
__device__ __forceinline__ int meta_src(int m) { return (m >> 16) & 3; }
__device__ __forceinline__ int meta_save(int m) { return ((m >> 18) & 31) - 1; }
__device__ __forceinline__ int meta_load(int m) { return (m >> 24) & 31; }

// The decay gate a = exp(g), compiled once so that every caller (the
// producer warp and the recompute path) gets identical bits.
__device__ __noinline__ float gdn_gate(float g) { return expf(g); }

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
    int rows, warps, chunk, ring, slots;
    int persist_last, validate;
    uint32_t off_ring, off_slots, off_tree, rec_stride;
};

// One node's state update on a lane's 2 rows x 16 columns (packed as float2).
// Used by the main walk and by the recompute path; explicit intrinsics keep
// both bit-identical.
template <int LR>
__device__ __forceinline__ void gdn_step(float2 (&S)[kRowsPerLane][8], const float2 (&k2)[8],
                                         const float (&vr)[kRowsPerLane], float a, float beta)
{
    float w[kRowsPerLane];
#pragma unroll
    for (int r = 0; r < kRowsPerLane; ++r) {
        float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int t = 0; t < 8; t += 2) {
            acc0 = __ffma2_rn(S[r][t], k2[t], acc0);
            acc1 = __ffma2_rn(S[r][t + 1], k2[t + 1], acc1);
        }
        w[r] = __fadd_rn(__fadd_rn(acc0.x, acc0.y), __fadd_rn(acc1.x, acc1.y));
    }
#pragma unroll
    for (int off = 1; off < LR; off <<= 1) {
#pragma unroll
        for (int r = 0; r < kRowsPerLane; ++r)
            w[r] = __fadd_rn(w[r], __shfl_xor_sync(0xffffffffu, w[r], off));
    }
    const float2 a2 = make_float2(a, a);
#pragma unroll
    for (int r = 0; r < kRowsPerLane; ++r) {
        const float u = __fmul_rn(beta, __fsub_rn(vr[r], __fmul_rn(a, w[r])));
        const float2 u2 = make_float2(u, u);
#pragma unroll
        for (int t = 0; t < 8; ++t)
            S[r][t] = __ffma2_rn(u2, k2[t], __fmul2_rn(a2, S[r][t]));
    }
}

template <int LR>
__device__ __forceinline__ void gdn_output(const float2 (&S)[kRowsPerLane][8], const float2 (&q2)[8],
                                           float scale, float (&o)[kRowsPerLane])
{
#pragma unroll
    for (int r = 0; r < kRowsPerLane; ++r) {
        float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int t = 0; t < 8; t += 2) {
            acc0 = __ffma2_rn(S[r][t], q2[t], acc0);
            acc1 = __ffma2_rn(S[r][t + 1], q2[t + 1], acc1);
        }
        o[r] = __fadd_rn(__fadd_rn(acc0.x, acc0.y), __fadd_rn(acc1.x, acc1.y));
    }
#pragma unroll
    for (int off = 1; off < LR; off <<= 1) {
#pragma unroll
        for (int r = 0; r < kRowsPerLane; ++r)
            o[r] = __fadd_rn(o[r], __shfl_xor_sync(0xffffffffu, o[r], off));
    }
#pragma unroll
    for (int r = 0; r < kRowsPerLane; ++r)
        o[r] = __fmul_rn(scale, o[r]);
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

// Builds the depth-first walk of one tree (tree mode; thread 0 runs the
// sequential passes, the rest of the CTA the parallel ones).  Returns false
// (on every thread) if the tree is malformed.
__device__ bool build_walk(const KParams& p, int b, int* tree)
{
    const int N = p.N;
    const int tid = threadIdx.x, nthr = blockDim.x;
    int* par = tree;
    int* ord = par + N;
    int* meta = ord + N;
    int* rstart = meta + N;
    int* nch = rstart + N;
    int* sz = nch + N;
    int* bd = sz + N;
    int* nxt = bd + N;

    bool bad = false;
    for (int n = tid; n < N; n += nthr) {
        const int pn = __ldg(p.parent + (size_t)b * N + n);
        par[n] = pn;
        nch[n] = 0;
        sz[n] = 1;
        bad |= (n == 0) ? (pn != -1) : (pn < 0 || pn >= n);
    }
    if (__syncthreads_or(bad))
        return false;
    for (int n = 1 + tid; n < N; n += nthr)
        atomicAdd(&nch[par[n]], 1);
    __syncthreads();
    if (tid == 0) {
        for (int n = N - 1; n >= 1; --n)
            sz[par[n]] += sz[n];
        bd[0] = 0;
        nxt[0] = 1;
        ord[0] = 0;
        for (int n = 1; n < N; ++n) {
            const int pp = par[n];
            bd[n] = bd[pp] + (nch[pp] >= 2 ? 1 : 0);
            const int pos = nxt[pp];
            nxt[pp] = pos + sz[n];
            nxt[n] = pos + 1;
            ord[pos] = n;
        }
    }
    __syncthreads();
    const int K = p.slots;
    for (int pos = tid; pos < N; pos += nthr) {
        const int n = ord[pos];
        const int pp = par[n];
        int src, ld = 0, start = -1;
        if (pos == 0) {
            src = kSrcRoot;
        } else if (pp == ord[pos - 1]) {
            src = kSrcCont;
        } else if (bd[pp] < K) {
            src = kSrcSlot;
            ld = bd[pp];
        } else {
            src = kSrcRecompute;
            // Deepest saved ancestor of pp: the branching ancestor with K - 1
            // branching ancestors above it (none when K == 0: start from the
            // root's parent state, state_in).
            int x = par[pp];
            while (x >= 0 && !(nch[x] >= 2 && bd[x] == K - 1))
                x = par[x];
            start = x;
        }
        const int save = (nch[n] >= 2 && bd[n] < K) ? bd[n] + 1 : 0;
        meta[pos] = n | (src << 16) | (save << 18) | (ld << 24);
        rstart[pos] = start;
    }
    __syncthreads();
    return true;
}

template <int DK, typename QT, typename ST, bool CHAIN>
__global__ void __launch_bounds__(kMaxThreads) gdn_verify_kernel(const KParams p)
{
    constexpr int LR = DK / kColsPerLane;           // lanes per row
    constexpr int RG = 32 / LR;                     // row groups per warp
    constexpr int RPW = kRowsPerLane * RG;          // rows per warp
    constexpr int EPC = 16 / sizeof(QT);            // elements per 16-byte chunk
    constexpr int QKCH = DK / EPC;                  // chunks per q (or k) row
    constexpr int VCH_MAX = kMaxWarps * RPW / EPC;  // chunks per v slice, upper bound
    constexpr int MAXT = (kChunkMax * (2 * QKCH + VCH_MAX) + 31) / 32;

    extern __shared__ __align__(16) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + p.ring;
    float* ring = reinterpret_cast<float*>(smem + p.off_ring);
    float* slotbuf = reinterpret_cast<float*>(smem + p.off_slots);
    int* tree = reinterpret_cast<int*>(smem + p.off_tree);

    const int N = p.N;
    const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int hk = h / p.G;
    const int row0 = tile * p.rows;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tid = threadIdx.x;

    if (tid == 0) {
        for (int i = 0; i < p.ring; ++i) {
            mbar_init(&full[i], 32);
            mbar_init(&empty[i], p.warps);
        }
        mbar_init_fence();
    }
    if constexpr (CHAIN) {
        bool bad = false;
        if (p.validate) {
            for (int n = tid; n < N; n += blockDim.x)
                bad |= __ldg(p.parent + (size_t)b * N + n) != n - 1;
        }
        if (__syncthreads_or(bad)) {
            if (tid == 0)
                report_status(p.status, GDN_ERR_BAD_TREE);
            return;
        }
    } else {
        __syncthreads();
        if (!build_walk(p, b, tree)) {
            if (tid == 0)
                report_status(p.status, GDN_ERR_BAD_TREE);
            return;
        }
    }
    const int* meta = tree + 2 * N;
    const int* rstart = tree + 3 * N;
    const int* par = tree;

    const int n_chunks = (N + p.chunk - 1) / p.chunk;
    const int rs = p.rec_stride;

    if (warp == p.warps) {
        // ------------------------------------------------------------ producer
        const QT* qg = static_cast<const QT*>(p.q);
        const QT* kg = static_cast<const QT*>(p.k);
        const QT* vg = static_cast<const QT*>(p.v);
        const int vch = p.rows / EPC;
        const int per_pos = 2 * QKCH + vch;
        for (int c = 0; c < n_chunks; ++c) {
            const int s = c % p.ring, use = c / p.ring;
            if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1)) {
                report_status(p.status, kStatusTimeout);
                return;
            }
            float* base = ring + (size_t)s * p.chunk * rs;
            const int p0 = c * p.chunk;
            const int cnt = min(p.chunk, N - p0);
            const int total = cnt * per_pos;
            uint4 regs[MAXT];
#pragma unroll
            for (int t = 0; t < MAXT; ++t) {
                const int idx = lane + 32 * t;
                if (idx < total) {
                    const int i = idx / per_pos, j = idx - i * per_pos;
                    const int pos = p0 + i;
                    const int n = CHAIN ? pos : meta_node(meta[pos]);
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
                const int n = CHAIN ? pos : meta_node(meta[pos]);
                const size_t gi = ((size_t)b * N + n) * p.Hv + h;
                float* rec = base + (size_t)lane * rs + 2 * DK + p.rows;
                rec[0] = gdn_gate(__ldg(p.g + gi));
                rec[1] = __ldg(p.beta + gi);
                rec[2] = __int_as_float(n);
            }
#pragma unroll
            for (int t = 0; t < MAXT; ++t) {
                const int idx = lane + 32 * t;
                if (idx < total) {
                    const int i = idx / per_pos, j = idx - i * per_pos;
                    float* rec = base + (size_t)i * rs;
                    float* dst = (j < 2 * QKCH) ? rec + j * EPC : rec + 2 * DK + (j - 2 * QKCH) * EPC;
                    Widen<QT>::store(dst, regs[t]);
                }
            }
            mbar_arrive(&full[s]);
        }
        return;
    }

    // ---------------------------------------------------------------- compute
    const int rg = lane / LR, cl = lane % LR;
    int rloc[kRowsPerLane];
#pragma unroll
    for (int r = 0; r < kRowsPerLane; ++r)
        rloc[r] = warp * RPW + rg + r * RG;
    const size_t head = (size_t)b * p.Hv + h;
    const float* sin = p.state_in + head * p.dv * DK;

    float2 S[kRowsPerLane][8];
#pragma unroll
    for (int r = 0; r < kRowsPerLane; ++r) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float4 x = __ldg(reinterpret_cast<const float4*>(
                sin + (size_t)(row0 + rloc[r]) * DK + 4 * (cl + m * LR)));
            S[r][2 * m] = make_float2(x.x, x.y);
            S[r][2 * m + 1] = make_float2(x.z, x.w);
        }
    }

    const int NS = p.persist_last ? 1 : N;
    ST* nst = static_cast<ST*>(p.node_states);

    for (int c = 0; c < n_chunks; ++c) {
        const int s = c % p.ring, use = c / p.ring;
        if (!mbar_wait(&full[s], use & 1)) {
            report_status(p.status, kStatusTimeout);
            return;
        }
        const float* base = ring + (size_t)s * p.chunk * rs;
        const int p0 = c * p.chunk;
        const int cnt = min(p.chunk, N - p0);
        for (int i = 0; i < cnt; ++i) {
            const int pos = p0 + i;
            const float* rec = base + (size_t)i * rs;
            int save = -1;
            if constexpr (!CHAIN) {
                const int m = meta[pos];
                save = meta_save(m);
                const int src = meta_src(m);
                if (src == kSrcSlot) {
                    const float* sl = slotbuf + (size_t)meta_load(m) * p.rows * DK;
#pragma unroll
                    for (int r = 0; r < kRowsPerLane; ++r) {
#pragma unroll
                        for (int mm = 0; mm < 4; ++mm) {
                            const float4 x = *reinterpret_cast<const float4*>(
                                sl + (size_t)rloc[r] * DK + 4 * (cl + mm * LR));
                            S[r][2 * mm] = make_float2(x.x, x.y);
                            S[r][2 * mm + 1] = make_float2(x.z, x.w);
                        }
                    }
                } else if (src == kSrcRecompute) {
                    // Rebuild the parent's state from the deepest saved ancestor
                    // (or from state_in), re-running the same update on each node
                    // of the path in between, with inputs read from global memory.
                    const int target = par[meta_node(m)];
                    const int start = rstart[pos];
                    int* path = tree + 8 * N + warp * N;
                    int len = 0;
                    for (int x = target; x != start; x = par[x])
                        path[len++] = x;  // every lane writes the same values
                    __syncwarp();
                    if (start >= 0) {
                        const float* sl = slotbuf + (size_t)(p.slots - 1) * p.rows * DK;
#pragma unroll
                        for (int r = 0; r < kRowsPerLane; ++r) {
#pragma unroll
                            for (int mm = 0; mm < 4; ++mm) {
                                const float4 x = *reinterpret_cast<const float4*>(
                                    sl + (size_t)rloc[r] * DK + 4 * (cl + mm * LR));
                                S[r][2 * mm] = make_float2(x.x, x.y);
                                S[r][2 * mm + 1] = make_float2(x.z, x.w);
                            }
                        }
                    } else {
#pragma unroll
                        for (int r = 0; r < kRowsPerLane; ++r) {
#pragma unroll
                            for (int mm = 0; mm < 4; ++mm) {
                                const float4 x = __ldg(reinterpret_cast<const float4*>(
                                    sin + (size_t)(row0 + rloc[r]) * DK + 4 * (cl + mm * LR)));
                                S[r][2 * mm] = make_float2(x.x, x.y);
                                S[r][2 * mm + 1] = make_float2(x.z, x.w);
                            }
                        }
                    }
                    const QT* kg = static_cast<const QT*>(p.k);
                    const QT* vg = static_cast<const QT*>(p.v);
                    for (int e = len - 1; e >= 0; --e) {
                        const int y = path[e];
                        const size_t node = (size_t)b * N + y;
                        float2 k2[8];
#pragma unroll
                        for (int mm = 0; mm < 4; ++mm) {
                            const float4 x = Widen<QT>::load4(kg + (node * p.Hk + hk) * DK +
                                                               4 * (cl + mm * LR));
                            k2[2 * mm] = make_float2(x.x, x.y);
                            k2[2 * mm + 1] = make_float2(x.z, x.w);
                        }
                        float vr[kRowsPerLane];
#pragma unroll
                        for (int r = 0; r < kRowsPerLane; ++r)
                            vr[r] = Widen<QT>::load1(vg + (node * p.Hv + h) * p.dv + row0 + rloc[r]);
                        const size_t gi = node * p.Hv + h;
                        const float a = gdn_gate(__ldg(p.g + gi));
                        const float be = __ldg(p.beta + gi);
                        gdn_step<LR>(S, k2, vr, a, be);
                    }
                    __syncwarp();
                }
            }
            float2 k2[8], q2[8];
#pragma unroll
            for (int mm = 0; mm < 4; ++mm) {
                const float4 x = *reinterpret_cast<const float4*>(rec + 4 * (cl + mm * LR));
                const float4 y = *reinterpret_cast<const float4*>(rec + DK + 4 * (cl + mm * LR));
                k2[2 * mm] = make_float2(x.x, x.y);
                k2[2 * mm + 1] = make_float2(x.z, x.w);
                q2[2 * mm] = make_float2(y.x, y.y);
                q2[2 * mm + 1] = make_float2(y.z, y.w);
            }
            float vr[kRowsPerLane];
#pragma unroll
            for (int r = 0; r < kRowsPerLane; ++r)
                vr[r] = rec[2 * DK + rloc[r]];
            const float a = rec[2 * DK + p.rows];
            const float be = rec[2 * DK + p.rows + 1];
            const int n = __float_as_int(rec[2 * DK + p.rows + 2]);

            gdn_step<LR>(S, k2, vr, a, be);

            float o[kRowsPerLane];
            gdn_output<LR>(S, q2, p.scale, o);
            if (cl == 0) {
#pragma unroll
                for (int r = 0; r < kRowsPerLane; ++r)
                    p.out[(((size_t)b * N + n) * p.Hv + h) * p.dv + row0 + rloc[r]] = o[r];
            }
            if (!p.persist_last || pos == N - 1) {
                const int ni = p.persist_last ? 0 : n;
                ST* dst = nst + (((size_t)b * NS + ni) * p.Hv + h) * p.dv * DK;
#pragma unroll
                for (int r = 0; r < kRowsPerLane; ++r) {
#pragma unroll
                    for (int mm = 0; mm < 4; ++mm)
                        Persist<ST>::store(dst + (size_t)(row0 + rloc[r]) * DK + 4 * (cl + mm * LR),
                                           S[r][2 * mm], S[r][2 * mm + 1]);
                }
            }
            if (save >= 0) {
                float* sl = slotbuf + (size_t)save * p.rows * DK;
#pragma unroll
                for (int r = 0; r < kRowsPerLane; ++r) {
#pragma unroll
                    for (int mm = 0; mm < 4; ++mm)
                        *reinterpret_cast<float4*>(sl + (size_t)rloc[r] * DK + 4 * (cl + mm * LR)) =
                            make_float4(S[r][2 * mm].x, S[r][2 * mm].y, S[r][2 * mm + 1].x,
                                        S[r][2 * mm + 1].y);
                }
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[s]);
    }
}

template <int DK, typename QT, typename ST, bool CHAIN>
cudaError_t launch_one(const KParams& kp, const VerifyArgs& a, const VerifyGeom& geom,
                       cudaStream_t stream)
{
    auto kern = gdn_verify_kernel<DK, QT, ST, CHAIN>;
    if (geom.smem > 48 * 1024) {
        // Opt in to more than 48 KB of dynamic shared memory once per device
        // for the largest size requested so far.
        static std::atomic<int> granted[kMaxDevices];
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess)
            return e;
        if (dev < 0 || dev >= kMaxDevices || granted[dev].load() < (int)geom.smem) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)geom.smem);
            if (e != cudaSuccess)
                return e;
            if (dev >= 0 && dev < kMaxDevices) {
                int cur = granted[dev].load();
                while (cur < (int)geom.smem && !granted[dev].compare_exchange_weak(cur, (int)geom.smem)) {
                }
            }
        }
    }
    dim3 grid(geom.tiles, a.n_v_heads, a.batch);
    dim3 block((geom.warps + 1) * 32);
    kern<<<grid, block, geom.smem, stream>>>(kp);
    return cudaGetLastError();
}

template <int DK, typename QT, typename ST>
cudaError_t launch_mode(const KParams& kp, const VerifyArgs& a, const VerifyGeom& g,
                        cudaStream_t s)
{
    if (a.flags & GDN_FLAG_CHAIN)
        return launch_one<DK, QT, ST, true>(kp, a, g, s);
    return launch_one<DK, QT, ST, false>(kp, a, g, s);
}

template <int DK, typename QT>
cudaError_t launch_state(const KParams& kp, const VerifyArgs& a, const VerifyGeom& g,
                         cudaStream_t s)
{
    if (a.state_dtype == GDN_F16)
        return launch_mode<DK, QT, __half>(kp, a, g, s);
    return launch_mode<DK, QT, float>(kp, a, g, s);
}

template <int DK>
cudaError_t launch_qkv(const KParams& kp, const VerifyArgs& a, const VerifyGeom& g,
                       cudaStream_t s)
{
    if (a.qkv_dtype == GDN_BF16)
        return launch_state<DK, __nv_bfloat16>(kp, a, g, s);
    return launch_state<DK, float>(kp, a, g, s);
}

}  // namespace

VerifyGeom verify_geometry(const VerifyArgs& a)
{
    VerifyGeom g{};
    const bool chain = (a.flags & GDN_FLAG_CHAIN) != 0;
    const int rpw = kRowsPerLane * 32 / (a.d_k / kColsPerLane);
    int warps = chain ? kMaxWarps : 2;
    while (warps > 1 && (a.d_v % (warps * rpw) != 0))
        warps >>= 1;
    g.warps = warps;
    g.rows = warps * rpw;
    g.tiles = (a.d_v % g.rows == 0) ? a.d_v / g.rows : 0;
    g.chunk = kChunkMax;
    g.ring = chain ? 4 : 2;
    if (chain) {
        g.slots = 0;
    } else {
        int k = 0;
        while ((2 << k) <= a.n_nodes)
            ++k;  // floor(log2(N))
        g.slots = k < 1 ? 1 : (k > 8 ? 8 : k);
    }
    const size_t rec = (size_t)(2 * a.d_k + g.rows + 4) * sizeof(float);
    size_t off = 64;  // barriers (2 * ring * 8 bytes <= 64)
    off += (size_t)g.ring * g.chunk * rec;
    off += (size_t)g.slots * g.rows * a.d_k * sizeof(float);
    if (!chain)
        off += (size_t)(8 + g.warps) * a.n_nodes * sizeof(int);
    g.smem = off;
    return g;
}

cudaError_t launch_verify(const VerifyArgs& a, const VerifyGeom& geom, cudaStream_t stream)
{
    KParams kp{};
    kp.q = a.q;
    kp.k = a.k;
    kp.v = a.v;
    kp.g = a.g;
    kp.beta = a.beta;
    kp.parent = a.parent;
    kp.state_in = a.state_in;
    kp.out = a.out;
    kp.node_states = a.node_states;
    kp.status = a.status;
    kp.N = a.n_nodes;
    kp.Hk = a.n_k_heads;
    kp.Hv = a.n_v_heads;
    kp.dv = a.d_v;
    kp.G = a.n_v_heads / a.n_k_heads;
    kp.scale = a.scale;
    kp.rows = geom.rows;
    kp.warps = geom.warps;
    kp.chunk = geom.chunk;
    kp.ring = geom.ring;
    kp.slots = geom.slots;
    kp.persist_last = (a.flags & GDN_FLAG_PERSIST_LAST) ? 1 : 0;
    kp.validate = (a.flags & GDN_FLAG_VALIDATE) ? 1 : 0;
    kp.rec_stride = (uint32_t)(2 * a.d_k + geom.rows + 4);
    kp.off_ring = 64;
    kp.off_slots = kp.off_ring + (uint32_t)(geom.ring * geom.chunk * kp.rec_stride * sizeof(float));
    kp.off_tree = kp.off_slots + (uint32_t)(geom.slots * geom.rows * a.d_k * sizeof(float));
    switch (a.d_k) {
        case 32: return launch_qkv<32>(kp, a, geom, stream);
        case 64: return launch_qkv<64>(kp, a, geom, stream);
        case 128: return launch_qkv<128>(kp, a, geom, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace gdn
