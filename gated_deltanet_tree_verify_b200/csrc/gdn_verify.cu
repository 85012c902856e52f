// gdn_verify.cu -- launch geometry and dispatch of the verify kernels (the
// kernels themselves are in gdn_verify.cuh, instantiated per head dim and
// lane shape in gdn_verify_d*_c*r*.cu).

#include <cstdint>

#include <cuda_runtime.h>

#include "gdn_internal.h"
#include "gdn_verify.cuh"

namespace gdn {
namespace verify {
#define GDN_EXTERN_SHAPE(DK, C, RL)                                                                \
    extern template cudaError_t launch_dk<DK, C, RL>(const KParams&, const VerifyArgs&,          \
                                                     const VerifyGeom&, cudaStream_t);
GDN_EXTERN_SHAPE(32, 2, 2)
GDN_EXTERN_SHAPE(32, 2, 1)
GDN_EXTERN_SHAPE(64, 2, 2)
GDN_EXTERN_SHAPE(64, 2, 1)
GDN_EXTERN_SHAPE(128, 2, 2)
GDN_EXTERN_SHAPE(128, 2, 1)
#undef GDN_EXTERN_SHAPE
}  // namespace verify

namespace {
size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

// Warps per SM below which a launch uses the lane shape with one row per
// lane (twice the warps, to hide the per-node dependency chain).
constexpr long long kWarpsPerSmTarget = 16;
constexpr long long kSms = 148;
// Large grids (two rows per lane): shared-memory stack slots per CTA for
// trees of <= 32, <= 96 and more nodes, and the warps per CTA of trees with
// shared-memory slots above 32 nodes (the node records are staged once per
// CTA, so wider CTAs spend less shared memory per row).
constexpr int kLargeGridSlots[3] = {1, 2, 3};
constexpr int kLargeTreeWarps = 8;
// Stack slots the wide kernel keeps in tensor memory (4 x 64 columns: two
// CTAs per SM fill its 512).
constexpr int kMaxTmemSlots = 4;
// Smallest tree that the wide kernel walks with tensor-memory slots; smaller
// trees stay on 4-warp CTAs (the wide kernel with tensor-memory slots measured
// 3-13 % slower for budgets 8-22 at batch 8, equal at batch 32).
// Layers whose k, q and v records total at most this many bytes prefetch them
// into L2 before the dependency wait (with GDN_FLAG_EARLY_TREE): the headline
// layer (one budget-22 tree, 48 v-heads) stages ~0.5 MB and gains ~2 %.
constexpr size_t kPrefetchMaxBytes = 2u << 20;
constexpr int kTmemMinNodes = 33;

template <int DK>
cudaError_t launch_shapes(const verify::KParams& kp, const VerifyArgs& a, const VerifyGeom& g,
                          cudaStream_t s)
{
    if (g.rows_per_lane == 2)
        return verify::launch_dk<DK, 2, 2>(kp, a, g, s);
    return verify::launch_dk<DK, 2, 1>(kp, a, g, s);
}
}  // namespace

using namespace verify;

VerifyGeom verify_geometry(const VerifyArgs& a, bool use_workspace)
{
    VerifyGeom g{};
    const bool chain = (a.flags & GDN_FLAG_CHAIN) != 0;
    const bool persist_last = (a.flags & GDN_FLAG_PERSIST_LAST) != 0;
    const size_t es = a.qkv_dtype == GDN_BF16 ? 2 : 4;

    // Lane shape: C = 2 chunks of 8 columns and RL rows per lane; two rows
    // (fewer instructions per row) unless that leaves fewer than
    // kWarpsPerSmTarget warps per SM.  (One chunk per lane, twice the warps
    // again, measured slower at every batch: the per-node overhead doubles.)
    auto rows_per_warp = [&](int c, int rl) { return rl * 32 * 8 * c / a.d_k; };
    auto total_warps = [&](int c, int rl) {
        return (long long)a.batch * a.n_v_heads * a.d_v / rows_per_warp(c, rl);
    };
    g.chunks = 2;
    g.rows_per_lane = total_warps(2, 2) >= kWarpsPerSmTarget * kSms ? 2 : 1;
    // f32 node states are the exact states, so an f32 tree can re-read a
    // branch's parent state from node_states and walk in index order.  On
    // large grids, trees above 32 nodes walk depth first with shared-memory
    // slots instead (measured 4-13 % faster at batch 8 and 32, budgets 32 to
    // 128); at one row per lane re-reading is faster at most budgets, and so
    // it is for packed trees of mixed sizes, whose shared memory is sized
    // for the largest.  Both give identical bits.
    g.reload = !chain && a.state_dtype == GDN_F32 && !persist_last &&
               !(g.rows_per_lane == 2 && a.n_nodes > 32 && a.cu_nodes == nullptr);
    int tmem_slots = 0;
    if (chain || g.reload) {
        g.slots = 0;
    } else {
        // floor(log2 N) slots make recomputation impossible.  In shared
        // memory fewer keep more CTAs resident: draft trees of budget <= 31
        // need at most 2, and with one about one node per tree is recomputed,
        // which pays off on large grids (more resident CTAs) but not on small
        // ones.  In a workspace only the size counts.
        int k = 0;
        while ((2 << k) <= a.n_nodes)
            ++k;
        g.gslots = use_workspace;
        // The wide kernel (two rows per lane, trees above 32 nodes) keeps
        // its slots in tensor memory, which the kernels do not otherwise
        // use: up to kMaxTmemSlots of them, none in shared memory.
        g.tslots = !chain && !g.reload && !g.gslots && a.n_nodes >= kTmemMinNodes && g.rows_per_lane == 2 &&
                   !persist_last && !(a.flags & GDN_FLAG_QK_L2NORM);
        const int size_class = a.n_nodes <= 32 ? 0 : (a.n_nodes <= 96 ? 1 : 2);
        const int cap = g.gslots ? 4 : (g.rows_per_lane == 2 ? kLargeGridSlots[size_class] : 2 + size_class);
        g.slots = k < 1 ? 1 : (k > cap ? cap : k);
        tmem_slots = k < 1 ? 1 : (k > kMaxTmemSlots ? kMaxTmemSlots : k);
    }
    const int rpw = rows_per_warp(g.chunks, g.rows_per_lane);
    // Staged kernel first (wide CTAs for large trees with shared-memory
    // slots on large grids, then the usual width), else the ring kernel
    // (which adds a producer warp).
    const bool wide = !chain && !g.reload && !g.gslots && g.rows_per_lane == 2 && (a.n_nodes > 32 || g.tslots);
    for (int pass = wide ? 0 : 1; pass < 3; ++pass) {
        const bool staged = pass < 2;
        int warps = pass == 0 ? kLargeTreeWarps : kSmallWarps;  // the ring kernel: kSmallWarps at most
        while (warps > 1 && a.d_v % (warps * rpw) != 0)
            --warps;
        const int rows = warps * rpw;
        if (a.d_v % rows != 0 || (rows * es) % 16 != 0)
            continue;
        const size_t raw_bytes = (size_t)(2 * a.d_k + rows) * es;
        // tensor-memory slots need the full 8 warps (a lane's 32 floats are
        // one 32-column store); otherwise shared-memory slots as usual
        const bool tmem = g.tslots && pass == 0 && warps == kLargeTreeWarps && rows * a.d_k == 32 * 32 * warps;
        const int slots = tmem ? tmem_slots : g.slots;
        const size_t slot_bytes = (g.gslots || tmem) ? 0 : (size_t)slots * rows * a.d_k * 4;
        size_t off = 64;  // mbarriers
        size_t off_raw = 0, off_desc = 0, off_ab = 0, off_slots = 0;
        if (staged) {
            off_raw = off;
            off += align16((size_t)a.n_nodes * raw_bytes);
            off_desc = off;
            off += (size_t)a.n_nodes * sizeof(PosDesc);
            off_ab = off;
            // g (then a) | beta', by node; with q/k normalisation also a' and
            // the output coefficient
            off += align16((size_t)((a.flags & GDN_FLAG_QK_L2NORM) ? 4 : 2) * a.n_nodes * 4);
        } else {
            off_ab = off;  // 1 / |k| by node (GDN_FLAG_QK_L2NORM trees)
            if ((a.flags & GDN_FLAG_QK_L2NORM) && !chain && !g.reload)
                off += align16((size_t)a.n_nodes * 4);
            off_raw = off;
            off += (size_t)kRing * (align16(kChunk * raw_bytes) + kChunk * (sizeof(PosDesc) + 4));
        }
        off_slots = off;
        off += align16(slot_bytes);
        // tree area: none for chains, the parent array for index order, the
        // warp-built walk (kWarpTreeInts ints), else the shared-memory walk
        const size_t off_tree = off;
        const bool warp_tree = staged && !chain && !g.reload && a.n_nodes <= 32;
        if (chain)
            off += 0;
        else if (g.reload)
            off += align16((size_t)a.n_nodes * 4);
        else if (warp_tree)
            off += kWarpTreeInts * 4;
        else  // the arrays, then the walk's per-warp path scratch (also the mask builder's)
            off += (size_t)(kTreeArrays + (warps > kMaskScratch ? warps : kMaskScratch)) * a.n_nodes * 4;
        if (staged && off > (size_t)kStagedMaxSmem)
            continue;
        g.staged = staged;
        g.warp_tree = warp_tree;
        g.warps = warps;
        g.rows = rows;
        g.tiles = a.d_v / rows;
        g.raw_bytes = (uint32_t)raw_bytes;
        g.off_raw = (uint32_t)off_raw;
        g.off_desc = (uint32_t)off_desc;
        g.off_ab = (uint32_t)off_ab;
        g.off_slots = (uint32_t)off_slots;
        g.off_tree = (uint32_t)off_tree;
        g.smem = off;
        g.ws_bytes = g.gslots ? (size_t)a.batch * a.n_v_heads * a.d_v * a.d_k * g.slots * 4 : 0;
        g.slots = slots;
        g.tslots = tmem;
        if (tmem) {
            // a lane's slot is 32 columns; the warps that share a lane
            // quarter sit side by side
            g.tmem_slot_cols = 32 * ((warps + 3) / 4);
            int cols = 32;
            while (cols < g.slots * g.tmem_slot_cols)
                cols *= 2;
            g.tmem_cols = cols;
        }
        break;
    }
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
    kp.slots = geom.slots;
    kp.persist_last = (a.flags & GDN_FLAG_PERSIST_LAST) ? 1 : 0;
    kp.validate = (a.flags & GDN_FLAG_VALIDATE) ? 1 : 0;
    kp.early_tree = (a.flags & GDN_FLAG_EARLY_TREE) ? 1 : 0;
    {
        // a layer's k, q and v bytes: the records the CTAs stage
        const size_t nodes = a.cu_nodes ? (size_t)a.total_nodes : (size_t)a.batch * a.n_nodes;
        const size_t esz = a.qkv_dtype == GDN_F32 ? 4 : 2;
        const size_t bytes = nodes * ((size_t)2 * a.n_k_heads * a.d_k + (size_t)a.n_v_heads * a.d_v) * esz;
        kp.prefetch = kp.early_tree && bytes <= kPrefetchMaxBytes;
    }
    kp.qk_norm = (a.flags & GDN_FLAG_QK_L2NORM) ? 1 : 0;
    kp.gates = (a.flags & GDN_FLAG_GATES) ? 1 : 0;
    kp.ws = geom.gslots ? a.workspace : nullptr;
    kp.tmem_cols = geom.tmem_cols;
    kp.tmem_slot_cols = geom.tmem_slot_cols;
    kp.cu = a.cu_nodes;
    kp.total = a.total_nodes;
    kp.raw_bytes = geom.raw_bytes;
    kp.off_raw = geom.off_raw;
    kp.off_desc = geom.off_desc;
    kp.off_ab = geom.off_ab;
    kp.off_slots = geom.off_slots;
    kp.off_tree = geom.off_tree;
    if (a.plan != nullptr) {
        const PlanGeom pg = plan_geometry(a);
        if (pg.needed) {
            kp.plan = a.plan;
            kp.plan_stride = pg.stride;
            kp.plan_sig = pg.sig;
        }
    }
    switch (a.d_k) {
        case 32: return launch_shapes<32>(kp, a, geom, stream);
        case 64: return launch_shapes<64>(kp, a, geom, stream);
        case 128: return launch_shapes<128>(kp, a, geom, stream);
        default: return cudaErrorInvalidValue;
    }
}

// ---------------------------------------------------------------------------
// Tree plans: the walk of each sequence built once, for every layer of a step
// ---------------------------------------------------------------------------

PlanGeom plan_geometry(const VerifyArgs& a)
{
    PlanGeom pg{};
    const VerifyGeom g = verify_geometry(a, false);
    const bool chain = (a.flags & GDN_FLAG_CHAIN) != 0;
    // Small grids (one row per lane) build walks while the previous layer
    // still runs (GDN_FLAG_EARLY_TREE), where they cost nothing: no plan.
    pg.needed = !chain && !g.reload && g.tiles > 0 && g.rows_per_lane == 2;
    pg.warp_kind = g.warp_tree;
    pg.slots = g.slots;
    pg.n_nodes = a.n_nodes;
    pg.stride = verify::kPlanHeader + (pg.warp_kind ? 128 : ((4 * a.n_nodes + 3) & ~3));
    pg.sig = 0x6D000000 | ((pg.warp_kind ? 1 : 2) << 20) | ((pg.slots & 15) << 16) | (a.n_nodes & 0xffff);
    return pg;
}

namespace verify {
namespace {

constexpr int kPlanThreads = 256;

// One CTA per sequence: the walk exactly as the staged kernels build it.
__global__ void __launch_bounds__(kPlanThreads)
    gdn_plan_kernel(const int32_t* parent, int N, int K, int warp_kind, int sig, int32_t* plan, int stride,
                    int32_t* status)
{
    extern __shared__ __align__(16) unsigned char smem[];
    int* tsm = reinterpret_cast<int*>(smem);
    pdl_wait_then_release();
    const int b = blockIdx.x, tid = threadIdx.x;
    const int32_t* prow = parent + (size_t)b * N;
    bool ok;
    if (warp_kind) {
        bool w_ok = true;
        if (tid < 32)
            w_ok = build_warp_walk(prow, N, K, tsm);
        ok = !__syncthreads_or(!w_ok);
    } else {
        const TreeView tv(tsm, N);
        ok = (N <= kMaskNodes && N <= (int)blockDim.x) ? build_walk_masked(prow, N, K, tv)
                                                        : build_walk(prow, N, K, tv);
    }
    int32_t* pl = plan + (size_t)b * stride;
    const int cnt = warp_kind ? 128 : 4 * N;
    if (ok)
        for (int i = tid; i < cnt; i += blockDim.x)
            pl[kPlanHeader + i] = tsm[i];
    if (tid == 0) {
        pl[0] = sig;
        pl[1] = ok ? 1 : 0;
        pl[2] = N;
        pl[3] = 0;
        if (!ok)
            report_status(status, GDN_ERR_BAD_TREE);
    }
}

}  // namespace
}  // namespace verify

cudaError_t launch_plan(const VerifyArgs& a, const PlanGeom& pg, int32_t* plan, cudaStream_t stream)
{
    const size_t smem = pg.warp_kind ? (size_t)kWarpTreeInts * 4
                                     : (size_t)(kTreeArrays + kMaskScratch) * a.n_nodes * 4;
    // The whole unified L1/shared array as shared memory: the split the
    // driver would pick for this small kernel stays in force for the verify
    // kernels after it, and with fewer of their CTAs resident the next
    // layer's could no longer start early (measured: ~4 us per layer).
    cudaError_t e = cudaFuncSetAttribute(verify::gdn_plan_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess)
        return e;
    if (smem > 48 * 1024) {
        e = cudaFuncSetAttribute(verify::gdn_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
    }
    // A plain launch: the verify launches that read the plan follow it with
    // an ordinary dependency (a programmatic one here was measured to slow
    // every layer of a captured 48-layer step by ~4 us).
    verify::gdn_plan_kernel<<<dim3(a.batch), dim3(verify::kPlanThreads), smem, stream>>>(
        a.parent, a.n_nodes, pg.slots, pg.warp_kind ? 1 : 0, pg.sig, plan, pg.stride, a.status);
    return cudaGetLastError();
}

}  // namespace gdn
