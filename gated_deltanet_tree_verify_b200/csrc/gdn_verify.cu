// gdn_verify.cu -- launch geometry and dispatch of the verify kernels (the
// kernels themselves are in gdn_verify.cuh).

#include <cstdint>

#include <cuda_runtime.h>

#include "gdn_internal.h"
#include "gdn_verify.cuh"

namespace gdn {
namespace verify {
extern template cudaError_t launch_dk<32>(const KParams&, const VerifyArgs&, const VerifyGeom&,
                                          cudaStream_t);
extern template cudaError_t launch_dk<64>(const KParams&, const VerifyArgs&, const VerifyGeom&,
                                          cudaStream_t);
extern template cudaError_t launch_dk<128>(const KParams&, const VerifyArgs&, const VerifyGeom&,
                                           cudaStream_t);
}  // namespace verify

namespace {
size_t align16(size_t x) { return (x + 15) & ~size_t(15); }
}  // namespace

using namespace verify;

VerifyGeom verify_geometry(const VerifyArgs& a)
{
    VerifyGeom g{};
    const bool chain = (a.flags & GDN_FLAG_CHAIN) != 0;
    const bool persist_last = (a.flags & GDN_FLAG_PERSIST_LAST) != 0;
    const int lr = a.d_k / kColsPerLane;
    const size_t es = a.qkv_dtype == GDN_BF16 ? 2 : 4;
    g.reload = !chain && a.state_dtype == GDN_F32 && !persist_last;
    if (chain || g.reload) {
        g.slots = 0;
    } else {
        // floor(log2 N) slots make recomputation impossible; fewer keep more
        // CTAs resident.  Draft trees of budget <= 31 need at most 2.
        int k = 0;
        while ((2 << k) <= a.n_nodes)
            ++k;
        const int cap = a.n_nodes <= 32 ? 2 : (a.n_nodes <= 96 ? 3 : 4);
        g.slots = k < 1 ? 1 : (k > cap ? cap : k);
    }
    // One row per lane when two would leave fewer than 8 warps per SM (148
    // SMs): more warps hide the per-node dependency chain of small batches.
    const long long warps_rl2 = (long long)a.batch * a.n_v_heads * a.d_v / (2 * 32 / lr);
    g.rows_per_lane = warps_rl2 < 8 * 148 ? 1 : 2;
    const int rpw = g.rows_per_lane * 32 / lr;
    // Staged kernel first, else the ring kernel (which adds a producer warp).
    for (int pass = 0; pass < 2; ++pass) {
        const bool staged = pass == 0;
        int warps = kMaxWarps;
        while (warps > 1 && a.d_v % (warps * rpw) != 0)
            --warps;
        const int rows = warps * rpw;
        if (a.d_v % rows != 0 || (rows * es) % 16 != 0)
            continue;
        const size_t raw_bytes = (size_t)(2 * a.d_k + rows) * es;
        const size_t rec_floats = (size_t)(2 * a.d_k + rows);
        const size_t slot_bytes = (size_t)g.slots * rows * a.d_k * 4;
        size_t off = 64;  // mbarriers
        size_t off_raw = 0, off_rec = 0, off_ab = 0, off_slots = 0;
        if (staged) {
            const size_t stage_raw = align16((size_t)a.n_nodes * raw_bytes);
            if (es == 2 && g.rows_per_lane == 1) {
                // raw bf16 records are read by the node loop itself
                off_raw = off_rec = off;
                off += stage_raw;
                off_slots = off;
                off += align16(slot_bytes);
            } else if (es == 2) {
                // raw rows are dead once widened: they share space with the stack
                off_raw = off_slots = off;
                off += stage_raw > slot_bytes ? stage_raw : align16(slot_bytes);
                off_rec = off;
                off += align16((size_t)a.n_nodes * rec_floats * 4);
            } else {
                off_raw = off_rec = off;  // f32 rows are the records
                off += stage_raw;
                off_slots = off;
                off += align16(slot_bytes);
            }
            off_ab = off;
            off += align16((size_t)3 * a.n_nodes * 4);  // a | beta | k.q per node
        } else {
            off_rec = off;
            off += (size_t)kRing * align16((kChunk * rec_floats + 3 * kChunk) * 4);
            off_slots = off;
            off += align16(slot_bytes);
        }
        // tree area: none for chains, the parent array for index order, the
        // register-built walk's 4 x 32 ints, else the shared-memory walk
        const size_t off_tree = off;
        const bool warp_tree = staged && !chain && !g.reload && a.n_nodes <= 32;
        if (chain)
            off += 0;
        else if (g.reload)
            off += align16((size_t)a.n_nodes * 4);
        else if (warp_tree)
            off += 4 * 32 * 4;
        else
            off += (size_t)(kTreeArrays + warps) * a.n_nodes * 4;
        if (staged && off > (size_t)kStagedMaxSmem)
            continue;
        g.staged = staged;
        g.warp_tree = warp_tree;
        g.warps = warps;
        g.rows = rows;
        g.tiles = a.d_v / rows;
        g.raw_bytes = (uint32_t)raw_bytes;
        g.rec_floats = (uint32_t)rec_floats;
        g.off_raw = (uint32_t)off_raw;
        g.off_rec = (uint32_t)off_rec;
        g.off_ab = (uint32_t)off_ab;
        g.off_slots = (uint32_t)off_slots;
        g.off_tree = (uint32_t)off_tree;
        g.smem = off;
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
    kp.reload = geom.reload ? 1 : 0;
    kp.early_tree = (a.flags & GDN_FLAG_EARLY_TREE) ? 1 : 0;
    kp.raw_bytes = geom.raw_bytes;
    kp.rec_floats = geom.rec_floats;
    kp.off_raw = geom.off_raw;
    kp.off_rec = geom.off_rec;
    kp.off_ab = geom.off_ab;
    kp.off_slots = geom.off_slots;
    kp.off_tree = geom.off_tree;
    switch (a.d_k) {
        case 32: return launch_dk<32>(kp, a, geom, stream);
        case 64: return launch_dk<64>(kp, a, geom, stream);
        case 128: return launch_dk<128>(kp, a, geom, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace gdn
