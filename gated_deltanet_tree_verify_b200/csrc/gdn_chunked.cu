// gdn_chunked.cu -- chains in chunks of 64 tokens on the Blackwell tensor
// cores (GDN_FLAG_CHUNKED: a prefill-style chain with last-only persistence).
//
// Within a chunk of T tokens starting from state S (d_v x d_k), with
// a_t = exp(g_t), Gamma_t = a_0 ... a_t and R[t][i] = a_{i+1} ... a_t (the
// decay from token i to token t), the recurrence
//
//     S_t = a_t S_{t-1} + beta_t (v_t - a_t S_{t-1} k_t) k_t^T,  o_t = scale S_t q_t
//
// unrolls to S_t = Gamma_t S + sum_{i <= t} R[t][i] u_i k_i^T, where the
// pseudo-values u_i = beta_i (v_i - a_i S_{i-1} k_i) solve the unit lower
// triangular system (I + L) U = diag(beta) (V - diag(Gamma) K S^T) with
// L = diag(beta) (K K^T o R) strictly below the diagonal (the delta rule's
// chunked "WY" form; the Gated Delta Networks paper by Yang, Kautz and
// Hatamizadeh derives it).  The inverse does not depend on the state, so
// with Ab = (I + L)^-1 diag(beta) and M = Q K^T o R (on and below the
// diagonal), transposed so that the state's d_v rows run down the tensor
// cores' M dimension:
//
//     X^T = S K^T,  Y^T = S Q^T                       [d_v x T]  (one product, N = 2T)
//     U^T = (V^T - X^T diag(Gamma)) Ab^T              [d_v x T]
//     O^T = scale (Y^T diag(Gamma) + U^T M^T)          [d_v x T]
//     S  <- Gamma_{T-1} S + (U^T diag(r)) K,  r_i = R[T-1][i]
//
// Only these four products (and elementwise work between them) lie on the
// chain from one chunk to the next; the decays, K K^T and Q K^T, L, M and
// the triangular inverse for chunk c + 1 are computed by other warps while
// chunk c runs.
//
// Every product is a tcgen05.mma (kind::f16, bf16 operands, f32 accumulation
// in tensor memory), issued by one thread.  Operands that are not exact in
// bf16 (the state, U, Ab, M) are split into bf16 parts, x = x1 + x2 + x3
// (x2 = bf16(x - x1), x3 = bf16(x - x1 - x2): 24 bits), and each product is
// formed from the part products down to ~2^-24 relative (S and U parts
// against the exact bf16 K and Q; 6 of the 9 part products for U^T Ab^T;
// 3 of 4 two-part products for the output-only U^T M^T), which keeps the
// chunked form at f32 accuracy.  Layout: the A operands (the state, P^T,
// U^T) live in tensor memory, written by the thread that owns the row
// (bf16 pairs per 32-bit column, the even element in the low half); the B
// operands (K, Q, K^T, Ab, M) in shared memory in the canonical K-major
// layout without swizzle (8 x 16-byte core matrices).  The state itself is
// the f32 accumulator of the update, in tensor memory for the whole chain.
//
// Rounding differs from the token-by-token path (different summation
// order), so this is an opt-in mode, not the chain fast path.
//
// One CTA per (sequence, v-head, 128 rows of d_v), 9 warps: warps 0-3 own
// the state rows (one row per thread: the elementwise steps between the
// products), warps 4-7 stage inputs and prepare each chunk's S-independent
// operands one chunk ahead, warp 8 issues the MMAs.  Hand-offs are
// mbarriers; every wait is bounded and a timeout is reported as a status.

#include <atomic>
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {
namespace chunked {
namespace {

constexpr int T = 64;           // tokens per chunk
constexpr int DK = 128;         // d_k
constexpr int TM = 128;         // state rows (d_v) per CTA: the MMAs' M
constexpr int kThreads = 288;   // warps 0-3 rows, 4-7 preparation, 8 MMA issue
constexpr int kPrep0 = 128;     // first preparation thread

// Tensor-memory columns (128 lanes x 512 columns of 32 bits, all of it).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;     // state S, f32 [d_v x d_k]
constexpr uint32_t kColAS = 128;  // S in 3 bf16 parts, 64 columns each (A of X^T | Y^T)
constexpr uint32_t kColAP = 128;  //   after that product: P^T in 3 parts of 32 columns
constexpr uint32_t kColU = 224;   //   and U^T, f32 [d_v x T]
constexpr uint32_t kColAUr = 128; //   after that: U^T diag(r) in 3 parts (A of the update)
constexpr uint32_t kColAU = 224;  //   and U^T in 2 parts (A of U^T M^T)
constexpr uint32_t kColX = 320;   // X^T, f32 [d_v x T]; later U^T M^T
constexpr uint32_t kColY = 384;   // Y^T, f32 [d_v x T]
constexpr uint32_t kColKQ = 448;  // [K; Q] K^T, f32 [2T x T] (lanes = K rows, then Q rows)

// Shared memory (bytes).  B operands in the canonical K-major layout: element
// (n, k) of an N-row operand at (k / 8) * N * 16 + (n / 8) * 128 + (n % 8) * 16
// + (k % 8) * 2.
constexpr int kKQBytes = 2 * T * DK * 2;  // [K; Q] of one chunk, 128 rows
constexpr int kVBytes = T * TM * 2;       // V of one chunk, [t][row]
constexpr int kTTBytes = T * T * 2;       // one bf16 part of a 64 x 64 operand
constexpr int kKTBytes = DK * T * 2;      // K^T, 128 rows x 64 tokens
constexpr int LST = T + 1;                // f32 row stride of L and M
constexpr int AST = T + 4;                // f32 row stride of the inverse (16-byte rows)
constexpr int kOffKQ = 0;                          // [2]
constexpr int kOffV = kOffKQ + 2 * kKQBytes;       // [2]
constexpr int kOffAb = kOffV + 2 * kVBytes;        // [3 parts]
constexpr int kOffM = kOffAb + 3 * kTTBytes;       // [2 parts]
constexpr int kOffKT = kOffM + 2 * kTTBytes;
constexpr int kOffL = kOffKT + kKTBytes;           // L, f32 [T][LST]
constexpr int kOffMf = kOffL + T * LST * 4;        // M, f32 [T][LST]
constexpr int kOffAi = kOffMf + T * LST * 4;       // (I + L)^-1, f32 [T][AST]
constexpr int kOffGB = kOffAi + T * AST * 4;       // [2][g | beta], f32
constexpr int kOffDec = kOffGB + 2 * 2 * T * 4;    // [3][Gamma | r], f32
constexpr int kOffA = kOffDec + 3 * 2 * T * 4;     // a = exp(g), f32 [T]
constexpr int kOffBar = kOffA + T * 4;             // mbarriers, tmem base, abort flag
constexpr int kSmem = kOffBar + 256;

// mbarriers (index into the array at kOffBar)
enum Bar {
    kKqFull0 = 0,  // chunk inputs staged in buffer 0 / 1 (128 preparation threads)
    kKqFull1 = 1,
    kKqMma = 2,    // [K; Q] K^T done (MMA commit)
    kKqFree = 3,   // [K; Q] K^T read out (128)
    kDec0 = 4,     // decays of a chunk written, slots 0..2 (128)
    kAsReady = 7,  // state parts written, previous outputs read (128 row threads)
    kXyDone = 8,   // X^T | Y^T done (commit)
    kApReady = 9,  // P^T parts written (128)
    kAbReady = 10, // Ab parts written (128)
    kUDone = 11,   // U^T done (commit)
    kAuReady = 12, // U^T parts written (128)
    kMktReady = 13,// M parts and K^T written (128)
    kCdDone = 14,  // update and U^T M^T done (commit)
    kFin = 15,     // all MMAs retired (commit)
    kNumBars = 16
};

struct Params {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    const float* g;
    const float* beta;
    const float* state_in;
    float* out;
    void* node_states;
    int32_t* status;
    int N, Hk, Hv, dv, G;
    float scale;
    int state_f16;
};

// ---- tcgen05 ----------------------------------------------------------------

// Shared-memory descriptor of a K-major operand without swizzle: start
// address, distance between 8-column pieces along K (lbo), between 8-row
// groups (128 bytes), descriptor version 1.
__device__ __forceinline__ uint64_t kdesc(uint32_t addr, uint32_t lbo)
{
    return (uint64_t)((addr >> 4) & 0x3fff) | ((uint64_t)((lbo >> 4) & 0x3fff) << 16) |
           ((uint64_t)(128 >> 4) << 32) | ((uint64_t)1 << 46);
}

// Instruction descriptor: f32 accumulator, bf16 A and B, both K-major, M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(int n)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((128u >> 4) << 24);
}

// D (tensor memory) (+)= A (shared memory) B^T
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

// D (tensor memory) (+)= A (tensor memory) B^T
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

// The barrier's phase completes once every MMA issued so far has retired.
__device__ __forceinline__ void mma_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---- bf16 splits --------------------------------------------------------------

__device__ __forceinline__ uint32_t pack_bf2(float a, float b)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// (a, b) = p1 + p2 + p3 in packed bf16 pairs (each remainder is exact in f32).
__device__ __forceinline__ void split3(float a, float b, uint32_t& p1, uint32_t& p2, uint32_t& p3)
{
    p1 = pack_bf2(a, b);
    float2 f = bf16x2_to_float2(p1);
    a = __fsub_rn(a, f.x);
    b = __fsub_rn(b, f.y);
    p2 = pack_bf2(a, b);
    f = bf16x2_to_float2(p2);
    p3 = pack_bf2(__fsub_rn(a, f.x), __fsub_rn(b, f.y));
}

__device__ __forceinline__ void split2(float a, float b, uint32_t& p1, uint32_t& p2)
{
    p1 = pack_bf2(a, b);
    const float2 f = bf16x2_to_float2(p1);
    p2 = pack_bf2(__fsub_rn(a, f.x), __fsub_rn(b, f.y));
}

// ---- synchronisation -------------------------------------------------------------

struct Sync {
    uint64_t* bar;
    volatile int* abort;
    int32_t* status;

    // Bounded wait for a phase; false once this or any other thread gave up.
    __device__ __forceinline__ bool wait(int b, uint32_t parity) const
    {
        if (mbar_try_wait(bar + b, parity))
            return true;
        const long long t0 = clock64();
        while (!mbar_try_wait_suspend(bar + b, parity, 20000u)) {
            if (*abort)
                return false;
            if (clock64() - t0 > (1ll << 31)) {
                *abort = 1;
                report_status(status, kStatusTimeout);
                return false;
            }
        }
        return true;
    }
    __device__ __forceinline__ void arrive(int b) const { mbar_arrive(bar + b); }
};

// Named barrier over the 128 preparation threads.
__device__ __forceinline__ void prep_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// The same barrier, returning whether ok holds for all 128 of them (so that
// they leave together and none is left waiting at a later barrier).
__device__ __forceinline__ bool prep_all(bool ok)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(ok ? 1u : 0u)
        : "memory");
    return r != 0;
}

// Whether ok holds for the whole warp (tensor-memory accesses are warp-wide).
__device__ __forceinline__ bool warp_all(bool ok) { return __all_sync(0xffffffffu, ok); }

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

// ---- preparation warps ---------------------------------------------------------------

// Stage chunk c's k and q rows (canonical layout, K rows 0..63 then Q rows),
// the CTA's 128-row slice of v ([t][row]), g and beta.  Tokens past the
// chain's end and rows past d_v are zero (k = q = v = 0, beta = 0, g = 0:
// they leave the state unchanged; their outputs are not written).
__device__ void stage_chunk(const Params& p, unsigned char* smem, int buf, int c, int b, int h, int hk, int row0,
                            int ptid)
{
    const int t0 = c * T;
    const uint32_t kq = smem_addr(smem + kOffKQ + buf * kKQBytes);
    const uint32_t vb = smem_addr(smem + kOffV + buf * kVBytes);
    for (int i = ptid; i < 2 * T * (DK / 8); i += 128) {
        const int which = i / (T * (DK / 8));
        const int t = (i / (DK / 8)) % T, pc = i % (DK / 8);
        const int n = which * T + t;
        const uint32_t dst = kq + pc * (2 * T * 16) + (n >> 3) * 128 + (n & 7) * 16;
        if (t0 + t < p.N) {
            const size_t node = (size_t)b * p.N + t0 + t;
            cp_async16(dst, (which == 0 ? p.k : p.q) + (node * p.Hk + hk) * DK + pc * 8);
        } else {
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0u) : "memory");
        }
    }
    for (int i = ptid; i < T * (TM / 8); i += 128) {
        const int t = i / (TM / 8), pc = i % (TM / 8);
        const uint32_t dst = vb + t * (TM * 2) + pc * 16;
        if (t0 + t < p.N && row0 + pc * 8 < p.dv) {
            const size_t node = (size_t)b * p.N + t0 + t;
            cp_async16(dst, p.v + (node * p.Hv + h) * p.dv + row0 + pc * 8);
        } else {
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0u) : "memory");
        }
    }
    {
        const int t = ptid & (T - 1), which = ptid >> 6;  // 0: g, 1: beta
        const uint32_t dst = smem_addr(smem + kOffGB) + (buf * 2 * T + which * T + t) * 4;
        if (t0 + t < p.N) {
            const size_t gi = ((size_t)b * p.N + t0 + t) * p.Hv + h;
            cp_async4(dst, (which == 0 ? p.g : p.beta) + gi);
        } else {
            asm volatile("st.shared.u32 [%0], %1;" ::"r"(dst), "r"(0u) : "memory");
        }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// (I + L)^-1 for the unit lower triangular I + L (L strictly lower, f32
// [T][LST]) into Ai (f32 [T][AST], whose entries above the diagonal stay 0):
// the four 16 x 16 diagonal blocks by forward substitution, one column per
// thread; then block rows 1..3, X = -L_(I, <I) Ai_(<I, <I) and
// Ai_(I, <I) = Ai_(I,I) X, 8 columns of one row per thread.
__device__ void invert_unit_lower(const float* L, float* Ai, int ptid)
{
    if (ptid < T) {
        const int blk = ptid >> 4, j = ptid & 15;
        const float* Lb = L + (16 * blk) * LST + 16 * blk;
        float d[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float acc = 0.f;
#pragma unroll
            for (int k = 0; k < i; ++k)
                acc = __fmaf_rn(Lb[i * LST + k], k >= j ? d[k] : 0.f, acc);
            d[i] = i < j ? 0.f : (i == j ? 1.f : -acc);
            Ai[(16 * blk + i) * AST + 16 * blk + j] = d[i];
        }
    }
    prep_sync();
#pragma unroll 1
    for (int I = 1; I < 4; ++I) {
        const int R0 = 16 * I;
        const int i = ptid & 15, c0 = 8 * (ptid >> 4);  // row of the block row, first of 8 columns
        const bool act = c0 < R0;
        float x[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (act) {
            const float* Lr = L + (R0 + i) * LST;
            for (int k = c0; k < R0; ++k) {  // Ai[k][c] = 0 for k < c
                const float l = Lr[k];
                const float4 a0 = *reinterpret_cast<const float4*>(Ai + k * AST + c0);
                const float4 a1 = *reinterpret_cast<const float4*>(Ai + k * AST + c0 + 4);
                x[0] = __fmaf_rn(-l, a0.x, x[0]);
                x[1] = __fmaf_rn(-l, a0.y, x[1]);
                x[2] = __fmaf_rn(-l, a0.z, x[2]);
                x[3] = __fmaf_rn(-l, a0.w, x[3]);
                x[4] = __fmaf_rn(-l, a1.x, x[4]);
                x[5] = __fmaf_rn(-l, a1.y, x[5]);
                x[6] = __fmaf_rn(-l, a1.z, x[6]);
                x[7] = __fmaf_rn(-l, a1.w, x[7]);
            }
            float* dst = Ai + (R0 + i) * AST + c0;  // X in the block's own place
            *reinterpret_cast<float4*>(dst) = make_float4(x[0], x[1], x[2], x[3]);
            *reinterpret_cast<float4*>(dst + 4) = make_float4(x[4], x[5], x[6], x[7]);
        }
        prep_sync();
        if (act) {
            float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            const float* Dr = Ai + (R0 + i) * AST + R0;  // the block's inverse, row i
            for (int i2 = 0; i2 <= i; ++i2) {
                const float dd = Dr[i2];
                const float4 a0 = *reinterpret_cast<const float4*>(Ai + (R0 + i2) * AST + c0);
                const float4 a1 = *reinterpret_cast<const float4*>(Ai + (R0 + i2) * AST + c0 + 4);
                y[0] = __fmaf_rn(dd, a0.x, y[0]);
                y[1] = __fmaf_rn(dd, a0.y, y[1]);
                y[2] = __fmaf_rn(dd, a0.z, y[2]);
                y[3] = __fmaf_rn(dd, a0.w, y[3]);
                y[4] = __fmaf_rn(dd, a1.x, y[4]);
                y[5] = __fmaf_rn(dd, a1.y, y[5]);
                y[6] = __fmaf_rn(dd, a1.z, y[6]);
                y[7] = __fmaf_rn(dd, a1.w, y[7]);
            }
            x[0] = y[0], x[1] = y[1], x[2] = y[2], x[3] = y[3];
            x[4] = y[4], x[5] = y[5], x[6] = y[6], x[7] = y[7];
        }
        prep_sync();
        if (act) {
            float* dst = Ai + (R0 + i) * AST + c0;
            *reinterpret_cast<float4*>(dst) = make_float4(x[0], x[1], x[2], x[3]);
            *reinterpret_cast<float4*>(dst + 4) = make_float4(x[4], x[5], x[6], x[7]);
        }
        prep_sync();
    }
}

__device__ void prep_role(const Params& p, unsigned char* smem, const Sync& sy, uint32_t tbase, int b, int h,
                          int hk, int row0, int n_chunks)
{
    const int ptid = threadIdx.x - kPrep0;
    const int pw = ptid >> 5;                  // lane quarter of tensor memory
    const bool qrow = ptid >= T;               // reads a Q row of [K; Q] K^T, else a K row
    const int t = ptid & (T - 1);              // that row's token
    float* L = reinterpret_cast<float*>(smem + kOffL);
    float* Mf = reinterpret_cast<float*>(smem + kOffMf);
    float* Ai = reinterpret_cast<float*>(smem + kOffAi);
    float* av = reinterpret_cast<float*>(smem + kOffA);

    for (int i = ptid; i < T * AST; i += 128)
        Ai[i] = 0.f;
    stage_chunk(p, smem, 0, 0, b, h, hk, row0, ptid);
    if (n_chunks > 1)
        stage_chunk(p, smem, 1, 1, b, h, hk, row0, ptid);

    for (int c = 0; c < n_chunks; ++c) {
        const int buf = c & 1, slot = c % 3;
        const float* gb = reinterpret_cast<const float*>(smem + kOffGB) + buf * 2 * T;
        float* Gam = reinterpret_cast<float*>(smem + kOffDec) + slot * 2 * T;
        float* rv = Gam + T;
        // 1. this chunk's inputs have landed
        if (c == 0 && n_chunks > 1)
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        else
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        fence_proxy_async();
        sy.arrive(kKqFull0 + buf);
        prep_sync();
        if (ptid < T)
            av[ptid] = expf(gb[ptid]);
        prep_sync();
        // 2. read this thread's row of [K; Q] K^T; the row's decays
        //    R[t][i] = a_{i+1} ... a_t come from a running product over i
        //    from t down to 0, which ends at Gamma_t
        if (!prep_all(sy.wait(kKqMma, c & 1)))
            return;
        tmem_fence_after_sync();
        uint32_t d[64];
        {
            uint32_t (&d0)[32] = *reinterpret_cast<uint32_t(*)[32]>(d);
            uint32_t (&d1)[32] = *reinterpret_cast<uint32_t(*)[32]>(d + 32);
            const uint32_t ta = tbase + ((uint32_t)(32 * pw) << 16) + kColKQ;
            tmem_ld32(ta, d0);
            tmem_ld32(ta + 32, d1);
        }
        tmem_fence_before_sync();
        sy.arrive(kKqFree);
        {
            const float bt = gb[T + t];
            float* row = (qrow ? Mf : L) + t * LST;
            float run = 1.f;
#pragma unroll
            for (int i = T - 1; i >= 0; --i) {
                const float kk = __uint_as_float(d[i]);
                float val;
                if (qrow)
                    val = i <= t ? __fmul_rn(kk, run) : 0.f;
                else
                    val = i < t ? __fmul_rn(bt, __fmul_rn(kk, run)) : 0.f;
                row[i] = val;
                if (!qrow && t == T - 1)
                    rv[i] = run;
                if (i <= t)
                    run = __fmul_rn(run, av[i]);
            }
            if (!qrow)
                Gam[t] = run;
        }
        sy.arrive(kDec0 + slot);
        prep_sync();
        // 3. Ai = (I + L)^-1
        invert_unit_lower(L, Ai, ptid);
        // 4. Ab = Ai diag(beta) in 3 bf16 parts, once the previous chunk's
        //    U^T product is done with them; then stage chunk c + 1 into the
        //    buffer the previous chunk has left
        if (c > 0) {
            if (!prep_all(sy.wait(kUDone, (c - 1) & 1)))
                return;
            if (c + 1 < n_chunks)
                stage_chunk(p, smem, (c + 1) & 1, c + 1, b, h, hk, row0, ptid);
        }
        for (int it = ptid; it < T * (T / 8); it += 128) {
            const int tt = it & (T - 1), pc = it >> 6;
            const float4 a0 = *reinterpret_cast<const float4*>(Ai + tt * AST + 8 * pc);
            const float4 a1 = *reinterpret_cast<const float4*>(Ai + tt * AST + 8 * pc + 4);
            const float4 b0 = *reinterpret_cast<const float4*>(gb + T + 8 * pc);
            const float4 b1 = *reinterpret_cast<const float4*>(gb + T + 8 * pc + 4);
            uint32_t p1[4], p2[4], p3[4];
            split3(__fmul_rn(a0.x, b0.x), __fmul_rn(a0.y, b0.y), p1[0], p2[0], p3[0]);
            split3(__fmul_rn(a0.z, b0.z), __fmul_rn(a0.w, b0.w), p1[1], p2[1], p3[1]);
            split3(__fmul_rn(a1.x, b1.x), __fmul_rn(a1.y, b1.y), p1[2], p2[2], p3[2]);
            split3(__fmul_rn(a1.z, b1.z), __fmul_rn(a1.w, b1.w), p1[3], p2[3], p3[3]);
            const uint32_t off = pc * (T * 16) + (tt >> 3) * 128 + (tt & 7) * 16;
            const uint32_t base = smem_addr(smem + kOffAb) + off;
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(base), "r"(p1[0]), "r"(p1[1]),
                         "r"(p1[2]), "r"(p1[3])
                         : "memory");
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(base + kTTBytes), "r"(p2[0]),
                         "r"(p2[1]), "r"(p2[2]), "r"(p2[3])
                         : "memory");
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(base + 2 * kTTBytes), "r"(p3[0]),
                         "r"(p3[1]), "r"(p3[2]), "r"(p3[3])
                         : "memory");
        }
        fence_proxy_async();
        sy.arrive(kAbReady);
        // 5. M in 2 bf16 parts and K^T, once the previous chunk's update and
        //    U^T M^T products are done with them
        if (c > 0 && !prep_all(sy.wait(kCdDone, (c - 1) & 1)))
            return;
        for (int it = ptid; it < T * (T / 8); it += 128) {
            const int tt = it & (T - 1), pc = it >> 6;
            const float* mr = Mf + tt * LST + 8 * pc;
            uint32_t p1[4], p2[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
                split2(mr[2 * e], mr[2 * e + 1], p1[e], p2[e]);
            const uint32_t base = smem_addr(smem + kOffM) + pc * (T * 16) + (tt >> 3) * 128 + (tt & 7) * 16;
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(base), "r"(p1[0]), "r"(p1[1]),
                         "r"(p1[2]), "r"(p1[3])
                         : "memory");
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(base + kTTBytes), "r"(p2[0]),
                         "r"(p2[1]), "r"(p2[2]), "r"(p2[3])
                         : "memory");
        }
        {
            // K^T: the 8 x 8 core matrix (token group tg, column group jg) of
            // K, transposed into core matrix (jg, tg) of K^T; 4 per ldmatrix.
            const uint32_t kq = smem_addr(smem + kOffKQ + buf * kKQBytes);
            const uint32_t kt = smem_addr(smem + kOffKT);
            const int lane = ptid & 31, mi = lane >> 3, r = lane & 7;
#pragma unroll
            for (int it = 0; it < 8; ++it) {
                const int blk = pw * 32 + it * 4 + mi;  // 128 core matrices
                const int tg = blk & 7, jg = blk >> 3;
                const uint32_t src = kq + jg * (2 * T * 16) + tg * 128 + r * 16;
                const uint32_t dst = kt + tg * (DK * 16) + jg * 128 + r * 16;
                uint32_t x0, x1, x2, x3;
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                             : "=r"(x0), "=r"(x1), "=r"(x2), "=r"(x3)
                             : "r"(src)
                             : "memory");
                asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(dst),
                             "r"(x0), "r"(x1), "r"(x2), "r"(x3)
                             : "memory");
            }
        }
        fence_proxy_async();
        sy.arrive(kMktReady);
    }
}

// ---- MMA warp -------------------------------------------------------------------------------

__device__ void mma_role(unsigned char* smem, const Sync& sy, uint32_t tbase, int n_chunks)
{
    const uint32_t kq0 = smem_addr(smem + kOffKQ);
    const uint32_t ab = smem_addr(smem + kOffAb);
    const uint32_t mm = smem_addr(smem + kOffM);
    const uint32_t kt = smem_addr(smem + kOffKT);
    constexpr uint32_t kKQLbo = 2 * T * 16, kTTLbo = T * 16, kKTLbo = DK * 16;

    // [K; Q] K^T of chunk cc: A = [K; Q] (128 rows), B = K (the first 64)
    auto kq_product = [&](int cc) {
        const uint32_t base = kq0 + (cc & 1) * kKQBytes;
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
            const uint64_t dsc = kdesc(base + ks * 2 * kKQLbo, kKQLbo);
            mma_ss(tbase + kColKQ, dsc, dsc, idesc_bf16(T), ks > 0 ? 1u : 0u);
        }
        mma_commit(sy.bar + kKqMma);
    };

    if (!sy.wait(kKqFull0, 0))
        return;
    tmem_fence_after_sync();
    kq_product(0);
    for (int c = 0; c < n_chunks; ++c) {
        const uint32_t kq = kq0 + (c & 1) * kKQBytes;
        // X^T | Y^T = S [K; Q]^T, S in 3 parts
        if (!sy.wait(kAsReady, c & 1))
            return;
        tmem_fence_after_sync();
#pragma unroll
        for (int part = 0; part < 3; ++part)
#pragma unroll
            for (int ks = 0; ks < DK / 16; ++ks)
                mma_ts(tbase + kColX, tbase + kColAS + 64 * part + 8 * ks, kdesc(kq + ks * 2 * kKQLbo, kKQLbo),
                       idesc_bf16(2 * T), (part | ks) != 0 ? 1u : 0u);
        mma_commit(sy.bar + kXyDone);
        // the next chunk's [K; Q] K^T
        if (c + 1 < n_chunks) {
            if (!sy.wait(kKqFull0 + ((c + 1) & 1), ((c + 1) >> 1) & 1) || !sy.wait(kKqFree, c & 1))
                return;
            tmem_fence_after_sync();
            kq_product(c + 1);
        }
        // U^T = P^T Ab^T: part products (P, Ab) with at most 2^-16 weight
        if (!sy.wait(kApReady, c & 1) || !sy.wait(kAbReady, c & 1))
            return;
        tmem_fence_after_sync();
        {
            const int pp[6] = {0, 0, 1, 0, 1, 2}, pa[6] = {0, 1, 0, 2, 1, 0};
#pragma unroll
            for (int q = 0; q < 6; ++q)
#pragma unroll
                for (int ks = 0; ks < T / 16; ++ks)
                    mma_ts(tbase + kColU, tbase + kColAP + 32 * pp[q] + 8 * ks,
                           kdesc(ab + pa[q] * kTTBytes + ks * 2 * kTTLbo, kTTLbo), idesc_bf16(T),
                           (q | ks) != 0 ? 1u : 0u);
        }
        mma_commit(sy.bar + kUDone);
        // S += (U^T diag(r)) K and U^T M^T
        if (!sy.wait(kAuReady, c & 1) || !sy.wait(kMktReady, c & 1))
            return;
        tmem_fence_after_sync();
#pragma unroll
        for (int part = 0; part < 3; ++part)
#pragma unroll
            for (int ks = 0; ks < T / 16; ++ks)
                mma_ts(tbase + kColS, tbase + kColAUr + 32 * part + 8 * ks, kdesc(kt + ks * 2 * kKTLbo, kKTLbo),
                       idesc_bf16(DK), 1u);
        {
            const int pu[3] = {0, 0, 1}, pm[3] = {0, 1, 0};
#pragma unroll
            for (int q = 0; q < 3; ++q)
#pragma unroll
                for (int ks = 0; ks < T / 16; ++ks)
                    mma_ts(tbase + kColX, tbase + kColAU + 32 * pu[q] + 8 * ks,
                           kdesc(mm + pm[q] * kTTBytes + ks * 2 * kTTLbo, kTTLbo), idesc_bf16(T),
                           (q | ks) != 0 ? 1u : 0u);
        }
        mma_commit(sy.bar + kCdDone);
    }
}

// ---- row warps ----------------------------------------------------------------------------------

// This thread's row of the previous chunk's outputs: scale (Gamma_t Y^T + U^T M^T).
__device__ __forceinline__ void write_outputs(const Params& p, uint32_t trow, const float* Gam, int b, int h,
                                              int row, int t0)
{
    const int Tc = min(T, p.N - t0);
#pragma unroll
    for (int hs = 0; hs < 2; ++hs) {
        uint32_t y[32], o[32];
        tmem_ld32(trow + kColY + 32 * hs, y);
        tmem_ld32(trow + kColX + 32 * hs, o);
        if (row < p.dv) {
            float* dst = p.out + ((size_t)b * p.N + t0) * p.Hv * p.dv + (size_t)h * p.dv + row;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int tt = 32 * hs + i;
                if (tt < Tc)
                    dst[(size_t)tt * p.Hv * p.dv] =
                        __fmul_rn(p.scale, __fmaf_rn(Gam[tt], __uint_as_float(y[i]), __uint_as_float(o[i])));
            }
        }
    }
}

__device__ void row_role(const Params& p, unsigned char* smem, const Sync& sy, uint32_t tbase, int b, int h,
                         int row0, int n_chunks)
{
    const int tid = threadIdx.x, warp = tid >> 5;
    const int m = tid;              // state row within the tile (lane quarter = warp)
    const int row = row0 + m;       // row of d_v
    const uint32_t trow = tbase + ((uint32_t)(32 * warp) << 16);
    const float* decs = reinterpret_cast<const float*>(smem + kOffDec);

    for (int c = 0; c < n_chunks; ++c) {
        const int slot = c % 3;
        const float* Gam = decs + slot * 2 * T;
        const float* rv = Gam + T;
        if (!warp_all(sy.wait(kDec0 + slot, (c / 3) & 1)))
            return;
        const float gT = Gam[T - 1];
        // 0. the previous chunk's outputs; S into 3 bf16 parts (A of X^T | Y^T),
        //    and Gamma_{T-1} S back as the update's accumulator
        if (c > 0) {
            if (!warp_all(sy.wait(kCdDone, (c - 1) & 1)))
                return;
            tmem_fence_after_sync();
            write_outputs(p, trow, decs + ((c - 1) % 3) * 2 * T, b, h, row, (c - 1) * T);
        }
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            uint32_t x[32];
            if (c == 0) {
                if (row < p.dv) {
                    const float4* src = reinterpret_cast<const float4*>(
                        p.state_in + (((size_t)b * p.Hv + h) * p.dv + row) * DK + 32 * s);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float4 f = __ldg(src + e);
                        x[4 * e] = __float_as_uint(f.x);
                        x[4 * e + 1] = __float_as_uint(f.y);
                        x[4 * e + 2] = __float_as_uint(f.z);
                        x[4 * e + 3] = __float_as_uint(f.w);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        x[e] = 0u;
                }
            } else {
                tmem_ld32(trow + kColS + 32 * s, x);
            }
            uint32_t p1[16], p2[16], p3[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
                split3(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1]), p1[e], p2[e], p3[e]);
            tmem_st16(trow + kColAS + 16 * s, p1);
            tmem_st16(trow + kColAS + 64 + 16 * s, p2);
            tmem_st16(trow + kColAS + 128 + 16 * s, p3);
#pragma unroll
            for (int e = 0; e < 32; ++e)
                x[e] = __float_as_uint(__fmul_rn(gT, __uint_as_float(x[e])));
            tmem_st32(trow + kColS + 32 * s, x);
        }
        tmem_wait_st();
        tmem_fence_before_sync();
        sy.arrive(kAsReady);

        // 1. P^T = V^T - X^T diag(Gamma) into 3 bf16 parts (A of U^T)
        if (!warp_all(sy.wait(kXyDone, c & 1) && sy.wait(kKqFull0 + (c & 1), (c >> 1) & 1)))
            return;
        tmem_fence_after_sync();
        {
            const unsigned short* V =
                reinterpret_cast<const unsigned short*>(smem + kOffV + (c & 1) * kVBytes) + m;
#pragma unroll
            for (int hs = 0; hs < 2; ++hs) {
                uint32_t x[32];
                tmem_ld32(trow + kColX + 32 * hs, x);
                uint32_t p1[16], p2[16], p3[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int tt = 32 * hs + 2 * e;
                    const float v0 = __uint_as_float((uint32_t)V[tt * TM] << 16);
                    const float v1 = __uint_as_float((uint32_t)V[(tt + 1) * TM] << 16);
                    split3(__fsub_rn(v0, __fmul_rn(Gam[tt], __uint_as_float(x[2 * e]))),
                           __fsub_rn(v1, __fmul_rn(Gam[tt + 1], __uint_as_float(x[2 * e + 1]))), p1[e], p2[e],
                           p3[e]);
                }
                tmem_st16(trow + kColAP + 16 * hs, p1);
                tmem_st16(trow + kColAP + 32 + 16 * hs, p2);
                tmem_st16(trow + kColAP + 64 + 16 * hs, p3);
            }
        }
        tmem_wait_st();
        tmem_fence_before_sync();
        sy.arrive(kApReady);

        // 2. U^T diag(r) in 3 parts (A of the update), U^T in 2 (A of U^T M^T)
        if (!warp_all(sy.wait(kUDone, c & 1)))
            return;
        tmem_fence_after_sync();
        {
            uint32_t u[64];
            {
                uint32_t (&u0)[32] = *reinterpret_cast<uint32_t(*)[32]>(u);
                uint32_t (&u1)[32] = *reinterpret_cast<uint32_t(*)[32]>(u + 32);
                tmem_ld32(trow + kColU, u0);
                tmem_ld32(trow + kColU + 32, u1);
            }
#pragma unroll
            for (int hs = 0; hs < 2; ++hs) {
                uint32_t p1[16], p2[16], p3[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int tt = 32 * hs + 2 * e;
                    split3(__fmul_rn(rv[tt], __uint_as_float(u[tt])), __fmul_rn(rv[tt + 1], __uint_as_float(u[tt + 1])),
                           p1[e], p2[e], p3[e]);
                }
                tmem_st16(trow + kColAUr + 16 * hs, p1);
                tmem_st16(trow + kColAUr + 32 + 16 * hs, p2);
                tmem_st16(trow + kColAUr + 64 + 16 * hs, p3);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int tt = 32 * hs + 2 * e;
                    split2(__uint_as_float(u[tt]), __uint_as_float(u[tt + 1]), p1[e], p2[e]);
                }
                tmem_st16(trow + kColAU + 16 * hs, p1);
                tmem_st16(trow + kColAU + 32 + 16 * hs, p2);
            }
        }
        tmem_wait_st();
        tmem_fence_before_sync();
        sy.arrive(kAuReady);
    }

    // the last chunk's outputs and the last state -> node_states[b][0][h][row][:]
    if (!warp_all(sy.wait(kCdDone, (n_chunks - 1) & 1)))
        return;
    tmem_fence_after_sync();
    write_outputs(p, trow, decs + ((n_chunks - 1) % 3) * 2 * T, b, h, row, (n_chunks - 1) * T);
    const size_t base = (((size_t)b * p.Hv + h) * p.dv + row) * DK;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        uint32_t x[32];
        tmem_ld32(trow + kColS + 32 * s, x);
        if (row >= p.dv)
            continue;
        if (p.state_f16) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__half*>(p.node_states) + base + 32 * s);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                uint32_t w[4];
#pragma unroll
                for (int f = 0; f < 4; ++f) {
                    const __half2 hh = __floats2half2_rn(__uint_as_float(x[8 * e + 2 * f]),
                                                         __uint_as_float(x[8 * e + 2 * f + 1]));
                    w[f] = *reinterpret_cast<const uint32_t*>(&hh);
                }
                dst[e] = make_uint4(w[0], w[1], w[2], w[3]);
            }
        } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.node_states) + base + 32 * s);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                dst[e] = make_float4(__uint_as_float(x[4 * e]), __uint_as_float(x[4 * e + 1]),
                                     __uint_as_float(x[4 * e + 2]), __uint_as_float(x[4 * e + 3]));
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1) gdn_chain_chunked(const Params p)
{
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + kOffBar + kNumBars * 8);
    int* abort_flag = reinterpret_cast<int*>(smem + kOffBar + kNumBars * 8 + 4);
    const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int hk = h / p.G;
    const int row0 = tile * TM;
    const int warp = threadIdx.x >> 5;
    const int n_chunks = (p.N + T - 1) / T;

    // the preceding kernel (and its tensor memory) is done before this CTA
    // allocates all 512 columns
    pdl_wait_then_release();
    if (threadIdx.x == 0) {
        const uint32_t counts[kNumBars] = {128, 128, 1, 128, 128, 128, 128, 128, 1, 128, 128, 1, 128, 128, 1, 1};
        for (int i = 0; i < kNumBars; ++i)
            mbar_init(bars + i, counts[i]);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == 0)
        tmem_alloc(tslot, kTmemCols);
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    const uint32_t tbase = *tslot;
    const Sync sy{bars, abort_flag, p.status};

    if (warp < 4) {
        row_role(p, smem, sy, tbase, b, h, row0, n_chunks);
    } else if (warp < 8) {
        prep_role(p, smem, sy, tbase, b, h, hk, row0, n_chunks);
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if ((threadIdx.x & 31) == 0) {
        mma_role(smem, sy, tbase, n_chunks);
        // every MMA issued has retired before the tensor memory is freed
        mma_commit(bars + kFin);
        const long long t0 = clock64();
        while (!mbar_try_wait_suspend(bars + kFin, 0, 20000u) && clock64() - t0 < (1ll << 31)) {
        }
    }
    tmem_fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tmem_fence_after_sync();
        tmem_free(tbase, kTmemCols);
    }
}

}  // namespace
}  // namespace chunked

bool chunked_supported(const VerifyArgs& a)
{
    return a.qkv_dtype == GDN_BF16 && a.d_k == chunked::DK && a.d_v % 64 == 0 &&
           (a.flags & GDN_FLAG_CHAIN) && (a.flags & GDN_FLAG_PERSIST_LAST) && a.cu_nodes == nullptr;
}

cudaError_t launch_chunked(const VerifyArgs& a, cudaStream_t stream)
{
    using namespace chunked;
    Params p{};
    p.q = static_cast<const __nv_bfloat16*>(a.q);
    p.k = static_cast<const __nv_bfloat16*>(a.k);
    p.v = static_cast<const __nv_bfloat16*>(a.v);
    p.g = a.g;
    p.beta = a.beta;
    p.state_in = a.state_in;
    p.out = a.out;
    p.node_states = a.node_states;
    p.status = a.status;
    p.N = a.n_nodes;
    p.Hk = a.n_k_heads;
    p.Hv = a.n_v_heads;
    p.dv = a.d_v;
    p.G = a.n_v_heads / a.n_k_heads;
    p.scale = a.scale;
    p.state_f16 = a.state_dtype == GDN_F16 ? 1 : 0;
    // opt in to kSmem bytes of dynamic shared memory, once per device
    static std::atomic<int> granted[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64 || granted[dev].load() == 0) {
        e = cudaFuncSetAttribute(gdn_chain_chunked, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess)
            return e;
        if (dev >= 0 && dev < 64)
            granted[dev].store(1);
    }
    dim3 grid((a.d_v + TM - 1) / TM, a.n_v_heads, a.batch);
    return launch_pdl(gdn_chain_chunked, grid, dim3(kThreads), (size_t)kSmem, stream, p);
}

}  // namespace gdn
