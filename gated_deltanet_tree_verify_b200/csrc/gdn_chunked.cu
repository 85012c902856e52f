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
// bf16 (the state, U, Ab, M) are split into bf16 parts, x = x1 + x2 (+ x3)
// (x2 = bf16(x - x1), x3 = bf16(x - x1 - x2): 16 or 24 bits).  The update
// adds U^T diag(r) in 3 parts against the exact bf16 K, and U^T Ab^T takes 6
// of the 9 part products (down to ~2^-16 relative); the state enters
// X^T | Y^T in 2 parts against the exact K and Q (its rounding there reaches
// the state only through U), and the output-only U^T M^T takes 3 of 4
// two-part products.  Over long chains the chunked form stays within a few
// times the f32 token walk's own rounding error.  Layout: the A operands (the state, P^T,
// U^T) live in tensor memory, written by the thread that owns the row
// (bf16 pairs per 32-bit column, the even element in the low half); the B
// operands (K, Q, K^T, Ab, M) in shared memory in the canonical K-major
// layout without swizzle (8 x 16-byte core matrices).  The state itself is
// the f32 accumulator of the update, in tensor memory for the whole chain.
//
// Rounding differs from the token-by-token path (different summation
// order), so this is an opt-in mode, not the chain fast path.
//
// One CTA per (sequence, v-head, 128 rows of d_v), 14 warps: warps 0-7 own
// the state rows (two threads per row, in warps w and w + 4, each with half
// of the columns of the elementwise steps between the products), warps 8-11
// prepare each chunk's S-independent operands one chunk ahead, warp 12
// issues the MMAs, warp 13 loads k, q, g and beta and computes the decays
// two chunks ahead.  k, q and v arrive by TMA (tensor maps over
// this GPU's q, k and v; one thread issues the copies, an mbarrier counts
// the bytes), and each chunk's outputs leave as one TMA store of a 64-token
// x 128-row tile staged in shared memory.  Hand-offs are mbarriers; every
// wait is bounded and a timeout is reported as a status.

#include <atomic>
#include <cstdint>
#include <mutex>

#include <cuda.h>
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
constexpr int kThreads = 448;   // warps 0-7 rows, 8-11 preparation, 12 MMA issue, 13 loads and decays
constexpr int kRows = 256;      // row threads: two per state row, each with half of every step
constexpr int kPrep0 = 256;     // first preparation thread

// Tensor-memory columns (128 lanes x 512 columns of 32 bits, all of it).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;     // state S, f32 [d_v x d_k]
constexpr uint32_t kColAS = 128;  // S in 2 bf16 parts, 64 columns each (A of X^T | Y^T)
constexpr uint32_t kColAP = 128;  //   after that product: P^T in 3 parts of 32 columns
constexpr uint32_t kColU = 224;   //   and U^T, f32 [d_v x T]
constexpr uint32_t kColAUr = 128; //   after that: U^T diag(r) in 3 parts (A of the update)
constexpr uint32_t kColAU0 = 288;  //   and U^T in 2 parts (A of U^T M^T): part 0 in the
constexpr uint32_t kColAU1 = 224;  //   spare columns, part 1 over the first half of U^T
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
constexpr int kOutBytes = T * TM * 4;     // one chunk's outputs, f32 [t][row]
constexpr int kOffKQ = 0;                          // [2]
constexpr int kOffV = kOffKQ + 2 * kKQBytes;
constexpr int kOffAb = kOffV + kVBytes;            // [3 parts]
constexpr int kOffM = kOffAb + 3 * kTTBytes;       // [2 parts]
constexpr int kOffKT = kOffM + 2 * kTTBytes;
constexpr int kOffOut = kOffKT + kKTBytes;
constexpr int kOffL = kOffOut + kOutBytes;         // L, f32 [T][LST]
constexpr int kOffMf = kOffL + T * LST * 4;        // M, f32 [T][LST]
constexpr int kOffAi = kOffMf + T * LST * 4;       // (I + L)^-1, f32 [T][AST]
// Per-token scalars of a chunk: for the preparation warps a = exp(g), beta
// and the inverse norms n_t = 1 / |k_t|, m_t = 1 / |q_t| (1 without
// GDN_FLAG_QK_L2NORM); for the row threads the decays as they use them,
// Gamma_t n_t (against X^T), r_t n_t (the update), Gamma_t m_t (against
// Y^T), and Gamma_{T-1}.
constexpr int kGB = 4 * T;                         // floats per buffer: a | beta | n | m
constexpr int kDec = 3 * T + 4;                    // floats per slot: Gamma n | r n | Gamma m | Gamma_{T-1}
constexpr int kOffGB = kOffAi + T * AST * 4;       // [2][kGB], f32
constexpr int kOffDec = kOffGB + 2 * kGB * 4;      // [3][kDec], f32
constexpr int kOffBar = kOffDec + 3 * kDec * 4;    // mbarriers, tmem base, abort flag
constexpr int kSmem = kOffBar + 256;
static_assert(kSmem <= 227 * 1024, "shared memory");

// mbarriers (index into the array at kOffBar)
enum Bar {
    kKqFull0 = 0,  // k, q of a chunk landed in buffer 0 / 1 (TMA bytes)
    kKqFull1 = 1,
    kKqMma = 2,    // [K; Q] K^T done (MMA commit)
    kDkqFree = 3,  // [K; Q] K^T read out (128)
    kDec0 = 4,     // decays of a chunk written, slots 0..2 (1)
    kAsReady = 7,  // state parts of d_k 0-31 and 64-95 written, previous outputs read (256 row threads)
    kXyDone = 8,   // X^T | Y^T done (commit)
    kApReady = 9,  // P^T parts written (256)
    kAbReady = 10, // Ab parts written (128)
    kUDone = 11,   // U^T done (commit)
    kAuReady = 12, // U^T parts written (256)
    kMktReady = 13,// M parts and K^T written (128)
    kCdDone = 14,  // update done, and U^T M^T before it (commit)
    kFin = 15,     // all MMAs retired (commit)
    kVFull = 16,   // v of a chunk landed (TMA bytes)
    kKqBuf0 = 17,  // k/q buffer 0 / 1 no longer read: the chunk's MMAs (commit) and K^T (128)
    kKqBuf1 = 18,
    kGb0 = 19,     // a and beta of a chunk written, buffer 0 / 1 (1)
    kGb1 = 20,
    kOutDone = 21, // U^T M^T done (commit): the chunk's outputs can be formed
    kAsReady2 = 22,// state parts of d_k 32-63 and 96-127 written (256)
    kNumBars = 23
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
    int gates;    // GDN_FLAG_GATES: g and beta hold the gates' pre-activations
    int qk_norm;  // GDN_FLAG_QK_L2NORM: q and k rows are normalised inside
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

// Whether the phase with the given parity has completed, without waiting.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

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

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Named barrier over the 256 row threads, and the same with a vote.
__device__ __forceinline__ void row_sync() { asm volatile("bar.sync 2, 256;" ::: "memory"); }

__device__ __forceinline__ bool row_all(bool ok)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 2, 256, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(ok ? 1u : 0u)
        : "memory");
    return r != 0;
}

// ---- TMA -------------------------------------------------------------------------------------

// The barrier's current phase also waits for `bytes` bytes of TMA data.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// Box of a 4-d tensor map at (x, y, z, w) into shared memory (no multicast);
// completion counted in bytes on bar.  Elements outside the tensor read 0.
__device__ __forceinline__ void tma_load(uint32_t dst, const CUtensorMap* tm, int x, int y, int z, int w,
                                         uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
        "[%6];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_addr(bar))
        : "memory");
}

// Shared memory to the box of a 4-d tensor map at (x, y, z, w); elements
// outside the tensor are not written.
__device__ __forceinline__ void tma_store(const CUtensorMap* tm, uint32_t src, int x, int y, int z, int w)
{
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(tm)),
                 "r"(src), "r"(x), "r"(y), "r"(z), "r"(w)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

struct Maps {
    CUtensorMap k, q, v, out;  // 4-d: (d, head, token, sequence)
};

// ---- preparation warps ---------------------------------------------------------------

// Chunk c's k and q rows into buffer buf in the canonical layout (K rows
// 0..63, then Q rows): one copy per 8-column piece, 64 tokens each.  Tokens
// past the chain's end read 0.  One thread.
__device__ __forceinline__ void load_kq(const Maps& mp, unsigned char* smem, uint64_t* bar, int buf, int c, int b,
                                        int hk)
{
    const uint32_t kq = smem_addr(smem + kOffKQ + buf * kKQBytes);
    mbar_expect_tx(bar, kKQBytes);
#pragma unroll 1
    for (int pc = 0; pc < DK / 8; ++pc) {
        tma_load(kq + pc * (2 * T * 16), &mp.k, 8 * pc, hk, c * T, b, bar);
        tma_load(kq + pc * (2 * T * 16) + T * 16, &mp.q, 8 * pc, hk, c * T, b, bar);
    }
}

// Chunk c's 128-row slice of v, [t][row]; rows past d_v and tokens past the
// end read 0.  One thread.
__device__ __forceinline__ void load_v(const Maps& mp, unsigned char* smem, uint64_t* bar, int c, int b, int h,
                                       int row0)
{
    mbar_expect_tx(bar, kVBytes);
    tma_load(smem_addr(smem + kOffV), &mp.v, row0, h, c * T, b, bar);
}

// Rows 16 I .. 16 I + 15 of block column J of (I + L)^-1, columns c0 ..
// c0 + NC - 1, for I = J + 1 .. 3, from the diagonal blocks' inverses already
// in Ai: X = -L_(I, J..I-1) Ai_(J..I-1, J), then Ai_(I, J) = Ai_(I, I) X.  One
// warp: lane = row i (lane % 16) and a parity kh (lane / 16); each sum runs
// over the terms of its parity and the two halves meet with one shuffle.  The
// rows the warp reads are its own.
template <int NC>
__device__ __forceinline__ void block_column(const float* L, float* Ai, int J, int c0, int lane)
{
    const int i = lane & 15, kh = lane >> 4;
#pragma unroll 1
    for (int I = J + 1; I < 4; ++I) {
        const int R0 = 16 * I;
        float x[NC];
#pragma unroll
        for (int e = 0; e < NC; ++e)
            x[e] = 0.f;
        const float* Lr = L + (R0 + i) * LST;
#pragma unroll 4
        for (int k = 16 * J + kh; k < R0; k += 2) {
            const float l = Lr[k];
#pragma unroll
            for (int e = 0; e < NC; e += 4) {
                const float4 a = *reinterpret_cast<const float4*>(Ai + k * AST + c0 + e);
                x[e] = __fmaf_rn(l, a.x, x[e]);
                x[e + 1] = __fmaf_rn(l, a.y, x[e + 1]);
                x[e + 2] = __fmaf_rn(l, a.z, x[e + 2]);
                x[e + 3] = __fmaf_rn(l, a.w, x[e + 3]);
            }
        }
#pragma unroll
        for (int e = 0; e < NC; ++e)
            x[e] = -__fadd_rn(x[e], __shfl_xor_sync(0xffffffffu, x[e], 16));
        float* dst = Ai + (R0 + i) * AST + c0;
        if (kh == 0) {
#pragma unroll
            for (int e = 0; e < NC; e += 4)
                *reinterpret_cast<float4*>(dst + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
        }
        __syncwarp();
        float y[NC];
#pragma unroll
        for (int e = 0; e < NC; ++e)
            y[e] = 0.f;
        const float* Dr = Ai + (R0 + i) * AST + R0;  // row i of the block's inverse
#pragma unroll 4
        for (int i2 = kh; i2 < 16; i2 += 2) {
            const float dd = i2 <= i ? Dr[i2] : 0.f;
#pragma unroll
            for (int e = 0; e < NC; e += 4) {
                const float4 a = *reinterpret_cast<const float4*>(Ai + (R0 + i2) * AST + c0 + e);
                y[e] = __fmaf_rn(dd, a.x, y[e]);
                y[e + 1] = __fmaf_rn(dd, a.y, y[e + 1]);
                y[e + 2] = __fmaf_rn(dd, a.z, y[e + 2]);
                y[e + 3] = __fmaf_rn(dd, a.w, y[e + 3]);
            }
        }
#pragma unroll
        for (int e = 0; e < NC; ++e)
            y[e] = __fadd_rn(y[e], __shfl_xor_sync(0xffffffffu, y[e], 16));
        __syncwarp();
        if (kh == 0) {
#pragma unroll
            for (int e = 0; e < NC; e += 4)
                *reinterpret_cast<float4*>(dst + e) = make_float4(y[e], y[e + 1], y[e + 2], y[e + 3]);
        }
        __syncwarp();
    }
}

// (I + L)^-1 for the unit lower triangular I + L (L strictly lower, f32
// [T][LST]) into Ai (f32 [T][AST], whose entries above the diagonal stay 0).
// Warp w inverts diagonal block w (one column per lane); then the block
// columns, in halves of 8 columns: warps 0 and 1 take block column 0 (three
// block rows), warps 2 and 3 block columns 1 and 2 (two and one), with no
// barrier between warps until the end.
__device__ void invert_unit_lower(const float* L, float* Ai, int ptid)
{
    const int pw = ptid >> 5, lane = ptid & 31;
    if (lane < 16) {
        const float* __restrict__ Lb = L + (16 * pw) * LST + 16 * pw;
        const int j = lane;
        float d[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
            for (int k = 0; k + 1 < i; k += 2) {  // d[k] = 0 for k < j
                acc0 = __fmaf_rn(Lb[i * LST + k], d[k], acc0);
                acc1 = __fmaf_rn(Lb[i * LST + k + 1], d[k + 1], acc1);
            }
            if (i & 1)
                acc0 = __fmaf_rn(Lb[i * LST + i - 1], d[i - 1], acc0);
            d[i] = i < j ? 0.f : (i == j ? 1.f : -__fadd_rn(acc0, acc1));
        }
        float* Ac = Ai + (16 * pw) * AST + 16 * pw + j;
#pragma unroll
        for (int i = 0; i < 16; ++i)
            Ac[i * AST] = d[i];
    }
    prep_sync();
    if (pw < 2) {
        block_column<8>(L, Ai, 0, 8 * pw, lane);
    } else {
        block_column<8>(L, Ai, 1, 16 + 8 * (pw - 2), lane);
        block_column<8>(L, Ai, 2, 32 + 8 * (pw - 2), lane);
    }
    prep_sync();
}

// This thread's row t of [K; Q] K^T (tensor memory at ta) times the row's
// decays R[t][i] = a_{i+1} ... a_t, a running product over i from t down to
// 0: row t of L = diag(beta) (K K^T o R) below the diagonal (K rows) or of
// M = Q K^T o R on and below it (Q rows).  NORM: the products are of the
// normalised rows, (x_t . k_i) / (|x_t| |k_i|), from the inverse norms in gb.
template <bool NORM>
__device__ __forceinline__ void lm_row(const float* gb, float* out, bool qrow, int t, uint32_t ta)
{
    const float bt = gb[T + t];
    const float nt = NORM ? gb[(qrow ? 3 : 2) * T + t] : 1.f;  // this row's 1 / |q_t| or 1 / |k_t|
    float* rowp = out + t * LST;
    float run = 1.f;
#pragma unroll 1
    for (int hs = 1; hs >= 0; --hs) {
        uint32_t d[32];
        float a[32], nn[32];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float4 x = reinterpret_cast<const float4*>(gb + 32 * hs)[e];
            a[4 * e] = x.x, a[4 * e + 1] = x.y, a[4 * e + 2] = x.z, a[4 * e + 3] = x.w;
            if (NORM) {
                const float4 y = reinterpret_cast<const float4*>(gb + 2 * T + 32 * hs)[e];
                nn[4 * e] = y.x, nn[4 * e + 1] = y.y, nn[4 * e + 2] = y.z, nn[4 * e + 3] = y.w;
            }
        }
        tmem_ld32(ta + 32 * hs, d);
        float val[32];
#pragma unroll
        for (int e = 31; e >= 0; --e) {
            const int i = 32 * hs + e;
            const float kk = NORM ? __fmul_rn(__uint_as_float(d[e]), __fmul_rn(nt, nn[e])) : __uint_as_float(d[e]);
            if (qrow)
                val[e] = i <= t ? __fmul_rn(kk, run) : 0.f;
            else
                val[e] = i < t ? __fmul_rn(bt, __fmul_rn(kk, run)) : 0.f;
            if (i <= t)
                run = __fmul_rn(run, a[e]);
        }
#pragma unroll
        for (int e = 0; e < 32; ++e)
            rowp[32 * hs + e] = val[e];
    }
}

__device__ void prep_role(unsigned char* smem, const Sync& sy, uint32_t tbase, int n_chunks, int p_qk_norm)
{
    const int ptid = threadIdx.x - kPrep0;
    const int pw = ptid >> 5;                  // lane quarter of tensor memory
    const bool qrow = ptid >= T;               // reads a Q row of [K; Q] K^T, else a K row
    const int t = ptid & (T - 1);              // that row's token
    float* L = reinterpret_cast<float*>(smem + kOffL);
    float* Mf = reinterpret_cast<float*>(smem + kOffMf);
    float* Ai = reinterpret_cast<float*>(smem + kOffAi);

    for (int i = ptid; i < T * AST; i += 128)
        Ai[i] = 0.f;

    for (int c = 0; c < n_chunks; ++c) {
        const int buf = c & 1;
        const float* gb = reinterpret_cast<const float*>(smem + kOffGB) + buf * kGB;
        // 1. this chunk's a and beta (written by the load warp), then this
        //    thread's row of [K; Q] K^T times the row's decays
        //    R[t][i] = a_{i+1} ... a_t, a running product over i from t down
        //    to 0: L (K rows) and M (Q rows)
        if (!prep_all(sy.wait(kGb0 + buf, (c >> 1) & 1) && sy.wait(kKqMma, c & 1)))
            return;
        tmem_fence_after_sync();
        if (p_qk_norm)
            lm_row<true>(gb, qrow ? Mf : L, qrow, t, tbase + ((uint32_t)(32 * pw) << 16) + kColKQ);
        else
            lm_row<false>(gb, qrow ? Mf : L, qrow, t, tbase + ((uint32_t)(32 * pw) << 16) + kColKQ);
        tmem_fence_before_sync();
        sy.arrive(kDkqFree);
        prep_sync();
        // 2. Ai = (I + L)^-1
        invert_unit_lower(L, Ai, ptid);
        // 3. Ab = Ai diag(beta) in 3 bf16 parts, once the previous chunk's
        //    U^T product is done with them
        if (c > 0 && !prep_all(sy.wait(kUDone, (c - 1) & 1)))
            return;
#pragma unroll 1
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
        // 4. M in 2 bf16 parts and K^T, once the previous chunk's update and
        //    U^T M^T products are done with them (and this chunk's k is in)
        if (!prep_all((c == 0 || sy.wait(kCdDone, (c - 1) & 1)) && sy.wait(kKqFull0 + buf, (c >> 1) & 1)))
            return;
#pragma unroll 1
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
        sy.arrive(kKqBuf0 + buf);
    }
}

// ---- loads and decays ----------------------------------------------------------------------

// Chunk c's per-token scalars (kGB floats into buffer buf, kDec into slot
// c % 3): a = exp(g) and beta; with raw gates, g = x and beta = y stand for
// g = -softplus(x) and beta = sigmoid(y), so a = 1 / (1 + e^x) and
// beta = 1 / (1 + e^-y) (the walk kernels' expressions; x = +inf resets);
// tokens past the end have a = 1, beta = 0.  The decays Gamma_t = a_0 ...
// a_t and r_t = a_{t+1} ... a_{T-1} by shuffle scans (lane l holds tokens
// 2 l and 2 l + 1).  With qk_norm the inverse norms of the chunk's k and q
// rows, read from its [K; Q] buffer (which must have landed), else 1 (and 1
// for tokens past the end).  One warp.
__device__ __forceinline__ void decays(const Params& p, unsigned char* smem, int buf, int c, int b, int h, int lane)
{
    float a[2], bt[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int t = c * T + 2 * lane + e;
        a[e] = 1.f;
        bt[e] = 0.f;
        if (t < p.N) {
            const size_t gi = ((size_t)b * p.N + t) * p.Hv + h;
            const float g = __ldg(p.g + gi), be = __ldg(p.beta + gi);
            if (p.gates) {
                a[e] = __fdiv_rn(1.f, __fadd_rn(1.f, expf(g)));
                bt[e] = __fdiv_rn(1.f, __fadd_rn(1.f, expf(-be)));
            } else {
                a[e] = expf(g);
                bt[e] = be;
            }
        }
    }
    // inverse norms of K rows (n) and Q rows (m) 2 lane and 2 lane + 1
    float nk[2] = {1.f, 1.f}, nq[2] = {1.f, 1.f};
    if (p.qk_norm) {
        const unsigned char* kq = smem + kOffKQ + buf * kKQBytes;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int n = (e >> 1) * T + 2 * lane + (e & 1);  // row of [K; Q]
            float ss = 0.f;
#pragma unroll 4
            for (int pc = 0; pc < DK / 8; ++pc) {
                const uint4 u = *reinterpret_cast<const uint4*>(kq + pc * (2 * T * 16) + (n >> 3) * 128 + (n & 7) * 16);
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int f = 0; f < 4; ++f) {
                    const float2 x = bf16x2_to_float2(w[f]);
                    ss = __fmaf_rn(x.x, x.x, ss);
                    ss = __fmaf_rn(x.y, x.y, ss);
                }
            }
            // tokens past the end are zero rows: they keep 1 (no 0 * inf)
            const float inv = c * T + 2 * lane + (e & 1) < p.N ? __fdiv_rn(1.f, __fsqrt_rn(ss)) : 1.f;
            if (e < 2)
                nk[e] = inv;
            else
                nq[e - 2] = inv;
        }
    }
    // inclusive prefix and suffix products of the lanes' pair products
    const float pr = __fmul_rn(a[0], a[1]);
    float pre = pr, suf = pr;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const float up = __shfl_up_sync(0xffffffffu, pre, d);
        const float dn = __shfl_down_sync(0xffffffffu, suf, d);
        if (lane >= d)
            pre = __fmul_rn(up, pre);
        if (lane + d < 32)
            suf = __fmul_rn(suf, dn);
    }
    float before = __shfl_up_sync(0xffffffffu, pre, 1);  // product of tokens < 2 lane
    float after = __shfl_down_sync(0xffffffffu, suf, 1);  // product of tokens > 2 lane + 1
    if (lane == 0)
        before = 1.f;
    if (lane == 31)
        after = 1.f;
    const float g0 = __fmul_rn(before, a[0]), g1 = __fmul_rn(g0, a[1]);  // Gamma
    const float r0 = __fmul_rn(a[1], after), r1 = after;                  // r
    float* gb = reinterpret_cast<float*>(smem + kOffGB) + buf * kGB;
    float* dec = reinterpret_cast<float*>(smem + kOffDec) + (c % 3) * kDec;
    *reinterpret_cast<float2*>(gb + 2 * lane) = make_float2(a[0], a[1]);
    *reinterpret_cast<float2*>(gb + T + 2 * lane) = make_float2(bt[0], bt[1]);
    *reinterpret_cast<float2*>(gb + 2 * T + 2 * lane) = make_float2(nk[0], nk[1]);
    *reinterpret_cast<float2*>(gb + 3 * T + 2 * lane) = make_float2(nq[0], nq[1]);
    *reinterpret_cast<float2*>(dec + 2 * lane) = make_float2(__fmul_rn(g0, nk[0]), __fmul_rn(g1, nk[1]));
    *reinterpret_cast<float2*>(dec + T + 2 * lane) = make_float2(__fmul_rn(r0, nk[0]), __fmul_rn(r1, nk[1]));
    *reinterpret_cast<float2*>(dec + 2 * T + 2 * lane) = make_float2(__fmul_rn(g0, nq[0]), __fmul_rn(g1, nq[1]));
    if (lane == 31)
        dec[3 * T] = g1;  // Gamma_{T-1}
}

// One warp: chunks 0 and 1, then chunk c + 2 into buffer c % 2 once chunk c's
// MMAs, K^T and preparation are done with it: k and q by TMA (lane 0),
// a, beta and the decays.  kq_loads[j]: TMA loads issued into buffer j.
__device__ void load_role(const Params& p, const Maps& mp, unsigned char* smem, const Sync& sy, int b, int h,
                          int hk, int n_chunks, int (&kq_loads)[2])
{
    const int lane = threadIdx.x & 31;
    for (int c = 0; c < n_chunks && c < 2; ++c) {
        if (lane == 0) {
            load_kq(mp, smem, sy.bar + kKqFull0 + c, c, c, b, hk);
            ++kq_loads[c];
        }
        if (p.qk_norm && !__all_sync(0xffffffffu, sy.wait(kKqFull0 + c, 0)))
            return;
        decays(p, smem, c, c, b, h, lane);
        __syncwarp();
        if (lane == 0) {
            sy.arrive(kGb0 + c);
            sy.arrive(kDec0 + c);
        }
    }
    for (int c = 0; c + 2 < n_chunks; ++c) {
        if (!__all_sync(0xffffffffu, sy.wait(kKqBuf0 + (c & 1), (c >> 1) & 1)))
            return;
        if (lane == 0) {
            load_kq(mp, smem, sy.bar + kKqFull0 + (c & 1), c & 1, c + 2, b, hk);
            ++kq_loads[c & 1];
        }
        if (p.qk_norm && !__all_sync(0xffffffffu, sy.wait(kKqFull0 + (c & 1), ((c + 2) >> 1) & 1)))
            return;
        decays(p, smem, c & 1, c + 2, b, h, lane);
        __syncwarp();
        if (lane == 0) {
            sy.arrive(kGb0 + (c & 1));
            sy.arrive(kDec0 + (c + 2) % 3);
        }
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
        // X^T | Y^T = S [K; Q]^T, S in 2 parts, in two stages of d_k as the
        // row threads write the parts: k-steps 0, 1, 4, 5, then 2, 3, 6, 7
#pragma unroll
        for (int stage = 0; stage < 2; ++stage) {
            if (!sy.wait(stage == 0 ? kAsReady : kAsReady2, c & 1))
                return;
            tmem_fence_after_sync();
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int part = q >> 2, ks = (q & 1) + ((q & 2) << 1) + 2 * stage;
                mma_ts(tbase + kColX, tbase + kColAS + 64 * part + 8 * ks, kdesc(kq + ks * 2 * kKQLbo, kKQLbo),
                       idesc_bf16(2 * T), stage + q != 0 ? 1u : 0u);
            }
        }
        mma_commit(sy.bar + kXyDone);
        mma_commit(sy.bar + kKqBuf0 + (c & 1));  // with [K; Q] K^T of c, issued before
        // the next chunk's [K; Q] K^T and this chunk's U^T = P^T Ab^T, in
        // the order their operands become ready; U^T from the part products
        // (P, Ab) of weight at least 2^-16
        bool kq_done = c + 1 >= n_chunks, u_done = false;
        const long long t0 = clock64();
        for (bool issued = true; !(kq_done && u_done); ) {
            if (!issued) {
                __nanosleep(32);  // leave the issue slots to the warps being waited for
                if (*sy.abort || clock64() - t0 > (1ll << 31)) {
                    *sy.abort = 1;
                    report_status(sy.status, kStatusTimeout);
                    return;
                }
            }
            issued = false;
            if (!kq_done && mbar_test(sy.bar + kKqFull0 + ((c + 1) & 1), ((c + 1) >> 1) & 1) &&
                mbar_test(sy.bar + kDkqFree, c & 1)) {
                tmem_fence_after_sync();
                kq_product(c + 1);
                kq_done = issued = true;
            }
            if (!u_done && mbar_test(sy.bar + kApReady, c & 1) && mbar_test(sy.bar + kAbReady, c & 1)) {
                tmem_fence_after_sync();
#pragma unroll
                for (int q = 0; q < 6 * (T / 16); ++q) {
                    const int pr = q >> 2, ks = q & 3;
                    const int pp = pr == 2 ? 1 : (pr == 4 ? 1 : (pr == 5 ? 2 : 0));  // (0,0) (0,1) (1,0) (0,2) (1,1) (2,0)
                    const int pa = pr == 1 ? 1 : (pr == 3 ? 2 : (pr == 4 ? 1 : 0));
                    mma_ts(tbase + kColU, tbase + kColAP + 32 * pp + 8 * ks,
                           kdesc(ab + pa * kTTBytes + ks * 2 * kTTLbo, kTTLbo), idesc_bf16(T), q != 0 ? 1u : 0u);
                }
                mma_commit(sy.bar + kUDone);
                u_done = issued = true;
            }
        }
        // U^T M^T, then S += (U^T diag(r)) K: the row threads form this
        // chunk's outputs while the update runs
        if (!sy.wait(kAuReady, c & 1) || !sy.wait(kMktReady, c & 1))
            return;
        tmem_fence_after_sync();
#pragma unroll
        for (int q = 0; q < 3 * (T / 16); ++q) {
            const int pr = q >> 2, ks = q & 3;  // (U, M) parts: (0,0) (0,1) (1,0)
            const uint32_t au = pr == 2 ? kColAU1 : kColAU0;
            mma_ts(tbase + kColX, tbase + au + 8 * ks, kdesc(mm + (pr == 1 ? kTTBytes : 0) + ks * 2 * kTTLbo, kTTLbo),
                   idesc_bf16(T), q != 0 ? 1u : 0u);
        }
        mma_commit(sy.bar + kOutDone);
#pragma unroll
        for (int q = 0; q < 3 * (T / 16); ++q) {
            const int part = q >> 2, ks = q & 3;
            mma_ts(tbase + kColS, tbase + kColAUr + 32 * part + 8 * ks, kdesc(kt + ks * 2 * kKTLbo, kKTLbo),
                   idesc_bf16(DK), 1u);
        }
        mma_commit(sy.bar + kCdDone);
    }
}

// ---- row warps ----------------------------------------------------------------------------------

// The previous chunk's outputs, scale (Gamma_t Y^T + U^T M^T) (Gam holds
// Gamma_t / |q_t| with q/k normalisation, Gamma_t without): each thread
// writes its row of the [t][row] tile in shared memory, then one thread
// stores the tile with TMA (after the previous store has read it).
__device__ __forceinline__ void write_outputs(const Params& p, const Maps& mp, unsigned char* smem, uint32_t trow,
                                              const float* Gam, int b, int h, int row0, int t0)
{
    const int m = threadIdx.x & (TM - 1), hs = threadIdx.x >> 7;  // row; half of the tokens
    float* tile = reinterpret_cast<float*>(smem + kOffOut) + m;
    if (threadIdx.x == 0)
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
    row_sync();
    {
        uint32_t y[32], o[32];
        float gm[32];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float4 x = reinterpret_cast<const float4*>(Gam + 32 * hs)[e];
            gm[4 * e] = x.x, gm[4 * e + 1] = x.y, gm[4 * e + 2] = x.z, gm[4 * e + 3] = x.w;
        }
        tmem_ld32(trow + kColY + 32 * hs, y);
        tmem_ld32(trow + kColX + 32 * hs, o);
#pragma unroll
        for (int i = 0; i < 32; ++i)
            tile[(32 * hs + i) * TM] =
                __fmul_rn(p.scale, __fmaf_rn(gm[i], __uint_as_float(y[i]), __uint_as_float(o[i])));
    }
    fence_proxy_async();
    row_sync();
    if (threadIdx.x == 0)
        tma_store(&mp.out, smem_addr(smem + kOffOut), row0, h, t0, b);
}

// v_loads: v loads this thread issued (thread 0 issues them all).
__device__ void row_role(const Params& p, const Maps& mp, unsigned char* smem, const Sync& sy, uint32_t tbase, int b,
                         int h, int row0, int n_chunks, int& v_loads)
{
    const int tid = threadIdx.x, warp = tid >> 5;
    const int m = tid & (TM - 1);   // state row within the tile (lane quarter = warp % 4)
    const int half = tid >> 7;      // which half of each step's columns
    const int row = row0 + m;       // row of d_v
    const uint32_t trow = tbase + ((uint32_t)(32 * (warp & 3)) << 16);
    const float* decs = reinterpret_cast<const float*>(smem + kOffDec);
    if (tid == 0) {
        load_v(mp, smem, sy.bar + kVFull, 0, b, h, row0);
        ++v_loads;
    }

    for (int c = 0; c < n_chunks; ++c) {
        const int slot = c % 3;
        const float* Gam = decs + slot * kDec;  // Gamma_t / |k_t|
        const float* rv = Gam + T;              // r_t / |k_t|
        if (!row_all(sy.wait(kDec0 + slot, (c / 3) & 1)))
            return;
        const float gT = Gam[3 * T];            // Gamma_{T-1}
        // 0. the previous chunk's outputs; S into 2 bf16 parts (A of X^T | Y^T),
        //    and Gamma_{T-1} S back as the update's accumulator
        if (c > 0) {
            if (!row_all(sy.wait(kOutDone, (c - 1) & 1)))
                return;
            tmem_fence_after_sync();
            write_outputs(p, mp, smem, trow, decs + ((c - 1) % 3) * kDec + 2 * T, b, h, row0, (c - 1) * T);
            if (!row_all(sy.wait(kCdDone, (c - 1) & 1)))
                return;
            tmem_fence_after_sync();
        }
#pragma unroll 1
        for (int s = 2 * half; s < 2 * half + 2; ++s) {
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
            uint32_t p1[16], p2[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
                split2(__uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1]), p1[e], p2[e]);
            tmem_st16(trow + kColAS + 16 * s, p1);
            tmem_st16(trow + kColAS + 64 + 16 * s, p2);
#pragma unroll
            for (int e = 0; e < 32; ++e)
                x[e] = __float_as_uint(__fmul_rn(gT, __uint_as_float(x[e])));
            tmem_st32(trow + kColS + 32 * s, x);
            tmem_wait_st();
            tmem_fence_before_sync();
            sy.arrive(s == 2 * half ? kAsReady : kAsReady2);
        }

        // 1. P^T = V^T - X^T diag(Gamma) into 3 bf16 parts (A of U^T)
        if (!row_all(sy.wait(kXyDone, c & 1) && sy.wait(kVFull, c & 1)))
            return;
        tmem_fence_after_sync();
        {
            const unsigned short* V = reinterpret_cast<const unsigned short*>(smem + kOffV) + m;
            {
                const int hs = half;
                uint32_t x[32];
                float gm[32], vv[32];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float4 g4 = reinterpret_cast<const float4*>(Gam + 32 * hs)[e];
                    gm[4 * e] = g4.x, gm[4 * e + 1] = g4.y, gm[4 * e + 2] = g4.z, gm[4 * e + 3] = g4.w;
                }
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    vv[e] = __uint_as_float((uint32_t)V[(32 * hs + e) * TM] << 16);
                tmem_ld32(trow + kColX + 32 * hs, x);
                uint32_t p1[16], p2[16], p3[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    split3(__fsub_rn(vv[2 * e], __fmul_rn(gm[2 * e], __uint_as_float(x[2 * e]))),
                           __fsub_rn(vv[2 * e + 1], __fmul_rn(gm[2 * e + 1], __uint_as_float(x[2 * e + 1]))), p1[e],
                           p2[e], p3[e]);
                tmem_st16(trow + kColAP + 16 * hs, p1);
                tmem_st16(trow + kColAP + 32 + 16 * hs, p2);
                tmem_st16(trow + kColAP + 64 + 16 * hs, p3);
            }
        }
        tmem_wait_st();
        tmem_fence_before_sync();
        sy.arrive(kApReady);

        // 2. U^T diag(r) in 3 parts (A of the update), U^T in 2 (A of U^T M^T);
        //    each half of U^T is read before anything is written over it.
        //    Every row thread is done with this chunk's v: the next one loads.
        if (!row_all(sy.wait(kUDone, c & 1)))
            return;
        if (tid == 0 && c + 1 < n_chunks) {
            load_v(mp, smem, sy.bar + kVFull, c + 1, b, h, row0);
            ++v_loads;
        }
        tmem_fence_after_sync();
        {
            const int hs = half;
            uint32_t u[32];
            float rr[32];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float4 r4 = reinterpret_cast<const float4*>(rv + 32 * hs)[e];
                rr[4 * e] = r4.x, rr[4 * e + 1] = r4.y, rr[4 * e + 2] = r4.z, rr[4 * e + 3] = r4.w;
            }
            tmem_ld32(trow + kColU + 32 * hs, u);
            uint32_t p1[16], p2[16], p3[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
                split3(__fmul_rn(rr[2 * e], __uint_as_float(u[2 * e])), __fmul_rn(rr[2 * e + 1], __uint_as_float(u[2 * e + 1])),
                       p1[e], p2[e], p3[e]);
            tmem_st16(trow + kColAUr + 16 * hs, p1);
            tmem_st16(trow + kColAUr + 32 + 16 * hs, p2);
            tmem_st16(trow + kColAUr + 64 + 16 * hs, p3);
#pragma unroll
            for (int e = 0; e < 16; ++e)
                split2(__uint_as_float(u[2 * e]), __uint_as_float(u[2 * e + 1]), p1[e], p2[e]);
            tmem_st16(trow + kColAU0 + 16 * hs, p1);
            // part 1 goes over the first half of U^T: both halves have read it
            tmem_fence_before_sync();
            row_sync();
            tmem_fence_after_sync();
            tmem_st16(trow + kColAU1 + 16 * hs, p2);
        }
        tmem_wait_st();
        tmem_fence_before_sync();
        sy.arrive(kAuReady);
    }

    // the last chunk's outputs and the last state -> node_states[b][0][h][row][:]
    if (!row_all(sy.wait(kCdDone, (n_chunks - 1) & 1)))
        return;
    tmem_fence_after_sync();
    write_outputs(p, mp, smem, trow, decs + ((n_chunks - 1) % 3) * kDec + 2 * T, b, h, row0, (n_chunks - 1) * T);
    const size_t base = (((size_t)b * p.Hv + h) * p.dv + row) * DK;
#pragma unroll 1
    for (int s = 2 * half; s < 2 * half + 2; ++s) {
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

// Bounded wait, ignoring the abort flag, for a phase of TMA data this thread
// asked for: the copy must land before the CTA's shared memory goes away.
__device__ __forceinline__ void drain(uint64_t* bar, uint32_t parity)
{
    const long long t0 = clock64();
    while (!mbar_try_wait_suspend(bar, parity, 20000u) && clock64() - t0 < (1ll << 31)) {
    }
}

__global__ void __launch_bounds__(kThreads, 1) gdn_chain_chunked(const Params p, const __grid_constant__ Maps mp)
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
        const uint32_t counts[kNumBars] = {1, 1, 1, 128, 1, 1, 1, kRows, 1, kRows, 128, 1, kRows, 128, 1, 1, 1, 129, 129, 1, 1, 1, kRows};
        for (int i = 0; i < kNumBars; ++i)
            mbar_init(bars + i, counts[i]);
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == 0)
        tmem_alloc(tslot, kTmemCols);
    if (threadIdx.x == 32) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mp.k)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mp.q)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mp.v)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mp.out)) : "memory");
    }
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    const uint32_t tbase = *tslot;
    const Sync sy{bars, abort_flag, p.status};

    // Each TMA load is waited for by the thread that issued it before the CTA
    // can leave (a barrier has at most one phase outstanding: a buffer is
    // reloaded only after its previous load was used).
    if (warp < 8) {
        int v_loads = 0;
        row_role(p, mp, smem, sy, tbase, b, h, row0, n_chunks, v_loads);
        if (threadIdx.x == 0) {
            if (v_loads > 0)
                drain(bars + kVFull, (uint32_t)(v_loads - 1) & 1);
            asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
        }
    } else if (warp < 12) {
        prep_role(smem, sy, tbase, n_chunks, p.qk_norm);
    } else if (warp == 13) {
        int kq_loads[2] = {0, 0};
        load_role(p, mp, smem, sy, b, h, hk, n_chunks, kq_loads);
        if ((threadIdx.x & 31) == 0) {
            if (kq_loads[0] > 0)
                drain(bars + kKqFull0, (uint32_t)(kq_loads[0] - 1) & 1);
            if (kq_loads[1] > 0)
                drain(bars + kKqFull1, (uint32_t)(kq_loads[1] - 1) & 1);
        }
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

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn()
{
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess && f)
            fn = reinterpret_cast<EncodeTiledFn>(f);
        cudaGetLastError();  // a failed lookup leaves no sticky error behind
    });
    return fn;
}

// A 4-d map (d, head, token, sequence) over a [batch][N][heads][d] tensor,
// boxes of (box_d, 1, 64, 1); elements outside read as zero.
bool encode_map(EncodeTiledFn fn, CUtensorMap* m, const void* base, CUtensorMapDataType type, size_t esize,
                uint64_t d, uint64_t heads, uint64_t N, uint64_t batch, uint32_t box_d)
{
    const cuuint64_t dims[4] = {d, heads, N, batch};
    const cuuint64_t strides[3] = {d * esize, heads * d * esize, N * heads * d * esize};
    const cuuint32_t box[4] = {box_d, 1, (cuuint32_t)chunked::T, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(m, type, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

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
    p.gates = (a.flags & GDN_FLAG_GATES) ? 1 : 0;
    p.qk_norm = (a.flags & GDN_FLAG_QK_L2NORM) ? 1 : 0;
    const EncodeTiledFn fn = encode_tiled_fn();
    if (fn == nullptr)
        return cudaErrorNotSupported;
    Maps mp;
    const uint64_t N = a.n_nodes, B = a.batch;
    if (!encode_map(fn, &mp.k, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, a.n_k_heads, N, B, 8) ||
        !encode_map(fn, &mp.q, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, DK, a.n_k_heads, N, B, 8) ||
        !encode_map(fn, &mp.v, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.d_v, a.n_v_heads, N, B, TM) ||
        !encode_map(fn, &mp.out, a.out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.d_v, a.n_v_heads, N, B, TM))
        return cudaErrorInvalidValue;
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
    return launch_pdl(gdn_chain_chunked, grid, dim3(kThreads), (size_t)kSmem, stream, p, mp);
}

}  // namespace gdn
