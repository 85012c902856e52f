// gdn_chunked.cu -- chains in chunks of 64 tokens on the tensor cores
// (GDN_FLAG_CHUNKED: a prefill-style chain with last-only persistence).
//
// Within a chunk of T tokens starting from state S_0 (d_v x d_k), with
// a_t = exp(g_t), Gamma_t = a_0 ... a_t and R[t][i] = a_{i+1} ... a_t (the
// decay from token i to token t), the recurrence
//
//     S_t = a_t S_{t-1} + beta_t (v_t - a_t S_{t-1} k_t) k_t^T,  o_t = scale S_t q_t
//
// unrolls to S_t = Gamma_t S_0 + sum_{i <= t} R[t][i] u_i k_i^T, where the
// pseudo-values u_i = beta_i (v_i - a_i S_{i-1} k_i) solve the unit lower
// triangular system
//
//     u_i + beta_i sum_{j < i} R[i][j] (k_i . k_j) u_j = beta_i (v_i - Gamma_i S_0 k_i).
//
// Hence, per chunk (the delta rule's chunked "WY" form; the Gated Delta
// Networks paper by Yang, Kautz and Hatamizadeh derives it):
//
//     P   = diag(beta) (V - diag(Gamma) K S_0^T)              [T x d_v]
//     U   = (I + L)^-1 P,  L = diag(beta) (K K^T o R), strictly lower
//     O   = scale (diag(Gamma) Q S_0^T + (Q K^T o R_incl) U)   [T x d_v]
//     S_T = Gamma_{T-1} S_0 + (diag(r) U)^T K,  r_i = R[T-1][i]
//
// The products are tensor-core mma.sync (bf16 for K K^T and Q K^T, whose
// operands are exact; tf32 otherwise).  f32 operands are split into two tf32
// parts, x = hi + lo, and products formed as hi*hi + hi*lo + lo*hi (bf16
// inputs are exact in tf32, so their lo part is 0 and that term is dropped),
// which keeps the chunked form at f32 accuracy.  The triangular system is
// solved by forward substitution on the CUDA cores, four threads per column.
// Rounding differs from the token-by-token path (different summation
// order), so this is an opt-in mode, not the chain fast path.
//
// One CTA per (sequence, v-head, 64 rows of d_v), 8 warps; chunk c + 1's
// inputs are staged with cp.async while chunk c is computed.

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

constexpr int T = 64;            // tokens per chunk
constexpr int DK = 128;          // d_k
constexpr int TV = 64;           // d_v rows per CTA
constexpr int kThreads = 256;    // 8 warps
constexpr int KST = DK + 8;      // bf16 row stride of K, Q (272 bytes)
constexpr int VST = TV + 8;      // bf16 row stride of the V tile
constexpr int SST = DK + 4;      // float2 row stride of the state tile: (value, tf32 remainder)
constexpr int MST = T + 4;       // f32 row stride of T x T matrices and U

struct Params {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    const float* g;
    const float* beta;
    const float* state_in;
    float* out;
    void* node_states;
    int N, Hk, Hv, dv, G;
    float scale;
    int state_f16;
};

// Shared memory layout (bytes), one CTA.
constexpr int kKQBytes = T * KST * 2;                 // one K or Q chunk
constexpr int kVBytes = T * VST * 2;                  // one V tile chunk
constexpr int kOffK = 0;                              // K[2]
constexpr int kOffQ = kOffK + 2 * kKQBytes;           // Q[2]
constexpr int kOffV = kOffQ + 2 * kKQBytes;           // V[2]
constexpr int kOffGB = kOffV + 2 * kVBytes;           // g[2][T], beta[2][T]
constexpr int kOffS = kOffGB + 4 * T * 4;             // S [TV][SST] float2
constexpr int kOffR = kOffS + TV * SST * 8;           // R [T][MST]
constexpr int kOffL = kOffR + T * MST * 4;            // L [T][MST]
constexpr int kOffM = kOffL + T * MST * 4;            // Q K^T o R_incl [T][MST]
constexpr int kOffU = kOffM + T * MST * 4;            // P, then U [T][MST]
constexpr int kOffA = kOffU + T * MST * 4;            // a [T], Gamma [T]
constexpr int kSmem = kOffA + 2 * T * 4;

__device__ __forceinline__ uint32_t f2tf32(float x)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// The tf32 remainder of x: x - tf32(x), itself rounded to tf32.
__device__ __forceinline__ float tf32_rem(float x)
{
    return __uint_as_float(f2tf32(__fsub_rn(x, __uint_as_float(f2tf32(x)))));
}

// x = hi + lo, both tf32 (lo is the rounding remainder, itself rounded).
__device__ __forceinline__ void split(float x, uint32_t& hi, uint32_t& lo)
{
    hi = f2tf32(x);
    lo = f2tf32(__fsub_rn(x, __uint_as_float(hi)));
}

__device__ __forceinline__ void mma_tf32(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bf16 element as a tf32 operand (exact: 8 of tf32's 10 mantissa bits)
__device__ __forceinline__ uint32_t bf2tf(const __nv_bfloat16* p)
{
    return static_cast<uint32_t>(*reinterpret_cast<const unsigned short*>(p)) << 16;
}

__device__ __forceinline__ float bf2f(const __nv_bfloat16* p) { return __uint_as_float(bf2tf(p)); }

__device__ __forceinline__ uint32_t ld32(const void* p) { return *reinterpret_cast<const uint32_t*>(p); }

__device__ __forceinline__ void cp_async16(void* dst, const void* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}

// Stage chunk c's k, q rows, the CTA's v slice, g and beta; tokens past the
// chain's end are zero (k = q = v = 0, beta = 0, g = 0: they leave the state
// unchanged and their outputs are not written).
__device__ void stage_chunk(const Params& p, unsigned char* smem, int buf, int c, int b, int h, int hk, int row0)
{
    const int tid = threadIdx.x;
    const int t0 = c * T;
    __nv_bfloat16* K = reinterpret_cast<__nv_bfloat16*>(smem + kOffK + buf * kKQBytes);
    __nv_bfloat16* Q = reinterpret_cast<__nv_bfloat16*>(smem + kOffQ + buf * kKQBytes);
    __nv_bfloat16* V = reinterpret_cast<__nv_bfloat16*>(smem + kOffV + buf * kVBytes);
    float* gb = reinterpret_cast<float*>(smem + kOffGB) + buf * 2 * T;
    // k, q: T rows x 16 chunks of 16 bytes each
    for (int i = tid; i < 2 * T * (DK / 8); i += kThreads) {
        const int which = i / (T * (DK / 8));
        const int r = (i / (DK / 8)) % T, ch = i % (DK / 8);
        __nv_bfloat16* dst = (which == 0 ? K : Q) + r * KST + ch * 8;
        if (t0 + r < p.N) {
            const size_t node = (size_t)b * p.N + t0 + r;
            const __nv_bfloat16* src = (which == 0 ? p.k : p.q) + (node * p.Hk + hk) * DK + ch * 8;
            cp_async16(dst, src);
        } else {
            *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
        }
    }
    // v: T rows x TV / 8 chunks
    for (int i = tid; i < T * (TV / 8); i += kThreads) {
        const int r = i / (TV / 8), ch = i % (TV / 8);
        __nv_bfloat16* dst = V + r * VST + ch * 8;
        if (t0 + r < p.N) {
            const size_t node = (size_t)b * p.N + t0 + r;
            cp_async16(dst, p.v + (node * p.Hv + h) * p.dv + row0 + ch * 8);
        } else {
            *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
        }
    }
    if (tid < 2 * T) {
        const int r = tid % T;
        float x = 0.f;
        if (t0 + r < p.N) {
            const size_t gi = ((size_t)b * p.N + t0 + r) * p.Hv + h;
            x = tid < T ? __ldg(p.g + gi) : __ldg(p.beta + gi);
        }
        gb[tid] = x;
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

__global__ void __launch_bounds__(kThreads, 1) gdn_chain_chunked(const Params p)
{
    extern __shared__ __align__(16) unsigned char smem[];
    float2* S = reinterpret_cast<float2*>(smem + kOffS);
    float* Rm = reinterpret_cast<float*>(smem + kOffR);
    float* Lp = reinterpret_cast<float*>(smem + kOffL);
    float* Mq = reinterpret_cast<float*>(smem + kOffM);
    float* U = reinterpret_cast<float*>(smem + kOffU);
    float* Av = reinterpret_cast<float*>(smem + kOffA);
    float* Gam = Av + T;

    const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int hk = h / p.G;
    const int row0 = tile * TV;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g8 = lane >> 2, t4 = lane & 3;          // mma fragment coordinates
    const int rb = (warp & 3) * 16;                   // this warp's 16 rows of a 64-row product
    const int n_chunks = (p.N + T - 1) / T;

    pdl_wait_then_release();
    // the state tile S_0 = state_in[b][h][row0 .. row0 + 63][:]
    {
        const float* src = p.state_in + (((size_t)b * p.Hv + h) * p.dv + row0) * DK;
        for (int i = tid; i < TV * DK / 4; i += kThreads) {
            const int r = i / (DK / 4), c4 = i % (DK / 4);
            const float4 x = __ldg(reinterpret_cast<const float4*>(src) + i);
            float4* d = reinterpret_cast<float4*>(S + r * SST + 4 * c4);
            d[0] = make_float4(x.x, tf32_rem(x.x), x.y, tf32_rem(x.y));
            d[1] = make_float4(x.z, tf32_rem(x.z), x.w, tf32_rem(x.w));
        }
    }
    stage_chunk(p, smem, 0, 0, b, h, hk, row0);

    for (int c = 0; c < n_chunks; ++c) {
        const int buf = c & 1;
        const int t0 = c * T;
        const int Tc = min(T, p.N - t0);
        if (c + 1 < n_chunks) {
            stage_chunk(p, smem, buf ^ 1, c + 1, b, h, hk, row0);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        const __nv_bfloat16* K = reinterpret_cast<const __nv_bfloat16*>(smem + kOffK + buf * kKQBytes);
        const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(smem + kOffQ + buf * kKQBytes);
        const __nv_bfloat16* V = reinterpret_cast<const __nv_bfloat16*>(smem + kOffV + buf * kVBytes);
        const float* gch = reinterpret_cast<const float*>(smem + kOffGB) + buf * 2 * T;
        const float* bch = gch + T;

        // 1. decays: a_t, Gamma_t = a_0 ... a_t, R[t][i] = a_{i+1} ... a_t for
        //    i <= t, r_i = R[T-1][i].  Row t by 4 threads, thread s covering
        //    i in [16 s, 16 s + 15]: a suffix product within its quarter
        //    times the products of the later quarters up to t.
        float* rvec = const_cast<float*>(gch);  // g is dead once a is known
        if (tid < T)
            Av[tid] = tid < Tc ? expf(gch[tid]) : 1.f;
        __syncthreads();
        {
            const int t = tid >> 2, q = tid & 3;
            const int lo = 16 * q, hi = min(16 * q + 15, t);
            float loc[16];
            float run = 1.f;
#pragma unroll
            for (int m = 15; m >= 0; --m) {
                // loc[m] = prod of a_j, j in (lo + m, hi]
                loc[m] = run;
                if (lo + m <= hi)
                    run = __fmul_rn(run, Av[lo + m]);
            }
            // run = prod of a_j, j in [lo, hi] (1 for a quarter past t)
            float tail = __shfl_down_sync(0xffffffffu, run, 1);  // quarters q + 1 ..
            const float t2 = __shfl_down_sync(0xffffffffu, tail, 1);
            const float t3 = __shfl_down_sync(0xffffffffu, t2, 1);
            tail = q == 3 ? 1.f : (q == 2 ? tail : (q == 1 ? __fmul_rn(tail, t2) : __fmul_rn(__fmul_rn(tail, t2), t3)));
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const int i = lo + m;
                if (i <= t) {
                    const float r = __fmul_rn(loc[m], tail);
                    Rm[t * MST + i] = r;
                    if (t == T - 1)
                        rvec[i] = r;
                    if (i == 0)
                        Gam[t] = __fmul_rn(r, Av[0]);
                }
            }
        }
        __syncthreads();

        // 2. K K^T and Q K^T (bf16, exact operands): this warp's 16 rows x 32
        //    columns of each; then L = beta (K K^T o R) below the diagonal and
        //    M = Q K^T o R on and below it
        {
            const int cb = (warp >> 2) * 32;
            float ck[4][4] = {}, cq[4][4] = {};
#pragma unroll
            for (int ks = 0; ks < DK; ks += 16) {
                const uint32_t ka0 = ld32(K + (rb + g8) * KST + ks + 2 * t4);
                const uint32_t ka1 = ld32(K + (rb + g8 + 8) * KST + ks + 2 * t4);
                const uint32_t ka2 = ld32(K + (rb + g8) * KST + ks + 2 * t4 + 8);
                const uint32_t ka3 = ld32(K + (rb + g8 + 8) * KST + ks + 2 * t4 + 8);
                const uint32_t qa0 = ld32(Q + (rb + g8) * KST + ks + 2 * t4);
                const uint32_t qa1 = ld32(Q + (rb + g8 + 8) * KST + ks + 2 * t4);
                const uint32_t qa2 = ld32(Q + (rb + g8) * KST + ks + 2 * t4 + 8);
                const uint32_t qa3 = ld32(Q + (rb + g8 + 8) * KST + ks + 2 * t4 + 8);
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    const int n = cb + nt * 8 + g8;
                    const uint32_t b0 = ld32(K + n * KST + ks + 2 * t4);
                    const uint32_t b1 = ld32(K + n * KST + ks + 2 * t4 + 8);
                    mma_bf16(ck[nt], ka0, ka1, ka2, ka3, b0, b1);
                    mma_bf16(cq[nt], qa0, qa1, qa2, qa3, b0, b1);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = rb + g8 + (e >> 1) * 8;
                    const int i = cb + nt * 8 + 2 * t4 + (e & 1);
                    const float rr = i <= t ? Rm[t * MST + i] : 0.f;
                    Lp[t * MST + i] = i < t ? __fmul_rn(bch[t], __fmul_rn(ck[nt][e], rr)) : 0.f;
                    Mq[t * MST + i] = __fmul_rn(cq[nt][e], rr);
                }
            }
        }

        // 3. P = beta (V - Gamma (K S^T)), and Q S^T for step 5 (kept in
        //    registers): this warp's 16 tokens x 32 of the 64 rows; K and Q
        //    exact in tf32, S split (the two products share its fragments)
        float qs[4][4] = {};
        {
            const int cb = (warp >> 2) * 32;
            float acc[4][4] = {};
#pragma unroll 2
            for (int ks = 0; ks < DK; ks += 8) {
                const uint32_t a0 = bf2tf(K + (rb + g8) * KST + ks + t4);
                const uint32_t a1 = bf2tf(K + (rb + g8 + 8) * KST + ks + t4);
                const uint32_t a2 = bf2tf(K + (rb + g8) * KST + ks + t4 + 4);
                const uint32_t a3 = bf2tf(K + (rb + g8 + 8) * KST + ks + t4 + 4);
                const uint32_t e0 = bf2tf(Q + (rb + g8) * KST + ks + t4);
                const uint32_t e1 = bf2tf(Q + (rb + g8 + 8) * KST + ks + t4);
                const uint32_t e2 = bf2tf(Q + (rb + g8) * KST + ks + t4 + 4);
                const uint32_t e3 = bf2tf(Q + (rb + g8 + 8) * KST + ks + t4 + 4);
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    const int n = cb + nt * 8 + g8;  // state row (d_v index)
                    const float2 s0 = S[n * SST + ks + t4], s1 = S[n * SST + ks + t4 + 4];
                    const uint32_t h0 = f2tf32(s0.x), l0 = __float_as_uint(s0.y);
                    const uint32_t h1 = f2tf32(s1.x), l1 = __float_as_uint(s1.y);
                    mma_tf32(acc[nt], a0, a1, a2, a3, h0, h1);
                    mma_tf32(acc[nt], a0, a1, a2, a3, l0, l1);
                    mma_tf32(qs[nt], e0, e1, e2, e3, h0, h1);
                    mma_tf32(qs[nt], e0, e1, e2, e3, l0, l1);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = rb + g8 + (e >> 1) * 8;
                    const int col = cb + nt * 8 + 2 * t4 + (e & 1);
                    const float vv = bf2f(V + t * VST + col);
                    U[t * MST + col] = __fmul_rn(bch[t], __fsub_rn(vv, __fmul_rn(Gam[t], acc[nt][e])));
                }
            }
        }
        __syncthreads();

        // 4. (I + L) U = P in blocks of 16 rows.  (a) the inverses D_b of the
        //    four unit lower triangular diagonal blocks, one column per
        //    thread; (b) per block b: X = P_b - L_{b,<b} U_{<b}, then
        //    U_b = D_b X, one row and 4 columns per thread.  D lives in this
        //    chunk's V buffer (dead after step 3).
        {
            float* D = reinterpret_cast<float*>(smem + kOffV + buf * kVBytes);  // [4][16][16]
            if (tid < T) {
                const int blk = tid >> 4, j = tid & 15;
                const float* Lb = Lp + (16 * blk) * MST + 16 * blk;
                float d[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float acc = 0.f;
#pragma unroll
                    for (int k = 0; k < i; ++k)
                        acc = __fmaf_rn(Lb[i * MST + k], k >= j ? d[k] : 0.f, acc);
                    d[i] = i < j ? 0.f : (i == j ? 1.f : -acc);
                    D[(blk * 16 + i) * 16 + j] = d[i];
                }
            }
            __syncthreads();
            const int r = tid >> 4, c0 = 4 * (tid & 15);  // a row of the block, 4 columns
#pragma unroll 1
            for (int blk = 0; blk < 4; ++blk) {
                const int row = 16 * blk + r;
                float4 x = *reinterpret_cast<const float4*>(U + row * MST + c0);
                for (int k0 = 0; k0 < 16 * blk; k0 += 16) {
#pragma unroll
                    for (int kk = 0; kk < 16; ++kk) {
                        const float l = Lp[row * MST + k0 + kk];
                        const float4 u = *reinterpret_cast<const float4*>(U + (k0 + kk) * MST + c0);
                        x.x = __fmaf_rn(-l, u.x, x.x);
                        x.y = __fmaf_rn(-l, u.y, x.y);
                        x.z = __fmaf_rn(-l, u.z, x.z);
                        x.w = __fmaf_rn(-l, u.w, x.w);
                    }
                }
                *reinterpret_cast<float4*>(U + row * MST + c0) = x;
                __syncthreads();
                float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
                const float* Dr = D + (blk * 16 + r) * 16;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    if (i <= r) {
                        const float dd = Dr[i];
                        const float4 xi = *reinterpret_cast<const float4*>(U + (16 * blk + i) * MST + c0);
                        y.x = __fmaf_rn(dd, xi.x, y.x);
                        y.y = __fmaf_rn(dd, xi.y, y.y);
                        y.z = __fmaf_rn(dd, xi.z, y.z);
                        y.w = __fmaf_rn(dd, xi.w, y.w);
                    }
                }
                __syncthreads();
                *reinterpret_cast<float4*>(U + row * MST + c0) = y;
                __syncthreads();
            }
        }

        // 5. O = scale (Gamma (Q S^T) + M U): 16 tokens x 32 rows per warp
        {
            const int cb = (warp >> 2) * 32;
            float mu[4][4] = {};
#pragma unroll 2
            for (int ks = 0; ks < T; ks += 8) {
                uint32_t ah[4], al[4];
                split(Mq[(rb + g8) * MST + ks + t4], ah[0], al[0]);
                split(Mq[(rb + g8 + 8) * MST + ks + t4], ah[1], al[1]);
                split(Mq[(rb + g8) * MST + ks + t4 + 4], ah[2], al[2]);
                split(Mq[(rb + g8 + 8) * MST + ks + t4 + 4], ah[3], al[3]);
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    const int n = cb + nt * 8 + g8;
                    uint32_t h0, l0, h1, l1;
                    split(U[(ks + t4) * MST + n], h0, l0);
                    split(U[(ks + t4 + 4) * MST + n], h1, l1);
                    mma_tf32(mu[nt], ah[0], ah[1], ah[2], ah[3], h0, h1);
                    mma_tf32(mu[nt], ah[0], ah[1], ah[2], ah[3], l0, l1);
                    mma_tf32(mu[nt], al[0], al[1], al[2], al[3], h0, h1);
                }
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = rb + g8 + (e >> 1) * 8;
                    const int col = cb + nt * 8 + 2 * t4 + (e & 1);
                    if (t < Tc) {
                        const float o = __fmul_rn(p.scale, __fmaf_rn(Gam[t], qs[nt][e], mu[nt][e]));
                        p.out[(((size_t)b * p.N + t0 + t) * p.Hv + h) * p.dv + row0 + col] = o;
                    }
                }
            }
        }

        // 6. S <- Gamma_{T-1} S + U^T diag(r) K, r_i = R[T-1][i]: this warp's
        //    16 rows of S x 64 of its columns
        {
            const int nb = (warp >> 2) * 64;
            const float gT = Gam[T - 1];
            float acc[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int m = rb + g8 + (e >> 1) * 8;
                    const int n = nb + nt * 8 + 2 * t4 + (e & 1);
                    acc[nt][e] = __fmul_rn(gT, S[m * SST + n].x);
                }
            }
#pragma unroll 2
            for (int ks = 0; ks < T; ks += 8) {
                // A[m][k] = r_k U[k][m] (split); B = K, exact in tf32
                const float r0 = rvec[ks + t4], r1 = rvec[ks + t4 + 4];
                uint32_t ah[4], al[4];
                split(__fmul_rn(r0, U[(ks + t4) * MST + rb + g8]), ah[0], al[0]);
                split(__fmul_rn(r0, U[(ks + t4) * MST + rb + g8 + 8]), ah[1], al[1]);
                split(__fmul_rn(r1, U[(ks + t4 + 4) * MST + rb + g8]), ah[2], al[2]);
                split(__fmul_rn(r1, U[(ks + t4 + 4) * MST + rb + g8 + 8]), ah[3], al[3]);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    const int n = nb + nt * 8 + g8;
                    const uint32_t b0 = bf2tf(K + (ks + t4) * KST + n);
                    const uint32_t b1 = bf2tf(K + (ks + t4 + 4) * KST + n);
                    mma_tf32(acc[nt], ah[0], ah[1], ah[2], ah[3], b0, b1);
                    mma_tf32(acc[nt], al[0], al[1], al[2], al[3], b0, b1);
                }
            }
            __syncthreads();  // every warp is done reading S (steps 3, 5) and U
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int m = rb + g8 + (e >> 1) * 8;
                    const int n = nb + nt * 8 + 2 * t4 + (e & 1);
                    S[m * SST + n] = make_float2(acc[nt][e], tf32_rem(acc[nt][e]));
                }
            }
        }
        __syncthreads();
    }

    // the last state -> node_states[b][0][h][row0 ..][:]
    const size_t base = (((size_t)b * p.Hv + h) * p.dv + row0) * DK;
    for (int i = tid; i < TV * DK / 4; i += kThreads) {
        const int r = i / (DK / 4), c4 = i % (DK / 4);
        const float4 s01 = *reinterpret_cast<const float4*>(S + r * SST + 4 * c4);
        const float4 s23 = *reinterpret_cast<const float4*>(S + r * SST + 4 * c4 + 2);
        const float4 x = make_float4(s01.x, s01.z, s23.x, s23.z);
        if (p.state_f16) {
            const __half2 lo = __float22half2_rn(make_float2(x.x, x.y));
            const __half2 hi = __float22half2_rn(make_float2(x.z, x.w));
            uint2 u;
            u.x = *reinterpret_cast<const uint32_t*>(&lo);
            u.y = *reinterpret_cast<const uint32_t*>(&hi);
            reinterpret_cast<uint2*>(static_cast<__half*>(p.node_states) + base)[i] = u;
        } else {
            reinterpret_cast<float4*>(static_cast<float*>(p.node_states) + base)[i] = x;
        }
    }
}

}  // namespace
}  // namespace chunked

bool chunked_supported(const VerifyArgs& a)
{
    return a.qkv_dtype == GDN_BF16 && a.d_k == chunked::DK && a.d_v % chunked::TV == 0 &&
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
    dim3 grid(a.d_v / TV, a.n_v_heads, a.batch);
    return launch_pdl(gdn_chain_chunked, grid, dim3(kThreads), (size_t)kSmem, stream, p);
}

}  // namespace gdn
