// Device helpers for libgdntree kernels (sm_100a): shared-memory barriers
// with bounded waits, exact bf16 widening, status reporting.
#pragma once

#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace gdn {

__device__ __forceinline__ uint32_t smem_addr(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier (shared::cta) -------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_init_fence()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Arrive with release semantics: this thread's earlier shared/global accesses
// happen before any thread that observes the phase flip.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// As mbar_try_wait, but the hardware may suspend the thread for up to
// `hint_ns` nanoseconds waiting for the phase, instead of returning at once,
// so a waiting warp issues no instructions.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t* bar, uint32_t parity,
                                                      uint32_t hint_ns)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return done != 0;
}

// Wait for the phase with the given parity to complete.  Bounded: gives up
// after ~2^32 SM cycles (about two seconds at B200 clocks) and returns false,
// so a logic error can never hang the GPU.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const long long t0 = clock64();
    while (!mbar_try_wait_suspend(bar, parity, 200000u)) {
        if (clock64() - t0 > (1ll << 32))
            return false;
    }
    return true;
}

// ---- tensor memory (TMEM) ----------------------------------------------------

// Allocates ncols columns (a power of two, 32..512) of this CTA's tensor
// memory and writes their address to *dst (shared memory).  One full warp
// calls it; the CTA then gives up its right to allocate more.  Tensor memory
// allocated by a CTA must be freed (tmem_free) before the CTA exits.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_free(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Orders tensor-memory accesses around a CTA barrier.
__device__ __forceinline__ void tmem_fence_before_sync()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_fence_after_sync()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 consecutive 32-bit columns of this thread's lane, starting at taddr
// (the warp's lane quarter in bits 31..16, the column in bits 15..0): one
// warp-wide store or load.  A load first waits for this thread's earlier
// stores, then for itself.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---- programmatic dependent launch -------------------------------------------

// Kernels are launched with programmatic stream serialization: the next
// kernel in the stream may become resident before this one finishes.  Every
// kernel first waits for the grid it depends on to complete (and its memory
// to be visible) before touching global memory, then lets its own dependents
// launch.  Without the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_wait_then_release()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// A hint that the 128-byte line holding p should be brought into L2.
__device__ __forceinline__ void prefetch_l2(const void* p)
{
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// ---- 256-bit global accesses ---------------------------------------------------

// 8 floats at a 32-byte-aligned global address in one access.  The load is a
// plain (coherent) load, so it sees this thread's earlier stores.
__device__ __forceinline__ void ld_global_v8(const float* p, float4& lo, float4& hi)
{
    asm volatile("ld.global.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=f"(lo.x), "=f"(lo.y), "=f"(lo.z), "=f"(lo.w), "=f"(hi.x), "=f"(hi.y), "=f"(hi.z),
                   "=f"(hi.w)
                 : "l"(p)
                 : "memory");
}

__device__ __forceinline__ void st_global_v8(float* p, float4 lo, float4 hi)
{
    asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "f"(lo.x), "f"(lo.y),
                 "f"(lo.z), "f"(lo.w), "f"(hi.x), "f"(hi.y), "f"(hi.z), "f"(hi.w)
                 : "memory");
}

// ---- status -----------------------------------------------------------------

__device__ __forceinline__ void report_status(int32_t* status, int32_t code)
{
    if (status != nullptr)
        atomicCAS(status, 0, code);
}

// ---- conversions ------------------------------------------------------------

// Two packed bf16 (low half = first element) widened exactly to f32.
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t x)
{
    return make_float2(__uint_as_float(x << 16), __uint_as_float(x & 0xffff0000u));
}

// 16 bytes of inputs widened to f32: 8 values for bf16, 4 for f32.
template <typename QT>
struct Widen;

template <>
struct Widen<__nv_bfloat16> {
    static constexpr int kPerChunk = 8;
    __device__ __forceinline__ static void store(float* dst, uint4 x)
    {
        const float2 a = bf16x2_to_float2(x.x), b = bf16x2_to_float2(x.y);
        const float2 c = bf16x2_to_float2(x.z), d = bf16x2_to_float2(x.w);
        reinterpret_cast<float4*>(dst)[0] = make_float4(a.x, a.y, b.x, b.y);
        reinterpret_cast<float4*>(dst)[1] = make_float4(c.x, c.y, d.x, d.y);
    }
    // 4 consecutive elements starting at p (8-byte aligned).
    __device__ __forceinline__ static float4 load4(const __nv_bfloat16* p)
    {
        const uint2 x = __ldg(reinterpret_cast<const uint2*>(p));
        const float2 a = bf16x2_to_float2(x.x), b = bf16x2_to_float2(x.y);
        return make_float4(a.x, a.y, b.x, b.y);
    }
    __device__ __forceinline__ static float load1(const __nv_bfloat16* p)
    {
        const unsigned short u = __ldg(reinterpret_cast<const unsigned short*>(p));
        return __uint_as_float(static_cast<uint32_t>(u) << 16);
    }
    // Same, from shared memory.
    __device__ __forceinline__ static float4 lds4(const __nv_bfloat16* p)
    {
        const uint2 x = *reinterpret_cast<const uint2*>(p);
        const float2 a = bf16x2_to_float2(x.x), b = bf16x2_to_float2(x.y);
        return make_float4(a.x, a.y, b.x, b.y);
    }
    __device__ __forceinline__ static float lds1(const __nv_bfloat16* p)
    {
        const unsigned short u = *reinterpret_cast<const unsigned short*>(p);
        return __uint_as_float(static_cast<uint32_t>(u) << 16);
    }
    // 8 consecutive elements starting at p (16-byte aligned) as 4 pairs, from
    // shared memory (lds8) or global memory (ldg8).
    __device__ __forceinline__ static void pairs(uint4 u, float2 (&x)[4])
    {
        x[0] = bf16x2_to_float2(u.x);
        x[1] = bf16x2_to_float2(u.y);
        x[2] = bf16x2_to_float2(u.z);
        x[3] = bf16x2_to_float2(u.w);
    }
    __device__ __forceinline__ static void lds8(const __nv_bfloat16* p, float2 (&x)[4])
    {
        pairs(*reinterpret_cast<const uint4*>(p), x);
    }
    __device__ __forceinline__ static void ldg8(const __nv_bfloat16* p, float2 (&x)[4])
    {
        pairs(__ldg(reinterpret_cast<const uint4*>(p)), x);
    }
};

template <>
struct Widen<float> {
    static constexpr int kPerChunk = 4;
    __device__ __forceinline__ static void store(float* dst, uint4 x)
    {
        reinterpret_cast<uint4*>(dst)[0] = x;
    }
    __device__ __forceinline__ static float4 load4(const float* p)
    {
        return __ldg(reinterpret_cast<const float4*>(p));
    }
    __device__ __forceinline__ static float load1(const float* p) { return __ldg(p); }
    __device__ __forceinline__ static float4 lds4(const float* p)
    {
        return *reinterpret_cast<const float4*>(p);
    }
    __device__ __forceinline__ static float lds1(const float* p) { return *p; }
    __device__ __forceinline__ static void pairs(float4 a, float4 b, float2 (&x)[4])
    {
        x[0] = make_float2(a.x, a.y);
        x[1] = make_float2(a.z, a.w);
        x[2] = make_float2(b.x, b.y);
        x[3] = make_float2(b.z, b.w);
    }
    __device__ __forceinline__ static void lds8(const float* p, float2 (&x)[4])
    {
        pairs(reinterpret_cast<const float4*>(p)[0], reinterpret_cast<const float4*>(p)[1], x);
    }
    __device__ __forceinline__ static void ldg8(const float* p, float2 (&x)[4])
    {
        pairs(__ldg(reinterpret_cast<const float4*>(p)), __ldg(reinterpret_cast<const float4*>(p) + 1), x);
    }
};

}  // namespace gdn
