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
