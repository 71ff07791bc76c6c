// Device helpers for the IF4 kernels (sm_100a).  Thin wrappers over PTX
// instructions; no IF4 policy lives here.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace if4dev {

// ------------------------------------------------------------ memory ----

// 256-bit read-only load, not kept in L1 (every byte is read once).
__device__ __forceinline__ void ld_nc_v8(const void *p, uint32_t (&r)[8])
{
    asm("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]),
          "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
        : "l"(p));
}

__device__ __forceinline__ void ld_nc_v4(const void *p, uint32_t &a, uint32_t &b,
                                         uint32_t &c, uint32_t &d)
{
    asm("ld.global.nc.L1::no_allocate.v4.b32 {%0,%1,%2,%3}, [%4];"
        : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "l"(p));
}

__device__ __forceinline__ void ld_nc_v2(const void *p, uint32_t &a, uint32_t &b)
{
    asm("ld.global.nc.L1::no_allocate.v2.b32 {%0,%1}, [%2];" : "=r"(a), "=r"(b) : "l"(p));
}

__device__ __forceinline__ uint32_t ld_nc_u32(const void *p)
{
    uint32_t v;
    asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_nc_u16(const void *p)
{
    uint16_t v;
    asm("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_nc_u8(const void *p)
{
    uint16_t v;
    asm("ld.global.nc.L1::no_allocate.u8 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// --------------------------------------------- L2 eviction priority ----
// A cache policy (createpolicy) passed with a load or store sets the L2
// eviction priority of the lines it touches: evict_first lines are replaced
// before normal ones, evict_last lines after them.

__device__ __forceinline__ uint64_t l2_evict_first()
{
    uint64_t p;
    asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_evict_normal()
{
    uint64_t p;
    asm("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_evict_last()
{
    uint64_t p;
    asm("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void ld_nc_v8_pol(const void *p, uint32_t (&r)[8], uint64_t pol)
{
    asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8], %9;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]),
          "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
        : "l"(p), "l"(pol));
}

__device__ __forceinline__ void ld_nc_v4_pol(const void *p, uint32_t &a, uint32_t &b, uint32_t &c,
                                             uint32_t &d, uint64_t pol)
{
    asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.b32 {%0,%1,%2,%3}, [%4], %5;"
        : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "l"(p), "l"(pol));
}

__device__ __forceinline__ void st_v8_pol(void *p, const uint32_t (&r)[8], uint64_t pol)
{
    asm volatile("st.global.L1::no_allocate.L2::cache_hint.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8}, %9;"
                 :: "l"(p), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]),
                    "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "l"(pol) : "memory");
}

__device__ __forceinline__ void st_v4_pol(void *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                          uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1,%2,%3,%4}, %5;"
                 :: "l"(p), "r"(a), "r"(b), "r"(c), "r"(d), "l"(pol) : "memory");
}

__device__ __forceinline__ void st_v2_pol(void *p, uint32_t a, uint32_t b, uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.v2.b32 [%0], {%1,%2}, %3;"
                 :: "l"(p), "r"(a), "r"(b), "l"(pol) : "memory");
}

__device__ __forceinline__ void st_u8_pol(void *p, uint32_t v, uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.u8 [%0], %1, %2;"
                 :: "l"(p), "h"((uint16_t)v), "l"(pol) : "memory");
}

__device__ __forceinline__ void st_v8(void *p, const uint32_t (&r)[8])
{
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                 :: "l"(p), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]),
                    "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]) : "memory");
}

__device__ __forceinline__ void st_v4(void *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};"
                 :: "l"(p), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void st_v2(void *p, uint32_t a, uint32_t b)
{
    asm volatile("st.global.v2.b32 [%0], {%1,%2};" :: "l"(p), "r"(a), "r"(b) : "memory");
}

__device__ __forceinline__ void st_u8(void *p, uint32_t v)
{
    asm volatile("st.global.u8 [%0], %1;" :: "l"(p), "h"((uint16_t)v) : "memory");
}

// ----------------------------------------------------- packed fp32 pairs --
// sm_100 executes these as one instruction on a 64-bit register pair.

typedef unsigned long long f2_t;

__device__ __forceinline__ f2_t f2_pack(float lo, float hi)
{
    f2_t r;
    asm("mov.b64 %0, {%1,%2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void f2_unpack(f2_t v, float &lo, float &hi)
{
    asm("mov.b64 {%0,%1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ f2_t f2_mul(f2_t a, f2_t b)
{
    f2_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ f2_t f2_add(f2_t a, f2_t b)
{
    f2_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ f2_t f2_sub(f2_t a, f2_t b)
{
    f2_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ f2_t f2_fma(f2_t a, f2_t b, f2_t c)
{
    f2_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// ------------------------------------------------------- conversions ----

// Two floats -> one byte of two E2M1 codes (lo -> bits 0-3, hi -> bits 4-7),
// round-to-nearest-even, saturating to +-6.
__device__ __forceinline__ uint32_t e2m1x2_from_f32(float lo, float hi)
{
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\t"
        "cvt.u32.u8 %0, t;\n\t}"
        : "=r"(r) : "f"(lo), "f"(hi));
    return r;
}

// One byte of two E2M1 codes -> f16x2 (bits 0-3 -> low half).
__device__ __forceinline__ uint32_t f16x2_from_e2m1x2(uint32_t byte)
{
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.u8.u32 t, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(r) : "r"(byte));
    return r;
}

// float -> E4M3 code, round-to-nearest-even, saturating to 448 (0x7E).
__device__ __forceinline__ uint32_t e4m3_from_f32(float f)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(f));
    return r & 0xFFu;
}

// E4M3 code (bits 0-6) -> float, exact (every E4M3 value is an f16 value).
__device__ __forceinline__ float f32_from_e4m3(uint32_t code)
{
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)(code & 0x7Fu)));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

__device__ __forceinline__ float f16lo_to_f32(uint32_t h2)
{
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

__device__ __forceinline__ float f16hi_to_f32(uint32_t h2)
{
    return __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
}

// two floats -> bf16x2 / f16x2, round-to-nearest-even (lo in bits 0-15)
__device__ __forceinline__ uint32_t bf16x2_from_f32(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ uint32_t f16x2_from_f32(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(lo), "f"(hi));
    return r;
}

// The two bf16 halves of w as an exact float pair (low half first).
__device__ __forceinline__ unsigned long long f2_from_bf16x2(uint32_t w)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(w << 16), "r"(w & 0xFFFF0000u));
    return r;
}

// Programmatic dependent launch, at the top of a kernel: the next kernel in
// the stream may be scheduled from now on (its blocks wait in the same
// call), then wait until every earlier kernel this one depends on has
// finished and its memory is visible.  The wait is a no-op when the kernel
// was launched without the programmatic-serialization attribute.
__device__ __forceinline__ void pdl_enter()
{
    asm volatile("griddepcontrol.launch_dependents;\n\tgriddepcontrol.wait;" ::: "memory");
}

// Let the next kernel in the stream be scheduled (it still waits for this
// one to finish before reading anything).
__device__ __forceinline__ void pdl_release()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Wall clock in nanoseconds, for bounded waits.
__device__ __forceinline__ unsigned long long globaltimer_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ----------------------------------------------------------- integers ----

__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// per 16-bit lane: max(|a|, |b|) with NaN propagated; the result's sign bit
// is sign(a) ^ sign(b) and must be masked off by the caller
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ uint32_t absmax_f16x2(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("max.NaN.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// max(|a|, |b|) as float bits with NaN propagated; the result's sign bit is
// sign(a) ^ sign(b) and must be masked off by the caller
__device__ __forceinline__ uint32_t absmax_f32(uint32_t a, float b)
{
    uint32_t r;
    asm("max.NaN.xorsign.abs.f32 %0, %1, %2;" : "=r"(r) : "r"(a), "f"(b));
    return r;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

}  // namespace if4dev
