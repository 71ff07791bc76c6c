// IF4 code decoding shared by the dequantizers and the fused-decode linear:
// the value of every 4-bit code from a 32-entry shared-memory table, read
// with one conflict-free load per element (sm_100a).
#pragma once

#include <cstdint>

#include "if4_device.cuh"
#include "if4_encode.cuh"

namespace {

using namespace if4dev;

// Decoded value of every code: lut[n] is the FP4 value of nibble n,
// lut[16 + n] the INT4 value fl(6k/7) of nibble n (k its sign extension).
// 32 floats, one per shared-memory bank, so any pattern of lookups by a warp
// is conflict-free.
__device__ __forceinline__ float code_value(uint32_t i)
{
    if (i < 16) {
        const uint32_t h = f16x2_from_e2m1x2(i);      // nibble in bits 0-3
        return f16lo_to_f32(h);
    }
    const float k = (float)((int)((i - 16) ^ 8u) - 8);
    return __fmul_rn(k, c67());
}

__device__ __forceinline__ float lds_f32(uint32_t addr)
{
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

// 8 decoded values (not yet scaled) of the 8 nibbles of w; base is the
// shared address of lut or lut + 16 floats.
__device__ __forceinline__ void decode_word(uint32_t w, uint32_t base, float (&q)[8])
{
    q[0] = lds_f32(base + ((w << 2) & 0x3Cu));
#pragma unroll
    for (int i = 1; i < 8; ++i) q[i] = lds_f32(base + ((w >> (4 * i - 2)) & 0x3Cu));
}

// ------------------------------------- byte-permute decode (16-bit out) --
// A group's 16-bit outputs without a table load per element.  The group's
// eight magnitudes are rounded once, t[m] = out(fl32(base[m] * eff)) with
// base = lut (FP4, m = 0..7) or lut + 16 (INT4, k = 0..7), exactly as the
// per-element path rounds them, and split into a low-byte and a high-byte
// plane of 8 bytes (two registers each).  Each element's magnitude index
// (FP4: n & 7; INT4, two's complement: n & 7 below 8, 8 - (n & 7) above) is
// formed for eight nibbles at once; prmt picks four elements' bytes from each
// plane; a prmt of the word and the word shifted by 4 puts each element's
// sign (bit 3 of its nibble) at bit 7 of its high byte, and a last prmt
// interleaves the planes into 16-bit pairs.  Rounding to nearest is symmetric
// in sign, so the sign bit on t[m] is the rounded negative value whenever
// eff is finite with its sign bit clear (the callers take the per-element
// path otherwise).  INT4 code 8 (k = -8, never emitted by the encoder) has
// index 8, which the planes cannot hold; it shows as bit 3 of the index and
// the callers decode such a group per element.

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ void lds_f32x4(uint32_t addr, float *v)
{
    asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]) : "r"(addr));
}

struct BytePlanes {
    uint32_t lo0, lo1, hi0, hi1;   // low / high bytes of t[0..3], t[4..7]
};

// base: shared address of the group's 8 magnitudes (16-byte aligned)
template <bool BF16>
__device__ __forceinline__ BytePlanes group_planes(uint32_t base, float eff)
{
    float b[8];
    lds_f32x4(base, b);
    lds_f32x4(base + 16u, b + 4);
    const f2_t E = f2_pack(eff, eff);
    uint32_t p[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float lo, hi;
        f2_unpack(f2_mul(f2_pack(b[2 * j], b[2 * j + 1]), E), lo, hi);
        p[j] = BF16 ? bf16x2_from_f32(lo, hi) : f16x2_from_f32(lo, hi);
    }
    return {prmt(p[0], p[1], 0x6420u), prmt(p[2], p[3], 0x6420u),
            prmt(p[0], p[1], 0x7531u), prmt(p[2], p[3], 0x7531u)};
}

// The 8 elements of code word w as four 16-bit pairs o[0..3] (element 2j in
// the low half of o[j]); im is all ones for an INT4 group, zero for FP4.
// Returns nonzero when an INT4 element holds code 8 (o is then not valid).
__device__ __forceinline__ uint32_t decode_word16(uint32_t w, uint32_t im, const BytePlanes &P,
                                                 uint32_t *o)
{
    const uint32_t s = (w >> 3) & 0x11111111u;          // sign bit of each nibble
    const uint32_t mag = ((w & 0x77777777u) ^ ((s * 7u) & im)) + (s & im);
    const uint32_t w4 = w << 4;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t sel = h ? mag >> 16 : mag;       // prmt reads the low 16 bits
        const uint32_t lo4 = prmt(P.lo0, P.lo1, sel);
        const uint32_t sg = prmt(w4, w, h ? 0x7362u : 0x5140u) & 0x80808080u;
        const uint32_t hi4 = prmt(P.hi0, P.hi1, sel) | sg;
        o[2 * h] = prmt(lo4, hi4, 0x5140u);
        o[2 * h + 1] = prmt(lo4, hi4, 0x7362u);
    }
    return mag & 0x88888888u;
}

// Whether the permute decode applies for this eff: finite, sign bit clear.
__device__ __forceinline__ bool permute_decode_ok(float eff)
{
    return __float_as_uint(eff) < 0x7F800000u;
}

}  // namespace
