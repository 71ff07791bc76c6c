// IF6 and IF3: the adaptive FP/INT choice of IF4 at 6 and 3 bits, on B200
// (sm_100a), and their C ABI.
//
// "Adaptive Block-Scaled Data Types" applies the IF4 idea to other bit widths
// and names IF3 and IF6 (abstract; companion "It Generalizes: IF3 and IF6";
// gist.science section 2 "Extensoes") without printing either grid.  The
// readings this file implements, the same as the CPU oracle's:
//   IF6: FP6 = E2M3 (largest 7.5) against INT6 k in [-31, 31] decoded as
//        fl(15k/62) and chosen as RNE(v * fl(62/15)); both grids reach 7.5.
//   IF3: FP3 = E2M0, magnitudes 0, 1, 2, 4, against INT3 k in [-3, 3] decoded
//        as fl(4k/3) and chosen as RNE(v * 3/4); both reach 4.
// Everything else follows IF4: block scale E4M3 of (amax/fpmax)/ts, tensor
// scale amax_T/(fpmax*448), v = x * fl(1/fl(E4M3*ts)), the lower squared
// error in the scaled domain wins with ties to FP, bit 7 of the scale byte
// marks INT, an FP zero keeps the sign of v, INT codes are two's complement,
// and element i's code sits at bits [w*i, w*i + w) of the group's
// little-endian code bytes (12 per group for IF6, 6 for IF3).
//
// Design: one thread per group of 16 in a grid-stride loop, element pairs in
// paired binary32 instructions.  FP6 codes come from the hardware E2M3
// conversion (round to nearest even, saturating), FP3 codes from three
// comparisons that give 1.0 or 0.0, summed and packed by exact FMAs; the INT
// integer from one fused multiply-add (a single rounding of the exact
// product).  The decision takes IF4's fast path: the two error sums in
// binary32, and the binary64 rule itself (its INT values the correctly
// rounded quotients, from a shared table) only for a group whose binary32
// margin is within the band; IF3 first tests its codes for an exact tie.

#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/if4.h"
#include "if4_device.cuh"

using namespace if4dev;

namespace {

enum { W_IF = IF4_W_ADAPTIVE, W_FP = IF4_W_FP_ONLY, W_INT = IF4_W_INT_ONLY };

template <int BITS>
struct Width;

template <>
struct Width<6> {
    static constexpr float fpmax = 7.5f;
    static constexpr int kmax = 31;
    static constexpr int code_bytes = 12;
};

template <>
struct Width<3> {
    static constexpr float fpmax = 4.0f;
    static constexpr int kmax = 3;
    static constexpr int code_bytes = 6;
};

constexpr float kMagic = 12582912.0f;           // 1.5 * 2^23

// FP code of v: sign in the top bit of the width, magnitude code below.
template <int BITS>
__device__ __forceinline__ uint32_t fp_code(float v)
{
    const float a = fabsf(v);
    uint32_t c;
    if constexpr (BITS == 6) {
        // E2M3: steps of 1/8 below 2, 1/4 below 4, 1/2 up to 7.5; the
        // scalings by 8, 4 and 2 are exact, __float2int_rn is RNE
        if (!(a <= 7.5f)) c = 31u;
        else if (a < 2.0f) c = (uint32_t)__float2int_rn(__fmul_rn(a, 8.0f));
        else if (a < 4.0f) c = (uint32_t)__float2int_rn(__fmul_rn(a, 4.0f)) + 8u;
        else c = (uint32_t)__float2int_rn(__fmul_rn(a, 2.0f)) + 16u;
        return c | (signbit(v) ? 0x20u : 0u);
    } else {
        // E2M0: 0, 1, 2, 4; ties to the even code (0.5 -> 0, 1.5 -> 2, 3 -> 2)
        if (!(a <= 3.0f)) c = 3u;
        else if (a >= 1.5f) c = 2u;
        else if (a > 0.5f) c = 1u;
        else c = 0u;
        return c | (signbit(v) ? 4u : 0u);
    }
}

// FP value of a code (exact in binary32).
template <int BITS>
__device__ __forceinline__ float fp_value(uint32_t code)
{
    float mag;
    if constexpr (BITS == 6) {
        const uint32_t e = (code >> 3) & 3u, m = code & 7u;
        mag = e == 0 ? __fmul_rn((float)m, 0.125f)
                     : ldexpf(__fadd_rn(1.0f, __fmul_rn((float)m, 0.125f)), (int)e - 1);
        return (code & 0x20u) ? -mag : mag;
    } else {
        const uint32_t c = code & 3u;
        mag = c == 0 ? 0.0f : (float)(1u << (c - 1));
        return (code & 4u) ? -mag : mag;
    }
}

// INT integer k = clamp(RNE(v * c), -kmax, kmax): one fused multiply-add
// rounds the exact product once when |v| < 2^19 (the product then stays below
// 2^22, where 1.5 * 2^23 + t keeps a unit ulp); beyond, k is clamped anyway.
template <int BITS>
__device__ __forceinline__ int int_k(float v, float c)
{
    constexpr int KM = Width<BITS>::kmax;
    if (!(fabsf(v) < 0x1p19f)) return v < 0.0f ? -KM : KM;
    const float r = __fmaf_rn(v, c, kMagic);
    int k = (int)__fsub_rn(r, kMagic);
    return k < -KM ? -KM : (k > KM ? KM : k);
}

template <int BITS>
__device__ __forceinline__ uint32_t int_code(int k)
{
    return (uint32_t)k & ((1u << BITS) - 1u);
}

// Shared tables: the INT value of every code (index = code), filled with the
// correctly rounded quotients 15k/62 or 4k/3.
template <int BITS>
__device__ __forceinline__ void fill_int_table(float *tab)
{
    constexpr int N = 1 << BITS;
    for (int c = threadIdx.x; c < N; c += blockDim.x) {
        const int k = (c & (N >> 1)) ? c - N : c;
        tab[c] = BITS == 6 ? __fdiv_rn((float)(15 * k), 62.0f) : __fdiv_rn((float)(4 * k), 3.0f);
    }
}

template <int DT>
__device__ __forceinline__ void words16(const uint32_t (&w)[8], float (&x)[16], float &amax,
                                        bool &nonfinite);

// 16 inputs of group g as floats; amax = max |x| and nonfinite (Inf or NaN
// present, after which the outputs are unspecified).  16-bit inputs take the
// maximum on the packed words, two elements per instruction.
template <int DT>
__device__ __forceinline__ void load16(const char *p, float (&x)[16], float &amax, bool &nonfinite)
{
    if constexpr (DT == IF4_F32) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t a, b, c, d;
            ld_nc_v4(p + 16 * q, a, b, c, d);
            x[4 * q] = __uint_as_float(a);
            x[4 * q + 1] = __uint_as_float(b);
            x[4 * q + 2] = __uint_as_float(c);
            x[4 * q + 3] = __uint_as_float(d);
        }
        amax = 0.0f;
        nonfinite = false;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float a = fabsf(x[i]);
            nonfinite |= !(a <= 3.4028235e38f);
            amax = a > amax ? a : amax;
        }
    } else {
        uint32_t w[8];
        ld_nc_v4(p, w[0], w[1], w[2], w[3]);
        ld_nc_v4(p + 16, w[4], w[5], w[6], w[7]);
        words16<DT>(w, x, amax, nonfinite);
    }
}

// The 16 inputs of a 16-bit group from its eight loaded words (as load16).
template <int DT>
__device__ __forceinline__ void words16(const uint32_t (&w)[8], float (&x)[16], float &amax,
                                        bool &nonfinite)
{
    uint32_t m = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        if constexpr (DT == IF4_BF16) {
            m = absmax_bf16x2(m, w[j]);
            x[2 * j] = __uint_as_float(w[j] << 16);
            x[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        } else {
            m = absmax_f16x2(m, w[j]);
            x[2 * j] = f16lo_to_f32(w[j]);
            x[2 * j + 1] = f16hi_to_f32(w[j]);
        }
    }
    const uint32_t m16 = max(m & 0x7FFFu, (m >> 16) & 0x7FFFu);
    if constexpr (DT == IF4_BF16) {
        nonfinite = m16 >= 0x7F80u;
        amax = __uint_as_float(m16 << 16);
    } else {
        nonfinite = m16 >= 0x7C00u;
        amax = f16lo_to_f32(m16);
    }
}

template <int DT>
__device__ __forceinline__ void load16(const char *p, float (&x)[16])
{
    float amax;
    bool nonfinite;
    load16<DT>(p, x, amax, nonfinite);
}

template <int DT>
__host__ __device__ constexpr int ebytes() { return DT == IF4_F32 ? 4 : 2; }

__device__ __forceinline__ const char *row_addr(const char *base, uint32_t g, uint32_t gpr,
                                                int64_t ld_bytes, int gbytes)
{
    const uint32_t row = g / gpr;
    return base + (int64_t)row * ld_bytes + (int64_t)(g - row * gpr) * gbytes;
}

// Store the 16 codes of an IF6 group, element i at bits [6i, 6i + 6): codes
// joined in quads (each code below 2^6, so the sums do not carry), the quads
// cut into three 32-bit words at a 4-byte aligned address.
__device__ __forceinline__ void store_codes6(uint8_t *p, const uint32_t (&c)[16])
{
    uint32_t q[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
        q[k] = c[4 * k] + (c[4 * k + 1] << 6) + (c[4 * k + 2] << 12) + (c[4 * k + 3] << 18);
    uint32_t *w = reinterpret_cast<uint32_t *>(p);
    w[0] = q[0] | (q[1] << 24);
    w[1] = (q[1] >> 8) | (q[2] << 16);
    w[2] = (q[2] >> 16) | (q[3] << 8);
}

// The code bytes of a group as three words (IF6: 12 bytes as three 32-bit
// loads; IF3: 6 bytes as three 16-bit loads), then the 16 codes from them.
template <int BITS>
__device__ __forceinline__ void load_code_words(const uint8_t *p, uint32_t (&w)[3])
{
    if constexpr (BITS == 6) {
        const uint32_t *q = reinterpret_cast<const uint32_t *>(p);
        w[0] = __ldg(q);
        w[1] = __ldg(q + 1);
        w[2] = __ldg(q + 2);
    } else {
        const uint16_t *q = reinterpret_cast<const uint16_t *>(p);
        w[0] = __ldg(q);
        w[1] = __ldg(q + 1);
        w[2] = __ldg(q + 2);
    }
}

template <int BITS>
__device__ __forceinline__ void unpack_code_words(const uint32_t (&w)[3], uint32_t (&c)[16])
{
    uint64_t lo, hi = 0;
    if constexpr (BITS == 6) {
        lo = (uint64_t)w[0] | ((uint64_t)w[1] << 32);
        hi = w[2];
    } else {
        lo = (uint64_t)w[0] | ((uint64_t)w[1] << 16) | ((uint64_t)w[2] << 32);
    }
    constexpr uint64_t M = (1u << BITS) - 1u;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int pos = BITS * i;
        if (pos + BITS <= 64) c[i] = (uint32_t)((lo >> pos) & M);
        else if (pos >= 64) c[i] = (uint32_t)((hi >> (pos - 64)) & M);
        else c[i] = (uint32_t)(((lo >> pos) | (hi << (64 - pos))) & M);
    }
}

__device__ __forceinline__ bool ts_ok(float ts) { return ts >= 0x1p-117f && ts <= 0x1p117f; }

// Block scale sb_f = fl(fl(amax / fpmax) / ts).  The first quotient is the
// exact amax * 1/4 for IF3 (amax >= 2^-124); for IF6 it is q = fl(amax y)
// with y = fl(1/7.5), corrected once to q + fl(amax - 7.5 q) y, which equals
// the IEEE division for every finite amax >= 2^-100 (checked on the CPU for
// every mantissa); below, and for Inf or NaN, the IEEE division.  The second
// quotient is Markstein's: with y = fl(1/ts), s = fl(a y), fl(s + fl(a - s
// ts) y) is the correctly rounded a / ts when neither quotient over- nor
// underflows.  Below a = 2^-100 the IEEE division is used; from s = 2^100 the
// unrefined s is returned (any such value saturates to 448, as the exact one
// does).
template <int BITS>
__device__ __forceinline__ float block_scale_w(float amax, float ts, float rts)
{
    float a;
    if constexpr (BITS == 3) {
        a = amax >= 0x1p-124f ? __fmul_rn(amax, 0.25f) : __fdiv_rn(amax, 4.0f);
    } else if (amax >= 0x1p-100f && amax <= 3.4028235e38f) {
        const float y = __uint_as_float(0x3E088889u);       // fl(1/7.5)
        const float q = __fmul_rn(amax, y);
        a = __fmaf_rn(__fmaf_rn(-q, 7.5f, amax), y, q);
    } else {
        a = __fdiv_rn(amax, Width<BITS>::fpmax);
    }
    const float s = __fmul_rn(a, rts);
    if (!(a >= 0x1p-100f && s < 0x1p100f)) return a >= 0x1p-100f ? s : __fdiv_rn(a, ts);
    return __fmaf_rn(__fmaf_rn(-s, ts, a), rts, s);
}

// E2M3 codes of an element pair (code of v0 in bits 0-5, of v1 in bits 8-13,
// sign in the code's bit 5) by the hardware conversion (round to nearest
// even, saturating at 7.5), and the differences qf - v, each exact (qf is v
// rounded to the grid, within a factor of two of it, or 0): one
// mixed-precision subtract of the code's f16 value.
__device__ __forceinline__ uint32_t e2m3_pair(float v0, float v1, float &d0, float &d1)
{
    uint32_t c;
    asm("{\n\t.reg .b16 b, l, u;\n\t.reg .b32 h;\n\t"
        "cvt.rn.satfinite.e2m3x2.f32 b, %4, %3;\n\t"
        "cvt.rn.f16x2.e2m3x2 h, b;\n\t"
        "mov.b32 {l, u}, h;\n\t"
        "sub.rn.f32.f16 %1, l, %3;\n\t"
        "sub.rn.f32.f16 %2, u, %4;\n\t"
        "cvt.u32.u16 %0, b;\n\t}"
        : "=r"(c), "=f"(d0), "=f"(d1) : "f"(v0), "f"(v1));
    return c;
}

// The decision rule itself, for a group whose binary32 margin is within its
// band: the two binary64 error sums in element order, from the group's
// inputs reloaded at p.  Returns true when INT wins.
template <int DT, int BITS>
__device__ __noinline__ bool ifw_int_wins_exact(const char *p, float inv, float c_int,
                                                const float *int_tab)
{
    float xv[16];
    load16<DT>(p, xv);
    double e_fp = 0.0, e_int = 0.0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float v = __fmul_rn(xv[i], inv);
        const double df = __dsub_rn((double)v, (double)fp_value<BITS>(fp_code<BITS>(v)));
        const double di =
            __dsub_rn((double)v, (double)int_tab[int_code<BITS>(int_k<BITS>(v, c_int))]);
        e_fp = __dadd_rn(e_fp, __dmul_rn(df, df));
        e_int = __dadd_rn(e_int, __dmul_rn(di, di));
    }
    return e_int < e_fp;
}

// IF6: FP and INT candidates of one group and their binary32 error sums (two
// lanes: lane 0 sums the even elements, lane 1 the odd ones).  CLAMP: |v|
// held below 2^19, as a subnormal or the largest block scale needs; the
// integer is clamped to [-31, 31] on every path (under the other block
// scales |v| <= 7.5 (1 + 2^-4) (1 + 4u), and v * 62/15 reaches 32.9).  Element
// pairs (2j, 2j + 1) go through paired binary32 instructions, each lane
// rounded as its scalar form (57.4 against 62.7 us for the scalar loop on the
// 8192 x 8192 activation).
template <bool CLAMP>
__device__ __forceinline__ void if6_candidates(const float (&xv)[16], float inv, float c_int,
                                               float nc_q, uint32_t (&cf)[16], uint32_t (&ci)[16],
                                               float (&ef)[2], float (&ei)[2])
{
    constexpr int KM = Width<6>::kmax;
    const f2_t INV = f2_pack(inv, inv), C = f2_pack(c_int, c_int);
    const f2_t M = f2_pack(kMagic, kMagic), NM = f2_pack(-kMagic, -kMagic);
    const f2_t NCQ = f2_pack(nc_q, nc_q);
    f2_t EF = f2_pack(ef[0], ef[1]), EI = f2_pack(ei[0], ei[1]);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const f2_t V = f2_mul(f2_pack(xv[2 * j], xv[2 * j + 1]), INV);
        float v[2], df[2];
        f2_unpack(V, v[0], v[1]);
        const uint32_t c2 = e2m3_pair(v[0], v[1], df[0], df[1]);
        cf[2 * j] = c2 & 0x3Fu;
        cf[2 * j + 1] = (c2 >> 8) & 0x3Fu;
        // k = clamp(RNE(v * c), -31, 31): one fused multiply-add rounds the
        // exact product once while |v| < 2^19
        f2_t VC = V;
        if constexpr (CLAMP)
            VC = f2_pack(fminf(fmaxf(v[0], -0x1p19f), 0x1p19f),
                         fminf(fmaxf(v[1], -0x1p19f), 0x1p19f));
        f2_t R = f2_fma(VC, C, M);
        float r[2];
        f2_unpack(R, r[0], r[1]);
#pragma unroll
        for (int l = 0; l < 2; ++l)
            r[l] = fminf(fmaxf(r[l], kMagic - (float)KM), kMagic + (float)KM);
        R = f2_pack(r[0], r[1]);
        ci[2 * j] = __float_as_uint(r[0]) & 0x3Fu;         // two's complement
        ci[2 * j + 1] = __float_as_uint(r[1]) & 0x3Fu;
        const f2_t DI = f2_fma(f2_add(R, NM), NCQ, V);      // v - k fl(c), one rounding
        const f2_t DF = f2_pack(df[0], df[1]);
        EF = f2_fma(DF, DF, EF);
        EI = f2_fma(DI, DI, EI);
    }
    f2_unpack(EF, ef[0], ef[1]);
    f2_unpack(EI, ei[0], ei[1]);
}

// 1.0f where the comparison holds, else 0.0f; the unordered forms (gtu, geu)
// hold for a NaN operand.
__device__ __forceinline__ float set_gtu(float a, float b)
{
    float d;
    asm("set.gtu.f32.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
    return d;
}

__device__ __forceinline__ float set_geu(float a, float b)
{
    float d;
    asm("set.geu.f32.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
    return d;
}

// 1.0f when the sign bit of v is set (a negative zero too), else 0.0f.
__device__ __forceinline__ float sign_bit_f(float v)
{
    float d;
    asm("set.lt.f32.s32 %0, %1, 0;" : "=f"(d) : "r"(__float_as_uint(v)));
    return d;
}

// IF3: both candidates of one group as four 12-bit quads of codes (element
// 4k + i at bits [3i, 3i + 3) of quad k), and the binary32 error sums in two
// lanes (even and odd elements, each in element order).
//
// E2M0 from three comparisons of a = |v| that give 1.0 or 0.0: s1 = [a > 1/2],
// s2 = [a >= 3/2], s3 = [a > 3].  The value is s1 + s2 + 2 s3 (0, 1, 2, 4),
// the magnitude code s1 + s2 + s3 (0 to 3): ties go to the even code (1/2 ->
// 0, 3/2 -> 2, 3 -> 2) and a NaN, every comparison holding, to 4.  The FP
// quad is accumulated as the exact float 2^23 + sum (code_i 8^i) and read from
// its low 12 bits; code_i = magnitude + 4 [sign bit of v].  |qf - v| = fl(q -
// a) (exact under the unclamped scales; otherwise the same rounding of the
// same difference) enters the sum squared.  The INT integer k = RNE(3v/4) from
// one fused multiply-add as in IF6 (CLAMP: |v| held below 2^19 and k clamped
// to [-3, 3]; under any other block scale |3v/4| < 3.5 needs neither).
template <bool CLAMP>
__device__ __forceinline__ void if3_candidates(const float (&xv)[16], float inv, float nc_q,
                                               uint32_t (&fq)[4], uint32_t (&iq)[4],
                                               float (&ef)[2], float (&ei)[2])
{
    // element pairs (4k + 2p, 4k + 2p + 1) in paired binary32 instructions,
    // each lane rounded as its scalar form (60.8 against 65.6 us scalar on
    // the 8192 x 8192 activation); the FP quad in two lanes (even elements
    // from 2^23, odd ones from 0) added at the end, exactly
    const f2_t INV = f2_pack(inv, inv), C = f2_pack(0.75f, 0.75f);
    const f2_t M = f2_pack(kMagic, kMagic), NM = f2_pack(-kMagic, -kMagic);
    const f2_t NCQ = f2_pack(nc_q, nc_q), TWO = f2_pack(2.0f, 2.0f), FOUR = f2_pack(4.0f, 4.0f);
    f2_t EF = f2_pack(ef[0], ef[1]), EI = f2_pack(ei[0], ei[1]);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        f2_t ACC = f2_pack(0x1p23f, 0.0f);
        uint32_t iw = 0;
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const int e = 4 * k + 2 * p;
            const f2_t W = f2_pack((float)(1 << (6 * p)), (float)(1 << (6 * p + 3)));   // 8^i
            const f2_t V = f2_mul(f2_pack(xv[e], xv[e + 1]), INV);
            float v0, v1;
            f2_unpack(V, v0, v1);
            const float a0 = fabsf(v0), a1 = fabsf(v1);
            const f2_t S1 = f2_pack(set_gtu(a0, 0.5f), set_gtu(a1, 0.5f));
            const f2_t S2 = f2_pack(set_geu(a0, 1.5f), set_geu(a1, 1.5f));
            const f2_t S3 = f2_pack(set_gtu(a0, 3.0f), set_gtu(a1, 3.0f));
            const f2_t SG = f2_pack(sign_bit_f(v0), sign_bit_f(v1));
            const f2_t A = f2_add(S1, S2);
            const f2_t DF = f2_sub(f2_fma(S3, TWO, A), f2_pack(a0, a1));
            ACC = f2_fma(A, W, ACC);
            ACC = f2_fma(f2_fma(SG, FOUR, S3), W, ACC);
            f2_t VC = V;
            if constexpr (CLAMP)
                VC = f2_pack(fminf(fmaxf(v0, -0x1p19f), 0x1p19f), fminf(fmaxf(v1, -0x1p19f), 0x1p19f));
            f2_t R = f2_fma(VC, C, M);
            float r0, r1;
            f2_unpack(R, r0, r1);
            if constexpr (CLAMP) {
                r0 = fminf(fmaxf(r0, kMagic - 3.0f), kMagic + 3.0f);
                r1 = fminf(fmaxf(r1, kMagic - 3.0f), kMagic + 3.0f);
                R = f2_pack(r0, r1);
            }
            iw |= ((__float_as_uint(r0) & 7u) << (6 * p)) |           // two's complement
                  ((__float_as_uint(r1) & 7u) << (6 * p + 3));
            const f2_t DI = f2_fma(f2_add(R, NM), NCQ, V);
            EF = f2_fma(DF, DF, EF);
            EI = f2_fma(DI, DI, EI);
        }
        float acc0, acc1;
        f2_unpack(ACC, acc0, acc1);
        fq[k] = __float_as_uint(__fadd_rn(acc0, acc1)) & 0xFFFu;
        iq[k] = iw;
    }
    f2_unpack(EF, ef[0], ef[1]);
    f2_unpack(EI, ei[0], ei[1]);
}

// IF3: true when the FP and INT values of every element coincide (both 0, or
// both +4 or both -4), found on the codes: a slot coincides exactly when its
// FP magnitude code is 0 or 3 (bits 0 and 1 equal) and bit 0 of the FP and
// INT codes agree.  Where the FP value is 0 (|v| <= 1/2) k is 0; where it is
// 4 (|v| > 3) |k| is 2 or 3 with the sign of v; so the codes pair as (000 or
// 100, 000), (011, 011 or 010), (111, 101 or 110), and the test keeps the
// first of each pair.
__device__ __forceinline__ bool if3_values_coincide(const uint32_t (&fq)[4], const uint32_t (&iq)[4])
{
    uint32_t t = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) t |= (fq[k] ^ (fq[k] >> 1)) | (fq[k] ^ iq[k]);
    return (t & 0x249u) == 0u;                 // bit 0 of each of the 4 slots
}

// The 6 code bytes of an IF3 group from its four quads.
__device__ __forceinline__ void store_quads3(uint8_t *p, const uint32_t (&q)[4])
{
    uint16_t *w = reinterpret_cast<uint16_t *>(p);
    const uint32_t lo = q[0] | (q[1] << 12) | (q[2] << 24);
    w[0] = (uint16_t)lo;
    w[1] = (uint16_t)(lo >> 16);
    w[2] = (uint16_t)((q[2] >> 8) | (q[3] << 4));
}

// The fast decision from the two binary32 sums: INT when e_fp - e_int
// exceeds the band 2^-16 (S + 1); near when the margin is within it and S !=
// 0 (S == 0: every error is zero or below 2^-75 where both candidates are 0,
// the sums tie and FP stays).
__device__ __forceinline__ bool fast_int(const float (&ef)[2], const float (&ei)[2], bool &near)
{
    const float e_fp = __fadd_rn(ef[0], ef[1]), e_int = __fadd_rn(ei[0], ei[1]);
    const float d = __fsub_rn(e_fp, e_int);
    const float S = __fadd_rn(e_fp, e_int);
    const float band = __fmul_rn(__fadd_rn(S, 1.0f), 0x1p-16f);
    near = !(fabsf(d) > band) && S != 0.0f;
    return d > band;
}

// Quantizer: one group per thread per round of a grid-stride loop.
//
// Decision, fast path (as IF4's): the two squared-error sums in binary32,
// two lanes of 8 fused multiply-adds each, then one add.  The FP differences
// are exact under every block scale but the clamped ones; an INT difference
// is one fused multiply-add v - k * fl(c) (c = 15/62 or 4/3), off from the
// rule's v - fl(num k / den) by at most 2^-20 plus one rounding.  Outside the band 2^-16 (S + 1) (S = the sum of both
// errors) the binary32 sign is the rule's; inside it the group is decided by
// the binary64 rule itself (ifw_int_wins_exact).
template <int DT, int BITS>
__global__ void __launch_bounds__(256, 4)     // four blocks per SM: IF3 3 % faster than three
ifw_quantize_kernel(const char *__restrict__ x, int64_t ld_bytes, uint32_t gpr, uint32_t ngroups,
                    int mode, uint8_t *__restrict__ codes, uint8_t *__restrict__ scales,
                    const float *__restrict__ ts_ptr, int *err, int check_ts)
{
    pdl_enter();
    constexpr int GB = 16 * ebytes<DT>();
    constexpr int CB = Width<BITS>::code_bytes;
    __shared__ float int_tab[1 << BITS];
    fill_int_table<BITS>(int_tab);
    const float ts = *ts_ptr;
    if (check_ts && blockIdx.x == 0 && threadIdx.x == 0 && !ts_ok(ts) && err)
        atomicOr(err, IF4_DEV_BAD_SCALE);
    const float c_int = BITS == 6 ? __fdiv_rn(62.0f, 15.0f) : 0.75f;
    const float nc_q = BITS == 6 ? -__fdiv_rn(15.0f, 62.0f) : -__fdiv_rn(4.0f, 3.0f);
    const float rts = __frcp_rn(ts);
    // IF3: inv = fl(1/fl(E4M3 * ts)) of every block scale byte, once per
    // block (58.6 against 59.2 us on the 8192 x 8192 activation; IF6 measured
    // 56.8 against 56.5 us with it and computes it per group)
    __shared__ float inv_tab[BITS == 3 ? 128 : 1];
    if (BITS == 3 && threadIdx.x < 128)
        inv_tab[threadIdx.x] =
            threadIdx.x == 0 ? 0.0f : __frcp_rn(__fmul_rn(f32_from_e4m3(threadIdx.x), ts));
    __syncthreads();
    bool nonfinite = false;
    const bool contig = ld_bytes == (int64_t)gpr * GB;
    const uint32_t stride = gridDim.x * blockDim.x;
    // a contiguous tensor needs no division for the group's address
    auto gaddr = [&](uint32_t g) {
        return contig ? x + (int64_t)g * GB : row_addr(x, g, gpr, ld_bytes, GB);
    };
    // bf16 inputs: the next group's words are loaded while this group is
    // encoded, two groups in flight per thread (IF3 60.6 -> 59.2 us, IF6
    // 57.1 -> 56.7 us on the 8192 x 8192 activation; with three blocks per
    // SM instead of four IF6 took 60.0 us); the words are unpacked before
    // the next load reuses their registers (no copies: IF3 58.5 -> 57.0 us,
    // IF6 56.4 -> 55.1 us)
    constexpr bool PF = DT == IF4_BF16;
    const uint32_t g0 = blockIdx.x * blockDim.x + threadIdx.x;
    uint32_t wn[8];
    if constexpr (PF) {
        if (g0 < ngroups) {
            const char *p0 = gaddr(g0);
            ld_nc_v4(p0, wn[0], wn[1], wn[2], wn[3]);
            ld_nc_v4(p0 + 16, wn[4], wn[5], wn[6], wn[7]);
        }
    }
    for (uint32_t g = g0; g < ngroups; g += stride) {
        const char *p = gaddr(g);
        float xv[16], amax;
        bool nf;
        if constexpr (PF) {
            // unpack first, then the same registers take the next group
            words16<DT>(wn, xv, amax, nf);
            if (g + stride < ngroups) {
                const char *pn = gaddr(g + stride);
                ld_nc_v4(pn, wn[0], wn[1], wn[2], wn[3]);
                ld_nc_v4(pn + 16, wn[4], wn[5], wn[6], wn[7]);
            }
        } else {
            load16<DT>(p, xv, amax, nf);
        }
        nonfinite |= nf;
        const uint32_t sb = e4m3_from_f32(block_scale_w<BITS>(amax, ts, rts)) & 0x7Fu;
        uint32_t scale = 0;
        // a subnormal or the largest block scale: v may leave the range the
        // unclamped path relies on
        const bool clamp = (sb - 1u) < 7u || sb == 0x7Eu;
        const float inv = BITS == 3 ? inv_tab[sb]
                          : (sb != 0 ? __frcp_rn(__fmul_rn(f32_from_e4m3(sb), ts)) : 0.0f);
        float ef[2] = {0.0f, 0.0f}, ei[2] = {0.0f, 0.0f};
        if constexpr (BITS == 6) {
            uint32_t out[16];
            if (sb == 0) {
#pragma unroll
                for (int i = 0; i < 16; ++i) out[i] = 0;
            } else {
                uint32_t cf[16], ci[16];
                if (clamp) if6_candidates<true>(xv, inv, c_int, nc_q, cf, ci, ef, ei);
                else if6_candidates<false>(xv, inv, c_int, nc_q, cf, ci, ef, ei);
                bool use_int = mode == W_INT;
                if (mode == W_IF) {
                    bool near;
                    use_int = fast_int(ef, ei, near);
                    if (near) use_int = ifw_int_wins_exact<DT, 6>(p, inv, c_int, int_tab);
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) out[i] = use_int ? ci[i] : cf[i];
                scale = sb | (use_int ? 0x80u : 0u);
            }
            store_codes6(codes + (int64_t)g * CB, out);
        } else {
            uint32_t out[4] = {0u, 0u, 0u, 0u};
            if (sb != 0) {
                uint32_t fq[4], iq[4];
                if (clamp) if3_candidates<true>(xv, inv, nc_q, fq, iq, ef, ei);
                else if3_candidates<false>(xv, inv, nc_q, fq, iq, ef, ei);
                bool use_int = mode == W_INT;
                if (mode == W_IF) {
                    bool near;
                    use_int = fast_int(ef, ei, near);
                    // a group whose FP and INT values coincide element by
                    // element (0 or +-4 on both grids: about one group in 17
                    // of the activations) ties exactly and keeps FP, without
                    // the binary64 rule
                    if (near)
                        use_int = if3_values_coincide(fq, iq)
                                      ? false
                                      : ifw_int_wins_exact<DT, 3>(p, inv, c_int, int_tab);
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) out[k] = use_int ? iq[k] : fq[k];
                scale = sb | (use_int ? 0x80u : 0u);
            }
            store_quads3(codes + (int64_t)g * CB, out);
        }
        scales[g] = (uint8_t)scale;
    }
    if (nonfinite && err) atomicOr(err, IF4_DEV_NONFINITE);
}

// Dequantizer: y = fl(q * fl(E4M3 * ts)), rounded to the output type.
template <int ODT, int BITS>
__global__ void __launch_bounds__(256)
ifw_dequantize_kernel(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scales,
                      const float *__restrict__ ts_ptr, uint32_t gpr, uint32_t ngroups,
                      char *__restrict__ y, int64_t ld_bytes)
{
    pdl_enter();
    constexpr int CB = Width<BITS>::code_bytes;
    constexpr int OB = ODT == IF4_F32 ? 4 : 2;
    __shared__ float int_tab[1 << BITS];
    __shared__ float fp_tab[1 << BITS];
    fill_int_table<BITS>(int_tab);
    for (int c = threadIdx.x; c < (1 << BITS); c += blockDim.x) fp_tab[c] = fp_value<BITS>(c);
    const float ts = *ts_ptr;
    __syncthreads();
    const bool contig = ld_bytes == (int64_t)gpr * (16 * OB);
    // a dense, 32-byte aligned output: every group's outputs start on a
    // 32-byte sector, so 256-bit stores write whole sectors (two 128-bit
    // stores would each write half of every sector they touch)
    const bool v8 = contig && (reinterpret_cast<uintptr_t>(y) & 31u) == 0u;
    const uint32_t stride = gridDim.x * blockDim.x;
    const uint32_t g0 = blockIdx.x * blockDim.x + threadIdx.x;
    // the next group's code words and scale byte are loaded once this
    // group's codes are unpacked, into the same registers
    uint32_t w[3] = {0u, 0u, 0u}, sbn = 0u;
    if (g0 < ngroups) {
        load_code_words<BITS>(codes + (int64_t)g0 * CB, w);
        sbn = __ldg(scales + g0);
    }
    for (uint32_t g = g0; g < ngroups; g += stride) {
        uint32_t c[16];
        unpack_code_words<BITS>(w, c);
        const uint32_t sb = sbn;
        if (g + stride < ngroups) {
            load_code_words<BITS>(codes + (int64_t)(g + stride) * CB, w);
            sbn = __ldg(scales + g + stride);
        }
        const float eff = __fmul_rn(f32_from_e4m3(sb & 0x7Fu), ts);
        const float *tab = (sb & 0x80u) ? int_tab : fp_tab;
        float yv[16];
        if constexpr (BITS == 6) {
            // FP groups: the magnitude (code & 31, the table's first half)
            // with the sign bit applied, so that +m and -m read one word:
            // in the 64-entry table they sit 32 words apart, in one bank,
            // and a warp holding both waited on the bank conflict (35.5 ->
            // 33.4 us on the 8192 x 8192 activation).  INT codes k and
            // k - 32 share a bank too, but large |k| is rare.
            const uint32_t mmask = (sb & 0x80u) ? 63u : 31u;
            const uint32_t smask = (sb & 0x80u) ? 0u : 0x80000000u;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t q = __float_as_uint(tab[c[i] & mmask]) ^ ((c[i] << 26) & smask);
                yv[i] = __fmul_rn(__uint_as_float(q), eff);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) yv[i] = __fmul_rn(tab[c[i]], eff);
        }
        char *p = contig ? y + (int64_t)g * (16 * OB)
                         : const_cast<char *>(row_addr(y, g, gpr, ld_bytes, 16 * OB));
        if constexpr (ODT == IF4_F32) {
            if (v8) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t o[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) o[j] = __float_as_uint(yv[8 * h + j]);
                    st_v8(p + 32 * h, o);
                }
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    st_v4(p + 16 * q, __float_as_uint(yv[4 * q]), __float_as_uint(yv[4 * q + 1]),
                          __float_as_uint(yv[4 * q + 2]), __float_as_uint(yv[4 * q + 3]));
            }
        } else {
            uint32_t o[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
                o[j] = ODT == IF4_BF16 ? bf16x2_from_f32(yv[2 * j], yv[2 * j + 1])
                                       : f16x2_from_f32(yv[2 * j], yv[2 * j + 1]);
            if (v8) {
                st_v8(p, o);
            } else {
                st_v4(p, o[0], o[1], o[2], o[3]);
                st_v4(p + 16, o[4], o[5], o[6], o[7]);
            }
        }
    }
}

// ts = amax / (fpmax * 448), 1 for amax == 0, floored at 2^-117; amax in *ts.
template <int BITS>
__global__ void ifw_tensor_scale_kernel(float *ts)
{
    pdl_enter();
    const float a = *ts;
    float t = 1.0f;
    if (a != 0.0f) {
        t = __fdiv_rn(a, Width<BITS>::fpmax * 448.0f);
        if (t < 0x1p-117f) t = 0x1p-117f;
    }
    *ts = t;
}

// ------------------------------------------------------------ host side ----

int elem_size(int dt) { return dt == IF4_F32 ? 4 : (dt == IF4_BF16 || dt == IF4_F16) ? 2 : 0; }

struct Shape {
    uint32_t gpr = 0, ngroups = 0;
    int64_t ld_bytes = 0;
};

int check_tensor(const void *p, int dt, int64_t rows, int64_t cols, int64_t ld, Shape &s)
{
    const int es = elem_size(dt);
    if (es == 0) return IF4_ERR_DTYPE;
    if (rows < 0 || cols < 0 || cols % 16 != 0 || ld < cols) return IF4_ERR_SHAPE;
    if (rows > 0 && (cols / 16) > 0 && rows > (int64_t)0x7FFFFFFF / (cols / 16)) return IF4_ERR_SHAPE;
    if (rows > 0 && cols > 0 && p == nullptr) return IF4_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(p) % 16 != 0 || (ld * es) % 16 != 0) return IF4_ERR_ALIGN;
    s.gpr = (uint32_t)(cols / 16);
    s.ngroups = (uint32_t)(rows * (cols / 16));
    s.ld_bytes = ld * es;
    return IF4_OK;
}

int check_sm100()
{
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return IF4_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return IF4_ERR_CUDA;
    return major == 10 ? IF4_OK : IF4_ERR_DEVICE;
}

unsigned grid_size(uint32_t work)
{
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const uint64_t want = ((uint64_t)work + 255) / 256;
    const uint64_t cap = (uint64_t)sms * 8;
    return (unsigned)(want < 1 ? 1 : (want < cap ? want : cap));
}

template <typename... KArgs, typename... Args>
int launch(void (*k)(KArgs...), unsigned grid, cudaStream_t st, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k, args...) != cudaSuccess) return IF4_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? IF4_OK : IF4_ERR_CUDA;
}

template <int BITS>
int quantize_w(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x, int mode,
               uint8_t *codes, uint8_t *scales, float *ts, int ts_mode, int *err_flag,
               void *stream)
{
    Shape s;
    int rc = check_tensor(x, x_dtype, rows, cols, ld_x, s);
    if (rc != IF4_OK) return rc;
    if (mode != W_IF && mode != W_FP && mode != W_INT) return IF4_ERR_MODE;
    if (ts_mode != IF4_TS_COMPUTE && ts_mode != IF4_TS_GIVEN) return IF4_ERR_MODE;
    if (ts == nullptr) return IF4_ERR_NULL;
    if (s.ngroups > 0 && (codes == nullptr || scales == nullptr)) return IF4_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(codes) % 4 != 0 || reinterpret_cast<uintptr_t>(ts) % 4 != 0)
        return IF4_ERR_ALIGN;
    rc = check_sm100();
    if (rc != IF4_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (ts_mode == IF4_TS_COMPUTE) {
        // max |x| into *ts (the IF4 amax pass), then the width's tensor scale
        rc = if4_tensor_amax(x, x_dtype, rows, cols, ld_x, ts, err_flag, stream);
        if (rc != IF4_OK) return rc;
        rc = launch(ifw_tensor_scale_kernel<BITS>, 1, st, ts);
        if (rc != IF4_OK) return rc;
    }
    if (s.ngroups == 0) return IF4_OK;
    const unsigned grid = grid_size(s.ngroups);
    const char *xc = static_cast<const char *>(x);
    const int check = ts_mode == IF4_TS_GIVEN ? 1 : 0;
    switch (x_dtype) {
    case IF4_F32:
        return launch(ifw_quantize_kernel<IF4_F32, BITS>, grid, st, xc, s.ld_bytes, s.gpr,
                      s.ngroups, mode, codes, scales, (const float *)ts, err_flag, check);
    case IF4_BF16:
        return launch(ifw_quantize_kernel<IF4_BF16, BITS>, grid, st, xc, s.ld_bytes, s.gpr,
                      s.ngroups, mode, codes, scales, (const float *)ts, err_flag, check);
    default:
        return launch(ifw_quantize_kernel<IF4_F16, BITS>, grid, st, xc, s.ld_bytes, s.gpr,
                      s.ngroups, mode, codes, scales, (const float *)ts, err_flag, check);
    }
}

template <int BITS>
int dequantize_w(const uint8_t *codes, const uint8_t *scales, const float *ts, int64_t rows,
                 int64_t cols, void *y, int y_dtype, int64_t ld_y, void *stream)
{
    Shape s;
    int rc = check_tensor(y, y_dtype, rows, cols, ld_y, s);
    if (rc != IF4_OK) return rc;
    if (ts == nullptr) return IF4_ERR_NULL;
    if (s.ngroups > 0 && (codes == nullptr || scales == nullptr)) return IF4_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(codes) % 4 != 0 || reinterpret_cast<uintptr_t>(ts) % 4 != 0)
        return IF4_ERR_ALIGN;
    rc = check_sm100();
    if (rc != IF4_OK) return rc;
    if (s.ngroups == 0) return IF4_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const unsigned grid = grid_size(s.ngroups);
    char *yc = static_cast<char *>(y);
    switch (y_dtype) {
    case IF4_F32:
        return launch(ifw_dequantize_kernel<IF4_F32, BITS>, grid, st, codes, scales, ts, s.gpr,
                      s.ngroups, yc, s.ld_bytes);
    case IF4_BF16:
        return launch(ifw_dequantize_kernel<IF4_BF16, BITS>, grid, st, codes, scales, ts, s.gpr,
                      s.ngroups, yc, s.ld_bytes);
    default:
        return launch(ifw_dequantize_kernel<IF4_F16, BITS>, grid, st, codes, scales, ts, s.gpr,
                      s.ngroups, yc, s.ld_bytes);
    }
}

}  // namespace

extern "C" {

int if6_quantize(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x, int mode,
                 uint8_t *codes, uint8_t *scales, float *ts, int ts_mode, int *err_flag,
                 void *stream)
{
    return quantize_w<6>(x, x_dtype, rows, cols, ld_x, mode, codes, scales, ts, ts_mode, err_flag,
                         stream);
}

int if3_quantize(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x, int mode,
                 uint8_t *codes, uint8_t *scales, float *ts, int ts_mode, int *err_flag,
                 void *stream)
{
    return quantize_w<3>(x, x_dtype, rows, cols, ld_x, mode, codes, scales, ts, ts_mode, err_flag,
                         stream);
}

int if6_dequantize(const uint8_t *codes, const uint8_t *scales, const float *ts, int64_t rows,
                   int64_t cols, void *y, int y_dtype, int64_t ld_y, void *stream)
{
    return dequantize_w<6>(codes, scales, ts, rows, cols, y, y_dtype, ld_y, stream);
}

int if3_dequantize(const uint8_t *codes, const uint8_t *scales, const float *ts, int64_t rows,
                   int64_t cols, void *y, int y_dtype, int64_t ld_y, void *stream)
{
    return dequantize_w<3>(codes, scales, ts, rows, cols, y, y_dtype, ld_y, stream);
}

}  // extern "C"
