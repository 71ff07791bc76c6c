// IF4 quantize / dequantize kernels for B200 (sm_100a) and their C ABI.
//
// Format and algorithm: "Adaptive Block-Scaled Data Types" (Cook et al.,
// arXiv 2603.28765).  Per group of 16 values along the contiguous dimension
// the quantizer forms an E2M1 FP4 candidate and a 7/6-scaled INT4 candidate
// under one E4M3 block scale, keeps the one with the lower squared error and
// writes the choice into the scale byte's sign bit (gist.science section 2
// "Metodologia": "Mecanismo de Selecao", "Codificacao Eficiente", "Metodo
// 6/7"; shd-paper.top technical framework, steps 1-5).  The arithmetic
// contract is spelled out in include/if4.h.
//
// Work decomposition: the path moves 2.5625 B per bf16 element for quantize
// (the single-candidate modes are HBM-bound; the IF4 encode, at about 200
// instructions per group, is bound by instruction issue), so one thread owns
// one whole group: a 256-bit load brings its 16 bf16 values, every reduction
// (amax, both squared-error sums) stays in the thread's registers, and the
// outputs are one 8-byte code store and one scale byte.  Lanes of a warp own
// consecutive groups, so each warp-wide load or store touches one contiguous
// span.  A grid-stride loop keeps the next group's load in flight while the
// current one is computed, and runs full rounds of a contiguous tensor
// without per-group range checks.  The group encoder itself (block scale,
// candidates, decision) is in if4_encode.cuh, shared with the linear's
// IF4-output epilogue.
//
// Kernels here: the tensor amax and tensor scale; the quantizer for IF4 and
// its comparators (NVFP4, NVINT4, 4/6), optionally on the random-sign
// Hadamard transform; the single-launch quantizer (amax, grid barrier, encode)
// in one cooperative launch, optionally also writing the bf16 round trip of
// its codes; the dequantizer and the fp16 operand decode of the linear.

#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/if4.h"
#include "if4_device.cuh"
#include "if4_decode.cuh"
#include "if4_encode.cuh"
#include "if4_internal.h"

using namespace if4dev;

namespace {

// --------------------------------------------------------- group loads ----

// Raw bits of one group: 16-bit types fill w[0..7], f32 fills w[0..15].
template <int DT>
struct Raw {
    uint32_t w[DT == DT_F32 ? 16 : 8];
};

template <int DT, bool V8>
__device__ __forceinline__ void load_group(const char *p, Raw<DT> &r)
{
    if constexpr (DT == DT_F32) {
        if constexpr (V8) {
            uint32_t a[8], b[8];
            ld_nc_v8(p, a);
            ld_nc_v8(p + 32, b);
#pragma unroll
            for (int i = 0; i < 8; ++i) { r.w[i] = a[i]; r.w[8 + i] = b[i]; }
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                ld_nc_v4(p + 16 * q, r.w[4 * q], r.w[4 * q + 1], r.w[4 * q + 2], r.w[4 * q + 3]);
        }
    } else {
        if constexpr (V8) {
            ld_nc_v8(p, r.w);
        } else {
            ld_nc_v4(p, r.w[0], r.w[1], r.w[2], r.w[3]);
            ld_nc_v4(p + 16, r.w[4], r.w[5], r.w[6], r.w[7]);
        }
    }
}

// The same loads with an L2 cache policy.
template <int DT, bool V8>
__device__ __forceinline__ void load_group_pol(const char *p, Raw<DT> &r, uint64_t pol)
{
    if constexpr (DT == DT_F32) {
        if constexpr (V8) {
            uint32_t a[8], b[8];
            ld_nc_v8_pol(p, a, pol);
            ld_nc_v8_pol(p + 32, b, pol);
#pragma unroll
            for (int i = 0; i < 8; ++i) { r.w[i] = a[i]; r.w[8 + i] = b[i]; }
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                ld_nc_v4_pol(p + 16 * q, r.w[4 * q], r.w[4 * q + 1], r.w[4 * q + 2], r.w[4 * q + 3],
                             pol);
        }
    } else {
        if constexpr (V8) {
            ld_nc_v8_pol(p, r.w, pol);
        } else {
            ld_nc_v4_pol(p, r.w[0], r.w[1], r.w[2], r.w[3], pol);
            ld_nc_v4_pol(p + 16, r.w[4], r.w[5], r.w[6], r.w[7], pol);
        }
    }
}

// Unpack to 8 float pairs (element 2j low, 2j+1 high) and the group's max |x|
// as float bits; *nonfinite is set for Inf/NaN.
template <int DT>
__device__ __forceinline__ float unpack_group(const Raw<DT> &r, f2_t (&x)[8], bool &nonfinite)
{
    if constexpr (DT == DT_F32) {
        // max |x| in two chains of one instruction per element (NaN
        // propagates; the sign bit it leaves is masked off)
        uint32_t m0 = 0, m1 = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t a = r.w[2 * j], b = r.w[2 * j + 1];
            m0 = absmax_f32(m0, __uint_as_float(a));
            m1 = absmax_f32(m1, __uint_as_float(b));
            x[j] = f2_pack(__uint_as_float(a), __uint_as_float(b));
        }
        const uint32_t m = absmax_f32(m0, __uint_as_float(m1)) & 0x7FFFFFFFu;
        nonfinite = m >= 0x7F800000u;
        return __uint_as_float(m);
    } else {
        // max(|a|, |b|) per 16-bit lane in one instruction (the sign bit it
        // leaves is ignored); NaN propagates, so Inf/NaN show up in the max
        uint32_t m = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t w = r.w[j];
            m = (DT == DT_BF16) ? absmax_bf16x2(m, w) : absmax_f16x2(m, w);
            if constexpr (DT == DT_BF16)
                x[j] = f2_from_bf16x2(w);
            else
                x[j] = f2_pack(f16lo_to_f32(w), f16hi_to_f32(w));
        }
        const uint32_t m16 = max(m & 0x7FFFu, (m >> 16) & 0x7FFFu);
        if constexpr (DT == DT_BF16) {
            nonfinite = m16 >= 0x7F80u;
            return __uint_as_float(m16 << 16);
        } else {
            nonfinite = m16 >= 0x7C00u;
            return f16lo_to_f32(m16);
        }
    }
}

// ------------------------------------- random-sign Hadamard transform ----
//
// y = H16 diag(s) x / 4 per group: the orthonormal random-sign transform the
// pages apply to weight gradients before quantizing them (gist.science
// section 1, second item; companion "Where the Gain Actually Comes From").
// Evaluated in binary32 as the fast Walsh-Hadamard transform, stages h = 1,
// 2, 4, 8 replacing (y[i], y[i+h]) by (y[i] + y[i+h], y[i] - y[i+h]) for i
// with bit h clear, then times 1/4 (exact).

// Sign flips as XOR masks on the raw words of a group: for 16-bit types word
// j holds elements 2j and 2j+1 (bits 15 and 31), for f32 word i element i.
struct SignMasks {
    uint32_t w[16];
};

// The transform on the 8 element pairs of a group (pair j = elements 2j,
// 2j+1): stage 1 inside each pair, stages 2, 4, 8 between pairs j and j + h/2.
// QUARTER: also the final times 1/4; without it x holds H x, for callers
// that fold the exact 1/4 into a later scaling.
template <bool QUARTER = true>
__device__ __forceinline__ void hadamard16(f2_t (&x)[8])
{
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float a, b;
        f2_unpack(x[j], a, b);
        x[j] = f2_pack(__fadd_rn(a, b), __fsub_rn(a, b));
    }
#pragma unroll
    for (int hp = 1; hp < 8; hp <<= 1) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if ((j & hp) == 0) {
                const f2_t a = x[j], b = x[j + hp];
                x[j] = f2_add(a, b);
                x[j + hp] = f2_sub(a, b);
            }
        }
    }
    if constexpr (QUARTER) {
        const f2_t Q = f2_pack(0.25f, 0.25f);
#pragma unroll
        for (int j = 0; j < 8; ++j) x[j] = f2_mul(x[j], Q);
    }
}

// The same transform on 16 scalars (the rare exact paths).
__device__ __forceinline__ void hadamard16_scalar(float (&y)[16], uint32_t signs)
{
#pragma unroll
    for (int j = 0; j < 16; ++j)
        if ((signs >> j) & 1u) y[j] = -y[j];
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            if ((i & h) == 0) {
                const float a = y[i], b = y[i + h];
                y[i] = __fadd_rn(a, b);
                y[i + h] = __fsub_rn(a, b);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) y[j] = __fmul_rn(y[j], 0.25f);
}

// Unpack with the transform: sign masks on the raw bits, pairs as in
// unpack_group, the transform, then max |y| over the transformed group
// (y = H x / 4).  QUARTER = false leaves x = H x (not y); the returned max is
// |y|'s either way: max fl(|H x| / 4) = fl(max |H x| / 4), rounding being
// monotone, subnormals included.
template <int DT, bool QUARTER = true>
__device__ __forceinline__ float unpack_group_rht(const Raw<DT> &r, const SignMasks &sm,
                                                  f2_t (&x)[8], bool &nonfinite)
{
    if constexpr (DT == DT_F32) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
            x[j] = f2_pack(__uint_as_float(r.w[2 * j] ^ sm.w[2 * j]),
                           __uint_as_float(r.w[2 * j + 1] ^ sm.w[2 * j + 1]));
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t w = r.w[j] ^ sm.w[j];
            if constexpr (DT == DT_BF16)
                x[j] = f2_from_bf16x2(w);
            else
                x[j] = f2_pack(f16lo_to_f32(w), f16hi_to_f32(w));
        }
    }
    hadamard16<false>(x);
    uint32_t m0 = 0, m1 = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float a, b;
        f2_unpack(x[j], a, b);
        m0 = absmax_f32(m0, a);
        m1 = absmax_f32(m1, b);
    }
    const uint32_t m = absmax_f32(m0, __uint_as_float(m1)) & 0x7FFFFFFFu;
    nonfinite = m >= 0x7F800000u;
    if constexpr (QUARTER) {
        const f2_t Q = f2_pack(0.25f, 0.25f);
#pragma unroll
        for (int k = 0; k < 8; ++k) x[k] = f2_mul(x[k], Q);
    }
    return __fmul_rn(__uint_as_float(m), 0.25f);
}

// The 16 (transformed, when RHT) inputs of a group, re-read from memory.
template <int DT, bool RHT>
__device__ __forceinline__ void reload_group(const char *p, uint32_t signs, float (&y)[16])
{
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        if constexpr (DT == DT_F32)
            y[i] = __ldg(reinterpret_cast<const float *>(p) + i);
        else if constexpr (DT == DT_BF16)
            y[i] = __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short *>(p) + i) << 16);
        else
            y[i] = __half2float(__ushort_as_half(__ldg(reinterpret_cast<const unsigned short *>(p) + i)));
    }
    if constexpr (RHT) hadamard16_scalar(y, signs);
}

__device__ __forceinline__ bool ts_valid(float ts)
{
    return ts >= kTsFloor && ts <= kTsCeil;   // false for NaN
}

template <int DT>
__host__ __device__ constexpr int elem_bytes() { return DT == DT_F32 ? 4 : 2; }

__device__ __forceinline__ const char *group_ptr(const char *x, uint32_t g, bool contig,
                                                 uint32_t gpr, int64_t ld_bytes, int gbytes)
{
    if (contig) return x + (int64_t)g * gbytes;
    uint32_t row = g / gpr;
    uint32_t col = g - row * gpr;
    return x + (int64_t)row * ld_bytes + (int64_t)col * gbytes;
}

// The encode with the INT4 clamp, for the rare groups whose scaled maximum
// can round past 7 (a saturated or subnormal block scale).
// It re-reads the group (still in L2) so that no registers of the common
// path are passed to it.
template <int DT, int MODE, bool RHT>
__device__ __noinline__ GroupCode encode_group_clamped(uint32_t sb, float inv, const char *p,
                                                       uint32_t signs)
{
    float y[16];
    reload_group<DT, RHT>(p, signs, y);
    f2_t x[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = f2_pack(y[2 * j], y[2 * j + 1]);
    return encode_group<MODE, true>(x, sb, inv, y);
}

// Address of group g of a [rows, gpr groups] tensor with row stride
// ld_bytes (a contiguous tensor is passed as one row of every group).
template <int GB>
__device__ __forceinline__ const char *group_addr(const char *x, uint32_t g, uint32_t gpr,
                                                  int64_t ld_bytes)
{
    const uint32_t row = g / gpr;
    return x + (int64_t)row * ld_bytes + (int64_t)(g - row * gpr) * GB;
}

// fl(fl(amax / 4) / ts): amax / 4 is exact (a power of two) above 2^-124,
// the quotient by ts is Markstein's, as in block_scale.
__device__ __forceinline__ float block_scale4(float amax, float ts, float rts)
{
    const float q = __fmul_rn(amax, 0.25f);
    const float s = __fmul_rn(q, rts);
    const float t = __fmaf_rn(__fmaf_rn(-s, ts, q), rts, s);
    if (!(amax >= 0x1p-100f && s < 0x1p100f))
        return amax >= 0x1p-100f ? s : block_scale_ieee(amax, 4.0f, ts);
    return t;
}

// Binary64 reconstruction errors of the two 4/6 candidates in element order
// (the rule itself), for groups whose binary32 margin is within rounding.
// The 16 inputs are all loaded before the sums start (one round trip).
template <int DT>
__device__ __noinline__ bool four_wins_exact(const char *p, float inv6, float eff6, float inv4,
                                             float eff4)
{
    float xv[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        if constexpr (DT == DT_F32)
            xv[i] = __ldg(reinterpret_cast<const float *>(p) + i);
        else if constexpr (DT == DT_BF16)
            xv[i] = __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short *>(p) + i) << 16);
        else
            xv[i] = __half2float(__ushort_as_half(__ldg(reinterpret_cast<const unsigned short *>(p) + i)));
    }
    double e6 = 0.0, e4 = 0.0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float x = xv[i];
        const float q6 = f16lo_to_f32(f16x2_from_e2m1x2(e2m1x2_from_f32(__fmul_rn(x, inv6), 0.0f)));
        const float q4 = f16lo_to_f32(f16x2_from_e2m1x2(e2m1x2_from_f32(__fmul_rn(x, inv4), 0.0f)));
        const double d6 = __dsub_rn((double)x, (double)__fmul_rn(q6, eff6));
        const double d4 = __dsub_rn((double)x, (double)__fmul_rn(q4, eff4));
        e6 = __dadd_rn(e6, __dmul_rn(d6, d6));
        e4 = __dadd_rn(e4, __dmul_rn(d4, d4));
    }
    return e4 < e6;
}

// 4/6 encode of one group: FP4 under the block scale of amax/6 and under that
// of amax/4, reconstruction errors sum (x - fl(q * eff))^2 compared, equal
// errors keep /6.  Fast path: each candidate's squared differences q - v in
// the scaled domain (exact mixed-precision subtracts), summed in two lanes
// and scaled by fl(eff^2).  eff (v - q) differs from the rule's x - fl(q *
// eff) by at most about 3.1 u X per element (v = fl(x fl(1/eff))), and with
// the sums' roundings the binary32 difference stays within 2^-19.3 S +
// 2^-20.4 X^2 of the rule (X = 6 max(eff6, eff4)), so outside the band 2^-18
// S + 2^-19 X^2 + 2^-126 its sign is the rule's.  Above X = 2^60 (where
// eff^2 may overflow), and when exactly one block scale is zero, the rule
// decides.
template <int DT>
__device__ __forceinline__ GroupCode encode_group_46(const f2_t (&x)[8], float amax, float ts,
                                                   float rts, const float *inv_tab,
                                                   const float *eff_tab, const char *xbase,
                                                   uint32_t g, uint32_t gpr, int64_t ld_bytes)
{
    const uint32_t sb6 = e4m3_from_f32(block_scale(amax, ts, rts)) & 0x7Fu;
    const uint32_t sb4 = e4m3_from_f32(block_scale4(amax, ts, rts)) & 0x7Fu;
    const float inv6 = inv_tab[sb6], eff6 = eff_tab[sb6];
    const float inv4 = inv_tab[sb4], eff4 = eff_tab[sb4];
    uint32_t w6[2], w4[2];
    f2_t e6 = f2_pack(0.0f, 0.0f), e4 = f2_pack(0.0f, 0.0f);
    const f2_t INV6 = f2_pack(inv6, inv6), INV4 = f2_pack(inv4, inv4);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        f2_t v6[4], v4[4], d6[4], d4[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            v6[j] = f2_mul(x[4 * h + j], INV6);
            v4[j] = f2_mul(x[4 * h + j], INV4);
        }
        w6[h] = fp4_word<true>(v6, d6);          // d = qf - v, exact
        w4[h] = fp4_word<true>(v4, d4);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            e6 = f2_fma(d6[j], d6[j], e6);
            e4 = f2_fma(d4[j], d4[j], e4);
        }
    }
    float a0, a1, b0, b1;
    f2_unpack(e6, a0, a1);
    f2_unpack(e4, b0, b1);
    // the scaled-domain sums times fl(eff^2): the x-domain sums, to within
    // the band below
    const float s6 = __fmul_rn(__fadd_rn(a0, a1), __fmul_rn(eff6, eff6));
    const float s4 = __fmul_rn(__fadd_rn(b0, b1), __fmul_rn(eff4, eff4));
    const float d = __fsub_rn(s6, s4);
    const float X = __fmul_rn(6.0f, fmaxf(eff6, eff4));
    const float band = __fmaf_rn(__fadd_rn(s6, s4), 0x1p-18f,
                                 __fmaf_rn(__fmul_rn(X, X), 0x1p-19f, 0x1p-126f));
    bool four = d > 0.0f;
    if (sb4 == sb6)
        four = false;                 // identical candidates: a tie, keep /6
    // the rule decides within the band; above X = 2^60, where eff^2 may
    // overflow; and when one block scale is zero (its v is 0, so the
    // scaled-domain sum is 0, while every output of that candidate is 0 and
    // its x-domain error the sum of x^2)
    else if (!(fabsf(d) > band) || X > 0x1p60f || sb6 == 0u || sb4 == 0u)
        four = four_wins_exact<DT>(group_addr<16 * elem_bytes<DT>()>(xbase, g, gpr, ld_bytes), inv6,
                                   eff6, inv4, eff4);
    GroupCode out;
    const uint32_t sb = four ? sb4 : sb6;
    out.c0 = four ? w4[0] : w6[0];
    out.c1 = four ? w4[1] : w6[1];
    out.scale = sb;
    if (sb == 0) out.c0 = out.c1 = 0u;
    return out;
}

// IF4 encode of one group, fast path.  Block scale by Markstein quotients
// (exact unless flagged below); both candidates without the INT4 clamp (it is
// the identity for every block scale E4M3 code 8..125: the largest |v| is
// then at most 6 * 17/16 = 6.375 and 6.375 * fl(7/6) < 7.5); the decision by
// binary32 error sums with the band of encode_group.  One branch leaves the
// path for every rare case: a flagged block scale (tiny amax, a quotient of
// 2^100 or more, Inf/NaN), a block scale code 1..7 or 126 (the clamp may
// act), or a margin within the band.
template <int DT, bool RHT>
__device__ __forceinline__ GroupCode encode_if4(const f2_t (&xv)[8], float amax, float ts,
                                              float rts, const float *inv_tab, const char *x,
                                              uint32_t g, uint32_t gpr, int64_t ld_bytes,
                                              uint32_t signs)
{
    constexpr int GB = 16 * elem_bytes<DT>();
    const If4Fast f = if4_fast<RHT>(xv, amax, ts, rts, inv_tab);
    return if4_finish(f, amax, ts, rts, inv_tab, [&](float (&y)[16]) {
        reload_group<DT, RHT>(group_addr<GB>(x, g, gpr, ld_bytes), signs, y);
    });
}

// ------------------------------------------ group decode (dequantizer) ----

template <int ODT>
__device__ __forceinline__ uint32_t pack_out2(float a, float b)
{
    if constexpr (ODT == DT_BF16) return bf16x2_from_f32(a, b);
    else return f16x2_from_f32(a, b);
}

// Decode one group (code words w0, w1, scale byte sb) and store its 16
// outputs at p: binary32 outputs by the per-element table; 16-bit outputs
// by the byte-permute decode (PERM), and by the table when the group holds
// INT4 code 8, eff is not finite with its sign bit clear, or !PERM (the same
// values).  POL: the 16-bit outputs are stored with the L2 cache policy pol.
template <int ODT, bool UNIT_TS, bool V8 = false, bool POL = false, bool PERM = true>
__device__ __forceinline__ void dequant_group(uint32_t w0, uint32_t w1, uint32_t sb, float ts,
                                              uint32_t lut_addr, char *p, uint64_t pol = 0)
{
    const float e4 = f32_from_e4m3(sb);
    const float eff = UNIT_TS ? e4 : __fmul_rn(e4, ts);
    const uint32_t base = lut_addr + ((sb >> 1) & 0x40u);        // INT4 half for bit 7
    // per-element table decode: values in binary32, then the output type
    auto table_decode = [&](f2_t (&ya)[4], f2_t (&yb)[4]) {
        float qa[8], qb[8];
        decode_word(w0, base, qa);
        decode_word(w1, base, qb);
        const f2_t EFF = f2_pack(eff, eff);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            ya[j] = f2_mul(f2_pack(qa[2 * j], qa[2 * j + 1]), EFF);
            yb[j] = f2_mul(f2_pack(qb[2 * j], qb[2 * j + 1]), EFF);
        }
    };
    if constexpr (ODT == DT_F32) {
        f2_t ya[4], yb[4];
        table_decode(ya, yb);
        uint32_t a[8], b[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float lo, hi;
            f2_unpack(ya[j], lo, hi);
            a[2 * j] = __float_as_uint(lo);
            a[2 * j + 1] = __float_as_uint(hi);
            f2_unpack(yb[j], lo, hi);
            b[2 * j] = __float_as_uint(lo);
            b[2 * j + 1] = __float_as_uint(hi);
        }
        if constexpr (V8) {
            st_v8(p, a);
            st_v8(p + 32, b);
        } else {
            st_v4(p, a[0], a[1], a[2], a[3]);
            st_v4(p + 16, a[4], a[5], a[6], a[7]);
            st_v4(p + 32, b[0], b[1], b[2], b[3]);
            st_v4(p + 48, b[4], b[5], b[6], b[7]);
        }
    } else {
        uint32_t o[8];
        if constexpr (!PERM) {
            f2_t ya[4], yb[4];
            table_decode(ya, yb);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float lo, hi;
                f2_unpack(ya[j], lo, hi);
                o[j] = pack_out2<ODT>(lo, hi);
                f2_unpack(yb[j], lo, hi);
                o[4 + j] = pack_out2<ODT>(lo, hi);
            }
        }
        uint32_t bad = 0u;
        if constexpr (PERM) {
            const uint32_t im = 0u - ((sb >> 7) & 1u);
            const BytePlanes P = group_planes<ODT == DT_BF16>(base, eff);
            bad = decode_word16(w0, im, P, o) | decode_word16(w1, im, P, o + 4);
            if (!permute_decode_ok(eff)) bad = 1u;
        }
        if (bad != 0u) {
            // per-element table decode, one pair at a time (few live values)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t w = i < 4 ? w0 : w1;
                const int sh = 8 * (i & 3);
                o[i] = pack_out2<ODT>(__fmul_rn(lds_f32(base + ((w >> sh << 2) & 0x3Cu)), eff),
                                      __fmul_rn(lds_f32(base + ((w >> (sh + 4) << 2) & 0x3Cu)),
                                                eff));
            }
        }
        // one 256-bit store fills a whole 32-byte sector; two 128-bit
        // stores would each write half of every sector they touch
        if constexpr (V8 && POL) {
            st_v8_pol(p, o, pol);
        } else if constexpr (V8) {
            st_v8(p, o);
        } else if constexpr (POL) {
            st_v4_pol(p, o[0], o[1], o[2], o[3], pol);
            st_v4_pol(p + 16, o[4], o[5], o[6], o[7], pol);
        } else {
            st_v4(p, o[0], o[1], o[2], o[3]);
            st_v4(p + 16, o[4], o[5], o[6], o[7]);
        }
    }
}

// Encode group g from its raw bits r and store its codes and scale byte.
// Returns true when an input element is Inf or NaN.  POL: every store
// carries the L2 cache policy pol.
template <int DT, int MODE, bool RHT, bool NV = false, bool DQ = false, bool POL = false>
__device__ __forceinline__ bool quantize_one(const Raw<DT> &r, uint32_t g, const char *x,
                                             int64_t ld_bytes, uint32_t gpr, float ts, float rts,
                                             const float *inv_tab, const float *eff_tab,
                                             uint8_t *codes, uint8_t *scales,
                                             const SignMasks &sm, uint32_t signs,
                                             uint8_t *nv_codes = nullptr,
                                             uint8_t *nv_scales = nullptr,
                                             char *y = nullptr, uint32_t lut_addr = 0u,
                                             uint64_t pol = 0)
{
    constexpr int GB = 16 * elem_bytes<DT>();
    f2_t xv[8];
    bool nonfinite;
    float amax;
    // IF4 with the transform keeps x = H x and folds the exact 1/4 into the
    // inverse block scale (if4_fast<true>); the other modes take y = H x / 4
    if constexpr (RHT)
        amax = unpack_group_rht<DT, MODE != Q_IF4>(r, sm, xv, nonfinite);
    else
        amax = unpack_group<DT>(r, xv, nonfinite);
    GroupCode out;
    if constexpr (MODE == Q_IF4) {
        out = encode_if4<DT, RHT>(xv, amax, ts, rts, inv_tab, x, g, gpr, ld_bytes, signs);
    } else if constexpr (MODE == Q_46) {
        out = encode_group_46<DT>(xv, amax, ts, rts, inv_tab, eff_tab, x, g, gpr, ld_bytes);
    } else {
        const uint32_t sb = e4m3_from_f32(block_scale(amax, ts, rts)) & 0x7Fu;
        // sb == 0: inv = 0 makes every candidate 0; the outputs are forced
        // to all-zero codes below
        const float inv = inv_tab[sb];
        // NVINT4: the clamp can act only under block scale codes 1..7 and
        // 126 (see encode_if4); FP4 saturates by itself
        if (MODE == Q_NVINT4 && ((sb - 1u) < 7u || sb == 0x7Eu))
            out = encode_group_clamped<DT, MODE, RHT>(sb, inv, group_addr<GB>(x, g, gpr, ld_bytes),
                                                      signs);
        else
            out = encode_group<MODE, false>(xv, sb, inv, nullptr);
        if (sb == 0) out.c0 = out.c1 = out.scale = 0u;
    }
    if constexpr (POL) {
        st_v2_pol(codes + (int64_t)g * 8, out.c0, out.c1, pol);
        st_u8_pol(scales + g, out.scale, pol);
    } else {
        st_v2(codes + (int64_t)g * 8, out.c0, out.c1);
        st_u8(scales + g, out.scale);
    }
    if constexpr (NV && MODE == Q_IF4) {
        // the NVFP4 comparator: the FP4 candidate under the same block scale
        if constexpr (POL) {
            st_v2_pol(nv_codes + (int64_t)g * 8, out.f0, out.f1, pol);
            st_u8_pol(nv_scales + g, out.scale & 0x7Fu, pol);
        } else {
            st_v2(nv_codes + (int64_t)g * 8, out.f0, out.f1);
            st_u8(nv_scales + g, out.scale & 0x7Fu);
        }
    }
    if constexpr (DQ) {
        // the round trip: this group's IF4 codes decoded as the dequantizer
        // decodes them, bf16 into a dense 32-byte aligned y
        dequant_group<DT_BF16, false, true, POL>(out.c0, out.c1, out.scale, ts, lut_addr,
                                                 y + (int64_t)g * 32, pol);
    }
    return nonfinite;
}

// Quantizer kernel: one group per thread per step of a grid-stride loop,
// the group's 32 (64) bytes in one (two) 256-bit loads, and the loads of the
// next PF groups in flight while the current one is encoded (PF = 2 for the
// light single-candidate modes, whose few instructions per group would not
// otherwise hide the memory latency; 1 for the rest, which keeps them at four
// resident blocks per SM).
template <int DT, int MODE, bool V8, bool RHT, int PF>
__global__ void __launch_bounds__(256, DT == DT_F32 ? 3 : 4)
quantize_kernel(const char *__restrict__ x, int64_t ld_bytes, uint32_t gpr,
                       uint32_t ngroups, int contig, uint8_t *__restrict__ codes,
                       uint8_t *__restrict__ scales, const float *__restrict__ ts_ptr, int *err,
                       int check_ts, const __grid_constant__ SignMasks sm, uint32_t signs)
{
    pdl_enter();
    constexpr int GB = 16 * elem_bytes<DT>();
    const float ts = *ts_ptr;
    if (check_ts && blockIdx.x == 0 && threadIdx.x == 0 && !ts_valid(ts) && err)
        atomicOr(err, IF4_DEV_BAD_SCALE);
    __shared__ float inv_tab[128];
    __shared__ float eff_tab[MODE == Q_46 ? 128 : 1];
    if (threadIdx.x < 128) {
        const float eff = __fmul_rn(f32_from_e4m3(threadIdx.x), ts);
        inv_tab[threadIdx.x] = threadIdx.x == 0 ? 0.0f : __frcp_rn(eff);
        if constexpr (MODE == Q_46) eff_tab[threadIdx.x] = eff;
    }
    const float rts = __frcp_rn(ts);
    __syncthreads();
    // the address of a group: contiguous tensors without a division
    const uint32_t gpr_eff = contig ? ngroups : gpr;
    auto addr = [&](uint32_t g) -> const char * {
        return contig ? x + (int64_t)g * GB : group_addr<GB>(x, g, gpr, ld_bytes);
    };
    const uint32_t stride = gridDim.x * blockDim.x;
    uint32_t g = blockIdx.x * blockDim.x + threadIdx.x;
    bool saw_nonfinite = false;
    // PF + 1 register buffers used in turn (g < 2^31 and the stride is far
    // below 2^31, so g + 2 * stride cannot wrap)
    Raw<DT> buf[PF + 1];
    if (g < ngroups) load_group<DT, V8>(addr(g), buf[0]);
    if (PF == 2 && g + stride < ngroups) load_group<DT, V8>(addr(g + stride), buf[1]);
    // Full rounds of a contiguous tensor, while every load of the round is in
    // range: no per-group range checks.  Worth 6-8 % for the IF4 encode (one
    // group in flight); the two-buffer loop of the single-candidate modes, and
    // the single launch's encode pass (which spilled with it), are left as
    // they are (they were no faster this way).
    if (PF == 1 && contig) {
        while ((uint64_t)g + (uint64_t)(2 * PF) * stride < ngroups) {
#pragma unroll
            for (int ph = 0; ph <= PF; ++ph) {
                load_group<DT, V8>(x + (int64_t)(g + PF * stride) * GB, buf[(ph + PF) % (PF + 1)]);
                saw_nonfinite |= quantize_one<DT, MODE, RHT>(buf[ph], g, x, ld_bytes, gpr_eff, ts,
                                                              rts, inv_tab, eff_tab, codes, scales, sm,
                                                              signs);
                g += stride;
            }
        }
    }
    // the rest (and strided tensors), one range check per group
    for (; g < ngroups;) {
#pragma unroll
        for (int ph = 0; ph <= PF; ++ph) {
            const uint32_t gp = g + PF * stride;
            if (gp < ngroups) load_group<DT, V8>(addr(gp), buf[(ph + PF) % (PF + 1)]);
            saw_nonfinite |= quantize_one<DT, MODE, RHT>(buf[ph], g, x, ld_bytes, gpr_eff, ts,
                                                          rts, inv_tab, eff_tab, codes, scales, sm,
                                                          signs);
            g += stride;
            if (g >= ngroups) break;
        }
    }
    if (saw_nonfinite && err) atomicOr(err, IF4_DEV_NONFINITE);
}

// ------------------------------------------ tensor amax and tensor scale --

// Float bits of max |x| over one group (NaN and Inf compare above every
// finite value, so they survive the integer max below).
template <int DT>
__device__ __forceinline__ uint32_t group_absmax_bits(const Raw<DT> &r)
{
    if constexpr (DT == DT_F32) {
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) m = max(m, r.w[i] & 0x7FFFFFFFu);
        return m;
    } else {
        uint32_t h = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            h = (DT == DT_BF16) ? absmax_bf16x2(h, r.w[i]) : absmax_f16x2(h, r.w[i]);
        const uint32_t h16 = max(h & 0x7FFFu, (h >> 16) & 0x7FFFu);
        return (DT == DT_BF16) ? (h16 << 16) : __float_as_uint(f16lo_to_f32(h16));
    }
}

// Tensor amax: max |x| over the tensor, accumulated as float bits with atomicMax into
// *amax_bits (zeroed by the caller's stream).  Each thread keeps eight group
// loads (four for f32) in flight.
template <int DT, bool V8, bool RHT>
__global__ void __launch_bounds__(256)
amax_kernel(const char *__restrict__ x, int64_t ld_bytes, uint32_t gpr, uint32_t ngroups,
            int contig, unsigned int *amax_bits, int *err, const __grid_constant__ SignMasks sm)
{
    pdl_enter();
    constexpr int GB = 16 * elem_bytes<DT>();
    constexpr int U = DT == DT_F32 ? 4 : 8;
    uint32_t m = 0;
    const uint32_t stride = gridDim.x * blockDim.x;
    for (uint64_t g0 = blockIdx.x * blockDim.x + threadIdx.x; g0 < ngroups;
         g0 += (uint64_t)U * stride) {
        Raw<DT> r[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint64_t g = g0 + (uint64_t)u * stride;
            if (g < ngroups) load_group<DT, V8>(group_ptr(x, (uint32_t)g, contig, gpr, ld_bytes, GB), r[u]);
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (g0 + (uint64_t)u * stride < ngroups) {
                if constexpr (RHT) {
                    f2_t xv[8];
                    bool nf;
                    m = max(m, __float_as_uint(unpack_group_rht<DT, false>(r[u], sm, xv, nf)));
                } else {
                    m = max(m, group_absmax_bits<DT>(r[u]));
                }
            }
    }
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    __shared__ uint32_t warp_max[8];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) warp_max[warp] = m;
    __syncthreads();
    if (warp == 0) {
        uint32_t v = lane < (int)(blockDim.x >> 5) ? warp_max[lane] : 0u;
        v = __reduce_max_sync(0xFFFFFFFFu, v);
        if (lane == 0 && v != 0u) {
            atomicMax(amax_bits, v);
            if (v >= 0x7F800000u && err) atomicOr(err, IF4_DEV_NONFINITE);
        }
    }
}

// ts = amax / 2688, 1 for amax == 0, floored at 2^-117 (NaN stays NaN).
__device__ __forceinline__ float tensor_scale_of(float a)
{
    float t = 1.0f;
    if (a != 0.0f) {
        t = __fdiv_rn(a, 2688.0f);
        if (t < kTsFloor) t = kTsFloor;
    }
    return t;
}

__global__ void tensor_scale_kernel(const float *amax, float *ts)
{
    pdl_enter();
    *ts = tensor_scale_of(*amax);
}

// ------------------------------------------- single-launch quantizer ----
//
// amax, tensor scale, IF4 quantize and (optionally) the NVFP4 comparator in
// one cooperative launch: every block is resident, so the blocks can meet
// at a grid barrier between the amax pass and the encode pass.  The encode
// pass reads the tensor a second time; for tensors that fit in the 126 MB
// L2 that read is served from L2.

constexpr unsigned long long kGridWaitNs = 1000000000ull;   // 1 s

// Grid barrier that also produces the tensor scale.  sync[0] counts
// arrivals and sync[1] accumulates the float bits of the tensor amax (one
// 128-byte line, written by the arriving blocks); sync[32] is the generation
// and sync[33] carries ts to the other blocks (another line, polled by the
// waiting blocks, read and written as one 64-bit word).  Each arriving block
// adds its maximum without waiting (a relaxed reduction) and then its
// arrival with acquire-release order, so the last block to arrive sees every
// maximum.  That block computes ts, stores it to *ts_out, puts sync[0] and
// sync[1] back to zero and publishes the next generation together with ts in
// one release store; the others poll that word (bounded) with acquire loads.
// `gen0` is the generation the block read at its start: it cannot move before
// every block, this one included, has arrived.  Called by one thread per
// block.  Returns false (and sets IF4_DEV_TIMEOUT) when the wait runs out.
__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __noinline__ bool grid_tensor_scale(uint32_t *sync, uint32_t gen0,
                                               uint32_t block_max_bits, float *ts_out, int *err,
                                               float &ts)
{
    if (block_max_bits != 0u)
        asm volatile("red.relaxed.gpu.global.max.u32 [%0], %1;"
                     :: "l"(sync + 1), "r"(block_max_bits) : "memory");
    uint32_t arrived;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                 : "=r"(arrived) : "l"(sync) : "memory");
    unsigned long long word;
    if (arrived == gridDim.x - 1) {
        const float t = tensor_scale_of(__uint_as_float(ld_relaxed_gpu(sync + 1)));
        *ts_out = t;
        asm volatile("st.relaxed.gpu.global.u32 [%0], 0;" :: "l"(sync + 1) : "memory");
        asm volatile("st.relaxed.gpu.global.u32 [%0], 0;" :: "l"(sync) : "memory");
        word = ((unsigned long long)__float_as_uint(t) << 32) | (unsigned long long)(gen0 + 1u);
        asm volatile("st.release.gpu.global.b64 [%0], %1;" :: "l"(sync + 32), "l"(word)
                     : "memory");
    } else {
        const unsigned long long t0 = globaltimer_ns();
        for (;;) {
            asm volatile("ld.acquire.gpu.global.b64 %0, [%1];" : "=l"(word) : "l"(sync + 32)
                         : "memory");
            if ((uint32_t)word != gen0) break;
            if (globaltimer_ns() - t0 > kGridWaitNs) {
                if (err) atomicOr(err, IF4_DEV_TIMEOUT);
                return false;
            }
            __nanosleep(100);
        }
    }
    ts = __uint_as_float((uint32_t)(word >> 32));
    return true;
}

// DQ: also write the round trip, the IF4 codes decoded to bf16 y (dense,
// 32-byte aligned), as the dequantizer would decode them.
template <int DT, bool V8, bool RHT, bool NV, bool DQ = false>
__global__ void __launch_bounds__(256, DT == DT_F32 ? 3 : 4)
quantize_fused_kernel(const char *__restrict__ x, int64_t ld_bytes, uint32_t gpr,
                      uint32_t ngroups, int contig, uint8_t *__restrict__ codes,
                      uint8_t *__restrict__ scales, uint8_t *__restrict__ nv_codes,
                      uint8_t *__restrict__ nv_scales, float *ts_out, uint32_t *sync, int *err,
                      const __grid_constant__ SignMasks sm, uint32_t signs,
                      char *__restrict__ y, uint32_t keep_from, int use_l2_policy)
{
    // wait for the previous kernel in the stream (programmatic launch)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const uint32_t gen0 = threadIdx.x == 0 ? ld_relaxed_gpu(sync + 32) : 0u;
    constexpr int GB = 16 * elem_bytes<DT>();
    __shared__ float inv_tab[128];
    __shared__ uint32_t warp_max[8];
    __shared__ float ts_sh;
    __shared__ int ok_sh;
    const uint32_t gpr_eff = contig ? ngroups : gpr;
    auto addr = [&](uint32_t g) -> const char * {
        return contig ? x + (int64_t)g * GB : group_addr<GB>(x, g, gpr, ld_bytes);
    };
    const uint32_t stride = gridDim.x * blockDim.x;
    const uint32_t g_first = blockIdx.x * blockDim.x + threadIdx.x;

    // L2 eviction priorities for a tensor larger than L2 can usefully keep
    // (use_l2_policy): pass 1 reads the groups from keep_from on, the last it
    // reads, with evict_last and the others with evict_first, so that at the
    // barrier L2 holds the tensor's tail; pass 2 walks the tensor backwards,
    // starting on that tail, and reads and writes with evict_first, so the
    // stream of outputs replaces lines already used rather than the tail
    // still to come.  Otherwise every access has the normal priority.
    // pass 1: max |x| (of the transform, with RHT), six loads in flight
    uint32_t m = 0;
    constexpr int U = (DT == DT_F32 || RHT) ? 3 : 6;
    {
    const uint64_t pol_first = use_l2_policy ? l2_evict_first() : l2_evict_normal();
    const uint64_t pol_last = use_l2_policy ? l2_evict_last() : l2_evict_normal();
    for (uint64_t g0 = g_first; g0 < ngroups; g0 += (uint64_t)U * stride) {
        Raw<DT> r[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint64_t g = g0 + (uint64_t)u * stride;
            if (g < ngroups)
                load_group_pol<DT, V8>(addr((uint32_t)g), r[u], g >= keep_from ? pol_last : pol_first);
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (g0 + (uint64_t)u * stride < ngroups) {
                if constexpr (RHT) {
                    f2_t xv[8];
                    bool nf;
                    m = max(m, __float_as_uint(unpack_group_rht<DT, false>(r[u], sm, xv, nf)));
                } else {
                    m = max(m, group_absmax_bits<DT>(r[u]));
                }
            }
    }
    }
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) warp_max[warp] = m;
    const uint64_t pol_first = use_l2_policy ? l2_evict_first() : l2_evict_normal();
    // pass 2 takes the j-th group of pass 1's order from the end: group
    // ngroups - 1 - j.  Its first group does not depend on ts: that load is
    // in flight while the block waits at the grid barrier.
    auto rev = [&](uint32_t j) -> uint32_t { return ngroups - 1u - j; };
    Raw<DT> buf[2];
    uint32_t g = g_first;
    if (g < ngroups) load_group_pol<DT, V8>(addr(rev(g)), buf[0], pol_first);
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) b = max(b, warp_max[w]);
        if (b >= 0x7F800000u && err) atomicOr(err, IF4_DEV_NONFINITE);
        float t = 1.0f;
        ok_sh = grid_tensor_scale(sync, gen0, b, ts_out, err, t) ? 1 : 0;
        ts_sh = t;
    }
    __syncthreads();
    if (!ok_sh) return;

    // pass 2: the encode, as quantize_kernel; the next kernel in the stream
    // may be scheduled as this grid's blocks finish
    pdl_release();
    const float ts = ts_sh;
    if (threadIdx.x < 128) {
        const float eff = __fmul_rn(f32_from_e4m3(threadIdx.x), ts);
        inv_tab[threadIdx.x] = threadIdx.x == 0 ? 0.0f : __frcp_rn(eff);
    }
    __shared__ __align__(128) float lut[DQ ? 32 : 1];
    if (DQ && threadIdx.x < 32) lut[threadIdx.x] = code_value(threadIdx.x);
    const uint32_t lut_addr = (uint32_t)__cvta_generic_to_shared(lut);
    const float rts = __frcp_rn(ts);
    __syncthreads();
    for (; g < ngroups;) {
#pragma unroll
        for (int ph = 0; ph < 2; ++ph) {
            const uint32_t gn = g + stride;
            if (gn < ngroups) load_group_pol<DT, V8>(addr(rev(gn)), buf[ph ^ 1], pol_first);
            quantize_one<DT, Q_IF4, RHT, NV, DQ, true>(buf[ph], rev(g), x, ld_bytes, gpr_eff, ts,
                                                       rts, inv_tab, nullptr, codes, scales, sm,
                                                       signs, nv_codes, nv_scales, y, lut_addr,
                                                       pol_first);
            g = gn;
            if (g >= ngroups) break;
        }
    }
}

// ------------------------------------------------------------ dequantize --

// ODT: output dtype.  UNIT_TS: leave the tensor scale out (the linear's
// operand decode), else multiply by *ts.  One thread per group (lanes of a
// warp own consecutive groups, so loads and stores are contiguous spans); the
// next group's codes and scale are loaded before the current one is decoded.
// 16-bit outputs: the unit-scale fp16 decode (the linear's operands) uses the
// byte-permute group decode, the dequantizer with a tensor scale the
// per-element table; on 134 MB tensors each is the faster of the two for its
// kernel (fp16 decode 31.3 against 31.7 us, bf16 dequantize 29.4 against
// 31.5 us).
template <int ODT, bool UNIT_TS, bool V8>
__global__ void __launch_bounds__(256)
dequantize_kernel(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scales,
                  const float *__restrict__ ts_ptr, uint32_t gpr, uint32_t ngroups,
                  char *__restrict__ y, int64_t ld_bytes, int contig)
{
    pdl_enter();
    constexpr int OB = ODT == DT_F32 ? 4 : 2;
    __shared__ __align__(128) float lut[32];
    if (threadIdx.x < 32) lut[threadIdx.x] = code_value(threadIdx.x);
    const float ts = UNIT_TS ? 1.0f : *ts_ptr;
    const uint32_t lut_addr = (uint32_t)__cvta_generic_to_shared(lut);
    __syncthreads();
    const uint32_t stride = gridDim.x * blockDim.x;
    uint32_t g = blockIdx.x * blockDim.x + threadIdx.x;
    uint32_t a0 = 0, a1 = 0, as = 0, b0 = 0, b1 = 0, bs = 0;
    if (g < ngroups) {
        ld_nc_v2(codes + (int64_t)g * 8, a0, a1);
        as = ld_nc_u8(scales + g);
    }
    // Full rounds of a contiguous output while both loads of the round are
    // in range: no per-group range checks (a0, a1, as hold group g at the top
    // of every round).  With it the kernel takes 39 registers (six resident
    // blocks per SM instead of eight) and runs 8 % faster on 134 MB tensors
    // (about 14 groups per thread); held to 32 registers it gains nothing.
    // Taken from six groups per thread on; at 4096 x 4096 (3-4 groups per
    // thread) the checked loop below does all the work.
    if (contig && ngroups / stride >= 6u) {
        while ((uint64_t)g + 2ull * stride < ngroups) {
            uint32_t gn = g + stride;
            ld_nc_v2(codes + (int64_t)gn * 8, b0, b1);
            bs = ld_nc_u8(scales + gn);
            dequant_group<ODT, UNIT_TS, V8, false, UNIT_TS>(a0, a1, as, ts, lut_addr,
                                                                y + (int64_t)g * (16 * OB));
            g = gn;
            gn = g + stride;
            ld_nc_v2(codes + (int64_t)gn * 8, a0, a1);
            as = ld_nc_u8(scales + gn);
            dequant_group<ODT, UNIT_TS, V8, false, UNIT_TS>(b0, b1, bs, ts, lut_addr,
                                                                y + (int64_t)g * (16 * OB));
            g = gn;
        }
    }
    while (g < ngroups) {
        uint32_t gn = g + stride;
        bool more = gn < ngroups && gn > g;
        if (more) {
            ld_nc_v2(codes + (int64_t)gn * 8, b0, b1);
            bs = ld_nc_u8(scales + gn);
        }
        dequant_group<ODT, UNIT_TS, V8, false, UNIT_TS>(
            a0, a1, as, ts, lut_addr,
            const_cast<char *>(group_ptr(y, g, contig, gpr, ld_bytes, 16 * OB)));
        if (!more) break;
        g = gn;
        gn = g + stride;
        more = gn < ngroups && gn > g;
        if (more) {
            ld_nc_v2(codes + (int64_t)gn * 8, a0, a1);
            as = ld_nc_u8(scales + gn);
        }
        dequant_group<ODT, UNIT_TS, V8, false, UNIT_TS>(
            b0, b1, bs, ts, lut_addr,
            const_cast<char *>(group_ptr(y, g, contig, gpr, ld_bytes, 16 * OB)));
        if (!more) break;
        g = gn;
    }
}

// ------------------------------------------------------------ host side ----

struct DeviceInfo {
    int sm_count = 0;
    int cc_major = 0;
};

bool device_info(DeviceInfo &out)
{
    static std::mutex mu;
    static DeviceInfo cache[64];
    static bool have[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::lock_guard<std::mutex> lock(mu);
    if (!have[dev]) {
        DeviceInfo d;
        if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return false;
        if (cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
            return false;
        cache[dev] = d;
        have[dev] = true;
    }
    out = cache[dev];
    return true;
}

int check_device(DeviceInfo &d)
{
    if (!device_info(d)) return IF4_ERR_CUDA;
    if (d.cc_major != 10) return IF4_ERR_DEVICE;
    return IF4_OK;
}

template <typename K>
int resident_blocks(K kernel, int threads)
{
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, 0) != cudaSuccess || n < 1)
        n = 1;
    return n;
}

int elem_size(int dt)
{
    switch (dt) {
    case IF4_F32: return 4;
    case IF4_BF16: return 2;
    case IF4_F16: return 2;
    default: return 0;
    }
}

struct Shape {
    uint32_t gpr = 0, ngroups = 0;
    int64_t ld_bytes = 0;
    bool contig = false, v8 = false;
};

// Validate a dense input or output tensor description.
int check_tensor(const void *p, int dt, int64_t rows, int64_t cols, int64_t ld, Shape &s)
{
    const int es = elem_size(dt);
    if (es == 0) return IF4_ERR_DTYPE;
    if (rows < 0 || cols < 0 || cols % 16 != 0 || ld < cols) return IF4_ERR_SHAPE;
    if (rows > 0 && (cols / 16) > 0 && rows > (int64_t)0x7FFFFFFF / (cols / 16)) return IF4_ERR_SHAPE;
    if (rows > 0 && cols > 0 && p == nullptr) return IF4_ERR_NULL;
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    if (a % 16 != 0 || (ld * es) % 16 != 0) return IF4_ERR_ALIGN;
    s.gpr = (uint32_t)(cols / 16);
    s.ngroups = (uint32_t)(rows * (cols / 16));
    s.ld_bytes = ld * es;
    s.contig = (ld == cols) || rows <= 1;
    s.v8 = (a % 32 == 0) && (s.ld_bytes % 32 == 0);
    return IF4_OK;
}

int launch_status()
{
    return cudaGetLastError() == cudaSuccess ? IF4_OK : IF4_ERR_CUDA;
}

// Launch of the stream-ordered kernels (amax, scale, quantize, dequantize)
// with programmatic dependent launch: each such kernel lets the next one be
// scheduled while it drains, and waits for its predecessor's results before
// reading anything (pdl_enter), so stream order holds as usual.
template <typename... KArgs, typename... Args>
int launch_k(void (*k)(KArgs...), unsigned grid, unsigned block, cudaStream_t st, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(block, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k, args...) != cudaSuccess) return IF4_ERR_CUDA;
    return launch_status();
}

// Blocks to launch: enough for every work item, capped at one full wave of
// resident blocks (the kernels are grid-stride loops).  `occ` is the number
// of resident blocks per SM, queried once per kernel instantiation.
// The linear's decode of both operands in one launch (internal_decode_f16_pair):
// group g < na is A's group g, the rest B's group g - na; each is decoded as
// if4_decode_f16 decodes it (dequant_group with a unit tensor scale and the
// byte-permute decode) into a dense, 32-byte aligned fp16 array.  The next
// group's codes and scale byte are loaded before the current group is
// decoded.  One launch instead of two saves a ramp and a tail: the operands
// of an 8192 x 4096 x 4096 linear are only 86 and 43 MB.
__global__ void __launch_bounds__(256)
decode_f16_pair_kernel(const uint8_t *__restrict__ ca, const uint8_t *__restrict__ sa,
                       uint32_t na, char *__restrict__ ya, const uint8_t *__restrict__ cb,
                       const uint8_t *__restrict__ sb, uint32_t nb, char *__restrict__ yb)
{
    pdl_enter();
    __shared__ __align__(128) float lut[32];
    if (threadIdx.x < 32) lut[threadIdx.x] = code_value(threadIdx.x);
    const uint32_t lut_addr = (uint32_t)__cvta_generic_to_shared(lut);
    __syncthreads();
    const uint32_t n = na + nb;                 // below 2^31 (checked on the host)
    const uint32_t stride = gridDim.x * blockDim.x;
    auto load = [&](uint32_t g, uint32_t &w0, uint32_t &w1, uint32_t &s) {
        const bool in_a = g < na;
        const uint32_t l = in_a ? g : g - na;
        ld_nc_v2((in_a ? ca : cb) + (int64_t)l * 8, w0, w1);
        s = ld_nc_u8((in_a ? sa : sb) + l);
    };
    uint32_t g = blockIdx.x * blockDim.x + threadIdx.x;
    uint32_t w0 = 0, w1 = 0, s = 0;
    if (g < n) load(g, w0, w1, s);
    for (; g < n; g += stride) {
        const uint32_t c0 = w0, c1 = w1, cs = s;
        if (g + stride < n) load(g + stride, w0, w1, s);
        const bool in_a = g < na;
        char *p = in_a ? ya + (int64_t)g * 32 : yb + (int64_t)(g - na) * 32;
        dequant_group<DT_F16, true, true, false, true>(c0, c1, cs, 1.0f, lut_addr, p);
    }
}

uint32_t grid_for(int occ, const DeviceInfo &d, uint32_t work_items, int threads)
{
    const uint64_t want = ((uint64_t)work_items + threads - 1) / threads;
    const uint64_t cap = (uint64_t)d.sm_count * (uint64_t)occ;
    return (uint32_t)std::max<uint64_t>(1, std::min(want, cap));
}

// Transform request of an entry point: off, or on with a 16-bit sign vector.
struct Rht {
    bool on = false;
    uint32_t signs = 0;
};

SignMasks sign_masks(int dt, uint32_t signs)
{
    SignMasks m{};
    for (int j = 0; j < 16; ++j) {
        if (dt == IF4_F32) {
            m.w[j] = ((signs >> j) & 1u) << 31;
        } else if (j < 8) {
            m.w[j] = (((signs >> (2 * j)) & 1u) << 15) | (((signs >> (2 * j + 1)) & 1u) << 31);
        }
    }
    return m;
}

template <int DT, bool V8, bool RHT>
int launch_amax(const Shape &s, const void *x, unsigned int *amax_bits, int *err,
                cudaStream_t st, const DeviceInfo &d, const SignMasks &sm)
{
    if (s.ngroups == 0) return IF4_OK;
    auto k = amax_kernel<DT, V8, RHT>;
    static const int occ = resident_blocks(k, 256);
    const uint32_t grid = grid_for(occ, d, s.ngroups, 256);
    return launch_k(k, grid, 256, st, static_cast<const char *>(x), s.ld_bytes, s.gpr, s.ngroups,
                    s.contig ? 1 : 0, amax_bits, err, sm);
}

template <int DT, bool RHT>
int dispatch_amax_dt(const Shape &s, const void *x, unsigned int *amax_bits, int *err,
                     cudaStream_t st, const DeviceInfo &d, const SignMasks &sm)
{
    return s.v8 ? launch_amax<DT, true, RHT>(s, x, amax_bits, err, st, d, sm)
                : launch_amax<DT, false, RHT>(s, x, amax_bits, err, st, d, sm);
}

int dispatch_amax(int dt, const Shape &s, const void *x, unsigned int *amax_bits, int *err,
                  cudaStream_t st, const DeviceInfo &d, Rht rht = Rht())
{
    const SignMasks sm = sign_masks(dt, rht.signs);
    switch (dt) {
    case IF4_F32:
        return rht.on ? dispatch_amax_dt<DT_F32, true>(s, x, amax_bits, err, st, d, sm)
                      : dispatch_amax_dt<DT_F32, false>(s, x, amax_bits, err, st, d, sm);
    case IF4_BF16:
        return rht.on ? dispatch_amax_dt<DT_BF16, true>(s, x, amax_bits, err, st, d, sm)
                      : dispatch_amax_dt<DT_BF16, false>(s, x, amax_bits, err, st, d, sm);
    default:
        return rht.on ? dispatch_amax_dt<DT_F16, true>(s, x, amax_bits, err, st, d, sm)
                      : dispatch_amax_dt<DT_F16, false>(s, x, amax_bits, err, st, d, sm);
    }
}

template <int DT, int MODE, bool RHT>
int launch_quant(const Shape &s, const void *x, uint8_t *codes, uint8_t *scales,
                 const float *ts, int *err, int check_ts, cudaStream_t st, const DeviceInfo &d,
                 const SignMasks &sm, uint32_t signs)
{
    if (s.ngroups == 0) return IF4_OK;
    constexpr int PF = (DT != DT_F32 && (MODE == Q_NVFP4 || MODE == Q_NVINT4)) ? 2 : 1;
    auto launch = [&](auto k) {
        static const int occ = resident_blocks(k, 256);
        const uint32_t grid = grid_for(occ, d, s.ngroups, 256);
        return launch_k(k, grid, 256, st, static_cast<const char *>(x), s.ld_bytes, s.gpr,
                        s.ngroups, s.contig ? 1 : 0, codes, scales, ts, err, check_ts, sm, signs);
    };
    return s.v8 ? launch(quantize_kernel<DT, MODE, true, RHT, PF>)
                : launch(quantize_kernel<DT, MODE, false, RHT, PF>);
}

template <int MODE, bool RHT>
int dispatch_quant(int dt, const Shape &s, const void *x, uint8_t *codes, uint8_t *scales,
                   const float *ts, int *err, int check_ts, cudaStream_t st, const DeviceInfo &d,
                   uint32_t signs)
{
    const SignMasks sm = sign_masks(dt, signs);
    switch (dt) {
    case IF4_F32:
        return launch_quant<DT_F32, MODE, RHT>(s, x, codes, scales, ts, err, check_ts, st, d,
                                                    sm, signs);
    case IF4_BF16:
        return launch_quant<DT_BF16, MODE, RHT>(s, x, codes, scales, ts, err, check_ts, st,
                                                     d, sm, signs);
    default:
        return launch_quant<DT_F16, MODE, RHT>(s, x, codes, scales, ts, err, check_ts, st, d,
                                                    sm, signs);
    }
}

template <int MODE, bool RHT = false>
int quantize_entry(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                   uint8_t *codes, uint8_t *scales, float *ts, int ts_mode, int *err_flag,
                   void *stream, uint32_t signs = 0)
{
    Shape s;
    int rc = check_tensor(x, x_dtype, rows, cols, ld_x, s);
    if (rc != IF4_OK) return rc;
    if (ts_mode != IF4_TS_COMPUTE && ts_mode != IF4_TS_GIVEN) return IF4_ERR_MODE;
    if (ts == nullptr) return IF4_ERR_NULL;
    if (s.ngroups > 0 && (codes == nullptr || scales == nullptr)) return IF4_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(codes) % 16 != 0 || reinterpret_cast<uintptr_t>(ts) % 4 != 0)
        return IF4_ERR_ALIGN;
    DeviceInfo d;
    rc = check_device(d);
    if (rc != IF4_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (ts_mode == IF4_TS_COMPUTE) {
        // the amax kernel accumulates max |x| as float bits into *ts, the
        // scale kernel turns it into ts
        if (cudaMemsetAsync(ts, 0, sizeof(float), st) != cudaSuccess) return IF4_ERR_CUDA;
        Rht rht;
        rht.on = RHT;
        rht.signs = signs;
        rc = dispatch_amax(x_dtype, s, x, reinterpret_cast<unsigned int *>(ts), err_flag, st, d,
                           rht);
        if (rc != IF4_OK) return rc;
        rc = launch_k(tensor_scale_kernel, 1, 1, st, (const float *)ts, ts);
        if (rc != IF4_OK) return rc;
    }
    return dispatch_quant<MODE, RHT>(x_dtype, s, x, codes, scales, ts, err_flag,
                                     ts_mode == IF4_TS_GIVEN ? 1 : 0, st, d, signs);
}

// The single-launch quantizer's L2 eviction priorities (see the kernel):
// used for inputs larger than 64 MB, keeping the last 48 MB in L2 for the
// encode pass.  On the 134 MB activation tensor the keep size was swept from
// 32 to 112 MB: 48 MB was fastest, and it cut the launch's DRAM reads from
// 267 to 218 MB.
constexpr uint64_t kL2PolicyMinBytes = 64ull << 20;
constexpr uint64_t kL2KeepBytes = 48ull << 20;

// Single-launch quantizer: a cooperative launch of at most one wave, so
// every block is resident when the blocks meet at the grid barrier.
template <int DT, bool V8, bool RHT, bool NV, bool DQ = false>
int launch_fused(const Shape &s, const void *x, uint8_t *codes, uint8_t *scales,
                 uint8_t *nv_codes, uint8_t *nv_scales, float *ts, uint32_t *sync, int *err,
                 cudaStream_t st, const DeviceInfo &d, const SignMasks &sm, uint32_t signs,
                 void *y = nullptr, int share = 1)
{
    auto k = quantize_fused_kernel<DT, V8, RHT, NV, DQ>;
    static const int occ = resident_blocks(k, 256);
    // a share of the device: floor(occ / share) blocks per SM, so that
    // `share` launches on other streams are resident at the same time
    const uint32_t grid = grid_for(std::max(1, occ / share), d, s.ngroups, 256);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    // L2 eviction priorities for inputs above kL2PolicyMinBytes: the last
    // kL2KeepBytes of the tensor are kept for the encode pass
    const uint64_t in_bytes = (uint64_t)s.ngroups * (uint64_t)(16 * elem_bytes<DT>());
    const bool use_pol = in_bytes > kL2PolicyMinBytes;
    const uint64_t keep_groups = kL2KeepBytes / (uint64_t)(16 * elem_bytes<DT>());
    const uint32_t keep_from = keep_groups >= s.ngroups ? 0u : (uint32_t)(s.ngroups - keep_groups);
    if (cudaLaunchKernelEx(&cfg, k, static_cast<const char *>(x), s.ld_bytes, s.gpr, s.ngroups,
                           s.contig ? 1 : 0, codes, scales, nv_codes, nv_scales, ts, sync, err, sm,
                           signs, static_cast<char *>(y), keep_from, use_pol ? 1 : 0) != cudaSuccess)
        return IF4_ERR_CUDA;
    return launch_status();
}

template <int DT, bool RHT>
int dispatch_fused_dt(const Shape &s, const void *x, uint8_t *codes, uint8_t *scales,
                      uint8_t *nv_codes, uint8_t *nv_scales, float *ts, uint32_t *sync, int *err,
                      cudaStream_t st, const DeviceInfo &d, const SignMasks &sm, uint32_t signs,
                      void *y, int share)
{
    const bool nv = nv_codes != nullptr;
    if constexpr (!RHT) {
        if (y != nullptr) {
            if (s.v8)
                return nv ? launch_fused<DT, true, false, true, true>(
                                s, x, codes, scales, nv_codes, nv_scales, ts, sync, err, st, d, sm,
                                signs, y, share)
                          : launch_fused<DT, true, false, false, true>(
                                s, x, codes, scales, nv_codes, nv_scales, ts, sync, err, st, d, sm,
                                signs, y, share);
            return nv ? launch_fused<DT, false, false, true, true>(
                            s, x, codes, scales, nv_codes, nv_scales, ts, sync, err, st, d, sm,
                            signs, y, share)
                      : launch_fused<DT, false, false, false, true>(
                            s, x, codes, scales, nv_codes, nv_scales, ts, sync, err, st, d, sm,
                            signs, y, share);
        }
    }
    if (s.v8)
        return nv ? launch_fused<DT, true, RHT, true>(s, x, codes, scales, nv_codes, nv_scales, ts,
                                                      sync, err, st, d, sm, signs, nullptr,
                                                      share)
                  : launch_fused<DT, true, RHT, false>(s, x, codes, scales, nv_codes, nv_scales,
                                                       ts, sync, err, st, d, sm, signs, nullptr,
                                                       share);
    return nv ? launch_fused<DT, false, RHT, true>(s, x, codes, scales, nv_codes, nv_scales, ts,
                                                   sync, err, st, d, sm, signs, nullptr, share)
              : launch_fused<DT, false, RHT, false>(s, x, codes, scales, nv_codes, nv_scales, ts,
                                                    sync, err, st, d, sm, signs, nullptr, share);
}

template <int ODT, bool UNIT_TS>
int launch_dequant(const Shape &s, const uint8_t *codes, const uint8_t *scales, const float *ts,
                   void *y, cudaStream_t st, const DeviceInfo &d)
{
    if (s.ngroups == 0) return IF4_OK;
    auto launch = [&](auto k) {
        static const int occ = resident_blocks(k, 256);
        const uint32_t grid = grid_for(occ, d, s.ngroups, 256);
        return launch_k(k, grid, 256, st, codes, scales, ts, s.gpr, s.ngroups,
                        static_cast<char *>(y), s.ld_bytes, s.contig ? 1 : 0);
    };
    // 32-byte aligned base and rows: 256-bit stores
    return s.v8 ? launch(dequantize_kernel<ODT, UNIT_TS, true>)
                : launch(dequantize_kernel<ODT, UNIT_TS, false>);
}

template <bool RHT>
int fused_entry(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                uint8_t *codes, uint8_t *scales, uint8_t *nv_codes, uint8_t *nv_scales, float *ts,
                uint32_t *sync_words, int *err_flag, void *stream, uint32_t signs,
                void *y = nullptr, int share = 1)
{
    Shape s;
    int rc = check_tensor(x, x_dtype, rows, cols, ld_x, s);
    if (rc != IF4_OK) return rc;
    if (share < 1 || share > 64) return IF4_ERR_SHAPE;
    if (ts == nullptr || sync_words == nullptr) return IF4_ERR_NULL;
    if ((nv_codes == nullptr) != (nv_scales == nullptr)) return IF4_ERR_NULL;
    if (s.ngroups > 0 && (codes == nullptr || scales == nullptr)) return IF4_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(codes) % 16 != 0 ||
        reinterpret_cast<uintptr_t>(nv_codes) % 16 != 0 ||
        reinterpret_cast<uintptr_t>(ts) % 4 != 0 || reinterpret_cast<uintptr_t>(sync_words) % 256 != 0)
        return IF4_ERR_ALIGN;
    DeviceInfo d;
    rc = check_device(d);
    if (rc != IF4_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (s.ngroups == 0) {
        // an empty tensor: amax 0, ts 1, nothing to encode
        if (cudaMemsetAsync(ts, 0, sizeof(float), st) != cudaSuccess) return IF4_ERR_CUDA;
        return launch_k(tensor_scale_kernel, 1, 1, st, (const float *)ts, ts);
    }
    const SignMasks sm = sign_masks(x_dtype, signs);
    switch (x_dtype) {
    case IF4_F32:
        return dispatch_fused_dt<DT_F32, RHT>(s, x, codes, scales, nv_codes, nv_scales, ts,
                                                sync_words, err_flag, st, d, sm, signs, y, share);
    case IF4_BF16:
        return dispatch_fused_dt<DT_BF16, RHT>(s, x, codes, scales, nv_codes, nv_scales, ts,
                                                 sync_words, err_flag, st, d, sm, signs, y, share);
    default:
        return dispatch_fused_dt<DT_F16, RHT>(s, x, codes, scales, nv_codes, nv_scales, ts,
                                                sync_words, err_flag, st, d, sm, signs, y, share);
    }
}

}  // namespace

// ================================================================ C ABI ====

extern "C" {

int if4_tensor_amax(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                    float *amax, int *err_flag, void *stream)
{
    Shape s;
    int rc = check_tensor(x, x_dtype, rows, cols, ld_x, s);
    if (rc != IF4_OK) return rc;
    if (amax == nullptr) return IF4_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(amax) % 4 != 0) return IF4_ERR_ALIGN;
    DeviceInfo d;
    rc = check_device(d);
    if (rc != IF4_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(amax, 0, sizeof(float), st) != cudaSuccess) return IF4_ERR_CUDA;
    return dispatch_amax(x_dtype, s, x, reinterpret_cast<unsigned int *>(amax), err_flag, st, d);
}

int if4_tensor_scale(const float *amax, float *ts, void *stream)
{
    if (amax == nullptr || ts == nullptr) return IF4_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(amax) % 4 != 0 || reinterpret_cast<uintptr_t>(ts) % 4 != 0)
        return IF4_ERR_ALIGN;
    DeviceInfo d;
    int rc = check_device(d);
    if (rc != IF4_OK) return rc;
    return launch_k(tensor_scale_kernel, 1, 1, static_cast<cudaStream_t>(stream), amax, ts);
}

int if4_quantize(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                 uint8_t *codes, uint8_t *scales, float *ts, int ts_mode, int *err_flag,
                 void *stream)
{
    return quantize_entry<Q_IF4>(x, x_dtype, rows, cols, ld_x, codes, scales, ts, ts_mode,
                                 err_flag, stream);
}

int nvfp4_quantize(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                   uint8_t *codes, uint8_t *scales, float *ts, int ts_mode, int *err_flag,
                   void *stream)
{
    return quantize_entry<Q_NVFP4>(x, x_dtype, rows, cols, ld_x, codes, scales, ts, ts_mode,
                                   err_flag, stream);
}

int nvint4_quantize(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                    uint8_t *codes, uint8_t *scales, float *ts, int ts_mode, int *err_flag,
                    void *stream)
{
    return quantize_entry<Q_NVINT4>(x, x_dtype, rows, cols, ld_x, codes, scales, ts, ts_mode,
                                    err_flag, stream);
}

int nvfp4_4over6_quantize(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                          uint8_t *codes, uint8_t *scales, float *ts, int ts_mode, int *err_flag,
                          void *stream)
{
    return quantize_entry<Q_46>(x, x_dtype, rows, cols, ld_x, codes, scales, ts, ts_mode,
                                err_flag, stream);
}

int if4_tensor_amax_rht(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                        uint32_t signs, float *amax, int *err_flag, void *stream)
{
    Shape s;
    int rc = check_tensor(x, x_dtype, rows, cols, ld_x, s);
    if (rc != IF4_OK) return rc;
    if (amax == nullptr) return IF4_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(amax) % 4 != 0) return IF4_ERR_ALIGN;
    DeviceInfo d;
    rc = check_device(d);
    if (rc != IF4_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(amax, 0, sizeof(float), st) != cudaSuccess) return IF4_ERR_CUDA;
    Rht rht;
    rht.on = true;
    rht.signs = signs & 0xFFFFu;
    return dispatch_amax(x_dtype, s, x, reinterpret_cast<unsigned int *>(amax), err_flag, st, d,
                         rht);
}

int if4_quantize_rht(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                     uint32_t signs, uint8_t *codes, uint8_t *scales, float *ts, int ts_mode,
                     int *err_flag, void *stream)
{
    return quantize_entry<Q_IF4, true>(x, x_dtype, rows, cols, ld_x, codes, scales, ts, ts_mode,
                                       err_flag, stream, signs & 0xFFFFu);
}

int if4_quantize_fused(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                       uint8_t *codes, uint8_t *scales, uint8_t *nv_codes, uint8_t *nv_scales,
                       float *ts, uint32_t *sync_words, int *err_flag, void *stream)
{
    return fused_entry<false>(x, x_dtype, rows, cols, ld_x, codes, scales, nv_codes, nv_scales, ts,
                              sync_words, err_flag, stream, 0u);
}

int if4_quantize_fused_shared(const void *x, int x_dtype, int64_t rows, int64_t cols,
                              int64_t ld_x, uint8_t *codes, uint8_t *scales, uint8_t *nv_codes,
                              uint8_t *nv_scales, float *ts, uint32_t *sync_words, int share,
                              int *err_flag, void *stream)
{
    return fused_entry<false>(x, x_dtype, rows, cols, ld_x, codes, scales, nv_codes, nv_scales, ts,
                              sync_words, err_flag, stream, 0u, nullptr, share);
}

int if4_quantize_fused_dequant(const void *x, int x_dtype, int64_t rows, int64_t cols,
                               int64_t ld_x, uint8_t *codes, uint8_t *scales, uint8_t *nv_codes,
                               uint8_t *nv_scales, float *ts, uint32_t *sync_words, void *y,
                               int *err_flag, void *stream)
{
    if (rows > 0 && cols > 0 && y == nullptr) return IF4_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(y) % 32 != 0) return IF4_ERR_ALIGN;
    return fused_entry<false>(x, x_dtype, rows, cols, ld_x, codes, scales, nv_codes, nv_scales, ts,
                              sync_words, err_flag, stream, 0u, y);
}

int if4_quantize_fused_dequant_shared(const void *x, int x_dtype, int64_t rows, int64_t cols,
                                      int64_t ld_x, uint8_t *codes, uint8_t *scales,
                                      uint8_t *nv_codes, uint8_t *nv_scales, float *ts,
                                      uint32_t *sync_words, void *y, int share, int *err_flag,
                                      void *stream)
{
    if (rows > 0 && cols > 0 && y == nullptr) return IF4_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(y) % 32 != 0) return IF4_ERR_ALIGN;
    return fused_entry<false>(x, x_dtype, rows, cols, ld_x, codes, scales, nv_codes, nv_scales, ts,
                              sync_words, err_flag, stream, 0u, y, share);
}

int if4_quantize_fused_rht(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                           uint32_t signs, uint8_t *codes, uint8_t *scales, uint8_t *nv_codes,
                           uint8_t *nv_scales, float *ts, uint32_t *sync_words, int *err_flag,
                           void *stream)
{
    return fused_entry<true>(x, x_dtype, rows, cols, ld_x, codes, scales, nv_codes, nv_scales, ts,
                             sync_words, err_flag, stream, signs & 0xFFFFu);
}

int if4_quantize_fused_rht_shared(const void *x, int x_dtype, int64_t rows, int64_t cols,
                                  int64_t ld_x, uint32_t signs, uint8_t *codes, uint8_t *scales,
                                  uint8_t *nv_codes, uint8_t *nv_scales, float *ts,
                                  uint32_t *sync_words, int share, int *err_flag, void *stream)
{
    return fused_entry<true>(x, x_dtype, rows, cols, ld_x, codes, scales, nv_codes, nv_scales, ts,
                             sync_words, err_flag, stream, signs & 0xFFFFu, nullptr, share);
}

int if4_dequantize(const uint8_t *codes, const uint8_t *scales, const float *ts, int64_t rows,
                   int64_t cols, void *y, int y_dtype, int64_t ld_y, void *stream)
{
    Shape s;
    int rc = check_tensor(y, y_dtype, rows, cols, ld_y, s);
    if (rc != IF4_OK) return rc;
    if (ts == nullptr) return IF4_ERR_NULL;
    if (s.ngroups > 0 && (codes == nullptr || scales == nullptr)) return IF4_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(codes) % 16 != 0 || reinterpret_cast<uintptr_t>(ts) % 4 != 0)
        return IF4_ERR_ALIGN;
    DeviceInfo d;
    rc = check_device(d);
    if (rc != IF4_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (y_dtype) {
    case IF4_F32: return launch_dequant<DT_F32, false>(s, codes, scales, ts, y, st, d);
    case IF4_BF16: return launch_dequant<DT_BF16, false>(s, codes, scales, ts, y, st, d);
    default: return launch_dequant<DT_F16, false>(s, codes, scales, ts, y, st, d);
    }
}

}  // extern "C"

int internal_decode_f16_pair(const uint8_t *a_codes, const uint8_t *a_scales, int64_t a_rows,
                             void *a_y, const uint8_t *b_codes, const uint8_t *b_scales,
                             int64_t b_rows, void *b_y, int64_t cols, void *stream)
{
    const int64_t na = a_rows * (cols / 16), nb = b_rows * (cols / 16);
    const bool aligned = reinterpret_cast<uintptr_t>(a_codes) % 16 == 0 &&
                         reinterpret_cast<uintptr_t>(b_codes) % 16 == 0 &&
                         reinterpret_cast<uintptr_t>(a_y) % 32 == 0 &&
                         reinterpret_cast<uintptr_t>(b_y) % 32 == 0;
    if (na + nb >= (int64_t)1 << 31 || !aligned || cols % 16 != 0 || na <= 0 || nb <= 0) {
        // two launches of the public decode
        int rc = if4_decode_f16(a_codes, a_scales, a_rows, cols, a_y, stream);
        return rc != IF4_OK ? rc : if4_decode_f16(b_codes, b_scales, b_rows, cols, b_y, stream);
    }
    if (!a_codes || !a_scales || !b_codes || !b_scales || !a_y || !b_y) return IF4_ERR_NULL;
    DeviceInfo d;
    int rc = check_device(d);
    if (rc != IF4_OK) return rc;
    static const int occ = resident_blocks(decode_f16_pair_kernel, 256);
    const uint32_t grid = grid_for(occ, d, (uint32_t)(na + nb), 256);
    return launch_k(decode_f16_pair_kernel, grid, 256, static_cast<cudaStream_t>(stream), a_codes,
                    a_scales, (uint32_t)na, static_cast<char *>(a_y), b_codes, b_scales,
                    (uint32_t)nb, static_cast<char *>(b_y));
}

extern "C" {

int if4_decode_f16(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t cols,
                   void *y, void *stream)
{
    Shape s;
    int rc = check_tensor(y, IF4_F16, rows, cols, cols, s);
    if (rc != IF4_OK) return rc;
    if (s.ngroups > 0 && (codes == nullptr || scales == nullptr)) return IF4_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(codes) % 16 != 0) return IF4_ERR_ALIGN;
    DeviceInfo d;
    rc = check_device(d);
    if (rc != IF4_OK) return rc;
    return launch_dequant<DT_F16, true>(s, codes, scales, nullptr, y,
                                        static_cast<cudaStream_t>(stream), d);
}

const char *if4_status_str(int status)
{
    switch (status) {
    case IF4_OK: return "ok";
    case IF4_ERR_NULL: return "a required pointer is NULL";
    case IF4_ERR_SHAPE: return "invalid shape (cols % 16, negative size, ld < cols, or too large)";
    case IF4_ERR_DTYPE: return "unknown dtype";
    case IF4_ERR_ALIGN: return "misaligned pointer or leading dimension";
    case IF4_ERR_MODE: return "unknown ts_mode";
    case IF4_ERR_WORKSPACE: return "workspace missing or too small";
    case IF4_ERR_CUDA: return "CUDA call or kernel launch failed";
    case IF4_ERR_DEVICE: return "current device is not sm_100 (B200)";
    default: return "unknown status";
    }
}

int if4_version(void) { return 100; }

}  // extern "C"
