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
// Work decomposition: the path is HBM-bound (2.5625 B per bf16 element for
// quantize), so one thread owns one whole group: a 256-bit load brings its 16
// bf16 values, every reduction (amax, both squared-error sums) stays in the
// thread's registers, and the outputs are one 8-byte code store and one scale
// byte.  Lanes of a warp own consecutive groups, so each warp-wide load or
// store touches one contiguous span.  A grid-stride loop keeps the next
// group's load in flight while the current one is computed.

#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/if4.h"
#include "if4_device.cuh"

using namespace if4dev;

namespace {

// fl(7/6) and fl(6/7) in binary32, and 1.5 * 2^23: adding it to |t| < 2^22
// leaves round-to-nearest-even(t) in the low mantissa bits.
__device__ __forceinline__ float c76() { return __uint_as_float(0x3F955555u); }
__device__ __forceinline__ float c67() { return __uint_as_float(0x3F5B6DB7u); }
constexpr float kMagic = 12582912.0f;
constexpr uint32_t kMagicBits = 0x4B400000u;

constexpr float kTsFloor = 0x1p-117f;
constexpr float kTsCeil = 0x1p117f;

enum { DT_F32 = IF4_F32, DT_BF16 = IF4_BF16, DT_F16 = IF4_F16 };

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

// Unpack to 8 float pairs (element 2j low, 2j+1 high) and the group's max |x|
// as float bits; *nonfinite is set for Inf/NaN.
template <int DT>
__device__ __forceinline__ float unpack_group(const Raw<DT> &r, f2_t (&x)[8], bool &nonfinite)
{
    if constexpr (DT == DT_F32) {
        uint32_t m = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            uint32_t a = r.w[2 * j], b = r.w[2 * j + 1];
            m = max(m, max(a & 0x7FFFFFFFu, b & 0x7FFFFFFFu));
            x[j] = f2_pack(__uint_as_float(a), __uint_as_float(b));
        }
        nonfinite = m >= 0x7F800000u;
        return __uint_as_float(m);
    } else {
        uint32_t m = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            uint32_t w = r.w[j];
            m = max_u16x2(m, w & 0x7FFF7FFFu);
            if constexpr (DT == DT_BF16)
                x[j] = f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
            else
                x[j] = f2_pack(f16lo_to_f32(w), f16hi_to_f32(w));
        }
        uint32_t m16 = max(m & 0xFFFFu, m >> 16);
        if constexpr (DT == DT_BF16) {
            nonfinite = m16 >= 0x7F80u;
            return __uint_as_float(m16 << 16);
        } else {
            nonfinite = m16 >= 0x7C00u;
            return f16lo_to_f32(m16);
        }
    }
}

// ------------------------------------------------------- the quantizer ----

// FP4 candidate of an element pair: the byte of two E2M1 nibbles (element
// 2j low) and the two decoded values.
__device__ __forceinline__ void fp4_pair(f2_t v, uint32_t &byte, f2_t &qf)
{
    float v0, v1;
    f2_unpack(v, v0, v1);
    byte = e2m1x2_from_f32(v0, v1);
    const uint32_t h = f16x2_from_e2m1x2(byte);
    qf = f2_pack(f16lo_to_f32(h), f16hi_to_f32(h));
}

// INT4 candidate of an element pair: r = 1.5*2^23 + RNE(v * fl(7/6)), one
// fused multiply-add, so the integer is the exact product rounded once (bits
// 0-3 of r are the nibble); qi = fl(k * fl(6/7)) = fl(6k/7) for |k| <= 7.
template <bool CLAMP>
__device__ __forceinline__ void int4_pair(f2_t v, f2_t &r, f2_t &qi)
{
    const f2_t C76 = f2_pack(c76(), c76());
    const f2_t M = f2_pack(kMagic, kMagic);
    r = f2_fma(v, C76, M);
    if constexpr (CLAMP) {
        float r0, r1;
        f2_unpack(r, r0, r1);
        r0 = fminf(fmaxf(r0, kMagic - 7.0f), kMagic + 7.0f);
        r1 = fminf(fmaxf(r1, kMagic - 7.0f), kMagic + 7.0f);
        r = f2_pack(r0, r1);
    }
    const f2_t C67 = f2_pack(c67(), c67());
    qi = f2_mul(f2_sub(r, M), C67);
}

// Pack the low nibbles of 8 magic-biased floats (elements 0..7) into a word,
// element 0 in bits 0-3.
__device__ __forceinline__ uint32_t pack_int4_nibbles(const f2_t (&r)[4])
{
    uint32_t e[4], o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float a, b;
        f2_unpack(r[j], a, b);
        e[j] = __float_as_uint(a);
        o[j] = __float_as_uint(b);
    }
    // gather byte 0 of each: even elements -> E, odd elements -> O
    uint32_t E = prmt(prmt(e[0], e[1], 0x0040u), prmt(e[2], e[3], 0x0040u), 0x5410u);
    uint32_t O = prmt(prmt(o[0], o[1], 0x0040u), prmt(o[2], o[3], 0x0040u), 0x5410u);
    return (E & 0x0F0F0F0Fu) | ((O << 4) & 0xF0F0F0F0u);
}

// Binary64 squared-error sums of both candidates in element order: the
// decision rule itself, used only when the binary32 margin of a group is too
// small to trust.  It re-reads the group's 16 inputs (still in L2) and walks
// them one by one, so the common path keeps no extra registers for it.  The
// INT4 integer is always clamped here; the clamp is the identity whenever the
// fast path skipped it.
template <int DT>
__device__ __noinline__ bool int4_wins_exact(const char *p, float inv)
{
    double ef = 0.0, ei = 0.0;
#pragma unroll 1
    for (int i = 0; i < 16; ++i) {
        float x;
        if constexpr (DT == DT_F32)
            x = __ldg(reinterpret_cast<const float *>(p) + i);
        else if constexpr (DT == DT_BF16)
            x = __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short *>(p) + i) << 16);
        else
            x = __half2float(__ushort_as_half(__ldg(reinterpret_cast<const unsigned short *>(p) + i)));
        const float v = __fmul_rn(x, inv);
        const uint32_t h = f16x2_from_e2m1x2(e2m1x2_from_f32(v, 0.0f));
        const float qf = f16lo_to_f32(h);
        float r = __fmaf_rn(v, c76(), kMagic);
        r = fminf(fmaxf(r, kMagic - 7.0f), kMagic + 7.0f);
        const float qi = __fmul_rn(__fsub_rn(r, kMagic), c67());
        const double df = __dsub_rn((double)v, (double)qf);
        const double di = __dsub_rn((double)v, (double)qi);
        ef = __dadd_rn(ef, __dmul_rn(df, df));
        ei = __dadd_rn(ei, __dmul_rn(di, di));
    }
    return ei < ef;
}

struct GroupCode {
    uint32_t c0, c1;   // codes of elements 0..7 and 8..15
    uint32_t scale;    // scale byte
};

// Encode one group from its 16 inputs x (pairs), the block scale byte sb, the
// reciprocal inv of the decoded scale and vmax = fl(amax * inv).
//
// Decision, fast path: each squared error is accumulated in binary32 from
// d = fma(x, -inv, q), an explicit single rounding of q - x*inv (the square
// does not see the sign).  Against the rule's d = v - q with v = fl(x*inv),
// every d is off by at most half an ulp of v plus one rounding, and each sum
// by at most 9 roundings; with Cauchy-Schwarz and vmax*sqrt(S) <= (vmax^2 +
// S)/2 the difference of the two sums is off by less than 2^-20 S + 2^-21
// vmax^2 + 2^-140.  Outside the band 2^-18 S + 2^-19 vmax^2 + 2^-126 the sign
// of the binary32 difference is therefore the sign of the binary64 rule;
// inside it the group is decided by the rule itself.
template <int DT, bool IF4, bool CLAMP>
__device__ __forceinline__ GroupCode encode_group(const f2_t (&x)[8], uint32_t sb, float inv,
                                                float vmax, const char *p)
{
    const f2_t INV = f2_pack(inv, inv);
    const f2_t NINV = f2_pack(-inv, -inv);
    uint32_t fp4[8];
    f2_t r[8];
    f2_t ef = f2_pack(0.0f, 0.0f), ei = f2_pack(0.0f, 0.0f);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const f2_t v = f2_mul(x[j], INV);
        f2_t qf;
        fp4_pair(v, fp4[j], qf);
        if constexpr (IF4) {
            f2_t qi;
            int4_pair<CLAMP>(v, r[j], qi);
            const f2_t df = f2_fma(x[j], NINV, qf);
            const f2_t di = f2_fma(x[j], NINV, qi);
            ef = f2_fma(df, df, ef);
            ei = f2_fma(di, di, ei);
        }
    }
    GroupCode out;
    out.c0 = fp4[0] | (fp4[1] << 8) | (fp4[2] << 16) | (fp4[3] << 24);
    out.c1 = fp4[4] | (fp4[5] << 8) | (fp4[6] << 16) | (fp4[7] << 24);
    out.scale = sb;
    if constexpr (IF4) {
        float a0, a1, b0, b1;
        f2_unpack(ef, a0, a1);
        f2_unpack(ei, b0, b1);
        const float e_fp = __fadd_rn(a0, a1), e_int = __fadd_rn(b0, b1);
        const float d = __fsub_rn(e_fp, e_int);
        const float band = __fmaf_rn(__fadd_rn(e_fp, e_int), 0x1p-18f,
                                     __fmaf_rn(__fmul_rn(vmax, vmax), 0x1p-19f, 0x1p-126f));
        bool int4;
        if (fabsf(d) > band)
            int4 = d > 0.0f;
        else
            int4 = int4_wins_exact<DT>(p, inv);
        if (int4) {
            const f2_t lo[4] = {r[0], r[1], r[2], r[3]};
            const f2_t hi[4] = {r[4], r[5], r[6], r[7]};
            out.c0 = pack_int4_nibbles(lo);
            out.c1 = pack_int4_nibbles(hi);
            out.scale = sb | 0x80u;
        }
    }
    return out;
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

template <int DT, bool IF4, bool V8>
__global__ void __launch_bounds__(256)
quantize_kernel(const char *__restrict__ x, int64_t ld_bytes, uint32_t gpr, uint32_t ngroups,
                int contig, uint8_t *__restrict__ codes, uint8_t *__restrict__ scales,
                const float *__restrict__ ts_ptr, int *err, int check_ts)
{
    constexpr int GB = 16 * elem_bytes<DT>();
    const float ts = *ts_ptr;
    if (check_ts && blockIdx.x == 0 && threadIdx.x == 0 && !ts_valid(ts) && err)
        atomicOr(err, IF4_DEV_BAD_SCALE);

    const uint32_t stride = gridDim.x * blockDim.x;
    uint32_t g = blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= ngroups) return;
    Raw<DT> cur;
    load_group<DT, V8>(group_ptr(x, g, contig, gpr, ld_bytes, GB), cur);
    bool saw_nonfinite = false;
    for (;;) {
        const uint32_t gn = g + stride;
        const bool more = gn < ngroups && gn > g;
        Raw<DT> nxt;
        if (more) load_group<DT, V8>(group_ptr(x, gn, contig, gpr, ld_bytes, GB), nxt);

        f2_t xv[8];
        bool nonfinite;
        const float amax = unpack_group<DT>(cur, xv, nonfinite);
        saw_nonfinite |= nonfinite;

        // A3: block scale
        const float sb_f = __fdiv_rn(__fdiv_rn(amax, 6.0f), ts);
        const uint32_t sb = e4m3_from_f32(sb_f);
        GroupCode out;
        if (sb == 0) {
            out.c0 = out.c1 = 0u;
            out.scale = 0u;
        } else {
            const float eff = __fmul_rn(f32_from_e4m3(sb), ts);
            const float inv = __frcp_rn(eff);
            const float vmax = __fmul_rn(amax, inv);
            const char *gp = group_ptr(x, g, contig, gpr, ld_bytes, GB);
            // The INT4 integer needs a clamp only if some |v| * fl(7/6) can
            // reach 7.5; |v| is monotonic in |x|, so the group's max decides.
            if (__fmul_rn(vmax, c76()) >= 7.5f)
                out = encode_group<DT, IF4, true>(xv, sb, inv, vmax, gp);
            else
                out = encode_group<DT, IF4, false>(xv, sb, inv, vmax, gp);
        }
        st_v2(codes + (int64_t)g * 8, out.c0, out.c1);
        st_u8(scales + g, out.scale);

        if (!more) break;
        g = gn;
        cur = nxt;
    }
    if (saw_nonfinite && err) atomicOr(err, IF4_DEV_NONFINITE);
}

// --------------------------------------------------------- A1 and A2 ----

template <int DT, bool V8>
__global__ void __launch_bounds__(256)
amax_kernel(const char *__restrict__ x, int64_t ld_bytes, uint32_t gpr, uint32_t ngroups,
            int contig, unsigned int *amax_bits, int *err)
{
    constexpr int GB = 16 * elem_bytes<DT>();
    uint32_t m = 0;   // float bits of the running max |x|
    const uint32_t stride = gridDim.x * blockDim.x;
    for (uint32_t g = blockIdx.x * blockDim.x + threadIdx.x; g < ngroups; g += stride) {
        Raw<DT> r;
        load_group<DT, V8>(group_ptr(x, g, contig, gpr, ld_bytes, GB), r);
        if constexpr (DT == DT_F32) {
#pragma unroll
            for (int i = 0; i < 16; ++i) m = max(m, r.w[i] & 0x7FFFFFFFu);
        } else {
            uint32_t h = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) h = max_u16x2(h, r.w[i] & 0x7FFF7FFFu);
            uint32_t h16 = max(h & 0xFFFFu, h >> 16);
            uint32_t f = (DT == DT_BF16) ? (h16 << 16) : __float_as_uint(f16lo_to_f32(h16));
            m = max(m, f);
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
__global__ void tensor_scale_kernel(const float *amax, float *ts)
{
    const float a = *amax;
    float t = 1.0f;
    if (a != 0.0f) {
        t = __fdiv_rn(a, 2688.0f);
        if (t < kTsFloor) t = kTsFloor;
    }
    *ts = t;
}

// ------------------------------------------------------------ A7 / K4 ----

template <int ODT>
__device__ __forceinline__ uint32_t pack_out2(float a, float b)
{
    if constexpr (ODT == DT_BF16) return bf16x2_from_f32(a, b);
    else return f16x2_from_f32(a, b);
}

// Decode 8 nibbles of one code word to 8 floats times eff.
__device__ __forceinline__ void decode_word(uint32_t w, bool is_int, float eff, float (&y)[8])
{
    if (is_int) {
        // (nibble ^ 8) = k + 8 placed in the mantissa of 2^23 * 1.5: exact
        const float bias = kMagic + 8.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t n = ((w >> (4 * i)) & 0xFu) ^ 0x8u;
            const float k = __fsub_rn(__uint_as_float(kMagicBits | n), bias);
            y[i] = __fmul_rn(__fmul_rn(k, c67()), eff);
        }
    } else {
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const uint32_t h = f16x2_from_e2m1x2((w >> (8 * b)) & 0xFFu);
            y[2 * b] = __fmul_rn(f16lo_to_f32(h), eff);
            y[2 * b + 1] = __fmul_rn(f16hi_to_f32(h), eff);
        }
    }
}

// ODT: output dtype.  UNIT_TS: leave the tensor scale out (the linear's
// operand decode), else multiply by *ts.
template <int ODT, bool UNIT_TS>
__global__ void __launch_bounds__(256)
dequantize_kernel(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scales,
                  const float *__restrict__ ts_ptr, uint32_t gpr, uint32_t ngroups,
                  char *__restrict__ y, int64_t ld_bytes, int contig)
{
    constexpr int OB = ODT == DT_F32 ? 4 : 2;
    const float ts = UNIT_TS ? 1.0f : *ts_ptr;
    const uint32_t stride = gridDim.x * blockDim.x;
    for (uint32_t g = blockIdx.x * blockDim.x + threadIdx.x; g < ngroups; g += stride) {
        uint32_t w0, w1;
        ld_nc_v2(codes + (int64_t)g * 8, w0, w1);
        const uint32_t sb = ld_nc_u8(scales + g);
        const float e4 = f32_from_e4m3(sb);
        const float eff = UNIT_TS ? e4 : __fmul_rn(e4, ts);
        const bool is_int = (sb & 0x80u) != 0u;
        float ya[8], yb[8];
        decode_word(w0, is_int, eff, ya);
        decode_word(w1, is_int, eff, yb);
        char *p = const_cast<char *>(group_ptr(y, g, contig, gpr, ld_bytes, 16 * OB));
        if constexpr (ODT == DT_F32) {
            uint32_t a[8], b[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) { a[i] = __float_as_uint(ya[i]); b[i] = __float_as_uint(yb[i]); }
            st_v4(p, a[0], a[1], a[2], a[3]);
            st_v4(p + 16, a[4], a[5], a[6], a[7]);
            st_v4(p + 32, b[0], b[1], b[2], b[3]);
            st_v4(p + 48, b[4], b[5], b[6], b[7]);
        } else {
            st_v4(p, pack_out2<ODT>(ya[0], ya[1]), pack_out2<ODT>(ya[2], ya[3]),
                  pack_out2<ODT>(ya[4], ya[5]), pack_out2<ODT>(ya[6], ya[7]));
            st_v4(p + 16, pack_out2<ODT>(yb[0], yb[1]), pack_out2<ODT>(yb[2], yb[3]),
                  pack_out2<ODT>(yb[4], yb[5]), pack_out2<ODT>(yb[6], yb[7]));
        }
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

template <typename K>
uint32_t grid_for(K kernel, const DeviceInfo &d, uint32_t work_items, int threads)
{
    static_assert(sizeof(K) > 0, "");
    const int occ = resident_blocks(kernel, threads);
    const uint64_t want = ((uint64_t)work_items + threads - 1) / threads;
    const uint64_t cap = (uint64_t)d.sm_count * (uint64_t)occ;
    return (uint32_t)std::max<uint64_t>(1, std::min(want, cap));
}

template <int DT, bool V8>
int launch_amax(const Shape &s, const void *x, unsigned int *amax_bits, int *err,
                cudaStream_t st, const DeviceInfo &d)
{
    if (s.ngroups == 0) return IF4_OK;
    auto k = amax_kernel<DT, V8>;
    const uint32_t grid = grid_for(k, d, s.ngroups, 256);
    k<<<grid, 256, 0, st>>>(static_cast<const char *>(x), s.ld_bytes, s.gpr, s.ngroups,
                            s.contig ? 1 : 0, amax_bits, err);
    return launch_status();
}

int dispatch_amax(int dt, const Shape &s, const void *x, unsigned int *amax_bits, int *err,
                  cudaStream_t st, const DeviceInfo &d)
{
    switch (dt) {
    case IF4_F32: return s.v8 ? launch_amax<DT_F32, true>(s, x, amax_bits, err, st, d)
                              : launch_amax<DT_F32, false>(s, x, amax_bits, err, st, d);
    case IF4_BF16: return s.v8 ? launch_amax<DT_BF16, true>(s, x, amax_bits, err, st, d)
                               : launch_amax<DT_BF16, false>(s, x, amax_bits, err, st, d);
    default: return s.v8 ? launch_amax<DT_F16, true>(s, x, amax_bits, err, st, d)
                         : launch_amax<DT_F16, false>(s, x, amax_bits, err, st, d);
    }
}

template <int DT, bool IF4, bool V8>
int launch_quant(const Shape &s, const void *x, uint8_t *codes, uint8_t *scales,
                 const float *ts, int *err, int check_ts, cudaStream_t st, const DeviceInfo &d)
{
    if (s.ngroups == 0) return IF4_OK;
    auto k = quantize_kernel<DT, IF4, V8>;
    const uint32_t grid = grid_for(k, d, s.ngroups, 256);
    k<<<grid, 256, 0, st>>>(static_cast<const char *>(x), s.ld_bytes, s.gpr, s.ngroups,
                            s.contig ? 1 : 0, codes, scales, ts, err, check_ts);
    return launch_status();
}

template <bool IF4>
int dispatch_quant(int dt, const Shape &s, const void *x, uint8_t *codes, uint8_t *scales,
                   const float *ts, int *err, int check_ts, cudaStream_t st, const DeviceInfo &d)
{
    switch (dt) {
    case IF4_F32:
        return s.v8 ? launch_quant<DT_F32, IF4, true>(s, x, codes, scales, ts, err, check_ts, st, d)
                    : launch_quant<DT_F32, IF4, false>(s, x, codes, scales, ts, err, check_ts, st, d);
    case IF4_BF16:
        return s.v8 ? launch_quant<DT_BF16, IF4, true>(s, x, codes, scales, ts, err, check_ts, st, d)
                    : launch_quant<DT_BF16, IF4, false>(s, x, codes, scales, ts, err, check_ts, st, d);
    default:
        return s.v8 ? launch_quant<DT_F16, IF4, true>(s, x, codes, scales, ts, err, check_ts, st, d)
                    : launch_quant<DT_F16, IF4, false>(s, x, codes, scales, ts, err, check_ts, st, d);
    }
}

template <bool IF4>
int quantize_entry(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                   uint8_t *codes, uint8_t *scales, float *ts, int ts_mode, int *err_flag,
                   void *stream)
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
        // A1 accumulates max |x| as float bits into *ts, A2 turns it into ts
        if (cudaMemsetAsync(ts, 0, sizeof(float), st) != cudaSuccess) return IF4_ERR_CUDA;
        rc = dispatch_amax(x_dtype, s, x, reinterpret_cast<unsigned int *>(ts), err_flag, st, d);
        if (rc != IF4_OK) return rc;
        tensor_scale_kernel<<<1, 1, 0, st>>>(ts, ts);
        rc = launch_status();
        if (rc != IF4_OK) return rc;
    }
    return dispatch_quant<IF4>(x_dtype, s, x, codes, scales, ts, err_flag,
                               ts_mode == IF4_TS_GIVEN ? 1 : 0, st, d);
}

template <int ODT, bool UNIT_TS>
int launch_dequant(const Shape &s, const uint8_t *codes, const uint8_t *scales, const float *ts,
                   void *y, cudaStream_t st, const DeviceInfo &d)
{
    if (s.ngroups == 0) return IF4_OK;
    auto k = dequantize_kernel<ODT, UNIT_TS>;
    const uint32_t grid = grid_for(k, d, s.ngroups, 256);
    k<<<grid, 256, 0, st>>>(codes, scales, ts, s.gpr, s.ngroups, static_cast<char *>(y),
                            s.ld_bytes, s.contig ? 1 : 0);
    return launch_status();
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
    tensor_scale_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(amax, ts);
    return launch_status();
}

int if4_quantize(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                 uint8_t *codes, uint8_t *scales, float *ts, int ts_mode, int *err_flag,
                 void *stream)
{
    return quantize_entry<true>(x, x_dtype, rows, cols, ld_x, codes, scales, ts, ts_mode,
                                err_flag, stream);
}

int nvfp4_quantize(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                   uint8_t *codes, uint8_t *scales, float *ts, int ts_mode, int *err_flag,
                   void *stream)
{
    return quantize_entry<false>(x, x_dtype, rows, cols, ld_x, codes, scales, ts, ts_mode,
                                 err_flag, stream);
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
