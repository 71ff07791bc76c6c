/*
 * IF4 / NVFP4 CPU ORACLE -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, scalar C statement of what the IF4 quantizer and dequantizer
 * compute, written from the pages on "Adaptive Block-Scaled Data Types"
 * (Cook et al., arXiv 2603.28765).  Only the test suite, the smoke check and
 * the CPU-baseline leg of the benchmark may load it.  It shares no code, table
 * or header with the CUDA library, and the CUDA library never calls it.
 *
 * Arithmetic: IEEE binary32 for every value the format defines (compile with
 * -O2 -ffp-contract=off, no fast-math, no flush-to-zero), binary64 for the
 * per-group squared-error sums that decide FP4 vs INT4.
 *
 * Sources, by page and section:
 *   [ABS]   the arXiv abstract (reprinted on shd-paper.top and fugumt.com):
 *           groups of 16 values, an E4M3 scale per group "as is done with
 *           NVFP4", the selected type kept in the scale's sign bit.
 *   [FRAME] shd-paper.top, "Adaptive Block-Scaled Data Types", method details,
 *           technical framework, steps 1-5: split into 16-blocks, evaluate the
 *           FP4 and INT4 error, keep the lower, scale by E4M3, record the type
 *           in the sign bit.
 *   [SEL]   gist.science (pt), same title, section 2 "Metodologia",
 *           "Mecanismo de Seleção": quantize to both, compute both MSEs, keep
 *           the smaller.
 *   [BIT]   gist.science section 2, "Codificação Eficiente": sign bit 0 = FP4,
 *           1 = scaled INT4; and the episode companion "Adaptive Block-Scaled
 *           Data Types for FP4 Training", "The Free Bit: Scale Factor Sign".
 *   [67]    gist.science section 2, "Método 6/7": INT4 values are multiplied
 *           by 7/6 before rounding and by 6/7 when used, so the largest value
 *           is 6, as for FP4; companion, "One Group, Two Candidate Encodings".
 *   [E2M1]  gist.science section 1 "O Problema": NVFP4 elements are E2M1.
 *   [E4M3]  fugumt.com related entry "FP8 Formats for Deep Learning": E4M3
 *           has no infinities and a single NaN mantissa pattern.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   tensor scale ts = amax/(6*448), 1 for an all-zero tensor, and never
 *   below 2^-117 so that every nonzero decoded block scale is a normal float;
 *   block scale = (amax_g/6)/ts rounded to E4M3 by round-to-nearest-even with
 *   saturation to 448 and subnormals kept; v = x * fl(1/eff); E2M1 is
 *   round-to-nearest-even of v; the INT4 integer is round-to-nearest-even of
 *   the exact product v * fl(7/6) (a single rounding); FP4 zero keeps the
 *   sign of v;
 *   INT4 codes are two's complement in [-7, 7]; the choice is INT4 only when
 *   its error is strictly lower; a group whose block scale rounds to zero is
 *   stored as all-zero FP4; the even element of a pair goes in the low nibble.
 *
 * The same adaptive choice at 6 and 3 bits (IF6, IF3) is at the end of this
 * file.  The pages name both but give neither grid; the grids used there
 * (FP6 = E2M3 against a 31-level INT6, FP3 = E2M0 against a 3-level INT3)
 * are readings, not fixed by the pages.
 *
 * Parity pins: every function here is checked by the non-GPU tests against
 * brute force over the grids, a library float8 cast, exact rationals,
 * closed-form values and hand-worked groups; none is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* E2M1 magnitudes indexed by the 3-bit code [E2M1]. */
static const float kE2M1Mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

/* ---------------------------------------------------------------- E4M3 ---- */

/* Value of an E4M3 byte with bit 7 ignored: 4 exponent bits (bias 7), 3
 * mantissa bits, exponent field 0 = subnormal (m * 2^-9), 0x7F = NaN. */
float orc_e4m3_value(uint8_t b)
{
    int code = b & 0x7F;
    int e = code >> 3, m = code & 7;
    if (code == 0x7F) return NAN;
    if (e == 0) return (float)ldexp((double)m, -9);
    return (float)ldexp((double)(8 + m), e - 10);
}

/* Nearest E4M3 code to a non-negative float, ties to the even code,
 * saturating at 448 (0x7E); never returns the NaN code for finite input. */
uint8_t orc_e4m3_encode(float f)
{
    if (f != f) return 0x7F;
    if (f <= 0.0f) return 0x00;
    if (f >= 448.0f) return 0x7E;
    int e2;
    (void)frexp((double)f, &e2);         /* f in [2^(e2-1), 2^e2) */
    int E = e2 - 1;
    if (E < -6) E = -6;                  /* subnormal range: step 2^-9 */
    /* f in units of 2^(E-3): exact power-of-two scaling, then RNE. */
    double q = rint(ldexp((double)f, 3 - E));
    /* normal: q in [8,16]; q == 16 carries into the next binade, which the
     * additive code form below produces by itself.  subnormal: q in [0,8]. */
    return (uint8_t)(((E + 7) << 3) + ((int)q - 8));
}

/* ---------------------------------------------------------------- E2M1 ---- */

/* 4-bit FP4 nibble of v: bit 3 = sign of v (so a negative v that rounds to
 * zero gives 0x8), bits 0-2 = magnitude code, round to nearest, ties to the
 * even code, saturating at 6. */
uint8_t orc_e2m1_nibble(float v)
{
    uint8_t sign = signbit(v) ? 8 : 0;
    double a = fabs((double)v);
    int c;
    if (!(a <= 6.0)) {
        c = 7;                           /* above 6 (or NaN): saturate */
    } else if (a < 2.0) {
        c = (int)rint(a * 2.0);          /* grid step 0.5, codes 0..4 */
    } else if (a < 4.0) {
        c = (int)rint(a) + 2;            /* grid step 1, codes 4..6 */
    } else {
        c = (int)rint(a * 0.5) + 4;      /* grid step 2, codes 6..7 */
        if (c > 7) c = 7;
    }
    return (uint8_t)(sign | c);
}

float orc_e2m1_value(uint8_t nib)
{
    float m = kE2M1Mag[nib & 7];
    return (nib & 8) ? -m : m;
}

/* ------------------------------------------------------ scaled INT4 ------- */

/* k = round-to-nearest-even(v * c) with c = fl(7/6), the product taken
 * exactly (one rounding, to the integer) [67]; k is clamped to [-7, 7] and
 * stored in 4-bit two's complement (0x8 is never produced).  Both factors
 * are binary32, so their product is exact in binary64. */
uint8_t orc_int4_nibble(float v)
{
    const float c76 = 7.0f / 6.0f;
    double k = rint((double)v * (double)c76);
    if (!(k >= -7.0)) k = -7.0;          /* also maps NaN to -7 */
    if (k > 7.0) k = 7.0;
    return (uint8_t)(((int)k) & 0xF);
}

/* Decoded INT4 value fl(6k/7), k the sign-extended nibble [67]. */
float orc_int4_value(uint8_t nib)
{
    int k = (nib & 8) ? (int)(nib & 0xF) - 16 : (int)(nib & 0xF);
    return (float)(6 * k) / 7.0f;
}

/* --------------------------------------- tensor amax and tensor scale ---- */

float orc_tensor_amax(const float *x, int64_t rows, int64_t cols, int64_t ld)
{
    float amax = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            float a = fabsf(x[r * ld + c]);
            if (a > amax || a != a) amax = a;
        }
    return amax;
}

/* ts = amax/(6*448) as an FP32 decode scale, as for NVFP4 [ABS]. */
float orc_tensor_scale(float amax)
{
    const float floor_ts = 0x1p-117f;
    if (amax == 0.0f) return 1.0f;
    float ts = amax / 2688.0f;
    return ts < floor_ts ? floor_ts : ts;
}

/* ------------------------------------------------------------ quantize ---- */

/* IF4: lower-error candidate per group.  NVFP4: FP4 always.  NVINT4: the
 * 7/6-scaled INT4 candidate always, bit 7 set (the all-INT4 format the pages
 * compare IF4 with: gist.science section 3, item 2; section 4, PTQ).
 * 4/6 ("Four Over Six"): NVFP4 whose block scale maps the group maximum to 6
 * or to 4, whichever reconstructs the group with the lower squared error in
 * the x domain (gist.science section 1, third item: adapting the block
 * maximum to 4 or 6); equal errors keep 6.  4/6 output is plain NVFP4. */
enum { ORC_MODE_IF4 = 0, ORC_MODE_NVFP4 = 1, ORC_MODE_NVINT4 = 2, ORC_MODE_4OVER6 = 3 };

/* Quantize one group of 16 floats.  Writes 8 code bytes and returns the
 * scale byte.  e_fp / e_int receive the binary64 squared errors of the two
 * candidates in the scaled domain; *near receives 1 when they differ by at
 * most 1e-6 relative (or both are zero). */
static uint8_t quantize_group(const float *x, float ts, int mode, uint8_t *codes,
                              double *e_fp_out, double *e_int_out, uint8_t *near_out)
{
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    float sb_f = (amax / 6.0f) / ts;
    uint8_t sb = orc_e4m3_encode(sb_f);
    if (sb == 0) {
        memset(codes, 0, 8);
        *e_fp_out = 0.0;
        *e_int_out = 0.0;
        *near_out = 1;
        return 0x00;
    }
    float eff = orc_e4m3_value(sb) * ts;
    float inv = 1.0f / eff;

    uint8_t nf[16], ni[16];
    double e_fp = 0.0, e_int = 0.0;
    for (int i = 0; i < 16; ++i) {
        float v = x[i] * inv;
        nf[i] = orc_e2m1_nibble(v);
        ni[i] = orc_int4_nibble(v);
        double df = (double)v - (double)orc_e2m1_value(nf[i]);
        double di = (double)v - (double)orc_int4_value(ni[i]);
        e_fp = e_fp + df * df;
        e_int = e_int + di * di;
    }
    int use_int4 = (mode == ORC_MODE_NVINT4) || ((mode == ORC_MODE_IF4) && (e_int < e_fp));
    const uint8_t *n = use_int4 ? ni : nf;
    for (int j = 0; j < 8; ++j)
        codes[j] = (uint8_t)(n[2 * j] | (n[2 * j + 1] << 4));
    double hi = e_fp > e_int ? e_fp : e_int;
    *e_fp_out = e_fp;
    *e_int_out = e_int;
    *near_out = (uint8_t)(fabs(e_fp - e_int) <= 1e-6 * hi);
    return (uint8_t)(sb | (use_int4 ? 0x80 : 0x00));
}

/* FP4 codes of a group under block scale byte sb; returns the binary64 sum
 * of (x - xhat)^2 with xhat = fl(q * fl(E4(sb) * ts)), the dequantized value. */
static double fp4_group_at_scale(const float *x, float ts, uint8_t sb, uint8_t *nib)
{
    float eff = orc_e4m3_value(sb) * ts;
    float inv = sb ? 1.0f / eff : 0.0f;
    double e = 0.0;
    for (int i = 0; i < 16; ++i) {
        float v = x[i] * inv;
        nib[i] = sb ? orc_e2m1_nibble(v) : 0;
        float xhat = orc_e2m1_value(nib[i]) * eff;
        double d = (double)x[i] - (double)xhat;
        e = e + d * d;
    }
    return e;
}

/* 4/6 for one group: candidates with block scales from amax/6 and amax/4. */
static uint8_t quantize_group_4over6(const float *x, float ts, uint8_t *codes, double *e6_out,
                                     double *e4_out, uint8_t *near_out)
{
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    uint8_t sb6 = orc_e4m3_encode((amax / 6.0f) / ts);
    uint8_t sb4 = orc_e4m3_encode((amax / 4.0f) / ts);
    uint8_t n6[16], n4[16];
    double e6 = fp4_group_at_scale(x, ts, sb6, n6);
    double e4 = fp4_group_at_scale(x, ts, sb4, n4);
    int use4 = e4 < e6;
    const uint8_t *n = use4 ? n4 : n6;
    for (int j = 0; j < 8; ++j)
        codes[j] = (uint8_t)(n[2 * j] | (n[2 * j + 1] << 4));
    double hi = e6 > e4 ? e6 : e4;
    *e6_out = e6;
    *e4_out = e4;
    *near_out = (uint8_t)(fabs(e6 - e4) <= 1e-6 * hi);
    return use4 ? sb4 : sb6;
}

/* x: float [rows, ld] row-major, cols % 16 == 0.  codes: [rows, cols/2],
 * scales: [rows, cols/16].  e_fp, e_int, near: [rows, cols/16] or NULL. */
void orc_quantize(const float *x, int64_t rows, int64_t cols, int64_t ld, float ts,
                  int mode, uint8_t *codes, uint8_t *scales, double *e_fp,
                  double *e_int, uint8_t *near, int nthreads)
{
    int64_t gpr = cols / 16;
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(static) num_threads(nthreads)
#endif
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < gpr; ++g) {
            double ef, ei;
            uint8_t nt;
            int64_t gi = r * gpr + g;
            if (mode == ORC_MODE_4OVER6)
                scales[gi] = quantize_group_4over6(x + r * ld + g * 16, ts,
                                                   codes + r * (cols / 2) + g * 8, &ef, &ei, &nt);
            else
                scales[gi] = quantize_group(x + r * ld + g * 16, ts, mode,
                                            codes + r * (cols / 2) + g * 8, &ef, &ei, &nt);
            if (e_fp) e_fp[gi] = ef;
            if (e_int) e_int[gi] = ei;
            if (near) near[gi] = nt;
        }
    }
    (void)nthreads;
}

/* --------------------------------- random-sign Hadamard transform ------ */

/* y = H16 diag(s) x / 4 for one group of 16, H16 the Sylvester Hadamard
 * matrix (entry (i, j) = (-1)^popcount(i & j)) and s_j = -1 where bit j of
 * `signs` is set: the orthonormal random-sign transform applied to weight
 * gradients before quantization (gist.science section 1, second item;
 * companion "Where the Gain Actually Comes From").  Evaluated as the fast
 * Walsh-Hadamard transform in binary32: stages h = 1, 2, 4, 8, each replacing
 * (y[i], y[i+h]) by (y[i] + y[i+h], y[i] - y[i+h]) for every i with bit h
 * clear, then multiplied by 1/4 (exact). */
void orc_rht16(const float *x, uint32_t signs, float *y)
{
    for (int j = 0; j < 16; ++j) y[j] = ((signs >> j) & 1u) ? -x[j] : x[j];
    for (int h = 1; h < 16; h <<= 1)
        for (int i = 0; i < 16; ++i)
            if ((i & h) == 0) {
                float a = y[i], b = y[i + h];
                y[i] = a + b;
                y[i + h] = a - b;
            }
    for (int j = 0; j < 16; ++j) y[j] = y[j] * 0.25f;
}

/* Apply orc_rht16 to every group of x [rows, ld] into y [rows, cols]. */
void orc_rht(const float *x, int64_t rows, int64_t cols, int64_t ld, uint32_t signs, float *y,
             int nthreads)
{
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(static) num_threads(nthreads)
#endif
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t g = 0; g < cols / 16; ++g)
            orc_rht16(x + r * ld + g * 16, signs, y + r * cols + g * 16);
    (void)nthreads;
}

/* ---------------------------------------------------------- dequantize ---- */

/* y[r, c] = fl(q * fl(E4(sb) * ts)), q decoded as FP4 or INT4 by bit 7. */
void orc_dequantize(const uint8_t *codes, const uint8_t *scales, float ts, int64_t rows,
                    int64_t cols, float *y, int nthreads)
{
    int64_t gpr = cols / 16;
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(static) num_threads(nthreads)
#endif
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < gpr; ++g) {
            uint8_t sb = scales[r * gpr + g];
            float eff = orc_e4m3_value(sb) * ts;
            for (int i = 0; i < 16; ++i) {
                uint8_t byte = codes[r * (cols / 2) + g * 8 + i / 2];
                uint8_t nib = (i & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
                float q = (sb & 0x80) ? orc_int4_value(nib) : orc_e2m1_value(nib);
                y[r * cols + g * 16 + i] = q * eff;
            }
        }
    }
    (void)nthreads;
}

/* ------------------------------------------- other widths: IF6 and IF3 ---
 *
 * The pages apply the same adaptive choice at 3 and 6 bits (abstract: "the
 * same insight ... for other bit-widths, including IF3 and IF6"; companion
 * "It Generalizes: IF3 and IF6"; gist.science section 2 "Extensoes") but give
 * neither grid.  Readings (each also listed in the design notes):
 *   IF6: FP candidate E2M3 (sign, two exponent bits with bias 1, three
 *        mantissa bits; magnitudes m/8 for exponent field 0, else
 *        (1 + m/8) 2^(e-1); largest 7.5), INT candidate k in [-31, 31]
 *        decoded as fl(15k/62) and chosen as the round-to-nearest-even of the
 *        exact product v * fl(62/15), so both grids reach 7.5, as FP4 and the
 *        7/6-scaled INT4 both reach 6.
 *   IF3: FP candidate E2M0 (sign, two exponent bits, no mantissa: magnitudes
 *        0, 1, 2, 4), INT candidate k in [-3, 3] decoded as fl(4k/3) and
 *        chosen as the round-to-nearest-even of v * 3/4; both reach 4.
 *   Both: the block scale is E4M3 of (amax/fpmax)/ts, the tensor scale
 *        amax_T/(fpmax * 448), ties between equal candidate errors keep FP,
 *        bit 7 of the scale byte set for INT, FP ties to the even code,
 *        saturating; an FP zero keeps the sign of v; INT codes two's
 *        complement.  Element i's code occupies bits [w*i, w*i + w) of the
 *        group's little-endian code bytes (12 bytes per group for IF6, 6 for
 *        IF3), so IF6 stores 6.5 and IF3 3.5 bits per value. */

enum { ORC_W_IF = 0, ORC_W_FP = 1, ORC_W_INT = 2 };

/* 6-bit E2M3 code of v: bit 5 = sign of v, bits 0-4 = magnitude code
 * (exponent << 3 | mantissa), round to nearest with ties to the even code,
 * saturating at 7.5.  The scalings by 8, 4 and 2 are exact. */
uint8_t orc_e2m3_code(float v)
{
    uint8_t sign = signbit(v) ? 0x20 : 0;
    double a = fabs((double)v);
    int c;
    if (!(a <= 7.5)) c = 31;                       /* above 7.5 (or NaN) */
    else if (a < 1.0) c = (int)rint(a * 8.0);      /* step 1/8: codes 0..8 */
    else if (a < 2.0) c = (int)rint(a * 8.0);      /* step 1/8: codes 8..16 */
    else if (a < 4.0) c = (int)rint(a * 4.0) + 8;  /* step 1/4: codes 16..24 */
    else c = (int)rint(a * 2.0) + 16;              /* step 1/2: codes 24..31 */
    return (uint8_t)(sign | c);
}

float orc_e2m3_value(uint8_t code)
{
    int e = (code >> 3) & 3, m = code & 7;
    double mag = e == 0 ? m / 8.0 : ldexp(1.0 + m / 8.0, e - 1);
    return (float)((code & 0x20) ? -mag : mag);
}

/* k = RNE(v * fl(62/15)), the product exact in binary64, clamped to
 * [-31, 31]; 6-bit two's complement. */
uint8_t orc_int6_code(float v)
{
    const float c = 62.0f / 15.0f;
    double k = rint((double)v * (double)c);
    if (!(k >= -31.0)) k = -31.0;
    if (k > 31.0) k = 31.0;
    return (uint8_t)(((int)k) & 0x3F);
}

float orc_int6_value(uint8_t code)
{
    int k = (code & 0x20) ? (int)(code & 0x3F) - 64 : (int)(code & 0x3F);
    return (float)(15 * k) / 62.0f;
}

/* 3-bit E2M0 code: bit 2 = sign of v, bits 0-1 = magnitude code of 0, 1, 2,
 * 4; ties to the even code (0.5 -> 0, 1.5 -> 2, 3 -> 2), saturating at 4. */
uint8_t orc_e2m0_code(float v)
{
    uint8_t sign = signbit(v) ? 4 : 0;
    double a = fabs((double)v);
    int c;
    if (!(a <= 3.0)) c = 3;
    else if (a >= 1.5) c = 2;
    else if (a > 0.5) c = 1;
    else c = 0;
    return (uint8_t)(sign | c);
}

float orc_e2m0_value(uint8_t code)
{
    static const float mag[4] = {0.0f, 1.0f, 2.0f, 4.0f};
    float m = mag[code & 3];
    return (code & 4) ? -m : m;
}

/* k = RNE(v * 3/4) clamped to [-3, 3]; 3-bit two's complement. */
uint8_t orc_int3_code(float v)
{
    double k = rint((double)v * 0.75);
    if (!(k >= -3.0)) k = -3.0;
    if (k > 3.0) k = 3.0;
    return (uint8_t)(((int)k) & 0x7);
}

float orc_int3_value(uint8_t code)
{
    int k = (code & 4) ? (int)(code & 7) - 8 : (int)(code & 7);
    return (float)(4 * k) / 3.0f;
}

static float width_fpmax(int bits) { return bits == 6 ? 7.5f : 4.0f; }

/* Tensor scale of the width-`bits` format: amax/(fpmax * 448), 1 for a zero
 * tensor, floored at 2^-117 as for IF4. */
float orc_tensor_scale_w(float amax, int bits)
{
    const float floor_ts = 0x1p-117f;
    if (amax == 0.0f) return 1.0f;
    float ts = amax / (width_fpmax(bits) * 448.0f);
    return ts < floor_ts ? floor_ts : ts;
}

static void put_code(uint8_t *bytes, int bits, int i, uint8_t code)
{
    for (int b = 0; b < bits; ++b)
        if ((code >> b) & 1) {
            int pos = bits * i + b;
            bytes[pos >> 3] |= (uint8_t)(1u << (pos & 7));
        }
}

static uint8_t get_code(const uint8_t *bytes, int bits, int i)
{
    uint8_t c = 0;
    for (int b = 0; b < bits; ++b) {
        int pos = bits * i + b;
        c |= (uint8_t)(((bytes[pos >> 3] >> (pos & 7)) & 1u) << b);
    }
    return c;
}

/* One group of 16 at width `bits` (6 or 3): code bytes (2 * bits of them),
 * returns the scale byte; the binary64 squared errors of both candidates in
 * the scaled domain and the near-tie flag as for IF4. */
static uint8_t quantize_group_w(const float *x, float ts, int bits, int mode, uint8_t *codes,
                                double *e_fp_out, double *e_int_out, uint8_t *near_out)
{
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    memset(codes, 0, (size_t)(2 * bits));
    uint8_t sb = orc_e4m3_encode((amax / width_fpmax(bits)) / ts);
    if (sb == 0) {
        *e_fp_out = 0.0;
        *e_int_out = 0.0;
        *near_out = 1;
        return 0x00;
    }
    float eff = orc_e4m3_value(sb) * ts;
    float inv = 1.0f / eff;
    uint8_t cf[16], ci[16];
    double e_fp = 0.0, e_int = 0.0;
    for (int i = 0; i < 16; ++i) {
        float v = x[i] * inv;
        float qf, qi;
        if (bits == 6) {
            cf[i] = orc_e2m3_code(v);
            ci[i] = orc_int6_code(v);
            qf = orc_e2m3_value(cf[i]);
            qi = orc_int6_value(ci[i]);
        } else {
            cf[i] = orc_e2m0_code(v);
            ci[i] = orc_int3_code(v);
            qf = orc_e2m0_value(cf[i]);
            qi = orc_int3_value(ci[i]);
        }
        double df = (double)v - (double)qf;
        double di = (double)v - (double)qi;
        e_fp = e_fp + df * df;
        e_int = e_int + di * di;
    }
    int use_int = (mode == ORC_W_INT) || ((mode == ORC_W_IF) && (e_int < e_fp));
    const uint8_t *c = use_int ? ci : cf;
    for (int i = 0; i < 16; ++i) put_code(codes, bits, i, c[i]);
    double hi = e_fp > e_int ? e_fp : e_int;
    *e_fp_out = e_fp;
    *e_int_out = e_int;
    *near_out = (uint8_t)(fabs(e_fp - e_int) <= 1e-6 * hi);
    return (uint8_t)(sb | (use_int ? 0x80 : 0x00));
}

/* x: float [rows, ld], cols % 16 == 0.  codes: [rows, cols * bits / 8],
 * scales: [rows, cols/16].  mode: ORC_W_IF, ORC_W_FP or ORC_W_INT. */
void orc_quantize_w(const float *x, int64_t rows, int64_t cols, int64_t ld, float ts, int bits,
                    int mode, uint8_t *codes, uint8_t *scales, double *e_fp, double *e_int,
                    uint8_t *near, int nthreads)
{
    int64_t gpr = cols / 16, cb = 2 * bits;
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(static) num_threads(nthreads)
#endif
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < gpr; ++g) {
            double ef, ei;
            uint8_t nt;
            int64_t gi = r * gpr + g;
            scales[gi] = quantize_group_w(x + r * ld + g * 16, ts, bits, mode,
                                          codes + r * gpr * cb + g * cb, &ef, &ei, &nt);
            if (e_fp) e_fp[gi] = ef;
            if (e_int) e_int[gi] = ei;
            if (near) near[gi] = nt;
        }
    }
    (void)nthreads;
}

/* y[r, c] = fl(q * fl(E4(sb) * ts)), q decoded as FP or INT by bit 7. */
void orc_dequantize_w(const uint8_t *codes, const uint8_t *scales, float ts, int64_t rows,
                      int64_t cols, int bits, float *y, int nthreads)
{
    int64_t gpr = cols / 16, cb = 2 * bits;
#ifdef _OPENMP
    if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(static) num_threads(nthreads)
#endif
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < gpr; ++g) {
            uint8_t sb = scales[r * gpr + g];
            float eff = orc_e4m3_value(sb) * ts;
            const uint8_t *gc = codes + r * gpr * cb + g * cb;
            for (int i = 0; i < 16; ++i) {
                uint8_t c = get_code(gc, bits, i);
                float q = bits == 6 ? ((sb & 0x80) ? orc_int6_value(c) : orc_e2m3_value(c))
                                    : ((sb & 0x80) ? orc_int3_value(c) : orc_e2m0_value(c));
                y[r * cols + g * 16 + i] = q * eff;
            }
        }
    }
    (void)nthreads;
}

int orc_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------- element functions over arrays ----- */
/* Used by the tests to sweep large value sets through the scalar functions. */

void orc_e4m3_encode_array(const float *f, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(f[i]);
}

void orc_e2m1_nibble_array(const float *v, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_nibble(v[i]);
}

void orc_int4_nibble_array(const float *v, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_int4_nibble(v[i]);
}

void orc_e2m3_code_array(const float *v, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m3_code(v[i]);
}

void orc_int6_code_array(const float *v, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_int6_code(v[i]);
}

void orc_e2m0_code_array(const float *v, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m0_code(v[i]);
}

void orc_int3_code_array(const float *v, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_int3_code(v[i]);
}
