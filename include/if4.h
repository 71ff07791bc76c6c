/*
 * if4.h -- C ABI of libif4.so: the IF4 (Int/Float 4) adaptive block-scaled
 * 4-bit format on NVIDIA B200 (sm_100a).
 *
 * The format ("Adaptive Block-Scaled Data Types", Cook et al., arXiv
 * 2603.28765; abstract, and gist.science section 2 "Metodologia"): a tensor
 * is cut into groups of 16 consecutive values along its contiguous (last)
 * dimension.  Each group shares one 8-bit E4M3 block scale, as in NVFP4, and
 * stores its 16 values as 4-bit codes, either as E2M1 FP4 or as INT4 scaled
 * by 7/6 (integers -7..7 that decode to k*6/7, so both grids end at 6; "Metodo
 * 6/7").  The quantizer forms both candidates and keeps the one with the
 * lower squared error ("Mecanismo de Selecao"; shd-paper.top, technical
 * framework steps 1-5).  The choice lives in the scale byte's sign bit, which
 * NVFP4 leaves unused: 0 = FP4, 1 = INT4 ("Codificacao Eficiente"; companion
 * page "The Free Bit: Scale Factor Sign").  Storage is NVFP4's, 4.5 bits per
 * value.  A per-tensor FP32 decode scale ts = amax/(6*448) sits above the
 * block scales, as in NVFP4.
 *
 * Arithmetic contract (every step IEEE binary32, round-to-nearest-even):
 *   ts    = amax_T / 2688  (1 if amax_T == 0; never below 2^-117)
 *   sb    = E4M3_RNE_satfinite((amax_g / 6) / ts), subnormals kept
 *   eff   = E4M3(sb) * ts,  inv = 1 / eff,  v_i = x_i * inv
 *   FP4   : nibble = sign(v) | RNE_E2M1(|v|) saturating at 6 (a negative v
 *           that rounds to zero keeps its sign: nibble 0x8)
 *   INT4  : k = clamp(RNE(v * fl(7/6)), -7, 7), nibble = k & 0xF,
 *           value fl(6k/7)
 *   choice: INT4 iff sum (v - q_int)^2 < sum (v - q_fp)^2, the sums taken in
 *           binary64 in element order; equal sums keep FP4.  (The kernels
 *           decide in binary32 and redo the binary64 sums for any group
 *           whose binary32 margin is within its rounding bound, so the
 *           result equals the binary64 rule everywhere.)
 *   sb == 0 (the block scale underflows): all nibbles 0, scale byte 0x00.
 *   dequantize: y = fl(q * fl(E4M3(sb & 0x7F) * ts)), then rounded to the
 *           output type.
 *
 * Layouts (all row-major, groups along the last dimension):
 *   x      [rows, cols], row stride ld_x elements, cols % 16 == 0
 *   codes  uint8 [rows, cols/2]  dense; byte j of a group holds element 2j in
 *          its low nibble and element 2j+1 in its high nibble
 *   scales uint8 [rows, cols/16] dense; bit 7 = type, bits 0-6 = E4M3 code
 *   ts     one float in device memory
 * NVFP4 output is valid IF4 with every bit 7 clear, so if4_dequantize also
 * decodes NVFP4.
 *
 * Ownership and ordering: the caller allocates every buffer (device memory
 * for all tensor and scalar arguments) and keeps it alive until the stream
 * work completes.  Entry points validate arguments on the host, enqueue
 * kernels on `stream` (a cudaStream_t; NULL = the legacy default stream) and
 * return without synchronising.  They allocate no memory, keep no state
 * between calls and may be called from several host threads.
 *
 * Errors: a nonzero if4_status is returned before anything is enqueued when
 * an argument is invalid; IF4_ERR_CUDA reports a launch failure.  Problems
 * only the device can see are OR-ed into *err_flag (a device int the caller
 * zeroes; may be NULL where stated) as IF4_DEV_* bits and never trap.
 */
#ifndef IF4_H
#define IF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    IF4_OK = 0,
    IF4_ERR_NULL = 1,        /* a required pointer is NULL                      */
    IF4_ERR_SHAPE = 2,       /* rows/cols < 0, cols % 16 != 0, ld too small, or
                                a size beyond the stated maximum               */
    IF4_ERR_DTYPE = 3,       /* unknown dtype code                              */
    IF4_ERR_ALIGN = 4,       /* pointer or leading dimension misaligned         */
    IF4_ERR_MODE = 5,        /* unknown ts_mode                                 */
    IF4_ERR_WORKSPACE = 6,   /* workspace NULL or smaller than required         */
    IF4_ERR_CUDA = 7,        /* a CUDA call or kernel launch failed             */
    IF4_ERR_DEVICE = 8       /* the current device is not sm_100 (B200)        */
} if4_status;

/* element types of dense tensors */
typedef enum { IF4_F32 = 0, IF4_BF16 = 1, IF4_F16 = 2 } if4_dtype;

/* tensor-scale modes of the quantizers */
enum {
    IF4_TS_COMPUTE = 0,      /* compute amax over x, write ts = amax/2688 to *ts */
    IF4_TS_GIVEN = 1         /* read the caller's ts from *ts                   */
};

/* device-side error bits OR-ed into *err_flag */
enum {
    IF4_DEV_NONFINITE = 1,   /* an input element is Inf or NaN: outputs unspecified */
    IF4_DEV_BAD_SCALE = 2,   /* a given ts is not finite or outside [2^-117, 2^117] */
    IF4_DEV_TIMEOUT = 4      /* a bounded wait (the linear's pipeline, the single-launch
                                quantizer's grid barrier) ran out: outputs unspecified */
};

/* Largest supported tensor: rows * cols / 16 < 2^31 groups. */

/*
 * Tensor amax: amax = max |x| over x[rows, cols] (device float).  x_dtype is IF4_F32,
 * IF4_BF16 or IF4_F16; x 16-byte aligned, ld_x*elem_size % 16 == 0.
 * err_flag may be NULL; otherwise IF4_DEV_NONFINITE is set for Inf/NaN.
 * (The tensor scale of NVFP4-style formats; arXiv abstract.)
 */
int if4_tensor_amax(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                    float *amax, int *err_flag, void *stream);

/* Tensor scale: ts = amax / 2688 (1 if amax == 0, floored at 2^-117), device to device. */
int if4_tensor_scale(const float *amax, float *ts, void *stream);

/*
 * IF4 quantize.  Per group of 16: the E4M3 block scale, the FP4 and
 * the 7/6-scaled INT4 candidates, the lower-error choice in bit 7 of the
 * scale byte (gist.science section 2; shd-paper.top framework steps 1-5).
 * ts_mode IF4_TS_COMPUTE runs the amax and scale steps first and writes *ts; IF4_TS_GIVEN reads
 * it.  codes must be 16-byte aligned.  err_flag may be NULL.
 */
int if4_quantize(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                 uint8_t *codes, uint8_t *scales, float *ts, int ts_mode,
                 int *err_flag, void *stream);

/*
 * NVFP4 quantize, the comparator: the FP4 candidate of if4_quantize for
 * every group, bit 7 of every scale byte 0.  Same arguments and rules.
 */
int nvfp4_quantize(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                   uint8_t *codes, uint8_t *scales, float *ts, int ts_mode,
                   int *err_flag, void *stream);

/*
 * Random-sign Hadamard transform fused into the quantizer, for weight
 * gradients (gist.science section 1, second item: a Hadamard transform makes
 * the data near-uniform, where INT4 does better; companion "Where the Gain
 * Actually Comes From").  Every group of 16 is replaced by y = H16 diag(s)
 * x_g / 4 before quantization: H16 the Sylvester Hadamard matrix, s_j = -1
 * where bit j of `signs` is set (bits 16-31 ignored).  The transform is
 * evaluated in binary32 as a fast Walsh-Hadamard transform with stages h = 1,
 * 2, 4, 8 (each (y[i], y[i+h]) -> (y[i] + y[i+h], y[i] - y[i+h]) for i with
 * bit h clear), then times 1/4.  The transformed tensor never reaches memory;
 * the codes are those of if4_quantize applied to it, and if4_dequantize gives
 * back the transformed values.
 */
int if4_tensor_amax_rht(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                        uint32_t signs, float *amax, int *err_flag, void *stream);
int if4_quantize_rht(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                     uint32_t signs, uint8_t *codes, uint8_t *scales, float *ts, int ts_mode,
                     int *err_flag, void *stream);

/*
 * Single-launch quantizer: tensor amax, tensor scale and IF4 quantize (as
 * if4_quantize with IF4_TS_COMPUTE), plus, when nv_codes / nv_scales are
 * given, the NVFP4 comparator of nvfp4_quantize under the same tensor scale,
 * all in one cooperative kernel launch that reads x for the amax and again
 * for the encode.  Results are byte-identical to those calls.
 *
 * sync_words: 64 uint32 (256 bytes) of device memory, 256-byte aligned,
 * owned by the caller, all zero before the first call.  Word 0 counts
 * arrivals at the grid barrier and word 1 accumulates the amax; every call
 * that completes leaves both at zero.  Word 32 counts barrier generations
 * and word 33 keeps the last ts; they may hold any value.  The rest is
 * unused.  So one allocation serves any number
 * of calls that run one after another; calls that may run at the same time
 * (other streams) need their own.  A call that set IF4_DEV_TIMEOUT (a
 * block waited more than 1 s at the grid barrier) leaves codes, scales, ts
 * and y unspecified: blocks that gave up wrote nothing, but a block that
 * arrived last, or was still waiting, may have encoded its groups.  Zero the
 * words and call again.
 *
 * nv_codes / nv_scales: both NULL (IF4 only) or both given.  err_flag may be
 * NULL; IF4_DEV_NONFINITE and IF4_DEV_TIMEOUT are reported there.  Other
 * rules as if4_quantize.  The pages have no counterpart: this is a fusion of
 * the steps above.
 */
int if4_quantize_fused(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                       uint8_t *codes, uint8_t *scales, uint8_t *nv_codes, uint8_t *nv_scales,
                       float *ts, uint32_t *sync_words, int *err_flag, void *stream);

/*
 * The single launch with the round trip: everything if4_quantize_fused does,
 * and also y, the IF4 codes it writes decoded exactly as if4_dequantize
 * decodes them to bf16: y = bf16_RNE(fl(q * fl(E4M3(sb) * ts))), byte-
 * identical to if4_dequantize(codes, scales, ts, ..., IF4_BF16) afterwards
 * ("Adaptive Block-Scaled Data Types", gist.science section 2, "Metodo 6/7",
 * and the companion's "MAC Unit: Decoding Two Formats from One Sign Bit").
 * The quantize-then-dequantize round trip of one tensor in one launch; the
 * codes are decoded while they are still in registers.
 *
 * y: bf16 [rows, cols], dense (row stride cols), base 32-byte aligned, owned
 * by the caller, not overlapping x or the other outputs.  Other arguments and
 * rules as if4_quantize_fused.  IF4_ERR_NULL for a null y of a non-empty
 * tensor, IF4_ERR_ALIGN for a y that is not 32-byte aligned.  After
 * IF4_DEV_TIMEOUT codes, scales, ts and y are unspecified, as for
 * if4_quantize_fused.
 */
int if4_quantize_fused_dequant(const void *x, int x_dtype, int64_t rows, int64_t cols,
                               int64_t ld_x, uint8_t *codes, uint8_t *scales, uint8_t *nv_codes,
                               uint8_t *nv_scales, float *ts, uint32_t *sync_words, void *y,
                               int *err_flag, void *stream);

/*
 * The single launches on a share of the device: if4_quantize_fused,
 * if4_quantize_fused_dequant and if4_quantize_fused_rht with one more
 * argument, share.  The launch sizes its grid to floor(R / share) blocks per
 * SM (at least one), R being the blocks of its kernel one SM holds, so that
 * `share` such calls on different streams, each with its own sync_words, are
 * resident together: the amax pass of one runs beside the encode pass of
 * another.  Independent tensors (consecutive steps, the layers of a model)
 * quantized this way on two streams take less time in total than one after
 * another on one stream, while each call alone takes longer.  share = 1 is
 * the plain call.  The outputs do not depend on share: they are
 * byte-identical to the plain call's.  IF4_ERR_SHAPE for share outside
 * [1, 64]; other arguments and rules as the plain call.  Each call waits
 * only for its own blocks, never for another launch.
 */
int if4_quantize_fused_shared(const void *x, int x_dtype, int64_t rows, int64_t cols,
                              int64_t ld_x, uint8_t *codes, uint8_t *scales, uint8_t *nv_codes,
                              uint8_t *nv_scales, float *ts, uint32_t *sync_words, int share,
                              int *err_flag, void *stream);
int if4_quantize_fused_dequant_shared(const void *x, int x_dtype, int64_t rows, int64_t cols,
                                      int64_t ld_x, uint8_t *codes, uint8_t *scales,
                                      uint8_t *nv_codes, uint8_t *nv_scales, float *ts,
                                      uint32_t *sync_words, void *y, int share, int *err_flag,
                                      void *stream);

/*
 * The same single launch on the random-sign Hadamard transform of x (see
 * if4_quantize_rht): the amax, the tensor scale, the IF4 codes and the
 * NVFP4 comparator are those of the transformed tensor, equal to
 * if4_quantize_rht(IF4_TS_COMPUTE) and nvfp4_quantize of the transformed
 * tensor under that ts.  signs: bits 0-15 as for if4_quantize_rht.
 */
int if4_quantize_fused_rht(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                           uint32_t signs, uint8_t *codes, uint8_t *scales, uint8_t *nv_codes,
                           uint8_t *nv_scales, float *ts, uint32_t *sync_words, int *err_flag,
                           void *stream);
/* if4_quantize_fused_rht on a share of the device, as the shared launches
 * above. */
int if4_quantize_fused_rht_shared(const void *x, int x_dtype, int64_t rows, int64_t cols,
                                  int64_t ld_x, uint32_t signs, uint8_t *codes, uint8_t *scales,
                                  uint8_t *nv_codes, uint8_t *nv_scales, float *ts,
                                  uint32_t *sync_words, int share, int *err_flag, void *stream);

/*
 * Comparator, all-INT4 ("NVINT4"): the 7/6-scaled INT4 candidate of
 * if4_quantize for every group, bit 7 set wherever the block scale is
 * nonzero (gist.science section 3, item 2, and section 4: IF4 is compared with
 * NVFP4 and NVINT4).  Same arguments and rules as if4_quantize; decoded by
 * if4_dequantize.
 */
int nvint4_quantize(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                    uint8_t *codes, uint8_t *scales, float *ts, int ts_mode,
                    int *err_flag, void *stream);

/*
 * Comparator, Four Over Six ("4/6"): NVFP4 whose block scale maps the group
 * maximum either to 6 (sb from amax/6, as NVFP4) or to 4 (sb from amax/4),
 * whichever reconstructs the group with the lower squared error
 * sum (x - fl(q * fl(E4M3 * ts)))^2 (binary64 rule, equal errors keep 6);
 * gist.science section 1, third item.  Output is plain NVFP4 (bit 7 clear),
 * decoded by if4_dequantize.  Same arguments and rules as if4_quantize.
 */
int nvfp4_4over6_quantize(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                          uint8_t *codes, uint8_t *scales, float *ts, int ts_mode,
                          int *err_flag, void *stream);

/*
 * Dequantize IF4 (or NVFP4) to y[rows, cols] of y_dtype (IF4_F32,
 * IF4_BF16 or IF4_F16), row stride ld_y elements: fl(q * fl(E4M3 * ts)),
 * then RNE to the output type.  codes 16-byte aligned; y 16-byte aligned and
 * ld_y*elem_size % 16 == 0.  (gist.science section 2, "Metodo 6/7";
 * companion, "MAC Unit: Decoding Two Formats from One Sign Bit".)
 */
int if4_dequantize(const uint8_t *codes, const uint8_t *scales, const float *ts,
                   int64_t rows, int64_t cols, void *y, int y_dtype, int64_t ld_y,
                   void *stream);

/*
 * First stage of the linear: y = fp16_RNE(fl(q * E4M3(sb))) [rows, cols],
 * dense, i.e. the dequantized value with the tensor scale left out (exact for
 * FP4 groups, rounded to 11 bits for INT4 groups).  y 16-byte aligned.
 */
int if4_decode_f16(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t cols,
                   void *y, void *stream);

/*
 * Second stage of the linear: C[M, N] = bf16_RNE(fl(a_ts * b_ts) * sum_k
 * A[m, k] * B[n, k]) with A fp16 [M, K], B fp16 [N, K] dense and K-contiguous,
 * products accumulated in fp32 by tcgen05 MMA.  a_ts, b_ts are device floats.
 * M, N >= 1, K % 16 == 0, K >= 16; A, B, C 16-byte aligned, N % 8 == 0.
 * err_flag must not be NULL (IF4_DEV_TIMEOUT).
 */
int if4_gemm_f16(const void *a, const void *b, const float *a_ts, const float *b_ts,
                 int64_t M, int64_t N, int64_t K, void *c, int *err_flag, void *stream);

/* Workspace the linear needs: two fp16 operand buffers, (M + N) * K * 2 bytes
 * plus alignment padding; 0 for invalid sizes. */
size_t if4_linear_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * IF4 x IF4 linear.  C[M, N] (bf16, dense) = sum_k A_hat[m, k] *
 * B_hat[n, k] where A (activations, [M, K]) and B (weights, [N, K], i.e. C =
 * A B^T) are both IF4 along K.  Runs if4_decode_f16 on both operands into
 * the caller's workspace, then if4_gemm_f16 with the two tensor scales in
 * its epilogue.  The pages' MAC routes each operand pair by the sign bit
 * into one of two decoders (companion, "MAC Unit: Decoding Two Formats from
 * One Sign Bit"); here both decoders run ahead of a dense tensor-core GEMM.
 * err_flag must not be NULL.
 */
int if4_linear(const uint8_t *a_codes, const uint8_t *a_scales, const float *a_ts,
               const uint8_t *b_codes, const uint8_t *b_scales, const float *b_ts,
               int64_t M, int64_t N, int64_t K, void *workspace, size_t ws_bytes,
               void *c, int *err_flag, void *stream);

/*
 * IF4 x IF4 linear with the decoders inside the GEMM: the same C as
 * if4_linear, bit for bit, without a workspace.  The pages' MAC decodes each
 * operand by its group's sign bit right before the multiply (companion, "MAC
 * Unit: Decoding Two Formats from One Sign Bit"); here warps of the GEMM
 * decode each 64-wide K step of both operands from the IF4 codes into the
 * tensor cores' shared-memory operand stages, so the fp16 operands never
 * exist in global memory.  Each operand row is decoded once per output tile
 * that uses it, so the decode work is repeated N/256 times for A and M/256
 * times for B (the separate decode of if4_linear runs once per element).
 *
 * K % 64 == 0; a_codes and b_codes 32-byte aligned, a_scales and b_scales
 * 4-byte aligned (row strides K/2 and K/16 bytes); other rules, errors and
 * err_flag as if4_linear (IF4_ERR_SHAPE for K % 64 != 0).
 */
int if4_linear_fused(const uint8_t *a_codes, const uint8_t *a_scales, const float *a_ts,
                     const uint8_t *b_codes, const uint8_t *b_scales, const float *b_ts,
                     int64_t M, int64_t N, int64_t K, void *c, int *err_flag, void *stream);

/*
 * IF4 x IF4 linear with an IF4 output: the product of if4_linear, rounded to
 * bf16 exactly as there, then quantized to IF4 along N (groups of 16
 * columns of each row of C) under the given tensor scale *c_ts, inside the
 * GEMM's epilogue.  The codes and scales equal those of
 * if4_quantize(C, IF4_BF16, M, N, N, ..., c_ts, IF4_TS_GIVEN) on the bf16
 * C of if4_linear.  The output never exists as a bf16 tensor unless c is
 * given (then it is written too, as by if4_linear).
 *
 * The tensor scale of C has to be known before the GEMM runs (for example
 * the previous step's, as with delayed scaling); an invalid one sets
 * IF4_DEV_BAD_SCALE, and Inf/NaN in C set IF4_DEV_NONFINITE.  The pages'
 * W4A4 training feeds quantized activations into the next linear (companion
 * "MAC Unit: Decoding Two Formats from One Sign Bit"); fusing that quantize
 * into the producing GEMM is this library's choice.
 *
 * c_codes: uint8 [M, N/2], 16-byte aligned; c_scales: uint8 [M, N/16];
 * c_ts: device float; c: bf16 [M, N] or NULL.  N % 16 == 0.  Other rules,
 * the workspace and the errors as if4_linear.
 */
int if4_linear_quantized(const uint8_t *a_codes, const uint8_t *a_scales, const float *a_ts,
                         const uint8_t *b_codes, const uint8_t *b_scales, const float *b_ts,
                         int64_t M, int64_t N, int64_t K, void *workspace, size_t ws_bytes,
                         void *c, uint8_t *c_codes, uint8_t *c_scales, const float *c_ts,
                         int *err_flag, void *stream);

/*
 * IF6 and IF3: the same adaptive FP/INT choice at 6 and 3 bits per value.
 * The pages name both formats and say the adaptive choice carries over to
 * other bit widths ("Adaptive Block-Scaled Data Types", abstract; companion
 * "It Generalizes: IF3 and IF6"; gist.science section 2, "Extensoes"), but
 * print neither grid.  The grids below are this library's reading, not fixed
 * by the pages:
 *   IF6: FP6 = E2M3 (sign, 2 exponent bits with bias 1, 3 mantissa bits;
 *        largest 7.5) against INT6 k in [-31, 31] decoded as fl(15k/62),
 *        k = clamp(RNE(v * fl(62/15))); both grids end at 7.5.
 *   IF3: FP3 = E2M0 (sign, magnitudes 0, 1, 2, 4) against INT3 k in [-3, 3]
 *        decoded as fl(4k/3), k = clamp(RNE(v * 3/4)); both end at 4.
 * Everything else is IF4's contract with fpmax (7.5 or 4) in place of 6:
 * ts = amax_T/(fpmax*448) with IF4_TS_COMPUTE, sb = E4M3((amax_g/fpmax)/ts),
 * v = x * fl(1/fl(E4M3(sb)*ts)), FP rounding to nearest with ties to the even
 * code, saturating, an FP zero keeping the sign of v, INT codes in two's
 * complement, the binary64 rule with ties to FP, bit 7 of the scale byte for
 * INT, sb == 0 giving zero codes and byte 0x00.
 *
 * mode: IF4_W_ADAPTIVE (the lower-error candidate), IF4_W_FP_ONLY (the FP
 * candidate everywhere, bit 7 clear: the fixed FP6/FP3 format at the same
 * block scale) or IF4_W_INT_ONLY (the INT candidate everywhere, bit 7 set
 * unless sb == 0).
 *
 * codes: uint8 [rows, cols*w/8] dense, w = 6 or 3: element i of a group is
 * the w-bit field at bits [w*i, w*i + w) of the group's little-endian code
 * bytes (12 bytes per group for IF6, 6 for IF3); 4-byte aligned base.
 * scales: uint8 [rows, cols/16].  Storage: 6.5 and 3.5 bits per value.
 * Other arguments, layouts and errors as if4_quantize (IF4_ERR_MODE also for
 * an unknown mode).  These formats are off the bench's step; the kernels take
 * the binary64 rule directly.
 */
enum { IF4_W_ADAPTIVE = 0, IF4_W_FP_ONLY = 1, IF4_W_INT_ONLY = 2 };

int if6_quantize(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x, int mode,
                 uint8_t *codes, uint8_t *scales, float *ts, int ts_mode, int *err_flag,
                 void *stream);
int if3_quantize(const void *x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x, int mode,
                 uint8_t *codes, uint8_t *scales, float *ts, int ts_mode, int *err_flag,
                 void *stream);

/*
 * Dequantize IF6 / IF3 (either mode's output): y = fl(q * fl(E4M3(sb & 0x7F)
 * * ts)), q decoded as FP or INT by bit 7, rounded to y_dtype.  Layouts and
 * errors as if4_dequantize; codes 4-byte aligned.
 */
int if6_dequantize(const uint8_t *codes, const uint8_t *scales, const float *ts, int64_t rows,
                   int64_t cols, void *y, int y_dtype, int64_t ld_y, void *stream);
int if3_dequantize(const uint8_t *codes, const uint8_t *scales, const float *ts, int64_t rows,
                   int64_t cols, void *y, int y_dtype, int64_t ld_y, void *stream);

/* Number of uint32 sync words if4_quantize_fused and its variants need. */
#define IF4_FUSED_SYNC_WORDS 64u

/* Size of the scratch array behind if4_linear_noalloc (32 MiB per device). */
#define IF4_LINEAR_NOALLOC_MAX_BYTES (32u * 1024u * 1024u)

/*
 * if4_linear without a workspace argument, for callers that cannot provide
 * device memory at the call: for example a plugin inside a framework that
 * owns all device memory through its own pool, or a latency-critical path
 * that must not risk the device synchronisation cudaMalloc can cause.  The
 * pages have no counterpart; this is a deployment variant of if4_linear.
 * Same arguments and result as if4_linear.  The decoded operands live in a
 * fixed scratch array in the library's device code (IF4_LINEAR_NOALLOC_MAX_BYTES
 * per device, held from when the library's device code is loaded on that
 * device until the process exits); it allocates nothing.  Problems whose
 * if4_linear_workspace_bytes exceeds that size return IF4_ERR_WORKSPACE
 * before anything is enqueued.  All calls on a device share the one array:
 * calls whose work overlaps on the GPU race and corrupt each other, so order
 * them (e.g. one stream).  The first call on each device looks up the
 * array's address with that device current; make that first call before any
 * stream capture.  That address belongs to the device's primary context:
 * after a cudaDeviceReset of the device, do not call if4_linear_noalloc on it
 * again in the same process.  Errors come in the order of if4_linear's: a
 * problem too large for the array returns IF4_ERR_WORKSPACE only when every
 * other argument is valid.
 */
int if4_linear_noalloc(const uint8_t *a_codes, const uint8_t *a_scales, const float *a_ts,
                       const uint8_t *b_codes, const uint8_t *b_scales, const float *b_ts,
                       int64_t M, int64_t N, int64_t K, void *c, int *err_flag, void *stream);

/* Static description of a status code. */
const char *if4_status_str(int status);

/* Library ABI version (major * 100 + minor). */
int if4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* IF4_H */
