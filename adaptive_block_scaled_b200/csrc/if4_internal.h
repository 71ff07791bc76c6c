// Library-internal entry points shared between the translation units of
// libif4.so.  Not part of the C ABI: the version script keeps these local.
#pragma once

#include <cstdint>

// The IF4 x IF4 linear's operand decode for both operands in one launch:
// A's groups, then B's, as one index space, each decoded as if4_decode_f16
// decodes it (fp16 of fl(q * E4M3(sb)), the tensor scale factored out) into
// a dense [rows, cols] fp16 array.  codes dense and 16-byte aligned, y
// 32-byte aligned.  Returns an IF4_* status.
int internal_decode_f16_pair(const uint8_t *a_codes, const uint8_t *a_scales, int64_t a_rows,
                             void *a_y, const uint8_t *b_codes, const uint8_t *b_scales,
                             int64_t b_rows, void *b_y, int64_t cols, void *stream);
