/* moe_pack.h -- host-side quantisation and packing of expert weights into the
 * layout the kernels read (moe_layer.codes / scales, described in moe.h).
 *
 * This is data preparation, not part of the hot path: a checkpoint converter
 * or a test harness calls it once per matrix.  The pages ship their experts as
 * group-quantised low-bit files ("Strata open-source runtime: a 12GB card runs
 * the 125B Qwen3 model", section "the cost": Q2_0 and IQ3 expert files) but
 * print no quantiser and no bit layout; the quantiser below is the plain
 * symmetric max-magnitude rule, and the layout is the one in moe.h.
 */
#ifndef MOE_PACK_H
#define MOE_PACK_H

#include "moe.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Quantise and pack one weight matrix.
 *  w:      host fp32 [rows][cols], row-major; groups of 32 run along cols (the
 *          contraction dimension K of the matrix in moe.h's layout).
 *  codes:  host uint8 [rows/16][cols/32 * 16 * (8 | 12)] (2-bit | 3-bit),
 *          16-row tiles laid out as moe.h describes.
 *  scales: host fp16 bits [rows/16][cols/32 * 16], tile-interleaved likewise.
 *  Quantiser, per row and group of 32 values w_0..w_31, in fp32:
 *    m = the w_j of largest magnitude (the first one on ties),
 *    s = fp16(m / -2^(b-1)), rounded to nearest even,
 *    q_j = clamp(round_half_even(w_j / s) + 2^(b-1), 0, 2^b - 1),
 *    and a group whose s is 0 stores q_j = 2^(b-1).
 *  The kernels and the oracle read w'_j = s * (q_j - 2^(b-1)).
 *  An expert's codes are pack(Wg), pack(Wu), pack(Wd) back to back (Wg, Wu
 *  [ffn][d]; Wd [d][ffn]) and its scales follow the same order: call three
 *  times with codes and scales advanced by each matrix's output size.
 *  Returns MOE_ERR_INVALID_ARG for a NULL pointer and
 *  MOE_ERR_UNSUPPORTED_SHAPE unless rows > 0, rows % 16 == 0, cols > 0,
 *  cols % 32 == 0 and bits is 2 or 3; nothing is written then.  Pure host
 *  code: no device, stream or allocation; the caller owns all three arrays. */
moe_status moe_pack_host(const float* w, int32_t rows, int32_t cols, int32_t bits,
                         uint8_t* codes, uint16_t* scales);

#ifdef __cplusplus
}
#endif

#endif /* MOE_PACK_H */
