/*
 * act.c -- per-tensor amax, dynamic activation quantization and its two-step
 * dequantization.  TEST INFRASTRUCTURE (see nv4_oracle.h).
 *
 * Definitions followed:
 *  amax      [CAL] section 2 step 1 (max calibration: largest absolute value of a
 *            weight or activation tensor).
 *  act quant [FLOW] 3.4-3.5: s2 = amax/6/448 from the calibrated amax; each block of
 *            16 consecutive elements along a row gets an E4M3 scale s_b for block_amax/6
 *            relative to s2; elements become E2M1 codes of x / (s_b*s2); [FLOW] 5.4: two
 *            FP4 codes per byte.  [CAL] format line: 16-element blocks, E4M3 scale, FP32
 *            second-level scale.
 *  RTN weight quant [FLOW] 3.5 (static weight quantization) and [CAL] section 2 step 1
 *            (max calibration gives the initial block scale): the same block arithmetic as
 *            the activation quantizer, applied once to a BF16 or FP32 weight tensor with its
 *            own amax.
 *  dequant   [FLOW] 3.4: DQ1 turns (E4M3 scale, FP32 s2) into the FP32 block scale
 *            S = s_b*s2; DQ2 multiplies each FP4 value by S and emits the high-precision
 *            type (BF16 by default, FP16 optional, [FLOW] 3.6).
 *
 * Readings where the pages are silent:
 *  - s2 is amax/2688 rounded once to FP32; a zero amax gives s2 = 0 and all-zero blocks.
 *  - the block scale is the nearest E4M3 value to the exact block_amax/(6*s2), ties to
 *    the even code, saturating at 448 (a calibrated amax below the live data saturates).
 *  - the E2M1 divisor is the FP32 block scale S = RN32(s_b*s2), the value DQ1 produces.
 *  - each E2M1 code keeps the sign of x, so -0 and small negatives give code 0x8.
 *  - byte i of a row holds element 2i in its low nibble and element 2i+1 in its high one.
 *  - NaN entries set the non-finite flag; outputs of a block holding one are unspecified.
 */
#include "nv4_oracle.h"

#include <math.h>
#include <string.h>

static double elem_value(const void* x, int dtype, int64_t i)
{
    if (dtype == ORC_F32) return (double)((const float*)x)[i];
    return orc_bf16_value(((const uint16_t*)x)[i]);
}

float orc_tensor_amax(const void* x, int dtype, int64_t n, uint32_t* flags)
{
    double amax = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        double v = elem_value(x, dtype, i);
        if (!isfinite(v)) *flags |= ORC_FLAG_NONFINITE;
        if (isnan(v)) continue;
        if (fabs(v) > amax) amax = fabs(v);
    }
    return (float)amax; /* exact: amax is one of the inputs */
}

float orc_act_quant(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, float amax,
                    int64_t row0, int64_t row1, uint8_t* q, uint8_t* scales, uint32_t* flags)
{
    return orc_block_quant(x, ORC_BF16, rows, cols, ld, amax, row0, row1, q, scales, flags);
}

float orc_block_quant(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld, float amax,
                      int64_t row0, int64_t row1, uint8_t* q, uint8_t* scales, uint32_t* flags)
{
    (void)rows;
    float s2 = orc_s2_from_amax(amax);
    if (!isfinite(s2)) *flags |= ORC_FLAG_OVERFLOW;
    const int64_t nblk = cols / 16;
    for (int64_t r = row0; r < row1; ++r) {
        for (int64_t b = 0; b < nblk; ++b) {
            double v[16];
            double a_b = 0.0;
            for (int i = 0; i < 16; ++i) {
                v[i] = elem_value(x, dtype, r * ld + 16 * b + i);
                if (!isfinite(v[i])) *flags |= ORC_FLAG_NONFINITE;
                if (fabs(v[i]) > a_b) a_b = fabs(v[i]);
            }
            /* block scale: nearest E4M3 to a_b / (6*s2) */
            unsigned code = orc_e4m3_encode(a_b, 6.0 * (double)s2);
            /* DQ1: the FP32 block scale (the product is exact in FP64, then rounded once) */
            float S = (float)(orc_e4m3_value(code) * (double)s2);
            scales[r * nblk + b] = (uint8_t)code;
            for (int i = 0; i < 16; i += 2) {
                unsigned lo = orc_e2m1_encode(v[i], (double)S);
                unsigned hi = orc_e2m1_encode(v[i + 1], (double)S);
                q[r * (cols / 2) + 8 * b + i / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
    return s2;
}

void orc_dequant(const uint8_t* q, const uint8_t* scales, float s2, int64_t rows, int64_t cols,
                 int out_dtype, int64_t row0, int64_t row1, void* out)
{
    (void)rows;
    const int64_t nblk = cols / 16;
    for (int64_t r = row0; r < row1; ++r) {
        for (int64_t c = 0; c < cols; ++c) {
            unsigned code = scales[r * nblk + c / 16];
            /* DQ1: S = RN32(s_b * s2) */
            float S = (float)(orc_e4m3_value(code) * (double)s2);
            unsigned byte = q[r * (cols / 2) + c / 2];
            unsigned nib = (c & 1) ? (byte >> 4) : (byte & 15u);
            /* DQ2: RN32(v * S); v has 2 significant bits, so the FP64 product is exact */
            float y = (float)(orc_e2m1_value(nib) * (double)S);
            int64_t o = r * cols + c;
            if (out_dtype == 0) ((uint16_t*)out)[o] = orc_f32_to_bf16(y);
            else if (out_dtype == 1) ((uint16_t*)out)[o] = orc_f32_to_f16(y);
            else ((float*)out)[o] = y;
        }
    }
}
