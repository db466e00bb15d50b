/*
 * variants.c -- format variants of the block quantizer: MXFP4 (32-element blocks,
 * E8M0 power-of-two scales) and FP8 E4M3 with one static per-tensor scale.
 * TEST INFRASTRUCTURE (see nv4_oracle.h).
 *
 * Definitions followed:
 *  MXFP4  [FP4] section 1.2 (32 elements per group, E8M0 scale: a pure power of two,
 *         E2M1 elements) and section 3.2 (power-aligned scales, shifts instead of
 *         multiplies).  Reading where the page is silent: the shared exponent of a block
 *         is floor(log2(amax)) - 2 (2 = the largest E2M1 exponent, so amax lands in
 *         [4, 8) before rounding), clamped to [-127, 127]; E8M0 code = exponent + 127;
 *         elements are the nearest E2M1 values to x / 2^e (ties to even, saturating at
 *         6, sign kept); an all-zero block gets code 0; a block holding NaN or Inf gets
 *         the NaN code 0xFF and sets the non-finite flag.  Byte i of a row holds element
 *         2i in its low nibble (as for NVFP4).
 *  FP8    [CAL] layer table (FP8 E4M3 W8A8 with static per-tensor scales) and the note
 *         under it (FP8 activations use the calibrated static scale).  Reading: the
 *         scale is s = RN32(amax / 448) and each element is the nearest E4M3 value to
 *         x / s (ties to even, saturating at 448, sign kept); s = 0 gives signed zeros.
 */
#include "nv4_oracle.h"

#include <math.h>

static double elem(const void* x, int dtype, int64_t i)
{
    if (dtype == ORC_F32) return (double)((const float*)x)[i];
    return orc_bf16_value(((const uint16_t*)x)[i]);
}

void orc_mxfp4_quant(const void* x, int dtype, int64_t cols, int64_t ld, int64_t row0, int64_t row1,
                     uint8_t* q, uint8_t* e8m0, uint32_t* flags)
{
    const int64_t nblk = cols / 32;
    for (int64_t r = row0; r < row1; ++r) {
        for (int64_t b = 0; b < nblk; ++b) {
            double v[32], amax = 0.0;
            int bad = 0;
            for (int i = 0; i < 32; ++i) {
                v[i] = elem(x, dtype, r * ld + 32 * b + i);
                if (!isfinite(v[i])) bad = 1;
                else if (fabs(v[i]) > amax) amax = fabs(v[i]);
            }
            uint8_t* qb = q + r * (cols / 2) + 16 * b;
            if (bad) {
                *flags |= ORC_FLAG_NONFINITE;
                e8m0[r * nblk + b] = 0xFF;
                for (int i = 0; i < 16; ++i) qb[i] = 0;
                continue;
            }
            int e = -127;
            if (amax > 0.0) {
                int ex;
                frexp(amax, &ex);              /* amax = f * 2^ex, f in [0.5, 1): floor(log2 amax) = ex - 1 */
                e = ex - 1 - 2;
                if (e < -127) e = -127;
                if (e > 127) e = 127;
            }
            e8m0[r * nblk + b] = (uint8_t)(e + 127);
            const double S = ldexp(1.0, e);
            for (int i = 0; i < 32; i += 2) {
                unsigned lo = orc_e2m1_encode(v[i], S), hi = orc_e2m1_encode(v[i + 1], S);
                qb[i / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
}

void orc_mxfp4_dequant(const uint8_t* q, const uint8_t* e8m0, int64_t cols, int64_t row0, int64_t row1,
                       int out_dtype, void* out)
{
    for (int64_t r = row0; r < row1; ++r) {
        for (int64_t c = 0; c < cols; ++c) {
            unsigned byte = q[r * (cols / 2) + c / 2];
            unsigned nib = (c & 1) ? (byte >> 4) : (byte & 15u);
            /* e2m1 * 2^k: exact in FP64, rounded once to FP32 (exact unless below FP32 range) */
            float y = (float)(orc_e2m1_value(nib) * orc_e8m0_value(e8m0[r * (cols / 32) + c / 32]));
            int64_t o = r * cols + c;
            if (out_dtype == 0) ((uint16_t*)out)[o] = orc_f32_to_bf16(y);
            else if (out_dtype == 1) ((uint16_t*)out)[o] = orc_f32_to_f16(y);
            else ((float*)out)[o] = y;
        }
    }
}

float orc_fp8_quant(const void* x, int dtype, int64_t cols, int64_t ld, float amax, int64_t row0, int64_t row1,
                    uint8_t* q, uint32_t* flags)
{
    const float s = (float)((double)amax / 448.0);   /* exact quotient rounded once to FP32 */
    if (!isfinite(s)) *flags |= ORC_FLAG_OVERFLOW;
    for (int64_t r = row0; r < row1; ++r) {
        for (int64_t c = 0; c < cols; ++c) {
            double v = elem(x, dtype, r * ld + c);
            if (!isfinite(v)) *flags |= ORC_FLAG_NONFINITE;
            unsigned sign = signbit(v) ? 0x80u : 0u;
            unsigned code = 0u;
            if (s > 0.0f && isfinite(v)) code = orc_e4m3_encode(fabs(v), (double)s);
            q[r * cols + c] = (uint8_t)(sign | code);
        }
    }
    return s;
}
