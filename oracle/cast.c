/*
 * cast.c -- closed-form MXFP4 -> NVFP4 cast.  TEST INFRASTRUCTURE.
 *
 * [CAST] section 2: an MXFP4 block of 32 E2M1 values carries one power-of-two scale
 * 2^k_j (E8M0).  Pin the global scale with global_amax = 6*448*2^(k_max-8), so the
 * NVFP4 second-level scale s2 = global_amax/(6*448) = 2^m with m = k_max-8.  Give every
 * NVFP4 block _amax = 6*2^k_j, so its block scale 2^(k_j-m) is exact in E4M3 and the
 * NVFP4 dequantized values equal the MXFP4 ones bit for bit, as long as
 * k_max - k_j <= 17.  Blocks outside that window fall back to a scale derived from the
 * data, max|w_block|.  The cast reports lossless layer/block fractions.
 * [DSPARK] stage 3: the E2M1 nibbles are reused unchanged and the scale bytes double
 * (32-element E8M0 -> 16-element E4M3).
 *
 * Readings where the pages are silent:
 *  - k_j is the unbiased exponent code-127; k_max is the maximum over one matrix.
 *  - an E8M0 code 0xFF (NaN) is rejected (flag) and never reaches the cast.
 *  - "w_block" in the fallback is the 16-element NVFP4 block of dequantized values
 *    e2m1*2^k_j (exact in FP32), re-quantized with the standard block-scale and element
 *    rules of act.c against s2 = 2^m.
 *  - a 16-block is lossless when its NVFP4 dequant (FP32, RN32(e2m1*S)) equals the
 *    MXFP4 dequant (FP32, e2m1*2^k_j) bit for bit.
 *  - nibble order: byte i of a row holds element 2i (low) and 2i+1 (high), both formats.
 */
#include "nv4_oracle.h"

#include <limits.h>
#include <math.h>
#include <string.h>

int orc_mx_kmax(const uint8_t* e8m0, int64_t n, uint32_t* flags)
{
    int kmax = INT_MIN;
    for (int64_t i = 0; i < n; ++i) {
        if (e8m0[i] == 0xFFu) { *flags |= ORC_FLAG_E8M0_NAN; continue; }
        int k = (int)e8m0[i] - 127;
        if (k > kmax) kmax = k;
    }
    return kmax;
}

void orc_mx_global(int k_max, float* s2, float* global_amax, uint32_t* flags)
{
    double p = ldexp(1.0, k_max - 8);         /* 2^m */
    *s2 = (float)p;                           /* exact for m in [-149, 127] */
    *global_amax = (float)(6.0 * 448.0 * p);  /* 6*448 = 21*2^7: exact unless it overflows */
    if (!isfinite(*s2) || !isfinite(*global_amax)) *flags |= ORC_FLAG_OVERFLOW;
}

static uint32_t f32_bits(double v)
{
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, 4);
    return u;
}

void orc_mxfp4_to_nvfp4(const uint8_t* mx_q, const uint8_t* e8m0, int64_t rows, int64_t cols,
                        int k_max, int64_t row0, int64_t row1, uint8_t* nv_q, uint8_t* nv_scales,
                        int64_t* counts)
{
    (void)rows;
    const int m = k_max - 8;
    const double s2 = ldexp(1.0, m);
    const int64_t nmx = cols / 32, nnv = cols / 16, nbytes = cols / 2;

    for (int64_t r = row0; r < row1; ++r) {
        for (int64_t j = 0; j < nmx; ++j) {
            const int k = (int)e8m0[r * nmx + j] - 127;
            for (int h = 0; h < 2; ++h) {            /* the two 16-element NVFP4 blocks */
                const int64_t byte0 = r * nbytes + 16 * j + 8 * h;
                unsigned nib[16];
                for (int i = 0; i < 8; ++i) {
                    nib[2 * i] = mx_q[byte0 + i] & 15u;
                    nib[2 * i + 1] = mx_q[byte0 + i] >> 4;
                }
                double w[16];
                for (int i = 0; i < 16; ++i) w[i] = orc_e2m1_value(nib[i]) * ldexp(1.0, k);

                unsigned code, out[16];
                if (k_max - k <= 17) {
                    /* in window: scale 2^(k_j - m) is an exact E4M3 value; nibbles unchanged */
                    code = orc_e4m3_encode(ldexp(1.0, k - m), 1.0);
                    for (int i = 0; i < 16; ++i) out[i] = nib[i];
                    counts[0] += 1;
                } else {
                    /* fallback: data-derived block amax, standard NVFP4 quantization */
                    double a_b = 0.0;
                    for (int i = 0; i < 16; ++i)
                        if (fabs(w[i]) > a_b) a_b = fabs(w[i]);
                    code = orc_e4m3_encode(a_b, 6.0 * s2);
                    float S = (float)(orc_e4m3_value(code) * s2);
                    for (int i = 0; i < 16; ++i) out[i] = orc_e2m1_encode(w[i], (double)S);
                    counts[1] += 1;
                }
                nv_scales[r * nnv + 2 * j + h] = (uint8_t)code;
                for (int i = 0; i < 8; ++i)
                    nv_q[byte0 + i] = (uint8_t)(out[2 * i] | (out[2 * i + 1] << 4));

                /* lossless: NVFP4 dequant == MXFP4 dequant, bit for bit in FP32 */
                float S = (float)(orc_e4m3_value(code) * s2);
                int same = 1;
                for (int i = 0; i < 16; ++i)
                    if (f32_bits(orc_e2m1_value(out[i]) * (double)S) != f32_bits(w[i])) { same = 0; break; }
                counts[2] += same;
            }
        }
    }
}
