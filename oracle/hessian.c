/*
 * hessian.c -- local Hessian per 16-input-channel block.  TEST INFRASTRUCTURE.
 *
 * [CAL] section 2 step 2: with full-precision weights, run the calibration forward
 * again and, at every layer input, accumulate H = sum X^T X per block of 16 channels.
 * Block b covers channels 16b..16b+15, so H_b[i][j] = sum_t x[t][16b+i] * x[t][16b+j].
 *
 * Reading where the page is silent: a plain sum over tokens (not a mean; the sweep's argmin does
 * not change under a positive scale), no damping term, and X is whatever the caller
 * passes.  Accumulation (+=) lets calibration run over many token batches.
 *
 * Arithmetic: BF16 values are exact in FP64 and so are their products (16 significant
 * bits); the sums carry FP64 rounding only (relative 2^-53 per add).
 */
#include "nv4_oracle.h"

void orc_hessian_accum(const uint16_t* x, int64_t tokens, int64_t cols, int64_t ld,
                       int64_t blk0, int64_t blk1, double* H)
{
    (void)cols;
    for (int64_t b = blk0; b < blk1; ++b) {
        double acc[256] = {0.0};
        for (int64_t t = 0; t < tokens; ++t) {
            double v[16];
            for (int i = 0; i < 16; ++i) v[i] = orc_bf16_value(x[t * ld + 16 * b + i]);
            for (int i = 0; i < 16; ++i)
                for (int j = 0; j < 16; ++j)
                    acc[16 * i + j] += v[i] * v[j];
        }
        for (int k = 0; k < 256; ++k) H[b * 256 + k] += acc[k];
    }
}
