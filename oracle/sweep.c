/*
 * sweep.c -- Hessian-weighted E4M3 block-scale sweep with the NVFP4 pack of the
 * winner.  TEST INFRASTRUCTURE.
 *
 * [CAL] section 2 step 3: for every 16-element weight block, try the FP8 E4M3 block
 * scale over all its values and keep the one that minimises (W - Wq)^T H (W - Wq),
 * with H the block's local Hessian (step 2).  Step 1 supplies the weight amax, which
 * fixes the FP32 second-level scale s2 = amax/6/448 ([FLOW] 3.4).
 *
 * For block w (16 values) and candidate code c:
 *     S_c  = RN32(e4m3(c) * s2)                       (DQ1 of [FLOW] 3.4)
 *     q_i  = E2M1 code of w_i / S_c                   (nearest, ties to even)
 *     e_i  = w_i - e2m1(q_i) * S_c
 *     cost = sum_i sum_j e_i H[i][j] e_j
 * The winner is the smallest cost, ties to the lowest code.
 *
 * Readings where the pages are silent:
 *  - candidates are the 127 finite non-negative codes 0x00..0x7E; the page's count of
 *    128 values is the 7-bit code space, whose last point 0x7F is NaN;
 *  - code 0 (S = 0, an all-zero block) is a candidate; nothing is clipped;
 *  - e uses the exact product e2m1*S_c (FP64); it is exact whenever w_i and the product
 *    lie within 2^26 of each other in magnitude, and otherwise off by at most 2^-53
 *    relative, far below any tolerance used on costs;
 *  - cost2 is the best cost among codes whose dequantized block differs from the
 *    winner's (as real numbers, so -0 == +0), +inf when every code gives the same block.
 */
#include "nv4_oracle.h"

#include <math.h>

static double elem_value(const void* w, int dtype, int64_t i)
{
    if (dtype == ORC_F32) return (double)((const float*)w)[i];
    return orc_bf16_value(((const uint16_t*)w)[i]);
}

void orc_scale_sweep(const void* w, int dtype, int64_t rows, int64_t cols, int64_t ld,
                     const double* H, float amax_w, int64_t row0, int64_t row1,
                     uint8_t* codes, uint8_t* q, double* cost1, double* cost2, uint32_t* flags)
{
    (void)rows;
    const float s2 = orc_s2_from_amax(amax_w);
    if (!isfinite(s2)) *flags |= ORC_FLAG_OVERFLOW;
    const int64_t nblk = cols / 16;

    for (int64_t r = row0; r < row1; ++r) {
        for (int64_t b = 0; b < nblk; ++b) {
            const double* Hb = H + b * 256;
            double wv[16];
            for (int i = 0; i < 16; ++i) {
                wv[i] = elem_value(w, dtype, r * ld + 16 * b + i);
                if (!isfinite(wv[i])) *flags |= ORC_FLAG_NONFINITE;
            }

            double cost[127];
            double deq[127][16];
            unsigned qc[127][16];
            for (unsigned c = 0; c < 127; ++c) {
                float S = (float)(orc_e4m3_value(c) * (double)s2);
                double e[16];
                for (int i = 0; i < 16; ++i) {
                    qc[c][i] = orc_e2m1_encode(wv[i], (double)S);
                    deq[c][i] = orc_e2m1_value(qc[c][i]) * (double)S;
                    e[i] = wv[i] - deq[c][i];
                }
                double s = 0.0;
                for (int i = 0; i < 16; ++i)
                    for (int j = 0; j < 16; ++j)
                        s += e[i] * Hb[16 * i + j] * e[j];
                cost[c] = s;
            }

            unsigned best = 0;
            for (unsigned c = 1; c < 127; ++c)
                if (cost[c] < cost[best]) best = c;

            double second = INFINITY;
            for (unsigned c = 0; c < 127; ++c) {
                int same = 1;
                for (int i = 0; i < 16; ++i)
                    if (deq[c][i] != deq[best][i]) { same = 0; break; }
                if (!same && cost[c] < second) second = cost[c];
            }

            codes[r * nblk + b] = (uint8_t)best;
            if (q)
                for (int i = 0; i < 16; i += 2)
                    q[r * (cols / 2) + 8 * b + i / 2] = (uint8_t)(qc[best][i] | (qc[best][i + 1] << 4));
            if (cost1) cost1[r * nblk + b] = cost[best];
            if (cost2) cost2[r * nblk + b] = second;
        }
    }
}
