/*
 * nv4_oracle.h -- plain, slow CPU oracle for the NVFP4 block-numerics hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant with the CUDA library, and it never includes it.
 *
 * Arithmetic is FP64 with exact comparisons.  Every rounding decision the
 * method takes (E4M3 block scale, E2M1 element) is decided by comparing the
 * operand with "midpoint x divisor", a product that is exact in FP64 for the
 * operand widths used here (see formats.c).  Nothing here is blocked, fused or
 * reordered beyond the definition each function cites.
 *
 * Sources (web pages on NVFP4, cited by title and section):
 *  [CAL]  "Coder390 NVFP4 calibration method" (evaluation/NVFP4_CALIBRATION_METHOD.md), section 2
 *         (max calibration, local Hessian H = sum X^T X per 16 channels, fp8_scale_sweep) and the
 *         format line under it (E2M1, 16-element blocks, E4M3 scale, FP32 second-level scale).
 *  [FLOW] "NVFP4 quantization and export flow" (Gemma-2B decoder to TensorRT), sections 3.4-3.5
 *         (per-tensor scale amax/6/448, dynamic activation quantize, two DequantizeLinear) and
 *         5.4 (two FP4 values packed in one byte).
 *  [CAST] "From MXFP4 to NVFP4: Model Optimizer mixed-precision format conversion", section 2
 *         (global_amax = 6*448*2^(k_max-8), per-block _amax = 6*2^k_j, window k_max-k_j <= 17,
 *         fallback to max|w_block|).
 *  [FP4]  "FP4 quantization overview", sections 1.1 (E2M1 values) and 1.2 (MXFP4 vs NVFP4 table).
 *  [DSPARK] "From calibration to export: the three-stage NVFP4 recipe of DeepSeek-V4-Pro-0813-nvfp4-DSpark",
 *         stage 3 (lossless MXFP4 -> NVFP4: nibbles reused, scale bytes double).
 *
 * Parity status: every function below is pinned by a test under tests/ that does
 * not call the oracle's own arithmetic (exact rationals, torch float8 casts,
 * numpy matmul, brute force).  No function is "parity unpinned".
 */
#ifndef NV4_ORACLE_H
#define NV4_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- formats (formats.c) ---------------------------------------------- */
double orc_e2m1_value(unsigned code);          /* 4-bit code SEEM -> signed value          */
double orc_e4m3_value(unsigned code);          /* 8-bit E4M3 (fn) code -> value, NaN 0x7F/FF */
double orc_e8m0_value(unsigned code);          /* 2^(code-127), NaN for 0xFF               */
unsigned orc_e4m3_encode(double num, double den); /* nearest non-negative E4M3 to num/den   */
unsigned orc_e2m1_encode(double x, double S);  /* sign | nearest grid magnitude to |x|/S   */
float orc_s2_from_amax(float amax);            /* RN32(amax / (6*448))                     */
double orc_bf16_value(uint16_t bits);          /* exact widening                           */
uint16_t orc_f32_to_bf16(float f);             /* IEEE round-to-nearest-even               */
uint16_t orc_f32_to_f16(float f);              /* IEEE round-to-nearest-even, overflow inf */

/* ---- data-dependent flags (same meaning as the product's flag word) ---- */
#define ORC_FLAG_NONFINITE 1u
#define ORC_FLAG_E8M0_NAN  2u
#define ORC_FLAG_OVERFLOW  4u

/* element types of an input tensor */
#define ORC_BF16 0
#define ORC_F32  2

/* ---- per-tensor amax (act.c) -------------------------------------------
 * Returns max |v| over the finite and infinite entries (NaN is skipped) and
 * ORs ORC_FLAG_NONFINITE into *flags when a NaN or Inf is present. */
float orc_tensor_amax(const void* x, int dtype, int64_t n, uint32_t* flags);

/* ---- dynamic activation quantization (act.c) ----------------------------
 * x: bf16 bits, row-major [rows, cols] with leading dimension ld (elements).
 * Rows [row0, row1) are processed.  q: [rows, cols/2] bytes, scales: [rows, cols/16]
 * E4M3 codes, both contiguous.  Returns s2. */
float orc_act_quant(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, float amax,
                    int64_t row0, int64_t row1, uint8_t* q, uint8_t* scales, uint32_t* flags);

/* ---- round-to-nearest block quantization of a BF16 or FP32 tensor (act.c) --
 * The activation quantizer's arithmetic for dtype ORC_BF16 or ORC_F32 input (RTN
 * weight quantization with max-calibrated block scales). */
float orc_block_quant(const void* x, int dtype, int64_t rows, int64_t cols, int64_t ld, float amax,
                      int64_t row0, int64_t row1, uint8_t* q, uint8_t* scales, uint32_t* flags);

/* ---- format variants (variants.c) ----------------------------------------
 * MXFP4: 32-element blocks, E8M0 shared power-of-two scale (q [rows, cols/2], e8m0
 * [rows, cols/32]).  FP8: E4M3 codes with one static per-tensor scale s = amax/448
 * (returned).  x: dtype ORC_BF16 or ORC_F32, leading dimension ld; rows [row0, row1). */
void orc_mxfp4_quant(const void* x, int dtype, int64_t cols, int64_t ld, int64_t row0, int64_t row1,
                     uint8_t* q, uint8_t* e8m0, uint32_t* flags);
void orc_mxfp4_dequant(const uint8_t* q, const uint8_t* e8m0, int64_t cols, int64_t row0, int64_t row1,
                       int out_dtype, void* out);
float orc_fp8_quant(const void* x, int dtype, int64_t cols, int64_t ld, float amax, int64_t row0, int64_t row1,
                    uint8_t* q, uint32_t* flags);

/* ---- two-step dequantization (act.c) ------------------------------------
 * out_dtype: 0 = bf16 bits (uint16), 1 = fp16 bits (uint16), 2 = fp32. */
void orc_dequant(const uint8_t* q, const uint8_t* scales, float s2, int64_t rows, int64_t cols,
                 int out_dtype, int64_t row0, int64_t row1, void* out);

/* ---- local Hessian (hessian.c) ------------------------------------------
 * H[b][i][j] += sum_t x[t][16b+i] * x[t][16b+j] for blocks [blk0, blk1).
 * x: bf16 bits [tokens, cols] with leading dimension ld.  H: double [cols/16][16][16]. */
void orc_hessian_accum(const uint16_t* x, int64_t tokens, int64_t cols, int64_t ld,
                       int64_t blk0, int64_t blk1, double* H);

/* ---- Hessian-weighted E4M3 scale sweep (sweep.c) --------------------------
 * w: [rows, cols] (dtype ORC_BF16 or ORC_F32), ld in elements.  H: double [cols/16][16][16].
 * Rows [row0, row1).  codes: [rows, cols/16]; q: [rows, cols/2] (may be NULL);
 * cost1 / cost2: double [rows, cols/16] (may be NULL). */
void orc_scale_sweep(const void* w, int dtype, int64_t rows, int64_t cols, int64_t ld,
                     const double* H, float amax_w, int64_t row0, int64_t row1,
                     uint8_t* codes, uint8_t* q, double* cost1, double* cost2, uint32_t* flags);

/* ---- MXFP4 -> NVFP4 closed-form cast (cast.c) -------------------------- */
/* Largest unbiased exponent k_max over an E8M0 array; ORs ORC_FLAG_E8M0_NAN. */
int orc_mx_kmax(const uint8_t* e8m0, int64_t n, uint32_t* flags);
/* Rows [row0, row1) of one matrix [rows, cols]; mx_q [rows, cols/2]; e8m0 [rows, cols/32].
 * nv_q [rows, cols/2]; nv_scales [rows, cols/16].  counts[0] += in-window 16-blocks,
 * counts[1] += fallback 16-blocks, counts[2] += lossless 16-blocks. */
void orc_mxfp4_to_nvfp4(const uint8_t* mx_q, const uint8_t* e8m0, int64_t rows, int64_t cols,
                        int k_max, int64_t row0, int64_t row1, uint8_t* nv_q, uint8_t* nv_scales,
                        int64_t* counts);
/* s2 = 2^(k_max-8) and global_amax = 6*448*2^(k_max-8) as FP32; ORs ORC_FLAG_OVERFLOW. */
void orc_mx_global(int k_max, float* s2, float* global_amax, uint32_t* flags);

#ifdef __cplusplus
}
#endif
#endif
