/*
 * nv4.h -- C ABI of libnv4.so, a B200 (sm_100a) NVFP4 block-numerics engine.
 *
 * NVFP4 stores 16-element blocks of E2M1 (FP4) values, each block with one E4M3
 * scale, plus one FP32 second-level scale per tensor.  The library implements
 * the data-parallel hot path of Hessian-weighted NVFP4 post-training
 * quantization as described on these pages (cited by title and section):
 *
 *  [CAL]    "Coder390 NVFP4 calibration method", section 2: max calibration, local
 *           Hessian H = sum X^T X per 16 input channels, Hessian-weighted E4M3 scale
 *           sweep (fp8_scale_sweep); format line: E2M1, 16-element blocks, E4M3 block
 *           scale, FP32 second-level scale.
 *  [FLOW]   "NVFP4 quantization and export flow" (Gemma-2B decoder), sections 3.4-3.6:
 *           per-tensor scale amax/6/448, dynamic activation quantize, DQ1/DQ2;
 *           section 5.4: two FP4 values per byte.
 *  [CAST]   "From MXFP4 to NVFP4: Model Optimizer mixed-precision format conversion",
 *           section 2: closed-form cast, global_amax = 6*448*2^(k_max-8), window 17.
 *  [DSPARK] "From calibration to export: the DSpark three-stage NVFP4 recipe", stage 3:
 *           nibbles reused, scale bytes double.
 *  [FP4]    "FP4 quantization overview", sections 1.1-1.2: E2M1 values, MXFP4 vs NVFP4.
 *
 * Conventions for every entry point
 *  - The caller owns all memory.  The library allocates nothing: no device memory,
 *    no host memory that outlives a call.
 *  - Pointers named d_* and all tensor pointers are DEVICE pointers.  Job arrays
 *    of the *_batched calls are HOST arrays, read during the call only.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  No call synchronizes the host.  Device scalars (amax, s2)
 *    travel by device pointer, so a chain of calls needs no host round trip.
 *  - The return status covers argument validation and launch errors.  Data-dependent
 *    conditions are OR-ed into the caller's flag word *d_flags (device, uint32,
 *    zeroed by the caller; may be NULL to ignore them).  Kernels never trap.
 *  - Layouts are row-major.  `ld` is a leading dimension in elements.  A 16-element
 *    block b of a row covers columns 16b..16b+15.  Packed FP4: byte i of a row holds
 *    element 2i in bits 0-3 and element 2i+1 in bits 4-7; an E2M1 code is
 *    sign(bit 3) | exponent(bits 2-1) | mantissa(bit 0).  Block scales are raw E4M3
 *    (fn) bytes, [rows, cols/16].
 *  - Alignment: tensor pointers 16-byte aligned and ld*element_size a multiple of
 *    16 bytes, else NV4_ERR_ALIGN (there is no slower unaligned path).
 *  - Calls on different streams that write the same buffers race; the library adds
 *    no ordering of its own.
 */
#ifndef NV4_H
#define NV4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NV4_API __attribute__((visibility("default")))
#else
#define NV4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NV4_OK = 0,
    NV4_ERR_NULL = 1,    /* a required pointer is NULL                               */
    NV4_ERR_SHAPE = 2,   /* negative size, cols % 16 != 0 (% 32 for MXFP4), ld < cols */
    NV4_ERR_ALIGN = 3,   /* pointer or ld*element_size not a multiple of 16 bytes    */
    NV4_ERR_DTYPE = 4,   /* element type not supported by this entry point           */
    NV4_ERR_CUDA = 5,    /* a CUDA runtime call or kernel launch failed              */
    NV4_ERR_LIMIT = 6    /* a size exceeds what one call supports (see the call)     */
} nv4_status;

typedef enum { NV4_BF16 = 0, NV4_FP16 = 1, NV4_FP32 = 2 } nv4_dtype;

/* data-dependent flags OR-ed into *d_flags */
#define NV4_FLAG_NONFINITE 1u  /* a NaN or Inf was read; affected outputs are unspecified */
#define NV4_FLAG_E8M0_NAN  2u  /* an E8M0 scale byte 0xFF (NaN) was read                  */
#define NV4_FLAG_OVERFLOW  4u  /* a second-level scale or global amax is not finite       */
#define NV4_FLAG_TIMEOUT   8u  /* a bounded wait inside a kernel gave up; outputs of that
                                  call are incomplete                                     */

/* Human-readable name of a status code (static storage). */
NV4_API const char* nv4_status_str(nv4_status s);

/* Library ABI version (major*100 + minor). */
NV4_API int nv4_version(void);

/* ---------------------------------------------------------------------------
 * nv4_tensor_amax -- per-tensor absolute maximum, as a running maximum.
 * [CAL] section 2 step 1 (max calibration records the largest |w| and |x| of each
 * layer over the calibration data, the initial scales); [FLOW] 3.4 (the calibrated
 * amax gives the per-tensor scale).
 *
 *   *d_amax = max(*d_amax, max_i |x[i]|)
 *
 * x      : n elements of type dt (NV4_BF16 or NV4_FP32), contiguous, 16-byte aligned.
 * d_amax : one float on the device, holding +0.0 or a previous amax before the first
 *          call (a running max over calibration batches needs no reset between them).
 * NaN elements are skipped; NaN or Inf sets NV4_FLAG_NONFINITE.  n == 0 is a no-op.
 */
NV4_API nv4_status nv4_tensor_amax(const void* x, nv4_dtype dt, int64_t n, float* d_amax,
                           uint32_t* d_flags, void* stream);

/* Batched form: the amax of several tensors of one dtype in one launch, each into its
 * own d_amax (e.g. the 15 activation shapes of a quantization sweep).  Per job the
 * rules of nv4_tensor_amax; n < 2^37 elements per job; at most 128 jobs (NV4_ERR_LIMIT
 * beyond). */
typedef struct {
    const void* x;      /* n elements, contiguous, 16-byte aligned */
    int64_t n;
    float* d_amax;
} nv4_amax_job;

NV4_API nv4_status nv4_tensor_amax_batched(const nv4_amax_job* jobs, int n_jobs, nv4_dtype dt,
                                   uint32_t* d_flags, void* stream);

/* ---------------------------------------------------------------------------
 * nv4_act_quant -- dynamic NVFP4 quantization of activations.  [FLOW] 3.4-3.5:
 * the per-tensor scale comes from a (calibrated or just measured) amax, the block
 * scales are computed at run time from the data; [CAL] format line; [FLOW] 5.4.
 *
 *   s2        = RN32(amax / 2688)                       (2688 = 6 * 448)
 *   per block : a_b = max|x|, s_b = E4M3 nearest to a_b / (6*s2) (ties to even code,
 *               saturating at 448), S = RN32(s_b * s2),
 *               code_i = sign(x_i) | E2M1 magnitude nearest to |x_i| / S (ties to even)
 *   amax == 0 gives s2 = 0, block scale 0 and sign-only codes.
 *
 * x      : bf16 [rows, cols], leading dimension ld (ld % 8 == 0).  cols % 16 == 0.
 * d_amax : device float (e.g. the output of nv4_tensor_amax), read on the device.
 * q      : [rows, cols/2] bytes, contiguous.   scales : [rows, cols/16] E4M3 bytes.
 * d_s2   : device float receiving s2, also when rows or cols is 0 (then x, q and scales
 *          are not read and may be NULL).  The same holds for every entry point below that
 *          writes a second-level scale (d_s2, d_scale) from d_amax.
 * Limit: rows * cols/16 < 2^30 blocks per call (NV4_ERR_LIMIT beyond).
 */
NV4_API nv4_status nv4_act_quant(const void* x, int64_t rows, int64_t cols, int64_t ld,
                         const float* d_amax, uint8_t* q, uint8_t* scales, float* d_s2,
                         uint32_t* d_flags, void* stream);

/* Batched form: several BF16 tensors, each with its own amax and s2, in one launch.
 * Per job the rules, layouts and limits of nv4_act_quant; at most 128 jobs. */
typedef struct {
    const void* x;      /* bf16 [rows, cols], leading dimension ld */
    int64_t rows, cols, ld;
    const float* d_amax;
    uint8_t* q;         /* [rows, cols/2] */
    uint8_t* scales;    /* [rows, cols/16] */
    float* d_s2;
} nv4_act_job;

NV4_API nv4_status nv4_act_quant_batched(const nv4_act_job* jobs, int n_jobs, uint32_t* d_flags,
                                 void* stream);

/* ---------------------------------------------------------------------------
 * nv4_weight_quant_rtn -- static round-to-nearest NVFP4 quantization of a weight
 * tensor with max-calibrated block scales: [FLOW] 3.5 (weights quantized once, ahead
 * of time) with the block arithmetic of nv4_act_quant; [CAL] section 2 step 1 (max
 * calibration gives the initial scale that the sweep of nv4_scale_sweep improves on).
 *
 * w      : [rows, cols] of dt (NV4_BF16 or NV4_FP32), leading dimension ld (16-byte
 *          multiple), 16-byte aligned.  cols % 16 == 0.
 * d_amax : device float, the weight tensor's amax.  Other arguments as nv4_act_quant.
 * Limit: rows * cols/16 < 2^30 blocks per call (NV4_ERR_LIMIT beyond).
 */
NV4_API nv4_status nv4_weight_quant_rtn(const void* w, nv4_dtype dt, int64_t rows, int64_t cols, int64_t ld,
                                const float* d_amax, uint8_t* q, uint8_t* scales, float* d_s2,
                                uint32_t* d_flags, void* stream);

/* Batched form: several weight tensors of one dtype (e.g. a layer's projections), each
 * with its own amax and s2, in one launch.  Per job the rules, layouts and limits of
 * nv4_weight_quant_rtn (the job struct is nv4_act_job with w in place of x).
 * jobs: host array of n_jobs descriptors, read before the call returns (caller-owned).
 * n_jobs == 0 is a no-op; n_jobs < 0 gives NV4_ERR_SHAPE, a null table NV4_ERR_NULL and
 * more than 128 jobs NV4_ERR_LIMIT; jobs with rows or cols == 0 quantize nothing but still
 * receive their s2 (their x, q and scales may be NULL).  Every job
 * is validated before anything is launched. */
NV4_API nv4_status nv4_weight_quant_rtn_batched(const nv4_act_job* jobs, int n_jobs, nv4_dtype dt,
                                        uint32_t* d_flags, void* stream);

/* ---------------------------------------------------------------------------
 * nv4_fake_qdq -- fused fake quantization: nv4_act_quant followed by nv4_dequant in
 * one pass, without materializing codes or scales ([FLOW] 3.4: quantizer, then DQ1
 * and DQ2; the quantize-dequantize a calibration forward pass runs on activations).
 * out = RN_out(RN32(e2m1(code) * S)) with code, S exactly as nv4_act_quant.
 *
 * x      : bf16 [rows, cols], leading dimension ld (ld % 8 == 0), 16-byte aligned.
 * out    : [rows, cols] of out_dt (NV4_BF16, NV4_FP16 or NV4_FP32), leading dimension
 *          ld_out (a 16-byte multiple), 16-byte aligned; may equal x when out_dt is
 *          NV4_BF16 and ld_out == ld (in place).
 * d_amax, d_s2, d_flags as nv4_act_quant.  Limit: rows * cols/16 < 2^30 blocks.
 */
NV4_API nv4_status nv4_fake_qdq(const void* x, int64_t rows, int64_t cols, int64_t ld, const float* d_amax,
                        nv4_dtype out_dt, void* out, int64_t ld_out, float* d_s2, uint32_t* d_flags,
                        void* stream);

/* ---------------------------------------------------------------------------
 * nv4_dequant -- the two-step dequantization of [FLOW] 3.4 / 5.4:
 *   DQ1: S = RN32(s_b * s2);  DQ2: y = RN32(e2m1(code) * S), then rounded to out_dt
 *   (NV4_BF16 default, NV4_FP16, or NV4_FP32 as is), ties to even, overflow to inf.
 * q [rows, cols/2], scales [rows, cols/16] (both 16-byte aligned), d_s2 device float; out [rows, cols]
 * contiguous, 16-byte aligned.  cols % 16 == 0.  Limit: rows * cols/16 < 2^30 blocks
 * per call (NV4_ERR_LIMIT beyond).
 */
NV4_API nv4_status nv4_dequant(const uint8_t* q, const uint8_t* scales, const float* d_s2,
                       int64_t rows, int64_t cols, nv4_dtype out_dt, void* out, void* stream);

/* Batched form: several tensors to one out_dt in one launch; per job the rules,
 * layouts and limits of nv4_dequant; at most 128 jobs. */
typedef struct {
    const uint8_t* q;       /* [rows, cols/2] */
    const uint8_t* scales;  /* [rows, cols/16] */
    const float* d_s2;
    int64_t rows, cols;
    void* out;              /* [rows, cols] of out_dt, contiguous */
} nv4_dequant_job;

NV4_API nv4_status nv4_dequant_batched(const nv4_dequant_job* jobs, int n_jobs, nv4_dtype out_dt,
                               void* stream);

/* ---------------------------------------------------------------------------
 * nv4_hessian_accum -- local Hessian per 16-input-channel block, [CAL] section 2
 * step 2 (full-precision forward, H = sum X^T X accumulated per 16 channels at the
 * layer input):
 *
 *   H[b][i][j] += sum_t x[t][16b+i] * x[t][16b+j]      (FP32 accumulation)
 *
 * x : bf16 [tokens, cols], leading dimension ld (ld % 8 == 0), cols % 16 == 0.
 * H : float [cols/16][16][16] on the device, accumulated (+=); zero it before the
 *     first calibration batch.  The result is deterministic (fixed reduction order).
 * A non-finite partial sum sets NV4_FLAG_NONFINITE.
 */
NV4_API nv4_status nv4_hessian_accum(const void* x, int64_t tokens, int64_t cols, int64_t ld,
                             float* H, uint32_t* d_flags, void* stream);

typedef struct {
    const void* x;      /* bf16 [tokens, cols], leading dimension ld */
    int64_t tokens, cols, ld;
    float* H;           /* [cols/16][16][16], +=; distinct jobs need distinct H */
} nv4_hessian_job;

/* Batched form: all jobs in one launch (e.g. the experts of an MoE layer).
 * At most 128 jobs and 65535 64-column slabs in total per call (NV4_ERR_LIMIT beyond). */
NV4_API nv4_status nv4_hessian_accum_batched(const nv4_hessian_job* jobs, int n_jobs,
                                     uint32_t* d_flags, void* stream);

/* ---------------------------------------------------------------------------
 * nv4_scale_sweep -- Hessian-weighted E4M3 block-scale search with NVFP4 pack of
 * the winner, [CAL] section 2 step 3 (fp8_scale_sweep over all E4M3 scale values,
 * minimising (W - Wq)^T H (W - Wq) per 16-element weight block).
 *
 *   s2 = RN32(amax_w / 2688)
 *   for every block w and code c in 0x00..0x7E (the 127 finite non-negative codes):
 *     S_c = RN32(e4m3(c) * s2), q = E2M1(w / S_c) as in nv4_act_quant,
 *     e = w - e2m1(q) * S_c, cost_c = e^T H_b e
 *   winner = argmin cost_c, ties to the lowest code.
 *
 * w        : [rows, cols] of dt (NV4_BF16 or NV4_FP32), leading dimension ld.
 * H        : float [cols/16][16][16] (symmetric; e.g. from nv4_hessian_accum).
 * d_amax_w : device float, the weight tensor's amax.
 * codes    : [rows, cols/16] winning E4M3 codes.
 * q        : [rows, cols/2] packed E2M1 codes at the winning scale, or NULL.
 * cost1    : [rows, cols/16] float winning cost, or NULL.
 * cost2    : [rows, cols/16] float smallest cost above the winner's (+inf if none),
 *            or NULL -- a near-tie diagnostic.
 * Accuracy: the winner is the exact argmin except where the two best costs lie within
 * 1e-5 relative of each other.  Costs are evaluated in FP32 where the block column's
 * Hessian bounds their error well enough for that (error <= 29 * 2^-24 * (2 - rho) / mu
 * relative, rho the Gershgorin ratio and mu a certified lower bound of the smallest
 * eigenvalue of the diagonally scaled H_b; certified when <= 4e-6); in the other
 * columns a block whose FP32 runner-up is within three times that error of the winner
 * or ties it exactly, every block when cost1 or cost2 is requested, and every block of
 * a column without a valid bound (mu < 1/32, error bound above 2^-12, indefinite or
 * non-finite H_b) is searched exhaustively with FP64 costs.  cost1 and cost2 are then
 * the FP64 costs rounded to FP32.
 * The search is exact over all 127 codes but skips the cost of candidates that a
 * lower bound proves cannot be the winner or, when cost2 is requested, the runner-up
 * (sweep.cu states the bounds): codes and q are the same with or without the cost
 * outputs, and cheapest without cost2.  The optional per-job work counter reports
 * how much of the search ran: candidate halves (8 elements each: a candidate is visited
 * half by half and its second half only when the first does not rule it out) and
 * quadratic forms evaluated.
 */
NV4_API nv4_status nv4_scale_sweep(const void* w, nv4_dtype dt, int64_t rows, int64_t cols, int64_t ld,
                           const float* H, const float* d_amax_w, uint8_t* codes, uint8_t* q,
                           float* cost1, float* cost2, uint32_t* d_flags, void* stream);

typedef struct {
    const void* w;      /* [rows, cols] of the call's dt, leading dimension ld */
    int64_t rows, cols, ld;
    const float* H;     /* [cols/16][16][16] */
    const float* d_amax_w;
    uint8_t* codes;     /* [rows, cols/16] */
    uint8_t* q;         /* [rows, cols/2] or NULL */
    float* cost1;       /* or NULL */
    float* cost2;       /* or NULL */
    unsigned long long* d_work;  /* or NULL: [0] += half-candidates visited (8 elements each),
                                    [1] += costs evaluated */
} nv4_sweep_job;

/* Batched form (e.g. all gate/up/down matrices of an expert stack) in one launch.
 * At most 192 jobs per call (NV4_ERR_LIMIT beyond). */
NV4_API nv4_status nv4_scale_sweep_batched(const nv4_sweep_job* jobs, int n_jobs, nv4_dtype dt,
                                   uint32_t* d_flags, void* stream);

/* ---------------------------------------------------------------------------
 * nv4_mxfp4_to_nvfp4 -- closed-form MXFP4 -> NVFP4 cast of one matrix, [CAST] section 2,
 * [DSPARK] stage 3.
 *
 *   k_j = e8m0_j - 127, k_max = max_j k_j over the matrix, m = k_max - 8
 *   *d_s2 = 2^m, *d_global_amax = 6*448*2^m (FP32; NV4_FLAG_OVERFLOW if not finite)
 *   each 32-element MX block j gives two 16-element NVFP4 blocks:
 *     k_max - k_j <= 17 : scale code encodes 2^(k_j - m) exactly, nibbles copied
 *     otherwise         : re-quantized from the exact values e2m1*2^k_j with the
 *                         nv4_act_quant rules (block amax max|w_block|, s2 = 2^m)
 *
 * mx_q [rows, cols/2] nibbles, e8m0 [rows, cols/32]; cols % 32 == 0.
 * nv_q [rows, cols/2] (may equal mx_q: then only fallback blocks are rewritten),
 * nv_scales [rows, cols/16].  d_counts: 3 unsigned long long on the device,
 * accumulated (+=): [0] in-window 16-blocks, [1] fallback 16-blocks, [2] lossless
 * 16-blocks (NVFP4 dequant equal to the MXFP4 dequant bit for bit).  An E8M0 byte
 * 0xFF sets NV4_FLAG_E8M0_NAN and is excluded from k_max; its blocks are unspecified.
 */
NV4_API nv4_status nv4_mxfp4_to_nvfp4(const uint8_t* mx_q, const uint8_t* e8m0, int64_t rows, int64_t cols,
                              uint8_t* nv_q, uint8_t* nv_scales, float* d_global_amax, float* d_s2,
                              unsigned long long* d_counts, uint32_t* d_flags, void* stream);

typedef struct {
    const uint8_t* mx_q;
    const uint8_t* e8m0;
    int64_t rows, cols;
    uint8_t* nv_q;
    uint8_t* nv_scales;
    float* d_global_amax;
    float* d_s2;
    int32_t group;      /* < 0: the matrix has its own scale_2.  Jobs of one call with the
                           same group id >= 0 share one scale_2 ([CAST] section 3: routed
                           experts' w1 and w3 with one scale_2): k_max is the largest
                           exponent over all of their E8M0 codes, each member's window and
                           fallback are taken against it, and every member's d_s2 and
                           d_global_amax receive the shared values. */
} nv4_cast_job;

/* Batched form: one launch for many matrices (each with its own k_max unless grouped).
 * At most 128 jobs per call (NV4_ERR_LIMIT beyond). */
NV4_API nv4_status nv4_mxfp4_to_nvfp4_batched(const nv4_cast_job* jobs, int n_jobs,
                                      unsigned long long* d_counts, uint32_t* d_flags, void* stream);

/* ---------------------------------------------------------------------------
 * W4A4 GEMM on the Blackwell block-scaled tensor cores ([FP4] section 4.1: tcgen05.mma
 * with reorganized scale factors; [CAST] section 4: activations and weights NVFP4).
 *
 * nv4_mma_scale_bytes / nv4_scales_to_mma_layout -- the block scales [rows, cols/16]
 * written by nv4_act_quant, nv4_weight_quant_rtn or nv4_scale_sweep, rearranged into
 * the layout the MMA reads: 512-byte atoms of 128 rows x 4 scales; atom (r/128, j/4)
 * starts at ((r/128) * ceil(cols/64) + j/4) * 512 and holds scale (r, j) at byte
 * (r%32)*16 + ((r%128)/32)*4 + j%4.  Rows pad to 128 and scale columns to 4, with
 * zeros.  out: nv4_mma_scale_bytes(rows, cols) bytes, 16-byte aligned.  The size
 * function returns 0 for invalid shapes.
 *
 * nv4_gemm_nvfp4 -- D[m, n] = s2_A * s2_B * sum_k A[m, k] * B[n, k] for NVFP4 operands
 * given as packed codes qa [M, K/2], qb [N, K/2] (contiguous, 16-byte aligned), their
 * scales in the MMA layout, and device FP32 second-level scales d_s2a, d_s2b.  Products
 * of E2M1 values and E4M3 scales are exact; accumulation is FP32 on the tensor cores;
 * out (NV4_BF16 or NV4_FP32, [M, N] with leading dimension ldd) is RN of the FP32
 * accumulator times RN32(s2_A * s2_B).  Shapes: M % 128 == 0, N % 128 == 0,
 * K % 256 == 0 (NV4_ERR_SHAPE otherwise).
 */
NV4_API size_t nv4_mma_scale_bytes(int64_t rows, int64_t cols);
NV4_API nv4_status nv4_scales_to_mma_layout(const uint8_t* scales, int64_t rows, int64_t cols, uint8_t* out,
                                    void* stream);
NV4_API nv4_status nv4_gemm_nvfp4(const uint8_t* qa, const uint8_t* sfa_mma, const float* d_s2a,
                          const uint8_t* qb, const uint8_t* sfb_mma, const float* d_s2b,
                          int64_t M, int64_t N, int64_t K, nv4_dtype out_dt, void* out, int64_t ldd,
                          uint32_t* d_flags, void* stream);

/* ---------------------------------------------------------------------------
 * Format variants ([FP4] sections 1.2 and 3.2; [CAL] layer table and the note under it).
 *
 * nv4_mxfp4_quant -- MXFP4 round-to-nearest quantization: 32-element blocks along a row,
 * one E8M0 scale 2^e per block with e = floor(log2 amax_block) - 2 clamped to [-127, 127]
 * (code e + 127; an all-zero block gets code 0), elements E2M1 nearest to x / 2^e (ties to
 * even, saturating at 6, sign kept).  A block holding NaN or Inf gets code 0xFF and sets
 * NV4_FLAG_NONFINITE.  x: [rows, cols] of dt (NV4_BF16 or NV4_FP32), leading dimension ld
 * (16-byte multiple), cols % 32 == 0.  q [rows, cols/2] (two codes per byte, low nibble =
 * even element) and e8m0 [rows, cols/32], contiguous.  The output feeds
 * nv4_mxfp4_to_nvfp4 directly.
 * nv4_mxfp4_dequant -- out = RN_out(RN32(e2m1(code) * 2^(e8m0 - 127))) as NV4_BF16/FP16/FP32
 * (NaN for code 0xFF).  out [rows, cols] contiguous, 16-byte aligned.
 *
 * nv4_fp8_quant -- FP8 E4M3 with one static per-tensor scale (W8A8 layers with calibrated
 * scales): s = RN32(amax / 448) written to *d_scale, code = sign | E4M3 nearest to |x| / s
 * (ties to even, saturating at 448); s = 0 gives signed zeros.  x as above with
 * cols % 16 == 0; q [rows, cols] contiguous.
 * nv4_fp8_dequant -- out = RN_out(RN32(e4m3(code) * s)), as nv4_dequant's DQ2.
 * Limits: fewer than 2^31 16-element groups per call (NV4_ERR_LIMIT beyond).
 */
NV4_API nv4_status nv4_mxfp4_quant(const void* x, nv4_dtype dt, int64_t rows, int64_t cols, int64_t ld,
                           uint8_t* q, uint8_t* e8m0, uint32_t* d_flags, void* stream);
NV4_API nv4_status nv4_mxfp4_dequant(const uint8_t* q, const uint8_t* e8m0, int64_t rows, int64_t cols,
                             nv4_dtype out_dt, void* out, void* stream);
NV4_API nv4_status nv4_fp8_quant(const void* x, nv4_dtype dt, int64_t rows, int64_t cols, int64_t ld,
                         const float* d_amax, uint8_t* q, float* d_scale, uint32_t* d_flags, void* stream);
NV4_API nv4_status nv4_fp8_dequant(const uint8_t* q, const float* d_scale, int64_t rows, int64_t cols,
                           nv4_dtype out_dt, void* out, void* stream);

/* ---------------------------------------------------------------------------
 * Block Hadamard rotation fused with FP4 quantization ([FP4] section 3.1: blocks rotated
 * by H / sqrt(n) so that outliers spread before quantization; section 4.1: transform
 * kernels for block sizes 16, 32, 64 and 128).  Along each row of x (bf16 [rows, cols],
 * leading dimension ld, ld % 8 == 0, 16-byte aligned, cols % 128 == 0), blocks of n in
 * {16, 32, 64, 128} consecutive values become y = RN32(RN64(x_block H_n) * RN64(1/sqrt(n)))
 * with H_n the natural-order (Sylvester) Hadamard matrix; the sums are exact in FP64 for
 * BF16 inputs whose values in a block span fewer than ~38 binades.
 *
 * nv4_hadamard_amax        -- *d_amax = max(*d_amax, max |y|) (running max, as nv4_tensor_amax).
 * nv4_hadamard_mxfp4_quant -- MXFP4 codes and E8M0 scales of y, as nv4_mxfp4_quant.
 * nv4_hadamard_nvfp4_quant -- NVFP4 codes and E4M3 scales of y with s2 = RN32(amax / 2688)
 *                             from *d_amax (e.g. from nv4_hadamard_amax), as nv4_act_quant.
 * Limits: fewer than 2^31 32-element row chunks per call (NV4_ERR_LIMIT).
 */
NV4_API nv4_status nv4_hadamard_amax(const void* x, int64_t rows, int64_t cols, int64_t ld, int n,
                             float* d_amax, uint32_t* d_flags, void* stream);
NV4_API nv4_status nv4_hadamard_mxfp4_quant(const void* x, int64_t rows, int64_t cols, int64_t ld, int n,
                                    uint8_t* q, uint8_t* e8m0, uint32_t* d_flags, void* stream);
NV4_API nv4_status nv4_hadamard_nvfp4_quant(const void* x, int64_t rows, int64_t cols, int64_t ld, int n,
                                    const float* d_amax, uint8_t* q, uint8_t* scales, float* d_s2,
                                    uint32_t* d_flags, void* stream);

/* ---------------------------------------------------------------------------
 * Two-sided block Hadamard rotation of weight tiles fused with FP4 quantization ([FP4]
 * section 3.1: the weight matrix is cut into n x n tiles, n = 16 or 32, and each tile B
 * becomes (H_n / sqrt(n)) B (H_n / sqrt(n))^T = H_n B H_n / n before quantization; H_n is the
 * natural-order (Sylvester) Hadamard matrix, which is symmetric).  Per tile:
 *
 *   y = RN32(exact(H_n B H_n) / n)        (1/n is a power of two: one rounding, to FP32)
 *
 * The kernels form the sums in FP64, exact while a tile's values, as multiples of its
 * smallest unit in the last place, fit 53 bits with 2*log2(n) bits of growth (BF16 tiles
 * spanning fewer than ~35 binades, FP32 tiles fewer than ~19); beyond that the FP64 sum
 * carries a relative error below 2^-52 before the final rounding.
 *
 * w : [rows, cols] of dt (NV4_BF16 or NV4_FP32), leading dimension ld (a 16-byte multiple),
 *     16-byte aligned; rows % n == 0 and cols % 32 == 0 (NV4_ERR_SHAPE otherwise).
 * nv4_hadamard2_rotate       -- out: y as FP32 [rows, cols], contiguous, 16-byte aligned.
 * nv4_hadamard2_amax         -- *d_amax = max(*d_amax, max |y|) (running max, as nv4_tensor_amax).
 * nv4_hadamard2_mxfp4_quant  -- MXFP4 of y along rows (32-element blocks), as nv4_mxfp4_quant.
 * nv4_hadamard2_nvfp4_quant  -- NVFP4 of y along rows with s2 = RN32(amax / 2688) from *d_amax
 *                               (e.g. from nv4_hadamard2_amax), as nv4_weight_quant_rtn.
 * Limits: fewer than 2^31 strips of n x 32 per call.  A NaN or Inf in y sets
 * NV4_FLAG_NONFINITE.
 */
NV4_API nv4_status nv4_hadamard2_rotate(const void* w, nv4_dtype dt, int64_t rows, int64_t cols, int64_t ld, int n,
                                float* out, uint32_t* d_flags, void* stream);
NV4_API nv4_status nv4_hadamard2_amax(const void* w, nv4_dtype dt, int64_t rows, int64_t cols, int64_t ld, int n,
                              float* d_amax, uint32_t* d_flags, void* stream);
NV4_API nv4_status nv4_hadamard2_mxfp4_quant(const void* w, nv4_dtype dt, int64_t rows, int64_t cols, int64_t ld,
                                     int n, uint8_t* q, uint8_t* e8m0, uint32_t* d_flags, void* stream);
NV4_API nv4_status nv4_hadamard2_nvfp4_quant(const void* w, nv4_dtype dt, int64_t rows, int64_t cols, int64_t ld,
                                     int n, const float* d_amax, uint8_t* q, uint8_t* scales, float* d_s2,
                                     uint32_t* d_flags, void* stream);

/* ---------------------------------------------------------------------------
 * nv4_selftest -- checks, on the current device, the hardware FP4/FP8 conversion
 * instructions the kernels rely on (lane order, rounding, sign of zero, saturation).
 * Writes 64 uint32 results to d_out (device); d_out[0] is a bit mask of failed
 * checks (0 = all passed), the rest are the raw values observed.  Not a paper
 * operation: a diagnostic of the build on the GPU it runs on.
 */
NV4_API nv4_status nv4_selftest(uint32_t* d_out, void* stream);

/* ---------------------------------------------------------------------------
 * nv4_fp32_probe -- a microbenchmark of the FP32 pipe, the denominator of the scale
 * sweep's roofline.  Launches `blocks` CTAs of 256 threads; every thread runs `iters`
 * iterations of 128 FLOP of independent fused multiply-adds (16 chains, 4 steps each), as
 * scalar FP32 FMAs (packed = 0) or as packed two-lane FMAs (packed = 1), so one launch does
 * blocks * 256 * iters * 128 FLOP; time it with events.  d_sink: one float per CTA on the device, written only if a
 * chain went NaN (never, for the built-in operands); it keeps the work from being
 * optimized away.  blocks <= 2^20 and iters <= 2^24 (NV4_ERR_LIMIT beyond).
 * Not a paper operation: a measurement of the GPU it runs on.
 */
NV4_API nv4_status nv4_fp32_probe(int packed, uint32_t blocks, uint32_t iters, float* d_sink, void* stream);

/* ---------------------------------------------------------------------------
 * nv4_selftest_wait -- exercises the bounded wait that every pipeline kernel uses (no
 * kernel of this library waits without a time limit): one thread polls the device word
 * *d_flag until it is non-zero or limit_ns (<= 2 s, the kernels' own limit; NV4_ERR_LIMIT
 * beyond) of GPU time has passed.  d_status[0] = 0 if the flag was seen, NV4_FLAG_TIMEOUT
 * if the wait gave up; d_status[1] = microseconds waited.  The kernel always returns.
 * Not a paper operation: the failure-detection path, testable without any fault.
 */
NV4_API nv4_status nv4_selftest_wait(const uint32_t* d_flag, uint64_t limit_ns, uint32_t* d_status, void* stream);

#ifdef __cplusplus
}
#endif
#endif
