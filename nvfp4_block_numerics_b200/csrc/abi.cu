// abi.cu -- the extern "C" entry points of libnv4.so (declared in include/nv4.h):
// argument validation, then one stream-ordered kernel launch per call.
#include <cstdint>

#include "nv4_common.cuh"
#include "nv4_internal.h"

namespace nv4 {

int num_sms()
{
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0u; }

static nv4_status from_cuda(cudaError_t e) { return e == cudaSuccess ? NV4_OK : NV4_ERR_CUDA; }

// ---------------------------------------------------------------- self-test
__global__ void selftest_kernel(uint32_t* out)
{
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    uint32_t fail = 0u;
    // E2M1 pack: lane order, RNE ties (2.5 -> 2), saturation (7 -> 6), sign of zero
    const float v[8] = {0.5f, 6.0f, -1.0f, 0.0f, -0.0f, -0.1f, 7.0f, 2.5f};
    const uint32_t p = cvt_e2m1x8(v);
    out[1] = p;
    if (p != 0x47880A71u) fail |= 1u;
    // E4M3 pair: lane order and saturation
    const uint32_t a = cvt_e4m3x2(1.0f, 448.0f);
    out[2] = a;
    if (a != 0x7E38u) fail |= 2u;
    const uint32_t b = cvt_e4m3x2(0x1p-10f, 0x1.8p-10f);   // tie to even (0), nearest subnormal (1)
    out[3] = b;
    if (b != 0x0100u) fail |= 4u;
    const uint32_t c = cvt_e4m3x2(500.0f, 1e30f);
    out[4] = c;
    if (c != 0x7E7Eu) fail |= 8u;
    // E2M1 -> FP16 decode: lane order and sign
    uint32_t h[4];
    cvt_e2m1x8_to_f16x8(0x47880A71u, h);
    for (int i = 0; i < 4; ++i) out[5 + i] = h[i];
    if (h[0] != 0x46003800u || h[1] != 0x0000BC00u || h[2] != 0x80008000u || h[3] != 0x40004600u) fail |= 16u;
    // BF16 pair packing order and rounding
    uint32_t bf;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(bf) : "f"(3.0f), "f"(1.0f + 0x1p-9f));
    out[9] = bf;
    if (bf != 0x40403F80u) fail |= 32u;
    // E4M3 values used by the kernels
    if (e4m3_value(0x7Eu) != 448.0f || e4m3_value(1u) != 0x1p-9f || e4m3_value(0x38u) != 1.0f) fail |= 64u;
    // exact fallbacks against known answers
    if (e4m3_code_exact(448.0f * 6.0f, 1.0f) != 0x7Eu || e4m3_code_exact(6.0f * 0x1p-10f, 1.0f) != 0u ||
        e4m3_code_exact(6.0f * 0x1.8p-10f, 1.0f) != 1u)
        fail |= 128u;
    if (e2m1_code_exact(2.5f, 1.0f) != 4u || e2m1_code_exact(-0.25f, 1.0f) != 8u ||
        e2m1_code_exact(0.75f, 1.0f) != 2u || e2m1_code_exact(100.0f, 1.0f) != 7u)
        fail |= 256u;
    FastDiv fd(7u);
    if (fd.div(48u) != 6u || fd.div(0xFFFFFFFFu) != 0xFFFFFFFFu / 7u) fail |= 512u;
    out[0] = fail;
}

cudaError_t launch_selftest(uint32_t* d_out, cudaStream_t s)
{
    selftest_kernel<<<1, 32, 0, s>>>(d_out);
    return cudaGetLastError();
}

// The bounded wait every pipeline kernel uses, exercised alone: thread 0 polls *flag
// until it is non-zero or limit_ns of %globaltimer time has passed, then reports which.
__global__ void wait_selftest_kernel(const volatile uint32_t* flag, uint64_t limit_ns, uint32_t* status)
{
    if (threadIdx.x != 0) return;
    const uint64_t t0 = global_ns();
    uint32_t st = kFlagTimeout;
    while (global_ns() - t0 <= limit_ns) {
        if (*flag != 0u) {
            st = 0u;
            break;
        }
        __nanosleep(1000);
    }
    status[0] = st;
    status[1] = (uint32_t)((global_ns() - t0) / 1000u);   // microseconds waited
}

cudaError_t launch_wait_selftest(const uint32_t* flag, uint64_t limit_ns, uint32_t* status, cudaStream_t s)
{
    wait_selftest_kernel<<<1, 32, 0, s>>>(flag, limit_ns, status);
    return cudaGetLastError();
}

// FP32 pipe microbenchmark: every thread runs `iters` iterations of 4 steps of 16
// independent fused multiply-add chains, as scalar fma.rn.f32 (kPacked = false) or as 8
// packed fma.rn.f32x2 (true); 128 FLOP per thread and iteration either way.  The multiplier and addend come from
// the arguments, so nothing folds; the chains end in one store that no input makes
// happen (the sum is finite, never NaN), which keeps them live.
template <bool kPacked>
__global__ void __launch_bounds__(256) fma_probe_kernel(uint32_t iters, float m, float c, float* sink)
{
    const float x0 = __uint2float_rn(threadIdx.x) * 0x1p-20f;
    float sum = 0.0f;
    if constexpr (kPacked) {
        float2 a[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) a[k] = make_float2(x0 + (float)k, x0 - (float)k);
        const float2 m2 = make_float2(m, m), c2 = make_float2(c, c);
#pragma unroll 1
        for (uint32_t it = 0; it < iters; ++it) {
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int k = 0; k < 8; ++k) a[k] = __ffma2_rn(a[k], m2, c2);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) sum += a[k].x + a[k].y;
    } else {
        float a[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) a[k] = x0 + (float)k;
#pragma unroll 1
        for (uint32_t it = 0; it < iters; ++it) {
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int k = 0; k < 16; ++k) a[k] = fmaf(a[k], m, c);
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) sum += a[k];
    }
    if (isnan(sum)) sink[blockIdx.x] = sum;
}

cudaError_t launch_fma_probe(int packed, uint32_t blocks, uint32_t iters, float* sink, cudaStream_t s)
{
    if (packed) fma_probe_kernel<true><<<blocks, 256, 0, s>>>(iters, 0.9999999f, 1e-7f, sink);
    else fma_probe_kernel<false><<<blocks, 256, 0, s>>>(iters, 0.9999999f, 1e-7f, sink);
    return cudaGetLastError();
}

}  // namespace nv4

using namespace nv4;

extern "C" {

const char* nv4_status_str(nv4_status s)
{
    switch (s) {
    case NV4_OK: return "NV4_OK";
    case NV4_ERR_NULL: return "NV4_ERR_NULL: a required pointer is NULL";
    case NV4_ERR_SHAPE: return "NV4_ERR_SHAPE: invalid size or shape";
    case NV4_ERR_ALIGN: return "NV4_ERR_ALIGN: pointer or leading dimension not 16-byte aligned";
    case NV4_ERR_DTYPE: return "NV4_ERR_DTYPE: unsupported element type";
    case NV4_ERR_CUDA: return "NV4_ERR_CUDA: CUDA runtime or launch error";
    case NV4_ERR_LIMIT: return "NV4_ERR_LIMIT: size beyond what one call supports";
    }
    return "unknown nv4_status";
}

int nv4_version(void) { return 100; }

// ---------------------------------------------------------------- amax, act quant, dequant
static nv4_status check_amax(const void* x, int64_t n, const float* d_amax)
{
    if (n < 0) return NV4_ERR_SHAPE;
    if (n == 0) return NV4_OK;
    if (x == nullptr || d_amax == nullptr) return NV4_ERR_NULL;
    if (!aligned16(x)) return NV4_ERR_ALIGN;
    if (n >= (int64_t)1 << 37) return NV4_ERR_LIMIT;
    return NV4_OK;
}

nv4_status nv4_tensor_amax(const void* x, nv4_dtype dt, int64_t n, float* d_amax, uint32_t* d_flags, void* stream)
{
    if (n < 0) return NV4_ERR_SHAPE;
    if (n == 0) return NV4_OK;
    if (x == nullptr || d_amax == nullptr) return NV4_ERR_NULL;
    if (dt != NV4_BF16 && dt != NV4_FP32) return NV4_ERR_DTYPE;
    const nv4_status st = check_amax(x, n, d_amax);
    if (st != NV4_OK) return st;
    const AmaxTask t = {x, n, d_amax};
    return from_cuda(launch_amax(&t, 1, dt == NV4_BF16 ? 0 : 2, d_flags, (cudaStream_t)stream));
}

nv4_status nv4_tensor_amax_batched(const nv4_amax_job* jobs, int n_jobs, nv4_dtype dt, uint32_t* d_flags,
                                   void* stream)
{
    if (n_jobs < 0) return NV4_ERR_SHAPE;
    if (n_jobs == 0) return NV4_OK;
    if (jobs == nullptr) return NV4_ERR_NULL;
    if (n_jobs > kMaxActJobs) return NV4_ERR_LIMIT;
    if (dt != NV4_BF16 && dt != NV4_FP32) return NV4_ERR_DTYPE;
    AmaxTask t[kMaxActJobs];
    for (int i = 0; i < n_jobs; ++i) {
        const nv4_status st = check_amax(jobs[i].x, jobs[i].n, jobs[i].d_amax);
        if (st != NV4_OK) return st;
        t[i] = {jobs[i].x, jobs[i].n, jobs[i].d_amax};
    }
    return from_cuda(launch_amax(t, n_jobs, dt == NV4_BF16 ? 0 : 2, d_flags, (cudaStream_t)stream));
}

// ld_mult: the row pitch that keeps rows 16-byte aligned (8 BF16 or 4 FP32 elements).
static nv4_status check_act(const void* x, int64_t rows, int64_t cols, int64_t ld, const float* d_amax,
                            const uint8_t* q, const uint8_t* scales, const float* d_s2, int64_t ld_mult = 8)
{
    if (rows < 0 || cols < 0 || cols % 16 != 0 || ld < cols) return NV4_ERR_SHAPE;
    if (d_amax == nullptr || d_s2 == nullptr) return NV4_ERR_NULL;
    if (rows == 0 || cols == 0) return NV4_OK;
    if (x == nullptr || q == nullptr || scales == nullptr) return NV4_ERR_NULL;
    if (!aligned16(x) || !aligned16(q) || ld % ld_mult != 0) return NV4_ERR_ALIGN;
    if (rows * (cols / 16) >= (int64_t)1 << 30) return NV4_ERR_LIMIT;
    return NV4_OK;
}

nv4_status nv4_act_quant(const void* x, int64_t rows, int64_t cols, int64_t ld, const float* d_amax, uint8_t* q,
                         uint8_t* scales, float* d_s2, uint32_t* d_flags, void* stream)
{
    const nv4_status st = check_act(x, rows, cols, ld, d_amax, q, scales, d_s2);
    if (st != NV4_OK) return st;
    const QuantTask t = {x, rows, cols, ld, d_amax, q, scales, nullptr, 0, d_s2};
    return from_cuda(launch_block_quant(&t, 1, 0, -1, d_flags, (cudaStream_t)stream));
}

nv4_status nv4_act_quant_batched(const nv4_act_job* jobs, int n_jobs, uint32_t* d_flags, void* stream)
{
    if (n_jobs < 0) return NV4_ERR_SHAPE;
    if (n_jobs == 0) return NV4_OK;
    if (jobs == nullptr) return NV4_ERR_NULL;
    if (n_jobs > kMaxActJobs) return NV4_ERR_LIMIT;
    QuantTask t[kMaxActJobs];
    for (int i = 0; i < n_jobs; ++i) {
        const nv4_act_job& J = jobs[i];
        const nv4_status st = check_act(J.x, J.rows, J.cols, J.ld, J.d_amax, J.q, J.scales, J.d_s2);
        if (st != NV4_OK) return st;
        t[i] = {J.x, J.rows, J.cols, J.ld, J.d_amax, J.q, J.scales, nullptr, 0, J.d_s2};
    }
    return from_cuda(launch_block_quant(t, n_jobs, 0, -1, d_flags, (cudaStream_t)stream));
}

nv4_status nv4_weight_quant_rtn(const void* w, nv4_dtype dt, int64_t rows, int64_t cols, int64_t ld,
                                const float* d_amax, uint8_t* q, uint8_t* scales, float* d_s2, uint32_t* d_flags,
                                void* stream)
{
    if (dt != NV4_BF16 && dt != NV4_FP32) return NV4_ERR_DTYPE;
    if (rows < 0 || cols < 0 || cols % 16 != 0 || ld < cols) return NV4_ERR_SHAPE;
    if (d_amax == nullptr || d_s2 == nullptr) return NV4_ERR_NULL;
    if (rows != 0 && cols != 0) {
        if (w == nullptr || q == nullptr || scales == nullptr) return NV4_ERR_NULL;
        if (!aligned16(w) || !aligned16(q) || ld % (dt == NV4_BF16 ? 8 : 4) != 0) return NV4_ERR_ALIGN;
        if (rows * (cols / 16) >= (int64_t)1 << 30) return NV4_ERR_LIMIT;
    }
    const QuantTask t = {w, rows, cols, ld, d_amax, q, scales, nullptr, 0, d_s2};
    return from_cuda(launch_block_quant(&t, 1, dt == NV4_BF16 ? 0 : 2, -1, d_flags, (cudaStream_t)stream));
}

nv4_status nv4_weight_quant_rtn_batched(const nv4_act_job* jobs, int n_jobs, nv4_dtype dt, uint32_t* d_flags,
                                        void* stream)
{
    if (n_jobs < 0) return NV4_ERR_SHAPE;
    if (n_jobs == 0) return NV4_OK;
    if (jobs == nullptr) return NV4_ERR_NULL;
    if (n_jobs > kMaxActJobs) return NV4_ERR_LIMIT;
    if (dt != NV4_BF16 && dt != NV4_FP32) return NV4_ERR_DTYPE;
    QuantTask t[kMaxActJobs];
    for (int i = 0; i < n_jobs; ++i) {
        const nv4_act_job& J = jobs[i];
        const nv4_status st = check_act(J.x, J.rows, J.cols, J.ld, J.d_amax, J.q, J.scales, J.d_s2,
                                        dt == NV4_BF16 ? 8 : 4);
        if (st != NV4_OK) return st;
        t[i] = {J.x, J.rows, J.cols, J.ld, J.d_amax, J.q, J.scales, nullptr, 0, J.d_s2};
    }
    return from_cuda(launch_block_quant(t, n_jobs, dt == NV4_BF16 ? 0 : 2, -1, d_flags, (cudaStream_t)stream));
}

nv4_status nv4_fake_qdq(const void* x, int64_t rows, int64_t cols, int64_t ld, const float* d_amax,
                        nv4_dtype out_dt, void* out, int64_t ld_out, float* d_s2, uint32_t* d_flags, void* stream)
{
    if (out_dt != NV4_BF16 && out_dt != NV4_FP16 && out_dt != NV4_FP32) return NV4_ERR_DTYPE;
    if (rows < 0 || cols < 0 || cols % 16 != 0 || ld < cols || ld_out < cols) return NV4_ERR_SHAPE;
    if (d_amax == nullptr || d_s2 == nullptr) return NV4_ERR_NULL;
    if (rows != 0 && cols != 0) {
        if (x == nullptr || out == nullptr) return NV4_ERR_NULL;
        if (!aligned16(x) || !aligned16(out) || ld % 8 != 0 || ld_out % (out_dt == NV4_FP32 ? 4 : 8) != 0)
            return NV4_ERR_ALIGN;
        if (rows * (cols / 16) >= (int64_t)1 << 30) return NV4_ERR_LIMIT;
    }
    const QuantTask t = {x, rows, cols, ld, d_amax, nullptr, nullptr, out, ld_out, d_s2};
    return from_cuda(launch_block_quant(&t, 1, 0, (int)out_dt, d_flags, (cudaStream_t)stream));
}

static nv4_status check_dequant(const uint8_t* q, const uint8_t* scales, const float* d_s2, int64_t rows,
                                int64_t cols, const void* out)
{
    if (rows < 0 || cols < 0 || cols % 16 != 0) return NV4_ERR_SHAPE;
    if (rows == 0 || cols == 0) return NV4_OK;
    if (q == nullptr || scales == nullptr || d_s2 == nullptr || out == nullptr) return NV4_ERR_NULL;
    if (!aligned16(q) || !aligned16(scales) || !aligned16(out)) return NV4_ERR_ALIGN;
    if (rows * (cols / 16) >= (int64_t)1 << 30) return NV4_ERR_LIMIT;
    return NV4_OK;
}

nv4_status nv4_dequant(const uint8_t* q, const uint8_t* scales, const float* d_s2, int64_t rows, int64_t cols,
                       nv4_dtype out_dt, void* out, void* stream)
{
    if (rows < 0 || cols < 0 || cols % 16 != 0) return NV4_ERR_SHAPE;
    if (out_dt != NV4_BF16 && out_dt != NV4_FP16 && out_dt != NV4_FP32) return NV4_ERR_DTYPE;
    const nv4_status st = check_dequant(q, scales, d_s2, rows, cols, out);
    if (st != NV4_OK || rows == 0 || cols == 0) return st;
    const DequantTask t = {q, scales, d_s2, rows, cols, out};
    return from_cuda(launch_dequant(&t, 1, (int)out_dt, (cudaStream_t)stream));
}

nv4_status nv4_dequant_batched(const nv4_dequant_job* jobs, int n_jobs, nv4_dtype out_dt, void* stream)
{
    if (n_jobs < 0) return NV4_ERR_SHAPE;
    if (n_jobs == 0) return NV4_OK;
    if (jobs == nullptr) return NV4_ERR_NULL;
    if (n_jobs > kMaxActJobs) return NV4_ERR_LIMIT;
    if (out_dt != NV4_BF16 && out_dt != NV4_FP16 && out_dt != NV4_FP32) return NV4_ERR_DTYPE;
    DequantTask t[kMaxActJobs];
    for (int i = 0; i < n_jobs; ++i) {
        const nv4_dequant_job& J = jobs[i];
        const nv4_status st = check_dequant(J.q, J.scales, J.d_s2, J.rows, J.cols, J.out);
        if (st != NV4_OK) return st;
        t[i] = {J.q, J.scales, J.d_s2, J.rows, J.cols, J.out};
    }
    return from_cuda(launch_dequant(t, n_jobs, (int)out_dt, (cudaStream_t)stream));
}

static nv4_status check_hessian_job(const nv4_hessian_job& J)
{
    if (J.tokens < 0 || J.cols < 0 || J.cols % 16 != 0 || J.ld < J.cols) return NV4_ERR_SHAPE;
    if (J.tokens == 0 || J.cols == 0) return NV4_OK;
    if (J.x == nullptr || J.H == nullptr) return NV4_ERR_NULL;
    if (!aligned16(J.x) || J.ld % 8 != 0) return NV4_ERR_ALIGN;
    if (J.tokens >= ((int64_t)1 << 31) || J.cols >= ((int64_t)1 << 31)) return NV4_ERR_LIMIT;
    return NV4_OK;
}

nv4_status nv4_hessian_accum_batched(const nv4_hessian_job* jobs, int n_jobs, uint32_t* d_flags, void* stream)
{
    if (n_jobs < 0) return NV4_ERR_SHAPE;
    if (n_jobs == 0) return NV4_OK;
    if (jobs == nullptr) return NV4_ERR_NULL;
    if (n_jobs > kMaxHessianJobs) return NV4_ERR_LIMIT;
    int64_t slabs = 0;
    for (int i = 0; i < n_jobs; ++i) {
        const nv4_status st = check_hessian_job(jobs[i]);
        if (st != NV4_OK) return st;
        slabs += (jobs[i].cols + 63) / 64;
    }
    if (slabs > 65535) return NV4_ERR_LIMIT;
    int bad = -1;
    const cudaError_t e = launch_hessian(jobs, n_jobs, d_flags, (cudaStream_t)stream, &bad);
    if (bad >= 0) return NV4_ERR_ALIGN;   // the TMA descriptor rejected the tensor's layout
    return from_cuda(e);
}

nv4_status nv4_hessian_accum(const void* x, int64_t tokens, int64_t cols, int64_t ld, float* H, uint32_t* d_flags,
                             void* stream)
{
    nv4_hessian_job j;
    j.x = x; j.tokens = tokens; j.cols = cols; j.ld = ld; j.H = H;
    return nv4_hessian_accum_batched(&j, 1, d_flags, stream);
}

static nv4_status check_sweep_job(const nv4_sweep_job& J, nv4_dtype dt)
{
    if (J.rows < 0 || J.cols < 0 || J.cols % 16 != 0 || J.ld < J.cols) return NV4_ERR_SHAPE;
    if (J.d_amax_w == nullptr) return NV4_ERR_NULL;
    if (J.rows == 0 || J.cols == 0) return NV4_OK;
    if (J.w == nullptr || J.H == nullptr || J.codes == nullptr) return NV4_ERR_NULL;
    const int64_t esz = dt == NV4_FP32 ? 4 : 2;
    if (!aligned16(J.w) || (J.ld * esz) % 16 != 0 || (J.q != nullptr && !aligned16(J.q))) return NV4_ERR_ALIGN;
    if (J.rows >= ((int64_t)1 << 31) || J.cols >= ((int64_t)1 << 31)) return NV4_ERR_LIMIT;
    return NV4_OK;
}

nv4_status nv4_scale_sweep_batched(const nv4_sweep_job* jobs, int n_jobs, nv4_dtype dt, uint32_t* d_flags,
                                   void* stream)
{
    if (n_jobs < 0) return NV4_ERR_SHAPE;
    if (dt != NV4_BF16 && dt != NV4_FP32) return NV4_ERR_DTYPE;
    if (n_jobs == 0) return NV4_OK;
    if (jobs == nullptr) return NV4_ERR_NULL;
    if (n_jobs > kMaxSweepJobs) return NV4_ERR_LIMIT;
    int64_t ctas = 0;
    for (int i = 0; i < n_jobs; ++i) {
        const nv4_status st = check_sweep_job(jobs[i], dt);
        if (st != NV4_OK) return st;
        ctas += ((jobs[i].rows + 127) / 128) * (jobs[i].cols / 16);
    }
    if (ctas >= ((int64_t)1 << 31)) return NV4_ERR_LIMIT;
    return from_cuda(launch_sweep(jobs, n_jobs, dt == NV4_BF16 ? 0 : 2, d_flags, (cudaStream_t)stream));
}

nv4_status nv4_scale_sweep(const void* w, nv4_dtype dt, int64_t rows, int64_t cols, int64_t ld, const float* H,
                           const float* d_amax_w, uint8_t* codes, uint8_t* q, float* cost1, float* cost2,
                           uint32_t* d_flags, void* stream)
{
    nv4_sweep_job j;
    j.w = w; j.rows = rows; j.cols = cols; j.ld = ld; j.H = H; j.d_amax_w = d_amax_w;
    j.codes = codes; j.q = q; j.cost1 = cost1; j.cost2 = cost2; j.d_work = nullptr;
    return nv4_scale_sweep_batched(&j, 1, dt, d_flags, stream);
}

static nv4_status check_cast_job(const nv4_cast_job& J)
{
    if (J.rows < 0 || J.cols < 0 || J.cols % 32 != 0) return NV4_ERR_SHAPE;
    if (J.rows == 0 || J.cols == 0) return NV4_OK;
    if (J.mx_q == nullptr || J.e8m0 == nullptr || J.nv_q == nullptr || J.nv_scales == nullptr ||
        J.d_global_amax == nullptr || J.d_s2 == nullptr)
        return NV4_ERR_NULL;
    if (!aligned16(J.mx_q) || !aligned16(J.e8m0) || !aligned16(J.nv_q) || !aligned16(J.nv_scales))
        return NV4_ERR_ALIGN;
    if (J.rows * (J.cols / 32) >= ((int64_t)1 << 31)) return NV4_ERR_LIMIT;
    // in-place is allowed only as exact aliasing of the nibble buffers
    const uint8_t* a = J.mx_q;
    const uint8_t* b = J.nv_q;
    const int64_t bytes = J.rows * (J.cols / 2);
    if (a != b && a < b + bytes && b < a + bytes) return NV4_ERR_SHAPE;
    return NV4_OK;
}

nv4_status nv4_mxfp4_to_nvfp4_batched(const nv4_cast_job* jobs, int n_jobs, unsigned long long* d_counts,
                                      uint32_t* d_flags, void* stream)
{
    if (n_jobs < 0) return NV4_ERR_SHAPE;
    if (n_jobs == 0) return NV4_OK;
    if (jobs == nullptr) return NV4_ERR_NULL;
    if (n_jobs > kMaxCastJobs) return NV4_ERR_LIMIT;
    for (int i = 0; i < n_jobs; ++i) {
        const nv4_status st = check_cast_job(jobs[i]);
        if (st != NV4_OK) return st;
    }
    return from_cuda(launch_cast(jobs, n_jobs, d_counts, d_flags, (cudaStream_t)stream));
}

nv4_status nv4_mxfp4_to_nvfp4(const uint8_t* mx_q, const uint8_t* e8m0, int64_t rows, int64_t cols, uint8_t* nv_q,
                              uint8_t* nv_scales, float* d_global_amax, float* d_s2, unsigned long long* d_counts,
                              uint32_t* d_flags, void* stream)
{
    nv4_cast_job j;
    j.mx_q = mx_q; j.e8m0 = e8m0; j.rows = rows; j.cols = cols; j.nv_q = nv_q; j.nv_scales = nv_scales;
    j.d_global_amax = d_global_amax; j.d_s2 = d_s2; j.group = -1;
    return nv4_mxfp4_to_nvfp4_batched(&j, 1, d_counts, d_flags, stream);
}

nv4_status nv4_selftest(uint32_t* d_out, void* stream)
{
    if (d_out == nullptr) return NV4_ERR_NULL;
    return from_cuda(launch_selftest(d_out, (cudaStream_t)stream));
}

nv4_status nv4_fp32_probe(int packed, uint32_t blocks, uint32_t iters, float* d_sink, void* stream)
{
    if (d_sink == nullptr) return NV4_ERR_NULL;
    if (blocks == 0 || blocks > (1u << 20) || iters == 0 || iters > (1u << 24)) return NV4_ERR_LIMIT;
    return from_cuda(launch_fma_probe(packed, blocks, iters, d_sink, (cudaStream_t)stream));
}

nv4_status nv4_selftest_wait(const uint32_t* d_flag, uint64_t limit_ns, uint32_t* d_status, void* stream)
{
    if (d_flag == nullptr || d_status == nullptr) return NV4_ERR_NULL;
    if (limit_ns > kWaitLimitNs) return NV4_ERR_LIMIT;
    return from_cuda(launch_wait_selftest(d_flag, limit_ns, d_status, (cudaStream_t)stream));
}

}  // extern "C"

// ------------------------------------------------------------------ W4A4 GEMM
size_t nv4_mma_scale_bytes(int64_t rows, int64_t cols)
{
    if (rows <= 0 || cols <= 0 || cols % 16 != 0) return 0;
    return mma_scale_bytes(rows, cols / 16);
}

nv4_status nv4_scales_to_mma_layout(const uint8_t* scales, int64_t rows, int64_t cols, uint8_t* out, void* stream)
{
    if (rows < 0 || cols < 0 || cols % 16 != 0) return NV4_ERR_SHAPE;
    if (rows == 0 || cols == 0) return NV4_OK;
    if (scales == nullptr || out == nullptr) return NV4_ERR_NULL;
    if (!aligned16(out)) return NV4_ERR_ALIGN;
    if (mma_scale_bytes(rows, cols / 16) >= ((size_t)1 << 34)) return NV4_ERR_LIMIT;
    return from_cuda(launch_mma_scale_layout(scales, rows, cols / 16, out, (cudaStream_t)stream));
}

nv4_status nv4_gemm_nvfp4(const uint8_t* qa, const uint8_t* sfa_mma, const float* d_s2a, const uint8_t* qb,
                          const uint8_t* sfb_mma, const float* d_s2b, int64_t M, int64_t N, int64_t K,
                          nv4_dtype out_dt, void* out, int64_t ldd, uint32_t* d_flags, void* stream)
{
    if (out_dt != NV4_BF16 && out_dt != NV4_FP32) return NV4_ERR_DTYPE;
    if (M < 0 || N < 0 || K < 0 || M % 128 != 0 || N % 128 != 0 || K % 256 != 0 || ldd < N) return NV4_ERR_SHAPE;
    if (M == 0 || N == 0) return NV4_OK;
    if (K == 0) return NV4_ERR_SHAPE;
    if (qa == nullptr || sfa_mma == nullptr || d_s2a == nullptr || qb == nullptr || sfb_mma == nullptr ||
        d_s2b == nullptr || out == nullptr)
        return NV4_ERR_NULL;
    if (!aligned16(qa) || !aligned16(qb) || !aligned16(sfa_mma) || !aligned16(sfb_mma) || !aligned16(out) ||
        ldd % (out_dt == NV4_FP32 ? 4 : 8) != 0)
        return NV4_ERR_ALIGN;
    if (M / 128 * (N / 128) >= ((int64_t)1 << 31) || K / 2 >= ((int64_t)1 << 32)) return NV4_ERR_LIMIT;
    return from_cuda(launch_gemm_nvfp4(qa, sfa_mma, d_s2a, qb, sfb_mma, d_s2b, M, N, K, (int)out_dt, out, ldd,
                                       d_flags, (cudaStream_t)stream));
}

// ------------------------------------------------------------------ format variants
nv4_status nv4_mxfp4_quant(const void* x, nv4_dtype dt, int64_t rows, int64_t cols, int64_t ld, uint8_t* q,
                           uint8_t* e8m0, uint32_t* d_flags, void* stream)
{
    if (dt != NV4_BF16 && dt != NV4_FP32) return NV4_ERR_DTYPE;
    if (rows < 0 || cols < 0 || cols % 32 != 0 || ld < cols) return NV4_ERR_SHAPE;
    if (rows == 0 || cols == 0) return NV4_OK;
    if (x == nullptr || q == nullptr || e8m0 == nullptr) return NV4_ERR_NULL;
    if (!aligned16(x) || !aligned16(q) || ld % (dt == NV4_BF16 ? 8 : 4) != 0) return NV4_ERR_ALIGN;
    if (rows * (cols / 16) >= (int64_t)1 << 31) return NV4_ERR_LIMIT;
    return from_cuda(launch_mxfp4_quant(x, dt == NV4_BF16 ? 0 : 2, rows, cols, ld, q, e8m0, d_flags,
                                        (cudaStream_t)stream));
}

nv4_status nv4_mxfp4_dequant(const uint8_t* q, const uint8_t* e8m0, int64_t rows, int64_t cols, nv4_dtype out_dt,
                             void* out, void* stream)
{
    if (out_dt != NV4_BF16 && out_dt != NV4_FP16 && out_dt != NV4_FP32) return NV4_ERR_DTYPE;
    if (rows < 0 || cols < 0 || cols % 32 != 0) return NV4_ERR_SHAPE;
    if (rows == 0 || cols == 0) return NV4_OK;
    if (q == nullptr || e8m0 == nullptr || out == nullptr) return NV4_ERR_NULL;
    if (!aligned16(q) || !aligned16(out)) return NV4_ERR_ALIGN;
    if (rows * (cols / 8) >= (int64_t)1 << 31) return NV4_ERR_LIMIT;
    return from_cuda(launch_mxfp4_dequant(q, e8m0, rows, cols, (int)out_dt, out, (cudaStream_t)stream));
}

nv4_status nv4_fp8_quant(const void* x, nv4_dtype dt, int64_t rows, int64_t cols, int64_t ld, const float* d_amax,
                         uint8_t* q, float* d_scale, uint32_t* d_flags, void* stream)
{
    if (dt != NV4_BF16 && dt != NV4_FP32) return NV4_ERR_DTYPE;
    if (rows < 0 || cols < 0 || cols % 16 != 0 || ld < cols) return NV4_ERR_SHAPE;
    if (d_amax == nullptr || d_scale == nullptr) return NV4_ERR_NULL;
    if (rows == 0 || cols == 0)                  // an empty tensor still receives its scale
        return from_cuda(launch_scale_only(&d_amax, &d_scale, 1, 448.0f, d_flags, (cudaStream_t)stream));
    if (x == nullptr || q == nullptr) return NV4_ERR_NULL;
    if (!aligned16(x) || !aligned16(q) || ld % (dt == NV4_BF16 ? 8 : 4) != 0) return NV4_ERR_ALIGN;
    if (rows * (cols / 16) >= (int64_t)1 << 31) return NV4_ERR_LIMIT;
    return from_cuda(launch_fp8_quant(x, dt == NV4_BF16 ? 0 : 2, rows, cols, ld, d_amax, q, d_scale, d_flags,
                                      (cudaStream_t)stream));
}

nv4_status nv4_fp8_dequant(const uint8_t* q, const float* d_scale, int64_t rows, int64_t cols, nv4_dtype out_dt,
                           void* out, void* stream)
{
    if (out_dt != NV4_BF16 && out_dt != NV4_FP16 && out_dt != NV4_FP32) return NV4_ERR_DTYPE;
    if (rows < 0 || cols < 0 || cols % 16 != 0) return NV4_ERR_SHAPE;
    if (rows == 0 || cols == 0) return NV4_OK;
    if (q == nullptr || d_scale == nullptr || out == nullptr) return NV4_ERR_NULL;
    if (!aligned16(q) || !aligned16(out)) return NV4_ERR_ALIGN;
    if (rows * (cols / 16) >= (int64_t)1 << 31) return NV4_ERR_LIMIT;
    return from_cuda(launch_fp8_dequant(q, d_scale, rows, cols, (int)out_dt, out, (cudaStream_t)stream));
}

// ------------------------------------------------------------------ block Hadamard + FP4
static nv4_status check_hadamard(const void* x, int64_t rows, int64_t cols, int64_t ld, int n)
{
    if (n != 16 && n != 32 && n != 64 && n != 128) return NV4_ERR_SHAPE;
    if (rows < 0 || cols < 0 || cols % 128 != 0 || ld < cols) return NV4_ERR_SHAPE;
    if (rows == 0 || cols == 0) return NV4_OK;
    if (x == nullptr) return NV4_ERR_NULL;
    if (!aligned16(x) || ld % 8 != 0) return NV4_ERR_ALIGN;
    if (rows * (cols / 32) >= (int64_t)1 << 31) return NV4_ERR_LIMIT;      // the kernel's 32-element chunk count
    return NV4_OK;
}

nv4_status nv4_hadamard_amax(const void* x, int64_t rows, int64_t cols, int64_t ld, int n, float* d_amax,
                             uint32_t* d_flags, void* stream)
{
    nv4_status st = check_hadamard(x, rows, cols, ld, n);
    if (st != NV4_OK) return st;
    if (d_amax == nullptr) return NV4_ERR_NULL;
    if (rows == 0 || cols == 0) return NV4_OK;
    return from_cuda(launch_hadamard_quant(0, x, rows, cols, ld, n, d_amax, nullptr, nullptr, nullptr, d_flags,
                                           (cudaStream_t)stream));
}

nv4_status nv4_hadamard_mxfp4_quant(const void* x, int64_t rows, int64_t cols, int64_t ld, int n, uint8_t* q,
                                    uint8_t* e8m0, uint32_t* d_flags, void* stream)
{
    nv4_status st = check_hadamard(x, rows, cols, ld, n);
    if (st != NV4_OK) return st;
    if (rows == 0 || cols == 0) return NV4_OK;
    if (q == nullptr || e8m0 == nullptr) return NV4_ERR_NULL;
    if (!aligned16(q)) return NV4_ERR_ALIGN;
    return from_cuda(launch_hadamard_quant(1, x, rows, cols, ld, n, nullptr, q, e8m0, nullptr, d_flags,
                                           (cudaStream_t)stream));
}

nv4_status nv4_hadamard_nvfp4_quant(const void* x, int64_t rows, int64_t cols, int64_t ld, int n,
                                    const float* d_amax, uint8_t* q, uint8_t* scales, float* d_s2, uint32_t* d_flags,
                                    void* stream)
{
    nv4_status st = check_hadamard(x, rows, cols, ld, n);
    if (st != NV4_OK) return st;
    if (d_amax == nullptr || d_s2 == nullptr) return NV4_ERR_NULL;
    if (rows == 0 || cols == 0)                  // an empty tensor still receives its s2
        return from_cuda(launch_scale_only(&d_amax, &d_s2, 1, 2688.0f, d_flags, (cudaStream_t)stream));
    if (q == nullptr || scales == nullptr) return NV4_ERR_NULL;
    if (!aligned16(q)) return NV4_ERR_ALIGN;
    return from_cuda(launch_hadamard_quant(2, x, rows, cols, ld, n, const_cast<float*>(d_amax), q, scales, d_s2,
                                           d_flags, (cudaStream_t)stream));
}

// ------------------------------------------------------------------ two-sided block Hadamard of weight tiles
static nv4_status check_hadamard2(const void* w, nv4_dtype dt, int64_t rows, int64_t cols, int64_t ld, int n)
{
    if (dt != NV4_BF16 && dt != NV4_FP32) return NV4_ERR_DTYPE;
    if (n != 16 && n != 32) return NV4_ERR_SHAPE;
    if (rows < 0 || cols < 0 || rows % n != 0 || cols % 32 != 0 || ld < cols) return NV4_ERR_SHAPE;
    if (rows == 0 || cols == 0) return NV4_OK;
    if (w == nullptr) return NV4_ERR_NULL;
    if (!aligned16(w) || ld % (dt == NV4_BF16 ? 8 : 4) != 0) return NV4_ERR_ALIGN;
    if ((rows / n) * (cols / 32) >= (int64_t)1 << 31) return NV4_ERR_LIMIT;
    return NV4_OK;
}

nv4_status nv4_hadamard2_rotate(const void* w, nv4_dtype dt, int64_t rows, int64_t cols, int64_t ld, int n,
                                float* out, uint32_t* d_flags, void* stream)
{
    const nv4_status st = check_hadamard2(w, dt, rows, cols, ld, n);
    if (st != NV4_OK || rows == 0 || cols == 0) return st;
    if (out == nullptr) return NV4_ERR_NULL;
    if (!aligned16(out)) return NV4_ERR_ALIGN;
    return from_cuda(launch_hadamard2(3, w, dt == NV4_BF16 ? 0 : 2, rows, cols, ld, n, nullptr, nullptr, nullptr,
                                      nullptr, out, d_flags, (cudaStream_t)stream));
}

nv4_status nv4_hadamard2_amax(const void* w, nv4_dtype dt, int64_t rows, int64_t cols, int64_t ld, int n,
                              float* d_amax, uint32_t* d_flags, void* stream)
{
    const nv4_status st = check_hadamard2(w, dt, rows, cols, ld, n);
    if (st != NV4_OK) return st;
    if (d_amax == nullptr) return NV4_ERR_NULL;
    if (rows == 0 || cols == 0) return NV4_OK;
    return from_cuda(launch_hadamard2(0, w, dt == NV4_BF16 ? 0 : 2, rows, cols, ld, n, d_amax, nullptr, nullptr,
                                      nullptr, nullptr, d_flags, (cudaStream_t)stream));
}

nv4_status nv4_hadamard2_mxfp4_quant(const void* w, nv4_dtype dt, int64_t rows, int64_t cols, int64_t ld, int n,
                                     uint8_t* q, uint8_t* e8m0, uint32_t* d_flags, void* stream)
{
    const nv4_status st = check_hadamard2(w, dt, rows, cols, ld, n);
    if (st != NV4_OK || rows == 0 || cols == 0) return st;
    if (q == nullptr || e8m0 == nullptr) return NV4_ERR_NULL;
    if (!aligned16(q)) return NV4_ERR_ALIGN;
    return from_cuda(launch_hadamard2(1, w, dt == NV4_BF16 ? 0 : 2, rows, cols, ld, n, nullptr, q, e8m0, nullptr,
                                      nullptr, d_flags, (cudaStream_t)stream));
}

nv4_status nv4_hadamard2_nvfp4_quant(const void* w, nv4_dtype dt, int64_t rows, int64_t cols, int64_t ld, int n,
                                     const float* d_amax, uint8_t* q, uint8_t* scales, float* d_s2,
                                     uint32_t* d_flags, void* stream)
{
    const nv4_status st = check_hadamard2(w, dt, rows, cols, ld, n);
    if (st != NV4_OK) return st;
    if (d_amax == nullptr || d_s2 == nullptr) return NV4_ERR_NULL;
    if (rows == 0 || cols == 0)                  // an empty tensor still receives its s2
        return from_cuda(launch_scale_only(&d_amax, &d_s2, 1, 2688.0f, d_flags, (cudaStream_t)stream));
    if (q == nullptr || scales == nullptr) return NV4_ERR_NULL;
    if (!aligned16(q)) return NV4_ERR_ALIGN;
    return from_cuda(launch_hadamard2(2, w, dt == NV4_BF16 ? 0 : 2, rows, cols, ld, n, const_cast<float*>(d_amax),
                                      q, scales, d_s2, nullptr, d_flags, (cudaStream_t)stream));
}
