// nv4_internal.h -- declarations shared by the kernel files and the C-ABI layer.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "nv4.h"

namespace nv4 {

// Division of 32-bit unsigned integers by a fixed divisor d >= 1 with one
// multiply-high, one add and one shift (T. Granlund and P. L. Montgomery,
// "Division by invariant integers using multiplication", PLDI 1994, round-up
// method): with s = ceil(log2 d) and m = floor(2^32 (2^s - d) / d) + 1,
// n / d = (mulhi(n, m) + n) >> s for every n < 2^32.
struct FastDiv {
    uint32_t d = 1, m = 1, s = 0;
    __host__ __device__ FastDiv() {}
    __host__ __device__ explicit FastDiv(uint32_t div) : d(div)
    {
        s = 0;
        while ((1ull << s) < div) ++s;
        m = (uint32_t)((((1ull << 32) * ((1ull << s) - div)) / div) + 1ull);
    }
    __device__ __forceinline__ uint32_t div(uint32_t n) const
    {
        return (uint32_t)(((uint64_t)__umulhi(n, m) + n) >> s);
    }
};

int num_sms();

constexpr int kMaxHessianJobs = 128;
constexpr int kMaxSweepJobs = 192;
constexpr int kMaxCastJobs = 128;

// One tensor of a (batched) per-tensor amax, block quantization or dequantization call.
struct AmaxTask {
    const void* x;
    int64_t n;
    float* d_amax;
};
struct QuantTask {
    const void* x;
    int64_t rows, cols, ld;
    const float* d_amax;
    uint8_t* q;           // packed codes (code output) or null
    uint8_t* scales;
    void* out;            // fake quantize-dequantize output or null
    int64_t ld_out;
    float* d_s2;
};
struct DequantTask {
    const uint8_t* q;
    const uint8_t* scales;
    const float* d_s2;
    int64_t rows, cols;
    void* out;
};
constexpr int kMaxActJobs = 128;

cudaError_t launch_amax(const AmaxTask* tasks, int n, int dt, uint32_t* d_flags, cudaStream_t s);
// Second-level scales of empty tensors: d_out[i] = RN32(*d_amax[i] / divisor) for n pairs,
// NV4_FLAG_OVERFLOW where that is not finite (one small launch; nothing else is read).
cudaError_t launch_scale_only(const float* const* d_amax, float* const* d_out, int n, float divisor,
                              uint32_t* d_flags, cudaStream_t s);
cudaError_t launch_block_quant(const QuantTask* tasks, int n, int in_dt, int out_dt, uint32_t* d_flags,
                               cudaStream_t s);
cudaError_t launch_mxfp4_quant(const void* x, int in_dt, int64_t rows, int64_t cols, int64_t ld, uint8_t* q,
                               uint8_t* e8m0, uint32_t* d_flags, cudaStream_t s);
cudaError_t launch_mxfp4_dequant(const uint8_t* q, const uint8_t* e8m0, int64_t rows, int64_t cols, int out_dt,
                                 void* out, cudaStream_t s);
cudaError_t launch_fp8_quant(const void* x, int in_dt, int64_t rows, int64_t cols, int64_t ld, const float* d_amax,
                             uint8_t* q, float* d_scale, uint32_t* d_flags, cudaStream_t s);
cudaError_t launch_fp8_dequant(const uint8_t* q, const float* d_scale, int64_t rows, int64_t cols, int out_dt,
                               void* out, cudaStream_t s);
cudaError_t launch_hadamard2(int mode, const void* w, int dt, int64_t rows, int64_t cols, int64_t ld, int n,
                             float* d_amax, uint8_t* q, uint8_t* sc, float* d_s2, float* out, uint32_t* d_flags,
                             cudaStream_t s);
cudaError_t launch_hadamard_quant(int mode, const void* x, int64_t rows, int64_t cols, int64_t ld, int n,
                                  float* d_amax, uint8_t* q, uint8_t* sc, float* d_s2, uint32_t* d_flags,
                                  cudaStream_t s);
cudaError_t launch_wait_selftest(const uint32_t* flag, uint64_t limit_ns, uint32_t* status, cudaStream_t s);
size_t mma_scale_bytes(int64_t rows, int64_t kb);
cudaError_t launch_mma_scale_layout(const uint8_t* sc, int64_t rows, int64_t kb, uint8_t* out, cudaStream_t s);
cudaError_t launch_gemm_nvfp4(const uint8_t* qa, const uint8_t* sfa, const float* d_s2a, const uint8_t* qb,
                              const uint8_t* sfb, const float* d_s2b, int64_t M, int64_t N, int64_t K, int out_dt,
                              void* out, int64_t ldd, uint32_t* d_flags, cudaStream_t s);
cudaError_t launch_dequant(const DequantTask* tasks, int n, int out_dt, cudaStream_t s);
cudaError_t launch_hessian(const nv4_hessian_job* jobs, int n, uint32_t* d_flags, cudaStream_t s, int* bad_job);
cudaError_t launch_sweep(const nv4_sweep_job* jobs, int n, int dt, uint32_t* d_flags, cudaStream_t s);
cudaError_t launch_cast(const nv4_cast_job* jobs, int n, unsigned long long* d_counts, uint32_t* d_flags,
                        cudaStream_t s);
cudaError_t launch_selftest(uint32_t* d_out, cudaStream_t s);
cudaError_t launch_fma_probe(int packed, uint32_t blocks, uint32_t iters, float* sink, cudaStream_t s);

}  // namespace nv4
