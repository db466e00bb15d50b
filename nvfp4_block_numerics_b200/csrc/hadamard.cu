// hadamard.cu -- block Hadamard rotation fused with FP4 quantization (sm_100a).
//
// [FP4] section 3.1 (blocks rotated by H / sqrt(n) before quantization, spreading
// outliers) and section 4.1 (quantization-transform kernels with block sizes 16, 32, 64
// and 128).  y = RN32(RN64(x_block H_n) * RN64(1/sqrt(n))) along each row, then:
//   mode 0: running max |y| into *d_amax (the per-tensor amax that NVFP4 needs);
//   mode 1: MXFP4 quantization of y (32-element blocks, E8M0 scales);
//   mode 2: NVFP4 quantization of y with s2 = RN32(amax / 2688).
//
// Mapping: a half-warp owns a 128-element row segment, 8 consecutive elements per lane
// (one 16-byte load).  The fast Walsh-Hadamard transform runs in FP64: three butterfly
// stages inside a lane, then log2(n / 8) stages across lanes with shuffles, so every
// sum is exact for BF16 inputs spanning fewer than ~38 binades in a block.  The
// quantizers then work on FP32 y exactly as nv4_mxfp4_quant / nv4_act_quant do: MXFP4
// blocks are 4 lanes (maxima combined with two shuffles), NVFP4 blocks 2 lanes.
#include <cmath>

#include "nv4_common.cuh"
#include "nv4_internal.h"

namespace nv4 {

constexpr int kHadThreads = 256;

// FWHT of 128 / n independent blocks of n values spread over a half-warp, 8 per lane.
__device__ __forceinline__ void fwht(double v[8], int n, uint32_t lane)
{
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {                 // in-lane stages (bits 0..2 of the index)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i & h) continue;
            const double a = v[i], b = v[i + h];
            v[i] = a + b;
            v[i + h] = a - b;
        }
    }
    for (int d = 1; d < n / 8; d <<= 1) {             // across lanes (bits 3.. of the index)
        const bool upper = (lane & (uint32_t)d) != 0u;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const double o = __shfl_xor_sync(0xFFFFFFFFu, v[i], d);
            v[i] = upper ? o - v[i] : v[i] + o;
        }
    }
}

// floor(log2(a)) for a finite positive FP32 bit pattern.
__device__ __forceinline__ int had_floor_log2(uint32_t b)
{
    const int e = (int)(b >> 23);
    return e != 0 ? e - 127 : -149 + (31 - __clz(b));
}

__device__ __forceinline__ float had_pow2(int k)
{
    return k >= -126 ? __uint_as_float((uint32_t)(k + 127) << 23) : __uint_as_float(1u << (k + 149));
}

template <int kMode>
__global__ void __launch_bounds__(kHadThreads)
hadamard_quant_kernel(const uint16_t* x, uint32_t rows, uint32_t segs_per_row, int64_t ld, FastDiv div_spr, int n,
                      double c, float* __restrict__ d_amax, uint8_t* __restrict__ q, uint8_t* __restrict__ sc,
                      float* __restrict__ d_s2, uint32_t* __restrict__ d_flags)
{
    const uint32_t lane = threadIdx.x & 31u, sub = lane & 15u, half = lane >> 4;
    const uint32_t total = rows * segs_per_row;
    const uint32_t warps = gridDim.x * (kHadThreads / 32);
    uint32_t flags = 0u, mx_bits = 0u;

    float s2 = 0.0f, k_lo = 0.0f, k_hi = 0.0f;
    bool fast_scale = false;
    if constexpr (kMode == 2) {
        s2 = __fdiv_rn(*d_amax, 2688.0f);
        if (blockIdx.x == 0 && threadIdx.x == 0) *d_s2 = s2;
        fast_scale = s2 >= kTinyScale && s2 <= 0x1p100f;
        const float k = __frcp_rn(__fmul_rn(6.0f, s2));
        k_lo = __fmul_rn(k, kLoMargin);
        k_hi = __fmul_rn(k, kHiMargin);
        if (!isfinite(s2)) flags |= kFlagOverflow;
    }

    for (uint32_t w = blockIdx.x * (kHadThreads / 32) + (threadIdx.x >> 5); 2u * w < total; w += warps) {
        const uint32_t seg = 2u * w + half;
        const bool live = seg < total;
        uint32_t r = 0u, s = 0u;
        double v[8];
        if (live) {
            r = div_spr.div(seg);
            s = seg - r * segs_per_row;
            const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(x + (int64_t)r * ld + 128 * (int64_t)s + 8 * sub));
            const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                v[2 * j] = (double)bf16_lo(wv[j]);
                v[2 * j + 1] = (double)bf16_hi(wv[j]);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = 0.0;
        }
        fwht(v, n, lane);
        float y[8];
        uint32_t ab = 0u;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            y[j] = (float)(v[j] * c);                    // RN32(RN64(z * c))
            ab = max(ab, __float_as_uint(y[j]) & 0x7FFFFFFFu);
        }
        if (ab >= 0x7F800000u && live) flags |= kFlagNonFinite;

        if constexpr (kMode == 0) {
            if (live && ab <= 0x7F800000u) mx_bits = max(mx_bits, ab);
        } else if constexpr (kMode == 1) {
            // MXFP4 block = 4 lanes (32 elements)
            uint32_t bm = max(ab, __shfl_xor_sync(0xFFFFFFFFu, ab, 1));
            bm = max(bm, __shfl_xor_sync(0xFFFFFFFFu, bm, 2));
            if (live) {
                uint32_t code, c0 = 0u;
                if (bm >= 0x7F800000u) {
                    code = 0xFFu;
                } else {
                    const int e = bm == 0u ? -127 : max(had_floor_log2(bm) - 2, -127);
                    code = (uint32_t)(e + 127);
                    const float inv = had_pow2(-e);
                    float t[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) t[j] = __fmul_rn(y[j], inv);   // exact
                    c0 = cvt_e2m1x8(t);
                }
                const int64_t col = 128 * (int64_t)s + 8 * sub;              // first element of this lane
                const int64_t cols = (int64_t)segs_per_row * 128;
                *reinterpret_cast<uint32_t*>(q + (int64_t)r * (cols / 2) + col / 2) = c0;
                if ((sub & 3u) == 0u) sc[(int64_t)r * (cols / 32) + col / 32] = (uint8_t)code;
            }
        } else {
            // NVFP4 block = 2 lanes (16 elements)
            const uint32_t bm = max(ab, __shfl_xor_sync(0xFFFFFFFFu, ab, 1));
            if (live) {
                const float a_b = __uint_as_float(bm);
                uint32_t code;
                if (fast_scale) {
                    const uint32_t cc = cvt_e4m3x2(__fmul_rn(a_b, k_lo), __fmul_rn(a_b, k_hi));
                    code = cc & 0xFFu;
                    if (code != (cc >> 8)) code = e4m3_fix(code, a_b, s2);
                } else {
                    code = e4m3_code_exact(a_b, s2);
                }
                code &= 0x7Fu;
                const float S = __fmul_rn(e4m3_value(code), s2);           // DQ1: RN32(s_b * s2)
                uint32_t c0 = 0u;
                if (S == 0.0f) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) c0 |= ((__float_as_uint(y[j]) >> 28) & 8u) << (4 * j);
                } else if (S >= kTinyScale && S <= 0x1p100f) {
                    const float rr = __frcp_rn(S);
                    const float rl = __fmul_rn(rr, kLoMargin), rh = __fmul_rn(rr, kHiMargin);
                    float lo[8], hi[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        lo[j] = __fmul_rn(y[j], rl);
                        hi[j] = __fmul_rn(y[j], rh);
                    }
                    c0 = cvt_e2m1x8(lo);
                    const uint32_t h0 = cvt_e2m1x8(hi);
                    if (c0 != h0) c0 = e2m1_fix8(y, S, c0, h0);
                } else {
#pragma unroll 1
                    for (int j = 0; j < 8; ++j) c0 |= e2m1_code_exact(y[j], S) << (4 * j);
                }
                const int64_t col = 128 * (int64_t)s + 8 * sub;
                const int64_t cols = (int64_t)segs_per_row * 128;
                *reinterpret_cast<uint32_t*>(q + (int64_t)r * (cols / 2) + col / 2) = c0;
                if ((sub & 1u) == 0u) sc[(int64_t)r * (cols / 16) + col / 16] = (uint8_t)code;
            }
        }
    }
    if constexpr (kMode == 0) {
        mx_bits = __reduce_max_sync(0xFFFFFFFFu, mx_bits);
        if (lane == 0 && mx_bits != 0u) atomicMax(reinterpret_cast<unsigned int*>(d_amax), mx_bits);
    }
    flags = __reduce_or_sync(0xFFFFFFFFu, flags);
    if (lane == 0) flag_or(d_flags, flags);
}

cudaError_t launch_hadamard_quant(int mode, const void* x, int64_t rows, int64_t cols, int64_t ld, int n,
                                  float* d_amax, uint8_t* q, uint8_t* sc, float* d_s2, uint32_t* d_flags,
                                  cudaStream_t s)
{
    const uint32_t spr = (uint32_t)(cols / 128);
    const int64_t segs = rows * (int64_t)spr;
    const int64_t warps_needed = (segs + 1) / 2;
    const int64_t need = (warps_needed + kHadThreads / 32 - 1) / (kHadThreads / 32);
    const int64_t cap = (int64_t)num_sms() * 8;
    const int grid = (int)(need < cap ? (need > 0 ? need : 1) : cap);
    const double c = 1.0 / std::sqrt((double)n);
    const uint16_t* xx = static_cast<const uint16_t*>(x);
    if (mode == 0)
        hadamard_quant_kernel<0><<<grid, kHadThreads, 0, s>>>(xx, (uint32_t)rows, spr, ld, FastDiv(spr), n, c, d_amax,
                                                              q, sc, d_s2, d_flags);
    else if (mode == 1)
        hadamard_quant_kernel<1><<<grid, kHadThreads, 0, s>>>(xx, (uint32_t)rows, spr, ld, FastDiv(spr), n, c, d_amax,
                                                              q, sc, d_s2, d_flags);
    else
        hadamard_quant_kernel<2><<<grid, kHadThreads, 0, s>>>(xx, (uint32_t)rows, spr, ld, FastDiv(spr), n, c, d_amax,
                                                              q, sc, d_s2, d_flags);
    return cudaGetLastError();
}

}  // namespace nv4
