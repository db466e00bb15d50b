// hadamard.cu -- block Hadamard rotation fused with FP4 quantization (sm_100a).
//
// [FP4] section 3.1 (blocks rotated by H / sqrt(n) before quantization, spreading
// outliers) and section 4.1 (quantization-transform kernels with block sizes 16, 32, 64
// and 128).  y = RN32(RN64(x_block H_n) * RN64(1/sqrt(n))) along each row, then:
//   mode 0: running max |y| into *d_amax (the per-tensor amax that NVFP4 needs);
//   mode 1: MXFP4 quantization of y (32-element blocks, E8M0 scales);
//   mode 2: NVFP4 quantization of y with s2 = RN32(amax / 2688).
//
// Mapping: a lane owns 32 consecutive elements of a row (four 16-byte loads); four lanes
// cover a 128-element segment.  The fast Walsh-Hadamard transform runs in FP64: up to
// five butterfly stages inside a lane, then log2(n / 32) stages across lanes with
// shuffles (n = 64, 128), so every sum is exact for BF16 inputs spanning fewer than ~38
// binades in a block.  n is a template parameter: with static stage counts the kernel
// needs 104 registers instead of 160 (4 CTAs per SM instead of 3), 0.63 ms instead of
// 0.70 ms for n = 128 on a [65536, 7168] BF16 input and 0.37 ms instead of 0.49 ms for
// n = 32.  The quantizers then work on FP32 y exactly as nv4_mxfp4_quant /
// nv4_act_quant do; an MXFP4 block is one lane's 32 values, an NVFP4 block half of them.
#include <cmath>

#include "nv4_common.cuh"
#include "nv4_internal.h"

namespace nv4 {

constexpr int kHadThreads = 128;

// FWHT of blocks of n values, 32 consecutive values per lane: five butterfly stages
// inside the lane, then log2(n / 32) stages across neighbouring lanes (n = 64, 128).
template <int kN>
__device__ __forceinline__ void fwht32(double v[32], uint32_t lane)
{
    constexpr int n = kN;
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
        if (h >= n) break;                            // blocks of 16: only four in-lane stages
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (i & h) continue;
            const double a = v[i], b = v[i + h];
            v[i] = a + b;
            v[i + h] = a - b;
        }
    }
#pragma unroll
    for (int d = 1; d < n / 32; d <<= 1) {
        const bool upper = (lane & (uint32_t)d) != 0u;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
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

template <int kMode, int kN>
__global__ void __launch_bounds__(kHadThreads)
hadamard_quant_kernel(const uint16_t* x, uint32_t rows, uint32_t chunks_per_row, int64_t ld, FastDiv div_cpr,
                      double c, float* __restrict__ d_amax, uint8_t* __restrict__ q, uint8_t* __restrict__ sc,
                      float* __restrict__ d_s2, uint32_t* __restrict__ d_flags)
{
    // one lane = one 32-element chunk of a row (4 lanes = one 128-element segment)
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t total = rows * chunks_per_row;                 // multiple of 4
    const uint32_t stride = gridDim.x * kHadThreads;
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
    const int64_t cols = (int64_t)chunks_per_row * 32;

    // warp-uniform trip count (lanes of one 128-element segment exchange values); the
    // next chunk's four loads are issued before the current chunk is transformed
    auto load = [&](uint32_t ch, uint4 raw[4]) {
        const uint32_t rr = div_cpr.div(ch), c2 = ch - rr * chunks_per_row;
        const uint4* src = reinterpret_cast<const uint4*>(x + (int64_t)rr * ld + 32 * (int64_t)c2);
#pragma unroll
        for (int k = 0; k < 4; ++k) raw[k] = __ldcs(src + k);
    };
    uint4 nxt[4];
    {
        const uint32_t ch0 = blockIdx.x * kHadThreads + (threadIdx.x & ~31u) + lane;
        if (ch0 < total) load(ch0, nxt);
    }
    for (uint32_t c0 = blockIdx.x * kHadThreads + (threadIdx.x & ~31u); c0 < total; c0 += stride) {
        const uint32_t ch = c0 + lane;
        const bool live = ch < total;                              // segments are all-live or all-dead
        uint32_t r = 0u, cc = 0u;
        double v[32];
        if (live) {
            r = div_cpr.div(ch);
            cc = ch - r * chunks_per_row;
            uint4 raw[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) raw[k] = nxt[k];
            if (ch + stride < total) load(ch + stride, nxt);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t wv[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    v[8 * k + 2 * j] = (double)bf16_lo(wv[j]);
                    v[8 * k + 2 * j + 1] = (double)bf16_hi(wv[j]);
                }
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = 0.0;
        }
        fwht32<kN>(v, lane);
        if (!live) continue;

        float y[32];
        uint32_t ab = 0u;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            y[j] = (float)(v[j] * c);                              // RN32(RN64(z * c))
            ab = max(ab, __float_as_uint(y[j]) & 0x7FFFFFFFu);
        }
        if (ab >= 0x7F800000u) flags |= kFlagNonFinite;
        const int64_t col = 32 * (int64_t)cc;

        if constexpr (kMode == 0) {
            if (ab <= 0x7F800000u) mx_bits = max(mx_bits, ab);
        } else if constexpr (kMode == 1) {
            uint32_t code, w[4] = {0u, 0u, 0u, 0u};
            if (ab >= 0x7F800000u) {
                code = 0xFFu;
            } else {
                const int e = ab == 0u ? -127 : max(had_floor_log2(ab) - 2, -127);
                code = (uint32_t)(e + 127);
                const float inv = had_pow2(-e);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float t[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) t[j] = __fmul_rn(y[8 * k + j], inv);   // exact
                    w[k] = cvt_e2m1x8(t);
                }
            }
            __stcs(reinterpret_cast<uint4*>(q + (int64_t)r * (cols / 2) + col / 2), make_uint4(w[0], w[1], w[2], w[3]));
            sc[(int64_t)r * (cols / 32) + col / 32] = (uint8_t)code;
        } else {
            uint32_t w[4], codes2 = 0u;
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {                       // two NVFP4 blocks of 16
                uint32_t bm = 0u;
#pragma unroll
                for (int j = 0; j < 16; ++j) bm = max(bm, __float_as_uint(y[16 * hb + j]) & 0x7FFFFFFFu);
                const float a_b = __uint_as_float(bm);
                uint32_t code;
                if (fast_scale) {
                    const uint32_t cv = cvt_e4m3x2(__fmul_rn(a_b, k_lo), __fmul_rn(a_b, k_hi));
                    code = cv & 0xFFu;
                    if (code != (cv >> 8)) code = e4m3_fix(code, a_b, s2);
                } else {
                    code = e4m3_code_exact(a_b, s2);
                }
                code &= 0x7Fu;
                codes2 |= code << (8 * hb);
                const float S = __fmul_rn(e4m3_value(code), s2);   // DQ1: RN32(s_b * s2)
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const float* yy = y + 16 * hb + 8 * k;
                    uint32_t c8 = 0u;
                    if (S == 0.0f) {
#pragma unroll
                        for (int j = 0; j < 8; ++j) c8 |= ((__float_as_uint(yy[j]) >> 28) & 8u) << (4 * j);
                    } else if (S >= kTinyScale && S <= 0x1p100f) {
                        const float rr = __frcp_rn(S);
                        const float rl = __fmul_rn(rr, kLoMargin), rh = __fmul_rn(rr, kHiMargin);
                        float lo[8], hi[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            lo[j] = __fmul_rn(yy[j], rl);
                            hi[j] = __fmul_rn(yy[j], rh);
                        }
                        c8 = cvt_e2m1x8(lo);
                        const uint32_t h8 = cvt_e2m1x8(hi);
                        if (c8 != h8) c8 = e2m1_fix8(yy, S, c8, h8);
                    } else {
#pragma unroll
                        for (int j = 0; j < 8; ++j) c8 |= e2m1_code_exact(yy[j], S) << (4 * j);
                    }
                    w[2 * hb + k] = c8;
                }
            }
            __stcs(reinterpret_cast<uint4*>(q + (int64_t)r * (cols / 2) + col / 2), make_uint4(w[0], w[1], w[2], w[3]));
            *reinterpret_cast<uint16_t*>(sc + (int64_t)r * (cols / 16) + col / 16) = (uint16_t)codes2;
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
    const uint32_t spr = (uint32_t)(cols / 32);                  // 32-element chunks per row
    const int64_t chunks = rows * (int64_t)spr;
    const int64_t need = (chunks + kHadThreads - 1) / kHadThreads;
    const int64_t cap = (int64_t)num_sms() * 8;
    const int grid = (int)(need < cap ? (need > 0 ? need : 1) : cap);
    const double c = 1.0 / std::sqrt((double)n);
    const uint16_t* xx = static_cast<const uint16_t*>(x);
#define NV4_HAD(M, N) hadamard_quant_kernel<M, N><<<grid, kHadThreads, 0, s>>>(xx, (uint32_t)rows, spr, ld, FastDiv(spr), \
                                                                         c, d_amax, q, sc, d_s2, d_flags)
#define NV4_HAD_N(M) do { if (n == 16) NV4_HAD(M, 16); else if (n == 32) NV4_HAD(M, 32); \
                          else if (n == 64) NV4_HAD(M, 64); else NV4_HAD(M, 128); } while (0)
    if (mode == 0) NV4_HAD_N(0);
    else if (mode == 1) NV4_HAD_N(1);
    else NV4_HAD_N(2);
#undef NV4_HAD_N
#undef NV4_HAD
    return cudaGetLastError();
}

}  // namespace nv4
