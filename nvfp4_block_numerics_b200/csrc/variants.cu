// variants.cu -- format variants of the block quantizer (sm_100a): MXFP4 (32-element
// blocks, E8M0 power-of-two scale) and FP8 E4M3 with one static per-tensor scale.
//
// MXFP4 ([FP4] sections 1.2, 3.2): shared exponent e = floor(log2 amax) - 2, clamped to
// [-127, 127]; elements = E2M1 nearest to x / 2^e.  Dividing by a power of two is exact
// in FP32 here (|x| / 2^e < 8 and 2^-e is a normal number for every finite amax), so one
// hardware round-to-nearest-even conversion gives the exact code: no bracket is needed.
// One thread handles half a block (16 elements); the two lanes of a block exchange their
// maxima with one shuffle.
//
// FP8 ([CAL] layer table, W8A8 with static per-tensor scales): s = RN32(amax / 448),
// code = sign | E4M3 nearest to |x| / s.  The quotient is bracketed between two FP32
// products by 1/s with a 2^-20 margin and both ends converted with the hardware's RNE
// E4M3 conversion; when they differ, one exact FMA comparison with the midpoint decides.
#include <cuda_fp16.h>

#include "nv4_common.cuh"
#include "nv4_internal.h"

namespace nv4 {

constexpr int kVarThreads = 256;

template <int kIn>
__device__ __forceinline__ void load16(const void* x, int64_t off, float v[16], uint32_t& amax_bits)
{
    amax_bits = 0u;
    if constexpr (kIn == 0) {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + off);
        const uint4 a = __ldcs(src), b = __ldcs(src + 1);
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t m = 0u;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            m = __vmaxu2(m, w[j] & 0x7FFF7FFFu);
            v[2 * j] = bf16_lo(w[j]);
            v[2 * j + 1] = bf16_hi(w[j]);
        }
        amax_bits = max(m & 0xFFFFu, m >> 16) << 16;
    } else {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const float*>(x) + off);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint4 t = __ldcs(src + k);
            const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                amax_bits = max(amax_bits, w[j] & 0x7FFFFFFFu);
                v[4 * k + j] = __uint_as_float(w[j]);
            }
        }
    }
}

// floor(log2(a)) for a finite positive FP32 bit pattern (normal or subnormal).
__device__ __forceinline__ int floor_log2_bits(uint32_t b)
{
    const int e = (int)(b >> 23);
    return e != 0 ? e - 127 : -149 + (31 - __clz(b));
}

// 2^k as FP32 for k in [-149, 127] (exact).
__device__ __forceinline__ float pow2f(int k)
{
    return k >= -126 ? __uint_as_float((uint32_t)(k + 127) << 23) : __uint_as_float(1u << (k + 149));
}

// ------------------------------------------------------------------ MXFP4
template <int kIn>
__global__ void __launch_bounds__(kVarThreads)
mxfp4_quant_kernel(const void* x, uint32_t rows, uint32_t halves_per_row, int64_t ld, FastDiv div_hpr,
                   uint8_t* __restrict__ q, uint8_t* __restrict__ e8m0, uint32_t* __restrict__ d_flags)
{
    const uint32_t total = rows * halves_per_row;                 // even: two halves per block
    const uint32_t stride = gridDim.x * kVarThreads;
    const uint32_t lane = threadIdx.x & 31u;
    uint32_t flags = 0u;
    // warp-uniform trip count, so the pair shuffle always has both lanes present
    for (uint32_t h0 = blockIdx.x * kVarThreads + (threadIdx.x & ~31u); h0 < total; h0 += stride) {
        const uint32_t h = h0 + lane;
        const bool live = h < total;                               // partners are both live or both not
        float v[16];
        uint32_t ab = 0u;
        if (live) {
            const uint32_t r = div_hpr.div(h), hh = h - r * halves_per_row;
            load16<kIn>(x, (int64_t)r * ld + 16 * (int64_t)hh, v, ab);
        }
        ab = max(ab, __shfl_xor_sync(0xFFFFFFFFu, ab, 1));         // the partner half of the block
        if (!live) continue;
        uint32_t code, c0 = 0u, c1 = 0u;
        if (ab >= 0x7F800000u) {                                   // NaN or Inf in the block
            flags |= kFlagNonFinite;
            code = 0xFFu;
        } else {
            const int e = ab == 0u ? -127 : max(floor_log2_bits(ab) - 2, -127);
            code = (uint32_t)(e + 127);
            const float inv = pow2f(-e);                           // normal: -e in [-125, 127]
            float y[16];
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
                const float2 t = __fmul2_rn(make_float2(v[i], v[i + 1]), make_float2(inv, inv));
                y[i] = t.x;
                y[i + 1] = t.y;
            }
            c0 = cvt_e2m1x8(y);
            c1 = cvt_e2m1x8(y + 8);
        }
        *reinterpret_cast<uint2*>(q + (int64_t)h * 8) = make_uint2(c0, c1);
        if ((h & 1u) == 0u) e8m0[h >> 1] = (uint8_t)code;
    }
    flags = __reduce_or_sync(__activemask(), flags);
    if ((threadIdx.x & 31) == 0) flag_or(d_flags, flags);
}

// One thread per 8 outputs: 4 code bytes, the block's E8M0 byte, 8 outputs.
template <int kOut>
__global__ void __launch_bounds__(kVarThreads)
mxfp4_dequant_kernel(const uint8_t* __restrict__ q, const uint8_t* __restrict__ e8m0, uint32_t total8, void* out)
{
    const uint32_t* qw = reinterpret_cast<const uint32_t*>(q);
    for (uint32_t h = blockIdx.x * kVarThreads + threadIdx.x; h < total8; h += gridDim.x * kVarThreads) {
        const uint32_t c = e8m0[h >> 2];
        const float S = c == 0xFFu ? __uint_as_float(0x7FC00000u) : pow2f((int)c - 127);
        uint32_t hv[4];
        cvt_e2m1x8_to_f16x8(__ldcs(qw + h), hv);
        float y[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float a, b;
            f16x2_to_f32(hv[j], a, b);
            y[2 * j] = __fmul_rn(a, S);
            y[2 * j + 1] = __fmul_rn(b, S);
        }
        if constexpr (kOut == 2) {
            float4* o = reinterpret_cast<float4*>(out) + 2 * (int64_t)h;
            __stcs(o, make_float4(y[0], y[1], y[2], y[3]));
            __stcs(o + 1, make_float4(y[4], y[5], y[6], y[7]));
        } else {
            uint32_t p[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if constexpr (kOut == 0)
                    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(p[j]) : "f"(y[2 * j + 1]), "f"(y[2 * j]));
                else
                    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(p[j]) : "f"(y[2 * j + 1]), "f"(y[2 * j]));
            }
            __stcs(reinterpret_cast<uint4*>(out) + h, make_uint4(p[0], p[1], p[2], p[3]));
        }
    }
}

// ------------------------------------------------------------------ FP8 E4M3, static per-tensor scale
// Nearest E4M3 code (0..126) to a / s, a >= 0, s > 0, ties to the even code, saturating;
// exact FP64 comparisons (value * s has at most 28 significant bits).
static __device__ __noinline__ uint32_t e4m3_div_exact(float a, float s)
{
    const double den = (double)s, num = (double)a;
    uint32_t lo = 0u, hi = 126u;                                 // largest code with value * den <= num
    while (lo < hi) {
        const uint32_t mid = (lo + hi + 1u) >> 1;
        if ((double)e4m3_value(mid) * den <= num) lo = mid; else hi = mid - 1u;
    }
    if (lo == 126u) return 126u;
    const double t = 0.5 * ((double)e4m3_value(lo) + (double)e4m3_value(lo + 1u)) * den;
    if (num > t) return lo + 1u;
    if (num == t) return (lo & 1u) ? lo + 1u : lo;
    return lo;
}

// Exact E4M3 code (sign kept) of x / s when the bracket ends gave codes lo and hi for |x|.
__device__ __forceinline__ uint32_t fp8_fix(float x, float s, uint32_t lo, uint32_t hi)
{
    const uint32_t sign = lo & 0x80u;
    uint32_t c = min(lo & 0x7Fu, hi & 0x7Fu);                     // the bracket's lower magnitude code
    if ((lo & 0x7Fu) != (hi & 0x7Fu)) {                           // adjacent codes: one exact comparison
        const float mid = 0.5f * (e4m3_value(c) + e4m3_value(c + 1u));
        const float d = fmaf(mid, s, -fabsf(x));
        c = d < 0.0f ? c + 1u : (d > 0.0f ? c : c + (c & 1u));
    }
    return sign | c;
}

// Two E4M3 codes (bits 0-7 and 8-15) to their values as FP16 (exact), low code in the
// low half.
__device__ __forceinline__ __half2 e4m3x2_to_half2(uint32_t codes)
{
    uint32_t r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"((unsigned short)codes));
    return *reinterpret_cast<const __half2*>(&r);
}

// Codes of 16 elements against s (bracket r_lo <= 1/s <= r_hi).  The hardware conversion
// keeps the sign, so signed products convert directly; a pair is exact when both ends of
// the bracket agree on both codes.
__device__ __forceinline__ void fp8_codes16(const float v[16], float s, float r_lo, float r_hi, int mode,
                                            uint32_t out[4])
{
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        uint32_t half[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float x0 = v[4 * w + 2 * h], x1 = v[4 * w + 2 * h + 1];
            if (mode == 1) {
                const float2 pl = __fmul2_rn(make_float2(x0, x1), make_float2(r_lo, r_lo));
                const float2 ph = __fmul2_rn(make_float2(x0, x1), make_float2(r_hi, r_hi));
                const uint32_t lo = cvt_e4m3x2(pl.x, pl.y), hi = cvt_e4m3x2(ph.x, ph.y);
                half[h] = lo;
                if (lo != hi)
                    half[h] = fp8_fix(x0, s, lo & 0xFFu, hi & 0xFFu) | (fp8_fix(x1, s, lo >> 8, hi >> 8) << 8);
            } else {
                const uint32_t s0 = (__float_as_uint(x0) >> 24) & 0x80u, s1 = (__float_as_uint(x1) >> 24) & 0x80u;
                const uint32_t c0 = mode == 0 ? 0u : e4m3_div_exact(fabsf(x0), s);
                const uint32_t c1 = mode == 0 ? 0u : e4m3_div_exact(fabsf(x1), s);
                half[h] = (s0 | c0) | ((s1 | c1) << 8);
            }
        }
        out[w] = half[0] | (half[1] << 16);
    }
}

// Every group this thread owns when s is zero or far from 1 (mode 0 or 2): no bracket,
// exact FP64 divisions.  Out of line and entered once, so the streaming loop below keeps
// few registers.
template <int kIn>
static __device__ __noinline__ uint32_t fp8_quant_exact_all(const void* x, uint32_t total, uint32_t groups_per_row,
                                                            int64_t ld, FastDiv div_gpr, uint8_t* q, int64_t ldq,
                                                            float s, int mode)
{
    uint32_t flags = 0u;
    for (uint32_t g = blockIdx.x * kVarThreads + threadIdx.x; g < total; g += gridDim.x * kVarThreads) {
        const uint32_t row = div_gpr.div(g), gg = g - row * groups_per_row;
        float v[16];
        uint32_t ab;
        load16<kIn>(x, (int64_t)row * ld + 16 * (int64_t)gg, v, ab);
        if (ab >= 0x7F800000u) flags |= kFlagNonFinite;
        uint32_t w[4];
        fp8_codes16(v, s, 0.0f, 0.0f, mode, w);
        __stcs(reinterpret_cast<uint4*>(q + (int64_t)row * ldq + 16 * (int64_t)gg), make_uint4(w[0], w[1], w[2], w[3]));
    }
    return flags;
}

// One thread per group of 16 elements, grid-stride, with the next group's loads in flight
// while this one is converted: two scaled products per element (the bracket
// r_lo <= 1/s <= r_hi) and two hardware conversions per pair; the rare elements whose
// bracket ends disagree get one exact FMA comparison each.
template <int kIn>
__global__ void __launch_bounds__(kVarThreads)
fp8_quant_kernel(const void* x, uint32_t rows, uint32_t groups_per_row, int64_t ld, FastDiv div_gpr,
                 const float* __restrict__ d_amax, uint8_t* __restrict__ q, int64_t ldq, float* __restrict__ d_scale,
                 uint32_t* __restrict__ d_flags)
{
    const float s = __fdiv_rn(*d_amax, 448.0f);                   // RN32(amax / 448)
    if (blockIdx.x == 0 && threadIdx.x == 0) *d_scale = s;
    const int mode = s == 0.0f ? 0 : (s >= 0x1p-100f && s <= 0x1p100f ? 1 : 2);
    uint32_t flags = isfinite(s) ? 0u : kFlagOverflow;
    const uint32_t total = rows * groups_per_row;
    if (mode != 1) {
        flags |= fp8_quant_exact_all<kIn>(x, total, groups_per_row, ld, div_gpr, q, ldq, s, mode);
    } else {
        const float r = __frcp_rn(s);
        const float r_lo = __fmul_rn(r, kLoMargin), r_hi = __fmul_rn(r, kHiMargin);
        const uint32_t stride = gridDim.x * kVarThreads;
        constexpr int kWords = kIn == 0 ? 2 : 4;
        constexpr int kElem = kIn == 0 ? 2 : 4;
        auto offset = [&](uint32_t g) {
            const uint32_t row = div_gpr.div(g);
            return (int64_t)row * ld + 16 * (int64_t)(g - row * groups_per_row);
        };
        uint4 nxt[kWords];
        uint32_t g = blockIdx.x * kVarThreads + threadIdx.x;
        if (g < total) {
            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const char*>(x) + offset(g) * kElem);
#pragma unroll
            for (int k = 0; k < kWords; ++k) nxt[k] = __ldcs(src + k);
        }
        for (; g < total; g += stride) {
            const uint32_t row = div_gpr.div(g), gg = g - row * groups_per_row;
            uint4 cur[kWords];
#pragma unroll
            for (int k = 0; k < kWords; ++k) cur[k] = nxt[k];
            if (g + stride < total) {
                const uint4* src =
                    reinterpret_cast<const uint4*>(static_cast<const char*>(x) + offset(g + stride) * kElem);
#pragma unroll
                for (int k = 0; k < kWords; ++k) nxt[k] = __ldcs(src + k);
            }
            float v[16];
            uint32_t ab = 0u;
            const uint32_t* cw = reinterpret_cast<const uint32_t*>(cur);
            if constexpr (kIn == 0) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    ab = __vmaxu2(ab, cw[j] & 0x7FFF7FFFu);
                    v[2 * j] = bf16_lo(cw[j]);
                    v[2 * j + 1] = bf16_hi(cw[j]);
                }
                ab = max(ab & 0xFFFFu, ab >> 16) << 16;
            } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    ab = max(ab, cw[j] & 0x7FFFFFFFu);
                    v[j] = __uint_as_float(cw[j]);
                }
            }
            if (ab >= 0x7F800000u) flags |= kFlagNonFinite;
            uint32_t lo[8], straddle = 0u;                        // codes of pairs (2j, 2j+1)
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float2 p = make_float2(v[2 * j], v[2 * j + 1]);
                const float2 pl = __fmul2_rn(p, make_float2(r_lo, r_lo));
                const float2 ph = __fmul2_rn(p, make_float2(r_hi, r_hi));
                lo[j] = cvt_e4m3x2(pl.x, pl.y);
                straddle |= (lo[j] != cvt_e4m3x2(ph.x, ph.y) ? 1u : 0u) << j;
            }
            uint8_t* dst = q + (int64_t)row * ldq + 16 * (int64_t)gg;
            __stcs(reinterpret_cast<uint4*>(dst), make_uint4(lo[0] | (lo[1] << 16), lo[2] | (lo[3] << 16),
                                                            lo[4] | (lo[5] << 16), lo[6] | (lo[7] << 16)));
            // Pairs whose bracket ends disagree (about one element in a hundred when s is
            // close to a short rational, as for amax = 752): the pair is re-read (it is
            // still in L2), both elements decided exactly and its two bytes rewritten; the
            // loop runs over the set bits so a warp pays for its busiest lane only.
            const char* src = static_cast<const char*>(x) + ((int64_t)row * ld + 16 * (int64_t)gg) * kElem;
            while (straddle != 0u) {
                const int j = __ffs(straddle) - 1;
                straddle &= straddle - 1u;
                float2 p;
                if constexpr (kIn == 0) {
                    const uint32_t w2 = __ldcs(reinterpret_cast<const uint32_t*>(src) + j);
                    p = make_float2(bf16_lo(w2), bf16_hi(w2));
                } else {
                    p = __ldcs(reinterpret_cast<const float2*>(src) + j);
                }
                const float2 pl = __fmul2_rn(p, make_float2(r_lo, r_lo));
                const float2 ph = __fmul2_rn(p, make_float2(r_hi, r_hi));
                const uint32_t l2 = cvt_e4m3x2(pl.x, pl.y), h2 = cvt_e4m3x2(ph.x, ph.y);
                // the midpoint between each element's two candidate codes (exact in FP16:
                // at most 5 significant bits), then one exact FMA comparison per element
                const __half2 vl = e4m3x2_to_half2(l2 & 0x7F7Fu), vh = e4m3x2_to_half2(h2 & 0x7F7Fu);
                const float2 mid = __half22float2(__hmul2(__hadd2(vl, vh), __float2half2_rn(0.5f)));
                const float2 d = __ffma2_rn(mid, make_float2(s, s), make_float2(-fabsf(p.x), -fabsf(p.y)));
                const bool up0 = d.x < 0.0f || (d.x == 0.0f && (l2 & 1u));
                const bool up1 = d.y < 0.0f || (d.y == 0.0f && ((l2 >> 8) & 1u));
                reinterpret_cast<unsigned short*>(dst)[j] =
                    (unsigned short)(((up0 ? h2 : l2) & 0xFFu) | ((up1 ? h2 : l2) & 0xFF00u));
            }
        }
    }
    flags = __reduce_or_sync(__activemask(), flags);
    if ((threadIdx.x & 31) == 0) flag_or(d_flags, flags);
}

// One thread per 16 outputs: out = RN(e4m3(code) * s).
template <int kOut>
__global__ void __launch_bounds__(kVarThreads)
fp8_dequant_kernel(const uint8_t* __restrict__ q, const float* __restrict__ d_scale, uint32_t total16, void* out)
{
    const float s = *d_scale;
    for (uint32_t g = blockIdx.x * kVarThreads + threadIdx.x; g < total16; g += gridDim.x * kVarThreads) {
        const uint4 c = __ldcs(reinterpret_cast<const uint4*>(q) + g);
        const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
        float y[16];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t b = (cw[w] >> (8 * i)) & 0xFFu;
                const float v = (b & 0x7Fu) == 0x7Fu ? __uint_as_float(0x7FC00000u) : e4m3_value(b & 0x7Fu);
                y[4 * w + i] = __fmul_rn(b & 0x80u ? -v : v, s);
            }
        }
        if constexpr (kOut == 2) {
            float4* o = reinterpret_cast<float4*>(out) + 4 * (int64_t)g;
#pragma unroll
            for (int k = 0; k < 4; ++k) __stcs(o + k, make_float4(y[4 * k], y[4 * k + 1], y[4 * k + 2], y[4 * k + 3]));
        } else {
            uint32_t p[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if constexpr (kOut == 0)
                    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(p[j]) : "f"(y[2 * j + 1]), "f"(y[2 * j]));
                else
                    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(p[j]) : "f"(y[2 * j + 1]), "f"(y[2 * j]));
            }
            uint4* o = reinterpret_cast<uint4*>(out) + 2 * (int64_t)g;
            __stcs(o, make_uint4(p[0], p[1], p[2], p[3]));
            __stcs(o + 1, make_uint4(p[4], p[5], p[6], p[7]));
        }
    }
}

// ------------------------------------------------------------------ launchers
static int var_grid(int64_t work)
{
    const int64_t need = (work + kVarThreads - 1) / kVarThreads;
    const int64_t cap = (int64_t)num_sms() * 8;
    return (int)(need < cap ? (need > 0 ? need : 1) : cap);
}

cudaError_t launch_mxfp4_quant(const void* x, int in_dt, int64_t rows, int64_t cols, int64_t ld, uint8_t* q,
                               uint8_t* e8m0, uint32_t* d_flags, cudaStream_t s)
{
    const uint32_t hpr = (uint32_t)(cols / 16);
    const int64_t total = rows * (int64_t)hpr;
    const int g = var_grid(total);
    if (in_dt == 0)
        mxfp4_quant_kernel<0><<<g, kVarThreads, 0, s>>>(x, (uint32_t)rows, hpr, ld, FastDiv(hpr), q, e8m0, d_flags);
    else
        mxfp4_quant_kernel<2><<<g, kVarThreads, 0, s>>>(x, (uint32_t)rows, hpr, ld, FastDiv(hpr), q, e8m0, d_flags);
    return cudaGetLastError();
}

cudaError_t launch_mxfp4_dequant(const uint8_t* q, const uint8_t* e8m0, int64_t rows, int64_t cols, int out_dt,
                                 void* out, cudaStream_t s)
{
    const uint32_t total8 = (uint32_t)(rows * (cols / 8));
    const int g = var_grid(total8);
    if (out_dt == 0) mxfp4_dequant_kernel<0><<<g, kVarThreads, 0, s>>>(q, e8m0, total8, out);
    else if (out_dt == 1) mxfp4_dequant_kernel<1><<<g, kVarThreads, 0, s>>>(q, e8m0, total8, out);
    else mxfp4_dequant_kernel<2><<<g, kVarThreads, 0, s>>>(q, e8m0, total8, out);
    return cudaGetLastError();
}

cudaError_t launch_fp8_quant(const void* x, int in_dt, int64_t rows, int64_t cols, int64_t ld, const float* d_amax,
                             uint8_t* q, float* d_scale, uint32_t* d_flags, cudaStream_t s)
{
    const uint32_t gpr = (uint32_t)(cols / 16);
    const int g = var_grid(rows * (int64_t)gpr);
    if (in_dt == 0)
        fp8_quant_kernel<0><<<g, kVarThreads, 0, s>>>(x, (uint32_t)rows, gpr, ld, FastDiv(gpr), d_amax, q, cols,
                                                       d_scale, d_flags);
    else
        fp8_quant_kernel<2><<<g, kVarThreads, 0, s>>>(x, (uint32_t)rows, gpr, ld, FastDiv(gpr), d_amax, q, cols,
                                                       d_scale, d_flags);
    return cudaGetLastError();
}

cudaError_t launch_fp8_dequant(const uint8_t* q, const float* d_scale, int64_t rows, int64_t cols, int out_dt,
                               void* out, cudaStream_t s)
{
    const uint32_t total16 = (uint32_t)(rows * (cols / 16));
    const int g = var_grid(total16);
    if (out_dt == 0) fp8_dequant_kernel<0><<<g, kVarThreads, 0, s>>>(q, d_scale, total16, out);
    else if (out_dt == 1) fp8_dequant_kernel<1><<<g, kVarThreads, 0, s>>>(q, d_scale, total16, out);
    else fp8_dequant_kernel<2><<<g, kVarThreads, 0, s>>>(q, d_scale, total16, out);
    return cudaGetLastError();
}

}  // namespace nv4
