// nv4_common.cuh -- device helpers shared by the NVFP4 kernels (sm_100a).
//
// Number formats (see include/nv4.h for the page citations):
//   E2M1 (FP4) code  sign(bit 3) | exponent(2 bits, bias 1) | mantissa(1 bit):
//                    magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6.
//   E4M3 (fn)        bias 7, subnormals m*2^-9, largest 448 (0x7E), 0x7F NaN.
//
// Rounding strategy.  Every code the library emits is the nearest representable
// value to an EXACT real quotient (ties to the even code).  The fast path brackets
// the quotient between two FP32 products q_lo <= q <= q_hi and converts both with
// the hardware's round-to-nearest-even FP4/FP8 conversion.  Rounding to a grid is
// monotone, so when both ends give the same code that code is the exact answer.
// When they differ (the quotient sits within ~2^-20 relative of a rounding
// boundary) one exact FP32 comparison decides: fma(boundary, divisor, -numerator)
// rounds the exact difference once, so its sign is exact (see the fix-ups below).
// Divisors outside [2^-100, 2^100] take exact FP64 comparisons instead.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace nv4 {

// relative margin of the bracket; covers the < 2^-21.4 relative error of
// a product by a reciprocal that was itself rounded up to three times
constexpr float kLoMargin = 1.0f - 0x1p-20f;
constexpr float kHiMargin = 1.0f + 0x1p-20f;
// below this a quotient bracket could leave the normal FP32 range: use exact paths
constexpr float kTinyScale = 0x1p-100f;

constexpr uint32_t kFlagNonFinite = 1u;
constexpr uint32_t kFlagE8M0Nan = 2u;
constexpr uint32_t kFlagOverflow = 4u;
constexpr uint32_t kFlagTimeout = 8u;

__device__ __forceinline__ void flag_or(uint32_t* flags, uint32_t bits)
{
    if (flags != nullptr && bits != 0u) atomicOr(flags, bits);
}

// ---------------------------------------------------------------- BF16
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ---------------------------------------------------------------- E4M3
// Value of a non-negative finite E4M3 code c in [0, 126].
__device__ __forceinline__ float e4m3_value(uint32_t c)
{
    const uint32_t e = c >> 3, m = c & 7u;
    return e == 0u ? __uint2float_rn(m) * 0x1p-9f : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Hardware conversion of two non-negative FP32 values to E4M3 codes (RNE,
// saturating at 448).  Returns lo's code in bits 0-7 and hi's in bits 8-15.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi)
{
    unsigned short r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// ---------------------------------------------------------------- E2M1
// Hardware conversion of 8 FP32 values to 8 E2M1 codes (RNE, saturating at 6,
// sign kept); element k lands in bits 4k..4k+3.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float v[8])
{
    uint32_t r;
    asm("{\n\t"
        ".reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t"
        "}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

// Packed E2M1 codes of lo (bits 0-3) and hi (bits 4-7): RNE, saturating at 6, sign kept.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi)
{
    uint32_t r;
    asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %2, %1;\n\tcvt.u32.u8 %0, b;\n\t}"
        : "=r"(r)
        : "f"(lo), "f"(hi));
    return r;
}

// Hardware decode of the 8 E2M1 codes packed in w (element k in bits 4k..4k+3)
// to FP16 pairs: h[j] holds elements 2j (low half) and 2j+1 (high half).  E2M1
// values are exact in FP16.
__device__ __forceinline__ void cvt_e2m1x8_to_f16x8(uint32_t w, uint32_t h[4])
{
    asm("{\n\t"
        ".reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t"
        "}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
}

__device__ __forceinline__ void f16x2_to_f32(uint32_t h, float& lo, float& hi)
{
    unsigned short a = (unsigned short)(h & 0xFFFFu), b = (unsigned short)(h >> 16);
    asm("cvt.f32.f16 %0, %1;" : "=f"(lo) : "h"(a));
    asm("cvt.f32.f16 %0, %1;" : "=f"(hi) : "h"(b));
}

// ---------------------------------------------------------------- exact fallbacks
// Nearest E4M3 code (0..126) to the real num / (6*s2), num >= 0, ties to the even
// code, saturating at 448.  6*s2 has 26 significant bits and a midpoint of two
// E4M3 values at most 5, so every product below is exact in FP64.
static __device__ __noinline__ uint32_t e4m3_code_exact(float num, float s2)
{
    if (!(s2 > 0.0f)) return 0u;
    const double den = 6.0 * (double)s2;
    const double a = (double)num;
    uint32_t lo = 0u, hi = 126u;            // largest code with value*den <= a
    while (lo < hi) {
        const uint32_t mid = (lo + hi + 1u) >> 1;
        if ((double)e4m3_value(mid) * den <= a) lo = mid; else hi = mid - 1u;
    }
    if (lo == 126u) return 126u;
    const double t = 0.5 * ((double)e4m3_value(lo) + (double)e4m3_value(lo + 1u)) * den;
    if (a > t) return lo + 1u;
    if (a == t) return (lo & 1u) ? lo + 1u : lo;
    return lo;
}

// E2M1 code of x under the FP32 block scale S: sign bit of x, magnitude nearest
// to |x|/S, ties to even, saturating at 6; S == 0 gives magnitude 0.  The grid
// midpoints have at most 3 significant bits, so mid*S is exact in FP64.
static __device__ __noinline__ uint32_t e2m1_code_exact(float x, float S)
{
    const uint32_t sign = (__float_as_uint(x) >> 28) & 8u;
    if (!(S > 0.0f)) return sign;
    const double a = fabs((double)x), s = (double)S;
    // boundaries between magnitude codes k and k+1, and whether a tie goes up
    const double mids[7] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};
    uint32_t k = 0u;
    while (k < 7u) {
        const double t = mids[k] * s;
        if (a < t) break;
        if (a == t) {                      // tie: the even code of k, k+1
            if (k & 1u) ++k;
            break;
        }
        ++k;
    }
    return sign | k;
}

// ---------------------------------------------------------------- exact fix-ups (FP32)
// When the two ends of a bracket convert to different codes, the quotient lies
// within ~2^-19 of exactly one rounding boundary, so the two codes are adjacent and
// one comparison decides.  fma(b, D, -a) rounds the exact b*D - a once, so its sign
// is exact, and it is zero only on an exact tie (no underflow: D >= 2^-100 on these
// paths and the operands agree to ~19 bits).

// Boundary between E2M1 magnitudes k and k+1: 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.
__device__ __forceinline__ float e2m1_boundary(uint32_t k)
{
    const uint64_t quarters = 0x00140E0A07050301ull;    // 4 x boundary, one byte per k
    return (float)((uint32_t)(quarters >> (8u * k)) & 0xFFu) * 0.25f;
}

// Corrects the packed codes lo (8 elements x[0..7], element i in bits 4i..4i+3) at
// every nibble where the bracket's other end hi disagrees; S is the block scale.  The
// loop runs over the differing nibbles only (usually one), so a warp whose lanes take
// this path at different elements pays for its busiest lane, not for every position
// (an unrolled test of all 8 positions measured 4% slower in the sweep, 1% in the
// activation quantizer).
__device__ __forceinline__ uint32_t e2m1_fix8(const float x[8], float S, uint32_t lo, uint32_t hi)
{
    uint32_t diff = lo ^ hi;
    while (diff != 0u) {
        const uint32_t sh = (uint32_t)(__ffs(diff) - 1) & ~3u;   // 4 x the element index
        diff &= ~(15u << sh);
        float xi = x[0];
#pragma unroll
        for (int j = 1; j < 8; ++j) xi = sh == 4u * j ? x[j] : xi;
        const uint32_t cl = (lo >> sh) & 15u, kl = cl & 7u;
        const float d = fmaf(e2m1_boundary(kl), S, -fabsf(xi));
        const uint32_t k = d < 0.0f ? kl + 1u : (d > 0.0f ? kl : kl + (kl & 1u));
        lo = (lo & ~(15u << sh)) | ((k | (cl & 8u)) << sh);
    }
    return lo;
}

// E4M3 block-scale code when the bracket gave codes c and c+1 for a / (6*s2):
// compares a with the midpoint times 6*s2 ((v_c + v_c+1) * 3 has <= 7 bits: exact).
__device__ __forceinline__ uint32_t e4m3_fix(uint32_t c, float a, float s2)
{
    const float mid6 = (e4m3_value(c) + e4m3_value(c + 1u)) * 3.0f;
    const float d = fmaf(mid6, s2, -a);
    return d < 0.0f ? c + 1u : (d > 0.0f ? c : c + (c & 1u));
}

// ---------------------------------------------------------------- time / waits
__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Upper bound of any wait inside a kernel.  A pipeline that has not made progress
// for this long is abandoned with NV4_FLAG_TIMEOUT instead of spinning forever.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

}  // namespace nv4
