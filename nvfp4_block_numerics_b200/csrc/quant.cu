// quant.cu -- per-tensor amax, dynamic NVFP4 activation quantization and the
// two-step dequantization (sm_100a).
//
// Operations and their sources are documented at the entry points in
// include/nv4.h ([CAL] section 2 step 1; [FLOW] sections 3.4-3.6 and 5.4).
//
// All three kernels are HBM-bound streams: one pass over the input, 128-bit
// loads and stores, a grid of a few CTAs per SM striding over the data.
#include "nv4_common.cuh"
#include "nv4_internal.h"

namespace nv4 {

// ============================================================== amax
// Running maximum of |x|.  The maximum of BF16 (or FP32) magnitudes is taken on
// their bit patterns: for non-negative IEEE values the unsigned order of the bit
// patterns is the numeric order, and NaN patterns sort above +Inf.  A thread whose
// data holds a NaN re-scans its own elements without the NaN entries (rare path).
template <int kThreads>
__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, uint32_t* red)
{
    v = __reduce_max_sync(0xFFFFFFFFu, v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < kThreads / 32 ? red[lane] : 0u;
        v = __reduce_max_sync(0xFFFFFFFFu, v);
    }
    return v;
}

__device__ __forceinline__ uint32_t absmax_bf16x8(const uint4& v)
{
    const uint32_t a = __vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu);
    const uint32_t b = __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu);
    return __vmaxu2(a, b);
}

__device__ __forceinline__ uint32_t absmax_bf16x8_no_nan(const uint4& v)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t m = 0u;
    for (int j = 0; j < 4; ++j) {
        const uint32_t lo = w[j] & 0x7FFFu, hi = (w[j] >> 16) & 0x7FFFu;
        if (lo <= 0x7F80u) m = max(m, lo);
        if (hi <= 0x7F80u) m = max(m, hi);
    }
    return m;
}

template <int kThreads>
__global__ void __launch_bounds__(kThreads)
amax_bf16_kernel(const uint4* __restrict__ x, int64_t nvec, const uint16_t* __restrict__ tail, int ntail,
                 float* __restrict__ d_amax, uint32_t* __restrict__ d_flags)
{
    __shared__ uint32_t red[kThreads / 32];
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    const int64_t i0 = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    uint32_t m = 0u;                                   // two packed 16-bit maxima
    int64_t i = i0;
    for (; i + 3 * stride < nvec; i += 4 * stride) {   // four independent loads in flight
        const uint4 v0 = __ldcs(x + i), v1 = __ldcs(x + i + stride);
        const uint4 v2 = __ldcs(x + i + 2 * stride), v3 = __ldcs(x + i + 3 * stride);
        m = __vmaxu2(m, __vmaxu2(__vmaxu2(absmax_bf16x8(v0), absmax_bf16x8(v1)),
                                 __vmaxu2(absmax_bf16x8(v2), absmax_bf16x8(v3))));
    }
    for (; i < nvec; i += stride) m = __vmaxu2(m, absmax_bf16x8(__ldcs(x + i)));
    uint32_t amax = max(m & 0xFFFFu, m >> 16);
    if (blockIdx.x == 0)
        for (int t = threadIdx.x; t < ntail; t += kThreads) amax = max(amax, (uint32_t)(tail[t] & 0x7FFFu));
    uint32_t flags = amax >= 0x7F80u ? kFlagNonFinite : 0u;
    if (amax > 0x7F80u) {                              // a NaN: recompute without NaN entries
        amax = 0u;
        for (int64_t k = i0; k < nvec; k += stride) amax = max(amax, absmax_bf16x8_no_nan(x[k]));
        if (blockIdx.x == 0)
            for (int t = threadIdx.x; t < ntail; t += kThreads) {
                const uint32_t a = tail[t] & 0x7FFFu;
                if (a <= 0x7F80u) amax = max(amax, a);
            }
    }
    flags = __reduce_or_sync(0xFFFFFFFFu, flags);
    if ((threadIdx.x & 31) == 0) flag_or(d_flags, flags);
    amax = block_max_u32<kThreads>(amax << 16, red);   // BF16 bits -> FP32 bits
    if (threadIdx.x == 0 && amax != 0u) atomicMax(reinterpret_cast<unsigned int*>(d_amax), amax);
}

template <int kThreads>
__global__ void __launch_bounds__(kThreads)
amax_f32_kernel(const uint4* __restrict__ x, int64_t nvec, const uint32_t* __restrict__ tail, int ntail,
                float* __restrict__ d_amax, uint32_t* __restrict__ d_flags)
{
    __shared__ uint32_t red[kThreads / 32];
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    const int64_t i0 = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    uint32_t m = 0u;
    int64_t i = i0;
    for (; i + 1 * stride < nvec; i += 2 * stride) {
        const uint4 v0 = __ldcs(x + i), v1 = __ldcs(x + i + stride);
        m = max(m, max(max(v0.x & 0x7FFFFFFFu, v0.y & 0x7FFFFFFFu), max(v0.z & 0x7FFFFFFFu, v0.w & 0x7FFFFFFFu)));
        m = max(m, max(max(v1.x & 0x7FFFFFFFu, v1.y & 0x7FFFFFFFu), max(v1.z & 0x7FFFFFFFu, v1.w & 0x7FFFFFFFu)));
    }
    for (; i < nvec; i += stride) {
        const uint4 v = __ldcs(x + i);
        m = max(m, max(max(v.x & 0x7FFFFFFFu, v.y & 0x7FFFFFFFu), max(v.z & 0x7FFFFFFFu, v.w & 0x7FFFFFFFu)));
    }
    if (blockIdx.x == 0)
        for (int t = threadIdx.x; t < ntail; t += kThreads) m = max(m, tail[t] & 0x7FFFFFFFu);
    uint32_t flags = m >= 0x7F800000u ? kFlagNonFinite : 0u;
    if (m > 0x7F800000u) {
        m = 0u;
        for (int64_t k = i0; k < nvec; k += stride) {
            const uint4 v = x[k];
            const uint32_t w[4] = {v.x & 0x7FFFFFFFu, v.y & 0x7FFFFFFFu, v.z & 0x7FFFFFFFu, v.w & 0x7FFFFFFFu};
            for (int j = 0; j < 4; ++j)
                if (w[j] <= 0x7F800000u) m = max(m, w[j]);
        }
        if (blockIdx.x == 0)
            for (int t = threadIdx.x; t < ntail; t += kThreads) {
                const uint32_t a = tail[t] & 0x7FFFFFFFu;
                if (a <= 0x7F800000u) m = max(m, a);
            }
    }
    flags = __reduce_or_sync(0xFFFFFFFFu, flags);
    if ((threadIdx.x & 31) == 0) flag_or(d_flags, flags);
    m = block_max_u32<kThreads>(m, red);
    if (threadIdx.x == 0 && m != 0u) atomicMax(reinterpret_cast<unsigned int*>(d_amax), m);
}

// ============================================================== act quant
// Tables of E4M3 values and their FP32 reciprocals, built per CTA in shared memory.
struct E4M3Tables {
    float dec[128];
    float rcp[128];
};

__device__ __forceinline__ void fill_e4m3_tables(E4M3Tables& t)
{
    for (int c = threadIdx.x; c < 128; c += blockDim.x) {
        const float v = c < 127 ? e4m3_value((uint32_t)c) : 0.0f;
        t.dec[c] = v;
        t.rcp[c] = c > 0 && c < 127 ? __frcp_rn(v) : 0.0f;
    }
}

// Quantizes 16 values x[] with block scale S into two words of packed E2M1 codes.
// r_lo / r_hi bracket 1/S (see nv4_common.cuh); exact == true forces the FP64 path
// (only for a block scale outside [2^-100, 2^100]).  S == 0 passes r_lo = r_hi = 0:
// the products keep the sign of x and convert to sign-only codes.
__device__ __forceinline__ void quantize16(const float x[16], float S, float r_lo, float r_hi, bool exact,
                                           uint32_t& w0, uint32_t& w1)
{
    if (!exact) {
        float lo[16], hi[16];
        const float2 rl = make_float2(r_lo, r_lo), rh = make_float2(r_hi, r_hi);
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            const float2 xv = make_float2(x[i], x[i + 1]);
            const float2 a = __fmul2_rn(xv, rl), b = __fmul2_rn(xv, rh);
            lo[i] = a.x; lo[i + 1] = a.y;
            hi[i] = b.x; hi[i + 1] = b.y;
        }
        w0 = cvt_e2m1x8(lo);
        w1 = cvt_e2m1x8(lo + 8);
        const uint32_t h0 = cvt_e2m1x8(hi), h1 = cvt_e2m1x8(hi + 8);
        if (w0 != h0) w0 = e2m1_fix8(x, S, w0, h0);
        if (w1 != h1) w1 = e2m1_fix8(x + 8, S, w1, h1);
        return;
    }
    w0 = w1 = 0u;
    for (int i = 0; i < 8; ++i) w0 |= e2m1_code_exact(x[i], S) << (4 * i);
    for (int i = 0; i < 8; ++i) w1 |= e2m1_code_exact(x[8 + i], S) << (4 * i);
}

constexpr int kActThreads = 256;

// One 16-element block of the input: BF16 (two 128-bit words) or FP32 (four).
template <int kIn>
struct BlockIn {
    uint4 v[kIn == 0 ? 2 : 4];
};

template <int kIn>
__device__ __forceinline__ void load_block_in(const void* x, int64_t off, BlockIn<kIn>& blk)
{
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const char*>(x) + off * (kIn == 0 ? 2 : 4));
#pragma unroll
    for (int k = 0; k < (kIn == 0 ? 2 : 4); ++k) blk.v[k] = __ldcs(src + k);
}

// Block max magnitude bits (as an FP32 bit pattern) and the 16 values as floats.
template <int kIn>
__device__ __forceinline__ uint32_t unpack_block(const BlockIn<kIn>& blk, float xv[16])
{
    if constexpr (kIn == 0) {
        const uint32_t w[8] = {blk.v[0].x, blk.v[0].y, blk.v[0].z, blk.v[0].w,
                               blk.v[1].x, blk.v[1].y, blk.v[1].z, blk.v[1].w};
        uint32_t m = 0u;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            m = __vmaxu2(m, w[j] & 0x7FFF7FFFu);
            xv[2 * j] = bf16_lo(w[j]);
            xv[2 * j + 1] = bf16_hi(w[j]);
        }
        return max(m & 0xFFFFu, m >> 16) << 16;
    } else {
        uint32_t m = 0u;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t w[4] = {blk.v[k].x, blk.v[k].y, blk.v[k].z, blk.v[k].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                m = max(m, w[j] & 0x7FFFFFFFu);
                xv[4 * k + j] = __uint_as_float(w[j]);
            }
        }
        return m;
    }
}

// Fake quantize-dequantize output of one block: DQ2 RN32(v * S), then the output type.
template <int kOut>
__device__ __forceinline__ void store_qdq(uint32_t q0, uint32_t q1, float S, void* out, int64_t off)
{
    uint32_t h[8];
    cvt_e2m1x8_to_f16x8(q0, h);
    cvt_e2m1x8_to_f16x8(q1, h + 4);
    float y[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float a, c;
        f16x2_to_f32(h[j], a, c);
        const float2 r = __fmul2_rn(make_float2(a, c), make_float2(S, S));
        y[2 * j] = r.x;
        y[2 * j + 1] = r.y;
    }
    if constexpr (kOut == 2) {
        float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + off);
#pragma unroll
        for (int k = 0; k < 4; ++k) __stcs(o + k, make_float4(y[4 * k], y[4 * k + 1], y[4 * k + 2], y[4 * k + 3]));
    } else {
        uint32_t p[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if constexpr (kOut == 0) {
                asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(p[j]) : "f"(y[2 * j + 1]), "f"(y[2 * j]));
            } else {
                asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(p[j]) : "f"(y[2 * j + 1]), "f"(y[2 * j]));
            }
        }
        uint4* o = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + off);
        __stcs(o, make_uint4(p[0], p[1], p[2], p[3]));
        __stcs(o + 1, make_uint4(p[4], p[5], p[6], p[7]));
    }
}

// Block quantizer over a [rows, cols] tensor: one thread per 16-block, grid-stride,
// with the next block's loads in flight while the current one is quantized.
// kIn: 0 BF16, 2 FP32 input.  kOut: -1 writes packed codes + E4M3 scales; 0/1/2 writes
// the fake quantize-dequantize values as BF16/FP16/FP32 (leading dimension ld_out).
// Every block is read and written by the same thread, read first, so out may alias x.
template <int kIn, int kOut>
__global__ void __launch_bounds__(kActThreads)
act_quant_kernel(const void* x, uint32_t rows, uint32_t bpr, int64_t ld, FastDiv div_bpr,
                 const float* __restrict__ d_amax, uint8_t* __restrict__ q, uint8_t* __restrict__ scales,
                 void* out, int64_t ld_out, float* __restrict__ d_s2, uint32_t* __restrict__ d_flags)
{
    __shared__ E4M3Tables tab;
    fill_e4m3_tables(tab);
    __syncthreads();

    const float amax = *d_amax;
    const float s2 = __fdiv_rn(amax, 2688.0f);                  // RN32(amax / (6*448))
    if (blockIdx.x == 0 && threadIdx.x == 0) *d_s2 = s2;
    const bool fast_scale = s2 >= kTinyScale && s2 <= 0x1p100f;
    const float k = __frcp_rn(__fmul_rn(6.0f, s2));             // ~ 1/(6*s2)
    const float k_lo = __fmul_rn(k, kLoMargin), k_hi = __fmul_rn(k, kHiMargin);
    const float rs2 = __frcp_rn(s2);                            // ~ 1/s2
    uint32_t flags = isfinite(s2) ? 0u : kFlagOverflow;

    const uint32_t total = rows * bpr;
    const uint32_t stride = gridDim.x * kActThreads;
    auto offset = [&](uint32_t u, int64_t l) {
        const uint32_t r = div_bpr.div(u), bb = u - r * bpr;
        return (int64_t)r * l + 16 * (int64_t)bb;
    };
    uint32_t u = blockIdx.x * kActThreads + threadIdx.x;
    BlockIn<kIn> nxt;
    if (u < total) load_block_in<kIn>(x, offset(u, ld), nxt);
    for (; u < total; u += stride) {
        const BlockIn<kIn> cur = nxt;
        if (u + stride < total) load_block_in<kIn>(x, offset(u + stride, ld), nxt);
        float xv[16];
        const uint32_t ab = unpack_block<kIn>(cur, xv);
        if (ab >= 0x7F800000u) flags |= kFlagNonFinite;
        const float a_b = __uint_as_float(ab);

        // block scale: nearest E4M3 to a_b / (6*s2)
        uint32_t code;
        if (fast_scale) {
            const uint32_t cc = cvt_e4m3x2(__fmul_rn(a_b, k_lo), __fmul_rn(a_b, k_hi));
            code = cc & 0xFFu;
            if (code != (cc >> 8)) code = e4m3_fix(code, a_b, s2);
        } else {
            code = e4m3_code_exact(a_b, s2);
        }
        code &= 0x7Fu;                                            // non-negative inputs only
        const float S = __fmul_rn(tab.dec[code], s2);            // DQ1: RN32(s_b * s2)

        const bool exact = S != 0.0f && !(S >= kTinyScale && S <= 0x1p100f);
        const float rr = S == 0.0f ? 0.0f : __fmul_rn(tab.rcp[code], rs2);   // ~ 1/S
        uint32_t q0, q1;
        quantize16(xv, S, __fmul_rn(rr, kLoMargin), __fmul_rn(rr, kHiMargin), exact, q0, q1);

        if constexpr (kOut < 0) {
            *reinterpret_cast<uint2*>(q + (int64_t)u * 8) = make_uint2(q0, q1);
            scales[u] = (uint8_t)code;
        } else {
            store_qdq<kOut>(q0, q1, S, out, offset(u, ld_out));
        }
    }
    flags = __reduce_or_sync(__activemask(), flags);
    if ((threadIdx.x & 31) == 0) flag_or(d_flags, flags);
}

// ============================================================== dequant
__device__ __forceinline__ float e4m3_value_signed(uint32_t c)
{
    if ((c & 0x7Fu) == 0x7Fu) return __uint_as_float(0x7FC00000u);
    const float v = e4m3_value(c & 0x7Fu);
    return (c & 0x80u) ? -v : v;
}

// One thread handles eight outputs (half a 16-block): 4 code bytes and the block's
// scale byte in, 16 (BF16/FP16) or 32 (FP32) bytes out, so a warp reads 128
// contiguous code bytes and writes 512 or 1024 contiguous output bytes per step.
template <int kOut>
__device__ __forceinline__ void dequant8(uint32_t qw, uint32_t sc, float s2, void* __restrict__ out, int64_t h)
{
    const float S = __fmul_rn(e4m3_value_signed(sc), s2);      // DQ1: RN32(s_b * s2)
    uint32_t hv[4];
    cvt_e2m1x8_to_f16x8(qw, hv);
    float y[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float a, b;
        f16x2_to_f32(hv[j], a, b);
        const float2 r = __fmul2_rn(make_float2(a, b), make_float2(S, S));   // DQ2: RN32(v * S)
        y[2 * j] = r.x;
        y[2 * j + 1] = r.y;
    }
    if constexpr (kOut == 2) {
        float4* o = reinterpret_cast<float4*>(out) + h * 2;
        __stcs(o, make_float4(y[0], y[1], y[2], y[3]));
        __stcs(o + 1, make_float4(y[4], y[5], y[6], y[7]));
    } else {
        uint32_t p[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if constexpr (kOut == 0) {
                asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(p[j]) : "f"(y[2 * j + 1]), "f"(y[2 * j]));
            } else {
                asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(p[j]) : "f"(y[2 * j + 1]), "f"(y[2 * j]));
            }
        }
        __stcs(reinterpret_cast<uint4*>(out) + h, make_uint4(p[0], p[1], p[2], p[3]));
    }
}

template <int kOut>   // 0 bf16, 1 fp16, 2 fp32
__global__ void __launch_bounds__(kActThreads)
dequant_kernel(const uint8_t* __restrict__ q, const uint8_t* __restrict__ scales, const float* __restrict__ d_s2,
               uint32_t total, void* __restrict__ out)
{
    const float s2 = *d_s2;
    const uint32_t halves = 2u * total;
    const uint32_t stride = gridDim.x * kActThreads;
    const uint32_t* qw = reinterpret_cast<const uint32_t*>(q);
    uint32_t h = blockIdx.x * kActThreads + threadIdx.x;
    for (; h + 3u * stride < halves; h += 4u * stride) {          // four independent steps in flight
        uint32_t a[4], c[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            a[k] = __ldcs(qw + h + k * stride);
            c[k] = scales[(h + k * stride) >> 1];
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) dequant8<kOut>(a[k], c[k], s2, out, h + k * stride);
    }
    for (; h < halves; h += stride) dequant8<kOut>(__ldcs(qw + h), scales[h >> 1], s2, out, h);
}

// ============================================================== launchers
static int grid_for(int64_t work, int threads, int per_sm)
{
    const int64_t need = (work + threads - 1) / threads;
    const int64_t cap = (int64_t)num_sms() * per_sm;
    return (int)(need < cap ? (need > 0 ? need : 1) : cap);
}

cudaError_t launch_amax(const void* x, int dt, int64_t n, float* d_amax, uint32_t* d_flags, cudaStream_t s)
{
    constexpr int T = 512;
    if (dt == 0) {
        const int64_t nvec = n / 8;
        const int ntail = (int)(n - nvec * 8);
        const uint16_t* tail = static_cast<const uint16_t*>(x) + nvec * 8;
        amax_bf16_kernel<T><<<grid_for(nvec, T, 4), T, 0, s>>>(static_cast<const uint4*>(x), nvec, tail, ntail,
                                                                 d_amax, d_flags);
    } else {
        const int64_t nvec = n / 4;
        const int ntail = (int)(n - nvec * 4);
        const uint32_t* tail = static_cast<const uint32_t*>(x) + nvec * 4;
        amax_f32_kernel<T><<<grid_for(nvec, T, 4), T, 0, s>>>(static_cast<const uint4*>(x), nvec, tail, ntail,
                                                                d_amax, d_flags);
    }
    return cudaGetLastError();
}

cudaError_t launch_act_quant(const void* x, int64_t rows, int64_t cols, int64_t ld, const float* d_amax,
                             uint8_t* q, uint8_t* scales, float* d_s2, uint32_t* d_flags, cudaStream_t s)
{
    return launch_block_quant(x, 0, rows, cols, ld, d_amax, q, scales, -1, nullptr, 0, d_s2, d_flags, s);
}

cudaError_t launch_block_quant(const void* x, int in_dt, int64_t rows, int64_t cols, int64_t ld,
                               const float* d_amax, uint8_t* q, uint8_t* scales, int out_dt, void* out,
                               int64_t ld_out, float* d_s2, uint32_t* d_flags, cudaStream_t s)
{
    const uint32_t bpr = (uint32_t)(cols / 16);
    const uint32_t total = (uint32_t)rows * bpr;
    const int g = grid_for(total, kActThreads, 8);
#define NV4_BQ(I, O) act_quant_kernel<I, O><<<g, kActThreads, 0, s>>>(x, (uint32_t)rows, bpr, ld, FastDiv(bpr), \
        d_amax, q, scales, out, ld_out, d_s2, d_flags)
    if (in_dt == 0) {
        if (out_dt < 0) NV4_BQ(0, -1); else if (out_dt == 0) NV4_BQ(0, 0); else if (out_dt == 1) NV4_BQ(0, 1); else NV4_BQ(0, 2);
    } else {
        if (out_dt < 0) NV4_BQ(2, -1); else if (out_dt == 0) NV4_BQ(2, 0); else if (out_dt == 1) NV4_BQ(2, 1); else NV4_BQ(2, 2);
    }
#undef NV4_BQ
    return cudaGetLastError();
}

cudaError_t launch_dequant(const uint8_t* q, const uint8_t* scales, const float* d_s2, int64_t rows, int64_t cols,
                           int out_dt, void* out, cudaStream_t s)
{
    const uint32_t total = (uint32_t)(rows * (cols / 16));
    const int g = grid_for((int64_t)total * 2, kActThreads, 8);
    if (out_dt == 0) dequant_kernel<0><<<g, kActThreads, 0, s>>>(q, scales, d_s2, total, out);
    else if (out_dt == 1) dequant_kernel<1><<<g, kActThreads, 0, s>>>(q, scales, d_s2, total, out);
    else dequant_kernel<2><<<g, kActThreads, 0, s>>>(q, scales, d_s2, total, out);
    return cudaGetLastError();
}

}  // namespace nv4
