// hadamard.cu -- block Hadamard rotation fused with FP4 quantization (sm_100a).
//
// [FP4] section 3.1 (blocks rotated by H / sqrt(n) before quantization, spreading
// outliers) and section 4.1 (quantization-transform kernels with block sizes 16, 32, 64
// and 128).  y = RN32(RN64(x_block H_n) * RN64(1/sqrt(n))) along each row, then:
//   mode 0: running max |y| into *d_amax (the per-tensor amax that NVFP4 needs);
//   mode 1: MXFP4 quantization of y (32-element blocks, E8M0 scales);
//   mode 2: NVFP4 quantization of y with s2 = RN32(amax / 2688).
//
// Mapping: a lane owns 32 consecutive elements of a row (four 16-byte loads); n / 32 lanes
// cover a segment of n elements.  The fast Walsh-Hadamard transform runs in FP64, so every
// sum is exact for BF16 inputs spanning fewer than ~38 binades in a block: up to five
// butterfly stages inside a lane, then log2(n / 32) stages across the segment's lanes.  For
// n = 64 the one cross-lane stage is a shuffle and one FMA with a factor of +-1; for n = 128
// the lanes exchange their values through shared memory, each lane takes an eighth of every
// chunk of its segment and runs both stages in registers, and the rounded FP32 outputs go
// back through shared memory so that the quantizers again see one chunk per lane (the
// amax of mode 0 skips that second exchange).  On a [65536, 7168] BF16 input: n = 128
// MXFP4 in 0.51 ms (0.63 ms with two shuffle stages of 2 shuffles and a select per value),
// NVFP4 0.58 ms (0.68), the amax pass 0.43 ms (0.54); n = 64 MXFP4 0.43 ms (0.50), n = 32
// 0.37 ms.  The quantizers then work on FP32 y exactly as nv4_mxfp4_quant / nv4_act_quant
// do; an MXFP4 block is one lane's 32 values, an NVFP4 block half of them.
#include <cmath>

#include "nv4_common.cuh"
#include "nv4_internal.h"

namespace nv4 {

constexpr int kHadThreads = 128;

// The in-lane part of the FWHT of blocks of n values, 32 consecutive values per lane: up to
// five butterfly stages (four for n = 16).
template <int kN>
__device__ __forceinline__ void fwht_lane(double v[32])
{
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
        if (h >= kN) break;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (i & h) continue;
            const double a = v[i], b = v[i + h];
            v[i] = a + b;
            v[i + h] = a - b;
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


// MXFP4 scale code of a block whose largest |y| has the bit pattern ab: the E8M0 code of
// 2^(floor(log2 amax) - 2) clamped to [-127, 127], 0 for an all-zero block, 0xFF (NaN) for
// a block holding NaN or Inf.
__device__ __forceinline__ uint32_t mx_block_code(uint32_t ab)
{
    if (ab >= 0x7F800000u) return 0xFFu;
    const int e = ab == 0u ? -127 : max(had_floor_log2(ab) - 2, -127);
    return (uint32_t)(e + 127);
}

// E2M1 codes of kCount values (16 or 32) under the MXFP4 scale `code`: scaling by 2^-e is
// exact, so one hardware RNE conversion per pair gives the exact codes.  w: kCount / 8 words.
template <int kCount>
__device__ __forceinline__ void mx_encode(const float* y, uint32_t code, uint32_t* w)
{
    if (code == 0xFFu) {
#pragma unroll
        for (int k = 0; k < kCount / 8; ++k) w[k] = 0u;
        return;
    }
    const float inv = had_pow2(127 - (int)code);
#pragma unroll
    for (int k = 0; k < kCount / 8; ++k) {
        float t[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) t[j] = __fmul_rn(y[8 * k + j], inv);   // exact
        w[k] = cvt_e2m1x8(t);
    }
}

// NVFP4 block scale code (E4M3, 7 bits) of a block whose largest |y| has the bit pattern bm,
// under s2 (k_lo, k_hi: the bracket of 1/(6 s2); fast: s2 inside [2^-100, 2^100]), as
// nv4_act_quant computes it.
__device__ __forceinline__ uint32_t nv_block_code(uint32_t bm, float s2, float k_lo, float k_hi, bool fast)
{
    const float a_b = __uint_as_float(bm);
    uint32_t code;
    if (fast) {
        const uint32_t cv = cvt_e4m3x2(__fmul_rn(a_b, k_lo), __fmul_rn(a_b, k_hi));
        code = cv & 0xFFu;
        if (code != (cv >> 8)) code = e4m3_fix(code, a_b, s2);
    } else {
        code = e4m3_code_exact(a_b, s2);
    }
    return code & 0x7Fu;
}

// E2M1 codes of 8 values of a block whose dequantization scale is S = RN32(s_b * s2).
__device__ __forceinline__ uint32_t nv_encode8(const float* yy, float S)
{
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
    return c8;
}

// NVFP4 of one 16-element block y: the scale code (returned) and the 16 E2M1 codes in w[0..1].
__device__ __forceinline__ uint32_t nv_block16(const float* y, float s2, float k_lo, float k_hi, bool fast,
                                               uint32_t* w)
{
    uint32_t bm = 0u;
#pragma unroll
    for (int j = 0; j < 16; ++j) bm = max(bm, __float_as_uint(y[j]) & 0x7FFFFFFFu);
    const uint32_t code = nv_block_code(bm, s2, k_lo, k_hi, fast);
    const float S = __fmul_rn(e4m3_value(code), s2);   // DQ1: RN32(s_b * s2)
    w[0] = nv_encode8(y, S);
    w[1] = nv_encode8(y + 8, S);
    return code;
}

template <int kMode, int kN>
__global__ void __launch_bounds__(kHadThreads)
hadamard_quant_kernel(const uint16_t* x, uint32_t rows, uint32_t chunks_per_row, int64_t ld, FastDiv div_cpr,
                      double c, float* __restrict__ d_amax, uint8_t* __restrict__ q, uint8_t* __restrict__ sc,
                      float* __restrict__ d_s2, uint32_t* __restrict__ d_flags)
{
    // one lane = one 32-element chunk of a row; kG lanes = one segment of n elements
    constexpr int kG = kN > 32 ? kN / 32 : 1;
    constexpr int kPitch = 34;                                     // doubles per lane in the exchange buffer
    __shared__ __align__(16) double xbuf[kG == 4 ? kHadThreads : 1][kPitch];
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t t = lane & (uint32_t)(kG - 1);                  // this lane's place in its segment
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

    // warp-uniform trip count (the lanes of a segment exchange values); the next chunk's
    // four loads are issued before the current chunk is transformed
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
        fwht_lane<kN>(v);
        if constexpr (kG == 2) {
            // n = 64: the last stage pairs neighbouring lanes; the upper lane forms lower - upper
            // as one FMA with a factor of -1 (a single rounding, like the subtraction)
            const double sg = (lane & 1u) != 0u ? -1.0 : 1.0;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const double o = __shfl_xor_sync(0xFFFFFFFFu, v[i], 1);
                v[i] = fma(sg, v[i], o);
            }
        } else if constexpr (kG == 4) {
            // n = 128: the two stages across the 4 lanes of a segment, through shared memory.
            // Lane a of the segment holds z_a[0..31] (its chunk after the in-lane stages);
            // afterwards lane t holds, for every a', the outputs a' * 32 + i of the segment for
            // i = 8 t .. 8 t + 7, out[a'][ii] = sum over a of (-1)^popcount(a' & a) z_a[i], formed
            // in the butterfly order of one stage per lane bit (lower + upper, lower - upper).
            // A lane's 16 pairs go to positions (k % 4) * 4 + k / 4 of its row (a 272-byte
            // pitch), so that the writes and the segment-wise reads each touch 32 distinct banks.
            double* mine = &xbuf[threadIdx.x][0];
#pragma unroll
            for (int k = 0; k < 16; ++k)
                *reinterpret_cast<double2*>(mine + 2 * ((k % 4) * 4 + k / 4)) = make_double2(v[2 * k], v[2 * k + 1]);
            __syncwarp();
            const double* grp = &xbuf[threadIdx.x & ~3u][0] + 2 * t;
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const double2 d2 = *reinterpret_cast<const double2*>(grp + a * kPitch + 8 * kk);
                    v[8 * a + 2 * kk] = d2.x;
                    v[8 * a + 2 * kk + 1] = d2.y;
                }
            __syncwarp();                                          // before the buffer is written again
#pragma unroll
            for (int h = 1; h < 4; h <<= 1)
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    if (a & h) continue;
#pragma unroll
                    for (int ii = 0; ii < 8; ++ii) {
                        const double lo = v[8 * a + ii], hi = v[8 * (a + h) + ii];
                        v[8 * a + ii] = lo + hi;
                        v[8 * (a + h) + ii] = lo - hi;
                    }
                }
        }
        float y[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) y[j] = (float)(v[j] * c);    // RN32(RN64(z * c))
        if constexpr (kG == 4 && kMode != 0) {
            // back to one chunk per lane for the quantizers (the maximum of mode 0 takes the
            // values in any order), through shared memory as FP32: output chunk k (four
            // values) of lane a' goes to 16-byte slot (k + 2 a') % 8 of a' 's 128-byte row, the
            // segments 1088 bytes apart plus 16 for odd ones, so that both sides touch 32
            // distinct banks
            const uint32_t sw = lane >> 2;                         // the segment's place in its warp
            float* segbuf = reinterpret_cast<float*>(&xbuf[threadIdx.x & ~31u][0]) + sw * 272u + 4u * (sw & 1u);
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const uint32_t k = 2u * t + (uint32_t)j;       // the chunk's place in row a
                    *reinterpret_cast<float4*>(segbuf + 32 * a + 4 * ((k + 2u * a) & 7u)) =
                        make_float4(y[8 * a + 4 * j], y[8 * a + 4 * j + 1], y[8 * a + 4 * j + 2], y[8 * a + 4 * j + 3]);
                }
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float4 f4 = *reinterpret_cast<const float4*>(segbuf + 32 * t + 4 * ((k + 2u * t) & 7u));
                y[4 * k] = f4.x; y[4 * k + 1] = f4.y; y[4 * k + 2] = f4.z; y[4 * k + 3] = f4.w;
            }
            __syncwarp();                                          // before the next chunk's writes
        }
        if (!live) continue;

        uint32_t ab = 0u;
#pragma unroll
        for (int j = 0; j < 32; ++j) ab = max(ab, __float_as_uint(y[j]) & 0x7FFFFFFFu);
        if (ab >= 0x7F800000u) flags |= kFlagNonFinite;
        const int64_t col = 32 * (int64_t)cc;

        if constexpr (kMode == 0) {
            if (ab <= 0x7F800000u) mx_bits = max(mx_bits, ab);
        } else if constexpr (kMode == 1) {
            uint32_t w[4];
            const uint32_t code = mx_block_code(ab);
            mx_encode<32>(y, code, w);
            __stcs(reinterpret_cast<uint4*>(q + (int64_t)r * (cols / 2) + col / 2), make_uint4(w[0], w[1], w[2], w[3]));
            sc[(int64_t)r * (cols / 32) + col / 32] = (uint8_t)code;
        } else {
            uint32_t w[4], codes2 = 0u;
#pragma unroll
            for (int hb = 0; hb < 2; ++hb)                         // two NVFP4 blocks of 16
                codes2 |= nv_block16(y + 16 * hb, s2, k_lo, k_hi, fast_scale, w + 2 * hb) << (8 * hb);
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


// ---------------------------------------------------------------- two-sided rotation of weight tiles
// [FP4] section 3.1: the weight matrix is cut into n x n tiles (n = 16 or 32) and each tile
// B becomes (H / sqrt(n)) B (H / sqrt(n))^T = H B H / n (H_n is symmetric), before FP4
// quantization.  y = RN32(exact(H B H) / n): 1/n is a power of two, and the FP64 sums are
// exact while the tile's values, as multiples of its smallest unit in the last place, fit
// 53 bits with the 2 log2(n) bits of growth (BF16 tiles spanning up to ~35 binades, FP32
// tiles up to ~19); beyond that the sum carries a relative error below 2^-52 before the
// one rounding to FP32.
//
// One warp per strip of n rows x 32 columns (one 32 x 32 tile, or two 16 x 16 tiles side by
// side), with the next strip's loads issued before the current one is transformed.  Lane l
// holds one row of its tile (n = 32: row l; n = 16: row l % 16 of tile l / 16) and runs that
// row's FWHT in FP64 registers; a transpose through shared memory (rows written as 16-byte
// pairs) gives lane l column l of the strip for the column FWHTs; the scaled, rounded values
// go back through shared memory as FP32 (rows read as 16-byte quads) so that lane l again
// holds its row for quantization:
//   mode 0: running max |y| into *d_amax;  mode 1: MXFP4 (32-element blocks along the row:
//   one lane's row for n = 32, lanes l and l + 16 together for n = 16);  mode 2: NVFP4
//   (16-element blocks) with s2 = RN32(amax / 2688);  mode 3: y itself, FP32 [rows, cols].
constexpr int kHad2Warps = 4;

template <int kN>
__device__ __forceinline__ void fwht_regs(double* v)
{
#pragma unroll
    for (int h = 1; h < kN; h <<= 1) {
#pragma unroll
        for (int i = 0; i < kN; ++i) {
            if (i & h) continue;
            const double a = v[i], b = v[i + h];
            v[i] = a + b;
            v[i + h] = a - b;
        }
    }
}

template <int kMode, int kN, int kDt>   // kDt 0 BF16, 2 FP32
__global__ void __launch_bounds__(32 * kHad2Warps)
hadamard2_kernel(const void* __restrict__ w, uint32_t strips, uint32_t strips_per_band, int64_t ld, int64_t cols,
                 float* __restrict__ d_amax, uint8_t* __restrict__ q, uint8_t* __restrict__ sc,
                 float* __restrict__ d_s2, float* __restrict__ out, uint32_t* __restrict__ d_flags)
{
    __shared__ __align__(16) double tbuf[kHad2Warps][kN][34];
    const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
    double (*T)[34] = tbuf[warp];                                         // rows 16-byte aligned
    float (*Y)[36] = reinterpret_cast<float (*)[36]>(&tbuf[warp][0][0]);   // kN x 36 floats fit
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
    const uint32_t r = kN == 32 ? lane : (lane & 15u);            // this lane's row in the strip
    const uint32_t cb = kN == 32 ? 0u : 16u * (lane >> 4);         // and its first column

    constexpr int kRaw = kN * (kDt == 0 ? 2 : 4) / 16;            // 16-byte loads per lane and strip
    const uint32_t stride = gridDim.x * kHad2Warps;
    auto load = [&](uint32_t st, uint4 raw[kRaw]) {
        const uint32_t band = st / strips_per_band, cs = st - band * strips_per_band;
        const int64_t row = (int64_t)band * kN + r;
        const int64_t col = 32 * (int64_t)cs + cb;
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const char*>(w) +
                                                          (row * ld + col) * (kDt == 0 ? 2 : 4));
#pragma unroll
        for (int k = 0; k < kRaw; ++k) raw[k] = __ldcs(src + k);
    };
    uint4 nxt[kRaw];
    if (blockIdx.x * kHad2Warps + warp < strips) load(blockIdx.x * kHad2Warps + warp, nxt);
    for (uint32_t st = blockIdx.x * kHad2Warps + warp; st < strips; st += stride) {
        const uint32_t band = st / strips_per_band, cs = st - band * strips_per_band;
        const int64_t row = (int64_t)band * kN + r;
        const int64_t col = 32 * (int64_t)cs + cb;
        uint4 raw[kRaw];
#pragma unroll
        for (int k = 0; k < kRaw; ++k) raw[k] = nxt[k];
        if (st + stride < strips) load(st + stride, nxt);         // the next strip's loads in flight
        double v[kN];
#pragma unroll
        for (int k = 0; k < kRaw; ++k) {
            const uint32_t u[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
            if constexpr (kDt == 0) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    v[8 * k + 2 * j] = (double)bf16_lo(u[j]);
                    v[8 * k + 2 * j + 1] = (double)bf16_hi(u[j]);
                }
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) v[4 * k + j] = (double)__uint_as_float(u[j]);
            }
        }
        fwht_regs<kN>(v);                                          // row transform: B H
#pragma unroll
        for (int j = 0; j < kN; j += 2)
            *reinterpret_cast<double2*>(&T[r][cb + j]) = make_double2(v[j], v[j + 1]);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < kN; ++i) v[i] = T[i][lane];            // column `lane` of the strip
        __syncwarp();
        fwht_regs<kN>(v);                                          // column transform: H (B H)
#pragma unroll
        for (int i = 0; i < kN; ++i) Y[i][lane] = (float)(v[i] * (1.0 / kN));   // exact scaling, one rounding
        __syncwarp();
        float y[kN];
        uint32_t ab = 0u;
#pragma unroll
        for (int j = 0; j < kN; j += 4) {
            const float4 f4 = *reinterpret_cast<const float4*>(&Y[r][cb + j]);
            y[j] = f4.x; y[j + 1] = f4.y; y[j + 2] = f4.z; y[j + 3] = f4.w;
        }
#pragma unroll
        for (int j = 0; j < kN; ++j) ab = max(ab, __float_as_uint(y[j]) & 0x7FFFFFFFu);
        __syncwarp();                                              // before the next strip reuses T
        if (ab >= 0x7F800000u) flags |= kFlagNonFinite;

        if constexpr (kMode == 0) {
            if (ab <= 0x7F800000u) mx_bits = max(mx_bits, ab);
        } else if constexpr (kMode == 3) {
            float4* dst = reinterpret_cast<float4*>(out + row * cols + col);
#pragma unroll
            for (int k = 0; k < kN / 4; ++k) __stcs(dst + k, make_float4(y[4 * k], y[4 * k + 1], y[4 * k + 2], y[4 * k + 3]));
        } else if constexpr (kMode == 1) {
            uint32_t bm = ab;
            if constexpr (kN == 16) bm = max(bm, __shfl_xor_sync(0xFFFFFFFFu, bm, 16));   // the row's other half
            const uint32_t code = mx_block_code(bm);
            uint32_t wv[kN / 8];
            mx_encode<kN>(y, code, wv);
            uint8_t* qd = q + row * (cols / 2) + col / 2;
            if constexpr (kN == 32) __stcs(reinterpret_cast<uint4*>(qd), make_uint4(wv[0], wv[1], wv[2], wv[3]));
            else __stcs(reinterpret_cast<uint2*>(qd), make_uint2(wv[0], wv[1]));
            if (cb == 0u) sc[row * (cols / 32) + col / 32] = (uint8_t)code;
        } else {
            uint32_t wv[kN / 8], codes = 0u;
#pragma unroll
            for (int hb = 0; hb < kN / 16; ++hb)
                codes |= nv_block16(y + 16 * hb, s2, k_lo, k_hi, fast_scale, wv + 2 * hb) << (8 * hb);
            uint8_t* qd = q + row * (cols / 2) + col / 2;
            if constexpr (kN == 32) {
                __stcs(reinterpret_cast<uint4*>(qd), make_uint4(wv[0], wv[1], wv[2], wv[3]));
                *reinterpret_cast<uint16_t*>(sc + row * (cols / 16) + col / 16) = (uint16_t)codes;
            } else {
                __stcs(reinterpret_cast<uint2*>(qd), make_uint2(wv[0], wv[1]));
                sc[row * (cols / 16) + col / 16] = (uint8_t)codes;
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

cudaError_t launch_hadamard2(int mode, const void* w, int dt, int64_t rows, int64_t cols, int64_t ld, int n,
                             float* d_amax, uint8_t* q, uint8_t* sc, float* d_s2, float* out, uint32_t* d_flags,
                             cudaStream_t s)
{
    const uint32_t spb = (uint32_t)(cols / 32);                 // strips per band of n rows
    const uint32_t strips = (uint32_t)(rows / n) * spb;
    const int64_t need = ((int64_t)strips + kHad2Warps - 1) / kHad2Warps;
    const int64_t cap = (int64_t)num_sms() * 8;
    const int grid = (int)(need < cap ? (need > 0 ? need : 1) : cap);
#define NV4_H2(M, N, D) hadamard2_kernel<M, N, D><<<grid, 32 * kHad2Warps, 0, s>>>(w, strips, spb, ld, cols, d_amax, q, \
                                                                                 sc, d_s2, out, d_flags)
#define NV4_H2_ND(M) do { if (n == 16) { if (dt == 0) NV4_H2(M, 16, 0); else NV4_H2(M, 16, 2); } \
                          else { if (dt == 0) NV4_H2(M, 32, 0); else NV4_H2(M, 32, 2); } } while (0)
    if (mode == 0) NV4_H2_ND(0);
    else if (mode == 1) NV4_H2_ND(1);
    else if (mode == 2) NV4_H2_ND(2);
    else NV4_H2_ND(3);
#undef NV4_H2_ND
#undef NV4_H2
    return cudaGetLastError();
}

}  // namespace nv4
