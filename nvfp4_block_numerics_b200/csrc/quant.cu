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

// Jobs: one or more tensors, each split into tiles of kAmaxTile 16-byte vectors; a
// tile belongs to one job, and a CTA strides over the tiles of all jobs (so the grid
// sweeps one region of memory at a time).  A CTA keeps a running maximum while its
// tiles stay in one job and folds it into that job's amax when the job changes.
constexpr int kAmaxThreads = 512;
constexpr uint32_t kAmaxVec = 4;                                // vectors per thread per tile
constexpr uint32_t kAmaxTile = kAmaxThreads * kAmaxVec;

struct AmaxJobDev {
    const uint4* x;
    const void* tail;                                           // the n % (elements per vector) last ones
    int64_t nvec;
    int ntail;
    float* d_amax;
    uint32_t tile_begin, tile_end;
};

struct AmaxParams {
    int n;
    uint32_t tiles;
    uint32_t* d_flags;
    AmaxJobDev jobs[kMaxActJobs];
};

// The job holding tile t (jobs are ordered by their first tile and own at least one).
template <class P>
__device__ __forceinline__ int job_of_tile(const P& p, uint32_t t)
{
    int lo = 0, hi = p.n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.jobs[mid].tile_begin <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Largest magnitude of a 16-byte vector as an FP32 bit pattern (NaN patterns included:
// they sort above +Inf); kDt 0: eight BF16, 2: four FP32.
template <int kDt>
__device__ __forceinline__ uint32_t vec_absmax(const uint4& v)
{
    if constexpr (kDt == 0) {
        const uint32_t m = absmax_bf16x8(v);
        return max(m & 0xFFFFu, m >> 16) << 16;
    } else {
        return max(max(v.x & 0x7FFFFFFFu, v.y & 0x7FFFFFFFu), max(v.z & 0x7FFFFFFFu, v.w & 0x7FFFFFFFu));
    }
}

template <int kDt>
__device__ __forceinline__ uint32_t vec_absmax_no_nan(const uint4& v)
{
    if constexpr (kDt == 0) {
        return absmax_bf16x8_no_nan(v) << 16;
    } else {
        const uint32_t w[4] = {v.x & 0x7FFFFFFFu, v.y & 0x7FFFFFFFu, v.z & 0x7FFFFFFFu, v.w & 0x7FFFFFFFu};
        uint32_t m = 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (w[j] <= 0x7F800000u) m = max(m, w[j]);
        return m;
    }
}

template <int kDt>
__device__ __forceinline__ uint32_t tail_abs(const void* tail, int i)
{
    if constexpr (kDt == 0) return (uint32_t)(static_cast<const uint16_t*>(tail)[i] & 0x7FFFu) << 16;
    else return static_cast<const uint32_t*>(tail)[i] & 0x7FFFFFFFu;
}

__device__ __forceinline__ void amax_fold(float* d_amax, uint32_t m, uint32_t* red)
{
    m = block_max_u32<kAmaxThreads>(m, red);
    if (threadIdx.x == 0 && m != 0u) atomicMax(reinterpret_cast<unsigned int*>(d_amax), m);
    __syncthreads();                                            // red is reused by the next fold
}

template <int kDt>
__global__ void __launch_bounds__(kAmaxThreads)
amax_kernel(const __grid_constant__ AmaxParams p)
{
    __shared__ uint32_t red[kAmaxThreads / 32];
    int cur = -1;                                               // job of the running maximum (CTA-uniform)
    uint32_t m = 0u, flags = 0u;
    for (uint32_t t = blockIdx.x; t < p.tiles; t += gridDim.x) {
        const int j = job_of_tile(p, t);
        if (j != cur) {
            if (cur >= 0) amax_fold(p.jobs[cur].d_amax, m, red);
            cur = j;
            m = 0u;
        }
        const AmaxJobDev& job = p.jobs[j];
        const int64_t base = (int64_t)(t - job.tile_begin) * kAmaxTile + threadIdx.x;
        uint4 v[kAmaxVec];
#pragma unroll
        for (uint32_t k = 0; k < kAmaxVec; ++k) {                 // four independent loads in flight
            const int64_t i = base + k * kAmaxThreads;
            v[k] = i < job.nvec ? __ldcs(job.x + i) : make_uint4(0u, 0u, 0u, 0u);
        }
        const bool tail = t + 1u == job.tile_end && (int)threadIdx.x < job.ntail;
        uint32_t tm = tail ? tail_abs<kDt>(job.tail, threadIdx.x) : 0u;
#pragma unroll
        for (uint32_t k = 0; k < kAmaxVec; ++k) tm = max(tm, vec_absmax<kDt>(v[k]));
        if (tm >= 0x7F800000u) {
            flags |= kFlagNonFinite;
            if (tm > 0x7F800000u) {                             // a NaN: these elements again without NaN entries
                tm = 0u;
                if (tail) {
                    const uint32_t a = tail_abs<kDt>(job.tail, threadIdx.x);
                    if (a <= 0x7F800000u) tm = a;
                }
#pragma unroll
                for (uint32_t k = 0; k < kAmaxVec; ++k) tm = max(tm, vec_absmax_no_nan<kDt>(v[k]));
            }
        }
        m = max(m, tm);
    }
    if (cur >= 0) amax_fold(p.jobs[cur].d_amax, m, red);
    flags = __reduce_or_sync(0xFFFFFFFFu, flags);
    if ((threadIdx.x & 31) == 0 && flags) flag_or(p.d_flags, flags);
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

// Block quantizer over one or more [rows, cols] tensors (jobs): one thread per 16-block.
// Tiles of kActThreads blocks belong to one job; a CTA takes every gridDim.x-th tile of
// the concatenation (job by job, the job's fields and per-tensor constants -- s2 and
// its brackets -- in registers) with the next block's loads in flight while the
// current one is quantized.
// kIn: 0 BF16, 2 FP32 input.  kOut: -1 writes packed codes + E4M3 scales; 0/1/2 writes
// the fake quantize-dequantize values as BF16/FP16/FP32 (leading dimension ld_out).
// Every block is read and written by the same thread, read first, so out may alias x.
struct QuantJobDev {
    const void* x;
    void* out;
    uint8_t* q;
    uint8_t* scales;
    const float* d_amax;
    float* d_s2;
    int64_t ld, ld_out;
    FastDiv div_bpr;
    uint32_t bpr, units, tile_begin;
};

struct QuantParams {
    int n;
    uint32_t tiles;
    uint32_t* d_flags;
    QuantJobDev jobs[kMaxActJobs];
};

template <int kIn, int kOut>
__global__ void __launch_bounds__(kActThreads)
act_quant_kernel(const __grid_constant__ QuantParams p)
{
    __shared__ E4M3Tables tab;
    fill_e4m3_tables(tab);
    __syncthreads();

    uint32_t flags = 0u;
    const uint32_t G = gridDim.x;
    // jobs in order; within a job the CTA takes the tiles t = blockIdx.x (mod G), with the
    // job's fields and constants in registers and the next block's loads in flight
    for (int j = 0; j < p.n; ++j) {
        const void* x = p.jobs[j].x;
        const int64_t ld = p.jobs[j].ld;
        const uint32_t bpr = p.jobs[j].bpr, units = p.jobs[j].units, tb = p.jobs[j].tile_begin;
        const FastDiv div_bpr = p.jobs[j].div_bpr;
        uint8_t* const q = p.jobs[j].q;
        uint8_t* const scales = p.jobs[j].scales;
        void* const out = p.jobs[j].out;
        const int64_t ld_out = p.jobs[j].ld_out;
        const uint32_t t0 = tb + (blockIdx.x + G - tb % G) % G;     // first tile of this CTA in the job
        uint32_t u = (t0 - tb) * kActThreads + threadIdx.x;
        if ((t0 - tb) * kActThreads >= units) continue;            // (CTA-uniform)
        auto offset = [&](uint32_t uu, int64_t l) {
            const uint32_t r = div_bpr.div(uu), bb = uu - r * bpr;
            return (int64_t)r * l + 16 * (int64_t)bb;
        };

        const float s2 = __fdiv_rn(*p.jobs[j].d_amax, 2688.0f);  // RN32(amax / (6*448))
        if (t0 == tb && threadIdx.x == 0) *p.jobs[j].d_s2 = s2;
        const bool fast_scale = s2 >= kTinyScale && s2 <= 0x1p100f;
        const float k = __frcp_rn(__fmul_rn(6.0f, s2));           // ~ 1/(6*s2)
        const float k_lo = __fmul_rn(k, kLoMargin), k_hi = __fmul_rn(k, kHiMargin);
        const float rs2 = __frcp_rn(s2);                          // ~ 1/s2
        if (!isfinite(s2)) flags |= kFlagOverflow;

        const uint32_t stride = G * kActThreads;
        BlockIn<kIn> nxt;
        if (u < units) load_block_in<kIn>(x, offset(u, ld), nxt);
        for (; u < units; u += stride) {
            const BlockIn<kIn> blk = nxt;
            if (u + stride < units) load_block_in<kIn>(x, offset(u + stride, ld), nxt);
            float xv[16];
            const uint32_t ab = unpack_block<kIn>(blk, xv);
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
            code &= 0x7Fu;                                        // non-negative inputs only
            const float S = __fmul_rn(tab.dec[code], s2);        // DQ1: RN32(s_b * s2)

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
    }
    flags = __reduce_or_sync(0xFFFFFFFFu, flags);
    if ((threadIdx.x & 31) == 0 && flags) flag_or(p.d_flags, flags);
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

// Jobs: tiles of kDeqTile half-blocks, each in one job; a CTA strides over the tiles of
// all jobs, four half-blocks per thread in flight.
constexpr uint32_t kDeqTile = kActThreads * 4;

struct DeqJobDev {
    const uint32_t* qw;
    const uint8_t* scales;
    const float* d_s2;
    void* out;
    uint32_t halves, tile_begin;
};

struct DeqParams {
    int n;
    uint32_t tiles;
    DeqJobDev jobs[kMaxActJobs];
};

template <int kOut>   // 0 bf16, 1 fp16, 2 fp32
__global__ void __launch_bounds__(kActThreads)
dequant_kernel(const __grid_constant__ DeqParams p)
{
    int cur = -1;
    float s2 = 0.0f;
    for (uint32_t t = blockIdx.x; t < p.tiles; t += gridDim.x) {
        const int j = job_of_tile(p, t);
        const DeqJobDev& job = p.jobs[j];
        if (j != cur) {
            cur = j;
            s2 = *job.d_s2;
        }
        const uint32_t base = (t - job.tile_begin) * kDeqTile + threadIdx.x;
        uint32_t a[4], c[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {                             // four independent steps in flight
            const uint32_t h = base + k * kActThreads;
            if (h < job.halves) {
                a[k] = __ldcs(job.qw + h);
                c[k] = job.scales[h >> 1];
            }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t h = base + k * kActThreads;
            if (h < job.halves) dequant8<kOut>(a[k], c[k], s2, job.out, h);
        }
    }
}

// ============================================================== launchers
static int grid_for(int64_t work, int per_sm)
{
    const int64_t cap = (int64_t)num_sms() * per_sm;
    return (int)(work < cap ? (work > 0 ? work : 1) : cap);
}

cudaError_t launch_amax(const AmaxTask* tasks, int n, int dt, uint32_t* d_flags, cudaStream_t s)
{
    AmaxParams p;
    p.d_flags = d_flags;
    const int64_t per_vec = dt == 0 ? 8 : 4;                    // elements per 16-byte vector
    int m = 0;
    uint32_t tiles = 0;
    for (int i = 0; i < n; ++i) {
        const AmaxTask& T = tasks[i];
        if (T.n == 0) continue;
        AmaxJobDev& d = p.jobs[m++];
        d.x = static_cast<const uint4*>(T.x);
        d.nvec = T.n / per_vec;
        d.ntail = (int)(T.n - d.nvec * per_vec);
        d.tail = static_cast<const char*>(T.x) + d.nvec * 16;
        d.d_amax = T.d_amax;
        d.tile_begin = tiles;
        const int64_t nt = (d.nvec + kAmaxTile - 1) / kAmaxTile;
        tiles += (uint32_t)(nt > 0 ? nt : 1);
        d.tile_end = tiles;
    }
    p.n = m;
    p.tiles = tiles;
    if (m == 0) return cudaSuccess;
    const int g = grid_for(tiles, 4);
    if (dt == 0) amax_kernel<0><<<g, kAmaxThreads, 0, s>>>(p);
    else amax_kernel<2><<<g, kAmaxThreads, 0, s>>>(p);
    return cudaGetLastError();
}

struct ScaleOnlyParams {
    int n;
    float divisor;
    uint32_t* d_flags;
    const float* d_amax[kMaxActJobs];
    float* d_out[kMaxActJobs];
};

__global__ void __launch_bounds__(kMaxActJobs)
scale_only_kernel(const __grid_constant__ ScaleOnlyParams p)
{
    const int i = threadIdx.x;
    if (i >= p.n) return;
    const float s2 = __fdiv_rn(*p.d_amax[i], p.divisor);
    *p.d_out[i] = s2;
    if (!isfinite(s2)) flag_or(p.d_flags, kFlagOverflow);
}

cudaError_t launch_scale_only(const float* const* d_amax, float* const* d_out, int n, float divisor,
                              uint32_t* d_flags, cudaStream_t s)
{
    if (n <= 0) return cudaSuccess;
    ScaleOnlyParams p;
    p.n = n < kMaxActJobs ? n : kMaxActJobs;
    p.divisor = divisor;
    p.d_flags = d_flags;
    for (int i = 0; i < p.n; ++i) {
        p.d_amax[i] = d_amax[i];
        p.d_out[i] = d_out[i];
    }
    scale_only_kernel<<<1, kMaxActJobs, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_block_quant(const QuantTask* tasks, int n, int in_dt, int out_dt, uint32_t* d_flags,
                               cudaStream_t s)
{
    // empty tensors still receive their s2
    const float* e_amax[kMaxActJobs];
    float* e_out[kMaxActJobs];
    int ne = 0;
    for (int i = 0; i < n; ++i)
        if (tasks[i].rows == 0 || tasks[i].cols == 0) {
            e_amax[ne] = tasks[i].d_amax;
            e_out[ne++] = tasks[i].d_s2;
        }
    if (ne > 0) {
        const cudaError_t e = launch_scale_only(e_amax, e_out, ne, 2688.0f, d_flags, s);
        if (e != cudaSuccess) return e;
    }

    QuantParams p;
    p.d_flags = d_flags;
    int m = 0;
    uint32_t tiles = 0;
    for (int i = 0; i < n; ++i) {
        const QuantTask& T = tasks[i];
        if (T.rows == 0 || T.cols == 0) continue;
        QuantJobDev& d = p.jobs[m++];
        d.x = T.x; d.out = T.out; d.q = T.q; d.scales = T.scales; d.d_amax = T.d_amax; d.d_s2 = T.d_s2;
        d.ld = T.ld; d.ld_out = T.ld_out;
        d.bpr = (uint32_t)(T.cols / 16);
        d.div_bpr = FastDiv(d.bpr);
        d.units = (uint32_t)T.rows * d.bpr;
        d.tile_begin = tiles;
        tiles += (d.units + kActThreads - 1) / kActThreads;
    }
    p.n = m;
    p.tiles = tiles;
    if (m == 0) return cudaSuccess;
    const int g = grid_for(tiles, 8);
#define NV4_BQ(I, O) act_quant_kernel<I, O><<<g, kActThreads, 0, s>>>(p)
    if (in_dt == 0) {
        if (out_dt < 0) NV4_BQ(0, -1); else if (out_dt == 0) NV4_BQ(0, 0); else if (out_dt == 1) NV4_BQ(0, 1); else NV4_BQ(0, 2);
    } else {
        if (out_dt < 0) NV4_BQ(2, -1); else if (out_dt == 0) NV4_BQ(2, 0); else if (out_dt == 1) NV4_BQ(2, 1); else NV4_BQ(2, 2);
    }
#undef NV4_BQ
    return cudaGetLastError();
}

cudaError_t launch_dequant(const DequantTask* tasks, int n, int out_dt, cudaStream_t s)
{
    DeqParams p;
    int m = 0;
    uint32_t tiles = 0;
    for (int i = 0; i < n; ++i) {
        const DequantTask& T = tasks[i];
        if (T.rows == 0 || T.cols == 0) continue;
        DeqJobDev& d = p.jobs[m++];
        d.qw = reinterpret_cast<const uint32_t*>(T.q);
        d.scales = T.scales;
        d.d_s2 = T.d_s2;
        d.out = T.out;
        d.halves = (uint32_t)(2 * T.rows * (T.cols / 16));
        d.tile_begin = tiles;
        tiles += (d.halves + kDeqTile - 1) / kDeqTile;
    }
    p.n = m;
    p.tiles = tiles;
    if (m == 0) return cudaSuccess;
    const int g = grid_for(tiles, 8);
    if (out_dt == 0) dequant_kernel<0><<<g, kActThreads, 0, s>>>(p);
    else if (out_dt == 1) dequant_kernel<1><<<g, kActThreads, 0, s>>>(p);
    else dequant_kernel<2><<<g, kActThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace nv4
