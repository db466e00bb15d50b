// cast.cu -- closed-form MXFP4 -> NVFP4 cast (sm_100a).
//
// [CAST] section 2; [DSPARK] stage 3 (see nv4.h).  Per matrix:
//   k_max = max_j (e8m0_j - 127);  m = k_max - 8;  s2 = 2^m;  global_amax = 6*448*2^m
//   MX block j with d = k_max - k_j <= 17: both NVFP4 scales encode 2^(k_j - m) = 2^(8-d)
//   exactly in E4M3 and the 16 nibble bytes are reused; otherwise the block is
//   re-quantized from its exact values e2m1 * 2^k_j (rare fallback path).
//
// Two stream-ordered kernels, no scratch memory:
//  1. cast_kmax_kernel: one thread-block cluster of kKmaxCluster CTAs per scale_2 set (a
//     matrix, or a group of matrices sharing one scale_2, [CAST] section 3) reads only
//     the E8M0 bytes, reduces the largest valid code through distributed shared memory
//     and writes every member's outputs s2 = 2^m and global_amax = 6*448*2^m;
//  2. cast_rewrite_kernel: one resident wave of warps striding over 256-block tiles
//     (lane-interleaved so each instruction moves contiguous bytes).  It recovers k_max
//     = m + 8 exactly from the s2 it reads back, writes the two E4M3 scale bytes per
//     block and, out of place, copies the 16 nibble bytes with 128-bit streaming loads
//     and stores; rare blocks (NaN code, outside the window) are handled by the whole
//     warp, one element per lane.  Launched as a programmatic dependent of kernel 1, it
//     copies the nibbles of each warp's first tiles while kernel 1 runs, then waits for
//     kernel 1.
#include "nv4_async.cuh"
#include "nv4_common.cuh"
#include "nv4_internal.h"

namespace nv4 {

constexpr int kKmaxThreads = 512;
constexpr int kKmaxCluster = 8;                  // CTAs reducing one matrix's largest E8M0 code

struct CastJobDev {
    const uint8_t* mx_q;
    const uint8_t* e8m0;
    uint8_t* nv_q;
    uint8_t* nv_scales;
    float* d_ga;
    float* d_s2;
    uint32_t nb;                                  // MX blocks in the matrix (rows * cols / 32)
    uint32_t tile_begin;                         // prefix sum of kTile-block tiles over jobs
};

struct CastParams {
    int n;
    int n_sets;                                   // scale_2 groups (sets of jobs sharing k_max)
    uint16_t set_begin[kMaxCastJobs + 1];         // members of set g: set_jobs[set_begin[g] .. set_begin[g+1])
    uint16_t set_jobs[kMaxCastJobs];
    uint32_t tiles;                               // total kTile-block tiles over all jobs
    unsigned long long* d_counts;
    uint32_t* d_flags;
    CastJobDev jobs[kMaxCastJobs];
};


// 2^e as FP32 for e in [-149, 127] (exact; subnormal below -126).
__device__ __forceinline__ float exp2_exact(int e)
{
    return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(1u << (e + 149));
}

// E4M3 code of 2^E for E in [-9, 8].
__device__ __forceinline__ uint32_t e4m3_code_pow2(int E)
{
    return E >= -6 ? (uint32_t)(E + 7) << 3 : 1u << (E + 9);
}

// Value of E2M1 code c (sign in bit 3) times 2^k, exact in FP32 for k >= -127.
__device__ __forceinline__ float e2m1_times_pow2(uint32_t c, int k)
{
    const uint32_t mag = c & 7u;
    const float v = mag < 2u ? 0.5f * (float)mag
                             : __uint_as_float(((126u + (mag >> 1)) << 23) | ((mag & 1u) << 22));
    const float r = v * exp2_exact(k);                    // power-of-two scaling: exact
    return (c & 8u) ? -r : r;
}

// One rare MX block g (E8M0 code c; arguments warp-uniform), handled by the whole warp:
// lanes 0-15 take the first 16-element half, lanes 16-31 the second, one element per
// lane.  A NaN code copies the nibbles (out of place) and writes zero scales.  Otherwise
// each half is re-quantized from its exact values e2m1 * 2^k with the activation-
// quantizer rules: block amax a_b, scale code = nearest E4M3 to a_b/(6*s2), codes =
// nearest E2M1 to w/S with S = RN32(s_b * s2).  Both roundings take the FP32 bracket
// (hardware conversion of both ends, an exact FMA comparison when they disagree);
// scales outside [2^-100, 2^100] take the exact FP64 encoders.  Every lane reads its
// source byte before any lane writes, so nv_q may equal mx_q.
__device__ __noinline__ void cast_rare_warp(const uint8_t* mx_q, uint8_t* nv_q, uint8_t* nv_scales, uint32_t g,
                                            uint32_t c, float s2, bool copy, uint32_t lane, uint32_t* n_fb,
                                            uint32_t* n_ll)
{
    const uint32_t h = lane >> 4, e = lane & 15u;
    const size_t at = (size_t)16 * g + 8u * h + (e >> 1);
    const uint32_t byte = mx_q[at];
    if (c == 0xFFu) {
        if (copy && (e & 1u) == 0u) nv_q[at] = (uint8_t)byte;
        if (lane == 0u) reinterpret_cast<uint16_t*>(nv_scales)[g] = 0;
        return;
    }
    const float w = e2m1_times_pow2((byte >> (4u * (e & 1u))) & 15u, (int)c - 127);
    uint32_t ab = __float_as_uint(w) & 0x7FFFFFFFu;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) ab = max(ab, __shfl_xor_sync(0xFFFFFFFFu, ab, o));   // within the half
    const float a_b = __uint_as_float(ab);

    uint32_t code;                                              // nearest E4M3 to a_b / (6*s2)
    if (s2 >= kTinyScale && s2 <= 0x1p100f) {
        const float kk = __frcp_rn(__fmul_rn(6.0f, s2));
        const uint32_t cc = cvt_e4m3x2(__fmul_rn(a_b, __fmul_rn(kk, kLoMargin)), __fmul_rn(a_b, __fmul_rn(kk, kHiMargin)));
        code = cc & 0xFFu;
        if (code != (cc >> 8)) code = e4m3_fix(code, a_b, s2);
        code &= 0x7Fu;
    } else {
        code = e4m3_code_exact(a_b, s2);
    }
    const float S = __fmul_rn(e4m3_value(code), s2);           // DQ1: RN32(s_b * s2)

    uint32_t q;                                                 // nearest E2M1 to w / S
    if (S == 0.0f) {
        q = (__float_as_uint(w) >> 28) & 8u;                    // sign only
    } else if (S >= kTinyScale && S <= 0x1p100f) {
        const float r = __frcp_rn(S);
        const uint32_t cc = cvt_e2m1x2(__fmul_rn(w, __fmul_rn(r, kLoMargin)), __fmul_rn(w, __fmul_rn(r, kHiMargin)));
        q = cc & 15u;
        if (q != (cc >> 4)) {                                   // near a rounding boundary
            const uint32_t kl = q & 7u;
            const float d = fmaf(e2m1_boundary(kl), S, -fabsf(w));
            const uint32_t k = d < 0.0f ? kl + 1u : (d > 0.0f ? kl : kl + (kl & 1u));
            q = k | (q & 8u);
        }
    } else {
        q = e2m1_code_exact(w, S);
    }
    // lossless: the NVFP4 value of every element equals its MXFP4 value
    const uint32_t mag = q & 7u;
    const float v = mag < 2u ? 0.5f * (float)mag : __uint_as_float(((126u + (mag >> 1)) << 23) | ((mag & 1u) << 22));
    const float y = __fmul_rn((q & 8u) ? -v : v, S);
    const uint32_t same = __ballot_sync(0xFFFFFFFFu, __float_as_uint(y) == __float_as_uint(w));
    const uint32_t partner = __shfl_xor_sync(0xFFFFFFFFu, q, 1);
    if ((e & 1u) == 0u) nv_q[at] = (uint8_t)(q | (partner << 4));
    if (e == 0u) nv_scales[(size_t)2 * g + h] = (uint8_t)code;
    if (lane == 0u) {
        *n_fb += 2u;
        *n_ll += ((same & 0xFFFFu) == 0xFFFFu ? 1u : 0u) + ((same >> 16) == 0xFFFFu ? 1u : 0u);
    }
}

// ------------------------------------------------------------------ kernel 1: k_max
__global__ void __launch_bounds__(kKmaxThreads)
cast_kmax_kernel(const __grid_constant__ CastParams p)
{
    __shared__ uint32_t red[kKmaxThreads / 32];
    __shared__ uint32_t cta_max;
    // the rewrite kernel may start its set-up and first loads now; it waits for this
    // grid to complete before it reads scale_2
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint32_t rank = cluster_ctarank();
    const int set = blockIdx.x / kKmaxCluster;
    const int m0 = p.set_begin[set], m1 = p.set_begin[set + 1];

    uint32_t mx = 0u, flags = 0u;                                   // four per-byte maxima
    auto scan = [&](const uint4& w) {
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            // bytes equal to 0xFF are NaN codes: flag them and keep them out of the max
            const uint32_t nan = __vcmpeq4(ws[k], 0xFFFFFFFFu);
            if (nan) flags |= kFlagE8M0Nan;
            mx = __vmaxu4(mx, ws[k] & ~nan);
        }
    };
    uint32_t mtail = 0u;                                            // scalar maximum of the tails
    for (int mi = m0; mi < m1; ++mi) {                              // every matrix of the set
        const CastJobDev& job = p.jobs[p.set_jobs[mi]];
        // share of this CTA, 16-aligned so it moves in 16-byte words
        const uint32_t per = ((job.nb + kKmaxCluster - 1) / kKmaxCluster + 15u) & ~15u;
        const uint32_t g0 = min(job.nb, rank * per), g1 = min(job.nb, g0 + per);
        const uint32_t nvec = (g1 - g0) / 16u;
        const uint4* src = reinterpret_cast<const uint4*>(job.e8m0 + g0);
        uint32_t v = threadIdx.x;
        for (; v + 3u * kKmaxThreads < nvec; v += 4u * kKmaxThreads) {  // four loads in flight
            uint4 w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) w[k] = __ldcs(src + v + k * kKmaxThreads);
#pragma unroll
            for (int k = 0; k < 4; ++k) scan(w[k]);
        }
        for (; v < nvec; v += kKmaxThreads) scan(__ldcs(src + v));
        for (uint32_t g = g0 + nvec * 16u + threadIdx.x; g < g1; g += kKmaxThreads) {
            const uint32_t c = job.e8m0[g];
            if (c == 0xFFu) flags |= kFlagE8M0Nan; else mtail = max(mtail, c);
        }
    }
    mx = max(max(max(mx & 0xFFu, (mx >> 8) & 0xFFu), max((mx >> 16) & 0xFFu, mx >> 24)), mtail);
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t m = 0u;
        for (int w = 0; w < kKmaxThreads / 32; ++w) m = max(m, red[w]);
        cta_max = m;
    }
    cluster_sync();
    if (rank == 0 && threadIdx.x < 32) {                           // one warp gathers the partial maxima
        uint32_t c = threadIdx.x < kKmaxCluster ? ld_dsmem_u32(&cta_max, threadIdx.x) : 0u;
        c = __reduce_max_sync(0xFFFFFFFFu, c);
        const float s2 = exp2_exact((int)c - 127 - 8);               // m = k_max - 8 in [-135, 119]
        const float ga = __fmul_rn(2688.0f, s2);                     // 6*448*2^m
        for (int mi = m0 + (int)threadIdx.x; mi < m1; mi += 32) {    // every member gets the set's scale_2
            const CastJobDev& job = p.jobs[p.set_jobs[mi]];
            *job.d_s2 = s2;
            *job.d_ga = ga;
        }
        if (threadIdx.x == 0 && !isfinite(ga)) flags |= kFlagOverflow;
    }
    cluster_sync();                                               // all remote reads done
    flags = __reduce_or_sync(0xFFFFFFFFu, flags);
    if ((threadIdx.x & 31) == 0) flag_or(p.d_flags, flags);
}

// m with s2 = 2^m exactly (s2 a power of two, normal or subnormal).
__device__ __forceinline__ int exact_log2(float s2)
{
    const uint32_t b = __float_as_uint(s2);
    const int e = (int)((b >> 23) & 0xFFu);
    return e != 0 ? e - 127 : -149 + (31 - __clz(b));
}

// ------------------------------------------------------------------ kernel 2: rewrite
// A tile is kTile consecutive MX blocks of one matrix; lane t of a warp takes blocks
// tile + 32i + t (i = 0..7), so every load and store instruction of the warp moves
// contiguous bytes (32 code bytes, 512 nibble bytes, 64 scale bytes).  Warps stride over
// the tiles (warp w takes tiles w, w + W, ...), so at any moment the grid sweeps one
// region of memory.  The nibble copy of a warp's first kPreTiles tiles needs nothing
// from kernel 1: under programmatic dependent launch it runs while kernel 1 is still
// reducing k_max, and the main pass then only writes those tiles' scale bytes.
constexpr uint32_t kTile = 256;
constexpr int kRwThreads = 256;
constexpr int kRwCtasPerSm = 2;
constexpr uint32_t kPreTiles = 3;

// The job holding global tile ti (jobs are ordered by their first tile).
__device__ __forceinline__ int cast_job_of(const CastParams& p, uint32_t ti)
{
    int lo = 0, hi = p.n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.jobs[mid].tile_begin <= ti) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(kRwThreads, kRwCtasPerSm)
cast_rewrite_kernel(const __grid_constant__ CastParams p)
{
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp_id = (blockIdx.x * kRwThreads + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * kRwThreads) >> 5;

    // ---- nibble copy of the first tiles (out of place), before kernel 1 has finished
    {
        uint32_t k = 0u;
        for (uint32_t ti = warp_id; k < kPreTiles && ti < p.tiles; ti += nwarps, ++k) {
            const CastJobDev& job = p.jobs[cast_job_of(p, ti)];
            if (job.nv_q == job.mx_q) continue;
            const uint32_t base = kTile * (ti - job.tile_begin);
            uint4 qv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t g = base + 32u * i + lane;
                if (g < job.nb) qv[i] = __ldcs(reinterpret_cast<const uint4*>(job.mx_q) + g);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t g = base + 32u * i + lane;
                if (g < job.nb) __stcs(reinterpret_cast<uint4*>(job.nv_q) + g, qv[i]);
            }
        }
    }
    // kernel 1's scale_2 values are visible from here on (a no-op without programmatic
    // dependent launch)
    asm volatile("griddepcontrol.wait;" ::: "memory");

    uint32_t n_in = 0u, n_fb = 0u, n_ll = 0u;
    uint32_t k = 0u;
    for (uint32_t ti = warp_id; ti < p.tiles; ti += nwarps, ++k) {
        const CastJobDev& job = p.jobs[cast_job_of(p, ti)];
        const float s2 = *job.d_s2;
        const int k_max = exact_log2(s2) + 8;
        const bool copy = job.nv_q != job.mx_q && k >= kPreTiles;     // nibbles still to copy
        const uint32_t base = kTile * (ti - job.tile_begin);
        uint32_t c[8];
        uint4 qv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t g = base + 32u * i + lane;
            c[i] = g < job.nb ? (uint32_t)__ldcs(job.e8m0 + g) : 0u;
        }
        if (copy) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t g = base + 32u * i + lane;
                if (g < job.nb) qv[i] = __ldcs(reinterpret_cast<const uint4*>(job.mx_q) + g);
            }
        }
        uint32_t rare = 0u;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t g = base + 32u * i + lane;
            if (g >= job.nb) continue;
            const int d = k_max - ((int)c[i] - 127);
            if (c[i] != 0xFFu && d <= 17) {
                const uint32_t e = e4m3_code_pow2(8 - d);
                __stcs(reinterpret_cast<unsigned short*>(job.nv_scales) + g, (unsigned short)(e | (e << 8)));
                if (copy) __stcs(reinterpret_cast<uint4*>(job.nv_q) + g, qv[i]);
                n_in += 2u;
            } else {
                rare |= 1u << i;
            }
        }
        // rare blocks, one at a time by the whole warp; the warp barrier orders every
        // lane's earlier nibble stores (a pre-copied tile) before other lanes rewrite them
        if (__ballot_sync(0xFFFFFFFFu, rare != 0u)) {
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                uint32_t m = __ballot_sync(0xFFFFFFFFu, (rare >> i) & 1u);
                while (m) {
                    const uint32_t L = __ffs(m) - 1u;
                    m &= m - 1u;
                    const uint32_t cL = __shfl_sync(0xFFFFFFFFu, c[i], L);
                    cast_rare_warp(job.mx_q, job.nv_q, job.nv_scales, base + 32u * i + L, cL, s2, copy, lane, &n_fb,
                                   &n_ll);
                }
            }
        }
    }
    // counters: one set of atomics per warp, no CTA barrier (warps retire independently)
    n_ll += n_in;                                                    // in-window blocks are lossless
    n_in = __reduce_add_sync(0xFFFFFFFFu, n_in);
    n_fb = __reduce_add_sync(0xFFFFFFFFu, n_fb);
    n_ll = __reduce_add_sync(0xFFFFFFFFu, n_ll);
    if (lane == 0 && p.d_counts != nullptr) {
        if (n_in) atomicAdd(p.d_counts + 0, (unsigned long long)n_in);
        if (n_fb) atomicAdd(p.d_counts + 1, (unsigned long long)n_fb);
        if (n_ll) atomicAdd(p.d_counts + 2, (unsigned long long)n_ll);
    }
}

cudaError_t launch_cast(const nv4_cast_job* jobs, int n, unsigned long long* d_counts, uint32_t* d_flags,
                        cudaStream_t s)
{
    CastParams p;
    p.d_counts = d_counts;
    p.d_flags = d_flags;
    int m = 0;
    uint32_t tiles = 0;
    for (int i = 0; i < n; ++i) {
        const nv4_cast_job& J = jobs[i];
        if (J.rows == 0 || J.cols == 0) continue;
        CastJobDev& d = p.jobs[m++];
        d.mx_q = J.mx_q; d.e8m0 = J.e8m0; d.nv_q = J.nv_q; d.nv_scales = J.nv_scales;
        d.d_ga = J.d_global_amax; d.d_s2 = J.d_s2;
        d.nb = (uint32_t)(J.rows * (J.cols / 32));
        d.tile_begin = tiles;
        tiles += (d.nb + kTile - 1u) / kTile;
    }
    p.n = m;
    p.tiles = tiles;
    if (m == 0) return cudaSuccess;
    // scale_2 sets: jobs with the same non-negative group id share one k_max
    {
        int order[kMaxCastJobs];
        int32_t gid[kMaxCastJobs];
        int mm = 0;
        for (int i = 0; i < n; ++i)
            if (jobs[i].rows != 0 && jobs[i].cols != 0) gid[mm++] = jobs[i].group;
        bool taken[kMaxCastJobs] = {};
        int k = 0, sets = 0;
        for (int i = 0; i < m; ++i) {
            if (taken[i]) continue;
            p.set_begin[sets++] = (uint16_t)k;
            order[k++] = i;
            taken[i] = true;
            if (gid[i] < 0) continue;
            for (int j = i + 1; j < m; ++j)
                if (!taken[j] && gid[j] == gid[i]) { order[k++] = j; taken[j] = true; }
        }
        p.set_begin[sets] = (uint16_t)k;
        p.n_sets = sets;
        for (int i = 0; i < m; ++i) p.set_jobs[i] = (uint16_t)order[i];
    }

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.n_sets * kKmaxCluster), 1, 1);
    cfg.blockDim = dim3(kKmaxThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kKmaxCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, cast_kmax_kernel, p);
    if (e != cudaSuccess) return e;

    // a single resident wave, launched as a programmatic dependent of the k_max kernel
    // so that its first loads overlap that kernel; it waits for the k_max results
    // before using them
    const uint64_t warps_needed = tiles;            // one warp per tile at most
    const uint64_t cap = (uint64_t)num_sms() * kRwCtasPerSm;
    const uint64_t need = (warps_needed + kRwThreads / 32 - 1) / (kRwThreads / 32);
    const int grid = (int)(need < cap ? need : cap);
    cudaLaunchConfig_t cfg2 = {};
    cfg2.gridDim = dim3((unsigned)grid, 1, 1);
    cfg2.blockDim = dim3(kRwThreads, 1, 1);
    cfg2.dynamicSmemBytes = 0;
    cfg2.stream = s;
    cudaLaunchAttribute attr2[1];
    attr2[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr2[0].val.programmaticStreamSerializationAllowed = 1;
    cfg2.attrs = attr2;
    cfg2.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg2, cast_rewrite_kernel, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace nv4
