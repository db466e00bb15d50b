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
//  2. cast_rewrite_kernel: a flat grid over the MX blocks of every matrix (a warp takes
//     256 consecutive blocks per step, lane-interleaved so each instruction moves
//     contiguous bytes) recovers k_max = m + 8 exactly from the s2 it reads back, writes
//     the two E4M3 scale bytes per block and, out of place, copies the 16 nibble bytes
//     with 128-bit streaming loads and stores; rare blocks (NaN code, outside the
//     window) take a separate exact path.
#include "nv4_common.cuh"
#include "nv4_internal.h"

namespace nv4 {

constexpr int kCastThreads = 256;
constexpr int kKmaxCluster = 8;                  // CTAs reducing one matrix's largest E8M0 code

struct CastJobDev {
    const uint8_t* mx_q;
    const uint8_t* e8m0;
    uint8_t* nv_q;
    uint8_t* nv_scales;
    float* d_ga;
    float* d_s2;
    uint32_t nb;                                  // MX blocks in the matrix (rows * cols / 32)
    uint32_t group_begin;                         // prefix sum of 256-block tiles over jobs
};

struct CastParams {
    int n;
    int n_sets;                                   // scale_2 groups (sets of jobs sharing k_max)
    uint16_t set_begin[kMaxCastJobs + 1];         // members of set g: set_jobs[set_begin[g] .. set_begin[g+1])
    uint16_t set_jobs[kMaxCastJobs];
    uint32_t groups;                              // total 256-block tiles
    unsigned long long* d_counts;
    uint32_t* d_flags;
    CastJobDev jobs[kMaxCastJobs];
};

__device__ __forceinline__ uint32_t cluster_rank_c()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_c()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t ld_dsmem_u32(const uint32_t* local, uint32_t rank)
{
    uint32_t remote, v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
                 : "=r"(remote)
                 : "r"((uint32_t)__cvta_generic_to_shared(local)), "r"(rank));
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(remote) : "memory");
    return v;
}

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

// Re-quantizes one 16-element half of an MX block outside the window.  Returns the
// E4M3 code, writes the packed nibbles to out[2], and sets *lossless.
__device__ __noinline__ uint32_t cast_fallback16(const uint32_t nib_words[2], int k, float s2,
                                                 uint32_t out[2], uint32_t* lossless)
{
    float w[16];
    float a_b = 0.0f;
    for (int i = 0; i < 16; ++i) {
        w[i] = e2m1_times_pow2((nib_words[i >> 3] >> (4 * (i & 7))) & 15u, k);
        a_b = fmaxf(a_b, fabsf(w[i]));
    }
    const uint32_t code = e4m3_code_exact(a_b, s2);
    const float S = __fmul_rn(e4m3_value(code), s2);
    out[0] = out[1] = 0u;
    uint32_t same = 1u;
    for (int i = 0; i < 16; ++i) {
        const uint32_t c = e2m1_code_exact(w[i], S);
        out[i >> 3] |= c << (4 * (i & 7));
        const uint32_t mag = c & 7u;
        const float v = mag < 2u ? 0.5f * (float)mag
                                 : __uint_as_float(((126u + (mag >> 1)) << 23) | ((mag & 1u) << 22));
        const float y = __fmul_rn((c & 8u) ? -v : v, S);
        if (__float_as_uint(y) != __float_as_uint(w[i])) same = 0u;
    }
    *lossless = same;
    return code;
}

// A block whose E8M0 code is NaN (nibbles copied, scales 0; flagged in phase 1) or lies
// outside the window (re-quantized).  Returns the two scale bytes; adds to the fallback
// and lossless counters.
__device__ __noinline__ uint32_t cast_rare_block(const uint8_t* __restrict__ mx_q, uint8_t* __restrict__ nv_q,
                                                 uint32_t g, uint32_t c, int k_max, float s2, bool copy,
                                                 uint32_t* n_fb, uint32_t* n_ll)
{
    const uint4 qv = *reinterpret_cast<const uint4*>(mx_q + (int64_t)g * 16);
    if (c == 0xFFu) {
        if (copy) *reinterpret_cast<uint4*>(nv_q + (int64_t)g * 16) = qv;
        return 0u;
    }
    const int k = (int)c - 127;
    const uint32_t lo_words[2] = {qv.x, qv.y}, hi_words[2] = {qv.z, qv.w};
    uint32_t out_lo[2], out_hi[2], ll0, ll1;
    const uint32_t s_lo = cast_fallback16(lo_words, k, s2, out_lo, &ll0);
    const uint32_t s_hi = cast_fallback16(hi_words, k, s2, out_hi, &ll1);
    *reinterpret_cast<uint4*>(nv_q + (int64_t)g * 16) = make_uint4(out_lo[0], out_lo[1], out_hi[0], out_hi[1]);
    *n_fb += 2u;
    *n_ll += ll0 + ll1;
    return s_lo | (s_hi << 8);
}

// ------------------------------------------------------------------ kernel 1: k_max
__global__ void __launch_bounds__(kCastThreads)
cast_kmax_kernel(const __grid_constant__ CastParams p)
{
    __shared__ uint32_t red[kCastThreads / 32];
    __shared__ uint32_t cta_max;
    const uint32_t rank = cluster_rank_c();
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
        for (; v + 3u * kCastThreads < nvec; v += 4u * kCastThreads) {  // four loads in flight
            uint4 w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) w[k] = __ldcs(src + v + k * kCastThreads);
#pragma unroll
            for (int k = 0; k < 4; ++k) scan(w[k]);
        }
        for (; v < nvec; v += kCastThreads) scan(__ldcs(src + v));
        for (uint32_t g = g0 + nvec * 16u + threadIdx.x; g < g1; g += kCastThreads) {
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
        for (int w = 0; w < kCastThreads / 32; ++w) m = max(m, red[w]);
        cta_max = m;
    }
    cluster_sync_c();
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
    cluster_sync_c();                                               // all remote reads done
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
// A warp step covers a tile of 256 consecutive MX blocks of one matrix: lane t takes
// blocks tile + 32i + t (i = 0..7), so every load and store instruction of the warp
// moves contiguous bytes (32 code bytes, 512 nibble bytes, 64 scale bytes).
constexpr uint32_t kTile = 256;

__global__ void __launch_bounds__(kCastThreads)
cast_rewrite_kernel(const __grid_constant__ CastParams p)
{
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t warp_id = (blockIdx.x * kCastThreads + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * kCastThreads) >> 5;
    uint32_t n_in = 0u, n_fb = 0u, n_ll = 0u;
    for (uint32_t ti = warp_id; ti < p.groups; ti += nwarps) {      // p.groups counts 256-block tiles here
        int j = 0;
        {
            int lo = 0, hi = p.n - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (p.jobs[mid].group_begin <= ti) lo = mid; else hi = mid - 1;
            }
            j = lo;
        }
        const CastJobDev& job = p.jobs[j];
        const float s2 = *job.d_s2;
        const int k_max = exact_log2(s2) + 8;
        const bool copy = job.nv_q != job.mx_q;
        const uint32_t base = kTile * (ti - job.group_begin);
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
                if (g < job.nb) qv[i] = __ldcs(reinterpret_cast<const uint4*>(job.mx_q + (int64_t)g * 16));
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
                __stcs(reinterpret_cast<unsigned short*>(job.nv_scales + (int64_t)g * 2), (unsigned short)(e | (e << 8)));
                if (copy) __stcs(reinterpret_cast<uint4*>(job.nv_q + (int64_t)g * 16), qv[i]);
                n_in += 2u;
            } else {
                rare |= 1u << i;
            }
        }
        if (rare) {                                                  // after the copies: nothing else live
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (rare & (1u << i)) {
                    const uint32_t g = base + 32u * i + lane;
                    const uint32_t v = cast_rare_block(job.mx_q, job.nv_q, g, c[i], k_max, s2, copy, &n_fb, &n_ll);
                    *reinterpret_cast<uint16_t*>(job.nv_scales + (int64_t)g * 2) = (uint16_t)v;
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
    uint32_t groups = 0;
    for (int i = 0; i < n; ++i) {
        const nv4_cast_job& J = jobs[i];
        if (J.rows == 0 || J.cols == 0) continue;
        CastJobDev& d = p.jobs[m++];
        d.mx_q = J.mx_q; d.e8m0 = J.e8m0; d.nv_q = J.nv_q; d.nv_scales = J.nv_scales;
        d.d_ga = J.d_global_amax; d.d_s2 = J.d_s2;
        d.nb = (uint32_t)(J.rows * (J.cols / 32));
        d.group_begin = groups;
        groups += (d.nb + kTile - 1u) / kTile;
    }
    p.n = m;
    p.groups = groups;
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
    cfg.blockDim = dim3(kCastThreads, 1, 1);
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

    // a single resident wave (two CTAs per SM at this kernel's register count); warps
    // stride over the tiles
    const int64_t need = ((int64_t)groups + kCastThreads / 32 - 1) / (kCastThreads / 32);   // one warp per tile
    const int64_t cap = (int64_t)num_sms() * 2;
    const int grid = (int)(need < cap ? (need > 0 ? need : 1) : cap);
    cast_rewrite_kernel<<<grid, kCastThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace nv4
