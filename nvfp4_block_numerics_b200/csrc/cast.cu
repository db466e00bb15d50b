// cast.cu -- closed-form MXFP4 -> NVFP4 cast (sm_100a).
//
// [CAST] section 2; [DSPARK] stage 3 (see nv4.h).  Per matrix:
//   k_max = max_j (e8m0_j - 127);  m = k_max - 8;  s2 = 2^m;  global_amax = 6*448*2^m
//   MX block j with d = k_max - k_j <= 17: both NVFP4 scales encode 2^(k_j - m) = 2^(8-d)
//   exactly in E4M3 and the 16 nibble bytes are reused; otherwise the block is
//   re-quantized from its exact values e2m1 * 2^k_j (rare fallback path).
//
// One thread-block cluster of kCastCluster CTAs handles one matrix.  Phase 1: each
// CTA reduces the largest E8M0 code of its share of the matrix (and keeps that share
// in shared memory); the cluster exchanges the partial maxima through distributed
// shared memory, so k_max needs no second launch and no scratch memory.  Phase 2:
// one thread per MX block writes the two E4M3 scale bytes and, out of place, copies
// the 16 nibble bytes with 128-bit loads and stores.
#include "nv4_common.cuh"
#include "nv4_internal.h"

namespace nv4 {

constexpr int kCastThreads = 512;
constexpr int kCastCluster = 8;
constexpr uint32_t kCastSmemCodes = 32768;       // cached E8M0 bytes per CTA

struct CastJobDev {
    const uint8_t* mx_q;
    const uint8_t* e8m0;
    uint8_t* nv_q;
    uint8_t* nv_scales;
    float* d_ga;
    float* d_s2;
    uint32_t rows, nmx;                           // nmx = cols / 32
    FastDiv div_nmx;
};

struct CastParams {
    int n;
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

__global__ void __launch_bounds__(kCastThreads)
cast_kernel(const __grid_constant__ CastParams p)
{
    __shared__ alignas(16) uint8_t codes[kCastSmemCodes];
    __shared__ uint32_t red[kCastThreads / 32];
    __shared__ uint32_t cta_max;
    __shared__ unsigned long long cnt[3];

    const uint32_t rank = cluster_rank_c();
    const CastJobDev& job = p.jobs[blockIdx.x / kCastCluster];
    const uint32_t nb = job.rows * job.nmx;                       // MX blocks in the matrix
    // share of this CTA, 16-aligned so the bulk can move in 16-byte words
    const uint32_t per = ((nb + kCastCluster - 1) / kCastCluster + 15u) & ~15u;
    const uint32_t g0 = min(nb, rank * per), g1 = min(nb, g0 + per);
    const bool cached = (g1 - g0) <= kCastSmemCodes;

    if (threadIdx.x < 3) cnt[threadIdx.x] = 0ull;

    // ---------------- phase 1: largest valid E8M0 code of the share
    uint32_t mx = 0u, flags = 0u;
    {
        const uint32_t nvec = (g1 - g0) / 16u;
        const uint4* src = reinterpret_cast<const uint4*>(job.e8m0 + g0);
        for (uint32_t v = threadIdx.x; v < nvec; v += kCastThreads) {
            const uint4 w = __ldcs(src + v);
            if (cached) reinterpret_cast<uint4*>(codes)[v] = w;
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    const uint32_t c = (ws[k] >> (8 * b)) & 0xFFu;
                    if (c == 0xFFu) flags |= kFlagE8M0Nan; else mx = max(mx, c);
                }
            }
        }
        for (uint32_t g = g0 + nvec * 16u + threadIdx.x; g < g1; g += kCastThreads) {
            const uint32_t c = job.e8m0[g];
            if (cached) codes[g - g0] = (uint8_t)c;
            if (c == 0xFFu) flags |= kFlagE8M0Nan; else mx = max(mx, c);
        }
    }
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t m = 0u;
        for (int w = 0; w < kCastThreads / 32; ++w) m = max(m, red[w]);
        cta_max = m;
    }
    cluster_sync_c();
    uint32_t kcode = 0u;
    for (uint32_t r = 0; r < kCastCluster; ++r) kcode = max(kcode, ld_dsmem_u32(&cta_max, r));
    cluster_sync_c();                                               // all remote reads done

    const int k_max = (int)kcode - 127, m = k_max - 8;
    const float s2 = exp2_exact(m);                                 // m in [-135, 119]
    if (rank == 0 && threadIdx.x == 0 && nb > 0) {
        const float ga = __fmul_rn(2688.0f, s2);                    // 6*448*2^m
        *job.d_s2 = s2;
        *job.d_ga = ga;
        if (!isfinite(ga)) flags |= kFlagOverflow;
    }

    // ---------------- phase 2: one thread per MX block
    const bool copy = job.nv_q != job.mx_q;
    uint32_t n_in = 0u, n_fb = 0u, n_ll = 0u;
    for (uint32_t g = g0 + threadIdx.x; g < g1; g += kCastThreads) {
        const uint32_t c = cached ? codes[g - g0] : job.e8m0[g];
        const uint32_t r = job.div_nmx.div(g), jb = g - r * job.nmx;
        const int64_t qoff = ((int64_t)r * job.nmx + jb) * 16;      // 16 nibble bytes per MX block
        uint16_t sc2;
        if (c == 0xFFu) {
            sc2 = 0;                                                // flagged in phase 1
            if (copy) *reinterpret_cast<uint4*>(job.nv_q + qoff) = *reinterpret_cast<const uint4*>(job.mx_q + qoff);
        } else {
            const int k = (int)c - 127, d = k_max - k;
            if (d <= 17) {
                const uint32_t sc = e4m3_code_pow2(8 - d);
                sc2 = (uint16_t)(sc | (sc << 8));
                if (copy)
                    __stcs(reinterpret_cast<uint4*>(job.nv_q + qoff), __ldcs(reinterpret_cast<const uint4*>(job.mx_q + qoff)));
                n_in += 2u;
                n_ll += 2u;
            } else {
                const uint4 qv = *reinterpret_cast<const uint4*>(job.mx_q + qoff);
                const uint32_t lo_words[2] = {qv.x, qv.y}, hi_words[2] = {qv.z, qv.w};
                uint32_t out_lo[2], out_hi[2], ll0, ll1;
                const uint32_t s_lo = cast_fallback16(lo_words, k, s2, out_lo, &ll0);
                const uint32_t s_hi = cast_fallback16(hi_words, k, s2, out_hi, &ll1);
                *reinterpret_cast<uint4*>(job.nv_q + qoff) = make_uint4(out_lo[0], out_lo[1], out_hi[0], out_hi[1]);
                sc2 = (uint16_t)(s_lo | (s_hi << 8));
                n_fb += 2u;
                n_ll += ll0 + ll1;
            }
        }
        *reinterpret_cast<uint16_t*>(job.nv_scales + ((int64_t)r * job.nmx + jb) * 2) = sc2;
    }

    // ---------------- counters and flags
    n_in = __reduce_add_sync(0xFFFFFFFFu, n_in);
    n_fb = __reduce_add_sync(0xFFFFFFFFu, n_fb);
    n_ll = __reduce_add_sync(0xFFFFFFFFu, n_ll);
    flags = __reduce_or_sync(0xFFFFFFFFu, flags);
    if ((threadIdx.x & 31) == 0) {
        if (n_in) atomicAdd(&cnt[0], (unsigned long long)n_in);
        if (n_fb) atomicAdd(&cnt[1], (unsigned long long)n_fb);
        if (n_ll) atomicAdd(&cnt[2], (unsigned long long)n_ll);
        flag_or(p.d_flags, flags);
    }
    __syncthreads();
    if (threadIdx.x < 3 && p.d_counts != nullptr && cnt[threadIdx.x] != 0ull)
        atomicAdd(p.d_counts + threadIdx.x, cnt[threadIdx.x]);
}

cudaError_t launch_cast(const nv4_cast_job* jobs, int n, unsigned long long* d_counts, uint32_t* d_flags,
                        cudaStream_t s)
{
    CastParams p;
    p.d_counts = d_counts;
    p.d_flags = d_flags;
    int m = 0;
    for (int i = 0; i < n; ++i) {
        const nv4_cast_job& J = jobs[i];
        if (J.rows == 0 || J.cols == 0) continue;
        CastJobDev& d = p.jobs[m++];
        d.mx_q = J.mx_q; d.e8m0 = J.e8m0; d.nv_q = J.nv_q; d.nv_scales = J.nv_scales;
        d.d_ga = J.d_global_amax; d.d_s2 = J.d_s2;
        d.rows = (uint32_t)J.rows;
        d.nmx = (uint32_t)(J.cols / 32);
        d.div_nmx = FastDiv(d.nmx);
    }
    p.n = m;
    if (m == 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(m * kCastCluster), 1, 1);
    cfg.blockDim = dim3(kCastThreads, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCastCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, cast_kernel, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace nv4
