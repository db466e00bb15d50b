// sweep.cu -- Hessian-weighted E4M3 block-scale sweep with NVFP4 pack (sm_100a).
//
// [CAL] section 2 step 3: for every 16-element weight block, try every E4M3 block
// scale and keep the one minimising (w - dq(w))^T H_b (w - dq(w)); see nv4.h.
//
// Mapping: one thread owns one (row, 16-block) pair; a CTA covers 128 rows of one
// block column b, so the block's Hessian H_b (136 distinct entries of a symmetric
// 16x16 matrix) is loaded once per CTA and kept in registers by every thread.
// The 127 candidate scales S_c (and the reciprocal brackets used to round w/S_c)
// depend only on the matrix's s2; they sit in a shared-memory table.
//
// Per candidate, per thread:
//   E2M1 codes of w/S_c   : bracketed hardware conversion, exact FP64 fix-up near
//                           a rounding boundary (nv4_common.cuh)
//   e_i = fma(-v_i, S_c, w_i)       (one rounding of the exact difference)
//   cost = sum_i e_i (H_ii e_i + sum_{j>i} (H_ij + H_ji) e_j)     136 + 16 FMA
// The loop runs over codes in increasing order and keeps a strictly smaller cost,
// so ties go to the lowest code.  Identical dequantized blocks produce identical e
// and therefore identical costs, so such ties are resolved exactly as well.
#include "nv4_common.cuh"
#include "nv4_internal.h"

namespace nv4 {

constexpr int kSweepThreads = 128;

struct SweepJobDev {
    const void* w;
    const float* H;
    const float* d_amax;
    uint8_t* codes;
    uint8_t* q;
    float* cost1;
    float* cost2;
    int64_t ld;
    uint32_t rows, nblk, row_tiles, cta_begin;
};

struct SweepParams {
    int n, dt;
    uint32_t* d_flags;
    SweepJobDev jobs[kMaxSweepJobs];
};

// E2M1 codes of the 16 weights at candidate scale S; t = {S, r_lo, r_hi, exact}.
__device__ __forceinline__ void codes16(const float w[16], const float4& t, uint32_t& c0, uint32_t& c1)
{
    if (t.w == 0.0f) {
        float lo[16], hi[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            lo[i] = __fmul_rn(w[i], t.y);
            hi[i] = __fmul_rn(w[i], t.z);
        }
        c0 = cvt_e2m1x8(lo);
        c1 = cvt_e2m1x8(lo + 8);
        const uint32_t h0 = cvt_e2m1x8(hi), h1 = cvt_e2m1x8(hi + 8);
        if (c0 == h0 && c1 == h1) return;
    }
    c0 = c1 = 0u;
    for (int i = 0; i < 8; ++i) c0 |= e2m1_code_exact(w[i], t.x) << (4 * i);
    for (int i = 0; i < 8; ++i) c1 |= e2m1_code_exact(w[8 + i], t.x) << (4 * i);
}

__device__ __forceinline__ void decode16(uint32_t c0, uint32_t c1, float v[16])
{
    uint32_t h[8];
    cvt_e2m1x8_to_f16x8(c0, h);
    cvt_e2m1x8_to_f16x8(c1, h + 4);
#pragma unroll
    for (int j = 0; j < 8; ++j) f16x2_to_f32(h[j], v[2 * j], v[2 * j + 1]);
}

template <int kDt>   // 0 bf16, 2 fp32
__global__ void __launch_bounds__(kSweepThreads, 2)
sweep_kernel(const __grid_constant__ SweepParams p)
{
    __shared__ float4 tab[128];
    __shared__ float hs[256];

    // locate job and tile
    int j = 0;
    {
        int lo = 0, hi = p.n - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.jobs[mid].cta_begin <= blockIdx.x) lo = mid; else hi = mid - 1;
        }
        j = lo;
    }
    const SweepJobDev& job = p.jobs[j];
    const uint32_t local = blockIdx.x - job.cta_begin;
    const uint32_t b = local % job.nblk, tile = local / job.nblk;

    // candidate table: S_c = RN32(e4m3(c) * s2) and a bracket of 1/S_c
    const float s2 = __fdiv_rn(*job.d_amax, 2688.0f);
    if (threadIdx.x < 128) {
        const uint32_t c = threadIdx.x;
        float4 t = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (c < 127) {
            const float S = __fmul_rn(e4m3_value(c), s2);
            t.x = S;
            if (c == 0 || S == 0.0f) {
                t.w = S == 0.0f ? 0.0f : 1.0f;          // S == 0: sign-only codes, fast path exact
            } else if (S >= kTinyScale && S <= 0x1p100f) {
                const float r = __frcp_rn(S);
                t.y = __fmul_rn(r, kLoMargin);
                t.z = __fmul_rn(r, kHiMargin);
            } else {
                t.w = 1.0f;                              // exact FP64 path for this candidate
            }
        }
        tab[c] = t;
    }
    for (int k = threadIdx.x; k < 256; k += kSweepThreads) hs[k] = job.H[(int64_t)b * 256 + k];
    __syncthreads();

    const uint32_t row = tile * kSweepThreads + threadIdx.x;
    if (row >= job.rows) return;

    // H_b in registers: diagonal and (H_ij + H_ji) for j > i
    float hd[16], ho[120];
#pragma unroll
    for (int i = 0, o = 0; i < 16; ++i) {
        hd[i] = hs[17 * i];
#pragma unroll
        for (int k = i + 1; k < 16; ++k, ++o) ho[o] = hs[16 * i + k] + hs[16 * k + i];
    }

    float w[16];
    if constexpr (kDt == 0) {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(job.w) + (int64_t)row * job.ld + 16 * b);
        const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
        const uint32_t u[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            w[2 * k] = bf16_lo(u[k]);
            w[2 * k + 1] = bf16_hi(u[k]);
        }
    } else {
        const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(job.w) + (int64_t)row * job.ld + 16 * b);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float4 v = __ldg(src + k);
            w[4 * k] = v.x; w[4 * k + 1] = v.y; w[4 * k + 2] = v.z; w[4 * k + 3] = v.w;
        }
    }
    uint32_t flags = isfinite(s2) ? 0u : kFlagOverflow;
#pragma unroll
    for (int i = 0; i < 16; ++i)
        if (!isfinite(w[i])) flags |= kFlagNonFinite;

    float best = __int_as_float(0x7F800000), second = best;
    uint32_t best_c = 0u;
#pragma unroll 1
    for (uint32_t c = 0; c < 127; ++c) {
        const float4 t = tab[c];
        uint32_t c0, c1;
        codes16(w, t, c0, c1);
        float v[16], e[16];
        decode16(c0, c1, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) e[i] = fmaf(-v[i], t.x, w[i]);
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int i = 0, o = 0; i < 16; ++i) {
            float z = hd[i] * e[i];
#pragma unroll
            for (int k = i + 1; k < 16; ++k, ++o) z = fmaf(ho[o], e[k], z);
            acc[i & 3] = fmaf(e[i], z, acc[i & 3]);
        }
        const float cost = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        if (cost < best) {
            second = best;
            best = cost;
            best_c = c;
        } else if (cost > best && cost < second) {
            second = cost;
        }
    }
    if (!isfinite(best)) flags |= kFlagNonFinite;

    const int64_t blk = (int64_t)row * job.nblk + b;
    job.codes[blk] = (uint8_t)best_c;
    if (job.q != nullptr) {
        uint32_t c0, c1;
        codes16(w, tab[best_c], c0, c1);
        *reinterpret_cast<uint2*>(job.q + blk * 8) = make_uint2(c0, c1);
    }
    if (job.cost1 != nullptr) job.cost1[blk] = best;
    if (job.cost2 != nullptr) job.cost2[blk] = second;
    flag_or(p.d_flags, flags);
}

cudaError_t launch_sweep(const nv4_sweep_job* jobs, int n, int dt, uint32_t* d_flags, cudaStream_t s)
{
    SweepParams p;
    p.dt = dt;
    p.d_flags = d_flags;
    int m = 0;
    uint32_t ctas = 0;
    for (int i = 0; i < n; ++i) {
        const nv4_sweep_job& J = jobs[i];
        if (J.rows == 0 || J.cols == 0) continue;
        SweepJobDev& d = p.jobs[m++];
        d.w = J.w; d.H = J.H; d.d_amax = J.d_amax_w; d.codes = J.codes; d.q = J.q;
        d.cost1 = J.cost1; d.cost2 = J.cost2; d.ld = J.ld;
        d.rows = (uint32_t)J.rows;
        d.nblk = (uint32_t)(J.cols / 16);
        d.row_tiles = (d.rows + kSweepThreads - 1) / kSweepThreads;
        d.cta_begin = ctas;
        ctas += d.row_tiles * d.nblk;
    }
    p.n = m;
    if (m == 0) return cudaSuccess;
    if (dt == 0) sweep_kernel<0><<<ctas, kSweepThreads, 0, s>>>(p);
    else sweep_kernel<2><<<ctas, kSweepThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace nv4
