// sweep.cu -- Hessian-weighted E4M3 block-scale sweep with NVFP4 pack (sm_100a).
//
// [CAL] section 2 step 3: for every 16-element weight block, try every E4M3 block
// scale and keep the one minimising (w - dq(w))^T H_b (w - dq(w)); see nv4.h.
//
// Mapping: one thread owns one (row, 16-block) pair; a CTA covers 128 rows of one
// block column b and keeps that block's Hessian H_b in shared memory, laid out so
// every warp reads it with conflict-free broadcast 128-bit loads.  The 127 candidate
// scales S_c (and the reciprocal brackets used to round w/S_c) depend only on the
// matrix's s2; they sit in a shared-memory table.
//
// Per candidate, per thread (all FP32; pairs use the packed FP32 instructions):
//   E2M1 codes of w/S_c : bracketed hardware conversion; near a rounding boundary
//                         one exact FMA comparison fixes the code (nv4_common.cuh)
//   e_i = w_i - v_i*S_c   (one rounding of the exact difference)
//   cost = sum_i e_i (H_ii e_i + sum_{j>i} (H_ij + H_ji) e_j), evaluated two rows at
//          a time: 136 + 16 multiply-adds in 80 packed instructions
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

// E2M1 codes of the 16 weights w (as 8 pairs) at candidate t = {S, r_lo, r_hi, exact}.
__device__ __forceinline__ void codes16(const float2 w[8], const float4& t, uint32_t& c0, uint32_t& c1)
{
    if (t.w == 0.0f) {
        const float2 rl = make_float2(t.y, t.y), rh = make_float2(t.z, t.z);
        float lo[16], hi[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float2 a = __fmul2_rn(w[j], rl), b = __fmul2_rn(w[j], rh);
            lo[2 * j] = a.x; lo[2 * j + 1] = a.y;
            hi[2 * j] = b.x; hi[2 * j + 1] = b.y;
        }
        c0 = cvt_e2m1x8(lo);
        c1 = cvt_e2m1x8(lo + 8);
        const uint32_t h0 = cvt_e2m1x8(hi), h1 = cvt_e2m1x8(hi + 8);
        if (c0 != h0 || c1 != h1) {          // near a rounding boundary: exact FP32 fix-up
            float x[16];
#pragma unroll
            for (int j = 0; j < 8; ++j) { x[2 * j] = w[j].x; x[2 * j + 1] = w[j].y; }
            if (c0 != h0) c0 = e2m1_fix8(x, t.x, c0, h0);
            if (c1 != h1) c1 = e2m1_fix8(x + 8, t.x, c1, h1);
        }
        return;
    }
    // S outside [2^-100, 2^100] (degenerate second-level scale): exact FP64 decisions
    c0 = c1 = 0u;
    for (int i = 0; i < 8; ++i) c0 |= e2m1_code_exact(i & 1 ? w[i >> 1].y : w[i >> 1].x, t.x) << (4 * i);
    for (int i = 0; i < 8; ++i) c1 |= e2m1_code_exact(i & 1 ? w[4 + (i >> 1)].y : w[4 + (i >> 1)].x, t.x) << (4 * i);
}

// Signed E2M1 values of the packed codes, as 8 pairs.
__device__ __forceinline__ void decode16(uint32_t c0, uint32_t c1, float2 v[8])
{
    uint32_t h[8];
    cvt_e2m1x8_to_f16x8(c0, h);
    cvt_e2m1x8_to_f16x8(c1, h + 4);
#pragma unroll
    for (int j = 0; j < 8; ++j) f16x2_to_f32(h[j], v[j].x, v[j].y);
}

// Shared-memory image of one H_b for the row-pair quadratic form: for rows (2m, 2m+1)
// one float4 {H_2m,2m, H_2m+1,2m+1, H'_2m,2m+1, 0} then, for k = 2m+2, 2m+4, ..., 14,
// float4 {H'_2m,k, H'_2m+1,k, H'_2m,k+1, H'_2m+1,k+1}, with H'_ij = H_ij + H_ji.
constexpr int kHPairs = 36;

__device__ __forceinline__ float hsym(const float* H, int i, int j) { return H[16 * i + j] + H[16 * j + i]; }

__device__ void build_hpairs(const float* __restrict__ H, float4* hp)
{
    for (int idx = threadIdx.x; idx < kHPairs; idx += blockDim.x) {
        // locate (m, slot) of entry idx: row pair m owns 8 - m entries
        int m = 0, base = 0;
        while (idx >= base + (8 - m)) { base += 8 - m; ++m; }
        const int slot = idx - base;
        const int r0 = 2 * m, r1 = 2 * m + 1;
        float4 v;
        if (slot == 0) {
            v = make_float4(H[17 * r0], H[17 * r1], hsym(H, r0, r1), 0.0f);
        } else {
            const int k = 2 * m + 2 * slot;
            v = make_float4(hsym(H, r0, k), hsym(H, r1, k), hsym(H, r0, k + 1), hsym(H, r1, k + 1));
        }
        hp[idx] = v;
    }
}

// e^T H e with e as 8 pairs and H_b in the shared-memory image above.
__device__ __forceinline__ float quad_form(const float2 e[8], const float4* __restrict__ hp)
{
    float2 acc = make_float2(0.0f, 0.0f);
    int idx = 0;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const float4 d = hp[idx++];
        float2 z = __fmul2_rn(make_float2(d.x, d.y), e[m]);
        z.x = fmaf(d.z, e[m].y, z.x);
#pragma unroll
        for (int k2 = m + 1; k2 < 8; ++k2) {
            const float4 h = hp[idx++];
            z = __ffma2_rn(make_float2(h.x, h.y), make_float2(e[k2].x, e[k2].x), z);
            z = __ffma2_rn(make_float2(h.z, h.w), make_float2(e[k2].y, e[k2].y), z);
        }
        acc = __ffma2_rn(e[m], z, acc);
    }
    return acc.x + acc.y;
}

template <int kDt>   // 0 bf16, 2 fp32
__global__ void __launch_bounds__(kSweepThreads, 4)
sweep_kernel(const __grid_constant__ SweepParams p)
{
    __shared__ float4 tab[128];
    __shared__ float4 hp[kHPairs];
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
            if (S == 0.0f) {
                // zero scale: the products w*0 keep the sign, giving sign-only codes
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
    build_hpairs(hs, hp);
    __syncthreads();

    const uint32_t row = tile * kSweepThreads + threadIdx.x;
    if (row >= job.rows) return;

    float2 w[8];
    if constexpr (kDt == 0) {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(job.w) + (int64_t)row * job.ld + 16 * b);
        const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
        const uint32_t u[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) w[k] = make_float2(bf16_lo(u[k]), bf16_hi(u[k]));
    } else {
        const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(job.w) + (int64_t)row * job.ld + 16 * b);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float4 v = __ldg(src + k);
            w[2 * k] = make_float2(v.x, v.y);
            w[2 * k + 1] = make_float2(v.z, v.w);
        }
    }
    uint32_t flags = isfinite(s2) ? 0u : kFlagOverflow;
#pragma unroll
    for (int k = 0; k < 8; ++k)
        if (!isfinite(w[k].x) || !isfinite(w[k].y)) flags |= kFlagNonFinite;

    float best = __int_as_float(0x7F800000), second = best;
    uint32_t best_c = 0u;
#pragma unroll 1
    for (uint32_t c = 0; c < 127; ++c) {
        const float4 t = tab[c];
        uint32_t c0, c1;
        codes16(w, t, c0, c1);
        float2 v[8], e[8];
        decode16(c0, c1, v);
        const float2 nS = make_float2(-t.x, -t.x);
#pragma unroll
        for (int k = 0; k < 8; ++k) e[k] = __ffma2_rn(v[k], nS, w[k]);     // w - v*S, one rounding
        const float cost = quad_form(e, hp);
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
