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
// Per visited candidate, per thread (all FP32; pairs use the packed FP32 instructions),
// in two halves of 8 elements -- the second half only when the first half's part of
// bound (1) below does not already rule the candidate out:
//   E2M1 codes of w/S_c : for bound (1), the hardware conversion of the lower end of the
//                         bracket alone; for a candidate the bound leaves open, the exact
//                         codes (both ends converted, near a rounding boundary one exact FMA
//                         comparison fixes the code, nv4_common.cuh) and e again where they
//                         differ
//   e_i = w_i - v_i*S_c   (one rounding of the exact difference)
//   cost = sum_i e_i (H_ii e_i + sum_{j>i} (H_ij + H_ji) e_j), evaluated two rows at
//          a time: 136 + 16 multiply-adds in 80 packed instructions
//
// Exact search order (branch and bound).  The result is the argmin over all 127
// codes, but most candidates are ruled out by lower bounds instead of evaluated:
//   (1) Scaled eigenvalue bound.  With D = diag(H_b) > 0 and H' = D^-1/2 Hs D^-1/2 (Hs
//       the symmetric part), every mu <= lambda_min(H') gives, for every e:
//       e^T H_b e >= mu sum_i H_ii e_i^2.  Per block column, mu is the larger of
//       Gershgorin's rho = 1 - max_i sum_{j != i} |H'_ij| and a value that a
//       floating-point Cholesky factorization of H' - mu I certifies (block_bound).
//   (2) Every grid point of scale S is at most 6S in magnitude, so |e_i| >= |w_i| - 6S,
//       and the same holds at every smaller scale.
//   (3) An element with |w_i| <= S/2 is at least min(|w_i|, S/2 - |w_i|) away from every
//       grid point of every scale >= S (its nearest points there are 0 and S'/2 >= S/2),
//       so mu * sum_i H_ii min(.)^2 bounds the cost of every candidate from S upwards.
// The winner and the runner-up cost depend only on candidates whose cost is at most
// the running runner-up cost; when the runner-up is not an output, only the winner
// (ties to the lowest code) has to be found and the running best cost is the
// threshold instead.  A thread starts at the max-calibrated code (nearest E4M3 to
// amax_b / (6 s2)) and walks outwards, alternating down and up: a candidate whose
// bound (1) exceeds the threshold skips the quadratic form, and once bound (2) over
// the two largest |w_i| exceeds it, the downward walk ends; once bound (3) exceeds it,
// the upward walk ends (long upward walks: weights whose block amax is far below the
// tensor's, such as heavy-tailed expert weights).  The comparisons
// keep a relative margin of 2^-10, far above the FP32 evaluation error and the 2^-15 by
// which bound (1) from the lower-end codes can exceed the bound from the exact codes, so
// skipped candidates could not have changed the FP32 result either.  When mu < 1/32, or eta_b
// (below) exceeds 2^-12, or H_b has a zero diagonal entry with a nonzero row, or
// non-finite entries, the bounds are off and all 127 candidates are evaluated, in FP64.
//
// Accuracy.  An FP32 cost differs from the exact eT H_b e by at most
// gamma * |e|T |H_b| |e| with gamma = 29 * 2^-24 (the longest chain of roundings a term
// goes through in quad_form, plus the roundings of e and of H_ij + H_ji), and
// |e|T |H_b| |e| <= (2 - rho) sum_i H_ii e_i^2 <= (2 - rho) / mu * eT H_b e (Gershgorin
// for the absolute values, then bound (1)), so every cost of block column b is exact to
// eta_b = gamma (2 - rho) / mu relative.  When eta_b <= 4e-6 the FP32 argmin is within
// 1e-5 of the exact minimum, the tolerance of a near tie.  Otherwise the block is searched again in FP64 when its
// FP32 runner-up lies within 3 eta_b of the winner (or the costs are outputs), and
// without a valid bound it is searched in FP64 from the start: the FP64 costs carry
// errors ~1e-16 |e|T |H_b| |e|, so the winner is the exact argmin outside ties closer
// than that.  Pruning keeps its 2^-10 margin, at least 4 eta_b wherever the bounds are on.
//
// Ties: the lowest code wins among equal costs, and the runner-up is the smallest
// cost strictly above the winner's, independent of the visiting order.  In a column whose
// FP32 costs are not certified, two codes with exactly the same FP32 cost are a near tie
// like a runner-up within 3 eta_b: the block is searched again in FP64.  Identical
// dequantized blocks produce identical e and therefore identical costs.
#include "nv4_common.cuh"
#include "nv4_internal.h"

namespace nv4 {

constexpr int kSweepThreads = 128;
// Row tiles of 128 per CTA (the bounds' set-up is paid once per CTA): up to 4 for BF16
// weights (24 KB of shared memory, 7 CTAs per SM), 3 for FP32 (the staged blocks are
// twice as large)
template <int kDt> constexpr int kMaxTilesPerCta = kDt == 0 ? 4 : 3;
template <int kDt> constexpr int kMaxRowsPerCta = kMaxTilesPerCta<kDt> * kSweepThreads;
constexpr float kPruneScale = 1.0f - 0x1p-10f;   // bound * this must exceed the runner-up

struct SweepJobDev {
    const void* w;
    const float* H;
    const float* d_amax;
    uint8_t* codes;
    uint8_t* q;
    float* cost1;
    float* cost2;
    unsigned long long* d_work;
    int64_t ld;
    uint32_t rows, nblk, row_tiles, cta_begin;
};

struct SweepParams {
    int n, dt;
    uint32_t tiles_per_cta;
    uint32_t* d_flags;
    SweepJobDev jobs[kMaxSweepJobs];
};

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

// The scaled symmetric part M = D^-1/2 Hs D^-1/2 of H_b, row lane % 16 (both 16-lane
// halves of the warp hold the matrix; s_i = RN(1 / sqrt(H_ii)), 0 for a zero diagonal,
// whose row is then a unit row): m_ij = 0.5 (H_ij + H_ji) s_i s_j in FP32, at most 5
// roundings (3e-7 relative) from the exact value.
__device__ __forceinline__ float scaled_entry(const float* __restrict__ hs, float si, int j)
{
    const int i = threadIdx.x & 15;
    const float sj = __shfl_sync(0xffffffffu, si, j, 16);
    const float h = 0.5f * (hs[16 * i + j] + hs[16 * j + i]);
    return j == i ? 1.0f : __fmul_rn(__fmul_rn(h, si), sj);
}

// Whether M - (mu + 2^-13) I is positive definite, each 16-lane half of the warp testing
// its own mu: an FP32 Cholesky factorization (outer-product form), each column scaled by
// rsqrtf of its pivot (within 2 ulp).  If it completes with positive pivots,
// lambda_min(M) >= mu: the factorization's backward error is at most (gamma_17 + 3 *
// 2^-22) |L||L|^T, whose 2-norm is at most its trace, the trace of the factored matrix
// (< 16), so below 3e-5 (Rump's criterion for floating-point Cholesky); the rounding of
// the scaled entries (16 per row, < 1 each) adds less than 5e-6: both far below the
// 2^-13 (1.2e-4) shift.  Pivots below 2^-60 count as failures.  No early exit: both
// halves run all 16 steps (a failed half computes on, its result discarded), so every
// shuffle is executed by the whole warp.
__device__ __noinline__ bool chol_test(const float* __restrict__ hs, float si, float mu)
{
    const int ll = threadIdx.x & 15;
    const float d = __fadd_rn(mu, 0x1p-13f);
    float a[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) a[j] = scaled_entry(hs, si, j) - (j == ll ? d : 0.0f);
    bool ok = true;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const float piv = __shfl_sync(0xffffffffu, a[k], k, 16);
        ok = ok && piv >= 0x1p-60f;                            // smaller pivots count as failures
        const float l = ll > k ? a[k] * rsqrtf(fmaxf(piv, 0x1p-60f)) : 0.0f;
#pragma unroll
        for (int j = k + 1; j < 16; ++j) a[j] = fmaf(-l, __shfl_sync(0xffffffffu, l, j, 16), a[j]);
    }
    return ok;
}

// mu * H_ii for the lower bounds (1)-(3), or all zero with *ok = false when no bound is
// valid for this H_b.  Run by one full warp, lane i < 16 owning channel i.
//   Gershgorin: rho = 1 - max_i sum_{j != i} |H'_ij| (H' the scaled symmetric part), in
//   FP32 with explicit safety margins: rsqrtf is within 2 ulp and the 15-term sum of
//   positive products within 2^-19 relative, so r * (1 + 2^-16) + 2^-16 bounds the exact
//   radius from above.  Always a lower bound of lambda_min(H'), often a loose one.
//   Certified lambda_min: one trisection of [max(rho, 0), 1 - max |m_ij|] (the upper end
//   is the smaller eigenvalue of a 2 x 2 principal minor), the two halves of the warp
//   testing the two inner points with chol_test at once; a test that succeeds proves its
//   mu (on the bench's Hessians lambda_min is 1.2 to 1.35 x rho, and the larger factor
//   prunes more candidates in all three bounds; a second trisection round, or the
//   bisection with four sequential tests, cost more in the CTA's prologue than they save).
// mu = the larger of the two; the bounds are used when mu >= 1/32 and the FP32 cost error
// bound eta = gamma * (2 - rho) / mu (|e|T |H_b| |e| <= (1 + r) sum_i H_ii e_i^2 <=
// (2 - rho) / mu * eT H_b e) is at most 2^-12, below the pruning margin 2^-10.  *eta
// receives that relative error bound of this column's FP32 costs (+inf without a bound).
constexpr float kCostGamma = 29.0f * 0x1p-24f;     // roundings per term of quad_form, plus e and H_ij + H_ji
constexpr float kCertifiedEta = 4e-6f;             // FP32 argmin within 1e-5 of the exact minimum
__device__ void block_bound(const float* __restrict__ hs, float* rd, int* ok, float* eta)
{
    const int lane = threadIdx.x & 31;
    const int i = lane & 15;
    const float di = hs[17 * i];
    bool bad = lane < 16 && !(di >= 0.0f && di <= 3.0e38f);
    const float inv = di > 0.0f ? rsqrtf(di) : 0.0f;
    float r = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const float inv_j = __shfl_sync(0xffffffffu, inv, j);
        if (j == i) continue;
        const float hij = 0.5f * (hs[16 * i + j] + hs[16 * j + i]);
        if (!(fabsf(hij) <= 3.0e38f)) bad = true;
        else if (hij != 0.0f && (inv == 0.0f || inv_j == 0.0f)) bad = true;   // zero diagonal, nonzero row
        r = fmaf(fabsf(hij) * inv, inv_j, r);
    }
    for (int o = 8; o > 0; o >>= 1) r = fmaxf(r, __shfl_xor_sync(0xffffffffu, r, o));
    bad = __any_sync(0xffffffffu, bad || !(r <= 3.0e38f));
    const float rho = 1.0f - fmaf(r, 1.0f + 0x1p-16f, 0x1p-16f);
    float mu = rho;
    if (!bad) {
        const float si = di > 0.0f ? __frsqrt_rn(di) : 0.0f;
        float mmax = 0.0f;                                   // max |m_ij|, i != j
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float mij = scaled_entry(hs, si, j);       // every lane: it shuffles
            if (j != i) mmax = fabsf(mij) < 1.0f ? fmaxf(mmax, fabsf(mij)) : 2.0f;   // also NaN
        }
        for (int o = 16; o > 0; o >>= 1) mmax = fmaxf(mmax, __shfl_xor_sync(0xffffffffu, mmax, o));
        if (mmax < 1.0f) {                                   // warp-uniform; else lambda_min <= 0
            float lo = fmaxf(rho, 0.0f), hi = 1.0f - mmax;
#pragma unroll 1
            for (int round = 0; round < 1 && lo < hi; ++round) {
                const float t1 = fmaf(hi - lo, 1.0f / 3.0f, lo), t2 = fmaf(hi - lo, 2.0f / 3.0f, lo);
                const bool okh = chol_test(hs, si, lane < 16 ? t1 : t2);
                const bool ok1 = __shfl_sync(0xffffffffu, okh, 0), ok2 = __shfl_sync(0xffffffffu, okh, 16);
                if (ok2) lo = t2;
                else if (ok1) { lo = t1; hi = t2; }
                else hi = t1;
            }
            mu = fmaxf(rho, lo);
        }
    }
    const float gam = __fdiv_ru(__fmul_ru(kCostGamma, 2.0f - rho), mu);
    const bool good = !bad && mu >= 0x1p-5f && gam <= 0x1p-12f;
    if (lane < 16) rd[lane] = good ? __fmul_rd(mu, di) : 0.0f;
    if (lane == 0) {
        *ok = good ? 1 : 0;
        *eta = good ? gam : __int_as_float(0x7F800000);
    }
}

// E2M1 codes of 8 weights (4 pairs) at candidate t = {S, r_lo, r_hi, exact}: both ends of
// the bracket converted, an exact FP32 fix-up where they disagree; S outside
// [2^-100, 2^100] (a degenerate second-level scale) takes the exact FP64 decisions.
__device__ __forceinline__ void codes8h(const float2 w[4], const float4& t, uint32_t& c)
{
    if (t.w == 0.0f) {
        const float2 rl = make_float2(t.y, t.y), rh = make_float2(t.z, t.z);
        float lo[8], hi[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 a = __fmul2_rn(w[j], rl), b = __fmul2_rn(w[j], rh);
            lo[2 * j] = a.x; lo[2 * j + 1] = a.y;
            hi[2 * j] = b.x; hi[2 * j + 1] = b.y;
        }
        c = cvt_e2m1x8(lo);
        const uint32_t h = cvt_e2m1x8(hi);
        if (c != h) {                        // near a rounding boundary: exact FP32 fix-up
            float x[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) { x[2 * j] = w[j].x; x[2 * j + 1] = w[j].y; }
            c = e2m1_fix8(x, t.x, c, h);
        }
        return;
    }
    c = 0u;
    for (int i = 0; i < 8; ++i) c |= e2m1_code_exact(i & 1 ? w[i >> 1].y : w[i >> 1].x, t.x) << (4 * i);
}

// E2M1 codes of 8 weights from the lower end of the bracket alone.  They differ from the
// exact codes only where w/S_c lies within the bracket's relative width (2^-20) above a
// rounding midpoint m, and there the other neighbour is as far from w to within a relative
// 2 m 2^-20 / (half the grid spacing at m) <= 14 * 2^-20 < 2^-16: bound (1) from these codes
// exceeds the one from the exact codes by less than 2^-15 relative, far inside the pruning
// margin.
__device__ __forceinline__ uint32_t codes8h_lo(const float2 w[4], const float4& t)
{
    const float2 rl = make_float2(t.y, t.y);
    float lo[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 a = __fmul2_rn(w[j], rl);
        lo[2 * j] = a.x; lo[2 * j + 1] = a.y;
    }
    return cvt_e2m1x8(lo);
}

// The exact codes given the lower-end codes c (t.w == 0): the upper end converted, the
// exact FP32 fix-up where the two ends disagree.
__device__ __forceinline__ uint32_t codes8h_exact_from(const float2 w[4], const float4& t, uint32_t c)
{
    const float2 rh = make_float2(t.z, t.z);
    float hi[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 b = __fmul2_rn(w[j], rh);
        hi[2 * j] = b.x; hi[2 * j + 1] = b.y;
    }
    const uint32_t h = cvt_e2m1x8(hi);
    if (c != h) {
        float x[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) { x[2 * j] = w[j].x; x[2 * j + 1] = w[j].y; }
        c = e2m1_fix8(x, t.x, c, h);
    }
    return c;
}

// Signed E2M1 values of 8 packed codes, as 4 pairs.
__device__ __forceinline__ void decode8h(uint32_t c, float2 v[4])
{
    uint32_t h[4];
    cvt_e2m1x8_to_f16x8(c, h);
#pragma unroll
    for (int j = 0; j < 4; ++j) f16x2_to_f32(h[j], v[j].x, v[j].y);
}

// Lower bound (1) over 8 elements: sum_i rd_i e_i^2 (rd4: their mu * H_ii).
__device__ __forceinline__ float bound_half(const float2 e[4], const float4* __restrict__ rd4)
{
    float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const float4 d = rd4[k];
        acc = __ffma2_rn(__fmul2_rn(e[2 * k], make_float2(d.x, d.y)), e[2 * k], acc);
        acc = __ffma2_rn(__fmul2_rn(e[2 * k + 1], make_float2(d.z, d.w)), e[2 * k + 1], acc);
    }
    return acc.x + acc.y;
}

// Signed weights of a staged block (BF16 as its 32 bytes, FP32 as its 64).
template <int kDt>
__device__ __forceinline__ void unstage_block(const uint4* __restrict__ src, float2 w[8])
{
    if constexpr (kDt == 0) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint4 v = src[j];
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) w[4 * j + k] = make_float2(bf16_lo(u[k]), bf16_hi(u[k]));
        }
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 v = src[j];
            w[2 * j] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
            w[2 * j + 1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
        }
    }
}

struct Search64 {
    double best, second;
    uint32_t code;
};

// The exhaustive search of one block with every cost in FP64, by a whole warp: lane l
// takes candidates l, l + 32, l + 64, l + 96.  e_i = w_i - v_i S_c is exact in FP64
// (v_i S_c has at most 27 significant bits) and eT H_b e is summed as in quad_form; the
// element codes are the same exact decisions as in the FP32 search.  Winner: smallest
// cost, ties to the lowest code; runner-up: the smallest cost above the winner's.  Used
// for the blocks whose FP32 costs cannot certify the argmin, after the FP32 walk and
// out of line, so that it costs the walk no registers.
template <int kDt>
__device__ __noinline__ Search64 search_fp64_warp(const uint4* __restrict__ src, const float4* __restrict__ tab,
                                                  const float* __restrict__ hs)
{
    const uint32_t lane = threadIdx.x & 31u;
    const double inf = __longlong_as_double(0x7FF0000000000000ll);
    float2 w[8];
    unstage_block<kDt>(src, w);
    double b1 = inf, b2 = inf;       // this lane's best and its smallest cost above it
    uint32_t bc = 0u;
#pragma unroll 1
    for (uint32_t c = lane; c < 127u; c += 32u) {
        const float4 t = tab[c];
        uint32_t q0, q1;
        codes8h(w, t, q0);
        codes8h(w + 4, t, q1);
        float2 v[8];
        decode8h(q0, v);
        decode8h(q1, v + 4);
        double e[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            e[2 * j] = fma(-(double)v[j].x, (double)t.x, (double)w[j].x);
            e[2 * j + 1] = fma(-(double)v[j].y, (double)t.x, (double)w[j].y);
        }
        double cost = 0.0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            double z = (double)hs[17 * i] * e[i];
#pragma unroll
            for (int j = i + 1; j < 16; ++j) z = fma((double)hs[16 * i + j] + (double)hs[16 * j + i], e[j], z);
            cost = fma(e[i], z, cost);
        }
        if (cost < b1) { b2 = b1; b1 = cost; bc = c; }   // ascending c: equal costs keep the lower code
        else if (cost > b1 && cost < b2) b2 = cost;
    }
    double B = b1;
    uint32_t C = bc;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double ob = __shfl_xor_sync(0xffffffffu, B, o);
        const uint32_t oc = __shfl_xor_sync(0xffffffffu, C, o);
        if (ob < B || (ob == B && oc < C)) { B = ob; C = oc; }
    }
    double s2 = b1 > B ? b1 : b2;    // this lane's smallest cost above the winner's
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s2 = fmin(s2, __shfl_xor_sync(0xffffffffu, s2, o));
    return Search64{B, s2, C};
}

// The FP64 searches of a CTA's listed rows, one warp per row; lane 0 writes the outputs.
// Returns the number of rows this lane finished (lane 0 only), for the work counter.
template <int kDt>
__device__ __noinline__ uint32_t redo_phase(const SweepJobDev& job, uint32_t b, uint32_t nr,
                                            const uint16_t* __restrict__ list, const uint4 (*__restrict__ sw)[kDt == 0 ? 2 : 4],
                                            const uint32_t* __restrict__ srow, const float4* __restrict__ tab,
                                            const float* __restrict__ hs, uint32_t* d_flags)
{
    const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;
    uint32_t done = 0u;
#pragma unroll 1
    for (uint32_t i = warp; i < nr; i += kSweepThreads / 32) {
        const uint32_t slot = list[i];
        const Search64 r = search_fp64_warp<kDt>(sw[slot], tab, hs);
        if (lane == 0) {
            const int64_t blk = (int64_t)srow[slot] * job.nblk + b;
            job.codes[blk] = (uint8_t)r.code;
            if (job.q != nullptr) {
                float2 w[8];
                unstage_block<kDt>(sw[slot], w);
                uint32_t c0, c1;
                const float4 tw = tab[r.code];
                codes8h(w, tw, c0);
                codes8h(w + 4, tw, c1);
                *reinterpret_cast<uint2*>(job.q + blk * 8) = make_uint2(c0, c1);
            }
            if (job.cost1 != nullptr) job.cost1[blk] = (float)r.best;
            if (job.cost2 != nullptr) job.cost2[blk] = (float)r.second;
            if (!(fabs(r.best) <= 1.7e308)) flag_or(d_flags, kFlagNonFinite);
            ++done;
        }
    }
    return done;
}

constexpr uint32_t kNoRow = 0xFFFFFFFFu;

// One CTA = one block column b of one job and up to p.tiles_per_cta tiles of 128 rows.
// Per tile the rows are counting-sorted by their starting code, so the lanes of a warp
// walk similar candidate sequences in lockstep.  Occupancy is the lever on this
// latency-bound search: 7 CTAs per SM (72 registers, 3 row tiles of staged weights,
// BF16 blocks staged as their 32 bytes) measured 1.34 ms on the Gemma-like layer against
// 1.73 ms at 4 CTAs (128 registers, 4 tiles as FP32), 1.38 ms at 6 and 1.35 ms at 8.
template <int kDt>   // 0 bf16, 2 fp32
__global__ void __launch_bounds__(kSweepThreads, 7)
sweep_kernel(const __grid_constant__ SweepParams p)
{
    __shared__ float4 tab[128];
    __shared__ float4 hp[kHPairs];
    __shared__ float hs[256];
    __shared__ float4 rd4[4];
    __shared__ int bound_ok;
    __shared__ float eta_s;
    static_assert(kMaxRowsPerCta<kDt> <= 512, "the FP64 search list shares the sort's 1 KB");
    __shared__ uint32_t sortbuf[256];                         // bucket counts and bases of the sort,
    uint32_t* const hist = sortbuf;                           // then the list of rows left to the
    uint32_t* const base = sortbuf + 128;                     // FP64 search (one 16-bit slot per row)
    uint16_t* const redo_list = reinterpret_cast<uint16_t*>(sortbuf);
    __shared__ uint32_t n_redo;
    __shared__ uint4 sw[kMaxRowsPerCta<kDt>][kDt == 0 ? 2 : 4];  // the group's weight blocks (BF16 or FP32 bits), load order
    __shared__ uint32_t srow[kMaxRowsPerCta<kDt>];                 // their rows (kNoRow past the end)
    __shared__ uint16_t perm[kMaxRowsPerCta<kDt>];                 // sorted position -> load slot

    // locate job and tile group
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
    const uint32_t b = local % job.nblk, group = local / job.nblk;

    // candidate table: S_c = RN32(e4m3(c) * s2) and a bracket of 1/S_c
    const float s2 = __fdiv_rn(*job.d_amax, 2688.0f);
    {
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
        hist[c] = 0u;
    }
    for (int k = threadIdx.x; k < 256; k += kSweepThreads) hs[k] = job.H[(int64_t)b * 256 + k];
    __syncthreads();
    build_hpairs(hs, hp);
    // warp 3 computes the bounds while the others load their rows (read after the next barrier)
    if (threadIdx.x >= 96) block_bound(hs, reinterpret_cast<float*>(rd4), &bound_ok, &eta_s);
    const float k6 = __frcp_rn(__fmul_rn(6.0f, s2));            // ~ 1/(6 s2), for the starting code
    const float* rd = reinterpret_cast<const float*>(rd4);
    const uint32_t s2flag = isfinite(s2) ? 0u : kFlagOverflow;

    uint32_t nhalf = 0u, nfull = 0u;                     // half-visits (8 elements), quadratic forms
    // ---- load the group's rows (up to 4 tiles of 128), counting-sort them by starting code
    const uint32_t tile0 = group * p.tiles_per_cta;
    const uint32_t ntile = min(job.row_tiles - tile0, p.tiles_per_cta);
    uint32_t keys[kMaxTilesPerCta<kDt>], ranks[kMaxTilesPerCta<kDt>];
    // all of this thread's loads first (one memory latency instead of one per tile), then
    // the keys; the blocks are staged as their bits
    constexpr int kVec = kDt == 0 ? 2 : 4;                  // 16-byte pieces per block
    uint4 raw[kMaxTilesPerCta<kDt>][kVec];
#pragma unroll
    for (uint32_t k = 0; k < kMaxTilesPerCta<kDt>; ++k) {
        const uint32_t row = (tile0 + k) * kSweepThreads + threadIdx.x;
        const bool live = k < ntile && row < job.rows;
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(job.w) +
                                                          ((int64_t)row * job.ld + 16 * b) * (kDt == 0 ? 2 : 4));
        if (live) {
#pragma unroll
            for (int j = 0; j < kVec; ++j) raw[k][j] = __ldg(src + j);
        } else {
#pragma unroll
            for (int j = 0; j < kVec; ++j) raw[k][j] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
#pragma unroll
    for (uint32_t k = 0; k < kMaxTilesPerCta<kDt>; ++k) {
        if (k >= ntile) break;
        const uint32_t slot = k * kSweepThreads + threadIdx.x;
        uint32_t row = (tile0 + k) * kSweepThreads + threadIdx.x;
        uint32_t key = 127u;
        if (row < job.rows) {
            float2 w[8];
            unstage_block<kDt>(raw[k], w);
            float a1 = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j) a1 = fmaxf(a1, fmaxf(fabsf(w[j].x), fabsf(w[j].y)));
            if (a1 > 0.0f) {
                const float t0 = __fmul_rn(a1, k6);
                key = min(cvt_e4m3x2(t0, t0) & 0x7Fu, 126u);
            }
        } else {
            row = kNoRow;
        }
#pragma unroll
        for (int j = 0; j < kVec; ++j) sw[slot][j] = raw[k][j];
        srow[slot] = row;
        keys[k] = key;
        ranks[k] = atomicAdd(&hist[key], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {                     // exclusive scan of the 128 bucket counts
        const uint32_t l = threadIdx.x;
        const uint32_t h0 = hist[4 * l], h1 = hist[4 * l + 1], h2 = hist[4 * l + 2], h3 = hist[4 * l + 3];
        uint32_t sum = h0 + h1 + h2 + h3, incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
            if (l >= (uint32_t)o) incl += t;
        }
        const uint32_t ex = incl - sum;
        base[4 * l] = ex;
        base[4 * l + 1] = ex + h0;
        base[4 * l + 2] = ex + h0 + h1;
        base[4 * l + 3] = ex + h0 + h1 + h2;
    }
    __syncthreads();
#pragma unroll
    for (uint32_t k = 0; k < kMaxTilesPerCta<kDt>; ++k) {
        if (k >= ntile) break;
        perm[base[keys[k]] + ranks[k]] = (uint16_t)(k * kSweepThreads + threadIdx.x);
    }
    __syncthreads();
    if (threadIdx.x == 0) n_redo = 0u;                       // base[] has been read by every thread
    __syncthreads();

    // ---- each warp walks interleaved groups of 32 sorted rows, without further barriers
    const bool pr = bound_ok != 0;                           // written by warp 3 before the barriers above
    const uint32_t nslots = ntile * kSweepThreads;
    const uint32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;
#pragma unroll 1
    for (uint32_t g = warp; 32u * g < nslots; g += kSweepThreads / 32) {
        const uint32_t slot = perm[32u * g + lane];
        const uint32_t row = srow[slot];
        float2 w[8];
        unstage_block<kDt>(sw[slot], w);
        if (row == kNoRow) continue;

        // ---- the search for this thread's (row, b)
        uint32_t flags = s2flag;
        float a1 = 0.0f, a2 = 0.0f, d1 = 0.0f, d2 = 0.0f;   // two largest |w_i|, their bound weights
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float x = k & 1 ? w[k >> 1].y : w[k >> 1].x;
            if (!isfinite(x)) flags |= kFlagNonFinite;
            const float a = fabsf(x), d = rd[k];
            if (a > a1) { a2 = a1; d2 = d1; a1 = a; d1 = d; }
            else if (a > a2) { a2 = a; d2 = d; }
        }
        // the threshold a candidate's lower bound must exceed to be skipped: the
        // runner-up cost when it is an output, else the best cost
        const bool need2 = job.cost2 != nullptr;
        float best = __int_as_float(0x7F800000), second = best, thr = best;
        uint32_t best_c = 0u;
        bool redo = false, tie = false;   // tie: another code reached exactly the best FP32 cost
        if (a1 == 0.0f) {
            best = 0.0f;                  // all-zero block: every candidate has e = w = 0
        } else if (!pr || ((job.cost1 != nullptr || job.cost2 != nullptr) &&
                           *reinterpret_cast<volatile float*>(&eta_s) > kCertifiedEta)) {
            redo = true;                  // no valid bound, or costs that FP32 cannot certify:
        } else {                          // all 127 candidates, in FP64
            const float t0 = __fmul_rn(a1, k6);
            int c = (int)min(cvt_e4m3x2(t0, t0) & 0x7Fu, 126u);
            int dn = c - 1, up = c + 1;
            bool go_dn = true;
#pragma unroll 1
            while (c >= 0) {
                // scheduling fence: keeps the compiler from pulling the next candidate's
                // work into this iteration; without it the kernel spills 332 bytes at 72
                // registers and takes 1.71 ms instead of 1.34 ms on the Gemma-like layer
                { const uint32_t am = __activemask(); asm volatile("" :: "r"(am)); }
                const float4 t = tab[c];
                const float2 nS = make_float2(-t.x, -t.x);
                float2 e[8];
                // first half (elements 0..7): codes, e and its part of bound (1); the bound
                // takes the lower-end codes, the quadratic form the exact ones
                const bool exact_t = t.w != 0.0f;
                uint32_t c0, c1 = 0u;
                if (exact_t) codes8h(w, t, c0); else c0 = codes8h_lo(w, t);
                {
                    float2 v[4];
                    decode8h(c0, v);
#pragma unroll
                    for (int k = 0; k < 4; ++k) e[k] = __ffma2_rn(v[k], nS, w[k]);
                }
                float lb = bound_half(e, rd4);
                ++nhalf;
                if (!pr || !(lb * kPruneScale > thr)) {               // the second half is still needed
                    ++nhalf;
                    if (exact_t) codes8h(w + 4, t, c1); else c1 = codes8h_lo(w + 4, t);
                    {
                        float2 v[4];
                        decode8h(c1, v);
#pragma unroll
                        for (int k = 0; k < 4; ++k) e[4 + k] = __ffma2_rn(v[k], nS, w[4 + k]);
                    }
                    lb += bound_half(e + 4, rd4 + 2);
                    if (!pr || !(lb * kPruneScale > thr)) {
                        if (!exact_t) {                                 // exact codes, e where they differ
                            const uint32_t x0 = codes8h_exact_from(w, t, c0);
                            const uint32_t x1 = codes8h_exact_from(w + 4, t, c1);
                            if (x0 != c0) {
                                float2 v[4];
                                decode8h(x0, v);
#pragma unroll
                                for (int k = 0; k < 4; ++k) e[k] = __ffma2_rn(v[k], nS, w[k]);
                            }
                            if (x1 != c1) {
                                float2 v[4];
                                decode8h(x1, v);
#pragma unroll
                                for (int k = 0; k < 4; ++k) e[4 + k] = __ffma2_rn(v[k], nS, w[4 + k]);
                            }
                        }
                        ++nfull;
                        const float cost = quad_form(e, hp);
                        if (cost < best || (cost == best && (uint32_t)c < best_c)) {
                            if (cost < best) { second = best; tie = false; } else tie = true;
                            best = cost;
                            best_c = (uint32_t)c;
                        } else if (cost == best) {
                            tie = true;
                        } else if (cost < second) {
                            second = cost;
                        }
                        thr = need2 ? second : best;
                    }
                }
                // next candidate: alternate down / up; bound (2) closes the downward walk and
                // bound (3), checked at every fourth upward code up to 110 (long upward walks
                // only: rows whose starting code is low, such as heavy-tailed expert weights;
                // on the Gemma-like layer, whose starting codes are ~115, it would save less
                // than it costs), the upward one
                bool take_dn = dn >= 0 && (go_dn || up > 126);
                if (!take_dn && pr && (up & 3) == 0 && up <= 110) {
                    const float h = 0.5f * tab[up].x;
                    float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const float ax = fabsf(w[k].x), ay = fabsf(w[k].y);
                        const float gx = ax <= h ? fminf(ax, h - ax) : 0.0f;
                        const float gy = ay <= h ? fminf(ay, h - ay) : 0.0f;
                        const float4 d = rd4[k >> 1];
                        const float2 dk = (k & 1) ? make_float2(d.z, d.w) : make_float2(d.x, d.y);
                        acc = __ffma2_rn(__fmul2_rn(dk, make_float2(gx, gy)), make_float2(gx, gy), acc);
                    }
                    if ((acc.x + acc.y) * kPruneScale > thr) {
                        up = 127;
                        take_dn = dn >= 0;
                    }
                }
                if (take_dn && pr) {
                    const float S = tab[dn].x;
                    const float u1 = fmaxf(fmaf(-6.0f, S, a1), 0.0f), u2 = fmaxf(fmaf(-6.0f, S, a2), 0.0f);
                    if (fmaf(d1 * u1, u1, d2 * u2 * u2) * kPruneScale > thr) {
                        dn = -1;
                        take_dn = false;
                    }
                }
                if (take_dn) { c = dn--; go_dn = false; }
                else if (up <= 126) { c = up++; go_dn = true; }
                else c = -1;
            }
            // FP32 costs exact to eta relative: a runner-up within 3 eta of the winner (or
            // costs that are outputs) needs the FP64 search unless eta certifies the argmin
            // (eta and the cost outputs are read here, not held through the walk)
            const float eta = *reinterpret_cast<volatile float*>(&eta_s);
            redo = eta > kCertifiedEta && (job.cost1 != nullptr || job.cost2 != nullptr || tie ||
                                           !(second > fmaf(best, 3.0f * eta, best)));
        }
        if (redo) {                       // decided later by the FP64 search of a whole warp
            flag_or(p.d_flags, flags);
            redo_list[atomicAdd(&n_redo, 1u)] = (uint16_t)slot;
            continue;
        }
        if (!isfinite(best)) flags |= kFlagNonFinite;

        const int64_t blk = (int64_t)row * job.nblk + b;
        job.codes[blk] = (uint8_t)best_c;
        if (job.q != nullptr) {
            uint32_t c0, c1;
            const float4 tw = tab[best_c];
            codes8h(w, tw, c0);
            codes8h(w + 4, tw, c1);
            *reinterpret_cast<uint2*>(job.q + blk * 8) = make_uint2(c0, c1);
        }
        if (job.cost1 != nullptr) job.cost1[blk] = best;
        if (job.cost2 != nullptr) job.cost2[blk] = second;
        flag_or(p.d_flags, flags);
    }

    // ---- blocks whose FP32 costs do not certify the argmin: exhaustive FP64 search, one warp each
    __syncthreads();
    if (n_redo != 0u) {
        const uint32_t done = redo_phase<kDt>(job, b, n_redo, redo_list, sw, srow, tab, hs, p.d_flags);
        nhalf += 2u * 127u * done;
        nfull += 127u * done;
    }
    if (job.d_work != nullptr) {
        __syncwarp();
        const uint32_t sv = __reduce_add_sync(0xffffffffu, nhalf), sf = __reduce_add_sync(0xffffffffu, nfull);
        if ((threadIdx.x & 31) == 0 && sv != 0u) {
            atomicAdd(job.d_work, (unsigned long long)sv);
            atomicAdd(job.d_work + 1, (unsigned long long)sf);
        }
    }
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
        d.cost1 = J.cost1; d.cost2 = J.cost2; d.d_work = J.d_work; d.ld = J.ld;
        d.rows = (uint32_t)J.rows;
        d.nblk = (uint32_t)(J.cols / 16);
        d.row_tiles = (d.rows + kSweepThreads - 1) / kSweepThreads;
    }
    // tiles per CTA: amortize the per-column setup while keeping >= ~16 CTAs per SM
    uint64_t tiles = 0;
    for (int i = 0; i < m; ++i) tiles += (uint64_t)p.jobs[i].row_tiles * p.jobs[i].nblk;
    const uint64_t per = tiles / ((uint64_t)num_sms() * 16u);
    const uint64_t cap = (uint64_t)(dt == 0 ? kMaxTilesPerCta<0> : kMaxTilesPerCta<2>);
    p.tiles_per_cta = (uint32_t)(per < 1 ? 1 : (per > cap ? cap : per));
    for (int i = 0; i < m; ++i) {
        SweepJobDev& d = p.jobs[i];
        d.cta_begin = ctas;
        ctas += ((d.row_tiles + p.tiles_per_cta - 1) / p.tiles_per_cta) * d.nblk;
    }
    p.n = m;
    if (m == 0) return cudaSuccess;
    if (dt == 0) sweep_kernel<0><<<ctas, kSweepThreads, 0, s>>>(p);
    else sweep_kernel<2><<<ctas, kSweepThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace nv4
