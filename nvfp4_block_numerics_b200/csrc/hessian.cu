// hessian.cu -- local Hessian H_b += X_b^T X_b per 16-channel block (sm_100a).
//
// [CAL] section 2 step 2: with full-precision weights, accumulate H = sum X^T X per
// block of 16 input channels at each layer input (see nv4.h).
//
// The useful work is the block diagonal of the Gram matrix X^T X: 2*16 FLOP per
// byte of BF16 input, so at HBM speed the contraction needs ~100 TFLOP/s, above
// what the FP32 pipe delivers.  It runs on the tensor cores with the m16n8k16
// BF16 MMA, whose 16x16 output tile is exactly one H_b, so no FLOP is spent off
// the diagonal (a 64- or 128-wide tcgen05 tile would compute 4x-8x more than
// needed).  Products of BF16 values are exact; accumulation is FP32.
//
// Data movement:
//   * a CTA owns a slab of 16*kBlk channels (kBlk = 8 or 4 blocks: 128 or 64 channels)
//     and a range of 64-token tiles;
//   * one producer warp streams [64 tokens x slab] stages with 2-D TMA loads (boxes of
//     64 x 64 BF16, 128-byte swizzle) into a shared-memory ring guarded by mbarriers;
//     ragged token or channel edges are zero-filled by the TMA unit;
//   * consumer warp w owns blocks 2w and 2w+1 over every token of the stage: one
//     ldmatrix.x4.trans per 16x16 sub-tile yields the MMA A fragment of X_b^T, and the
//     same four registers are the B fragments of X_b (A[m][k] = X[k][m], B[k][n] =
//     X[k][n]); the MMA accumulators are flushed every 128 tokens into a second FP32
//     sum;
//   * the token range of a slab is split over the CTAs of a thread-block cluster;
//     partials are summed in a fixed order (cluster ranks, through distributed shared
//     memory) and added to H by cluster rank 0, so the result is bit-reproducible.
// Every mbarrier wait is bounded (kWaitLimitNs); on expiry the kernel sets
// NV4_FLAG_TIMEOUT, stops issuing, drains its own copies in flight and finishes.
#include <algorithm>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "nv4_async.cuh"
#include "nv4_common.cuh"
#include "nv4_internal.h"

namespace nv4 {

constexpr int kTok = 64;                 // tokens per stage
constexpr int kMaxCluster = 8;
constexpr uint32_t kBoxBytes = kTok * 64 * 2;   // one 64x64 BF16 TMA box

// Slab configuration: kBlk 16-channel blocks per CTA, two per consumer warp.
template <int kBlk>
struct HCfg {
    static constexpr int kWarpsC = kBlk / 2;
    static constexpr int kThreads = (kWarpsC + 1) * 32;
    static constexpr int kBoxes = kBlk / 4;
    static constexpr uint32_t kStageBytes = kBoxBytes * kBoxes;
    static constexpr int kStages = kBlk == 4 ? 8 : (kBlk == 8 ? 6 : 3);
    static constexpr uint32_t kFlushStages = 2;  // 128 tokens per FP32 accumulation chunk
};

struct HessJobDev {
    CUtensorMap tmap;                    // X as [tokens][cols] bf16, box 64x64, swizzle 128B
    float* H;
    uint32_t ntiles;                     // ceil(tokens / 64)
    uint32_t nblk;                       // cols / 16
    uint32_t slab_begin;                 // prefix sum of slabs over jobs
    uint32_t pad;
};

struct HessParams {
    int n;
    uint32_t* d_flags;
    HessJobDev jobs[kMaxHessianJobs];
};

template <int kBlk>
struct HessSmem {
    alignas(1024) uint8_t tiles[HCfg<kBlk>::kStages][HCfg<kBlk>::kStageBytes];
    alignas(8) uint64_t full[HCfg<kBlk>::kStages];
    uint64_t empty[HCfg<kBlk>::kStages];
    uint32_t consumed;                   // stages fully consumed (for draining on timeout)
    uint32_t timeout;
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t r[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                 "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}


// ------------------------------------------------------------------ kernel
template <int kBlk>
__global__ void __launch_bounds__(HCfg<kBlk>::kThreads)
hessian_kernel(const __grid_constant__ HessParams p)
{
    using Cfg = HCfg<kBlk>;
    constexpr int kStages = Cfg::kStages;
    extern __shared__ uint8_t smem_raw[];
    HessSmem<kBlk>& sm =
        *reinterpret_cast<HessSmem<kBlk>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    // job and slab of this CTA (blockIdx.y = global slab index)
    int j = 0;
    {
        int lo = 0, hi = p.n - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.jobs[mid].slab_begin <= blockIdx.y) lo = mid; else hi = mid - 1;
        }
        j = lo;
    }
    const HessJobDev& job = p.jobs[j];
    const uint32_t slab = blockIdx.y - job.slab_begin;
    const uint32_t rank = cluster_ctarank(), nrank = cluster_nctarank();
    const uint32_t t_begin = (uint32_t)(((uint64_t)job.ntiles * rank) / nrank);
    const uint32_t t_end = (uint32_t)(((uint64_t)job.ntiles * (rank + 1)) / nrank);
    const uint32_t ntile = t_end - t_begin;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], Cfg::kWarpsC);
        }
        sm.consumed = 0u;
        sm.timeout = 0u;
        mbar_init_fence();
    }
    __syncthreads();

    // acc: the MMA accumulators of the current 128-token chunk; tot: the sum of chunks.
    float acc[2][2][4], tot[2][2][4];
#pragma unroll
    for (int bk = 0; bk < 2; ++bk)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[bk][h][k] = tot[bk][h][k] = 0.0f;

    if (warp == Cfg::kWarpsC) {
        // ---------------- producer: one lane issues the TMA loads
        if (lane == 0) {
            uint32_t issued = 0;
            for (uint32_t i = 0; i < ntile; ++i) {
                const int s = (int)(i % kStages);
                if (i >= (uint32_t)kStages && !mbar_wait(&sm.empty[s], ((i / kStages) + 1u) & 1u)) {
                    atomicOr(&sm.timeout, 1u);
                    break;
                }
                if (*reinterpret_cast<volatile uint32_t*>(&sm.timeout)) break;
                mbar_arrive_expect_tx(&sm.full[s], Cfg::kStageBytes);
                const int x0 = (int)(slab * 16u * kBlk), y0 = (int)((t_begin + i) * kTok);
#pragma unroll
                for (int bx = 0; bx < Cfg::kBoxes; ++bx)
                    tma_load_2d(sm.tiles[s] + bx * kBoxBytes, &job.tmap, &sm.full[s], x0 + 64 * bx, y0);
                ++issued;
            }
            // drain: every issued copy must have landed before shared memory is reused
            const uint32_t done = *reinterpret_cast<volatile uint32_t*>(&sm.consumed);
            for (uint32_t i = done; i < issued; ++i)
                if (!mbar_wait(&sm.full[i % kStages], (i / kStages) & 1u)) atomicOr(&sm.timeout, 1u);
        }
    } else {
        // ---------------- consumers: warp w owns blocks 2w, 2w+1 of the slab
        const uint32_t row_in = (uint32_t)(lane & 7), mat = (uint32_t)(lane >> 3);
        const uint32_t box = (uint32_t)(2 * warp) / 4u;                      // both blocks share a box
        const uint32_t chunk0 = (uint32_t)(2 * (2 * warp % 4)) + (mat & 1u); // 16-byte chunk of block 2w
        for (uint32_t i = 0; i < ntile; ++i) {
            const int s = (int)(i % kStages);
            if (!mbar_wait(&sm.full[s], (i / kStages) & 1u)) {
                atomicOr(&sm.timeout, 1u);
                break;
            }
            const uint32_t base = smem_u32(sm.tiles[s] + box * kBoxBytes);
#pragma unroll
            for (int g = 0; g < 4; ++g) {                                  // 16-token groups
                const uint32_t tok = (uint32_t)(16 * g) + (mat >> 1) * 8u + row_in;
                const uint32_t rowb = base + tok * 128u;
#pragma unroll
                for (int bk = 0; bk < 2; ++bk) {
                    const uint32_t chunk = chunk0 + 2u * (uint32_t)bk;
                    uint32_t a[4];
                    ldmatrix_x4_trans(rowb + ((chunk ^ (tok & 7u)) << 4), a);
                    mma_bf16_16816(acc[bk][0], a, a[0], a[2]);
                    mma_bf16_16816(acc[bk][1], a, a[1], a[3]);
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm.empty[s]);
                if (warp == 0) atomicMax(&sm.consumed, i + 1u);
            }
            if ((i + 1u) % Cfg::kFlushStages == 0u) {
#pragma unroll
                for (int bk = 0; bk < 2; ++bk)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            tot[bk][h][k] += acc[bk][h][k];
                            acc[bk][h][k] = 0.0f;
                        }
            }
            if (*reinterpret_cast<volatile uint32_t*>(&sm.timeout)) break;
        }
#pragma unroll
        for (int bk = 0; bk < 2; ++bk)
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int k = 0; k < 4; ++k) tot[bk][h][k] += acc[bk][h][k];
    }
    __syncthreads();

    // ---------------- CTA partial in shared memory: [kBlk blocks][256]
    float* part = reinterpret_cast<float*>(sm.tiles[0]);
    if (warp < Cfg::kWarpsC) {
        const int g = lane >> 2, c = lane & 3;
#pragma unroll
        for (int bk = 0; bk < 2; ++bk)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float* P = part + (2 * warp + bk) * 256;
                const int n0 = 8 * h + 2 * c;
                P[g * 16 + n0] = tot[bk][h][0];
                P[g * 16 + n0 + 1] = tot[bk][h][1];
                P[(g + 8) * 16 + n0] = tot[bk][h][2];
                P[(g + 8) * 16 + n0 + 1] = tot[bk][h][3];
            }
    }
    cluster_sync();

    // ---------------- cluster rank 0 sums the ranks in order and adds into H
    uint32_t flags = 0u;
    if (rank == 0) {
        for (int e = threadIdx.x; e < kBlk * 256; e += Cfg::kThreads) {
            const uint32_t bk = slab * (uint32_t)kBlk + (uint32_t)(e >> 8);
            if (bk >= job.nblk) continue;
            float sum = part[e];
            for (uint32_t r = 1; r < nrank; ++r) sum += ld_dsmem_f32(part + e, r);
            float* dst = job.H + (int64_t)bk * 256 + (e & 255);
            const float v = *dst + sum;
            *dst = v;
            if (!isfinite(v)) flags |= kFlagNonFinite;
        }
    }
    if (sm.timeout) flags |= kFlagTimeout;
    cluster_sync();                                              // keep shared memory alive for readers
    flags = __reduce_or_sync(0xFFFFFFFFu, flags);
    if (lane == 0) flag_or(p.d_flags, flags);
}

// ------------------------------------------------------------------ host side
static PFN_cuTensorMapEncodeTiled_v12000 get_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

template <int kBlk>
static cudaError_t launch_width(const HessParams& p, uint32_t slabs, uint32_t max_tiles, cudaStream_t s)
{
    using Cfg = HCfg<kBlk>;
    const size_t smem = sizeof(HessSmem<kBlk>) + 1024;
    // once per device and width (the first, eager call sets it; later calls may be captured)
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(hessian_kernel<kBlk>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    // cluster size: the largest that keeps every CTA of the launch resident at once (a
    // single wave, so all slabs -- and so all HBM channels -- stream together), each
    // CTA keeping at least 8 stages of work
    const uint32_t per_sm = (uint32_t)(200 * 1024 / smem) > 0 ? (uint32_t)(200 * 1024 / smem) : 1u;
    const uint32_t target = (uint32_t)num_sms() * per_sm;
    uint32_t z = 1;
    while (z < (uint32_t)kMaxCluster && slabs * (2u * z) <= target && max_tiles / (2u * z) >= 8u) z *= 2u;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(z, slabs, 1);
    cfg.blockDim = dim3(Cfg::kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = z;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, hessian_kernel<kBlk>, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_hessian(const nv4_hessian_job* jobs, int n, uint32_t* d_flags, cudaStream_t s, int* bad_job)
{
    *bad_job = -1;
    auto encode = get_encoder();
    if (encode == nullptr) return cudaErrorNotSupported;

    // slab width: 128 channels (256-byte row segments; measured best for the layer
    // inputs here), or 64 when 128-wide slabs cannot give every SM two CTAs
    uint64_t slabs128 = 0;
    uint32_t max_tiles = 0;
    for (int i = 0; i < n; ++i) {
        if (jobs[i].tokens == 0 || jobs[i].cols == 0) continue;
        slabs128 += (uint64_t)((jobs[i].cols + 127) / 128);
        const uint32_t t = (uint32_t)((jobs[i].tokens + kTok - 1) / kTok);
        if (t > max_tiles) max_tiles = t;
    }
    const uint64_t zmax = std::min<uint64_t>(kMaxCluster, std::max<uint64_t>(1u, max_tiles / 16u));
    const uint32_t width = slabs128 * zmax >= (uint64_t)num_sms() * 2u ? 128u : 64u;

    HessParams p;          // ~25 KB, copied into the launch's parameter buffer
    p.d_flags = d_flags;
    int m = 0;
    uint32_t slabs = 0;
    for (int i = 0; i < n; ++i) {
        const nv4_hessian_job& J = jobs[i];
        if (J.tokens == 0 || J.cols == 0) continue;
        HessJobDev& d = p.jobs[m];
        const cuuint64_t dims[2] = {(cuuint64_t)J.cols, (cuuint64_t)J.tokens};
        const cuuint64_t strides[1] = {(cuuint64_t)J.ld * 2u};
        const cuuint32_t box[2] = {64u, (cuuint32_t)kTok};
        const cuuint32_t estr[2] = {1u, 1u};
        const CUresult r = encode(&d.tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(J.x), dims,
                                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            *bad_job = i;
            return cudaErrorInvalidValue;
        }
        d.H = J.H;
        d.ntiles = (uint32_t)((J.tokens + kTok - 1) / kTok);
        d.nblk = (uint32_t)(J.cols / 16);
        d.slab_begin = slabs;
        slabs += (uint32_t)((J.cols + width - 1) / width);
        ++m;
    }
    p.n = m;
    if (m == 0) return cudaSuccess;
    if (width == 128u) return launch_width<8>(p, slabs, max_tiles, s);
    return launch_width<4>(p, slabs, max_tiles, s);
}

}  // namespace nv4
