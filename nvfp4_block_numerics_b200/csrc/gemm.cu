// gemm.cu -- NVFP4 x NVFP4 block-scaled GEMM on the 5th-generation tensor cores (sm_100a).
//
// [FP4] section 4.1 (block-scaled FP4 matrix multiply with tcgen05.mma and scale
// factors reorganized for it), [CAST] section 4 (W4A4: activations and weights both
// NVFP4).  D[m, n] = s2_A * s2_B * sum_k (e2m1(a_mk) * sA[m, k/16]) * (e2m1(b_nk) * sB[n, k/16]),
// i.e. the product of the two dequantized matrices, accumulated in FP32 and written
// as BF16 or FP32.
//
// Kernel structure: persistent, one CTA per SM walking the 128 x kBN output tiles
// t = blockIdx.x, + gridDim.x, ... (kBN = 256 when N allows, else 128); 192 threads:
//   * warp 4, one lane: producer.  Per stage of 256 K-elements it loads the A and B code
//     tiles (128 rows x 128 bytes each) with 2-D TMA into 128-byte-swizzled shared
//     memory, and the stage's scale-factor atoms (4 x 512 bytes per operand, already in
//     the MMA layout, see nv4_scales_to_mma_layout) with 1-D bulk copies, all completing
//     on the stage's mbarrier.  A 4-stage ring that runs across tiles: while the epilogue
//     drains one tile, the first stages of the next are already loading.  A stage is
//     reused once the MMAs that read it have completed (tcgen05.commit on "empty").
//   * warp 5: allocates the tensor memory (the 128 x kBN FP32 accumulator and two
//     scale-factor buffers); one lane waits until the epilogue has read the previous
//     tile's accumulator ("acc_empty"), then per stage issues tcgen05.cp of the scale
//     atoms into tensor memory and four tcgen05.mma kind::mxf4nvf4 block16 (K = 64 each)
//     with both operands read from shared memory through matrix descriptors, and commits
//     "acc_full" after the tile's last stage.
//   * warps 0-3: epilogue.  Warp w reads accumulator lanes 32w..32w+31 with tcgen05.ld (one
//     output row per thread), multiplies by s2_A * s2_B, stores, and arrives on acc_empty.
// The accumulator is single-buffered (a second 256-column one does not fit the 512 columns
// next to the scale buffers), so the epilogue still runs between two tiles' MMAs.
// Every mbarrier wait is bounded (kWaitLimitNs); on expiry the kernel sets
// NV4_FLAG_TIMEOUT, every role stops, the stores are skipped, copies in flight are
// drained and the tensor memory is released.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "nv4_async.cuh"
#include "nv4_common.cuh"
#include "nv4_internal.h"

namespace nv4 {

namespace gemm {

constexpr int kBM = 128;
constexpr int kBK = 256;                          // FP4 elements per stage (128 bytes per row)
constexpr int kStages = 4;
constexpr int kThreads = 192;                     // warps 0-3 epilogue, 4 producer, 5 MMA issuer

// Tile width kBN = 128 or 256 (one MMA of 128 x kBN x 64 per K-step).
template <int kBN>
struct Cfg {
    static constexpr uint32_t kATile = 128 * 128;                    // A codes per stage
    static constexpr uint32_t kBTile = kBN * 128;                    // B codes per stage
    static constexpr uint32_t kSfA = 4 * 512;                        // 4 K-steps x one 128-row atom
    static constexpr uint32_t kSfB = (kBN / 128) * 4 * 512;
    static constexpr uint32_t kStageTx = kATile + kBTile + kSfA + kSfB;
    static constexpr uint32_t kTmemCols = kBN == 128 ? 256 : 512;   // power of two >= accumulator + scales
    static constexpr uint32_t kColSfA = kBN;                         // two 16-column buffers
    static constexpr uint32_t kSfBCols = 16 * (kBN / 128);           // per buffer
    static constexpr uint32_t kColSfB = kBN + 32;                    // two buffers
    // Instruction descriptor of kind::mxf4nvf4: A and B E2M1 (format 1), K-major, scale
    // factors UE4M3 (bit 23 = 0), N >> 3 in bits 17-22, M >> 4 in bits 24-28, dense K = 64.
    static constexpr uint32_t kIdesc =
        (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
};

template <int kBN>
struct Smem {
    uint8_t a[kStages][Cfg<kBN>::kATile];         // 1024-byte aligned (128-byte swizzle atoms)
    uint8_t b[kStages][Cfg<kBN>::kBTile];
    uint8_t sfa[kStages][Cfg<kBN>::kSfA];
    uint8_t sfb[kStages][Cfg<kBN>::kSfB];
    uint64_t full[kStages], empty[kStages], acc_full, acc_empty, drain;
    uint32_t tmem_base;
    uint32_t abort;                               // set by a wait that gave up
    uint32_t issued, consumed;                    // stages loaded / stages handed to the MMA
};

struct Params {
    CUtensorMap map_a, map_b;                     // codes [rows, K/2] bytes, 128 x 128-byte boxes
    const uint8_t* sfa;                           // scale atoms in the MMA layout
    const uint8_t* sfb;
    const float* d_s2a;
    const float* d_s2b;
    void* out;
    int64_t ldd;
    uint32_t n_tiles, k_stages, kt4;              // kt4 = K / 64: scale atoms per 128-row tile
    uint32_t tiles;                               // output tiles in all
    uint32_t* d_flags;
};

// ---------------------------------------------------------------- PTX helpers
// Shared-memory matrix descriptor (Blackwell format): start address, leading and
// stride byte offsets in 16-byte units, descriptor version 1 (bits 46-47) and the
// layout/swizzle mode in bits 61-63 (0 none, 2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout)
{
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)(lbo & 0x3FFFu) << 16) |
           ((uint64_t)(sbo & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Copies one 512-byte scale atom (32 rows x 16 bytes) into 4 tensor-memory columns,
// replicated over the four 32-lane sub-partitions.
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t desc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

__device__ __forceinline__ void mma_fp4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t sfa, uint32_t sfb, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
                 "}"
                 ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
                 : "memory");
}

// Arrives on mbar once every tcgen05 operation issued so far by this thread completes.
__device__ __forceinline__ void tc_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 consecutive FP32 accumulator columns of this warp's 32 lanes (one row per thread).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float v[32])
{
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
                 "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
                   "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
                   "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
                   "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

}  // namespace gemm

namespace gemm {

template <int kBN, int kOut>   // tile width 128 | 256; output 0 bf16, 2 fp32
__global__ void __launch_bounds__(kThreads, 1)
gemm_nvfp4_kernel(const __grid_constant__ Params p)
{
    using C = Cfg<kBN>;
    extern __shared__ uint8_t smem_raw[];
    Smem<kBN>& sm = *reinterpret_cast<Smem<kBN>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t KS = p.k_stages;

    if (threadIdx.x == 128) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.acc_full, 1);
        mbar_init(&sm.acc_empty, 4);                               // one arrival per epilogue warp
        mbar_init(&sm.drain, 1);
        sm.abort = 0u;
        sm.issued = sm.consumed = 0u;
        mbar_init_fence();
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.map_a)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.map_b)) : "memory");
    }
    if (warp == 5) tmem_alloc(&sm.tmem_base, C::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    uint32_t flags = 0u;
    auto aborted = [&]() { return *reinterpret_cast<volatile uint32_t*>(&sm.abort) != 0u; };

    if (warp == 4) {
        if (lane == 0) {                                           // producer, running ahead across tiles
            uint32_t g = 0;
            for (uint32_t t = blockIdx.x; t < p.tiles && !aborted(); t += gridDim.x) {
                const uint32_t n_tile = t % p.n_tiles, m_tile = t / p.n_tiles;
                for (uint32_t ks = 0; ks < KS; ++ks, ++g) {
                    const uint32_t s = g % kStages;
                    if (g >= (uint32_t)kStages && !mbar_wait(&sm.empty[s], ((g / kStages) - 1u) & 1u)) {
                        flags |= kFlagTimeout;
                        atomicOr(&sm.abort, 1u);
                    }
                    if (aborted()) break;
                    mbar_arrive_expect_tx(&sm.full[s], C::kStageTx);
                    tma_load_2d(sm.a[s], &p.map_a, &sm.full[s], (int)(ks * 128u), (int)(m_tile * kBM));
                    tma_load_2d(sm.b[s], &p.map_b, &sm.full[s], (int)(ks * 128u), (int)(n_tile * kBN));
                    bulk_load(sm.sfa[s], p.sfa + ((size_t)m_tile * p.kt4 + 4u * ks) * 512u, C::kSfA, &sm.full[s]);
#pragma unroll
                    for (uint32_t h = 0; h < (uint32_t)(kBN / 128); ++h)  // one run of 4 atoms per 128 rows
                        bulk_load(sm.sfb[s] + 2048u * h,
                                  p.sfb + ((size_t)(n_tile * (kBN / 128) + h) * p.kt4 + 4u * ks) * 512u, 2048u,
                                  &sm.full[s]);
                }
            }
            sm.issued = g;
        }
        __syncwarp();
    } else if (warp == 5) {
        if (lane == 0) {                                           // MMA issuer
            uint32_t g = 0, i = 0;
            for (uint32_t t = blockIdx.x; t < p.tiles && !aborted(); t += gridDim.x, ++i) {
                // the accumulator is free once the epilogue has read the previous tile
                if (i > 0 && !mbar_wait(&sm.acc_empty, (i - 1u) & 1u)) {
                    flags |= kFlagTimeout;
                    atomicOr(&sm.abort, 1u);
                    break;
                }
                tc_fence_after();
                for (uint32_t ks = 0; ks < KS; ++ks, ++g) {
                    const uint32_t s = g % kStages;
                    if (!mbar_wait(&sm.full[s], (g / kStages) & 1u)) {
                        flags |= kFlagTimeout;
                        atomicOr(&sm.abort, 1u);
                        break;
                    }
                    tc_fence_after();
                    const uint32_t buf = g & 1u;
                    // scale columns: A row r of K-step j at column ta + 4j + r/32; B row n at tb + nb*j + n/32
                    constexpr uint32_t nb = 4u * (kBN / 128);
                    const uint32_t ta = tmem + C::kColSfA + 16u * buf, tb = tmem + C::kColSfB + C::kSfBCols * buf;
#pragma unroll
                    for (uint32_t j = 0; j < 4; ++j) {
                        tmem_cp_sf(ta + 4u * j, smem_desc(smem_u32(sm.sfa[s] + 512u * j), 0u, 8u, 0u));
#pragma unroll
                        for (uint32_t h = 0; h < (uint32_t)(kBN / 128); ++h)
                            tmem_cp_sf(tb + nb * j + 4u * h, smem_desc(smem_u32(sm.sfb[s] + 2048u * h + 512u * j), 0u, 8u, 0u));
                    }
                    const uint32_t a0 = smem_u32(sm.a[s]), b0 = smem_u32(sm.b[s]);
#pragma unroll
                    for (uint32_t j = 0; j < 4; ++j)
                        mma_fp4(tmem, smem_desc(a0 + 32u * j, 1u, 64u, 2u), smem_desc(b0 + 32u * j, 1u, 64u, 2u),
                                C::kIdesc, ta + 4u * j, tb + nb * j, (ks | j) != 0u ? 1u : 0u);
                    tc_commit(&sm.empty[s]);                       // frees the stage when these MMAs finish
                }
                if (aborted()) break;
                tc_commit(&sm.acc_full);                           // this tile's accumulator is complete
            }
            sm.consumed = g;
            tc_commit(&sm.drain);                                  // every tensor-core operation issued
            if (!mbar_wait(&sm.drain, 0u)) flags |= kFlagTimeout;
        }
        __syncwarp();
    } else {
        // ---- epilogue warps 0-3: accumulator lanes 32w..32w+31, one output row per thread
        const float alpha = __fmul_rn(*p.d_s2a, *p.d_s2b);
        uint32_t i = 0;
        for (uint32_t t = blockIdx.x; t < p.tiles; t += gridDim.x, ++i) {
            const bool ok = !aborted() && mbar_wait(&sm.acc_full, i & 1u);
            if (!ok) {
                if (!aborted()) { flags |= kFlagTimeout; atomicOr(&sm.abort, 1u); }
                break;
            }
            tc_fence_after();
            __syncwarp();
            const uint32_t n_tile = t % p.n_tiles, m_tile = t / p.n_tiles;
            const int64_t row = (int64_t)m_tile * kBM + 32 * warp + lane;
#pragma unroll 1
            for (int cb = 0; cb < kBN / 32; ++cb) {
                float v[32];
                tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)(32 * cb), v);
                const int64_t col = (int64_t)n_tile * kBN + 32 * cb;
                if constexpr (kOut == 2) {
                    float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * p.ldd + col);
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        o[k] = make_float4(__fmul_rn(v[4 * k], alpha), __fmul_rn(v[4 * k + 1], alpha),
                                           __fmul_rn(v[4 * k + 2], alpha), __fmul_rn(v[4 * k + 3], alpha));
                } else {
                    uint32_t w[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        asm("cvt.rn.bf16x2.f32 %0, %1, %2;"
                            : "=r"(w[k])
                            : "f"(__fmul_rn(v[2 * k + 1], alpha)), "f"(__fmul_rn(v[2 * k], alpha)));
                    uint4* o = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + row * p.ldd + col);
#pragma unroll
                    for (int k = 0; k < 4; ++k) o[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.acc_empty);             // this warp has read the accumulator
        }
    }

    // ---- teardown: drain copies that were loaded but never consumed, free tensor memory
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 128) {
        for (uint32_t g = sm.consumed; g < sm.issued; ++g)
            if (!mbar_wait(&sm.full[g % kStages], (g / kStages) & 1u)) flags |= kFlagTimeout;
    }
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
    flags = __reduce_or_sync(0xFFFFFFFFu, flags);
    if (lane == 0) flag_or(p.d_flags, flags);
}

// Block scales [rows, kb] (row-major, kb = K/16) -> the MMA atom layout, one thread per
// 32-bit word (one row's 4 consecutive scales); padding rows and columns are zero.
__global__ void __launch_bounds__(256)
mma_scale_layout_kernel(const uint8_t* __restrict__ sc, uint32_t rows, uint32_t kb, uint32_t kt,
                        uint32_t total_words, uint32_t* __restrict__ out)
{
    for (uint32_t w = blockIdx.x * 256u + threadIdx.x; w < total_words; w += gridDim.x * 256u) {
        // word w = ((rt * kt) + g) * 128 + (r % 32) * 4 + (r % 128) / 32
        const uint32_t atom = w >> 7, in = w & 127u;
        const uint32_t rt = atom / kt, g = atom - rt * kt;
        const uint32_t r = rt * 128u + (in >> 2) + 32u * (in & 3u);
        uint32_t v = 0u;
        if (r < rows) {
            const uint8_t* src = sc + (size_t)r * kb + 4u * g;
#pragma unroll
            for (uint32_t j = 0; j < 4; ++j)
                if (4u * g + j < kb) v |= (uint32_t)src[j] << (8u * j);
        }
        out[w] = v;
    }
}

static PFN_cuTensorMapEncodeTiled_v12000 encoder()
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

static bool code_map(CUtensorMap* map, const uint8_t* q, int64_t rows, int64_t K, uint32_t box_rows)
{
    auto enc = encoder();
    if (enc == nullptr) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    const cuuint32_t box[2] = {128u, box_rows};
    const cuuint32_t es[2] = {1u, 1u};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(q), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace gemm

size_t mma_scale_bytes(int64_t rows, int64_t kb)
{
    return (size_t)((rows + 127) / 128) * 128u * (size_t)((kb + 3) / 4) * 4u;
}

cudaError_t launch_mma_scale_layout(const uint8_t* sc, int64_t rows, int64_t kb, uint8_t* out, cudaStream_t s)
{
    const uint32_t kt = (uint32_t)((kb + 3) / 4);
    const uint32_t words = (uint32_t)(mma_scale_bytes(rows, kb) / 4u);
    int64_t need = ((int64_t)words + 255) / 256;
    const int64_t cap = (int64_t)num_sms() * 8;
    const int grid = (int)(need < cap ? (need > 0 ? need : 1) : cap);
    gemm::mma_scale_layout_kernel<<<grid, 256, 0, s>>>(sc, (uint32_t)rows, (uint32_t)kb, kt, words,
                                                       reinterpret_cast<uint32_t*>(out));
    return cudaGetLastError();
}

cudaError_t launch_gemm_nvfp4(const uint8_t* qa, const uint8_t* sfa, const float* d_s2a, const uint8_t* qb,
                              const uint8_t* sfb, const float* d_s2b, int64_t M, int64_t N, int64_t K, int out_dt,
                              void* out, int64_t ldd, uint32_t* d_flags, cudaStream_t s)
{
    using namespace gemm;
    Params p;
    const bool wide = N % 256 == 0;
    const int bn = wide ? 256 : 128;
    if (!code_map(&p.map_a, qa, M, K, 128u) || !code_map(&p.map_b, qb, N, K, (uint32_t)bn)) return cudaErrorInvalidValue;
    p.sfa = sfa;
    p.sfb = sfb;
    p.d_s2a = d_s2a;
    p.d_s2b = d_s2b;
    p.out = out;
    p.ldd = ldd;
    p.n_tiles = (uint32_t)(N / bn);
    p.k_stages = (uint32_t)(K / kBK);
    p.kt4 = (uint32_t)(K / 64);
    p.tiles = (uint32_t)((M / kBM) * (N / bn));
    p.d_flags = d_flags;
    const size_t smem = (wide ? sizeof(Smem<256>) : sizeof(Smem<128>)) + 1024;
    static bool attr_set[4][64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int o = out_dt == 2 ? 1 : 0;
    const int v = 2 * (wide ? 1 : 0) + o;
    auto kern = wide ? (o ? gemm_nvfp4_kernel<256, 2> : gemm_nvfp4_kernel<256, 0>)
                     : (o ? gemm_nvfp4_kernel<128, 2> : gemm_nvfp4_kernel<128, 0>);
    if (dev < 0 || dev >= 64 || !attr_set[v][dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[v][dev] = true;
    }
    const unsigned grid = (unsigned)(p.tiles < (uint32_t)num_sms() ? p.tiles : (uint32_t)num_sms());
    kern<<<grid, kThreads, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace nv4
