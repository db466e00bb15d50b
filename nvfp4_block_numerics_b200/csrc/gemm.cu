// gemm.cu -- NVFP4 x NVFP4 block-scaled GEMM on the 5th-generation tensor cores (sm_100a).
//
// [FP4] section 4.1 (block-scaled FP4 matrix multiply with tcgen05.mma and scale
// factors reorganized for it), [CAST] section 4 (W4A4: activations and weights both
// NVFP4).  D[m, n] = s2_A * s2_B * sum_k (e2m1(a_mk) * sA[m, k/16]) * (e2m1(b_nk) * sB[n, k/16]),
// i.e. the product of the two dequantized matrices, accumulated in FP32 and written
// as BF16 or FP32.
//
// Kernel structure: persistent, one CTA per SM walking the 128 x kBN output tiles
// t = blockIdx.x, + gridDim.x, ... (kBN = 256 when N allows, else 128); 448 threads:
//   * warp 8, one lane: producer.  Per stage of 256 K-elements it loads the A and B code
//     tiles (128 rows x 128 bytes each) with 2-D TMA into 128-byte-swizzled shared
//     memory, and the stage's scale-factor atoms (4 x 512 bytes per operand, already in
//     the MMA layout, see nv4_scales_to_mma_layout) with 1-D bulk copies, all completing
//     on the stage's mbarrier.  A 4-stage ring that runs across tiles: while the epilogue
//     drains one tile, the first stages of the next are already loading.  A stage is
//     reused once the MMAs that read it have completed (tcgen05.commit on "empty").
//   * warps 4-7: scale writers, one per 32-lane tensor-memory sub-partition.  The
//     block-scaled MMA reads a K-step's scale factors from every sub-partition, so each
//     writer stores the stage's atoms into its own 32 lanes with tcgen05.st (48 or 32
//     columns per stage into one of kSfBufs buffers) and arrives on "sf_full".  Moving the
//     scales with tcgen05.st from four warps, instead of twelve tcgen05.cp 32x128b.warpx4
//     copies per stage issued by the MMA thread, takes the copies out of the tensor pipe's
//     instruction stream (8192^3: 2.85 -> 4.03 PFLOP/s; the copies cost per instruction,
//     not per byte).
//   * warp 9: allocates the tensor memory (the 128 x kBN FP32 accumulator and the scale
//     buffers); one lane waits until the epilogue has read the previous tile's accumulator
//     ("acc_empty"), then per stage waits for the codes and the scales and issues four
//     tcgen05.mma kind::mxf4nvf4 block16 (K = 64 each) with both operands read from shared
//     memory through matrix descriptors, commits "empty" and "sf_free", and commits
//     "acc_full" after the tile's last stage.
//   * warps 0-3 and 10-13: epilogue, two warps per 32-lane sub-partition, half the columns
//     each.  A warp reads its 32 rows x kBN/2 accumulator columns with tcgen05.ld (one row
//     per thread), multiplies by s2_A * s2_B and arrives on acc_empty; for BF16 the half
//     row is converted into registers first and stored only after the accumulator has been
//     released, so the stores overlap the next tile's MMAs, each 32 x 16 block transposed
//     through 1 KB of shared memory so that a store instruction writes 16 rows x 32
//     contiguous bytes instead of 32 rows x 16.
// The accumulator is single-buffered (a second 256-column one does not fit the 512 columns
// next to the scale buffers): the tensor pipe idles while the epilogue reads it.
//
// When M and N are multiples of 256 the product runs on CTA pairs instead (the kernel
// gemm_nvfp4_pair_kernel below: 256 x 256 tiles, the 2-SM MMA): 8192^3 +2%, 16384 x 16384 x
// 2048 +7%.  Its cross-CTA hand-offs use plain (CTA-scope) mbarrier waits and remote
// arrives: with cluster-scope acquire/release on them the same kernel ran 40% slower.
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
constexpr int kSfBufs = 4;                        // scale-factor buffers in tensor memory
constexpr int kThreads = 448;                     // warps 0-3, 10-13 epilogue, 4-7 scale writers, 8 producer, 9 MMA issuer
constexpr int kProducer = 256, kIssuer = 288;     // the two single-thread roles

// Tile width kBN = 128 or 256 (one MMA of 128 x kBN x 64 per K-step).
template <int kBN>
struct Cfg {
    static constexpr uint32_t kATile = 128 * 128;                    // A codes per stage
    static constexpr uint32_t kBTile = kBN * 128;                    // B codes per stage
    static constexpr uint32_t kSfA = 4 * 512;                        // 4 K-steps x one 128-row atom
    static constexpr uint32_t kSfB = (kBN / 128) * 4 * 512;
    static constexpr uint32_t kStageTx = kATile + kBTile + kSfA + kSfB;
    static constexpr uint32_t kTmemCols = kBN == 128 ? 256 : 512;   // power of two >= accumulator + scales
    static constexpr uint32_t kSfBCols = 16 * (kBN / 128);           // B scale columns per buffer
    static constexpr uint32_t kSfCols = 16 + kSfBCols;               // one buffer: A (16 columns), then B
    static_assert(kBN + kSfBufs * kSfCols <= kTmemCols, "tensor memory");
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
    uint8_t stg[8][1024];                         // per epilogue warp: 32 rows x 32 bytes, swizzled
    uint64_t full[kStages], empty[kStages], sf_full[kSfBufs], sf_free[kSfBufs], acc_full, acc_empty, drain;
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

// Writes n consecutive 32-bit tensor-memory columns of this warp's 32 lanes (one register
// per column and lane); the caller waits with tmem_st_wait before handing them on.
template <int n>
__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t (&v)[n]);

template <>
__device__ __forceinline__ void tmem_st<16>(uint32_t taddr, const uint32_t (&v)[16])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
                 "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
                 ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
                   "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
                   "r"(v[15])
                 : "memory");
}

template <>
__device__ __forceinline__ void tmem_st<32>(uint32_t taddr, const uint32_t (&v)[32])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
                 "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
                 "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
                 ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
                   "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
                   "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]),
                   "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]),
                   "r"(v[31])
                 : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

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

    if (threadIdx.x == kProducer) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < kSfBufs; ++b) {
            mbar_init(&sm.sf_full[b], 4);                          // one arrival per scale-writer warp
            mbar_init(&sm.sf_free[b], 1);
        }
        mbar_init(&sm.acc_full, 1);
        mbar_init(&sm.acc_empty, 8);                               // one arrival per epilogue warp
        mbar_init(&sm.drain, 1);
        sm.abort = 0u;
        sm.issued = sm.consumed = 0u;
        mbar_init_fence();
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.map_a)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.map_b)) : "memory");
    }
    if (warp == kIssuer / 32) tmem_alloc(&sm.tmem_base, C::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    uint32_t flags = 0u;
    auto aborted = [&]() { return *reinterpret_cast<volatile uint32_t*>(&sm.abort) != 0u; };

    if (warp == kProducer / 32) {
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
    } else if (warp == kIssuer / 32) {
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
                    const uint32_t b = g % kSfBufs;
                    if (!mbar_wait(&sm.full[s], (g / kStages) & 1u) ||
                        !mbar_wait(&sm.sf_full[b], (g / kSfBufs) & 1u)) {
                        flags |= kFlagTimeout;
                        atomicOr(&sm.abort, 1u);
                        break;
                    }
                    tc_fence_after();
                    // scale columns (written by the scale writers): A row r of K-step j at column
                    // ta + 4j + r/32, B row n at tb + nb*j + n/32
                    constexpr uint32_t nb = 4u * (kBN / 128);
                    const uint32_t ta = tmem + kBN + C::kSfCols * b, tb = ta + 16u;
                    const uint32_t a0 = smem_u32(sm.a[s]), b0 = smem_u32(sm.b[s]);
#pragma unroll
                    for (uint32_t j = 0; j < 4; ++j)
                        mma_fp4(tmem, smem_desc(a0 + 32u * j, 1u, 64u, 2u), smem_desc(b0 + 32u * j, 1u, 64u, 2u),
                                C::kIdesc, ta + 4u * j, tb + nb * j, (ks | j) != 0u ? 1u : 0u);
                    tc_commit(&sm.empty[s]);                       // frees the stage when these MMAs finish
                    tc_commit(&sm.sf_free[b]);                     // and the scale buffer
                }
                if (aborted()) break;
                tc_commit(&sm.acc_full);                           // this tile's accumulator is complete
            }
            sm.consumed = g;
            tc_commit(&sm.drain);                                  // every tensor-core operation issued
            if (!mbar_wait(&sm.drain, 0u)) flags |= kFlagTimeout;
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 8) {
        // ---- scale writers, warps 4-7 (tensor-memory sub-partition q = warp % 4, lanes
        // 32q..32q+31).  The block-scaled MMA reads the scale factors of a K-step from the
        // lanes of every sub-partition: row r of a 512-byte atom (32 rows x 16 bytes, rows r,
        // r+32, r+64, r+96 of the operand, 4 scales each) goes to lane 32q + r of every q, as
        // four consecutive columns.  Per stage each writer loads row `lane` of the stage's
        // atoms from shared memory and stores them with tcgen05.st into buffer g % kSfBufs:
        // 16 A columns (K-step j at 4j) and 16 or 32 B columns (K-step j, half h at nb*j + 4h).
        // Every lane waits on the barriers itself; the decision to stop is warp-uniform.
        const uint32_t lanes = (uint32_t)(32 * (warp & 3)) << 16;
        constexpr uint32_t nb = 4u * (kBN / 128);
        uint32_t g = 0;
        bool quit = false;
        for (uint32_t t = blockIdx.x; t < p.tiles && !quit; t += gridDim.x) {
            for (uint32_t ks = 0; ks < KS; ++ks, ++g) {
                const uint32_t s = g % kStages, b = g % kSfBufs;
                bool ok = mbar_wait(&sm.full[s], (g / kStages) & 1u);
                if (ok && g >= (uint32_t)kSfBufs) ok = mbar_wait(&sm.sf_free[b], ((g / kSfBufs) - 1u) & 1u);
                const bool timed_out = __any_sync(0xFFFFFFFFu, !ok);
                quit = timed_out || __any_sync(0xFFFFFFFFu, aborted());
                if (quit) {
                    if (timed_out && lane == 0) { flags |= kFlagTimeout; atomicOr(&sm.abort, 1u); }
                    break;
                }
                tc_fence_after();
                uint32_t va[16], vb[4 * nb];
#pragma unroll
                for (uint32_t j = 0; j < 4; ++j) {
                    const uint4 x = *reinterpret_cast<const uint4*>(sm.sfa[s] + 512u * j + 16u * lane);
                    va[4 * j] = x.x; va[4 * j + 1] = x.y; va[4 * j + 2] = x.z; va[4 * j + 3] = x.w;
#pragma unroll
                    for (uint32_t h = 0; h < (uint32_t)(kBN / 128); ++h) {
                        const uint4 y = *reinterpret_cast<const uint4*>(sm.sfb[s] + 2048u * h + 512u * j + 16u * lane);
                        const uint32_t c = nb * j + 4u * h;
                        vb[c] = y.x; vb[c + 1] = y.y; vb[c + 2] = y.z; vb[c + 3] = y.w;
                    }
                }
                const uint32_t ta = tmem + lanes + kBN + C::kSfCols * b;
                tmem_st<16>(ta, va);
                tmem_st<4 * nb>(ta + 16u, vb);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.sf_full[b]);
            }
        }
        __syncwarp();
    } else {
        // ---- epilogue warps 0-3 and 10-13: warp w reads accumulator lanes 32q..32q+31
        // (q = w % 4, one output row per thread), columns [h * kBN/2, (h + 1) * kBN/2) with
        // h = (w >= 10).  BF16: the half row is converted into registers, the accumulator is
        // released, and only then stored (overlapping the next tile's MMAs), each 32 x 16
        // block transposed through the warp's 1 KB of shared memory so that a store
        // instruction writes 16 rows x 32 contiguous bytes.  FP32: stored as read.
        const uint32_t q = (uint32_t)warp & 3u, h = warp >= 10 ? 1u : 0u;
        uint8_t* st = sm.stg[q + 4u * h];
        const float alpha = __fmul_rn(*p.d_s2a, *p.d_s2b);
        constexpr int kChunks = kBN / 64;                          // 32-column chunks per warp
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
            const int64_t row0 = (int64_t)m_tile * kBM + 32 * q;  // this warp's first row
            const int64_t col0 = (int64_t)n_tile * kBN + (int64_t)h * (kBN / 2);
            const uint32_t taddr = tmem + ((32u * q) << 16) + h * (uint32_t)(kBN / 2);
            if constexpr (kOut == 2) {
#pragma unroll 1
                for (int cb = 0; cb < kChunks; ++cb) {
                    float v[32];
                    tmem_ld32(taddr + (uint32_t)(32 * cb), v);
                    float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.out) + (row0 + lane) * p.ldd + col0 + 32 * cb);
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        o[k] = make_float4(__fmul_rn(v[4 * k], alpha), __fmul_rn(v[4 * k + 1], alpha),
                                           __fmul_rn(v[4 * k + 2], alpha), __fmul_rn(v[4 * k + 3], alpha));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.acc_empty);
            } else {
                uint32_t w[16 * kChunks];
#pragma unroll
                for (int cb = 0; cb < kChunks; ++cb) {
                    float v[32];
                    tmem_ld32(taddr + (uint32_t)(32 * cb), v);
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        asm("cvt.rn.bf16x2.f32 %0, %1, %2;"
                            : "=r"(w[16 * cb + k])
                            : "f"(__fmul_rn(v[2 * k + 1], alpha)), "f"(__fmul_rn(v[2 * k], alpha)));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.acc_empty);         // the accumulator is free
                // 16-byte piece p of staged row r at r * 32 + 16 * (p ^ ((r >> 2) & 1)):
                // conflict-free for the row-per-thread writes and the 16-rows-per-instruction reads
                const int pr = lane >> 1, pc = lane & 1;
#pragma unroll
                for (int c16 = 0; c16 < 2 * kChunks; ++c16) {
#pragma unroll
                    for (int k = 0; k < 2; ++k)
                        *reinterpret_cast<uint4*>(st + 32 * lane + 16 * (k ^ ((lane >> 2) & 1))) =
                            make_uint4(w[8 * c16 + 4 * k], w[8 * c16 + 4 * k + 1], w[8 * c16 + 4 * k + 2],
                                       w[8 * c16 + 4 * k + 3]);
                    __syncwarp();
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const int rr = pr + 16 * k;
                        const uint4 x = *reinterpret_cast<const uint4*>(st + 32 * rr + 16 * (pc ^ ((rr >> 2) & 1)));
                        *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + (row0 + rr) * p.ldd + col0 + 16 * c16 +
                                                  8 * pc) = x;
                    }
                    __syncwarp();
                }
            }
        }
    }

    // ---- teardown: drain copies that were loaded but never consumed, free tensor memory
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == kProducer) {
        for (uint32_t g = sm.consumed; g < sm.issued; ++g)
            if (!mbar_wait(&sm.full[g % kStages], (g / kStages) & 1u)) flags |= kFlagTimeout;
    }
    if (warp == kIssuer / 32) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
    flags = __reduce_or_sync(0xFFFFFFFFu, flags);
    if (lane == 0) flag_or(p.d_flags, flags);
}

// ---------------------------------------------------------------- the CTA-pair kernel
// 256 x 256 output tiles computed by a pair of CTAs (a 2-CTA cluster) with the 2-SM MMA
// (tcgen05.mma.cta_group::2, M = 256): CTA r of the pair holds rows 128r..128r+127 of the
// tile's A and of its B in its own shared memory, the full N = 256 of B's scale atoms, and
// its 128 x 256 FP32 accumulator.  The pair's MMA reads each B half once and shares it, so
// per SM a stage moves 16 KB less B through shared memory (TMA write and MMA read) than
// the single-CTA 128 x 256 tile does for the same work.  Roles per CTA as in the kernel
// above (producer, scale writers, epilogue); warp 9 of rank 0 issues the pair's MMAs and
// warp 9 of rank 1 forwards "this stage's codes have landed and its scales are written"
// to it (a cluster-scope mbarrier arrive).  The MMA thread's commits arrive on the
// barriers of both CTAs (tcgen05.commit ... multicast::cluster, mask 0b11); rank 1's
// epilogue warps release the accumulator on rank 0's acc_empty.  No load is multicast.
constexpr int kStages2 = 5;
constexpr int kSfBufs2 = 5;                       // 256 + 5 x 48 = 496 tensor-memory columns

struct Smem2 {
    uint8_t a[kStages2][128 * 128];               // this CTA's 128 rows of A (1024-byte aligned)
    uint8_t b[kStages2][128 * 128];               // this CTA's 128 rows of B
    uint8_t sfa[kStages2][4 * 512];               // A scale atoms of this CTA's rows
    uint8_t sfb[kStages2][8 * 512];               // B scale atoms of all 256 rows
    uint8_t stg[8][1024];                         // epilogue transposes
    uint64_t full[kStages2], empty[kStages2], peer_ready[kStages2], sf_full[kSfBufs2], sf_free[kSfBufs2];
    uint64_t acc_full, acc_empty, drain;
    uint32_t tmem_base;
    uint32_t abort;
    uint32_t issued, consumed;
};

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void mma_fp4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t sfa, uint32_t sfb, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
                 "}"
                 ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
                 : "memory");
}

// Arrives on the barrier at bar's offset in both CTAs of the pair once every tcgen05
// operation issued so far by this thread completes.
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 ::"r"(smem_u32(bar)), "h"((uint16_t)3u)
                 : "memory");
}

template <int kOut>
__global__ void __launch_bounds__(kThreads, 1)
gemm_nvfp4_pair_kernel(const __grid_constant__ Params p)
{
    using C = Cfg<256>;
    constexpr int kStages = kStages2;
    constexpr uint32_t kTx = 2u * 128u * 128u + 4u * 512u + 8u * 512u;
    // instruction descriptor: as Cfg<256>::kIdesc with M = 256 (the pair)
    constexpr uint32_t kIdesc2 = (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
    extern __shared__ uint8_t smem_raw[];
    Smem2& sm = *reinterpret_cast<Smem2*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t KS = p.k_stages;
    const uint32_t rank = cluster_ctarank();
    const uint32_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (threadIdx.x == kProducer) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
            mbar_init(&sm.peer_ready[s], 1);
        }
        for (int b = 0; b < kSfBufs2; ++b) {
            mbar_init(&sm.sf_full[b], 8);                          // the writers of both CTAs
            mbar_init(&sm.sf_free[b], 1);
        }
        mbar_init(&sm.acc_full, 1);
        mbar_init(&sm.acc_empty, 16);                              // 8 epilogue warps in each CTA
        mbar_init(&sm.drain, 1);
        sm.abort = 0u;
        sm.issued = sm.consumed = 0u;
        mbar_init_fence();
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.map_a)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.map_b)) : "memory");
    }
    if (warp == kIssuer / 32) tmem_alloc_pair(&sm.tmem_base, C::kTmemCols);
    tc_fence_before();
    cluster_sync();                                                // barriers of both CTAs initialised
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    uint32_t flags = 0u;
    auto aborted = [&]() { return *reinterpret_cast<volatile uint32_t*>(&sm.abort) != 0u; };
    auto give_up = [&]() { flags |= kFlagTimeout; atomicOr(&sm.abort, 1u); };

    if (warp == kProducer / 32) {
        if (lane == 0) {                                           // producer: this CTA's halves
            uint32_t g = 0;
            for (uint32_t t = pair; t < p.tiles && !aborted(); t += npairs) {
                const uint32_t n_tile = t % p.n_tiles, m_tile = t / p.n_tiles;
                const uint32_t mrow = 2u * m_tile + rank, nrow = 2u * n_tile + rank;   // 128-row tiles
                for (uint32_t ks = 0; ks < KS; ++ks, ++g) {
                    const uint32_t s = g % kStages;
                    if (g >= (uint32_t)kStages && !mbar_wait(&sm.empty[s], ((g / kStages) - 1u) & 1u)) give_up();
                    if (aborted()) break;
                    mbar_arrive_expect_tx(&sm.full[s], kTx);
                    tma_load_2d(sm.a[s], &p.map_a, &sm.full[s], (int)(ks * 128u), (int)(mrow * 128u));
                    tma_load_2d(sm.b[s], &p.map_b, &sm.full[s], (int)(ks * 128u), (int)(nrow * 128u));
                    bulk_load(sm.sfa[s], p.sfa + ((size_t)mrow * p.kt4 + 4u * ks) * 512u, 2048u, &sm.full[s]);
#pragma unroll
                    for (uint32_t h = 0; h < 2u; ++h)
                        bulk_load(sm.sfb[s] + 2048u * h, p.sfb + ((size_t)(2u * n_tile + h) * p.kt4 + 4u * ks) * 512u,
                                  2048u, &sm.full[s]);
                }
            }
            sm.issued = g;
        }
        __syncwarp();
    } else if (warp == kIssuer / 32) {
        if (lane == 0 && rank == 0) {                              // the pair's MMA issuer
            uint32_t g = 0, i = 0;
            for (uint32_t t = pair; t < p.tiles && !aborted(); t += npairs, ++i) {
                if (i > 0 && !mbar_wait(&sm.acc_empty, (i - 1u) & 1u)) {
                    give_up();
                    break;
                }
                tc_fence_after();
                for (uint32_t ks = 0; ks < KS; ++ks, ++g) {
                    const uint32_t s = g % kStages, b = g % kSfBufs2, ph = (g / kStages) & 1u;
                    if (!mbar_wait(&sm.full[s], ph) || !mbar_wait(&sm.sf_full[b], (g / kSfBufs2) & 1u) ||
                        !mbar_wait(&sm.peer_ready[s], ph)) {
                        give_up();
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ta = tmem + 256u + C::kSfCols * b, tb = ta + 16u;
                    const uint32_t a0 = smem_u32(sm.a[s]), b0 = smem_u32(sm.b[s]);
#pragma unroll
                    for (uint32_t j = 0; j < 4; ++j)
                        mma_fp4_pair(tmem, smem_desc(a0 + 32u * j, 1u, 64u, 2u), smem_desc(b0 + 32u * j, 1u, 64u, 2u),
                                     kIdesc2, ta + 4u * j, tb + 8u * j, (ks | j) != 0u ? 1u : 0u);
                    tc_commit_pair(&sm.empty[s]);
                    tc_commit_pair(&sm.sf_free[b]);
                }
                if (aborted()) break;
                tc_commit_pair(&sm.acc_full);
            }
            sm.consumed = g;
            tc_commit_pair(&sm.drain);
            if (!mbar_wait(&sm.drain, 0u)) flags |= kFlagTimeout;
        } else if (lane == 0) {                                    // rank 1: forwards its landed stages
            uint32_t g = 0;
            for (uint32_t t = pair; t < p.tiles && !aborted(); t += npairs) {
                for (uint32_t ks = 0; ks < KS; ++ks, ++g) {
                    const uint32_t s = g % kStages;
                    if (!mbar_wait(&sm.full[s], (g / kStages) & 1u)) {
                        give_up();
                        break;
                    }
                    mbar_arrive_cluster(&sm.peer_ready[s], 0u);
                }
            }
            sm.consumed = g;
        }
        __syncwarp();
    } else if (warp >= 4 && warp < 8) {
        // ---- scale writers: as in the single-CTA kernel, this CTA's rows of A, all of B
        const uint32_t lanes = (uint32_t)(32 * (warp & 3)) << 16;
        uint32_t g = 0;
        bool quit = false;
        for (uint32_t t = pair; t < p.tiles && !quit; t += npairs) {
            for (uint32_t ks = 0; ks < KS; ++ks, ++g) {
                const uint32_t s = g % kStages, b = g % kSfBufs2;
                bool ok = mbar_wait(&sm.full[s], (g / kStages) & 1u);
                if (ok && g >= (uint32_t)kSfBufs2) ok = mbar_wait(&sm.sf_free[b], ((g / kSfBufs2) - 1u) & 1u);
                const bool timed_out = __any_sync(0xFFFFFFFFu, !ok);
                quit = timed_out || __any_sync(0xFFFFFFFFu, aborted());
                if (quit) {
                    if (timed_out && lane == 0) give_up();
                    break;
                }
                tc_fence_after();
                uint32_t va[16], vb[32];
#pragma unroll
                for (uint32_t j = 0; j < 4; ++j) {
                    const uint4 x = *reinterpret_cast<const uint4*>(sm.sfa[s] + 512u * j + 16u * lane);
                    va[4 * j] = x.x; va[4 * j + 1] = x.y; va[4 * j + 2] = x.z; va[4 * j + 3] = x.w;
#pragma unroll
                    for (uint32_t h = 0; h < 2u; ++h) {
                        const uint4 y = *reinterpret_cast<const uint4*>(sm.sfb[s] + 2048u * h + 512u * j + 16u * lane);
                        const uint32_t c = 8u * j + 4u * h;
                        vb[c] = y.x; vb[c + 1] = y.y; vb[c + 2] = y.z; vb[c + 3] = y.w;
                    }
                }
                const uint32_t ta = tmem + lanes + 256u + C::kSfCols * b;
                tmem_st<16>(ta, va);
                tmem_st<32>(ta + 16u, vb);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {                                   // on the MMA issuer's CTA
                    if (rank == 0) mbar_arrive(&sm.sf_full[b]);
                    else mbar_arrive_cluster(&sm.sf_full[b], 0u);
                }
            }
        }
        __syncwarp();
    } else {
        // ---- epilogue warps 0-3 and 10-13, as in the single-CTA kernel; rows 128 * rank + ...
        const uint32_t q = (uint32_t)warp & 3u, h = warp >= 10 ? 1u : 0u;
        uint8_t* st = sm.stg[q + 4u * h];
        const float alpha = __fmul_rn(*p.d_s2a, *p.d_s2b);
        auto release = [&]() {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (rank == 0) mbar_arrive(&sm.acc_empty);
                else mbar_arrive_cluster(&sm.acc_empty, 0u);
            }
        };
        uint32_t i = 0;
        for (uint32_t t = pair; t < p.tiles; t += npairs, ++i) {
            const bool ok = !aborted() && mbar_wait(&sm.acc_full, i & 1u);
            if (!ok) {
                if (!aborted()) give_up();
                break;
            }
            tc_fence_after();
            __syncwarp();
            const uint32_t n_tile = t % p.n_tiles, m_tile = t / p.n_tiles;
            const int64_t row0 = (int64_t)m_tile * 256 + 128 * (int64_t)rank + 32 * q;
            const int64_t col0 = (int64_t)n_tile * 256 + (int64_t)h * 128;
            const uint32_t taddr = tmem + ((32u * q) << 16) + h * 128u;
            if constexpr (kOut == 2) {
#pragma unroll 1
                for (int cb = 0; cb < 4; ++cb) {
                    float v[32];
                    tmem_ld32(taddr + (uint32_t)(32 * cb), v);
                    float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.out) + (row0 + lane) * p.ldd + col0 + 32 * cb);
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        o[k] = make_float4(__fmul_rn(v[4 * k], alpha), __fmul_rn(v[4 * k + 1], alpha),
                                           __fmul_rn(v[4 * k + 2], alpha), __fmul_rn(v[4 * k + 3], alpha));
                }
                release();
            } else {
                uint32_t w[64];
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) {
                    float v[32];
                    tmem_ld32(taddr + (uint32_t)(32 * cb), v);
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        asm("cvt.rn.bf16x2.f32 %0, %1, %2;"
                            : "=r"(w[16 * cb + k])
                            : "f"(__fmul_rn(v[2 * k + 1], alpha)), "f"(__fmul_rn(v[2 * k], alpha)));
                }
                release();
                const int pr = lane >> 1, pc = lane & 1;
#pragma unroll
                for (int c16 = 0; c16 < 8; ++c16) {
#pragma unroll
                    for (int k = 0; k < 2; ++k)
                        *reinterpret_cast<uint4*>(st + 32 * lane + 16 * (k ^ ((lane >> 2) & 1))) =
                            make_uint4(w[8 * c16 + 4 * k], w[8 * c16 + 4 * k + 1], w[8 * c16 + 4 * k + 2],
                                       w[8 * c16 + 4 * k + 3]);
                    __syncwarp();
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const int rr = pr + 16 * k;
                        const uint4 x = *reinterpret_cast<const uint4*>(st + 32 * rr + 16 * (pc ^ ((rr >> 2) & 1)));
                        *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + (row0 + rr) * p.ldd + col0 + 16 * c16 +
                                                  8 * pc) = x;
                    }
                    __syncwarp();
                }
            }
        }
    }

    // ---- teardown: this CTA's loads drained, then the pair's barrier (rank 0 reaches it
    // only after its MMAs, which read both CTAs' shared memory, have completed), then the
    // pair's tensor memory is released
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == kProducer) {
        for (uint32_t g = sm.consumed; g < sm.issued; ++g)
            if (!mbar_wait(&sm.full[g % kStages], (g / kStages) & 1u)) flags |= kFlagTimeout;
    }
    tc_fence_before();
    cluster_sync();
    if (warp == kIssuer / 32) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, C::kTmemCols);
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
    static bool attr_set[6][64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int o = out_dt == 2 ? 1 : 0;
    if (M % 256 == 0 && N % 256 == 0) {
        // 256 x 256 tiles on CTA pairs (2-SM MMA)
        if (!code_map(&p.map_a, qa, M, K, 128u) || !code_map(&p.map_b, qb, N, K, 128u)) return cudaErrorInvalidValue;
        p.sfa = sfa;
        p.sfb = sfb;
        p.d_s2a = d_s2a;
        p.d_s2b = d_s2b;
        p.out = out;
        p.ldd = ldd;
        p.n_tiles = (uint32_t)(N / 256);
        p.k_stages = (uint32_t)(K / kBK);
        p.kt4 = (uint32_t)(K / 64);
        p.tiles = (uint32_t)((M / 256) * (N / 256));
        p.d_flags = d_flags;
        const size_t smem = sizeof(Smem2) + 1024;
        auto kern = o ? gemm_nvfp4_pair_kernel<2> : gemm_nvfp4_pair_kernel<0>;
        if (dev < 0 || dev >= 64 || !attr_set[4 + o][dev]) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            if (dev >= 0 && dev < 64) attr_set[4 + o][dev] = true;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        // persistent: as many pairs as can be resident at once (once per device and output type)
        static int resident[2][64] = {};
        int pairs_cap = dev >= 0 && dev < 64 ? resident[o][dev] : 0;
        if (pairs_cap <= 0) {
            cfg.gridDim = dim3(2u * (uint32_t)(num_sms() / 2), 1, 1);
            if (cudaOccupancyMaxActiveClusters(&pairs_cap, kern, &cfg) != cudaSuccess || pairs_cap <= 0) {
                (void)cudaGetLastError();
                pairs_cap = num_sms() / 2;
            }
            if (dev >= 0 && dev < 64) resident[o][dev] = pairs_cap;
        }
        const uint32_t npairs = p.tiles < (uint32_t)pairs_cap ? p.tiles : (uint32_t)pairs_cap;
        cfg.gridDim = dim3(2u * npairs, 1, 1);
        e = cudaLaunchKernelEx(&cfg, kern, p);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
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
