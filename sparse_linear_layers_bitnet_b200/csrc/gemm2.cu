// Persistent CTA-pair tensor-core GEMM (tcgen05 .cta_group::2, sm_100a).
//
// Same products as gemm.cu: the 2:4-sparse int8 x ternary forward
// ("BitNet b1.58: Ternary Weights for 1.58-bit LLMs", section "The mechanism";
// "Sparse-BitNet" (gist.science), section 2), the dense bf16 STE input
// gradient and the dense weight gradient dW = dY^T X ("Sparse-BitNet",
// section 2 "Training Strategie").  The forward results are identical to
// gemm.cu (integer accumulation is exact; the fp32 epilogue does the same
// operations in the same order).  Dense operands are K-major or MN-major
// (template mask MN): the input gradient reads Wq as bf16 rows (B MN-major),
// the weight gradient reads dY and X with the token index as the contraction
// (both MN-major), so no operand is ever transposed in memory.
//
// A cluster of two CTAs on two SMs computes one 256 x BN output tile with one
// MMA instruction stream: each CTA holds 128 rows of A and BN/2 rows of B in
// its own shared memory, and the pair's TMEM holds the 256 x BN accumulator
// (128 lanes per CTA).  Per SM this halves the B bytes per MMA compared with a
// 128 x BN single-CTA tile.  The CTA pair is persistent: it walks tiles
// pair_id, pair_id + pairs, ...; two TMEM accumulator buffers let the
// epilogue of one tile overlap the main loop of the next.
//   warp 0     TMA producer in both CTAs (2-SM TMA: completion counted on the
//              leader CTA's barrier), STAGES-deep ring;
//   warp 1     TMEM allocation in both CTAs; the leader's lane 0 copies the
//              2:4 metadata into TMEM and issues the MMAs; commits release the
//              ring stage and publish an accumulator in both CTAs;
//   warps 2-5  epilogue in both CTAs: TMEM -> registers -> scaled stores, then
//              release of the accumulator buffer to the leader.
// Every wait is bounded (2 s) and reports through the device status word.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace bitnet {

namespace pair {

__device__ __forceinline__ uint32_t cta_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// arrive on the barrier at the same shared-memory offset in CTA `rank`
__device__ __forceinline__ void arrive_remote(uint64_t *bar, uint32_t rank) {
    asm volatile(
        "{\n\t.reg .b32 ra;\n\t"
        "mapa.shared::cluster.u32 ra, %0, %1;\n\t"
        "mbarrier.arrive.release.cluster.shared::cluster.b64 _, [ra];\n\t}" ::"r"(smem_u32(bar)),
        "r"(rank)
        : "memory");
}

// 2-SM TMA load: data lands in this CTA's shared memory; the transaction bytes
// are counted on the leader CTA's barrier (same offset, peer bit cleared).
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap *map, uint64_t *bar, void *dst, int32_t c0,
                                                 int32_t c1) {
    const uint32_t leader_bar = smem_u32(bar) & 0xFEFFFFFFu;
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
        "[%2];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(leader_bar), "r"(c0), "r"(c1)
        : "memory");
}

// TMA tiled store shared -> global (bulk group), and its bookkeeping
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int32_t c0, int32_t c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_shared() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc2(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void mma_sp_i8_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t e,
                                               uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.sp.cta_group::2.kind::i8 [%0], %1, %2, [%5], %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(e)
        : "memory");
}

__device__ __forceinline__ void mma_bf16_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void tmem_cp_pair_128x128b(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.128x128b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void tmem_cp_pair_128x256b(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.128x256b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// arrive once on the barrier at this offset in both CTAs when the issued
// tcgen05 operations are complete
__device__ __forceinline__ void commit_both(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(static_cast<uint16_t>(3))
        : "memory");
}

}  // namespace pair

// MN (dense only), a mask: 1 = A, 2 = B stored with its M (A) or N (B)
// dimension contiguous ("MN-major"): its tiles arrive as 64-element-wide boxes
// of 64 k-rows, 128-byte swizzled; the descriptors step 8 KB between 64-wide
// boxes (leading byte offset) and 1 KB between groups of 8 k-rows (stride byte
// offset).  The other operand stays K-major.
template <bool SPARSE, int BN, int STAGES, int MN = 0>
struct PairCfg {
    static constexpr int kHalfN = BN / 2;                  // B rows per CTA
    static constexpr int kARowBytes = SPARSE ? 64 : 128;
    static constexpr int kBRowBytes = 128;
    static constexpr int kKStep = SPARSE ? 128 : 64;       // k of one k-step (one metadata block when sparse)
    // k-steps per ring stage: a sparse k-step is only 2 x 64 of k, about 150 ns of
    // MMA at the instruction's rate, so two share a stage and its barrier round trip
    static constexpr int kSub = SPARSE ? 2 : 1;
    static constexpr int kASub = 128 * kARowBytes;          // one k-step's A, B and metadata bytes
    static constexpr int kBSub = kHalfN * kBRowBytes;
    static constexpr int kESub = SPARSE ? 2048 : 0;
    static constexpr int kABytes = kSub * kASub;
    static constexpr int kBBytes = kSub * kBSub;
    static constexpr int kEBytes = kSub * kESub;
    static constexpr int kSubBytes = kASub + kBSub + kESub;
    static constexpr int kStageBytes = kSub * kSubBytes;   // per CTA
    static constexpr int kMmaPerStage = SPARSE ? 2 : 4;
    static constexpr int kAAdvance = 32;
    static constexpr int kBAdvance = SPARSE ? 64 : 32;
    static constexpr int kAccStride = 256;                // TMEM columns between the two accumulators
    static constexpr int kECol = 2 * kAccStride - 16;     // metadata columns (two groups of 8)
    static constexpr int kTmemCols = 512;
    static constexpr int kStageOutBytes = SPARSE ? 2 * 16 * 128 * 4 : 0;   // two [16 tokens][128 rows] fp32 chunks
    static constexpr int kSmemBytes = STAGES * kStageBytes + kStageOutBytes + 1024 + 2048;
    // M = 256 (two CTAs), N = BN
    static constexpr uint32_t kIdesc = (SPARSE ? (1u << 2) : 0u) | ((SPARSE ? 2u : 1u) << 4) | (1u << 7) |
                                       (1u << 10) | ((MN & 1) ? (1u << 15) : 0u) | ((MN & 2) ? (1u << 16) : 0u) |
                                       (static_cast<uint32_t>(BN >> 3) << 17) | (static_cast<uint32_t>(256 >> 4) << 24);
    static constexpr int kMnBox = 64 * 64 * 2;             // one 64 (MN) x 64 (k) bf16 box
    static constexpr int kMnAdvance = 2 * 1024;            // 16 k-rows per MMA
    static_assert(!SPARSE || (BN % 32 == 0 && BN <= 224), "sparse pair tiles: N multiple of 32, two buffers + metadata");
    static_assert(SPARSE || (BN % 32 == 0 && BN <= 256), "dense pair tiles: N multiple of 32");
    static_assert(kBSub % 1024 == 0, "B tile must keep the 128-byte swizzle atoms aligned");
    static_assert(!MN || (!SPARSE && (!(MN & 2) || kHalfN % 64 == 0)), "MN-major tiles: dense, whole 64-wide boxes");
};

struct PairParams {
    int64_t M, N, K;
    int tma_store;               // sparse: output chunks leave through TMA stores
    int64_t meta_rows;           // sparse: rows of one metadata k-block
    const float *gamma;
    const float *amax;           // sparse: per-token scale
    void *out;
    int out_bf16;
    int32_t *acc_out;
    uint32_t *status;
    int accumulate;              // dense fp32 output: out += result (else out = result)
};

template <bool SPARSE, int BN, int STAGES, int MN = 0>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
    k_umma_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmY, PairParams p) {
    using C = PairCfg<SPARSE, BN, STAGES, MN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = sA + STAGES * C::kABytes;
    uint8_t *sE = sB + STAGES * C::kBBytes;
    uint8_t *sOut = sE + STAGES * C::kEBytes;   // output staging (sparse)
    uint64_t *full = reinterpret_cast<uint64_t *>(sOut + C::kStageOutBytes);
    uint64_t *empty = full + STAGES;
    uint64_t *acc_full = empty + STAGES;       // [2]
    uint64_t *acc_empty = acc_full + 2;        // [2], leader: one arrival per CTA
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(acc_empty + 2);
    volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);
    float *s_scale = reinterpret_cast<float *>(s_tmem + 4);   // BN floats

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = pair::cta_rank();
    const bool leader = rank == 0;
    const int64_t pair_id = blockIdx.x >> 1, pairs = gridDim.x >> 1;
    const int64_t m_tiles = (p.M + 255) / 256, n_tiles = (p.N + BN - 1) / BN;
    const int64_t tiles = m_tiles * n_tiles;
    const int ksteps = static_cast<int>((p.K + C::kKStep - 1) / C::kKStep);
    // ring stages per tile.  When a tile has an odd number of sparse k-steps the
    // last stage's second one lies past K: TMA fills its A and B boxes with
    // zeros and its metadata load is clamped to the last valid block, so its
    // MMAs add exactly zero and every stage has the same shape.
    const int ktiles = (ksteps + C::kSub - 1) / C::kSub;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 2);
        }
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        pair::tmem_alloc2(s_tmem, C::kTmemCols);
        pair::tmem_relinquish2();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        if (SPARSE) prefetch_tensormap(&tmE);
    }
    tc_fence_before();
    pair::cluster_sync();   // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 0) {
        // ------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            int it = 0;
            for (int64_t t = pair_id; t < tiles && !*s_abort; t += pairs) {
                const int64_t mt = t / n_tiles, nt = t - mt * n_tiles;
                const int32_t a_row = static_cast<int32_t>(mt * 256 + 128 * rank);
                const int32_t b_row = static_cast<int32_t>(nt * BN + C::kHalfN * rank);
                // metadata rows past the padded end (a ragged last pair) read a valid block:
                // their A rows are zero-filled, so any valid index pattern gives zero
                int64_t e_row = mt * 256 + 128 * rank;
                if (e_row > p.meta_rows - 128) e_row = p.meta_rows - 128;
                for (int kt = 0; kt < ktiles; ++kt, ++it) {
                    const int s = it % STAGES;
                    if (it >= STAGES && !mbar_wait_bounded(&empty[s], ((it / STAGES) - 1) & 1, s_abort, p.status))
                        break;
                    if (leader) mbar_arrive_expect_tx(&full[s], 2 * C::kStageBytes);
                    if (SPARSE) {
#pragma unroll
                        for (int sub = 0; sub < C::kSub; ++sub) {
                            const int kk = kt * C::kSub + sub;
                            const int ke = kk < ksteps ? kk : ksteps - 1;   // a valid metadata block
                            pair::tma_load_2d_pair(&tmA, &full[s], sA + s * C::kABytes + sub * C::kASub,
                                                   kk * (C::kKStep / 2), a_row);
                            pair::tma_load_2d_pair(&tmB, &full[s], sB + s * C::kBBytes + sub * C::kBSub, kk * C::kKStep,
                                                   b_row);
                            pair::tma_load_2d_pair(&tmE, &full[s], sE + s * C::kEBytes + sub * C::kESub, 0,
                                                   static_cast<int32_t>((ke * p.meta_rows + e_row) / 8));
                        }
                    } else if (MN) {
                        // MN-major: boxes of 64 MN-elements x 64 k-rows (two for A's 128 rows, kHalfN / 64
                        // for B); K-major: one box of 64 k x all rows
                        if (MN & 1) {
#pragma unroll
                            for (int h = 0; h < 2; ++h)
                                pair::tma_load_2d_pair(&tmA, &full[s], sA + s * C::kABytes + h * C::kMnBox,
                                                       a_row + 64 * h, kt * C::kKStep);
                        } else {
                            pair::tma_load_2d_pair(&tmA, &full[s], sA + s * C::kABytes, kt * C::kKStep, a_row);
                        }
                        if (MN & 2) {
#pragma unroll
                            for (int h = 0; h < C::kHalfN / 64; ++h)
                                pair::tma_load_2d_pair(&tmB, &full[s], sB + s * C::kBBytes + h * C::kMnBox,
                                                       b_row + 64 * h, kt * C::kKStep);
                        } else {
                            pair::tma_load_2d_pair(&tmB, &full[s], sB + s * C::kBBytes, kt * C::kKStep, b_row);
                        }
                    } else {
                        pair::tma_load_2d_pair(&tmA, &full[s], sA + s * C::kABytes, kt * C::kKStep, a_row);
                        pair::tma_load_2d_pair(&tmB, &full[s], sB + s * C::kBBytes, kt * C::kKStep, b_row);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader CTA)
        if (leader && lane == 0) {
            int it = 0, local = 0;
            for (int64_t t = pair_id; t < tiles && !*s_abort; t += pairs, ++local) {
                const int b = local & 1;
                // both CTAs' epilogues must have drained this accumulator buffer
                if (local >= 2 && !mbar_wait_bounded(&acc_empty[b], ((local >> 1) - 1) & 1, s_abort, p.status)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + b * C::kAccStride;
                for (int kt = 0; kt < ktiles; ++kt, ++it) {
                    const int s = it % STAGES;
                    if (!mbar_wait_bounded(&full[s], (it / STAGES) & 1, s_abort, p.status)) break;
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(sA + s * C::kABytes);
                    const uint32_t b_base = smem_u32(sB + s * C::kBBytes);
                    if (SPARSE) {
                        // both k-steps' metadata in one copy of 128 lanes x 256 bits: k-step 0's block (the
                        // first 16-byte core-matrix column) lands in columns 0..3, k-step 1's (C::kESub bytes on)
                        // in 4..7; consecutive stages alternate between two groups of 8 columns
                        static_assert(!SPARSE || C::kSub == 2, "one 256-bit metadata copy covers two k-steps");
                        const uint32_t e_stage = tmem + C::kECol + 8u * (it & 1);
                        pair::tmem_cp_pair_128x256b(
                            e_stage, make_smem_desc(smem_u32(sE + s * C::kEBytes), C::kESub, 128, kSwizzleNone));
#pragma unroll
                        for (int sub = 0; sub < C::kSub; ++sub) {
                            const uint32_t e_col = e_stage + 4u * sub;
#pragma unroll
                            for (int j = 0; j < C::kMmaPerStage; ++j) {
                                const uint64_t ad = make_smem_desc(a_base + sub * C::kASub + j * C::kAAdvance, 16, 512,
                                                                   kSwizzle64B);
                                const uint64_t bd = make_smem_desc(b_base + sub * C::kBSub + j * C::kBAdvance, 16, 1024,
                                                                   kSwizzle128B);
                                pair::mma_sp_i8_pair(d_tmem, ad, bd, C::kIdesc, e_col + 2u * j, (kt | j | sub) != 0);
                            }
                        }
                    } else if (MN) {
#pragma unroll
                        for (int j = 0; j < C::kMmaPerStage; ++j) {
                            const uint64_t ad = (MN & 1) ? make_smem_desc(a_base + j * C::kMnAdvance, C::kMnBox, 1024, kSwizzle128B)
                                                         : make_smem_desc(a_base + j * C::kAAdvance, 16, 1024, kSwizzle128B);
                            const uint64_t bd = (MN & 2) ? make_smem_desc(b_base + j * C::kMnAdvance, C::kMnBox, 1024, kSwizzle128B)
                                                         : make_smem_desc(b_base + j * C::kBAdvance, 16, 1024, kSwizzle128B);
                            pair::mma_bf16_pair(d_tmem, ad, bd, C::kIdesc, (kt | j) != 0);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < C::kMmaPerStage; ++j) {
                            const uint64_t ad = make_smem_desc(a_base + j * C::kAAdvance, 16, 1024, kSwizzle128B);
                            const uint64_t bd = make_smem_desc(b_base + j * C::kBAdvance, 16, 1024, kSwizzle128B);
                            pair::mma_bf16_pair(d_tmem, ad, bd, C::kIdesc, (kt | j) != 0);
                        }
                    }
                    pair::commit_both(&empty[s]);
                }
                pair::commit_both(&acc_full[b]);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (warps 2..5, both CTAs)
        const int quarter = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(32 * quarter) << 16;
        int local = 0;
        int chunk_count = 0;   // output chunks staged so far (TMA-store double buffer)
        for (int64_t t = pair_id; t < tiles; t += pairs, ++local) {
            const int b = local & 1;
            const int64_t mt = t / n_tiles, nt = t - mt * n_tiles;
            const int64_t m0 = mt * 256 + 128 * rank;   // this CTA's accumulator rows
            const int64_t n0 = nt * BN;
            if (SPARSE) {
                const float g = *p.gamma;
                asm volatile("bar.sync 1, 128;" ::: "memory");   // previous tile's scales are no longer read
                for (int j = threadIdx.x - 64; j < BN; j += 128) {
                    const int64_t tok = n0 + j;
                    s_scale[j] = (tok < p.N) ? __fdiv_rn(__fmul_rn(g, p.amax[tok]), 127.0f) : 0.0f;
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
            }
            const bool ok = mbar_wait_bounded(&acc_full[b], (local >> 1) & 1, s_abort, p.status);
            tc_fence_after();
            const int64_t m = m0 + 32 * quarter + lane;
            const uint32_t taddr = tmem + lane_base + b * C::kAccStride;
            if (ok) {
#pragma unroll 1
                for (int c = 0; c < BN / 16; ++c) {
                    uint32_t r[16];
                    tmem_ld_32x32b_x16(taddr + 16 * c, r);
                    tmem_ld_wait();
                    if (SPARSE && p.tma_store) {
                        // stage [16 tokens][128 rows] and send it with one TMA store
                        const int buf = chunk_count & 1;
                        uint8_t *stg = sOut + buf * (16 * 128 * 4);
                        if (chunk_count >= 2) {
                            if (threadIdx.x == 64) pair::bulk_wait_read1();   // the store of 2 chunks ago has read this buffer
                            asm volatile("bar.sync 1, 128;" ::: "memory");
                        }
                        const int row = 32 * quarter + lane;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float y = __fmul_rn(__int2float_rn(static_cast<int>(r[j])), s_scale[16 * c + j]);
                            if (p.out_bf16)
                                reinterpret_cast<__nv_bfloat16 *>(stg)[j * 128 + row] = __float2bfloat16_rn(y);
                            else
                                reinterpret_cast<float *>(stg)[j * 128 + row] = y;
                        }
                        pair::fence_async_shared();
                        asm volatile("bar.sync 1, 128;" ::: "memory");
                        if (threadIdx.x == 64 && m0 < p.M && n0 + 16 * c < p.N) {
                            pair::tma_store_2d(&tmY, stg, static_cast<int32_t>(m0), static_cast<int32_t>(n0 + 16 * c));
                            pair::bulk_commit();
                        }
                        ++chunk_count;
                        if (p.acc_out && m < p.M) {
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const int64_t tok = n0 + 16 * c + j;
                                if (tok < p.N) p.acc_out[tok * p.M + m] = static_cast<int>(r[j]);
                            }
                        }
                        continue;
                    }
                    if (m >= p.M) continue;
                    if (SPARSE) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int64_t tok = n0 + 16 * c + j;
                            if (tok < p.N) {
                                const int acc = static_cast<int>(r[j]);
                                const float y = __fmul_rn(__int2float_rn(acc), s_scale[16 * c + j]);
                                if (p.out_bf16)
                                    static_cast<__nv_bfloat16 *>(p.out)[tok * p.M + m] = __float2bfloat16_rn(y);
                                else
                                    static_cast<float *>(p.out)[tok * p.M + m] = y;
                                if (p.acc_out) p.acc_out[tok * p.M + m] = acc;
                            }
                        }
                    } else {
                        const float g = p.gamma ? *p.gamma : 1.0f;
                        const int64_t nb = n0 + 16 * c;
                        if (nb + 16 <= p.N) {
                            if (p.out_bf16) {
                                uint32_t h[8];
#pragma unroll
                                for (int j = 0; j < 8; ++j) {
                                    const __nv_bfloat162 v = __floats2bfloat162_rn(
                                        __fmul_rn(__uint_as_float(r[2 * j]), g), __fmul_rn(__uint_as_float(r[2 * j + 1]), g));
                                    h[j] = *reinterpret_cast<const uint32_t *>(&v);
                                }
                                uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.out) + m * p.N + nb);
                                dst[0] = make_uint4(h[0], h[1], h[2], h[3]);
                                dst[1] = make_uint4(h[4], h[5], h[6], h[7]);
                            } else {
                                float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.out) + m * p.N + nb);
#pragma unroll
                                for (int j = 0; j < 4; ++j) {
                                    float4 y = make_float4(__fmul_rn(__uint_as_float(r[4 * j]), g),
                                                           __fmul_rn(__uint_as_float(r[4 * j + 1]), g),
                                                           __fmul_rn(__uint_as_float(r[4 * j + 2]), g),
                                                           __fmul_rn(__uint_as_float(r[4 * j + 3]), g));
                                    if (p.accumulate) {
                                        const float4 o = dst[j];
                                        y = make_float4(__fadd_rn(o.x, y.x), __fadd_rn(o.y, y.y), __fadd_rn(o.z, y.z),
                                                        __fadd_rn(o.w, y.w));
                                    }
                                    dst[j] = y;
                                }
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const int64_t n = nb + j;
                                if (n < p.N) {
                                    const float y = __fmul_rn(__uint_as_float(r[j]), g);
                                    if (p.out_bf16)
                                        static_cast<__nv_bfloat16 *>(p.out)[m * p.N + n] = __float2bfloat16_rn(y);
                                    else if (p.accumulate)
                                        static_cast<float *>(p.out)[m * p.N + n] =
                                            __fadd_rn(static_cast<float *>(p.out)[m * p.N + n], y);
                                    else
                                        static_cast<float *>(p.out)[m * p.N + n] = y;
                                }
                            }
                        }
                    }
                }
            }
            // this CTA is done with the buffer: one arrival on the leader's barrier
            tc_fence_before();
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (threadIdx.x == 64) pair::arrive_remote(&acc_empty[b], 0);
            if (!ok) break;
        }
    }
    if (SPARSE && p.tma_store && threadIdx.x == 64) pair::bulk_wait_all();   // stores have left shared memory
    tc_fence_before();
    __syncthreads();
    pair::cluster_sync();   // no CTA leaves while its peer may still signal it
    if (warp == 1) {
        tc_fence_after();
        pair::tmem_dealloc2(tmem, C::kTmemCols);
    }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*PFN_encodeTiled2)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                     const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                     CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static PFN_encodeTiled2 encode_fn() {
    static PFN_encodeTiled2 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_encodeTiled2>(ptr);
    });
    return fn;
}

static bool map2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
                  uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    PFN_encodeTiled2 enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {pitch_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool SPARSE, int BN, int STAGES, int MN = 0>
static cudaError_t run_pair(const CUtensorMap &a, const CUtensorMap &b, const CUtensorMap &e, const CUtensorMap &y,
                            const PairParams &p, cudaStream_t s) {
    using C = PairCfg<SPARSE, BN, STAGES, MN>;
    auto kern = k_umma_pair<SPARSE, BN, STAGES, MN>;
    {
        cudaError_t err = smem_attr(reinterpret_cast<const void *>(kern), C::kSmemBytes);
        if (err != cudaSuccess) return err;
    }
    const int64_t tiles = ((p.M + 255) / 256) * ((p.N + BN - 1) / BN);
    int64_t pairs = num_sms() / 2;
    if (pairs > tiles) pairs = tiles;
    if (pairs < 1) pairs = 1;
    kern<<<dim3(static_cast<unsigned>(2 * pairs)), 192, C::kSmemBytes, s>>>(a, b, e, y, p);
    return cudaGetLastError();
}

template <int BN>
static cudaError_t sp_pair(const int8_t *Xq, const float *amax, const float *gamma, const int8_t *vals,
                           const uint8_t *meta, int64_t T, int64_t n_out, int64_t k, void *Y, bool y_bf16, int32_t *acc,
                           uint32_t *status, cudaStream_t s) {
    PairParams p{};
    p.M = n_out;
    p.N = T;
    p.K = k;
    p.meta_rows = (n_out + 127) / 128 * 128;
    p.gamma = gamma;
    p.amax = amax;
    p.out = Y;
    p.out_bf16 = y_bf16 ? 1 : 0;
    p.acc_out = acc;
    p.status = status;
    CUtensorMap ma, mb, me;
    if (!map2d(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, vals, static_cast<uint64_t>(k / 2), static_cast<uint64_t>(n_out),
               static_cast<uint64_t>(k / 2), 64, 128, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    if (!map2d(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, Xq, static_cast<uint64_t>(k), static_cast<uint64_t>(T),
               static_cast<uint64_t>(k), 128, static_cast<uint32_t>(BN / 2), CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    // metadata as rows of 128 bytes: one k-step of a 128-row tile is 16 such rows (2 KB, contiguous)
    const uint64_t meta_total_rows = static_cast<uint64_t>((k + 127) / 128) * static_cast<uint64_t>(p.meta_rows);
    if (!map2d(&me, CU_TENSOR_MAP_DATA_TYPE_UINT8, meta, 128, meta_total_rows / 8, 128, 128, 16,
               CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    // output through TMA stores when the row pitch allows it (16-byte multiple)
    CUtensorMap my = ma;
    const size_t esz = y_bf16 ? 2 : 4;
    p.tma_store = (static_cast<size_t>(n_out) * esz) % 16 == 0;
    if (p.tma_store &&
        !map2d(&my, y_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Y,
               static_cast<uint64_t>(n_out), static_cast<uint64_t>(T), static_cast<uint64_t>(n_out) * esz, 128, 16,
               CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    return run_pair<true, BN, 4>(ma, mb, me, my, p, s);
}

// Tile width of the sparse pair GEMM over the T tokens: 192 unless 224-wide
// tiles waste clearly fewer padded columns.  Cost model: ceil(T / BN) x
// (BN + 32), the padded columns of one tile row plus a fixed cost per tile.
// With two k-steps per ring stage the 192-wide tiles measured faster even
// where the model has them slightly dearer: at T = 4096 (7B up and down)
// 3503 against 3355 TOPS; 160- and 128-wide tiles measured 3035 and 2683.
// T = 2048 is 9 x 224 + 32 (a last tile 86% padding) but 10 x 192 + 128.
cudaError_t launch_gemm_sp_pair(const int8_t *Xq, const float *amax, const float *gamma, const int8_t *vals,
                                const uint8_t *meta, int64_t T, int64_t n_out, int64_t k, void *Y, bool y_bf16,
                                int32_t *acc, uint32_t *status, cudaStream_t s) {
    auto cost = [&](int64_t bn) { return static_cast<double>((T + bn - 1) / bn) * static_cast<double>(bn + 32); };
    if (cost(224) < 0.95 * cost(192))
        return sp_pair<224>(Xq, amax, gamma, vals, meta, T, n_out, k, Y, y_bf16, acc, status, s);
    return sp_pair<192>(Xq, amax, gamma, vals, meta, T, n_out, k, Y, y_bf16, acc, status, s);
}

// dX = gamma dY . Wq with Wq as bf16 rows [n_out][k] (expanded from the group
// bytes without a transpose): B (N = k, K = n_out) is MN-major.
cudaError_t launch_gemm_bf16_pair(const void *dY, const __nv_bfloat16 *w, const float *gamma, int64_t T,
                                  int64_t n_out, int64_t k, void *dX, bool dx_bf16, uint32_t *status, cudaStream_t s) {
    constexpr int BN = 256;
    PairParams p{};
    p.M = T;
    p.N = k;
    p.K = n_out;
    p.gamma = gamma;
    p.out = dX;
    p.out_bf16 = dx_bf16 ? 1 : 0;
    p.status = status;
    CUtensorMap ma, mb;
    if (!map2d(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dY, static_cast<uint64_t>(n_out), static_cast<uint64_t>(T),
               static_cast<uint64_t>(n_out) * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!map2d(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w, static_cast<uint64_t>(k), static_cast<uint64_t>(n_out),
               static_cast<uint64_t>(k) * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    return run_pair<false, BN, 6, 2>(ma, mb, ma, ma, p, s);
}

// Weight gradient dW[n, k] (+)= sum_t dY[t, n] X[t, k]: A = dY and B = X both
// with the contraction index t as the outer (row) index, i.e. MN-major tiles.
cudaError_t launch_gemm_wgrad_pair(const void *dY, const void *X, int64_t T, int64_t n_out, int64_t k, float *dW,
                                   bool accumulate, uint32_t *status, cudaStream_t s) {
    constexpr int BN = 256;
    PairParams p{};
    p.M = n_out;
    p.N = k;
    p.K = T;
    p.gamma = nullptr;   // scale 1
    p.out = dW;
    p.out_bf16 = 0;
    p.accumulate = accumulate ? 1 : 0;
    p.status = status;
    CUtensorMap ma, mb;
    if (!map2d(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dY, static_cast<uint64_t>(n_out), static_cast<uint64_t>(T),
               static_cast<uint64_t>(n_out) * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!map2d(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, static_cast<uint64_t>(k), static_cast<uint64_t>(T),
               static_cast<uint64_t>(k) * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    return run_pair<false, BN, 6, 3>(ma, mb, ma, ma, p, s);
}

}  // namespace bitnet
