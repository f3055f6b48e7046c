// Tensor-core throughput ceilings, measured on the GPU that runs the GEMMs.
//
// The prefill GEMM issues tcgen05.mma.sp.cta_group::2.kind::i8 (M = 256,
// N = 224, K = 64 logical).  What the hardware sustains for that instruction
// form is the ceiling the GEMM is judged against, and the nominal "2x dense"
// ratio of 2:4 sparsity need not hold for it.  k_tensor_peak issues the same
// instruction (or its dense int8 / bf16 counterparts) back to back on operands
// that sit in shared memory, with no loads and no epilogue, so its rate is the
// most a GEMM built from that instruction can reach on this device.  One CTA
// pair per two SMs; the leader's lane 0 issues every MMA into one TMEM
// accumulator, as the GEMM's issuer does, and a final commit tells both CTAs
// when the tensor pipe has drained.
//
// Operand bytes are a fixed hash of their index (the multipliers toggle as
// with real data); the 2:4 metadata selects positions (0, 1) of every group,
// a valid pattern.  The results in TMEM are never read.
#include "../../include/bitnet_sparse.h"
#include "common.cuh"
#include "kernels.h"

namespace bitnet {

namespace peak {

__device__ __forceinline__ uint32_t cta_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
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
__device__ __forceinline__ void tmem_cp2_128x128b(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.128x128b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void mma_sp_i8_2(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t e, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.sp.cta_group::2.kind::i8 [%0], %1, %2, [%5], %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(e)
        : "memory");
}
__device__ __forceinline__ void mma_i8_2(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void mma_bf16_2(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void commit_both(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(static_cast<uint16_t>(3))
        : "memory");
}

}  // namespace peak

// Instruction forms (M = 256 over the CTA pair).
//   kind 0: 2:4-sparse int8, N = 224, K = 64 logical (32 stored bytes of A per row), two per 128-k stage
//   kind 1: dense int8, N = 256, K = 32, four per 128-byte stage
//   kind 2: dense bf16, N = 256, K = 16, four per 128-byte stage
//   kind 3: kind 0 with the stage's metadata copied into TMEM (tcgen05.cp) right before its two MMAs,
//           in a ring of two slots, as a GEMM stage does
//   kind 4: kind 3 with each copy issued four stages ahead of its MMAs (ring of eight slots)
struct PeakForm {
    int n, k, per_stage;
};
__host__ __device__ constexpr PeakForm peak_form(int kind) {
    return (kind == 0 || kind >= 3) ? PeakForm{224, 64, 2} : (kind == 1 ? PeakForm{256, 32, 4} : PeakForm{256, 16, 4});
}

constexpr int kPeakABytes = 128 * 128;   // 128 rows x 128 bytes (sparse: 64 used per row)
constexpr int kPeakBBytes = 128 * 128;   // up to 128 rows (N / 2 per CTA) x 128 bytes
constexpr int kPeakEBytes = 2048;        // 128 rows x 16 bytes of metadata
constexpr int kPeakSmem = kPeakABytes + kPeakBBytes + kPeakEBytes + 1024;

template <int KIND>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(128, 1) k_tensor_peak(int64_t iters, uint32_t *status) {
    constexpr PeakForm F = peak_form(KIND);
    // s32 (kinds 0, 1) or f32 (kind 2) accumulators; s8 / bf16 operands; M = 256, N = F.n
    constexpr bool kSparse = KIND == 0 || KIND >= 3;
    constexpr uint32_t kIdesc = (kSparse ? (1u << 2) : 0u) | ((KIND == 2 ? 1u : 2u) << 4) | (1u << 7) | (1u << 10) |
                                (static_cast<uint32_t>(F.n >> 3) << 17) | (static_cast<uint32_t>(256 >> 4) << 24);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = sA + kPeakABytes;
    uint8_t *sE = sB + kPeakBBytes;
    __shared__ __align__(8) uint64_t done;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool leader = peak::cta_rank() == 0;

    for (int i = threadIdx.x; i < (kPeakABytes + kPeakBBytes) / 4; i += blockDim.x) {
        uint32_t h = static_cast<uint32_t>(i) * 0x9E3779B1u + blockIdx.x * 0x85EBCA77u;
        h ^= h >> 15;
        h *= 0x2C1B3C6Du;
        h ^= h >> 12;
        if (KIND == 2) h &= 0xBFFFBFFFu;   // bf16 pairs with exponents below 2^1: finite, no overflow
        reinterpret_cast<uint32_t *>(sA)[i] = h;
    }
    for (int i = threadIdx.x; i < kPeakEBytes / 4; i += blockDim.x) reinterpret_cast<uint32_t *>(sE)[i] = 0x44444444u;
    if (threadIdx.x == 0) {
        mbar_init(&done, 1);
        s_abort = 0;
        fence_mbar_init();
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // operands written by threads, read by the tensor pipe
    if (warp == 0) {
        peak::tmem_alloc2(&s_tmem, 512);
        peak::tmem_relinquish2();
    }
    tc_fence_before();
    __syncthreads();
    peak::cluster_sync();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    if (leader && warp == 0 && lane == 0) {
        const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
        const uint32_t e_col = tmem + 256;
        const uint64_t e_desc = make_smem_desc(smem_u32(sE), 16, 128, kSwizzleNone);
        if (KIND == 0) peak::tmem_cp2_128x128b(e_col, e_desc);
        if (KIND == 4)
            for (int q = 0; q < 4; ++q) peak::tmem_cp2_128x128b(e_col + 4u * q, e_desc);
        for (int64_t it = 0, st = 0; it < iters; it += F.per_stage, ++st) {
            uint32_t e_stage = e_col;
            if (KIND == 3) {   // this stage's metadata, then its MMAs
                e_stage = e_col + 4u * static_cast<uint32_t>(st & 1);
                peak::tmem_cp2_128x128b(e_stage, e_desc);
            } else if (KIND == 4) {   // stage st + 4's metadata, then stage st's MMAs
                e_stage = e_col + 4u * static_cast<uint32_t>(st & 7);
                peak::tmem_cp2_128x128b(e_col + 4u * static_cast<uint32_t>((st + 4) & 7), e_desc);
            }
#pragma unroll
            for (int j = 0; j < F.per_stage; ++j) {
                const uint32_t acc = (it | j) != 0;
                if (kSparse) {
                    const uint64_t ad = make_smem_desc(a_base + j * 32, 16, 512, kSwizzle64B);
                    const uint64_t bd = make_smem_desc(b_base + j * 64, 16, 1024, kSwizzle128B);
                    peak::mma_sp_i8_2(tmem, ad, bd, kIdesc, e_stage + 2u * j, acc);
                } else if (KIND == 1) {
                    const uint64_t ad = make_smem_desc(a_base + j * 32, 16, 1024, kSwizzle128B);
                    const uint64_t bd = make_smem_desc(b_base + j * 32, 16, 1024, kSwizzle128B);
                    peak::mma_i8_2(tmem, ad, bd, kIdesc, acc);
                } else {
                    const uint64_t ad = make_smem_desc(a_base + j * 32, 16, 1024, kSwizzle128B);
                    const uint64_t bd = make_smem_desc(b_base + j * 32, 16, 1024, kSwizzle128B);
                    peak::mma_bf16_2(tmem, ad, bd, kIdesc, acc);
                }
            }
        }
        peak::commit_both(&done);
    }
    // both CTAs: the tensor pipe has finished every MMA of the pair (bounded wait)
    if (threadIdx.x == 0) mbar_wait_bounded(&done, 0, &s_abort, status);
    tc_fence_before();
    __syncthreads();
    peak::cluster_sync();
    if (warp == 0) {
        tc_fence_after();
        peak::tmem_dealloc2(tmem, 512);
    }
}

cudaError_t launch_tensor_peak(int kind, int64_t iters, uint32_t *status, double *ops, cudaStream_t s) {
    const int sms = num_sms();
    const int ctas = sms / 2 * 2;
    const PeakForm F = peak_form(kind);
    const int64_t per = (iters + F.per_stage - 1) / F.per_stage * F.per_stage;   // MMAs per pair
    *ops = 2.0 * 256.0 * F.n * F.k * static_cast<double>(per) * (ctas / 2);
    auto kern = kind == 0 ? k_tensor_peak<0>
                          : (kind == 1 ? k_tensor_peak<1>
                                       : (kind == 2 ? k_tensor_peak<2> : (kind == 3 ? k_tensor_peak<3> : k_tensor_peak<4>)));
    cudaError_t e = smem_attr(reinterpret_cast<const void *>(kern), kPeakSmem);
    if (e != cudaSuccess) return e;
    kern<<<dim3(static_cast<unsigned>(ctas)), 128, kPeakSmem, s>>>(per, status);
    return cudaGetLastError();
}

}  // namespace bitnet
