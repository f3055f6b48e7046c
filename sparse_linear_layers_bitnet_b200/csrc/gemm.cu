// Tensor-core GEMMs on tcgen05 (sm_100a): the prefill / training sparse
// int8 x ternary product, and the dense bf16 STE input gradient.
//
// Sparse product ("BitNet b1.58: Ternary Weights for 1.58-bit LLMs", section
// "The mechanism": signed accumulation of int8 activations by ternary weights;
// "Sparse-BitNet" (gist.science), section 2: the forward uses the 2:4-masked
// ternary weights, run on sparse tensor cores):
//     Y^T[n, t] = sum_k Wq[n, k] Xq[t, k]      (int32 in TMEM)
// The 2:4-sparse operand must be A of tcgen05.mma.sp, so A = the compressed
// weights (M = output features), B = int8 activations (N = tokens), K = input
// features; the epilogue dequantises and writes Y[t, n] (the transpose).
//
// STE gradient ("Sparse-BitNet", section 2 "Training Strategie"):
//     dX[t, k] = gamma * sum_n dY[t, n] Wq[n, k]      (bf16 in, fp32 in TMEM)
// with A = dY (M = tokens), B = Wq expanded to bf16 (N = input features),
// K = output features: here (T <= 128) as Wq^T, K-major; the CTA-pair kernel
// (gemm2.cu, T > 128) reads untransposed bf16 rows of Wq as an MN-major operand.
//
// One CTA computes a 128 x BN output tile:
//   warp 0      TMA producer: A and B tiles (and the 2 KB metadata block) per
//               k-step into a STAGES-deep ring of shared-memory buffers;
//   warp 1      allocates TMEM and issues the MMAs from one thread; for the
//               sparse kind it first copies the metadata block into TMEM
//               (tcgen05.cp), which the MMAs read in issue order;
//   warps 2-5   epilogue: tcgen05.ld of the accumulator, scale, store.
// Every mbarrier wait is bounded (2 s); a wait that gives up sets the device
// status word and the CTA drains its in-flight copies and MMAs and exits.
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace bitnet {

template <bool SPARSE, int BN, int STAGES>
struct GemmCfg {
    static constexpr int kBM = 128;
    // bytes of one row of A / B per k-step (one 128-byte or 64-byte swizzle row)
    static constexpr int kARowBytes = SPARSE ? 64 : 128;   // 128 logical int8 compressed 2:1 | 64 bf16
    static constexpr int kBRowBytes = 128;                 // 128 int8 | 64 bf16
    static constexpr int kKStep = SPARSE ? 128 : 64;       // logical K elements per stage
    static constexpr int kABytes = kBM * kARowBytes;
    static constexpr int kBBytes = BN * kBRowBytes;
    static constexpr int kEBytes = SPARSE ? 2048 : 0;
    static constexpr int kStageBytes = kABytes + kBBytes + kEBytes;
    static constexpr int kMmaPerStage = SPARSE ? 2 : 4;    // K = 64 (sparse i8) | 16 (bf16) per MMA
    static constexpr int kAAdvance = 32;                   // bytes of A per MMA along K
    static constexpr int kBAdvance = SPARSE ? 64 : 32;
    static constexpr int kECol = BN;                       // TMEM column of the metadata
    static constexpr int kTmemCols = (BN + (SPARSE ? 8 : 0)) <= 32    ? 32
                                     : (BN + (SPARSE ? 8 : 0)) <= 64  ? 64
                                     : (BN + (SPARSE ? 8 : 0)) <= 128 ? 128
                                     : (BN + (SPARSE ? 8 : 0)) <= 256 ? 256
                                                                      : 512;
    static constexpr int kSmemBytes = STAGES * kStageBytes + 1024 /*align*/ + 2048 /*barriers, scales*/;
    // instruction descriptor: sparse flag (bit 2), D format (bits 4-5: 1 = f32, 2 = s32),
    // A/B format (bits 7-9, 10-12: s8 = 1 | bf16 = 1), K-major A and B, N >> 3 (bits 17-22),
    // M >> 4 (bits 24-28).
    static constexpr uint32_t kIdesc = (SPARSE ? (1u << 2) : 0u) | ((SPARSE ? 2u : 1u) << 4) | (1u << 7) |
                                       (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                                       (static_cast<uint32_t>(kBM >> 4) << 24);
};

struct GemmParams {
    int64_t M, N, K;            // M rows of A, N rows of B, K logical contraction length
    const uint8_t *meta;        // sparse: metadata blocks
    int64_t meta_rows;          // sparse: rows per metadata k-block
    const float *gamma;
    const float *amax;          // sparse: per-token absmax
    void *out;
    int out_bf16;
    int32_t *acc_out;           // sparse: optional raw accumulators
    uint32_t *status;
};

template <bool SPARSE, int BN, int STAGES>
__global__ void __launch_bounds__(192, 1) k_umma_gemm(const __grid_constant__ CUtensorMap tmA,
                                                      const __grid_constant__ CUtensorMap tmB, GemmParams p) {
    using C = GemmCfg<SPARSE, BN, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + STAGES * C::kABytes;
    uint8_t *sE = sB + STAGES * C::kBBytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(sE + STAGES * C::kEBytes);
    uint64_t *empty = full + STAGES;
    uint64_t *acc_bar = empty + STAGES;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(acc_bar + 1);
    volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);
    float *s_scale = reinterpret_cast<float *>(s_tmem + 4);   // BN floats

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t m0 = static_cast<int64_t>(blockIdx.x) * C::kBM;
    const int64_t n0 = static_cast<int64_t>(blockIdx.y) * BN;
    const int ktiles = static_cast<int>((p.K + C::kKStep - 1) / C::kKStep);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_bar, 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(s_tmem, C::kTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 0) {
        // ------------------------------------------------ producer
        if (lane == 0) {
            int issued = 0;
            for (int kt = 0; kt < ktiles; ++kt) {
                const int s = kt % STAGES;
                if (kt >= STAGES && !mbar_wait_bounded(&empty[s], ((kt / STAGES) - 1) & 1, s_abort, p.status))
                    break;
                mbar_arrive_expect_tx(&full[s], C::kStageBytes);
                if (SPARSE) {
                    tma_load_2d(&tmA, &full[s], sA + s * C::kABytes, kt * (C::kKStep / 2), static_cast<int32_t>(m0));
                    tma_load_2d(&tmB, &full[s], sB + s * C::kBBytes, kt * C::kKStep, static_cast<int32_t>(n0));
                    const uint8_t *e = p.meta + ((static_cast<int64_t>(kt) * p.meta_rows + m0) << 4);
                    bulk_load(sE + s * C::kEBytes, e, C::kEBytes, &full[s]);
                } else {
                    tma_load_2d(&tmA, &full[s], sA + s * C::kABytes, kt * C::kKStep, static_cast<int32_t>(m0));
                    tma_load_2d(&tmB, &full[s], sB + s * C::kBBytes, kt * C::kKStep, static_cast<int32_t>(n0));
                }
                ++issued;
            }
            // drain: the most recent phase of each armed stage must have landed
            const int first = issued > STAGES ? issued - STAGES : 0;
            for (int kt = first; kt < issued; ++kt) {
                volatile int dummy = 0;
                mbar_wait_bounded(&full[kt % STAGES], (kt / STAGES) & 1, &dummy, p.status);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t tm_acc = tmem;
            for (int kt = 0; kt < ktiles; ++kt) {
                const int s = kt % STAGES;
                if (!mbar_wait_bounded(&full[s], (kt / STAGES) & 1, s_abort, p.status)) break;
                tc_fence_after();
                const uint32_t a_base = smem_u32(sA + s * C::kABytes);
                const uint32_t b_base = smem_u32(sB + s * C::kBBytes);
                if (SPARSE) {
                    const uint32_t e_col = tmem + C::kECol + 4u * (kt & 1);
                    // 128 rows x 16 bytes, 8-row core matrices of 128 contiguous bytes
                    tmem_cp_128x128b(e_col, make_smem_desc(smem_u32(sE + s * C::kEBytes), 16, 128, kSwizzleNone));
#pragma unroll
                    for (int j = 0; j < C::kMmaPerStage; ++j) {
                        const uint64_t ad = make_smem_desc(a_base + j * C::kAAdvance, 16, 512, kSwizzle64B);
                        const uint64_t bd = make_smem_desc(b_base + j * C::kBAdvance, 16, 1024, kSwizzle128B);
                        mma_sp_i8(tm_acc, ad, bd, C::kIdesc, e_col + 2u * j, (kt | j) != 0);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < C::kMmaPerStage; ++j) {
                        const uint64_t ad = make_smem_desc(a_base + j * C::kAAdvance, 16, 1024, kSwizzle128B);
                        const uint64_t bd = make_smem_desc(b_base + j * C::kBAdvance, 16, 1024, kSwizzle128B);
                        mma_bf16(tm_acc, ad, bd, C::kIdesc, (kt | j) != 0);
                    }
                }
                mma_commit(&empty[s]);   // frees the stage once these MMAs have read it
            }
            mma_commit(acc_bar);
            if (*s_abort) {   // make sure every issued MMA is done before TMEM is released
                volatile int dummy = 0;
                mbar_wait_bounded(acc_bar, 0, &dummy, p.status);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (warps 2..5)
        const int ep = threadIdx.x - 64;   // 0..127
        if (SPARSE) {
            const float g = *p.gamma;
            for (int j = ep; j < BN; j += 128) {
                const int64_t t = n0 + j;
                s_scale[j] = (t < p.N) ? __fdiv_rn(__fmul_rn(g, p.amax[t]), 127.0f) : 0.0f;
            }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const bool ok = mbar_wait_bounded(acc_bar, 0, s_abort, p.status);
        tc_fence_after();
        const int quarter = warp & 3;                 // TMEM lanes 32*quarter .. +31
        const int64_t m = m0 + 32 * quarter + lane;   // this thread's accumulator row
        const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * quarter) << 16);
        if (ok) {
#pragma unroll 1
            for (int c = 0; c < BN / 16; ++c) {
                uint32_t r[16];
                tmem_ld_32x32b_x16(taddr + 16 * c, r);
                tmem_ld_wait();
                if (m >= p.M) continue;
                if (SPARSE) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int64_t t = n0 + 16 * c + j;
                        if (t < p.N) {
                            const int acc = static_cast<int>(r[j]);
                            const float y = __fmul_rn(__int2float_rn(acc), s_scale[16 * c + j]);
                            if (p.out_bf16)
                                static_cast<__nv_bfloat16 *>(p.out)[t * p.M + m] = __float2bfloat16_rn(y);
                            else
                                static_cast<float *>(p.out)[t * p.M + m] = y;
                            if (p.acc_out) p.acc_out[t * p.M + m] = acc;
                        }
                    }
                } else {
                    const float g = *p.gamma;
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
                            for (int j = 0; j < 4; ++j)
                                dst[j] = make_float4(__fmul_rn(__uint_as_float(r[4 * j]), g),
                                                     __fmul_rn(__uint_as_float(r[4 * j + 1]), g),
                                                     __fmul_rn(__uint_as_float(r[4 * j + 2]), g),
                                                     __fmul_rn(__uint_as_float(r[4 * j + 3]), g));
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int64_t n = nb + j;
                            if (n < p.N) {
                                const float y = __fmul_rn(__uint_as_float(r[j]), g);
                                if (p.out_bf16)
                                    static_cast<__nv_bfloat16 *>(p.out)[m * p.N + n] = __float2bfloat16_rn(y);
                                else
                                    static_cast<float *>(p.out)[m * p.N + n] = y;
                            }
                        }
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*PFN_encodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                    const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static PFN_encodeTiled get_encode() {
    static PFN_encodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_encodeTiled>(ptr);
    });
    return fn;
}

// 2-D tensor map: inner dimension `inner` elements (contiguous), `outer` rows,
// row pitch `pitch_bytes`, box `box_inner` x `box_outer`, zero fill outside.
static bool make_map_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
                        uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    PFN_encodeTiled enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {pitch_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool SPARSE, int BN, int STAGES>
static cudaError_t run_gemm(const CUtensorMap &a, const CUtensorMap &b, const GemmParams &p, cudaStream_t s) {
    using C = GemmCfg<SPARSE, BN, STAGES>;
    auto kern = k_umma_gemm<SPARSE, BN, STAGES>;
    {
        cudaError_t e = smem_attr(reinterpret_cast<const void *>(kern), C::kSmemBytes);
        if (e != cudaSuccess) return e;
    }
    dim3 grid(static_cast<unsigned>((p.M + C::kBM - 1) / C::kBM), static_cast<unsigned>((p.N + BN - 1) / BN));
    kern<<<grid, 192, C::kSmemBytes, s>>>(a, b, p);
    return cudaGetLastError();
}

cudaError_t launch_gemm_sp(const int8_t *Xq, const float *amax, const float *gamma, const int8_t *vals,
                           const uint8_t *meta, int64_t T, int64_t n_out, int64_t k, void *Y, bool y_bf16,
                           int32_t *acc, uint32_t *status, cudaStream_t s) {
    GemmParams p{};
    p.M = n_out;
    p.N = T;
    p.K = k;
    p.meta = meta;
    p.meta_rows = (n_out + 127) / 128 * 128;
    p.gamma = gamma;
    p.amax = amax;
    p.out = Y;
    p.out_bf16 = y_bf16 ? 1 : 0;
    p.acc_out = acc;
    p.status = status;
    if (T > 128)   // CTA-pair persistent kernel (gemm2.cu)
        return launch_gemm_sp_pair(Xq, amax, gamma, vals, meta, T, n_out, k, Y, y_bf16, acc, status, s);
    const int bn = T <= 32 ? 32 : (T <= 128 ? 128 : 256);
    CUtensorMap ma, mb;
    if (!make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, vals, static_cast<uint64_t>(k / 2),
                     static_cast<uint64_t>(n_out), static_cast<uint64_t>(k / 2), 64, 128, CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    if (!make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, Xq, static_cast<uint64_t>(k), static_cast<uint64_t>(T),
                     static_cast<uint64_t>(k), 128, static_cast<uint32_t>(bn), CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (bn == 32) return run_gemm<true, 32, 6>(ma, mb, p, s);
    if (bn == 128) return run_gemm<true, 128, 6>(ma, mb, p, s);
    return run_gemm<true, 256, 5>(ma, mb, p, s);
}

// Wq^T in bf16: wt[k, n] = code of weight (n, k), from the canonical group bytes.
// Persistent CTAs walk 64 (n) x 64 (k) tiles.  Per tile, 64 threads bring the
// 64 rows of 16 group bytes in with one 16-byte load each (issued one tile
// ahead, so the load overlaps the previous tile's work) into a padded shared
// tile.  A 256-entry shared table holds, for every group byte, the bf16 values
// of its four positions (8 bytes).  Thread (g, c) looks up the four group
// bytes of rows n = 4c..4c+3 at group g and assembles the output rows
// k = 4g..4g+3 of those four columns with byte permutes, as 8-byte stores;
// sixteen threads cover one 128-byte output row segment.
constexpr int kExpandRowWords = 17;   // 68-byte shared rows: the 16 column groups fall in different banks

__device__ __forceinline__ uint4 expand_load(const uint8_t *__restrict__ gb, int64_t n_out, int64_t k, int64_t n,
                                            int64_t k0) {
    uint4 v = make_uint4(0x04040404u, 0x04040404u, 0x04040404u, 0x04040404u);   // idx (0,1), codes 0
    if (n < n_out) {
        const uint8_t *src = gb + n * (k / 4) + k0 / 4;
        if (k0 + 64 <= k && (reinterpret_cast<uintptr_t>(src) & 15) == 0) {
            v = __ldg(reinterpret_cast<const uint4 *>(src));
        } else {
            uint8_t tmp[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) tmp[j] = (k0 + 4 * j < k) ? src[j] : static_cast<uint8_t>(0x04);
            v = *reinterpret_cast<const uint4 *>(tmp);
        }
    }
    return v;
}

__global__ void __launch_bounds__(256) k_expand_wt(const uint8_t *__restrict__ gb, int64_t n_out, int64_t k,
                                                   __nv_bfloat16 *__restrict__ wt) {
    __shared__ __align__(16) uint32_t s_gb[64 * kExpandRowWords];
    __shared__ uint2 s_lut[256];
    const int tid = threadIdx.x;
    s_lut[tid] = group_bf16x4(static_cast<uint32_t>(tid));
    const int64_t ktiles = (k + 63) / 64, ntiles = (n_out + 63) / 64;
    const int64_t tiles = ktiles * ntiles;
    int64_t tile = blockIdx.x;
    uint4 v;
    if (tid < 64 && tile < tiles) v = expand_load(gb, n_out, k, (tile / ktiles) * 64 + tid, (tile % ktiles) * 64);
    const int g = tid >> 4, c = tid & 15;
    for (; tile < tiles; tile += gridDim.x) {
        const int64_t n0 = (tile / ktiles) * 64, k0 = (tile % ktiles) * 64;
        __syncthreads();   // the table is ready; the previous tile's reads of s_gb are done
        if (tid < 64) {
            uint32_t *row = s_gb + tid * kExpandRowWords;
            row[0] = v.x;
            row[1] = v.y;
            row[2] = v.z;
            row[3] = v.w;
        }
        __syncthreads();
        const int64_t next = tile + gridDim.x;
        if (tid < 64 && next < tiles) v = expand_load(gb, n_out, k, (next / ktiles) * 64 + tid, (next % ktiles) * 64);
        // values of the four group bytes: rows 4c + i, group g
        uint2 L[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t word = s_gb[(4 * c + i) * kExpandRowWords + (g >> 2)];
            L[i] = s_lut[(word >> (8 * (g & 3))) & 0xffu];
        }
        const int64_t nb = n0 + 4 * c;
#pragma unroll
        for (int pos = 0; pos < 4; ++pos) {
            const int64_t kk = k0 + 4 * g + pos;
            if (kk >= k) break;
            // position pos of columns nb..nb+3: bytes 2q, 2q+1 of the half holding it
            constexpr uint32_t kSel[2] = {0x5410u, 0x7632u};
            const uint32_t sel = kSel[pos & 1];
            const uint32_t h01 = __byte_perm(pos < 2 ? L[0].x : L[0].y, pos < 2 ? L[1].x : L[1].y, sel);
            const uint32_t h23 = __byte_perm(pos < 2 ? L[2].x : L[2].y, pos < 2 ? L[3].x : L[3].y, sel);
            __nv_bfloat16 *dst = wt + kk * n_out + nb;
            if (nb + 4 <= n_out) {
                *reinterpret_cast<uint2 *>(dst) = make_uint2(h01, h23);
            } else {
                const uint32_t h[4] = {h01 & 0xffffu, h01 >> 16, h23 & 0xffffu, h23 >> 16};
                for (int i = 0; i < 4; ++i)
                    if (nb + i < n_out) reinterpret_cast<uint16_t *>(dst)[i] = static_cast<uint16_t>(h[i]);
            }
        }
    }
}

// Wq as bf16 rows [n_out][k]: group byte i holds the weights 4i .. 4i + 3 of the
// row-major matrix, so the expansion is a linear map.  Lane-consecutive
// 16-byte output chunks (two group bytes each): loads and stores coalesced.
__global__ void __launch_bounds__(256) k_expand_w(const uint8_t *__restrict__ gb, int64_t nbytes,
                                                  __nv_bfloat16 *__restrict__ w) {
    __shared__ uint2 s_lut[256];
    s_lut[threadIdx.x] = group_bf16x4(threadIdx.x);
    __syncthreads();
    const int64_t nchunk = nbytes / 2;   // nbytes is even (k % 8 == 0)
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const uint16_t *src = reinterpret_cast<const uint16_t *>(gb);
    uint4 *dst = reinterpret_cast<uint4 *>(w);
    int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (; j + 3 * stride < nchunk; j += 4 * stride) {
        uint32_t b[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) b[u] = __ldg(src + j + u * stride);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const uint2 lo = s_lut[b[u] & 0xffu], hi = s_lut[b[u] >> 8];
            dst[j + u * stride] = make_uint4(lo.x, lo.y, hi.x, hi.y);
        }
    }
    for (; j < nchunk; j += stride) {
        const uint32_t b = __ldg(src + j);
        const uint2 lo = s_lut[b & 0xffu], hi = s_lut[b >> 8];
        dst[j] = make_uint4(lo.x, lo.y, hi.x, hi.y);
    }
}

cudaError_t launch_dgrad(const void *dY, const float *gamma, const uint8_t *gb, int64_t T, int64_t n_out, int64_t k,
                         void *dX, bool dx_bf16, void *ws, cudaStream_t s) {
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    __nv_bfloat16 *wt = reinterpret_cast<__nv_bfloat16 *>(w8 + kDgradWsHeader);
    if (T > 128) {   // CTA-pair persistent kernel (gemm2.cu) on Wq's untransposed bf16 rows
        const int64_t nchunk = n_out * k / 8;
        const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
        const int64_t blocks = (nchunk + 1023) / 1024;
        k_expand_w<<<static_cast<unsigned>(blocks < cap ? blocks : cap), 256, 0, s>>>(gb, n_out * k / 4, wt);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        return launch_gemm_bf16_pair(dY, wt, gamma, T, n_out, k, dX, dx_bf16,
                                     reinterpret_cast<uint32_t *>(w8 + kStatusOffset), s);
    }
    const int64_t tiles = ((k + 63) / 64) * ((n_out + 63) / 64);
    const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
    k_expand_wt<<<static_cast<unsigned>(tiles < cap ? tiles : cap), 256, 0, s>>>(gb, n_out, k, wt);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    GemmParams p{};
    p.M = T;
    p.N = k;
    p.K = n_out;
    p.gamma = gamma;
    p.out = dX;
    p.out_bf16 = dx_bf16 ? 1 : 0;
    p.status = reinterpret_cast<uint32_t *>(w8 + kStatusOffset);
    CUtensorMap ma, mb;
    if (!make_map_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dY, static_cast<uint64_t>(n_out),
                     static_cast<uint64_t>(T), static_cast<uint64_t>(n_out) * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    if (!make_map_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, wt, static_cast<uint64_t>(n_out),
                     static_cast<uint64_t>(k), static_cast<uint64_t>(n_out) * 2, 64, 256, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    return run_gemm<false, 256, 4>(ma, mb, p, s);
}

}  // namespace bitnet
