// Decode GEMV (T <= 8 tokens) over packed 2:4 ternary weights (sm_100a).
//
// "BitNet b1.58: Ternary Weights for 1.58-bit LLMs", section "The mechanism":
// at inference the ternary weights are stored packed and each output is a
// signed sum of activations; section "Algorithm / figure walkthrough" step 5
// (packed ternary weights at inference).  "Sparse-BitNet" (gist.science),
// section 4 "Snelheid en Efficientie": the speed-up comes from the sparse
// tensor cores.
//
// Two kernels:
//  * k_gemv_dec reads the decode layout: per 16-row x 64-k tile, every lane
//    loads 8 bytes = its 16 two-bit codes and its 8 metadata nibbles, expands
//    the codes to int8 in registers (shift, mask, one multiply-add per 4
//    values) and issues one warp-level m16n8k64 sparse MMA; the hardware
//    gathers the kept activations from the metadata.  Bytes read from HBM are
//    0.25 per weight.  Warps of a CTA split k; a shared-memory reduction and
//    the dequant epilogue finish the 16 x T outputs.
//  * k_gemv_gb reads canonical group bytes directly (one warp per row, dp4a on
//    CUDA cores).  It serves shapes the decode layout does not cover.
#include "common.cuh"
#include "kernels.h"

namespace bitnet {

constexpr int kDecRegTiles = 16;   // k-tiles (8 bytes each) prefetched per lane per round

// Warps per CTA so that one prefetch round holds every k-tile of a warp
// (K <= 4096: 4 warps; K <= 8192: 8 warps; beyond, several rounds).
inline int gemv_warps(int64_t k) { return (k / 64 + 3) / 4 <= kDecRegTiles ? 4 : 8; }

// int8 code of one activation: clamp(rint(fp32(x * s)), -127, 127)
__device__ __forceinline__ int8_t quant_code(float x, float s) {
    int q = __float2int_rn(__fmul_rn(x, s));
    q = q > 127 ? 127 : (q < -127 ? -127 : q);
    return static_cast<int8_t>(q);
}

__device__ __forceinline__ uint32_t expand_codes(uint32_t codes, int r) {
    // bytes of t hold 2-bit codes {0: 0, 1: +1, 3: -1}; int8 = (t & 1) | (t & 2) * 0x7f
    const uint32_t t = (codes >> (2 * r)) & 0x03030303u;
    return (t & 0x01010101u) + (t & 0x02020202u) * 0x7fu;
}

__device__ __forceinline__ void mma_sp_m16n8k64(int (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[4],
                                                uint32_t e) {
    asm volatile(
        "mma.sp::ordered_metadata.sync.aligned.m16n8k64.row.col.s32.s8.s8.s32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9, %10, %11}, {%0, %1, %2, %3}, %12, 0x0;"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]), "r"(b[2]), "r"(b[3]), "r"(e));
}

template <int kDecWarps>
__global__ void __launch_bounds__(kDecWarps * 32) k_gemv_dec(const uint2 *__restrict__ dec,
                                                              const int8_t *__restrict__ Xq,
                                                              const float *__restrict__ amax,
                                                              const float *__restrict__ gamma, int T, int64_t n_out,
                                                              int64_t K, void *__restrict__ Y, int y_bf16,
                                                              int32_t *__restrict__ acc_out) {
    __shared__ int s_part[kDecWarps][32][4];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tq = lane & 3;
    const int64_t rt = blockIdx.x;                 // 16-row tile
    const int64_t ktiles = K / 64;
    const int64_t per_warp = (ktiles + kDecWarps - 1) / kDecWarps;
    const int64_t kt0 = warp * per_warp;
    const int64_t kt1 = (kt0 + per_warp < ktiles) ? kt0 + per_warp : ktiles;
    const uint2 *src = dec + (rt * ktiles) * 32 + lane;
    const bool tok = gid < T;
    const int8_t *xrow = Xq + static_cast<int64_t>(tok ? gid : 0) * K + 4 * tq;

    // every weight record of this warp's first round is in flight before any use;
    // they do not depend on the previous kernel, so they are issued before the wait
    uint2 w[kDecRegTiles];
#pragma unroll
    for (int i = 0; i < kDecRegTiles; ++i)
        if (kt0 + i < kt1) w[i] = __ldg(src + (kt0 + i) * 32);
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    int d[4] = {0, 0, 0, 0};
    for (int64_t base = kt0; base < kt1; base += kDecRegTiles) {
        if (base != kt0) {
#pragma unroll
            for (int i = 0; i < kDecRegTiles; ++i)
                if (base + i < kt1) w[i] = __ldg(src + (base + i) * 32);
        }
#pragma unroll
        for (int i = 0; i < kDecRegTiles; ++i) {
            const int64_t kt = base + i;
            if (kt < kt1) {
                uint32_t a[4], b[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    b[j] = tok ? __ldg(reinterpret_cast<const uint32_t *>(xrow + kt * 64 + 16 * j)) : 0u;
#pragma unroll
                for (int r = 0; r < 4; ++r) a[r] = expand_codes(w[i].x, r);
                mma_sp_m16n8k64(d, a, b, w[i].y);
            }
        }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) s_part[warp][lane][q] = d[q];
    __syncthreads();
    if (warp != 0) return;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        int sum = 0;
#pragma unroll
        for (int w2 = 0; w2 < kDecWarps; ++w2) sum += s_part[w2][lane][q];
        d[q] = sum;
    }
    const float g = *gamma;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int row = gid + 8 * (q >> 1);
        const int t = 2 * tq + (q & 1);
        if (t >= T) continue;
        const int64_t n = rt * 16 + row;
        const float scale = __fdiv_rn(__fmul_rn(g, amax[t]), 127.0f);
        const float y = __fmul_rn(__int2float_rn(d[q]), scale);
        if (y_bf16)
            static_cast<__nv_bfloat16 *>(Y)[t * n_out + n] = __float2bfloat16_rn(y);
        else
            static_cast<float *>(Y)[t * n_out + n] = y;
        if (acc_out) acc_out[t * n_out + n] = d[q];
    }
}

// ---------------------------------------------------------------- canonical group bytes

__device__ __forceinline__ uint32_t group_to_int8x4(uint32_t b) {
    const uint32_t i0 = b & 3u, i1 = (b >> 2) & 3u, c0 = (b >> 4) & 3u, c1 = (b >> 6) & 3u;
    const uint32_t v0 = c0 | ((c0 >> 1) * 0xfeu);   // 0 -> 0, 1 -> 0x01, 3 -> 0xff
    const uint32_t v1 = c1 | ((c1 >> 1) * 0xfeu);
    return (v0 << (8 * i0)) | (v1 << (8 * i1));
}

__global__ void __launch_bounds__(256) k_gemv_gb(const uint8_t *__restrict__ gb, const int8_t *__restrict__ Xq,
                                                 const float *__restrict__ amax, const float *__restrict__ gamma,
                                                 int T, int64_t n_out, int64_t K, void *__restrict__ Y, int y_bf16,
                                                 int32_t *__restrict__ acc_out) {
    const int lane = threadIdx.x & 31;
    const int64_t gpr = K / 4;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t n = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); n < n_out;
         n += warps) {
        int acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        const uint8_t *row = gb + n * gpr;
        for (int64_t g = lane; g < gpr; g += 32) {
            const uint32_t w4 = group_to_int8x4(__ldg(row + g));
#pragma unroll
            for (int t = 0; t < 8; ++t)
                if (t < T) acc[t] = __dp4a(static_cast<int>(w4),
                                           __ldg(reinterpret_cast<const int *>(Xq + t * K) + g), acc[t]);
        }
#pragma unroll
        for (int t = 0; t < 8; ++t) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
        }
        if (lane == 0) {
            const float g = *gamma;
            for (int t = 0; t < T; ++t) {
                const float scale = __fdiv_rn(__fmul_rn(g, amax[t]), 127.0f);
                const float y = __fmul_rn(__int2float_rn(acc[t]), scale);
                if (y_bf16)
                    static_cast<__nv_bfloat16 *>(Y)[t * n_out + n] = __float2bfloat16_rn(y);
                else
                    static_cast<float *>(Y)[t * n_out + n] = y;
                if (acc_out) acc_out[t * n_out + n] = acc[t];
            }
        }
    }
}

// ---------------------------------------------------------------- fused quantisation + GEMV

// One kernel per projection for decode: the CTA first issues the loads of its
// packed weights (which do not depend on earlier kernels), then waits on the
// programmatic dependency (griddepcontrol.wait: the previous kernel of the
// stream has finished and its writes are visible), reads the T activation rows
// (fp32 or bf16), forms the per-token absmax scale exactly as bitnet_quant_act
// does, quantises its own B fragments in registers and runs the sparse MMAs.
// Launched with programmatic stream serialisation, consecutive projections
// overlap: the next kernel streams its weights while this one finishes.
constexpr int kFusedWarps = 8;
constexpr int kFusedRegTiles = 16;  // k-tiles prefetched per lane per round

template <bool BF16>
__device__ __forceinline__ float load_x(const void *X, int64_t idx) {
    if (BF16) return __uint_as_float(static_cast<uint32_t>(__ldg(static_cast<const unsigned short *>(X) + idx)) << 16);
    return __ldg(static_cast<const float *>(X) + idx);
}

// four consecutive activations (idx % 4 == 0) in one vector load
template <bool BF16>
__device__ __forceinline__ void load_x4(const void *X, int64_t idx, float (&v)[4]) {
    if (BF16) {
        const uint2 u = __ldg(reinterpret_cast<const uint2 *>(static_cast<const unsigned short *>(X) + idx));
        v[0] = __uint_as_float(u.x << 16);
        v[1] = __uint_as_float(u.x & 0xffff0000u);
        v[2] = __uint_as_float(u.y << 16);
        v[3] = __uint_as_float(u.y & 0xffff0000u);
    } else {
        const float4 f = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(X) + idx));
        v[0] = f.x;
        v[1] = f.y;
        v[2] = f.z;
        v[3] = f.w;
    }
}

template <bool BF16>
__device__ __forceinline__ uint32_t quant4(const void *X, int64_t idx, float s) {
    // four consecutive activations -> four int8 codes (same arithmetic as k_quant_act)
    float v[4];
    load_x4<BF16>(X, idx, v);
    uint32_t w = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) w |= static_cast<uint32_t>(static_cast<uint8_t>(quant_code(v[j], s))) << (8 * j);
    return w;
}

template <bool BF16>
__global__ void __launch_bounds__(kFusedWarps * 32, 2) k_gemv_fused(const uint2 *__restrict__ dec, const void *__restrict__ X,
                                                                 float eps, const float *__restrict__ gamma, int T,
                                                                 int64_t n_out, int64_t K, void *__restrict__ Y,
                                                                 int y_bf16, int32_t *__restrict__ acc_out,
                                                                 int8_t *__restrict__ xq_out, float *__restrict__ amax_out) {
    // dynamic shared memory: the int8 codes of the T activation rows, row pitch
    // K + 16 bytes so that the 8 token rows of a B fragment fall in different banks
    extern __shared__ __align__(16) int8_t s_xq[];
    __shared__ int s_part[kFusedWarps][32][4];
    __shared__ float s_red[kFusedWarps][8];
    __shared__ float s_amax[8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gid = lane >> 2, tq = lane & 3;
    const int64_t rt = blockIdx.x;
    const int64_t ktiles = K / 64;
    const int64_t pitch = K + 16;
    const int64_t per_warp = (ktiles + kFusedWarps - 1) / kFusedWarps;
    const int64_t kt0 = warp * per_warp;
    const int64_t kt1 = (kt0 + per_warp < ktiles) ? kt0 + per_warp : ktiles;
    const uint2 *src = dec + (rt * ktiles) * 32 + lane;

    // 1. weights: independent of the previous kernel, issued before the wait
    uint2 w[kFusedRegTiles];
#pragma unroll
    for (int i = 0; i < kFusedRegTiles; ++i)
        if (kt0 + i < kt1) w[i] = __ldg(src + (kt0 + i) * 32);
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // 2. per-token absmax over the whole row (every CTA recomputes it from L2)
    float m[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) m[t] = 0.0f;
    for (int64_t i = 4 * threadIdx.x; i < K; i += 4 * blockDim.x) {
#pragma unroll
        for (int t = 0; t < 8; ++t)
            if (t < T) {
                float v[4];
                load_x4<BF16>(X, t * K + i, v);
                m[t] = fmaxf(fmaxf(m[t], fmaxf(fabsf(v[0]), fabsf(v[1]))), fmaxf(fabsf(v[2]), fabsf(v[3])));
            }
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m[t] = fmaxf(m[t], __shfl_xor_sync(0xffffffffu, m[t], o));
    }
    if (lane == 0) {
#pragma unroll
        for (int t = 0; t < 8; ++t) s_red[warp][t] = m[t];
    }
    __syncthreads();
    if (threadIdx.x < 8) {
        float v = 0.0f;
        for (int q = 0; q < kFusedWarps; ++q) v = fmaxf(v, s_red[q][threadIdx.x]);
        s_amax[threadIdx.x] = v > eps ? v : eps;
    }
    __syncthreads();
    // 3. quantise the rows once into shared memory (four codes per thread step, L1/L2 hits)
    for (int t = 0; t < T; ++t) {
        const float st = __fdiv_rn(127.0f, s_amax[t]);
        for (int64_t i = 4 * threadIdx.x; i < K; i += 4 * blockDim.x)
            *reinterpret_cast<uint32_t *>(s_xq + t * pitch + i) = quant4<BF16>(X, t * K + i, st);
    }
    __syncthreads();

    // 4. sparse MMAs over this warp's k-range; B fragments from shared memory
    const bool tok = gid < T;
    const int8_t *xs = s_xq + (tok ? gid : 0) * pitch + 4 * tq;
    int d[4] = {0, 0, 0, 0};
    for (int64_t base = kt0; base < kt1; base += kFusedRegTiles) {
        if (base != kt0) {
#pragma unroll
            for (int i = 0; i < kFusedRegTiles; ++i)
                if (base + i < kt1) w[i] = __ldg(src + (base + i) * 32);
        }
#pragma unroll
        for (int i = 0; i < kFusedRegTiles; ++i) {
            const int64_t kt = base + i;
            if (kt < kt1) {
                uint32_t a[4], b[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    b[j] = tok ? *reinterpret_cast<const uint32_t *>(xs + kt * 64 + 16 * j) : 0u;
#pragma unroll
                for (int r = 0; r < 4; ++r) a[r] = expand_codes(w[i].x, r);
                mma_sp_m16n8k64(d, a, b, w[i].y);
            }
        }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) s_part[warp][lane][q] = d[q];
    __syncthreads();
    if (blockIdx.x == 0 && (xq_out || amax_out)) {   // optional copy of the int8 activations
        for (int64_t i = threadIdx.x; i < static_cast<int64_t>(T) * K; i += blockDim.x) {
            const int64_t t = i / K;
            if (xq_out) xq_out[i] = s_xq[t * pitch + (i - t * K)];
        }
        if (amax_out && threadIdx.x < T) amax_out[threadIdx.x] = s_amax[threadIdx.x];
    }
    if (warp != 0) return;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        int sum = 0;
#pragma unroll
        for (int w2 = 0; w2 < kFusedWarps; ++w2) sum += s_part[w2][lane][q];
        d[q] = sum;
    }
    const float g = *gamma;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int row = gid + 8 * (q >> 1);
        const int t = 2 * tq + (q & 1);
        if (t >= T) continue;
        const int64_t n = rt * 16 + row;
        const float scale = __fdiv_rn(__fmul_rn(g, s_amax[t]), 127.0f);
        const float y = __fmul_rn(__int2float_rn(d[q]), scale);
        if (y_bf16)
            static_cast<__nv_bfloat16 *>(Y)[t * n_out + n] = __float2bfloat16_rn(y);
        else
            static_cast<float *>(Y)[t * n_out + n] = y;
        if (acc_out) acc_out[t * n_out + n] = d[q];
    }
}

cudaError_t launch_gemv_fused(const void *X, bool x_bf16, float eps, const float *gamma, const uint8_t *dec,
                              int64_t T, int64_t n_out, int64_t k, void *Y, bool y_bf16, int32_t *acc,
                              int8_t *xq_out, float *amax_out, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n_out / 16));
    cfg.blockDim = dim3(kFusedWarps * 32);
    cfg.dynamicSmemBytes = static_cast<size_t>(T) * static_cast<size_t>(k + 16);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const uint2 *d2 = reinterpret_cast<const uint2 *>(dec);
    const int Ti = static_cast<int>(T);
    const int yb = y_bf16 ? 1 : 0;
    static bool attr_done[2] = {false, false};
    if (!attr_done[x_bf16 ? 1 : 0]) {
        cudaError_t e = x_bf16 ? cudaFuncSetAttribute(k_gemv_fused<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                      static_cast<int>(kFusedMaxSmem))
                               : cudaFuncSetAttribute(k_gemv_fused<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                      static_cast<int>(kFusedMaxSmem));
        if (e != cudaSuccess) return e;
        attr_done[x_bf16 ? 1 : 0] = true;
    }
    if (x_bf16)
        return cudaLaunchKernelEx(&cfg, k_gemv_fused<true>, d2, X, eps, gamma, Ti, n_out, k, Y, yb, acc, xq_out,
                                  amax_out);
    return cudaLaunchKernelEx(&cfg, k_gemv_fused<false>, d2, X, eps, gamma, Ti, n_out, k, Y, yb, acc, xq_out, amax_out);
}

cudaError_t launch_gemv_dec(const int8_t *Xq, const float *amax, const float *gamma, const uint8_t *dec,
                            int64_t T, int64_t n_out, int64_t k, void *Y, bool y_bf16, int32_t *acc,
                            cudaStream_t s) {
    const int warps = gemv_warps(k);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n_out / 16));
    cfg.blockDim = dim3(warps * 32);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const uint2 *d2 = reinterpret_cast<const uint2 *>(dec);
    if (warps == 4)
        return cudaLaunchKernelEx(&cfg, k_gemv_dec<4>, d2, Xq, amax, gamma, static_cast<int>(T), n_out, k, Y,
                                  y_bf16 ? 1 : 0, acc);
    return cudaLaunchKernelEx(&cfg, k_gemv_dec<8>, d2, Xq, amax, gamma, static_cast<int>(T), n_out, k, Y,
                              y_bf16 ? 1 : 0, acc);
}

cudaError_t launch_gemv_gb(const int8_t *Xq, const float *amax, const float *gamma, const uint8_t *gb,
                           int64_t T, int64_t n_out, int64_t k, void *Y, bool y_bf16, int32_t *acc,
                           cudaStream_t s) {
    int64_t blocks = (n_out + 7) / 8;
    const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
    if (blocks > cap) blocks = cap;
    k_gemv_gb<<<static_cast<unsigned>(blocks), 256, 0, s>>>(gb, Xq, amax, gamma, static_cast<int>(T), n_out, k, Y,
                                                            y_bf16 ? 1 : 0, acc);
    return cudaGetLastError();
}

}  // namespace bitnet
