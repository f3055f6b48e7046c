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
#include "frag.cuh"
#include "kernels.h"

namespace bitnet {

constexpr int kDecRegTiles = 16;   // k-tiles (8 bytes each) prefetched per lane per round

// Warps per CTA so that one prefetch round holds every k-tile of a warp
// (K <= 4096: 4 warps; K <= 8192: 8 warps; beyond, several rounds).
inline int gemv_warps(int64_t k) { return (k / 64 + 3) / 4 <= kDecRegTiles ? 4 : 8; }

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
