// Per-token absmax int8 activation quantisation (sm_100a).
//
// "BitNet b1.58: Ternary Weights for 1.58-bit LLMs", section "The mechanism"
// (Activations): every token is scaled to the symmetric range [-Q_b, Q_b]
// with no zero-point; Q_b = 127.
//   a = max(max_k |x_k|, eps),  s = 127 / a,  q_k = clamp(rint(x_k * s), -127, 127)
// Division, product and rounding are single IEEE operations (round to
// nearest even), so the codes are bit-exact.  The rounding is one fp32 add of
// 1.5 x 2^23 (codes4_fast / codes8_fast): |x s| <= 127 (1 + 2^-24) here, so
// the add rounds exactly as rint and the clamp never acts.
//
// Each token row is read once with 16-byte loads into registers, reduced to
// its absmax, then quantised from registers and written with vector stores:
// 2 bytes read + 1 byte written per bf16 element.
#include "common.cuh"
#include "kernels.h"

namespace bitnet {

constexpr int kQuantThreads = 256;
constexpr int kQuantMaxChunks = 8;   // 16-byte chunks kept in registers per thread

template <bool BF16>
struct Chunk {
    static constexpr int kElems = BF16 ? 8 : 4;
    uint4 raw;
    __device__ __forceinline__ float get(int j) const {
        const uint32_t w = (&raw.x)[BF16 ? (j >> 1) : j];
        if (BF16) return __uint_as_float((j & 1) ? (w & 0xffff0000u) : (w << 16));
        return __uint_as_float(w);
    }
};

// Running |x| max of a thread's chunks.  bf16: the sign-cleared bit patterns
// of each half-word under max.u16x2 (one instruction per element, the order of
// the patterns being the order of the magnitudes); fp32: fmaxf of |x|.
template <bool BF16>
struct AbsMax {
    uint32_t m2 = 0u;
    float mf = 0.0f;
    __device__ __forceinline__ void add(const Chunk<BF16> &c) {
        if constexpr (BF16) {
            const uint32_t k = 0x7fff7fffu;
            m2 = vmax_u16x2(m2, vmax_u16x2(vmax_u16x2(c.raw.x & k, c.raw.y & k), vmax_u16x2(c.raw.z & k, c.raw.w & k)));
        } else {
            mf = fmaxf(fmaxf(mf, fmaxf(fabsf(__uint_as_float(c.raw.x)), fabsf(__uint_as_float(c.raw.y)))),
                       fmaxf(fabsf(__uint_as_float(c.raw.z)), fabsf(__uint_as_float(c.raw.w))));
        }
    }
    __device__ __forceinline__ float value() const {
        if constexpr (BF16) {
            const uint32_t hi = m2 >> 16, lo = m2 & 0xffffu;
            return __uint_as_float((hi > lo ? hi : lo) << 16);
        } else {
            return mf;
        }
    }
};

// Codes of one chunk stored at out (chunk c of the row): 8 bytes for bf16, 4 for fp32.
template <bool BF16>
__device__ __forceinline__ void store_codes(const Chunk<BF16> &c, float s, int8_t *out) {
    if constexpr (BF16) {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = c.get(j);
        *reinterpret_cast<uint2 *>(out) = codes8_fast(v, s);
    } else {
        *reinterpret_cast<uint32_t *>(out) = codes4_fast(c.get(0), c.get(1), c.get(2), c.get(3), s);
    }
}

__device__ __forceinline__ float block_max(float v, float *s_red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) s_red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = (lane < (int)(blockDim.x >> 5)) ? s_red[lane] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) s_red[0] = v;
    }
    __syncthreads();
    return s_red[0];
}

// Loads the register-cached chunks of token group g: thread gt of token slot
// grp takes chunks gt, gt + kTpt, ... of its row.  Rows past T load nothing.
template <bool BF16, int TPC>
__device__ __forceinline__ void quant_load(Chunk<BF16> (&r)[kQuantMaxChunks], const uint4 *__restrict__ X, int64_t T,
                                           int64_t K, int64_t g, int grp, int gt) {
    using C = Chunk<BF16>;
    constexpr int kTpt = kQuantThreads / TPC;
    const int64_t t = g * TPC + grp;
    const int64_t nchunk = t < T ? K / C::kElems : 0;
    const uint4 *row = X + t * (K / C::kElems);
#pragma unroll
    for (int u = 0; u < kQuantMaxChunks; ++u) {
        const int64_t c = gt + static_cast<int64_t>(u) * kTpt;
        if (c < nchunk) r[u].raw = __ldg(row + c);
    }
}

// Absmax, scale and codes of token group g from its cached chunks (plus a
// second read of any chunks beyond the cache).  One CTA barrier: the token's
// warps publish their maxima in s_red.
template <bool BF16, int TPC>
__device__ __forceinline__ void quant_group(const Chunk<BF16> (&r)[kQuantMaxChunks], const uint4 *__restrict__ X,
                                            int64_t T, int64_t K, float eps, int8_t *__restrict__ Xq,
                                            float *__restrict__ amax, int64_t g, int grp, int gt, float *s_red) {
    using C = Chunk<BF16>;
    constexpr int kTpt = kQuantThreads / TPC;   // threads per token
    constexpr int kWpt = kTpt / 32;             // warps per token
    const int64_t t = g * TPC + grp;
    const bool valid = t < T;
    const int64_t nchunk = valid ? K / C::kElems : 0;
    const bool fits = nchunk <= static_cast<int64_t>(kQuantMaxChunks) * kTpt;
    const uint4 *row = X + t * (K / C::kElems);
    AbsMax<BF16> am;
#pragma unroll
    for (int u = 0; u < kQuantMaxChunks; ++u) {
        const int64_t c = gt + static_cast<int64_t>(u) * kTpt;
        if (c < nchunk) am.add(r[u]);
    }
    if (!fits) {   // rows longer than the register cache: a second read later
        for (int64_t c = gt + static_cast<int64_t>(kQuantMaxChunks) * kTpt; c < nchunk; c += kTpt) {
            C ch;
            ch.raw = __ldg(row + c);
            am.add(ch);
        }
    }
    float m = am.value();
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = m;
    __syncthreads();
    m = s_red[grp * kWpt];
#pragma unroll
    for (int w = 1; w < kWpt; ++w) m = fmaxf(m, s_red[grp * kWpt + w]);
    if (!valid) return;
    const float a = m > eps ? m : eps;
    const float s = __fdiv_rn(127.0f, a);
    if (gt == 0) amax[t] = a;
    int8_t *out = Xq + t * K;
#pragma unroll
    for (int u = 0; u < kQuantMaxChunks; ++u) {
        const int64_t c = gt + static_cast<int64_t>(u) * kTpt;
        if (c < nchunk) store_codes<BF16>(r[u], s, out + c * C::kElems);
    }
    if (!fits) {
        for (int64_t c = gt + static_cast<int64_t>(kQuantMaxChunks) * kTpt; c < nchunk; c += kTpt) {
            C ch;
            ch.raw = __ldg(row + c);
            store_codes<BF16>(ch, s, out + c * C::kElems);
        }
    }
}

// One token group of TPC tokens per CTA, kQuantThreads / TPC threads (a whole
// number of warps) per token: short rows pack several tokens into one CTA so
// that each thread keeps up to kQuantMaxChunks loads in flight.  At most 64
// registers, so four CTAs (32 warps) share an SM.  (A persistent form that
// keeps the next group's loads in flight while quantising the current one
// measured the same on the 4096 x 4096 and 4096 x 11008 prefill rows, with
// twice the registers.)
template <bool BF16, int TPC>
__global__ void __launch_bounds__(kQuantThreads, 4) k_quant_act(const uint4 *__restrict__ X, int64_t T, int64_t K,
                                                                float eps, int8_t *__restrict__ Xq,
                                                                float *__restrict__ amax) {
    __shared__ float s_red[kQuantThreads / 32];
    constexpr int kTpt = kQuantThreads / TPC;
    const int grp = threadIdx.x / kTpt, gt = threadIdx.x % kTpt;
    Chunk<BF16> r[kQuantMaxChunks];
    // X may be the output of the previous kernel of the stream
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    quant_load<BF16, TPC>(r, X, T, K, blockIdx.x, grp, gt);
    quant_group<BF16, TPC>(r, X, T, K, eps, Xq, amax, blockIdx.x, grp, gt, s_red);
}

template <bool BF16, int TPC>
static cudaError_t quant_launch(cudaLaunchConfig_t &cfg, const uint4 *x, int64_t T, int64_t K, float eps, int8_t *Xq,
                                float *amax) {
    cfg.gridDim = dim3(static_cast<unsigned>((T + TPC - 1) / TPC));
    return cudaLaunchKernelEx(&cfg, k_quant_act<BF16, TPC>, x, T, K, eps, Xq, amax);
}

cudaError_t launch_quant_act(const void *X, bool bf16, int64_t T, int64_t K, float eps, int8_t *Xq, float *amax,
                             cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    // tokens per CTA: the most whose rows still fit the register cache (and at least one chunk per thread)
    const int64_t nchunk = K / (bf16 ? 8 : 4);
    int tpc = 1;
    for (int c = 8; c > 1; c >>= 1)
        if (nchunk <= static_cast<int64_t>(kQuantMaxChunks) * (kQuantThreads / c) && nchunk >= kQuantThreads / c &&
            T >= 2 * c) {
            tpc = c;
            break;
        }
    // programmatic serialisation: the kernel that consumes Xq may start its own
    // independent loads while this one runs
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kQuantThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const uint4 *x = static_cast<const uint4 *>(X);
    switch (tpc) {
        case 8: return bf16 ? quant_launch<true, 8>(cfg, x, T, K, eps, Xq, amax) : quant_launch<false, 8>(cfg, x, T, K, eps, Xq, amax);
        case 4: return bf16 ? quant_launch<true, 4>(cfg, x, T, K, eps, Xq, amax) : quant_launch<false, 4>(cfg, x, T, K, eps, Xq, amax);
        case 2: return bf16 ? quant_launch<true, 2>(cfg, x, T, K, eps, Xq, amax) : quant_launch<false, 2>(cfg, x, T, K, eps, Xq, amax);
        default: return bf16 ? quant_launch<true, 1>(cfg, x, T, K, eps, Xq, amax) : quant_launch<false, 1>(cfg, x, T, K, eps, Xq, amax);
    }
}


// ---------------------------------------------------------------- activation lifting for 6:8 windows
//
// "Is 2:4 Sparsity Still Worth It? ..." (thelatestinai.com), its SlideSparse
// entry: the activation rearrangement that matches the window decomposition
// of the weights is done inside per-token quantisation.  For 6:8 each block of
// 8 activations x[8b .. 8b+7] becomes 12 codes, the three overlapping windows
// x[8b + 2w .. 8b + 2w + 3] (w = 0, 1, 2).  The scale is the token's absmax
// over its original row, so every code equals bitnet_quant_act's.
template <bool BF16>
__global__ void __launch_bounds__(kQuantThreads) k_quant_lift68(const uint8_t *__restrict__ X, int64_t K, float eps,
                                                                int8_t *__restrict__ Xl, float *__restrict__ amax) {
    __shared__ float s_red[32];
    const int64_t t = blockIdx.x;
    const int64_t esize = BF16 ? 2 : 4;
    const uint8_t *row = X + t * K * esize;
    const int64_t blocks = K / 8;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    float m = 0.0f;
    for (int64_t b = threadIdx.x; b < blocks; b += kQuantThreads) {
        float v[8];
        if (BF16) {
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(row) + b);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = __uint_as_float((j & 1) ? (w[j >> 1] & 0xffff0000u) : (w[j >> 1] << 16));
        } else {
            const float4 a = __ldg(reinterpret_cast<const float4 *>(row) + 2 * b);
            const float4 c = __ldg(reinterpret_cast<const float4 *>(row) + 2 * b + 1);
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = c.x; v[5] = c.y; v[6] = c.z; v[7] = c.w;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
    }
    m = block_max(m, s_red);
    const float a = m > eps ? m : eps;
    const float sc = __fdiv_rn(127.0f, a);
    if (threadIdx.x == 0) amax[t] = a;
    int8_t *out = Xl + t * (K / 2 * 3);
    for (int64_t b = threadIdx.x; b < blocks; b += kQuantThreads) {
        float v[8];
        if (BF16) {
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(row) + b);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = __uint_as_float((j & 1) ? (w[j >> 1] & 0xffff0000u) : (w[j >> 1] << 16));
        } else {
            const float4 a4 = __ldg(reinterpret_cast<const float4 *>(row) + 2 * b);
            const float4 c4 = __ldg(reinterpret_cast<const float4 *>(row) + 2 * b + 1);
            v[0] = a4.x; v[1] = a4.y; v[2] = a4.z; v[3] = a4.w; v[4] = c4.x; v[5] = c4.y; v[6] = c4.z; v[7] = c4.w;
        }
        const uint2 q = codes8_fast(v, sc);   // codes 0-3 | 4-7
        // windows 0, 1, 2: codes 0-3, 2-5, 4-7
        uint32_t *dst = reinterpret_cast<uint32_t *>(out + 12 * b);
        dst[0] = q.x;
        dst[1] = __byte_perm(q.x, q.y, 0x5432u);
        dst[2] = q.y;
    }
}

cudaError_t launch_quant_lift68(const void *X, bool bf16, int64_t T, int64_t K, float eps, int8_t *Xl, float *amax,
                                cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(T));
    cfg.blockDim = dim3(kQuantThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const uint8_t *x = static_cast<const uint8_t *>(X);
    if (bf16) return cudaLaunchKernelEx(&cfg, k_quant_lift68<true>, x, K, eps, Xl, amax);
    return cudaLaunchKernelEx(&cfg, k_quant_lift68<false>, x, K, eps, Xl, amax);
}

}  // namespace bitnet
