// Block epilogues fused into per-token int8 quantisation (sm_100a):
// RMSNorm -> quant and SwiGLU -> quant.
//
// "BitNet b1.58: Ternary Weights for 1.58-bit LLMs", "What this paper
// explains" item 3: the Transformer stack around BitLinear is LLaMA-alike
// (RMSNorm, SwiGLU, no biases); "The mechanism": the activations entering a
// BitLinear are quantised per token to [-127, 127].  Fusing the norm or the
// gate into the quantisation reads the bf16 activations once and writes int8.
//
// The pages fix no precision for these steps.  The definitions used (the
// oracle follows the same ones):
//  * RMSNorm: S = exact sum of x^2 over the row, rounded once to fp64;
//    ms = fp32(S / K); r = fp32(1 / fp32(sqrt(fp32(ms + eps))));
//    x_n = fp32(x * r), then fp32(x_n * w_k) when a weight vector is given.
//  * SwiGLU: h = fp32(silu(g) * u), silu(g) = fp32(g / fp32(1 + exp32(-g)));
//    exp32 is Cody-Waite range reduction (x = n ln2 + r, ln2 split in a short
//    high part and a correction) followed by the degree-6 Taylor polynomial of
//    e^r on |r| <= ln2 / 2, every step one IEEE fp32 operation.
// Then a = max(max_k |h_k|, eps), s = fp32(127 / a), q = clamp(rint(fp32(h s))),
// as in bitnet_quant_act.  Every step is a single IEEE operation in a fixed
// order, so the codes are bit-exact.
//
// The exact sum of squares: a bf16 value is M 2^(e) with an 8-bit
// significand M, so x^2 = M^2 2^te with M^2 < 2^16.  Squares with te in a
// window of 80 binary places go into a per-thread 128-bit fixed-point
// accumulator (at most 2^15 terms below 2^96 each: no overflow); the rest
// (tiny, huge, subnormal) go into per-exponent integer bins in shared memory.
// One thread turns window + bins into the nearest fp64 with 32-bit limbs.
#include "common.cuh"
#include "frag.cuh"
#include "kernels.h"

namespace bitnet {

constexpr int kBqThreads = 256;
constexpr int kSqTe0 = -74;                // window: x^2 = M^2 2^te with kSqTe0 <= te < kSqTe0 + 80
constexpr int kSqTeMin = -266;             // smallest te (subnormal bf16)
constexpr int kSqBins = 240 - kSqTeMin + 1;   // te in [-266, 240]
constexpr int kSqLimbs = 18;               // 576 bits from 2^-266 upward

__device__ __forceinline__ void add128_sq(uint64_t &lo, uint64_t &hi, uint64_t vlo, uint64_t vhi) {
    const uint64_t s = lo + vlo;
    hi += vhi + (s < lo ? 1ull : 0ull);
    lo = s;
}

// x^2 of one bf16 value (16 bits) into the window accumulator or the bins
__device__ __forceinline__ void sq_accumulate(uint32_t b16, uint64_t &lo, uint64_t &hi,
                                              unsigned long long *s_bins, int *s_rare) {
    const uint32_t E = (b16 >> 7) & 0xffu, m7 = b16 & 0x7fu;
    if (E == 0u && m7 == 0u) return;                       // +-0
    const uint32_t M = E ? (m7 | 0x80u) : m7;
    const int te = E ? 2 * static_cast<int>(E) - 268 : -266;
    const uint64_t M2 = static_cast<uint64_t>(M * M);
    const int sh = te - kSqTe0;
    if (sh >= 0 && sh < 80) {
        if (sh < 64) add128_sq(lo, hi, M2 << sh, sh ? (M2 >> (64 - sh)) : 0ull);
        else add128_sq(lo, hi, 0ull, M2 << (sh - 64));
    } else {
        atomicAdd(&s_bins[te - kSqTeMin], static_cast<unsigned long long>(M2));
        *s_rare = 1;
    }
}

// value += v 2^shift on little-endian 32-bit limbs
__device__ void sq_limbs_add(uint32_t *limb, uint64_t v, int shift) {
    const int q = shift >> 5, r = shift & 31;
    const uint64_t lo = v << r;
    const uint64_t hi = r ? (v >> (64 - r)) : 0ull;
    const uint64_t add[3] = {lo & 0xffffffffull, lo >> 32, hi};
    uint64_t carry = 0;
    for (int j = q; j < kSqLimbs; ++j) {
        const uint64_t a = (j - q < 3) ? add[j - q] : 0ull;
        if (j - q >= 3 && carry == 0) break;
        const uint64_t s2 = static_cast<uint64_t>(limb[j]) + a + carry;
        limb[j] = static_cast<uint32_t>(s2);
        carry = s2 >> 32;
    }
}

// nearest fp64 of the exact sum (window in units 2^kSqTe0, bins by te); one thread
__device__ double sq_finalize(uint64_t wlo, uint64_t whi, const unsigned long long *bins, bool rare, uint32_t *limb) {
    for (int j = 0; j < kSqLimbs; ++j) limb[j] = 0u;
    sq_limbs_add(limb, wlo, kSqTe0 - kSqTeMin);
    sq_limbs_add(limb, whi, kSqTe0 - kSqTeMin + 64);
    if (rare)
        for (int i = 0; i < kSqBins; ++i)
            if (bins[i]) sq_limbs_add(limb, bins[i], i);
    int L = -1;
    for (int j = kSqLimbs - 1; j >= 0; --j)
        if (limb[j]) {
            L = j;
            break;
        }
    if (L < 0) return 0.0;
    if (L <= 1) {
        const uint64_t v = (static_cast<uint64_t>(L == 1 ? limb[1] : 0u) << 32) | limb[0];
        return __ull2double_rn(v) * 0x1p-266;   // power-of-two scaling, exact in the normal range
    }
    // top 64 bits of the top three limbs, everything below folded into a sticky bit
    const int lz = __clz(limb[L]);
    const int shift = 32 - lz;   // bits of the top limb kept above the 64-bit window
    const uint64_t top = (static_cast<uint64_t>(limb[L]) << 32) | limb[L - 1];
    uint64_t w64 = shift == 32 ? top : ((top << (32 - shift)) | (limb[L - 2] >> shift));
    bool sticky = shift == 32 ? (limb[L - 2] != 0u) : ((limb[L - 2] & ((1u << shift) - 1u)) != 0u);
    for (int j = 0; j < L - 2 && !sticky; ++j) sticky = limb[j] != 0u;
    if (sticky) w64 |= 1ull;   // bit 0 lies below the 53-bit rounding position
    const int ex = 32 * (L - 2) + shift - 266;   // weight of bit 0 of w64 (2^ex)
    return __ull2double_rn(w64) * __longlong_as_double(static_cast<long long>(1023 + ex) << 52);
}

// exp in fp32, the definition above (x clamped to [-87, 88]; no fused multiply-add)
// Constants are given as fp32 bit patterns: log2(e), ln2 split into a 16-bit
// high part and the rest, and the Taylor coefficients 1/720, 1/120, 1/24, 1/6.
__device__ __forceinline__ float exp32(float x) {
    x = fminf(fmaxf(x, -87.0f), 88.0f);
    const float n = rintf(__fmul_rn(x, __uint_as_float(0x3fb8aa3bu)));
    float r = __fsub_rn(x, __fmul_rn(n, __uint_as_float(0x3f317200u)));
    r = __fsub_rn(r, __fmul_rn(n, __uint_as_float(0x35bfbe8eu)));
    float p = __uint_as_float(0x3ab60b61u);
    p = __fadd_rn(__fmul_rn(p, r), __uint_as_float(0x3c088889u));
    p = __fadd_rn(__fmul_rn(p, r), __uint_as_float(0x3d2aaaabu));
    p = __fadd_rn(__fmul_rn(p, r), __uint_as_float(0x3e2aaaabu));
    p = __fadd_rn(__fmul_rn(p, r), 0.5f);
    p = __fadd_rn(__fmul_rn(p, r), 1.0f);
    p = __fadd_rn(__fmul_rn(p, r), 1.0f);
    return __fmul_rn(p, __int_as_float((static_cast<int>(n) + 127) << 23));
}

__device__ __forceinline__ float bf16_at(const uint16_t *p, int64_t i) {
    return __uint_as_float(static_cast<uint32_t>(__ldg(p + i)) << 16);
}

__device__ __forceinline__ float bq_block_max(float v, float *s_red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) s_red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < static_cast<int>(blockDim.x >> 5) ? s_red[lane] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) s_red[0] = v;
    }
    __syncthreads();
    const float r = s_red[0];
    __syncthreads();
    return r;
}

// int8 code of one value with scale s (as bitnet_quant_act)
__device__ __forceinline__ uint32_t bq_code(float v, float s) { return static_cast<uint8_t>(quant_code(v, s)); }

// RMSNorm -> int8, one CTA per token.  X bf16 [T, K], optional fp32 weight w [K].
// Pass 1 sums x^2 exactly; thread 0 forms r; pass 2 normalises, takes the
// absmax; pass 3 writes the codes (the row is re-read from L1/L2).  rinv, when
// given, receives r per token (what the backward of the norm needs).
__global__ void __launch_bounds__(kBqThreads) k_rmsnorm_quant(const uint16_t *__restrict__ X, const float *__restrict__ w,
                                                              int64_t K, float eps_n, float eps_a,
                                                              int8_t *__restrict__ Xq, float *__restrict__ amax,
                                                              float *__restrict__ rinv) {
    __shared__ unsigned long long s_bins[kSqBins];
    __shared__ unsigned long long s_lo[kBqThreads / 32], s_hi[kBqThreads / 32];
    __shared__ uint32_t s_limb[kSqLimbs];
    __shared__ float s_red[32];
    __shared__ float s_r;
    __shared__ int s_rare;
    const int64_t t = blockIdx.x;
    const uint16_t *row = X + t * K;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < kSqBins; i += kBqThreads) s_bins[i] = 0ull;
    if (threadIdx.x == 0) s_rare = 0;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __syncthreads();
    uint64_t lo = 0, hi = 0;
    const int64_t nchunk = K / 8;   // 8 bf16 = 16 bytes
    for (int64_t c = threadIdx.x; c < nchunk; c += kBqThreads) {
        const uint4 u = __ldg(reinterpret_cast<const uint4 *>(row) + c);
        const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            sq_accumulate(wv[j] & 0xffffu, lo, hi, s_bins, &s_rare);
            sq_accumulate(wv[j] >> 16, lo, hi, s_bins, &s_rare);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t l2 = __shfl_xor_sync(0xffffffffu, lo, o), h2 = __shfl_xor_sync(0xffffffffu, hi, o);
        add128_sq(lo, hi, l2, h2);
    }
    if (lane == 0) {
        s_lo[warp] = lo;
        s_hi[warp] = hi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint64_t L = 0, H = 0;
        for (int i = 0; i < kBqThreads / 32; ++i) add128_sq(L, H, s_lo[i], s_hi[i]);
        const double S = sq_finalize(L, H, s_bins, s_rare != 0, s_limb);
        const float ms = __double2float_rn(__ddiv_rn(S, static_cast<double>(K)));
        s_r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps_n)));
        if (rinv) rinv[t] = s_r;
    }
    __syncthreads();
    const float r = s_r;
    float m = 0.0f;
    for (int64_t i = threadIdx.x; i < K; i += kBqThreads) {
        float v = __fmul_rn(bf16_at(row, i), r);
        if (w) v = __fmul_rn(v, __ldg(w + i));
        m = fmaxf(m, fabsf(v));
    }
    m = bq_block_max(m, s_red);
    const float a = m > eps_a ? m : eps_a;
    const float s = __fdiv_rn(127.0f, a);
    if (threadIdx.x == 0) amax[t] = a;
    int8_t *out = Xq + t * K;
    for (int64_t i0 = 4 * threadIdx.x; i0 < K; i0 += 4 * kBqThreads) {
        uint32_t q = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float v = __fmul_rn(bf16_at(row, i0 + j), r);
            if (w) v = __fmul_rn(v, __ldg(w + i0 + j));
            q |= bq_code(v, s) << (8 * j);
        }
        *reinterpret_cast<uint32_t *>(out + i0) = q;
    }
}

// SwiGLU -> int8, one CTA per token.  G, U bf16 with row stride ld (elements),
// F columns each.  h is kept in shared memory (F fp32) between the absmax and
// the codes.
__global__ void __launch_bounds__(kBqThreads) k_swiglu_quant(const uint16_t *__restrict__ G, const uint16_t *__restrict__ U,
                                                             int64_t ld, int64_t F, float eps_a,
                                                             int8_t *__restrict__ Xq, float *__restrict__ amax) {
    extern __shared__ float s_h[];
    __shared__ float s_red[32];
    const int64_t t = blockIdx.x;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    float m = 0.0f;
    for (int64_t i = threadIdx.x; i < F; i += kBqThreads) {
        const float g = bf16_at(G, t * ld + i), u = bf16_at(U, t * ld + i);
        const float silu = __fdiv_rn(g, __fadd_rn(1.0f, exp32(-g)));
        const float h = __fmul_rn(silu, u);
        s_h[i] = h;
        m = fmaxf(m, fabsf(h));
    }
    m = bq_block_max(m, s_red);   // also orders the s_h writes before the reads below
    const float a = m > eps_a ? m : eps_a;
    const float s = __fdiv_rn(127.0f, a);
    if (threadIdx.x == 0) amax[t] = a;
    int8_t *out = Xq + t * F;
    for (int64_t i0 = 4 * threadIdx.x; i0 < F; i0 += 4 * kBqThreads) {
        uint32_t q = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) q |= bq_code(s_h[i0 + j], s) << (8 * j);
        *reinterpret_cast<uint32_t *>(out + i0) = q;
    }
}

static cudaLaunchConfig_t bq_config(int64_t T, size_t smem, cudaStream_t s, cudaLaunchAttribute *attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(T));
    cfg.blockDim = dim3(kBqThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

cudaError_t launch_rmsnorm_quant(const void *X, const float *w, int64_t T, int64_t K, float eps_n, float eps_a,
                                 int8_t *Xq, float *amax, float *rinv, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = bq_config(T, 0, s, attr);
    return cudaLaunchKernelEx(&cfg, k_rmsnorm_quant, static_cast<const uint16_t *>(X), w, K, eps_n, eps_a, Xq, amax,
                              rinv);
}

size_t swiglu_smem_bytes(int64_t F) { return static_cast<size_t>(F) * 4; }

cudaError_t launch_swiglu_quant(const void *G, const void *U, int64_t ld, int64_t T, int64_t F, float eps_a,
                                int8_t *Xq, float *amax, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(k_swiglu_quant, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kSwigluMaxSmem));
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = bq_config(T, swiglu_smem_bytes(F), s, attr);
    return cudaLaunchKernelEx(&cfg, k_swiglu_quant, static_cast<const uint16_t *>(G), static_cast<const uint16_t *>(U),
                              ld, F, eps_a, Xq, amax);
}

}  // namespace bitnet
