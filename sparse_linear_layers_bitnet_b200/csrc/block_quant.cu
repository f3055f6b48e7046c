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
    uint64_t carry = 0;
    for (int j = q; j < kSqLimbs; ++j) {
        const int d = j - q;
        const uint64_t a = d == 0 ? (lo & 0xffffffffull) : d == 1 ? (lo >> 32) : d == 2 ? hi : 0ull;
        if (d >= 3 && carry == 0) break;
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
    // n = rint(x log2 e): adding 1.5 2^23 rounds to an integer (ties to even) for
    // |x log2 e| < 2^22 and leaves it in the low bits of the sum
    const float big = __fadd_rn(__fmul_rn(x, __uint_as_float(0x3fb8aa3bu)), 12582912.0f);
    const float n = __fsub_rn(big, 12582912.0f);
    const int ni = __float_as_int(big) - 0x4b400000;
    float r = __fsub_rn(x, __fmul_rn(n, __uint_as_float(0x3f317200u)));
    r = __fsub_rn(r, __fmul_rn(n, __uint_as_float(0x35bfbe8eu)));
    float p = __uint_as_float(0x3ab60b61u);
    p = __fadd_rn(__fmul_rn(p, r), __uint_as_float(0x3c088889u));
    p = __fadd_rn(__fmul_rn(p, r), __uint_as_float(0x3d2aaaabu));
    p = __fadd_rn(__fmul_rn(p, r), __uint_as_float(0x3e2aaaabu));
    p = __fadd_rn(__fmul_rn(p, r), 0.5f);
    p = __fadd_rn(__fmul_rn(p, r), 1.0f);
    p = __fadd_rn(__fmul_rn(p, r), 1.0f);
    return __fmul_rn(p, __int_as_float((ni + 127) << 23));
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

// int8 code of one value with scale s, as bitnet_quant_act: rint(v s) clamped
// to [-127, 127].  |v s| <= 127 (1 + 2^-23)^2 here (|v| <= a, s = fp32(127 / a)),
// so adding 1.5 2^23 rounds v s to an integer (ties to even) exactly as rint,
// and the integer is read from the low bits without a conversion instruction.
__device__ __forceinline__ uint32_t bq_code(float v, float s) {
    int q = __float_as_int(__fadd_rn(__fmul_rn(v, s), 12582912.0f)) - 0x4b400000;
    q = q > 127 ? 127 : (q < -127 ? -127 : q);
    return static_cast<uint32_t>(q) & 0xffu;
}

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

// ---------------------------------------------------------------- register-cached forms
//
// One CTA per token with the whole row held in registers: CPT 16-byte chunks
// per thread, threads = the row's chunks / CPT rounded up to a warp.  All the
// row's loads are issued before any arithmetic, so a CTA keeps its row's bytes
// in flight at once; the row is read from HBM exactly once.

// x^2 of one bf16 value into the window; returns true when it falls outside
__device__ __forceinline__ bool sq_window(uint32_t b16, uint64_t &lo, uint64_t &hi) {
    const uint32_t E = (b16 >> 7) & 0xffu, m7 = b16 & 0x7fu;
    const uint32_t M = E ? (m7 | 0x80u) : m7;
    const int sh = 2 * static_cast<int>(E) - 268 - kSqTe0;
    const uint64_t M2 = static_cast<uint64_t>(M * M);
    if (E != 0u && sh >= 0 && sh < 80) {
        if (sh < 64) add128_sq(lo, hi, M2 << sh, sh ? (M2 >> (64 - sh)) : 0ull);
        else add128_sq(lo, hi, 0ull, M2 << (sh - 64));
        return false;
    }
    return M2 != 0ull;   // +-0 contributes nothing; subnormals and out-of-window squares are rare
}

// window (units 2^kSqTe0) += s for s > 0 an fp64 multiple of 2^kSqTe0 below 2^(kSqTe0 + 116)
__device__ __forceinline__ void window_add_f64(double s, uint64_t &lo, uint64_t &hi) {
    const uint64_t b = static_cast<uint64_t>(__double_as_longlong(s));
    const int k = static_cast<int>(b >> 52) - 1075 - kSqTe0;   // s = m 2^(k + kSqTe0), m < 2^53
    const uint64_t m = (b & 0xfffffffffffffull) | 0x10000000000000ull;
    uint64_t vl, vh = 0ull;
    if (k >= 0) {
        vl = m << k;
        if (k) vh = m >> (64 - k);
    } else {
        vl = m >> (-k);   // exact: s is a multiple of 2^kSqTe0
    }
    add128_sq(lo, hi, vl, vh);
}


// |x| of a normal bf16 (15 bits: exponent E and 7 mantissa bits, at bit 13 of
// a word) as an fp64: the high word with the exponent rebiased by 1023 - 127
__device__ __forceinline__ double bf16abs_f64(uint32_t at13) {
    return __hiloint2double(static_cast<int>(at13 + (896u << 20)), 0);
}

// The squares of one 16-byte chunk (8 bf16) summed in fp64 with no rounding
// and added to the window, when all eight values are normal, in the window
// (97 <= E < 137) and with exponents at most 17 apart: then the squares are
// multiples of 2^te_min below 2^(te_max + 16), te_max - te_min <= 34, so every
// partial sum is a multiple of 2^te_min below 2^(te_min + 53) and each fused
// multiply-add is exact.  Returns false (nothing added) otherwise, zeros and
// subnormals included: the caller then takes the values one by one.
__device__ __forceinline__ bool sq_chunk_f64(const uint4 &v, uint64_t &lo, uint64_t &hi) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t amax2 = 0u, amin2 = 0xffffffffu;   // per 16-bit half: |x| bit patterns
    double s = 0.0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const uint32_t a = w[e] & 0x7fff7fffu;
        amax2 = vmax_u16x2(amax2, a);
        amin2 = vmin_u16x2(amin2, a);
        const double x0 = bf16abs_f64((w[e] & 0x7fffu) << 13);
        const double x1 = bf16abs_f64((w[e] >> 3) & 0x0fffe000u);
        s = __fma_rn(x0, x0, s);
        s = __fma_rn(x1, x1, s);
    }
    const uint32_t emax = max(amax2 & 0xffffu, amax2 >> 16) >> 7;
    const uint32_t emin = min(amin2 & 0xffffu, amin2 >> 16) >> 7;
    if (emin < 97u || emax >= 137u || emax - emin > 17u) return false;
    window_add_f64(s, lo, hi);
    return true;
}

// nearest fp64 of the window value (H:L) 2^kSqTe0
__device__ __forceinline__ double window_to_f64(uint64_t L, uint64_t H) {
    if (H == 0ull) return __ull2double_rn(L) * 0x1p-74;   // power-of-two scaling: exact
    const int lz = __clzll(static_cast<long long>(H));
    uint64_t top = lz ? ((H << lz) | (L >> (64 - lz))) : H;   // the 64 leading bits
    if (L << lz) top |= 1ull;                                 // sticky: bits below them
    return __ull2double_rn(top) * __longlong_as_double(static_cast<long long>(1023 - 10 - lz) << 52);
}

__device__ __forceinline__ void sq_rare_add(uint32_t b16, unsigned long long *s_bins) {
    const uint32_t E = (b16 >> 7) & 0xffu, m7 = b16 & 0x7fu;
    const uint32_t M = E ? (m7 | 0x80u) : m7;
    const int te = E ? 2 * static_cast<int>(E) - 268 : -266;
    const int sh = te - kSqTe0;
    if (M != 0u && !(E != 0u && sh >= 0 && sh < 80))
        atomicAdd(&s_bins[te - kSqTeMin], static_cast<unsigned long long>(M * M));
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// the eight bf16 of a chunk as fp32, in order
__device__ __forceinline__ void chunk_f32(const uint4 &u, float *f) {
    f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x); f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
    f[4] = bf16_lo(u.z); f[5] = bf16_hi(u.z); f[6] = bf16_lo(u.w); f[7] = bf16_hi(u.w);
}


__device__ __forceinline__ uint2 codes8(const float *v, float s) {
    uint2 q;
    q.x = bq_code(v[0], s) | (bq_code(v[1], s) << 8) | (bq_code(v[2], s) << 16) | (bq_code(v[3], s) << 24);
    q.y = bq_code(v[4], s) | (bq_code(v[5], s) << 8) | (bq_code(v[6], s) << 16) | (bq_code(v[7], s) << 24);
    return q;
}

// block max for CTAs of up to 8 warps (s_red: 8 floats); one call per kernel
__device__ __forceinline__ float rc_block_max(float v, float *s_red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    if (lane == 0) s_red[warp] = v;
    __syncthreads();
    float r = lane < nw ? s_red[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) r = fmaxf(r, __shfl_xor_sync(0xffffffffu, r, o));
    return r;   // every warp reduces the same values: no second barrier needed
}

template <int CPT>
__global__ void __launch_bounds__(256) k_rmsnorm_quant_rc(const uint4 *__restrict__ X, const float4 *__restrict__ w,
                                                         int K, float eps_n, float eps_a,
                                                         int8_t *__restrict__ Xq, float *__restrict__ amax,
                                                         float *__restrict__ rinv) {
    __shared__ unsigned long long s_bins[kSqBins];
    __shared__ unsigned long long s_lo[8], s_hi[8];
    __shared__ uint32_t s_limb[kSqLimbs];
    __shared__ float s_red[8];
    __shared__ float s_r;
    const int64_t t = blockIdx.x;
    const int nchunk = K >> 3;
    const uint4 *row = X + t * nchunk;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    uint4 v[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        const int c = threadIdx.x + j * blockDim.x;
        v[j] = c < nchunk ? __ldg(row + c) : make_uint4(0u, 0u, 0u, 0u);
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    uint64_t lo = 0, hi = 0;
    bool rare = false;
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        if (!sq_chunk_f64(v[j], lo, hi)) {   // a wide or out-of-window chunk: value by value
            const uint32_t wv[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                rare |= sq_window(wv[e] & 0xffffu, lo, hi);
                rare |= sq_window(wv[e] >> 16, lo, hi);
            }
        }
    }
    const bool any_rare = __syncthreads_or(rare) != 0;
    if (any_rare) {   // squares outside the window go to per-exponent bins (a second scan of the registers)
        for (int i = threadIdx.x; i < kSqBins; i += blockDim.x) s_bins[i] = 0ull;
        __syncthreads();
        if (rare) {
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                const uint32_t wv[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    sq_rare_add(wv[e] & 0xffffu, s_bins);
                    sq_rare_add(wv[e] >> 16, s_bins);
                }
            }
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
    if (warp == 0) {   // one warp forms the total and r (its lanes in step), the others wait at the barrier
        uint64_t L = 0, H = 0;
        for (int i = 0; i < nw; ++i) add128_sq(L, H, s_lo[i], s_hi[i]);
        double S;
        if (!any_rare) S = window_to_f64(L, H);
        else S = lane == 0 ? sq_finalize(L, H, s_bins, true, s_limb) : 0.0;
        if (lane == 0) {
            const float ms = __double2float_rn(__ddiv_rn(S, static_cast<double>(K)));
            const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps_n)));
            s_r = r;
            if (rinv) rinv[t] = r;
        }
    }
    __syncthreads();
    const float r = s_r;
    float xn[CPT][8];
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        const int c = threadIdx.x + j * blockDim.x;
        chunk_f32(v[j], xn[j]);   // chunks past the row are zero
        if (w) {
            float4 w0 = make_float4(0.f, 0.f, 0.f, 0.f), w1 = w0;
            if (c < nchunk) {
                w0 = __ldg(w + 2 * c);
                w1 = __ldg(w + 2 * c + 1);
            }
            const float wf[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) xn[j][e] = __fmul_rn(__fmul_rn(xn[j][e], r), wf[e]);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) xn[j][e] = __fmul_rn(xn[j][e], r);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(xn[j][e]));
    }
    m = rc_block_max(m, s_red);
    const float a = m > eps_a ? m : eps_a;
    const float s = __fdiv_rn(127.0f, a);
    if (threadIdx.x == 0) amax[t] = a;
    uint2 *out = reinterpret_cast<uint2 *>(Xq + t * K);
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        const int c = threadIdx.x + j * blockDim.x;
        if (c < nchunk) out[c] = codes8_fast(xn[j], s);
    }
}

// silu(g) * u of the definition above
__device__ __forceinline__ float swiglu1(float g, float u) {
    return __fmul_rn(__fdiv_rn(g, __fadd_rn(1.0f, exp32(-g))), u);
}

// exp32 of two values at once with the paired fp32 add and multiply of
// sm_100, which round each component exactly as the scalar __fadd_rn and
// __fmul_rn do: the same operations in the same order, so the results equal
// exp32's bit for bit.  A subtraction a - b is the addition a + fp32(n (-c))
// with the constant negated, which rounds to the same value.
__device__ __forceinline__ float2 exp32x2(float2 x) {
    x.x = fminf(fmaxf(x.x, -87.0f), 88.0f);
    x.y = fminf(fmaxf(x.y, -87.0f), 88.0f);
    const float l2e = __uint_as_float(0x3fb8aa3bu), hi = __uint_as_float(0xbf317200u), lo = __uint_as_float(0xb5bfbe8eu);
    const float2 big = __fadd2_rn(__fmul2_rn(x, make_float2(l2e, l2e)), make_float2(12582912.0f, 12582912.0f));
    const float2 n = __fadd2_rn(big, make_float2(-12582912.0f, -12582912.0f));
    const int n0 = __float_as_int(big.x) - 0x4b400000, n1 = __float_as_int(big.y) - 0x4b400000;
    float2 r = __fadd2_rn(x, __fmul2_rn(n, make_float2(hi, hi)));
    r = __fadd2_rn(r, __fmul2_rn(n, make_float2(lo, lo)));
    const float c5 = __uint_as_float(0x3ab60b61u), c4 = __uint_as_float(0x3c088889u), c3 = __uint_as_float(0x3d2aaaabu),
                c2 = __uint_as_float(0x3e2aaaabu);
    float2 p = make_float2(c5, c5);
    p = __fadd2_rn(__fmul2_rn(p, r), make_float2(c4, c4));
    p = __fadd2_rn(__fmul2_rn(p, r), make_float2(c3, c3));
    p = __fadd2_rn(__fmul2_rn(p, r), make_float2(c2, c2));
    p = __fadd2_rn(__fmul2_rn(p, r), make_float2(0.5f, 0.5f));
    p = __fadd2_rn(__fmul2_rn(p, r), make_float2(1.0f, 1.0f));
    p = __fadd2_rn(__fmul2_rn(p, r), make_float2(1.0f, 1.0f));
    return __fmul2_rn(p, make_float2(__int_as_float((n0 + 127) << 23), __int_as_float((n1 + 127) << 23)));
}

// swiglu1 of two (g, u) pairs; the divisions stay scalar IEEE divisions
__device__ __forceinline__ float2 swiglu2(float2 g, float2 u) {
    const float2 d = __fadd2_rn(make_float2(1.0f, 1.0f), exp32x2(make_float2(-g.x, -g.y)));
    return __fmul2_rn(make_float2(__fdiv_rn(g.x, d.x), __fdiv_rn(g.y, d.y)), u);
}

// h goes to shared memory (F fp32) between the absmax and the codes; the raw
// gate and up chunks stay in registers only until h is formed.
template <int CPT>
__global__ void __launch_bounds__(256) k_swiglu_quant_rc(const uint4 *__restrict__ G, const uint4 *__restrict__ U,
                                                        int64_t ld8, int F, float eps_a,
                                                        int8_t *__restrict__ Xq, float *__restrict__ amax) {
    extern __shared__ float4 s_h4[];
    __shared__ float s_red[8];
    const int64_t t = blockIdx.x;
    const int nchunk = F >> 3;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    uint4 gv[CPT], uv[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        const int c = threadIdx.x + j * blockDim.x;
        const bool in = c < nchunk;
        gv[j] = in ? __ldg(G + t * ld8 + c) : make_uint4(0u, 0u, 0u, 0u);
        uv[j] = in ? __ldg(U + t * ld8 + c) : make_uint4(0u, 0u, 0u, 0u);
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        const int c = threadIdx.x + j * blockDim.x;
        if (c < nchunk) {
            float g[8], u[8], h[8];
            chunk_f32(gv[j], g);
            chunk_f32(uv[j], u);
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
                const float2 hp = swiglu2(make_float2(g[e], g[e + 1]), make_float2(u[e], u[e + 1]));
                h[e] = hp.x;
                h[e + 1] = hp.y;
                m = fmaxf(m, fmaxf(fabsf(hp.x), fabsf(hp.y)));
            }
            s_h4[2 * c] = make_float4(h[0], h[1], h[2], h[3]);
            s_h4[2 * c + 1] = make_float4(h[4], h[5], h[6], h[7]);
        }
    }
    m = rc_block_max(m, s_red);   // its barrier also orders the s_h4 writes before the reads below
    const float a = m > eps_a ? m : eps_a;
    const float s = __fdiv_rn(127.0f, a);
    if (threadIdx.x == 0) amax[t] = a;
    uint2 *out = reinterpret_cast<uint2 *>(Xq + t * F);
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        const int c = threadIdx.x + j * blockDim.x;
        if (c < nchunk) {
            const float4 h0 = s_h4[2 * c], h1 = s_h4[2 * c + 1];
            const float h[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
            out[c] = codes8_fast(h, s);
        }
    }
}

static cudaLaunchConfig_t bq_config(int64_t T, int threads, size_t smem, cudaStream_t s, cudaLaunchAttribute *attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(T));
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

// chunks per thread for a row of nchunk 16-byte chunks: the smallest listed
// CPT that covers the row with at most max_threads threads (fewer threads per
// token: less per-token reduction work, more tokens resident per SM); threads =
// chunks / CPT rounded up to a warp.  Returns 0 when the row is longer than
// the largest listed CPT covers with max_threads.
static int pick_cpt(int64_t nchunk, const int *list, int n, int max_threads, int *threads) {
    for (int i = 0; i < n; ++i)
        if (nchunk <= static_cast<int64_t>(max_threads) * list[i]) {
            const int64_t th = (nchunk + list[i] - 1) / list[i];
            *threads = static_cast<int>((th + 31) / 32 * 32);
            return list[i];
        }
    return 0;
}

constexpr int kRmsCpt[] = {1, 2, 3, 4, 6, 8};   // larger CPT spills registers
constexpr int kSwiCpt[] = {1, 2, 3, 4, 6, 8};

template <int CPT>
static cudaError_t rms_rc(cudaLaunchConfig_t &cfg, const void *X, const float *w, int64_t K, float eps_n, float eps_a,
                          int8_t *Xq, float *amax, float *rinv) {
    return cudaLaunchKernelEx(&cfg, k_rmsnorm_quant_rc<CPT>, static_cast<const uint4 *>(X),
                              reinterpret_cast<const float4 *>(w), static_cast<int>(K), eps_n, eps_a, Xq, amax, rinv);
}

cudaError_t launch_rmsnorm_quant(const void *X, const float *w, int64_t T, int64_t K, float eps_n, float eps_a,
                                 int8_t *Xq, float *amax, float *rinv, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    cudaLaunchAttribute attr[1];
    int threads = 0;
    int cpt = 0;
    if (!(reinterpret_cast<uintptr_t>(w) & 15u)) {
        cpt = pick_cpt(K / 8, kRmsCpt, 6, 128, &threads);
        if (cpt == 0) cpt = pick_cpt(K / 8, kRmsCpt, 6, 256, &threads);
    }
    if (cpt == 0) {   // rows beyond the register cache, or a weight vector without 16-byte alignment
        cudaLaunchConfig_t cfg = bq_config(T, kBqThreads, 0, s, attr);
        return cudaLaunchKernelEx(&cfg, k_rmsnorm_quant, static_cast<const uint16_t *>(X), w, K, eps_n, eps_a, Xq,
                                  amax, rinv);
    }
    cudaLaunchConfig_t cfg = bq_config(T, threads, 0, s, attr);
    switch (cpt) {
        case 1: return rms_rc<1>(cfg, X, w, K, eps_n, eps_a, Xq, amax, rinv);
        case 2: return rms_rc<2>(cfg, X, w, K, eps_n, eps_a, Xq, amax, rinv);
        case 3: return rms_rc<3>(cfg, X, w, K, eps_n, eps_a, Xq, amax, rinv);
        case 4: return rms_rc<4>(cfg, X, w, K, eps_n, eps_a, Xq, amax, rinv);
        case 6: return rms_rc<6>(cfg, X, w, K, eps_n, eps_a, Xq, amax, rinv);
        default: return rms_rc<8>(cfg, X, w, K, eps_n, eps_a, Xq, amax, rinv);
    }
}

size_t swiglu_smem_bytes(int64_t F) { return static_cast<size_t>(F) * 4; }

template <int CPT>
static cudaError_t swi_rc(cudaLaunchConfig_t &cfg, const void *G, const void *U, int64_t ld, int64_t F, float eps_a,
                          int8_t *Xq, float *amax) {
    {
        cudaError_t e = smem_attr(reinterpret_cast<const void *>(k_swiglu_quant_rc<CPT>), static_cast<int>(kSwigluMaxSmem));
        if (e != cudaSuccess) return e;
    }
    return cudaLaunchKernelEx(&cfg, k_swiglu_quant_rc<CPT>, static_cast<const uint4 *>(G), static_cast<const uint4 *>(U),
                              ld / 8, static_cast<int>(F), eps_a, Xq, amax);
}

cudaError_t launch_swiglu_quant(const void *G, const void *U, int64_t ld, int64_t T, int64_t F, float eps_a,
                                int8_t *Xq, float *amax, cudaStream_t s) {
    if (T <= 0) return cudaSuccess;
    cudaLaunchAttribute attr[1];
    int threads = 0;
    const bool vec = !(reinterpret_cast<uintptr_t>(G) & 15u) && !(reinterpret_cast<uintptr_t>(U) & 15u) && ld % 8 == 0;
    const int cpt = vec ? pick_cpt(F / 8, kSwiCpt, 6, 256, &threads) : 0;
    if (cpt == 0) {   // rows beyond the register cache, or rows without 16-byte alignment
        {
            cudaError_t e = smem_attr(reinterpret_cast<const void *>(k_swiglu_quant), static_cast<int>(kSwigluMaxSmem));
            if (e != cudaSuccess) return e;
        }
        cudaLaunchConfig_t cfg = bq_config(T, kBqThreads, swiglu_smem_bytes(F), s, attr);
        return cudaLaunchKernelEx(&cfg, k_swiglu_quant, static_cast<const uint16_t *>(G),
                                  static_cast<const uint16_t *>(U), ld, F, eps_a, Xq, amax);
    }
    cudaLaunchConfig_t cfg = bq_config(T, threads, swiglu_smem_bytes(F), s, attr);
    switch (cpt) {
        case 1: return swi_rc<1>(cfg, G, U, ld, F, eps_a, Xq, amax);
        case 2: return swi_rc<2>(cfg, G, U, ld, F, eps_a, Xq, amax);
        case 3: return swi_rc<3>(cfg, G, U, ld, F, eps_a, Xq, amax);
        case 4: return swi_rc<4>(cfg, G, U, ld, F, eps_a, Xq, amax);
        case 6: return swi_rc<6>(cfg, G, U, ld, F, eps_a, Xq, amax);
        default: return swi_rc<8>(cfg, G, U, ld, F, eps_a, Xq, amax);
    }
}

}  // namespace bitnet
