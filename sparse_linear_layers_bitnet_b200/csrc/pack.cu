// Per-step mask + ternarise + pack of fp32 master weights (sm_100a).
//
// "Sparse-BitNet" (gist.science technical summary), section 2
// "Kerncomponenten": the N:M mask keeps the N largest master magnitudes of
// every M consecutive weights along k and is taken before quantisation; the
// forward pass quantises to ternary and then masks.  "Training Strategie": the
// mask is recomputed every step, which is why this kernel runs every step.
// "BitNet b1.58: Ternary Weights for 1.58-bit LLMs", section "The mechanism":
// gamma is the mean absolute value of the whole matrix; W/gamma is rounded and
// clipped to {-1, 0, 1}.
//
// Pass 1 (k_abs_sum) sums |W| exactly: every fp32 magnitude is an integer
// multiple of 2^-149, so the sum is an integer.  Magnitudes with biased
// exponent in [96, 128) (|w| in [2^-31, 2), which holds all weights of a
// trained or Gaussian-initialised layer) go to a per-thread 128-bit fixed-point
// accumulator; any other magnitude goes to per-exponent integer bins in shared
// memory.  Both are combined with integer atomics, so the result does not
// depend on the order of the additions.
// The finaliser turns the integer into the nearest fp64, forms gamma, and
// finds the smallest fp32 t with fp32(t / gamma) > 0.5: by monotonicity of
// correctly rounded division, a kept weight has a non-zero code exactly when
// |w| >= t, so pass 2 needs no division.
// Pass 2 (k_pack24) reads each group of 4 weights once (one float4 per
// thread, coalesced), ranks the magnitudes (ties to the lower position) and
// writes every requested layout.
#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "kernels.h"

namespace bitnet {

__device__ __forceinline__ void add128(uint64_t &lo, uint64_t &hi, uint64_t v) {
    const uint64_t s = lo + v;
    hi += (s < lo) ? 1ull : 0ull;
    lo = s;
}

__device__ __forceinline__ void accumulate_abs(uint32_t bits, uint64_t &lo, uint64_t &hi,
                                               unsigned long long *s_bins, int *s_rare) {
    const uint32_t a = bits & 0x7fffffffu;
    const uint32_t e = a >> 23;
    if (e - 96u < 32u) {
        const uint64_t m = static_cast<uint64_t>((a & 0x7fffffu) | 0x800000u);
        add128(lo, hi, m << (e - 96u));
    } else if (a != 0u) {
        const uint32_t m = (a & 0x7fffffu) | (e ? 0x800000u : 0u);
        atomicAdd(&s_bins[e], static_cast<unsigned long long>(m));
        *s_rare = 1;
    }
}

// ---------------------------------------------------------------- finaliser

// value += v * 2^shift on a little-endian array of 32-bit limbs (shared memory).
__device__ void limbs_add(uint32_t *limb, int nlimb, uint64_t v, int shift) {
    int q = shift >> 5, r = shift & 31;
    // v * 2^r spans at most three limbs
    const uint64_t lo = v << r;
    const uint64_t hi = r ? (v >> (64 - r)) : 0ull;
    uint64_t add[3] = {lo & 0xffffffffull, lo >> 32, hi};
    uint64_t carry = 0;
    for (int j = q; j < nlimb; ++j) {
        const uint64_t a = (j - q < 3) ? add[j - q] : 0ull;
        if (j - q >= 3 && carry == 0) break;
        const uint64_t s2 = static_cast<uint64_t>(limb[j]) + a + carry;
        limb[j] = static_cast<uint32_t>(s2);
        carry = s2 >> 32;
    }
}

constexpr int kLimbs = 12;   // 384 bits

// Turns the exact integer sum (window + bins, in units of 2^-149) into gamma
// and the code threshold.  Called by one thread; bins and limbs in shared memory.
__device__ void finalize_gamma(const unsigned long long *s_bins, const int *s_nz, int n_nz, uint64_t wlo,
                               uint64_t whi, int64_t n, float eps, uint32_t *limb, float *gamma, uint32_t *thr_out) {
    for (int j = 0; j < kLimbs; ++j) limb[j] = 0;
    // a magnitude with biased exponent e and significand m is m * 2^(max(e,1)-1)
    // units; window entries were pre-shifted by (e - 96), so they carry 2^95
    for (int i = 0; i < n_nz; ++i) {
        const int e = s_nz[i];
        limbs_add(limb, kLimbs, s_bins[e], (e == 0 ? 1 : e) - 1);
    }
    limbs_add(limb, kLimbs, wlo, 95);
    limbs_add(limb, kLimbs, whi, 95 + 64);
    // nearest fp64: the top 64 bits with everything below folded into a sticky
    // bit 0, then the correctly rounded u64 -> f64 conversion
    int L = -1;
    for (int j = kLimbs - 1; j >= 0; --j)
        if (limb[j]) {
            L = j;
            break;
        }
    double S = 0.0;
    if (L >= 0) {
        if (L <= 1) {
            const uint64_t v = (static_cast<uint64_t>(L == 1 ? limb[1] : 0u) << 32) | limb[0];
            S = __ull2double_rn(v) * 0x1p-149;   // power-of-two scaling, exact in the normal range
        } else {
            const unsigned __int128 top3 = (static_cast<unsigned __int128>(limb[L]) << 64) |
                                           (static_cast<unsigned __int128>(limb[L - 1]) << 32) | limb[L - 2];
            const int shift = 32 - __clz(limb[L]);          // keeps the top 64 bits of the 96
            uint64_t w64 = static_cast<uint64_t>(top3 >> shift);
            bool sticky = (top3 & ((static_cast<unsigned __int128>(1) << shift) - 1)) != 0;
            for (int j = 0; j < L - 2 && !sticky; ++j) sticky = limb[j] != 0u;
            if (sticky) w64 |= 1ull;   // bit 0 lies below the 53-bit rounding position
            const int ex = 32 * (L - 2) + shift - 149;       // weight of bit 0 of w64
            S = __ull2double_rn(w64) * __longlong_as_double(static_cast<long long>(1023 + ex) << 52);
        }
    }
    const double mean = __ddiv_rn(S, static_cast<double>(n));
    float g = __double2float_rn(mean);
    g = __fadd_rn(g, eps);
    *gamma = g;
    // smallest t >= 0 with fp32(t / g) > 0.5
    uint32_t t = __float_as_uint(__fmul_rn(g, 0.5f));
    int it = 0;
    if (__fdiv_rn(__uint_as_float(t), g) > 0.5f) {
        while (t > 0u && __fdiv_rn(__uint_as_float(t - 1u), g) > 0.5f && it < 64) {
            --t;
            ++it;
        }
    } else {
        while (!(__fdiv_rn(__uint_as_float(t), g) > 0.5f) && it < 64) {
            ++t;
            ++it;
        }
    }
    *thr_out = t;
}

__global__ void __launch_bounds__(256, 4) k_abs_sum(const float4 *__restrict__ W, int64_t n4,
                                                 unsigned long long *__restrict__ win,
                                                 unsigned long long *__restrict__ bins,
                                                 unsigned *__restrict__ counter, int64_t n_total, float eps,
                                                 float *__restrict__ gamma, uint32_t *__restrict__ thr) {
    __shared__ unsigned long long s_bins[256];
    __shared__ unsigned long long s_lo[8], s_hi[8];
    __shared__ int s_rare;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) s_bins[i] = 0ull;
    if (threadIdx.x == 0) s_rare = 0;
    __syncthreads();

    uint64_t lo = 0, hi = 0;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    // four independent 16-byte loads in flight per thread
    for (; i + 3 * stride < n4; i += 4 * stride) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = __ldg(W + i + u * stride);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            accumulate_abs(__float_as_uint(v[u].x), lo, hi, s_bins, &s_rare);
            accumulate_abs(__float_as_uint(v[u].y), lo, hi, s_bins, &s_rare);
            accumulate_abs(__float_as_uint(v[u].z), lo, hi, s_bins, &s_rare);
            accumulate_abs(__float_as_uint(v[u].w), lo, hi, s_bins, &s_rare);
        }
    }
    for (; i < n4; i += stride) {
        const float4 v = __ldg(W + i);
        accumulate_abs(__float_as_uint(v.x), lo, hi, s_bins, &s_rare);
        accumulate_abs(__float_as_uint(v.y), lo, hi, s_bins, &s_rare);
        accumulate_abs(__float_as_uint(v.z), lo, hi, s_bins, &s_rare);
        accumulate_abs(__float_as_uint(v.w), lo, hi, s_bins, &s_rare);
    }
    // 128-bit warp reduction
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t l2 = __shfl_xor_sync(0xffffffffu, lo, o);
        const uint64_t h2 = __shfl_xor_sync(0xffffffffu, hi, o);
        const uint64_t s = lo + l2;
        hi = hi + h2 + ((s < lo) ? 1ull : 0ull);
        lo = s;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        s_lo[warp] = lo;
        s_hi[warp] = hi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint64_t L = 0, H = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
            const uint64_t s = L + s_lo[w];
            H = H + s_hi[w] + ((s < L) ? 1ull : 0ull);
            L = s;
        }
        if (L | H) {
            const unsigned long long old = atomicAdd(&win[0], static_cast<unsigned long long>(L));
            const uint64_t carry = (static_cast<uint64_t>(old) + L < static_cast<uint64_t>(old)) ? 1ull : 0ull;
            atomicAdd(&win[1], static_cast<unsigned long long>(H + carry));
        }
    }
    if (s_rare) {
        for (int e = threadIdx.x; e < 256; e += blockDim.x)
            if (s_bins[e]) atomicAdd(&bins[e], s_bins[e]);
    }
    // the last block to finish turns the sums into gamma and the threshold
    __shared__ unsigned s_ticket;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_ticket = atomicAdd(counter, 1u);
    __syncthreads();
    if (s_ticket != gridDim.x - 1) return;
    __threadfence();
    __shared__ int s_nz[256];
    __shared__ int s_nnz;
    __shared__ uint32_t s_limb[kLimbs];
    if (threadIdx.x == 0) s_nnz = 0;
    __syncthreads();
    for (int e = threadIdx.x; e < 256; e += blockDim.x) {
        const unsigned long long b = atomicAdd(&bins[e], 0ull);   // coherent read of the final sums
        s_bins[e] = b;
        if (b) s_nz[atomicAdd(&s_nnz, 1)] = e;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // ascending exponent order is not needed (integer sums commute), but keep it deterministic
        for (int i = 1; i < s_nnz; ++i)
            for (int j = i; j > 0 && s_nz[j - 1] > s_nz[j]; --j) {
                const int tmp = s_nz[j];
                s_nz[j] = s_nz[j - 1];
                s_nz[j - 1] = tmp;
            }
        const uint64_t wlo = atomicAdd(&win[0], 0ull), whi = atomicAdd(&win[1], 0ull);
        finalize_gamma(s_bins, s_nz, s_nnz, wlo, whi, n_total, eps, s_limb, gamma, thr);
    }
}

// ---------------------------------------------------------------- pass 2 (2:4)

// Division of 32-bit indices by an invariant divisor with one multiply-high
// (Granlund and Montgomery, "Division by Invariant Integers using
// Multiplication", PLDI 1994, section 4: m = floor(2^32 (2^l - d) / d) + 1,
// q = (t + ((n - t) >> 1)) >> (l - 1) with t = umulhi(m, n), l = ceil(log2 d)).
struct FastDiv32 {
    uint32_t d, m, s1, s2;
};

static FastDiv32 make_fastdiv(uint32_t d) {
    FastDiv32 f;
    f.d = d;
    int l = 0;
    while ((1ull << l) < d) ++l;   // l = ceil(log2 d)
    f.m = static_cast<uint32_t>(((1ull << 32) * ((1ull << l) - d)) / d + 1);
    f.s1 = l > 0 ? 1u : 0u;
    f.s2 = l > 0 ? static_cast<uint32_t>(l - 1) : 0u;
    return f;
}

__device__ __forceinline__ uint32_t fastdiv(uint32_t n, const FastDiv32 &f) {
    const uint32_t t = __umulhi(f.m, n);
    return (t + ((n - t) >> f.s1)) >> f.s2;
}

struct Pack24Args {
    const float4 *W;
    int64_t n_groups;    // n_out * k / 4
    int64_t gpr;         // groups per row = k / 4
    FastDiv32 gpr_div;   // division by gpr (group indices < 2^32)
    int64_t n_out;
    int64_t k;
    int64_t meta_rows;   // rows of one metadata k-block = ceil(n_out/128)*128
    const uint32_t *thr;
    uint8_t *gb;         // [n_out, k/4] or null
    uint16_t *vals;      // [n_out, k/2] int8 pairs or null
    uint8_t *meta;       // blocks of 128 rows x 16 bytes or null
    uint8_t *mask;       // [n_out*k/8] or null
};

// Bit q set when position q is among the two largest magnitudes of the group
// (ties to the lower position).  Position p is ranked behind q < p when
// mag[q] >= mag[p], and behind q > p when mag[q] > mag[p]; p is kept when at
// most one position is ranked ahead of it.  Six comparisons.
__device__ __forceinline__ uint32_t top2_of_4(const uint32_t (&mag)[4]) {
    const uint32_t g01 = mag[0] >= mag[1], g02 = mag[0] >= mag[2], g03 = mag[0] >= mag[3];
    const uint32_t g12 = mag[1] >= mag[2], g13 = mag[1] >= mag[3], g23 = mag[2] >= mag[3];
    const uint32_t ahead0 = (1u - g01) + (1u - g02) + (1u - g03);
    const uint32_t ahead1 = g01 + (1u - g12) + (1u - g13);
    const uint32_t ahead2 = g02 + g12 + (1u - g23);
    const uint32_t ahead3 = g03 + g13 + g23;
    return (ahead0 < 2u ? 1u : 0u) | (ahead1 < 2u ? 2u : 0u) | (ahead2 < 2u ? 4u : 0u) | (ahead3 < 2u ? 8u : 0u);
}

// Ranks one group, writes every requested layout with threshold thr, and
// returns whether one of its kept magnitudes lies in [band_lo, band_hi].
__device__ __forceinline__ uint32_t pack_group(const Pack24Args &p, uint32_t thr, int lane, int64_t i, bool valid,
                                               const float4 v, uint32_t band_lo, uint32_t band_hi) {
    uint32_t bits[4] = {__float_as_uint(v.x), __float_as_uint(v.y), __float_as_uint(v.z), __float_as_uint(v.w)};
    uint32_t mag[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) mag[q] = bits[q] & 0x7fffffffu;   // |w| as ordered integers
    const uint32_t keep = top2_of_4(mag);
    const uint32_t i0 = __ffs(keep) - 1;
    const uint32_t i1 = 31 - __clz(keep);
    // register selects instead of a dynamically indexed array (no local memory)
    const uint32_t b0 = i0 == 0 ? bits[0] : (i0 == 1 ? bits[1] : (i0 == 2 ? bits[2] : bits[3]));
    const uint32_t b1 = i1 == 0 ? bits[0] : (i1 == 1 ? bits[1] : (i1 == 2 ? bits[2] : bits[3]));
    const uint32_t nz0 = (b0 & 0x7fffffffu) >= thr, nz1 = (b1 & 0x7fffffffu) >= thr;
    const uint32_t c0 = nz0 ? ((b0 >> 31) ? 3u : 1u) : 0u;
    const uint32_t c1 = nz1 ? ((b1 >> 31) ? 3u : 1u) : 0u;
    const uint32_t nib = i0 | (i1 << 2);
    if (valid && p.gb) p.gb[i] = static_cast<uint8_t>(nib | (c0 << 4) | (c1 << 6));
    if (valid && p.vals) {
        const uint32_t v0 = nz0 ? ((b0 >> 31) ? 0xffu : 0x01u) : 0u;
        const uint32_t v1 = nz1 ? ((b1 >> 31) ? 0xffu : 0x01u) : 0u;
        p.vals[i] = static_cast<uint16_t>(v0 | (v1 << 8));
    }
    // neighbouring groups share a byte in the metadata and the mask
    const uint32_t nib_hi = __shfl_xor_sync(0xffffffffu, nib, 1);
    const uint32_t keep_hi = __shfl_xor_sync(0xffffffffu, keep, 1);
    if (valid && (lane & 1) == 0) {
        const uint32_t row32 = fastdiv(static_cast<uint32_t>(i), p.gpr_div);
        const int64_t row = row32, g = i - row * p.gpr;
        if (p.meta) {
            const int64_t kb = g >> 5;
            const int64_t off = ((kb * p.meta_rows + row) << 4) + ((g & 31) >> 1);
            p.meta[off] = static_cast<uint8_t>(nib | (nib_hi << 4));
        }
        if (p.mask) p.mask[(row * p.k >> 3) + (g >> 1)] = static_cast<uint8_t>(keep | (keep_hi << 4));
    }
    const uint32_t m0 = b0 & 0x7fffffffu, m1 = b1 & 0x7fffffffu;
    return ((m0 >= band_lo && m0 <= band_hi) || (m1 >= band_lo && m1 <= band_hi)) ? 1u : 0u;
}

// Rewrites the threshold-dependent bytes of one group (group byte and values).
__device__ __forceinline__ void patch_group(const Pack24Args &p, uint32_t thr, int64_t i, const float4 v) {
    uint32_t bits[4] = {__float_as_uint(v.x), __float_as_uint(v.y), __float_as_uint(v.z), __float_as_uint(v.w)};
    uint32_t mag[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) mag[q] = bits[q] & 0x7fffffffu;
    const uint32_t keep = top2_of_4(mag);
    const uint32_t i0 = __ffs(keep) - 1, i1 = 31 - __clz(keep);
    const uint32_t b0 = i0 == 0 ? bits[0] : (i0 == 1 ? bits[1] : (i0 == 2 ? bits[2] : bits[3]));
    const uint32_t b1 = i1 == 0 ? bits[0] : (i1 == 1 ? bits[1] : (i1 == 2 ? bits[2] : bits[3]));
    const uint32_t nz0 = (b0 & 0x7fffffffu) >= thr, nz1 = (b1 & 0x7fffffffu) >= thr;
    const uint32_t c0 = nz0 ? ((b0 >> 31) ? 3u : 1u) : 0u;
    const uint32_t c1 = nz1 ? ((b1 >> 31) ? 3u : 1u) : 0u;
    if (p.gb) p.gb[i] = static_cast<uint8_t>(i0 | (i1 << 2) | (c0 << 4) | (c1 << 6));
    if (p.vals) {
        const uint32_t v0 = nz0 ? ((b0 >> 31) ? 0xffu : 0x01u) : 0u;
        const uint32_t v1 = nz1 ? ((b1 >> 31) ? 0xffu : 0x01u) : 0u;
        p.vals[i] = static_cast<uint16_t>(v0 | (v1 << 8));
    }
}

constexpr int kPackUnroll = 4;

__global__ void __launch_bounds__(256) k_pack24(Pack24Args p) {
    const uint32_t thr = *p.thr;
    const int lane = threadIdx.x & 31;
    const int64_t warp_stride = static_cast<int64_t>(gridDim.x) * blockDim.x * kPackUnroll;
    // each warp takes 32 * kPackUnroll consecutive groups per round; all loads of
    // the round are issued before any group is processed.  The iteration is
    // warp-uniform so that every lane takes part in the shuffles.
    for (int64_t base = (static_cast<int64_t>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31)) * kPackUnroll;
         base < p.n_groups; base += warp_stride) {
        float4 v[kPackUnroll];
#pragma unroll
        for (int u = 0; u < kPackUnroll; ++u) {
            const int64_t i = base + 32 * u + lane;
            v[u] = (i < p.n_groups) ? __ldg(p.W + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kPackUnroll; ++u) {
            const int64_t i = base + 32 * u + lane;
            pack_group(p, thr, lane, i, i < p.n_groups, v[u], 0u, 0u);
        }
    }
}

// ---------------------------------------------------------------- single-read update

// Smallest t >= 0 with fp32(t / g) > 0.5 (the code threshold of gamma g).
__device__ uint32_t code_threshold(float g) {
    uint32_t t = __float_as_uint(__fmul_rn(g, 0.5f));
    int it = 0;
    if (__fdiv_rn(__uint_as_float(t), g) > 0.5f) {
        while (t > 0u && __fdiv_rn(__uint_as_float(t - 1u), g) > 0.5f && it < 64) {
            --t;
            ++it;
        }
    } else {
        while (!(__fdiv_rn(__uint_as_float(t), g) > 0.5f) && it < 64) {
            ++t;
            ++it;
        }
    }
    return t;
}

struct UpdateArgs {
    Pack24Args p;              // layouts (p.thr unused here)
    const float *gamma_prev;   // previous gamma of this matrix (the hint), read before it is overwritten
    float *gamma;              // out (same buffer as gamma_prev)
    unsigned long long *win, *bins;
    unsigned *counter;
    uint32_t *thr;             // new threshold (out)
    uint32_t *mode;            // 1: patch the listed groups, 2: full second pass
    uint32_t *band;            // [t_lo, t_hi] of the hint, written by block 0
    uint32_t *list;            // group indices whose kept weights lie in the band
    unsigned *list_count;
    uint32_t list_cap;
    int64_t n_total;
    float eps;
};

// Pass 1 of the update: exact sum of |W| for the new gamma and, when a valid
// hint exists, every layout computed with the hint's threshold; kept weights
// whose magnitude lies within a relative 2^-10 of that threshold are listed.
// The last block forms the new gamma and threshold and chooses: if the new
// threshold lies inside the band (and the list did not overflow), only the
// listed groups can change and are patched; otherwise a full second pass runs.
__global__ void __launch_bounds__(256, 4) k_pack_update(UpdateArgs u) {
    __shared__ unsigned long long s_bins[256];
    __shared__ unsigned long long s_lo[8], s_hi[8];
    __shared__ int s_rare;
    __shared__ uint32_t s_t, s_tlo, s_thi;
    __shared__ int s_hint;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) s_bins[i] = 0ull;
    if (threadIdx.x == 0) {
        s_rare = 0;
        const float gp = *u.gamma_prev;
        s_hint = (gp > 0.0f && gp < 3.0e38f) ? 1 : 0;   // finite and positive
        if (s_hint) {
            s_t = code_threshold(gp);
            const float tf = __uint_as_float(s_t);
            s_tlo = __float_as_uint(__fmul_rd(tf, 1.0f - 0x1p-10f));
            s_thi = __float_as_uint(__fmul_ru(tf, 1.0f + 0x1p-10f));
            if (blockIdx.x == 0) {
                u.band[0] = s_tlo;
                u.band[1] = s_thi;
            }
        }
    }
    __syncthreads();
    const bool hint = s_hint != 0;
    const uint32_t t_old = s_t, t_lo = s_tlo, t_hi = s_thi;
    const Pack24Args &p = u.p;
    const int lane = threadIdx.x & 31;
    uint64_t lo = 0, hi = 0;
    const int64_t warp_stride = static_cast<int64_t>(gridDim.x) * blockDim.x * kPackUnroll;
    for (int64_t base = (static_cast<int64_t>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31)) * kPackUnroll;
         base < p.n_groups; base += warp_stride) {
        float4 v[kPackUnroll];
#pragma unroll
        for (int q = 0; q < kPackUnroll; ++q) {
            const int64_t i = base + 32 * q + lane;
            v[q] = (i < p.n_groups) ? __ldg(p.W + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int q = 0; q < kPackUnroll; ++q) {
            const int64_t i = base + 32 * q + lane;
            accumulate_abs(__float_as_uint(v[q].x), lo, hi, s_bins, &s_rare);
            accumulate_abs(__float_as_uint(v[q].y), lo, hi, s_bins, &s_rare);
            accumulate_abs(__float_as_uint(v[q].z), lo, hi, s_bins, &s_rare);
            accumulate_abs(__float_as_uint(v[q].w), lo, hi, s_bins, &s_rare);
            if (hint) {
                const uint32_t in_band = pack_group(p, t_old, lane, i, i < p.n_groups, v[q], t_lo, t_hi);
                if (in_band && i < p.n_groups) {
                    const unsigned slot = atomicAdd(u.list_count, 1u);
                    if (slot < u.list_cap) u.list[slot] = static_cast<uint32_t>(i);
                }
            }
        }
    }
    // exact-sum reduction, as in k_abs_sum
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t l2 = __shfl_xor_sync(0xffffffffu, lo, o);
        const uint64_t h2 = __shfl_xor_sync(0xffffffffu, hi, o);
        const uint64_t sum = lo + l2;
        hi = hi + h2 + ((sum < lo) ? 1ull : 0ull);
        lo = sum;
    }
    const int warp = threadIdx.x >> 5;
    if (lane == 0) {
        s_lo[warp] = lo;
        s_hi[warp] = hi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint64_t L = 0, H = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
            const uint64_t sum = L + s_lo[w];
            H = H + s_hi[w] + ((sum < L) ? 1ull : 0ull);
            L = sum;
        }
        if (L | H) {
            const unsigned long long old = atomicAdd(&u.win[0], static_cast<unsigned long long>(L));
            const uint64_t carry = (static_cast<uint64_t>(old) + L < static_cast<uint64_t>(old)) ? 1ull : 0ull;
            atomicAdd(&u.win[1], static_cast<unsigned long long>(H + carry));
        }
    }
    if (s_rare) {
        for (int e = threadIdx.x; e < 256; e += blockDim.x)
            if (s_bins[e]) atomicAdd(&u.bins[e], s_bins[e]);
    }
    __shared__ unsigned s_ticket;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_ticket = atomicAdd(u.counter, 1u);
    __syncthreads();
    if (s_ticket != gridDim.x - 1) return;
    __threadfence();
    __shared__ int s_nz[256];
    __shared__ int s_nnz;
    __shared__ uint32_t s_limb[kLimbs];
    if (threadIdx.x == 0) s_nnz = 0;
    __syncthreads();
    for (int e = threadIdx.x; e < 256; e += blockDim.x) {
        const unsigned long long b = atomicAdd(&u.bins[e], 0ull);
        s_bins[e] = b;
        if (b) s_nz[atomicAdd(&s_nnz, 1)] = e;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 1; i < s_nnz; ++i)
            for (int j = i; j > 0 && s_nz[j - 1] > s_nz[j]; --j) {
                const int tmp = s_nz[j];
                s_nz[j] = s_nz[j - 1];
                s_nz[j - 1] = tmp;
            }
        const uint64_t wlo = atomicAdd(&u.win[0], 0ull), whi = atomicAdd(&u.win[1], 0ull);
        finalize_gamma(s_bins, s_nz, s_nnz, wlo, whi, u.n_total, u.eps, s_limb, u.gamma, u.thr);
        const uint32_t t_new = *u.thr;
        const unsigned listed = atomicAdd(u.list_count, 0u);
        const bool patch = hint && t_new >= t_lo && t_new <= t_hi && listed <= u.list_cap;
        *u.mode = patch ? 1u : 2u;
    }
}

// Pass 2 of the update: either the full pass (mode 2) or a patch of the listed
// groups with the new threshold (mode 1; the mask and metadata do not depend on
// the threshold, so only the group bytes and the values are rewritten).
__global__ void __launch_bounds__(256) k_pack_finish(UpdateArgs u) {
    const uint32_t mode = *u.mode;
    const uint32_t thr = *u.thr;
    const Pack24Args &p = u.p;
    if (mode == 2u) {
        const int lane = threadIdx.x & 31;
        const int64_t warp_stride = static_cast<int64_t>(gridDim.x) * blockDim.x * kPackUnroll;
        for (int64_t base = (static_cast<int64_t>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31)) * kPackUnroll;
             base < p.n_groups; base += warp_stride) {
            float4 v[kPackUnroll];
#pragma unroll
            for (int q = 0; q < kPackUnroll; ++q) {
                const int64_t i = base + 32 * q + lane;
                v[q] = (i < p.n_groups) ? __ldg(p.W + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int q = 0; q < kPackUnroll; ++q) {
                const int64_t i = base + 32 * q + lane;
                pack_group(p, thr, lane, i, i < p.n_groups, v[q], 0u, 0u);
            }
        }
        return;
    }
    const unsigned listed = *u.list_count;
    for (unsigned j = blockIdx.x * blockDim.x + threadIdx.x; j < listed; j += gridDim.x * blockDim.x) {
        const int64_t i = u.list[j];
        const float4 v = __ldg(p.W + i);
        patch_group(p, thr, i, v);
    }
}

// ---------------------------------------------------------------- lane-quad kernels (k % 16 == 0)
//
// Leaner inner loop for the HBM-bound pass: each lane takes 4 consecutive
// groups of one row (16 weights), so its group bytes, values, metadata nibbles
// and mask bits leave as one 4-, 8-, 2- and 2-byte store, with no shuffles and
// one row division per 4 groups.  The exact sum of |W| takes an fp64 fast
// path: magnitudes in [2^-20, 2) are integer multiples of 2^-43, and up to
// 2^10 / 2^-43 = 2^53 units (fewer than 512 of them) add exactly in fp64; the
// per-lane fp64 sum is moved into the 128-bit integer accumulator (units of
// 2^-54) once per round.  A group with any other magnitude (a zero included)
// takes the exact path of accumulate_abs.

__device__ __forceinline__ void sum_float4(const float4 v, double &d, uint64_t &lo, uint64_t &hi,
                                           unsigned long long *s_bins, int *s_rare) {
    const uint32_t a0 = __float_as_uint(v.x) & 0x7fffffffu, a1 = __float_as_uint(v.y) & 0x7fffffffu;
    const uint32_t a2 = __float_as_uint(v.z) & 0x7fffffffu, a3 = __float_as_uint(v.w) & 0x7fffffffu;
    // all four magnitudes in [2^-20, 2): the smallest and the largest bit pattern
    // decide it (non-negative floats order like their bits); anything else,
    // zeros included, takes the exact path below
    const uint32_t mn = min(min(a0, a1), min(a2, a3)), mx = max(max(a0, a1), max(a2, a3));
    if (mn >= 0x35800000u && mx < 0x40000000u) {
        d += static_cast<double>(__uint_as_float(a0));
        d += static_cast<double>(__uint_as_float(a1));
        d += static_cast<double>(__uint_as_float(a2));
        d += static_cast<double>(__uint_as_float(a3));
    } else {
        accumulate_abs(a0, lo, hi, s_bins, s_rare);
        accumulate_abs(a1, lo, hi, s_bins, s_rare);
        accumulate_abs(a2, lo, hi, s_bins, s_rare);
        accumulate_abs(a3, lo, hi, s_bins, s_rare);
    }
}

// fp64 partial sum (a multiple of 2^-43 below 2^6) -> 128-bit accumulator
__device__ __forceinline__ void flush_sum(double &d, uint64_t &lo, uint64_t &hi) {
    const uint64_t q = __double2ull_rn(d * 0x1p43);   // exact: an integer below 2^49
    add128(lo, hi, q << 11);
    d = 0.0;
}

struct QuadOut {
    uint32_t gb;      // 4 group bytes
    uint32_t vlo, vhi;   // 8 int8 values
    uint32_t meta;    // 4 nibbles in the low 16 bits
    uint32_t mask;    // 4 keep nibbles in the low 16 bits
    uint32_t band;    // bit j: group j has a kept magnitude in [band_lo, band_hi]
};

// One group of four: the two kept positions by a tournament (pair winners,
// then the final; the runner-up is the final's loser or the champion's pair
// partner; every comparison is >= so that ties go to the lower position, the
// same selection as top2_of_4), then codes against thr, group byte, values,
// metadata nibble and whether a kept magnitude lies in [band_lo, band_lo + band_span].
__device__ __forceinline__ void one_group(const float4 v, uint32_t thr, uint32_t band_lo, uint32_t band_span,
                                          uint32_t &gbyte, uint32_t &vals16, uint32_t &nib, uint32_t &in_band) {
    const uint32_t b0 = __float_as_uint(v.x), b1 = __float_as_uint(v.y), b2 = __float_as_uint(v.z),
                   b3 = __float_as_uint(v.w);
    const uint32_t m0 = b0 & 0x7fffffffu, m1 = b1 & 0x7fffffffu, m2 = b2 & 0x7fffffffu, m3 = b3 & 0x7fffffffu;
    const bool pa = m0 >= m1, pb = m2 >= m3;                       // pair winners: 0 / 2 on ties
    const uint32_t wAm = pa ? m0 : m1, lAm = pa ? m1 : m0, wBm = pb ? m2 : m3, lBm = pb ? m3 : m2;
    const bool fa = wAm >= wBm;                                    // champion from the pair (0, 1)
    const bool k01 = fa && lAm >= wBm;                             // kept {0, 1}
    const bool k23 = !fa && !(wAm >= lBm);                         // kept {2, 3}
    const uint32_t wA = pa ? b0 : b1, wB = pb ? b2 : b3;           // otherwise kept: the two pair winners
    const uint32_t x0 = k01 ? b0 : (k23 ? b2 : wA), x1 = k01 ? b1 : (k23 ? b3 : wB);
    nib = k01 ? 0x4u : (k23 ? 0xeu : ((pa ? 0u : 1u) | ((pb ? 2u : 3u) << 2)));
    const uint32_t y0 = x0 & 0x7fffffffu, y1 = x1 & 0x7fffffffu;
    const uint32_t c0 = y0 >= thr ? ((x0 >> 30) & 2u) | 1u : 0u;   // {0, 1: +1, 3: -1}
    const uint32_t c1 = y1 >= thr ? ((x1 >> 30) & 2u) | 1u : 0u;
    gbyte = nib | (c0 << 4) | (c1 << 6);
    vals16 = ((c0 & 2u) * 0x7eu + c0) | (((c1 & 2u) * 0x7eu + c1) << 8);   // int8 +1 / -1 / 0
    in_band = (y0 - band_lo <= band_span || y1 - band_lo <= band_span) ? 1u : 0u;
}

// band: [band_lo, band_hi]; band_hi < band_lo (no hint) lists nothing
__device__ __forceinline__ QuadOut pack_quad(const float4 (&v)[4], uint32_t thr, uint32_t band_lo, uint32_t band_hi) {
    QuadOut o;
    o.gb = o.vlo = o.vhi = o.meta = o.mask = o.band = 0u;
    const uint32_t span = band_hi - band_lo;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint32_t gbyte, vals16, nib, inb;
        one_group(v[j], thr, band_lo, span, gbyte, vals16, nib, inb);
        o.gb |= gbyte << (8 * j);
        if (j < 2) o.vlo |= vals16 << (16 * j);
        else o.vhi |= vals16 << (16 * (j - 2));
        o.meta |= nib << (4 * j);
        o.band |= inb << j;
    }
    // keep bits of the four groups from their metadata nibbles
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t nb = (o.meta >> (4 * j)) & 0xfu;
        o.mask |= ((1u << (nb & 3u)) | (1u << (nb >> 2))) << (4 * j);
    }
    return o;
}

// quad q (4 consecutive groups starting at group 4q) -> its layouts
__device__ __forceinline__ void store_quad(const Pack24Args &p, uint32_t q, const QuadOut &o) {
    const uint32_t i = 4u * q;
    const uint32_t row = fastdiv(i, p.gpr_div);
    const uint32_t g = i - row * static_cast<uint32_t>(p.gpr);
    if (p.gb) *reinterpret_cast<uint32_t *>(p.gb + i) = o.gb;
    if (p.vals) *reinterpret_cast<uint2 *>(p.vals + i) = make_uint2(o.vlo, o.vhi);
    if (p.meta) {
        const size_t off = ((static_cast<size_t>(g >> 5) * static_cast<size_t>(p.meta_rows) + row) << 4) + ((g & 31u) >> 1);
        *reinterpret_cast<uint16_t *>(p.meta + off) = static_cast<uint16_t>(o.meta);
    }
    if (p.mask)
        *reinterpret_cast<uint16_t *>(p.mask + ((static_cast<size_t>(row) * static_cast<size_t>(p.k)) >> 3) + (g >> 1)) =
            static_cast<uint16_t>(o.mask);
}

constexpr int kQuadUnroll = 2;   // quads per lane per round (8 x 16-byte loads in flight)

// pass 1 of bitnet_pack_nm: exact sum of |W| (fast path), last block finalises
__global__ void __launch_bounds__(256, 4) k_abs_sum_fast(const float4 *__restrict__ W, int64_t n4,
                                                         unsigned long long *__restrict__ win,
                                                         unsigned long long *__restrict__ bins,
                                                         unsigned *__restrict__ counter, int64_t n_total, float eps,
                                                         float *__restrict__ gamma, uint32_t *__restrict__ thr) {
    __shared__ unsigned long long s_bins[256];
    __shared__ unsigned long long s_lo[8], s_hi[8];
    __shared__ int s_rare;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) s_bins[i] = 0ull;
    if (threadIdx.x == 0) s_rare = 0;
    __syncthreads();
    uint64_t lo = 0, hi = 0;
    double d = 0.0;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (; i + 7 * stride < n4; i += 8 * stride) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = __ldg(W + i + u * stride);
#pragma unroll
        for (int u = 0; u < 8; ++u) sum_float4(v[u], d, lo, hi, s_bins, &s_rare);
        flush_sum(d, lo, hi);
    }
    for (; i < n4; i += stride) sum_float4(__ldg(W + i), d, lo, hi, s_bins, &s_rare);
    flush_sum(d, lo, hi);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t l2 = __shfl_xor_sync(0xffffffffu, lo, o);
        const uint64_t h2 = __shfl_xor_sync(0xffffffffu, hi, o);
        const uint64_t sum = lo + l2;
        hi = hi + h2 + ((sum < lo) ? 1ull : 0ull);
        lo = sum;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        s_lo[warp] = lo;
        s_hi[warp] = hi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint64_t L = 0, H = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
            const uint64_t sum = L + s_lo[w];
            H = H + s_hi[w] + ((sum < L) ? 1ull : 0ull);
            L = sum;
        }
        if (L | H) {
            const unsigned long long old = atomicAdd(&win[0], static_cast<unsigned long long>(L));
            const uint64_t carry = (static_cast<uint64_t>(old) + L < static_cast<uint64_t>(old)) ? 1ull : 0ull;
            atomicAdd(&win[1], static_cast<unsigned long long>(H + carry));
        }
    }
    if (s_rare) {
        for (int e = threadIdx.x; e < 256; e += blockDim.x)
            if (s_bins[e]) atomicAdd(&bins[e], s_bins[e]);
    }
    __shared__ unsigned s_ticket;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_ticket = atomicAdd(counter, 1u);
    __syncthreads();
    if (s_ticket != gridDim.x - 1) return;
    __threadfence();
    __shared__ int s_nz[256];
    __shared__ int s_nnz;
    __shared__ uint32_t s_limb[kLimbs];
    if (threadIdx.x == 0) s_nnz = 0;
    __syncthreads();
    for (int e = threadIdx.x; e < 256; e += blockDim.x) {
        const unsigned long long b = atomicAdd(&bins[e], 0ull);
        s_bins[e] = b;
        if (b) s_nz[atomicAdd(&s_nnz, 1)] = e;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int a = 1; a < s_nnz; ++a)
            for (int j = a; j > 0 && s_nz[j - 1] > s_nz[j]; --j) {
                const int tmp = s_nz[j];
                s_nz[j] = s_nz[j - 1];
                s_nz[j - 1] = tmp;
            }
        const uint64_t wlo = atomicAdd(&win[0], 0ull), whi = atomicAdd(&win[1], 0ull);
        finalize_gamma(s_bins, s_nz, s_nnz, wlo, whi, n_total, eps, s_limb, gamma, thr);
    }
}

// ---------------------------------------------------------------- optimiser step emitting the next gamma
//
// "Sparse-BitNet" (gist.science), section 2 "Training Strategie": the
// gradient passes straight through the quantiser and the mask to every fp32
// master, so the optimiser updates all of them each step; the next step's pack
// needs the absmean of the updated masters ("BitNet b1.58 ...", section "The
// mechanism").  The update kernel therefore also sums |W_new| exactly (the
// same accumulators as k_abs_sum_fast) and its last block forms gamma and the
// code threshold: the following pack reads W once and needs no sum.
//
// AdamW, every step one IEEE fp32 operation in this order (no fused
// multiply-add): m = b1 m + (1 - b1) g; v = b2 v + (1 - b2) (g g);
// u = (m / c1) / (sqrt(v / c2) + eps); w = w - lr (u + wd w), with the bias
// corrections c1 = 1 - b1^t and c2 = 1 - b2^t given by the caller.
struct AdamWArgs {
    float4 *W;
    const float4 *G;
    float4 *M, *V;
    int64_t n4;
    float lr, b1, b2, eps, wd, c1, c2;
    unsigned long long *win, *bins;
    unsigned *counter;
    int64_t n_total;
    float eps_gamma;
    float *gamma;
    uint32_t *thr;
};

__device__ __forceinline__ float adamw1(float w, float g, float &m, float &v, const AdamWArgs &a, float omb1,
                                        float omb2) {
    m = __fadd_rn(__fmul_rn(a.b1, m), __fmul_rn(omb1, g));
    v = __fadd_rn(__fmul_rn(a.b2, v), __fmul_rn(omb2, __fmul_rn(g, g)));
    const float u = __fdiv_rn(__fdiv_rn(m, a.c1), __fadd_rn(__fsqrt_rn(__fdiv_rn(v, a.c2)), a.eps));
    return __fsub_rn(w, __fmul_rn(a.lr, __fadd_rn(u, __fmul_rn(a.wd, w))));
}

__global__ void __launch_bounds__(256, 6) k_adamw_gamma(const __grid_constant__ AdamWArgs a) {
    __shared__ unsigned long long s_bins[256];
    __shared__ unsigned long long s_lo[8], s_hi[8];
    __shared__ int s_rare;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) s_bins[i] = 0ull;
    if (threadIdx.x == 0) s_rare = 0;
    __syncthreads();
    const float omb1 = __fsub_rn(1.0f, a.b1), omb2 = __fsub_rn(1.0f, a.b2);
    uint64_t lo = 0, hi = 0;
    double d = 0.0;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    constexpr int kU = 1;   // one float4 group per thread per round, latency hidden by 48 warps per SM (3B block:
                            // 0.65 ms; four groups per thread at 32 warps: 0.77 ms; 64 warps spill registers)
    for (; i < a.n4; i += kU * stride) {
        float4 w[kU], g[kU], m[kU], v[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t j = i + u * stride;
            if (j < a.n4) {
                w[u] = a.W[j];
                g[u] = __ldg(a.G + j);
                m[u] = a.M[j];
                v[u] = a.V[j];
            } else {
                w[u] = g[u] = m[u] = v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t j = i + u * stride;
            if (j < a.n4) {
                float4 wn;
                wn.x = adamw1(w[u].x, g[u].x, m[u].x, v[u].x, a, omb1, omb2);
                wn.y = adamw1(w[u].y, g[u].y, m[u].y, v[u].y, a, omb1, omb2);
                wn.z = adamw1(w[u].z, g[u].z, m[u].z, v[u].z, a, omb1, omb2);
                wn.w = adamw1(w[u].w, g[u].w, m[u].w, v[u].w, a, omb1, omb2);
                a.W[j] = wn;
                a.M[j] = m[u];
                a.V[j] = v[u];
                sum_float4(wn, d, lo, hi, s_bins, &s_rare);
            }
        }
        flush_sum(d, lo, hi);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t l2 = __shfl_xor_sync(0xffffffffu, lo, o);
        const uint64_t h2 = __shfl_xor_sync(0xffffffffu, hi, o);
        const uint64_t sum = lo + l2;
        hi = hi + h2 + ((sum < lo) ? 1ull : 0ull);
        lo = sum;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        s_lo[warp] = lo;
        s_hi[warp] = hi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint64_t L = 0, H = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
            const uint64_t sum = L + s_lo[w];
            H = H + s_hi[w] + ((sum < L) ? 1ull : 0ull);
            L = sum;
        }
        if (L | H) {
            const unsigned long long old = atomicAdd(&a.win[0], static_cast<unsigned long long>(L));
            const uint64_t carry = (static_cast<uint64_t>(old) + L < static_cast<uint64_t>(old)) ? 1ull : 0ull;
            atomicAdd(&a.win[1], static_cast<unsigned long long>(H + carry));
        }
    }
    if (s_rare) {
        for (int e = threadIdx.x; e < 256; e += blockDim.x)
            if (s_bins[e]) atomicAdd(&a.bins[e], s_bins[e]);
    }
    __shared__ unsigned s_ticket;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_ticket = atomicAdd(a.counter, 1u);
    __syncthreads();
    if (s_ticket != gridDim.x - 1) return;
    __threadfence();
    __shared__ int s_nz[256];
    __shared__ int s_nnz;
    __shared__ uint32_t s_limb[kLimbs];
    if (threadIdx.x == 0) s_nnz = 0;
    __syncthreads();
    for (int e = threadIdx.x; e < 256; e += blockDim.x) {
        const unsigned long long b = atomicAdd(&a.bins[e], 0ull);
        s_bins[e] = b;
        if (b) s_nz[atomicAdd(&s_nnz, 1)] = e;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int q = 1; q < s_nnz; ++q)
            for (int j = q; j > 0 && s_nz[j - 1] > s_nz[j]; --j) {
                const int tmp = s_nz[j];
                s_nz[j] = s_nz[j - 1];
                s_nz[j - 1] = tmp;
            }
        const uint64_t wlo = atomicAdd(&a.win[0], 0ull), whi = atomicAdd(&a.win[1], 0ull);
        finalize_gamma(s_bins, s_nz, s_nnz, wlo, whi, a.n_total, a.eps_gamma, s_limb, a.gamma, a.thr);
    }
}

// pass 2 of bitnet_pack_nm (and the full pass of the update): lane quads
__device__ __forceinline__ void quad_pass(const Pack24Args &p, uint32_t thr) {
    const uint32_t n_quads = static_cast<uint32_t>(p.n_groups >> 2);
    const uint32_t lane = threadIdx.x & 31;
    const uint32_t warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t warps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t base = warp_global * 32u * kQuadUnroll; base < n_quads; base += warps * 32u * kQuadUnroll) {
        float4 v[kQuadUnroll][4];
#pragma unroll
        for (int u = 0; u < kQuadUnroll; ++u) {
            const uint32_t q = base + 32u * u + lane;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                v[u][j] = q < n_quads ? __ldg(p.W + 4u * q + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kQuadUnroll; ++u) {
            const uint32_t q = base + 32u * u + lane;
            if (q < n_quads) store_quad(p, q, pack_quad(v[u], thr, 0u, 0u));
        }
    }
}

__global__ void __launch_bounds__(256) k_pack24_quad(Pack24Args p) { quad_pass(p, *p.thr); }

// single-read update, lane quads: sum + layouts with the hint's threshold + band list
__global__ void __launch_bounds__(256, 4) k_pack_update_quad(UpdateArgs u) {
    __shared__ unsigned long long s_bins[256];
    __shared__ unsigned long long s_lo[8], s_hi[8];
    __shared__ int s_rare;
    __shared__ uint32_t s_t, s_tlo, s_thi;
    __shared__ int s_hint;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) s_bins[i] = 0ull;
    if (threadIdx.x == 0) {
        s_rare = 0;
        const float gp = *u.gamma_prev;
        s_hint = (gp > 0.0f && gp < 3.0e38f) ? 1 : 0;
        s_t = s_tlo = s_thi = 0u;
        if (s_hint) {
            s_t = code_threshold(gp);
            const float tf = __uint_as_float(s_t);
            s_tlo = __float_as_uint(__fmul_rd(tf, 1.0f - 0x1p-10f));
            s_thi = __float_as_uint(__fmul_ru(tf, 1.0f + 0x1p-10f));
            if (blockIdx.x == 0) {
                u.band[0] = s_tlo;
                u.band[1] = s_thi;
            }
        }
    }
    __syncthreads();
    const bool hint = s_hint != 0;
    const uint32_t t_old = s_t, t_lo = s_tlo, t_hi = s_thi;
    const Pack24Args &p = u.p;
    const uint32_t n_quads = static_cast<uint32_t>(p.n_groups >> 2);
    const uint32_t lane = threadIdx.x & 31;
    const uint32_t warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t warps = (gridDim.x * blockDim.x) >> 5;
    uint64_t lo = 0, hi = 0;
    double d = 0.0;
    for (uint32_t base = warp_global * 32u * kQuadUnroll; base < n_quads; base += warps * 32u * kQuadUnroll) {
        float4 v[kQuadUnroll][4];
#pragma unroll
        for (int k2 = 0; k2 < kQuadUnroll; ++k2) {
            const uint32_t q = base + 32u * k2 + lane;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                v[k2][j] = q < n_quads ? __ldg(p.W + 4u * q + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int k2 = 0; k2 < kQuadUnroll; ++k2) {
            const uint32_t q = base + 32u * k2 + lane;
#pragma unroll
            for (int j = 0; j < 4; ++j) sum_float4(v[k2][j], d, lo, hi, s_bins, &s_rare);
            if (hint && q < n_quads) {
                const QuadOut o = pack_quad(v[k2], t_old, t_lo, t_hi);
                store_quad(p, q, o);
                if (o.band) {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if ((o.band >> j) & 1u) {
                            const unsigned slot = atomicAdd(u.list_count, 1u);
                            if (slot < u.list_cap) u.list[slot] = 4u * q + j;
                        }
                }
            }
        }
        flush_sum(d, lo, hi);
    }
    flush_sum(d, lo, hi);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint64_t l2 = __shfl_xor_sync(0xffffffffu, lo, o);
        const uint64_t h2 = __shfl_xor_sync(0xffffffffu, hi, o);
        const uint64_t sum = lo + l2;
        hi = hi + h2 + ((sum < lo) ? 1ull : 0ull);
        lo = sum;
    }
    const int warp = threadIdx.x >> 5;
    if (lane == 0) {
        s_lo[warp] = lo;
        s_hi[warp] = hi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        uint64_t L = 0, H = 0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
            const uint64_t sum = L + s_lo[w];
            H = H + s_hi[w] + ((sum < L) ? 1ull : 0ull);
            L = sum;
        }
        if (L | H) {
            const unsigned long long old = atomicAdd(&u.win[0], static_cast<unsigned long long>(L));
            const uint64_t carry = (static_cast<uint64_t>(old) + L < static_cast<uint64_t>(old)) ? 1ull : 0ull;
            atomicAdd(&u.win[1], static_cast<unsigned long long>(H + carry));
        }
    }
    if (s_rare) {
        for (int e = threadIdx.x; e < 256; e += blockDim.x)
            if (s_bins[e]) atomicAdd(&u.bins[e], s_bins[e]);
    }
    __shared__ unsigned s_ticket;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_ticket = atomicAdd(u.counter, 1u);
    __syncthreads();
    if (s_ticket != gridDim.x - 1) return;
    __threadfence();
    __shared__ int s_nz[256];
    __shared__ int s_nnz;
    __shared__ uint32_t s_limb[kLimbs];
    if (threadIdx.x == 0) s_nnz = 0;
    __syncthreads();
    for (int e = threadIdx.x; e < 256; e += blockDim.x) {
        const unsigned long long b = atomicAdd(&u.bins[e], 0ull);
        s_bins[e] = b;
        if (b) s_nz[atomicAdd(&s_nnz, 1)] = e;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int a = 1; a < s_nnz; ++a)
            for (int j = a; j > 0 && s_nz[j - 1] > s_nz[j]; --j) {
                const int tmp = s_nz[j];
                s_nz[j] = s_nz[j - 1];
                s_nz[j - 1] = tmp;
            }
        const uint64_t wlo = atomicAdd(&u.win[0], 0ull), whi = atomicAdd(&u.win[1], 0ull);
        finalize_gamma(s_bins, s_nz, s_nnz, wlo, whi, u.n_total, u.eps, s_limb, u.gamma, u.thr);
        const uint32_t t_new = *u.thr;
        const unsigned listed = atomicAdd(u.list_count, 0u);
        const bool patch = hint && t_new >= t_lo && t_new <= t_hi && listed <= u.list_cap;
        *u.mode = patch ? 1u : 2u;
    }
}

__global__ void __launch_bounds__(256) k_pack_finish_quad(UpdateArgs u) {
    const uint32_t mode = *u.mode;
    const uint32_t thr = *u.thr;
    if (mode == 2u) {
        quad_pass(u.p, thr);
        return;
    }
    const unsigned listed = *u.list_count;
    for (unsigned j = blockIdx.x * blockDim.x + threadIdx.x; j < listed; j += gridDim.x * blockDim.x) {
        const int64_t i = u.list[j];
        patch_group(u.p, thr, i, __ldg(u.p.W + i));
    }
}

// Metadata padding: rows >= n_out of every k-block, and the groups past k in
// the last k-block, hold idx (0, 1) = nibble 0x4, so the tensor-core product
// sees zero values at valid positions.
__global__ void k_meta_pad(uint8_t *meta, int64_t n_out, int64_t k, int64_t meta_rows) {
    const int64_t kblocks = (k + 127) / 128;
    const int64_t tail_groups = (k / 4) - (kblocks - 1) * 32;   // valid groups of the last block
    const int64_t pad_rows = meta_rows - n_out;
    const int64_t n_a = kblocks * pad_rows * 16;                  // bytes of padded rows
    const int64_t tail_first_byte = (tail_groups + 1) / 2;        // first byte with no valid group
    const int64_t n_b = (tail_groups < 32) ? n_out * (16 - tail_first_byte) : 0;
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < n_a + n_b;
         j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        if (j < n_a) {
            const int64_t kb = j / (pad_rows * 16), rem = j - kb * pad_rows * 16;
            meta[(kb * meta_rows + n_out) * 16 + rem] = 0x44;
        } else {
            const int64_t jj = j - n_a, per = 16 - tail_first_byte;
            const int64_t row = jj / per, byte = tail_first_byte + (jj - row * per);
            meta[((kblocks - 1) * meta_rows + row) * 16 + byte] = 0x44;
        }
    }
    // a half-valid byte (odd number of valid groups): high nibble is padding
    if ((tail_groups & 1) && blockIdx.x == 0) {
        for (int64_t row = threadIdx.x; row < n_out; row += blockDim.x) {
            uint8_t *b = meta + ((kblocks - 1) * meta_rows + row) * 16 + tail_groups / 2;
            *b = static_cast<uint8_t>((*b & 0x0f) | 0x40);
        }
    }
}

// ---------------------------------------------------------------- mask, general N:M

__global__ void __launch_bounds__(256) k_mask_nm(const float *__restrict__ W, int64_t n_groups, int n, int m,
                                                 uint8_t *__restrict__ mask) {
    // one thread per group of m (m in {4, 8}); m = 8 writes one byte, m = 4 one nibble
    // via a neighbour exchange, as in k_pack24.
    const int lane = threadIdx.x & 31;
    const int64_t warp_stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t base = (static_cast<int64_t>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31)); base < n_groups;
         base += warp_stride) {
        const int64_t i = base + lane;
        const bool valid = i < n_groups;
        uint32_t mag[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) mag[q] = (valid && q < m) ? (__float_as_uint(__ldg(W + i * m + q)) & 0x7fffffffu) : 0u;
        uint32_t keep = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            if (q >= m) break;
            int before = 0;
#pragma unroll
            for (int r = 0; r < 8; ++r)
                if (r < m) before += (mag[r] > mag[q]) || (r < q && mag[r] == mag[q]);
            keep |= (before < n ? 1u : 0u) << q;
        }
        if (m == 8) {
            if (valid) mask[i] = static_cast<uint8_t>(keep);
        } else {
            const uint32_t hi = __shfl_xor_sync(0xffffffffu, keep, 1);
            if (valid && (lane & 1) == 0) mask[i >> 1] = static_cast<uint8_t>(keep | (hi << 4));
        }
    }
}

// ---------------------------------------------------------------- decode layout

// One thread per (16-row x 64-k tile, lane): 8 bytes = 16 two-bit codes (the
// lane's A fragment of the warp-level m16n8k64 sparse MMA) + 8 metadata nibbles.
// Fragment ownership (lane = 4*gid + tq):
//   values : register r in 0..3, byte j in 0..3 holds row gid + 8*(r&1),
//            compressed column 4*tq + j + 16*(r>>1) (two columns per group);
//            its 2-bit code sits at bit 8*j + 2*r of the code word.
//   meta   : row gid + 8*(lane&1), groups 8*((lane>>1)&1) .. +7 of the tile,
//            nibble q of the word for group 8*((lane>>1)&1) + q.
__global__ void __launch_bounds__(256) k_make_dec(const uint8_t *__restrict__ gb, int64_t n_out, int64_t k,
                                                  uint2 *__restrict__ dec) {
    const int64_t gpr = k / 4, ktiles = k / 64, rtiles = n_out / 16;
    const int64_t total = rtiles * ktiles * 32;
    for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int lane = static_cast<int>(idx & 31);
        const int64_t tile = idx >> 5;
        const int64_t rt = tile / ktiles, kt = tile - rt * ktiles;
        const int gid = lane >> 2, tq = lane & 3;
        const int64_t row0 = rt * 16, g0 = kt * 16;   // first row, first group of the tile
        uint32_t codes = 0;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int64_t row = row0 + gid + 8 * (r & 1);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int col = 4 * tq + j + 16 * (r >> 1);   // compressed column in 0..31
                const uint8_t b = gb[row * gpr + g0 + (col >> 1)];
                const uint32_t c = (col & 1) ? ((b >> 6) & 3u) : ((b >> 4) & 3u);
                codes |= c << (8 * j + 2 * r);
            }
        }
        uint32_t meta = 0;
        {
            const int64_t row = row0 + gid + 8 * (lane & 1);
            const int gs = 8 * ((lane >> 1) & 1);
#pragma unroll
            for (int q = 0; q < 8; ++q) meta |= static_cast<uint32_t>(gb[row * gpr + g0 + gs + q] & 0x0f) << (4 * q);
        }
        dec[idx] = make_uint2(codes, meta);
    }
}

// ---------------------------------------------------------------- host side

// SM count of the current device, looked up once per device (a process may
// drive several GPUs; each keeps its own entry).
int num_sms() {
    constexpr int kMaxDev = 64;
    static std::atomic<int> sms[kMaxDev];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= kMaxDev) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        return n > 0 ? n : 148;
    }
    int n = sms[dev].load(std::memory_order_relaxed);
    if (n <= 0) {
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
        sms[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// Raises a kernel's dynamic shared-memory limit to bytes on the current
// device.  The attribute belongs to the function in one device's context, so
// the record of what was set is kept per (device, function); a second device
// in the same process gets its own call.
cudaError_t smem_attr(const void *func, int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    struct Entry {
        int dev;
        const void *func;
        int bytes;
    };
    static std::mutex mu;
    static std::vector<Entry> done;
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry &d : done)
        if (d.dev == dev && d.func == func && d.bytes >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    for (Entry &d : done)
        if (d.dev == dev && d.func == func) {
            d.bytes = bytes;
            return cudaSuccess;
        }
    done.push_back(Entry{dev, func, bytes});
    return cudaSuccess;
}

static unsigned grid_for(int64_t work, int threads, int per_sm) {
    const int64_t need = (work + threads - 1) / threads;
    const int64_t cap = static_cast<int64_t>(num_sms()) * per_sm;
    return static_cast<unsigned>(need < cap ? (need > 0 ? need : 1) : cap);
}

cudaError_t launch_pack(const float *W, int64_t n_out, int64_t k, int n, int m, float eps, float *gamma,
                        uint8_t *gb, int8_t *vals, uint8_t *meta, uint8_t *dec, uint8_t *mask, void *ws,
                        cudaStream_t s) {
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    uint32_t *thr = reinterpret_cast<uint32_t *>(w8 + kPackWsThrOffset);
    unsigned long long *win = reinterpret_cast<unsigned long long *>(w8 + kPackWsWinOffset);
    unsigned long long *bins = reinterpret_cast<unsigned long long *>(w8 + kPackWsBinsOffset);
    cudaError_t err = cudaMemsetAsync(ws, 0, kPackWsBytes, s);
    if (err != cudaSuccess) return err;
    const int64_t n_el = n_out * k;
    unsigned *counter = reinterpret_cast<unsigned *>(w8 + kPackWsCounterOffset);
    k_abs_sum_fast<<<grid_for(n_el / 4, 256, 4), 256, 0, s>>>(reinterpret_cast<const float4 *>(W), n_el / 4, win,
                                                             bins, counter, n_el, eps, gamma, thr);
    const bool packed = gb || vals || meta || dec;
    if (packed) {
        Pack24Args a;
        a.W = reinterpret_cast<const float4 *>(W);
        a.n_groups = n_el / 4;
        a.gpr = k / 4;
        a.gpr_div = make_fastdiv(static_cast<uint32_t>(k / 4));
        a.n_out = n_out;
        a.k = k;
        a.meta_rows = (n_out + 127) / 128 * 128;
        a.thr = thr;
        a.gb = gb;
        a.vals = reinterpret_cast<uint16_t *>(vals);
        a.meta = meta;
        a.mask = (n == 2 && m == 4) ? mask : nullptr;
        if (k % 16 == 0)
            k_pack24_quad<<<grid_for((a.n_groups / 4 + kQuadUnroll - 1) / kQuadUnroll, 256, 8), 256, 0, s>>>(a);
        else
            k_pack24<<<grid_for((a.n_groups + kPackUnroll - 1) / kPackUnroll, 256, 8), 256, 0, s>>>(a);
        if (meta && (a.meta_rows != n_out || (k % 128) != 0))
            k_meta_pad<<<grid_for(((k + 127) / 128) * (a.meta_rows - n_out) * 16 + n_out * 16, 256, 4), 256, 0, s>>>(
                meta, n_out, k, a.meta_rows);
        if (dec)
            k_make_dec<<<grid_for(n_out / 16 * (k / 64) * 32, 256, 8), 256, 0, s>>>(gb, n_out, k,
                                                                                    reinterpret_cast<uint2 *>(dec));
    }
    if (mask && !(packed && n == 2 && m == 4)) {
        const int64_t groups = n_el / m;
        k_mask_nm<<<grid_for(groups, 256, 8), 256, 0, s>>>(W, groups, n, m, mask);
    }
    return cudaGetLastError();
}

cudaError_t launch_adamw_gamma(float *W, const float *G, float *M, float *V, int64_t n, float lr, float b1, float b2,
                               float eps, float wd, float c1, float c2, float eps_gamma, float *gamma, void *ws,
                               cudaStream_t s) {
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    cudaError_t err = cudaMemsetAsync(ws, 0, kPackWsBytes, s);
    if (err != cudaSuccess) return err;
    AdamWArgs a;
    a.W = reinterpret_cast<float4 *>(W);
    a.G = reinterpret_cast<const float4 *>(G);
    a.M = reinterpret_cast<float4 *>(M);
    a.V = reinterpret_cast<float4 *>(V);
    a.n4 = n / 4;
    a.lr = lr;
    a.b1 = b1;
    a.b2 = b2;
    a.eps = eps;
    a.wd = wd;
    a.c1 = c1;
    a.c2 = c2;
    a.win = reinterpret_cast<unsigned long long *>(w8 + kPackWsWinOffset);
    a.bins = reinterpret_cast<unsigned long long *>(w8 + kPackWsBinsOffset);
    a.counter = reinterpret_cast<unsigned *>(w8 + kPackWsCounterOffset);
    a.n_total = n;
    a.eps_gamma = eps_gamma;
    a.gamma = gamma;
    a.thr = reinterpret_cast<uint32_t *>(w8 + kPackWsThrOffset);
    k_adamw_gamma<<<grid_for(a.n4, 256, 6), 256, 0, s>>>(a);
    return cudaGetLastError();
}

// The same AdamW step over a list of matrices in one launch: every matrix is cut
// into chunks of kAdamWChunk float4 groups and every CTA takes a contiguous
// range of the global chunk list (so it meets one or two matrices); per matrix
// the exact partial sums go to its own workspace header, and the CTA that
// completes its last chunk forms its gamma.
constexpr uint32_t kAdamWChunk = 2048;   // float4 groups per chunk (8192 weights)

struct AdamWBatchItem {
    float4 *W;
    const float4 *G;
    float4 *M, *V;
    int64_t n4;
    float *gamma;
    uint8_t *hdr;             // kPackWsBytes scratch header (zeroed before the launch)
    uint32_t chunk0, nchunks;
};

struct AdamWBatchParams {
    AdamWBatchItem it[kAdamWBatchMax];
    int32_t n;
    uint32_t total_chunks;
    float lr, b1, b2, eps, wd, c1, c2, eps_gamma;
};

__device__ __forceinline__ int adamw_item_of(const AdamWBatchParams &bp, uint32_t c) {
    int lo = 0, hi = bp.n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (bp.it[mid].chunk0 <= c) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(256, 6) k_adamw_gamma_batch(const __grid_constant__ AdamWBatchParams bp) {
    __shared__ unsigned long long s_bins[256];
    __shared__ unsigned long long s_lo[8], s_hi[8];
    __shared__ int s_rare;
    __shared__ unsigned s_ticket;
    __shared__ int s_nz[256];
    __shared__ int s_nnz;
    __shared__ uint32_t s_limb[kLimbs];
    const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t G = gridDim.x;
    const uint32_t c_begin = static_cast<uint32_t>((static_cast<uint64_t>(blockIdx.x) * bp.total_chunks) / G);
    const uint32_t c_end = static_cast<uint32_t>((static_cast<uint64_t>(blockIdx.x + 1) * bp.total_chunks) / G);
    for (int i = threadIdx.x; i < 256; i += blockDim.x) s_bins[i] = 0ull;
    if (threadIdx.x == 0) s_rare = 0;
    __syncthreads();
    AdamWArgs a;   // the scalar hyper-parameters in the form adamw1 takes them
    a.lr = bp.lr;
    a.b1 = bp.b1;
    a.b2 = bp.b2;
    a.eps = bp.eps;
    a.wd = bp.wd;
    a.c1 = bp.c1;
    a.c2 = bp.c2;
    const float omb1 = __fsub_rn(1.0f, bp.b1), omb2 = __fsub_rn(1.0f, bp.b2);
    uint32_t c = c_begin;
    while (c < c_end) {
        const int item = adamw_item_of(bp, c);
        const AdamWBatchItem &I = bp.it[item];
        const uint32_t seg_end = min(c_end, I.chunk0 + I.nchunks);
        uint64_t lo = 0, hi = 0;
        double d = 0.0;
        for (uint32_t ch = c; ch < seg_end; ++ch) {
            const int64_t base = static_cast<int64_t>(ch - I.chunk0) * kAdamWChunk;
            const int64_t end = min(base + static_cast<int64_t>(kAdamWChunk), I.n4);
            for (int64_t j = base + threadIdx.x; j < end; j += blockDim.x) {
                const float4 w = I.W[j], g = __ldg(I.G + j);
                float4 m = I.M[j], v = I.V[j];
                float4 wn;
                wn.x = adamw1(w.x, g.x, m.x, v.x, a, omb1, omb2);
                wn.y = adamw1(w.y, g.y, m.y, v.y, a, omb1, omb2);
                wn.z = adamw1(w.z, g.z, m.z, v.z, a, omb1, omb2);
                wn.w = adamw1(w.w, g.w, m.w, v.w, a, omb1, omb2);
                I.W[j] = wn;
                I.M[j] = m;
                I.V[j] = v;
                sum_float4(wn, d, lo, hi, s_bins, &s_rare);
            }
            flush_sum(d, lo, hi);   // at most 8 groups (32 magnitudes) per thread per chunk
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const uint64_t l2 = __shfl_xor_sync(0xffffffffu, lo, o);
            const uint64_t h2 = __shfl_xor_sync(0xffffffffu, hi, o);
            const uint64_t sum = lo + l2;
            hi = hi + h2 + ((sum < lo) ? 1ull : 0ull);
            lo = sum;
        }
        if (lane == 0) {
            s_lo[warp] = lo;
            s_hi[warp] = hi;
        }
        __syncthreads();
        unsigned long long *win = reinterpret_cast<unsigned long long *>(I.hdr + kPackWsWinOffset);
        unsigned long long *bins = reinterpret_cast<unsigned long long *>(I.hdr + kPackWsBinsOffset);
        if (threadIdx.x == 0) {
            uint64_t L = 0, H = 0;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
                const uint64_t sum = L + s_lo[w];
                H = H + s_hi[w] + ((sum < L) ? 1ull : 0ull);
                L = sum;
            }
            if (L | H) {
                const unsigned long long old = atomicAdd(&win[0], static_cast<unsigned long long>(L));
                const uint64_t carry = (static_cast<uint64_t>(old) + L < static_cast<uint64_t>(old)) ? 1ull : 0ull;
                atomicAdd(&win[1], static_cast<unsigned long long>(H + carry));
            }
        }
        if (s_rare) {
            for (int e = threadIdx.x; e < 256; e += blockDim.x)
                if (s_bins[e]) {
                    atomicAdd(&bins[e], s_bins[e]);
                    s_bins[e] = 0ull;
                }
        }
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) {
            s_rare = 0;
            const unsigned done = seg_end - c;
            s_ticket = atomicAdd(reinterpret_cast<unsigned *>(I.hdr + kPackWsCounterOffset), done) + done;
        }
        __syncthreads();
        if (s_ticket == I.nchunks) {   // every chunk of this matrix is summed: its gamma
            __threadfence();
            if (threadIdx.x == 0) s_nnz = 0;
            __syncthreads();
            for (int e = threadIdx.x; e < 256; e += blockDim.x) {
                const unsigned long long b = atomicAdd(&bins[e], 0ull);
                s_bins[e] = b;
                if (b) s_nz[atomicAdd(&s_nnz, 1)] = e;
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                for (int q = 1; q < s_nnz; ++q)
                    for (int j = q; j > 0 && s_nz[j - 1] > s_nz[j]; --j) {
                        const int tmp = s_nz[j];
                        s_nz[j] = s_nz[j - 1];
                        s_nz[j - 1] = tmp;
                    }
                const uint64_t wlo = atomicAdd(&win[0], 0ull), whi = atomicAdd(&win[1], 0ull);
                finalize_gamma(s_bins, s_nz, s_nnz, wlo, whi, I.n4 * 4, bp.eps_gamma, s_limb, I.gamma,
                               reinterpret_cast<uint32_t *>(I.hdr + kPackWsThrOffset));
            }
            __syncthreads();
            for (int e = threadIdx.x; e < 256; e += blockDim.x) s_bins[e] = 0ull;
            __syncthreads();
        }
        c = seg_end;
    }
}

cudaError_t launch_adamw_gamma_batch(const AdamWItemHost *items, int n_items, float lr, float b1, float b2, float eps,
                                     float wd, float c1, float c2, float eps_gamma, void *ws, cudaStream_t s) {
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    cudaError_t err = cudaMemsetAsync(ws, 0, static_cast<size_t>(n_items) * kPackWsBytes, s);
    if (err != cudaSuccess) return err;
    for (int base = 0; base < n_items; base += kAdamWBatchMax) {
        const int n = (n_items - base) < kAdamWBatchMax ? (n_items - base) : kAdamWBatchMax;
        AdamWBatchParams bp;
        uint32_t chunks = 0;
        for (int i = 0; i < n; ++i) {
            const AdamWItemHost &h = items[base + i];
            AdamWBatchItem &I = bp.it[i];
            I.W = reinterpret_cast<float4 *>(h.W);
            I.G = reinterpret_cast<const float4 *>(h.G);
            I.M = reinterpret_cast<float4 *>(h.M);
            I.V = reinterpret_cast<float4 *>(h.V);
            I.n4 = h.n / 4;
            I.gamma = h.gamma;
            I.hdr = w8 + static_cast<size_t>(base + i) * kPackWsBytes;
            I.chunk0 = chunks;
            I.nchunks = static_cast<uint32_t>((I.n4 + kAdamWChunk - 1) / kAdamWChunk);
            chunks += I.nchunks;
        }
        bp.n = n;
        bp.total_chunks = chunks;
        bp.lr = lr;
        bp.b1 = b1;
        bp.b2 = b2;
        bp.eps = eps;
        bp.wd = wd;
        bp.c1 = c1;
        bp.c2 = c2;
        bp.eps_gamma = eps_gamma;
        const uint32_t want = static_cast<uint32_t>(num_sms() * 6);
        const unsigned grid = chunks < want ? chunks : want;
        k_adamw_gamma_batch<<<grid, 256, 0, s>>>(bp);
    }
    return cudaGetLastError();
}

cudaError_t launch_pack_update(const float *W, int64_t n_out, int64_t k, float eps, float *gamma, uint8_t *gb,
                               int8_t *vals, uint8_t *meta, uint8_t *dec, uint8_t *mask, void *ws, size_t ws_bytes,
                               cudaStream_t s) {
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    cudaError_t err = cudaMemsetAsync(ws, 0, kPackWsBytes, s);
    if (err != cudaSuccess) return err;
    const int64_t n_el = n_out * k;
    UpdateArgs u;
    u.p.W = reinterpret_cast<const float4 *>(W);
    u.p.n_groups = n_el / 4;
    u.p.gpr = k / 4;
    u.p.gpr_div = make_fastdiv(static_cast<uint32_t>(k / 4));
    u.p.n_out = n_out;
    u.p.k = k;
    u.p.meta_rows = (n_out + 127) / 128 * 128;
    u.p.thr = nullptr;
    u.p.gb = gb;
    u.p.vals = reinterpret_cast<uint16_t *>(vals);
    u.p.meta = meta;
    u.p.mask = mask;
    u.gamma_prev = gamma;
    u.gamma = gamma;
    u.win = reinterpret_cast<unsigned long long *>(w8 + kPackWsWinOffset);
    u.bins = reinterpret_cast<unsigned long long *>(w8 + kPackWsBinsOffset);
    u.counter = reinterpret_cast<unsigned *>(w8 + kPackWsCounterOffset);
    u.thr = reinterpret_cast<uint32_t *>(w8 + kPackWsThrOffset);
    u.mode = reinterpret_cast<uint32_t *>(w8 + kPackWsModeOffset);
    u.band = reinterpret_cast<uint32_t *>(w8 + kPackWsBandOffset);
    u.list_count = reinterpret_cast<unsigned *>(w8 + kPackWsListCountOffset);
    u.list = reinterpret_cast<uint32_t *>(w8 + kPackWsBytes);
    u.list_cap = static_cast<uint32_t>((ws_bytes - kPackWsBytes) / 4);
    u.n_total = n_el;
    u.eps = eps;
    if (k % 16 == 0) {
        const unsigned grid = grid_for((u.p.n_groups / 4 + kQuadUnroll - 1) / kQuadUnroll, 256, 4);
        k_pack_update_quad<<<grid, 256, 0, s>>>(u);
        k_pack_finish_quad<<<grid, 256, 0, s>>>(u);
    } else {
        const unsigned grid = grid_for((u.p.n_groups + kPackUnroll - 1) / kPackUnroll, 256, 4);
        k_pack_update<<<grid, 256, 0, s>>>(u);
        k_pack_finish<<<grid, 256, 0, s>>>(u);
    }
    if (meta && (u.p.meta_rows != n_out || (k % 128) != 0))
        k_meta_pad<<<grid_for(((k + 127) / 128) * (u.p.meta_rows - n_out) * 16 + n_out * 16, 256, 4), 256, 0, s>>>(
            meta, n_out, k, u.p.meta_rows);
    if (dec)
        k_make_dec<<<grid_for(n_out / 16 * (k / 64) * 32, 256, 8), 256, 0, s>>>(gb, n_out, k,
                                                                                reinterpret_cast<uint2 *>(dec));
    return cudaGetLastError();
}


// ---------------------------------------------------------------- batched per-step pack (lane quads)
//
// bitnet_pack_nm_update over a list of matrices in two launches instead of
// three or four per matrix.  The matrices' quads are cut into chunks of
// kBatchChunkQuads; the update kernel gives every CTA a contiguous range of
// the global chunk list, so a CTA meets one or two matrices.  Per matrix it
// does what k_pack_update_quad does (exact sum, layouts with the previous
// gamma's threshold, band list), with a per-matrix chunk counter in place of
// the block ticket: the CTA that completes a matrix's last chunk forms its
// gamma, threshold and mode.  The finish kernel then patches every listed
// group (mode 1), reruns the layouts of the matrices whose threshold left the
// band (mode 2) and writes the metadata padding, each over one flattened
// index space across the matrices.  Results are those of
// bitnet_pack_nm_update on each matrix, bit for bit.

struct BatchItem {
    Pack24Args p;              // layouts (p.thr unused)
    float *gamma;              // previous gamma in (the hint), new gamma out
    uint8_t *hdr;              // this matrix's kPackWsBytes scratch header (zeroed before the launch)
    uint32_t *list;            // band list
    uint32_t list_cap;
    uint32_t chunk0, nchunks;  // this matrix's range of the global chunk list
    uint32_t pad_bytes;        // metadata padding bytes (0: none)
    uint32_t w_bf16;           // 1: the masters (p.W) are bf16, widened exactly to fp32 on load
    uint32_t gamma_known;      // 1: *gamma already is the exact gamma of W (no sum, no band, gamma kept)
    int64_t n_total;
};

struct BatchParams {
    BatchItem it[kPackBatchMax];
    int32_t n;
    uint32_t total_chunks;
    float eps;
};

constexpr uint32_t kBatchChunkQuads = 512;   // 256 threads x 2 quads

// four bf16 masters (8 bytes) widened exactly to fp32
__device__ __forceinline__ float4 bf16x4_to_float4(uint2 u) {
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u), __uint_as_float(u.y << 16),
                       __uint_as_float(u.y & 0xffff0000u));
}

// the four groups (16 masters) of quad q, fp32 or bf16 storage
__device__ __forceinline__ void load_quad(const Pack24Args &p, bool bf16, uint32_t q, float4 (&v)[4]) {
    if (bf16) {
        const uint4 *Wb = reinterpret_cast<const uint4 *>(p.W);
        const uint4 a = __ldg(Wb + 2u * q), b = __ldg(Wb + 2u * q + 1u);
        v[0] = bf16x4_to_float4(make_uint2(a.x, a.y));
        v[1] = bf16x4_to_float4(make_uint2(a.z, a.w));
        v[2] = bf16x4_to_float4(make_uint2(b.x, b.y));
        v[3] = bf16x4_to_float4(make_uint2(b.z, b.w));
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = __ldg(p.W + 4u * q + j);
    }
}

__device__ __forceinline__ float4 load_group(const Pack24Args &p, bool bf16, int64_t i) {
    if (bf16) return bf16x4_to_float4(__ldg(reinterpret_cast<const uint2 *>(p.W) + i));
    return __ldg(p.W + i);
}

__device__ __forceinline__ int batch_item_of(const BatchParams &bp, uint32_t c) {
    int lo = 0, hi = bp.n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (bp.it[mid].chunk0 <= c) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// One CTA's run of chunks [c, seg_end) of one matrix: exact partial sum of
// |W| (into lo, hi) and, with a hint, every layout with the hint's threshold
// plus the band list.  BF16: the masters are bf16.
template <bool BF16, bool KNOWN>
__device__ __forceinline__ void batch_segment(const BatchItem &I, uint32_t c, uint32_t seg_end, bool hint,
                                              uint32_t t_old, uint32_t t_lo, uint32_t t_hi, unsigned *list_count,
                                              uint64_t &lo, uint64_t &hi, unsigned long long *s_bins, int *s_rare) {
    const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const Pack24Args &p = I.p;
    const uint32_t n_quads = static_cast<uint32_t>(p.n_groups >> 2);
    double d = 0.0;
    for (uint32_t ch = c; ch < seg_end; ++ch) {
        const uint32_t qbase = (ch - I.chunk0) * kBatchChunkQuads + warp * (32u * kQuadUnroll);
        float4 v[kQuadUnroll][4];
#pragma unroll
        for (int k2 = 0; k2 < kQuadUnroll; ++k2) {
            const uint32_t q = qbase + 32u * k2 + lane;
            if (q < n_quads) {
                load_quad(p, BF16, q, v[k2]);
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) v[k2][j] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int k2 = 0; k2 < kQuadUnroll; ++k2) {
            const uint32_t q = qbase + 32u * k2 + lane;
            if (!KNOWN) {
#pragma unroll
                for (int j = 0; j < 4; ++j) sum_float4(v[k2][j], d, lo, hi, s_bins, s_rare);
            }
            if (hint && q < n_quads) {
                const QuadOut o = pack_quad(v[k2], t_old, t_lo, t_hi);
                store_quad(p, q, o);
                if (o.band) {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if ((o.band >> j) & 1u) {
                            const unsigned slot = atomicAdd(list_count, 1u);
                            if (slot < I.list_cap) I.list[slot] = 4u * q + j;
                        }
                }
            }
        }
        flush_sum(d, lo, hi);
    }
}

__global__ void __launch_bounds__(256, 4) k_pack_update_batch(const __grid_constant__ BatchParams bp) {
    __shared__ unsigned long long s_bins[256];
    __shared__ unsigned long long s_lo[8], s_hi[8];
    __shared__ int s_rare;
    __shared__ uint32_t s_t, s_tlo, s_thi;
    __shared__ int s_hint;
    __shared__ unsigned s_ticket;
    __shared__ int s_nz[256];
    __shared__ int s_nnz;
    __shared__ uint32_t s_limb[kLimbs];
    const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t G = gridDim.x;
    const uint32_t c_begin = static_cast<uint32_t>((static_cast<uint64_t>(blockIdx.x) * bp.total_chunks) / G);
    const uint32_t c_end = static_cast<uint32_t>((static_cast<uint64_t>(blockIdx.x + 1) * bp.total_chunks) / G);
    for (int i = threadIdx.x; i < 256; i += blockDim.x) s_bins[i] = 0ull;
    uint32_t c = c_begin;
    while (c < c_end) {
        const int item = batch_item_of(bp, c);
        const BatchItem &I = bp.it[item];
        const uint32_t seg_end = min(c_end, I.chunk0 + I.nchunks);
        uint8_t *hdr = I.hdr;
        if (threadIdx.x == 0) {
            s_rare = 0;
            const float gp = *I.gamma;
            s_hint = (gp > 0.0f && gp < 3.0e38f) ? 1 : 0;
            s_t = s_tlo = s_thi = 0u;
            if (s_hint) {
                s_t = code_threshold(gp);
                const float tf = __uint_as_float(s_t);
                s_tlo = __float_as_uint(__fmul_rd(tf, 1.0f - 0x1p-10f));
                s_thi = __float_as_uint(__fmul_ru(tf, 1.0f + 0x1p-10f));
                if (c == I.chunk0) {
                    reinterpret_cast<uint32_t *>(hdr + kPackWsBandOffset)[0] = s_tlo;
                    reinterpret_cast<uint32_t *>(hdr + kPackWsBandOffset)[1] = s_thi;
                }
            }
        }
        __syncthreads();
        const bool hint = s_hint != 0;
        const uint32_t t_old = s_t, t_lo = s_tlo, t_hi = s_thi;
        const bool wbf16 = I.w_bf16 != 0u;
        unsigned *list_count = reinterpret_cast<unsigned *>(hdr + kPackWsListCountOffset);
        uint64_t lo = 0, hi = 0;
        const bool known = hint && I.gamma_known != 0u;
        if (known) {   // codes against the exact threshold: nothing to sum, no band to list
            if (wbf16)
                batch_segment<true, true>(I, c, seg_end, true, t_old, 0xffffffffu, 0xffffffffu, list_count, lo, hi,
                                          s_bins, &s_rare);
            else
                batch_segment<false, true>(I, c, seg_end, true, t_old, 0xffffffffu, 0xffffffffu, list_count, lo, hi,
                                           s_bins, &s_rare);
        } else if (wbf16) {
            batch_segment<true, false>(I, c, seg_end, hint, t_old, t_lo, t_hi, list_count, lo, hi, s_bins, &s_rare);
        } else {
            batch_segment<false, false>(I, c, seg_end, hint, t_old, t_lo, t_hi, list_count, lo, hi, s_bins, &s_rare);
        }
        // this segment's exact partial sum into the matrix's accumulators
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const uint64_t l2 = __shfl_xor_sync(0xffffffffu, lo, o);
            const uint64_t h2 = __shfl_xor_sync(0xffffffffu, hi, o);
            const uint64_t sum = lo + l2;
            hi = hi + h2 + ((sum < lo) ? 1ull : 0ull);
            lo = sum;
        }
        if (lane == 0) {
            s_lo[warp] = lo;
            s_hi[warp] = hi;
        }
        __syncthreads();
        unsigned long long *win = reinterpret_cast<unsigned long long *>(hdr + kPackWsWinOffset);
        unsigned long long *bins = reinterpret_cast<unsigned long long *>(hdr + kPackWsBinsOffset);
        if (threadIdx.x == 0) {
            uint64_t L = 0, H = 0;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
                const uint64_t sum = L + s_lo[w];
                H = H + s_hi[w] + ((sum < L) ? 1ull : 0ull);
                L = sum;
            }
            if (L | H) {
                const unsigned long long old = atomicAdd(&win[0], static_cast<unsigned long long>(L));
                const uint64_t carry = (static_cast<uint64_t>(old) + L < static_cast<uint64_t>(old)) ? 1ull : 0ull;
                atomicAdd(&win[1], static_cast<unsigned long long>(H + carry));
            }
        }
        if (s_rare) {
            for (int e = threadIdx.x; e < 256; e += blockDim.x)
                if (s_bins[e]) {
                    atomicAdd(&bins[e], s_bins[e]);
                    s_bins[e] = 0ull;
                }
        }
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) {
            const unsigned done = seg_end - c;
            s_ticket = atomicAdd(reinterpret_cast<unsigned *>(hdr + kPackWsCounterOffset), done) + done;
        }
        __syncthreads();
        if (s_ticket == I.nchunks && !known) {
            // every chunk of this matrix is summed: form gamma, threshold and mode
            __threadfence();
            if (threadIdx.x == 0) s_nnz = 0;
            __syncthreads();
            for (int e = threadIdx.x; e < 256; e += blockDim.x) {
                const unsigned long long b = atomicAdd(&bins[e], 0ull);
                s_bins[e] = b;
                if (b) s_nz[atomicAdd(&s_nnz, 1)] = e;
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                for (int a = 1; a < s_nnz; ++a)
                    for (int j = a; j > 0 && s_nz[j - 1] > s_nz[j]; --j) {
                        const int tmp = s_nz[j];
                        s_nz[j] = s_nz[j - 1];
                        s_nz[j - 1] = tmp;
                    }
                const uint64_t wlo = atomicAdd(&win[0], 0ull), whi = atomicAdd(&win[1], 0ull);
                uint32_t *thr = reinterpret_cast<uint32_t *>(hdr + kPackWsThrOffset);
                finalize_gamma(s_bins, s_nz, s_nnz, wlo, whi, I.n_total, bp.eps, s_limb, I.gamma, thr);
                const uint32_t t_new = *thr;
                const unsigned listed = atomicAdd(list_count, 0u);
                const bool patch = hint && t_new >= t_lo && t_new <= t_hi && listed <= I.list_cap;
                *reinterpret_cast<uint32_t *>(hdr + kPackWsModeOffset) = patch ? 1u : 2u;
            }
            __syncthreads();
            for (int e = threadIdx.x; e < 256; e += blockDim.x) s_bins[e] = 0ull;
        }
        __syncthreads();
        c = seg_end;
    }
}

// index of the last entry of pref[0..n] that is <= x (pref ascending, pref[0] = 0)
__device__ __forceinline__ int batch_bucket(const uint32_t *pref, int n, uint32_t x) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pref[mid] <= x) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Byte j of the metadata padding of one matrix (k % 16 == 0, so no half-valid
// bytes): the rows >= n_out of every k-block, then the bytes past the last
// valid group of the last k-block.  Same bytes as k_meta_pad.
__device__ __forceinline__ void meta_pad_at(const Pack24Args &p, uint32_t j) {
    const int64_t kblocks = (p.k + 127) / 128;
    const int64_t tail_groups = (p.k / 4) - (kblocks - 1) * 32;
    const int64_t pad_rows = p.meta_rows - p.n_out;
    const int64_t n_a = kblocks * pad_rows * 16;
    if (static_cast<int64_t>(j) < n_a) {
        const int64_t kb = j / (pad_rows * 16), rem = j - kb * pad_rows * 16;
        p.meta[(kb * p.meta_rows + p.n_out) * 16 + rem] = 0x44;
    } else {
        const int64_t tail_first_byte = (tail_groups + 1) / 2;
        const int64_t jj = j - n_a, per = 16 - tail_first_byte;
        const int64_t row = jj / per, byte = tail_first_byte + (jj - row * per);
        p.meta[((kblocks - 1) * p.meta_rows + row) * 16 + byte] = 0x44;
    }
}

uint32_t meta_pad_bytes(int64_t n_out, int64_t k) {
    const int64_t meta_rows = (n_out + 127) / 128 * 128;
    const int64_t kblocks = (k + 127) / 128;
    const int64_t tail_groups = (k / 4) - (kblocks - 1) * 32;
    const int64_t n_a = kblocks * (meta_rows - n_out) * 16;
    const int64_t n_b = (tail_groups < 32) ? n_out * (16 - (tail_groups + 1) / 2) : 0;
    return static_cast<uint32_t>(n_a + n_b);
}

__global__ void __launch_bounds__(256) k_pack_finish_batch(const __grid_constant__ BatchParams bp) {
    __shared__ uint32_t s_thr[kPackBatchMax];
    __shared__ uint32_t s_patch[kPackBatchMax + 1], s_quads[kPackBatchMax + 1], s_pad[kPackBatchMax + 1];
    const int n = bp.n;
    if (threadIdx.x < n) {
        const BatchItem &I = bp.it[threadIdx.x];
        const uint32_t mode = *reinterpret_cast<const uint32_t *>(I.hdr + kPackWsModeOffset);
        const unsigned listed = *reinterpret_cast<const unsigned *>(I.hdr + kPackWsListCountOffset);
        s_thr[threadIdx.x] = *reinterpret_cast<const uint32_t *>(I.hdr + kPackWsThrOffset);
        s_patch[threadIdx.x + 1] = mode == 1u ? (listed < I.list_cap ? listed : I.list_cap) : 0u;
        s_quads[threadIdx.x + 1] = mode == 2u ? static_cast<uint32_t>(I.p.n_groups >> 2) : 0u;
        s_pad[threadIdx.x + 1] = I.pad_bytes;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        s_patch[0] = s_quads[0] = s_pad[0] = 0u;
        for (int i = 1; i <= n; ++i) {
            s_patch[i] += s_patch[i - 1];
            s_quads[i] += s_quads[i - 1];
            s_pad[i] += s_pad[i - 1];
        }
    }
    __syncthreads();
    const uint32_t gtid = blockIdx.x * blockDim.x + threadIdx.x;
    const uint32_t gstride = gridDim.x * blockDim.x;
    // 1. listed groups of the matrices whose threshold stayed in the band
    for (uint32_t x = gtid; x < s_patch[n]; x += gstride) {
        const int item = batch_bucket(s_patch, n, x);
        const BatchItem &I = bp.it[item];
        const int64_t i = I.list[x - s_patch[item]];
        patch_group(I.p, s_thr[item], i, load_group(I.p, I.w_bf16 != 0u, i));
    }
    // 2. every quad of the matrices whose threshold left the band (or had no hint)
    for (uint32_t x = gtid; x < s_quads[n]; x += gstride) {
        const int item = batch_bucket(s_quads, n, x);
        const BatchItem &I = bp.it[item];
        const uint32_t q = x - s_quads[item];
        float4 v[4];
        load_quad(I.p, I.w_bf16 != 0u, q, v);
        store_quad(I.p, q, pack_quad(v, s_thr[item], 0u, 0u));
    }
    // 3. metadata padding
    for (uint32_t x = gtid; x < s_pad[n]; x += gstride) {
        const int item = batch_bucket(s_pad, n, x);
        meta_pad_at(bp.it[item].p, x - s_pad[item]);
    }
}

size_t pack_batch_ws_bytes(const int64_t *n_out, const int64_t *k, int n_items) {
    size_t b = static_cast<size_t>(n_items) * kPackWsBytes;
    for (int i = 0; i < n_items; ++i) b += update_list_bytes(n_out[i], k[i]);
    return b;
}

cudaError_t launch_pack_update_batch(const PackBatchItemHost *items, int n_items, float eps, void *ws, cudaStream_t s) {
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    // every header first, then the lists: one memset clears all headers
    cudaError_t err = cudaMemsetAsync(ws, 0, static_cast<size_t>(n_items) * kPackWsBytes, s);
    if (err != cudaSuccess) return err;
    uint8_t *lists = w8 + static_cast<size_t>(n_items) * kPackWsBytes;
    for (int base = 0; base < n_items; base += kPackBatchMax) {
        const int n = (n_items - base) < kPackBatchMax ? (n_items - base) : kPackBatchMax;
        BatchParams bp;
        uint32_t chunks = 0;
        for (int i = 0; i < n; ++i) {
            const PackBatchItemHost &h = items[base + i];
            BatchItem &I = bp.it[i];
            const int64_t n_el = h.n_out * h.k;
            I.p.W = reinterpret_cast<const float4 *>(h.W);
            I.w_bf16 = h.w_bf16 ? 1u : 0u;
            I.gamma_known = h.gamma_known ? 1u : 0u;
            I.p.n_groups = n_el / 4;
            I.p.gpr = h.k / 4;
            I.p.gpr_div = make_fastdiv(static_cast<uint32_t>(h.k / 4));
            I.p.n_out = h.n_out;
            I.p.k = h.k;
            I.p.meta_rows = (h.n_out + 127) / 128 * 128;
            I.p.thr = nullptr;
            I.p.gb = h.gb;
            I.p.vals = reinterpret_cast<uint16_t *>(h.vals);
            I.p.meta = h.meta;
            I.p.mask = h.mask;
            I.gamma = h.gamma;
            I.hdr = w8 + static_cast<size_t>(base + i) * kPackWsBytes;
            I.list = reinterpret_cast<uint32_t *>(lists);
            const size_t lb = update_list_bytes(h.n_out, h.k);
            I.list_cap = static_cast<uint32_t>(lb / 4);
            lists += lb;
            const uint32_t quads = static_cast<uint32_t>(I.p.n_groups / 4);
            I.chunk0 = chunks;
            I.nchunks = (quads + kBatchChunkQuads - 1) / kBatchChunkQuads;
            chunks += I.nchunks;
            I.pad_bytes = (h.meta && (I.p.meta_rows != h.n_out || (h.k % 128) != 0)) ? meta_pad_bytes(h.n_out, h.k) : 0u;
            I.n_total = n_el;
        }
        bp.n = n;
        bp.total_chunks = chunks;
        bp.eps = eps;
        const unsigned grid = static_cast<unsigned>(num_sms() * 4);
        k_pack_update_batch<<<grid, 256, 0, s>>>(bp);
        k_pack_finish_batch<<<grid, 256, 0, s>>>(bp);
        for (int i = 0; i < n; ++i) {
            const PackBatchItemHost &h = items[base + i];
            if (h.dec)
                k_make_dec<<<grid_for(h.n_out / 16 * (h.k / 64) * 32, 256, 8), 256, 0, s>>>(
                    h.gb, h.n_out, h.k, reinterpret_cast<uint2 *>(h.dec));
        }
    }
    return cudaGetLastError();
}


// ---------------------------------------------------------------- 6:8 through 2:4 windows
//
// "Sparse-BitNet" (gist.science), section 4 "Resultaten": the method trains
// at 6:8.  "Is 2:4 Sparsity Still Worth It? ..." (thelatestinai.com), its
// SlideSparse entry: a (2N-2):2N block is rewritten, without loss, as N-1
// overlapping 2:4-compliant windows, and the activations are rearranged to
// match during per-token quantisation.  For 6:8 (N = 4) the three windows of
// every block of 8 start at positions 0, 2 and 4 and are 4 wide.  The pages
// do not give the assignment of kept positions to windows; here each kept
// position goes, in increasing order, to the leftmost window that covers it
// and has a free slot.  A position's windows form a contiguous range, so this
// greedy assignment fills all six slots for every choice of six kept
// positions.  The result is a canonical 2:4 matrix over k' = 3k/2 whose
// product with the lifted activations equals the 6:8 product exactly.

// one thread per block of 8 weights -> three group bytes of the window layout
__global__ void __launch_bounds__(256) k_pack68(const float4 *__restrict__ W, int64_t n_blocks,
                                               const uint32_t *__restrict__ thr_p, uint8_t *__restrict__ gbw) {
    const uint32_t thr = *thr_p;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < n_blocks; b += stride) {
        const float4 v0 = __ldg(W + 2 * b), v1 = __ldg(W + 2 * b + 1);
        const uint32_t bits[8] = {__float_as_uint(v0.x), __float_as_uint(v0.y), __float_as_uint(v0.z),
                                  __float_as_uint(v0.w), __float_as_uint(v1.x), __float_as_uint(v1.y),
                                  __float_as_uint(v1.z), __float_as_uint(v1.w)};
        uint32_t mag[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mag[i] = bits[i] & 0x7fffffffu;
        // position i is kept when fewer than six positions rank ahead of it
        // (larger magnitude, or equal magnitude at a lower position)
        uint32_t keep = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t ahead = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j != i) ahead += (j < i) ? (mag[j] >= mag[i] ? 1u : 0u) : (mag[j] > mag[i] ? 1u : 0u);
            keep |= (ahead < 6u ? 1u : 0u) << i;
        }
        // greedy leftmost windows: positions 0,1 -> window 0; 2,3 -> 0 or 1; 4,5 -> 1 or 2; 6,7 -> 2
        uint32_t g[3] = {0u, 0u, 0u}, f[3] = {0u, 0u, 0u};
#pragma unroll
        for (int pos = 0; pos < 8; ++pos) {
            if (!((keep >> pos) & 1u)) continue;
            const uint32_t c = mag[pos] >= thr ? (((bits[pos] >> 30) & 2u) | 1u) : 0u;
            int w;
            if (pos < 2) w = 0;
            else if (pos < 4) w = f[0] < 2u ? 0 : 1;
            else if (pos < 6) w = f[1] < 2u ? 1 : 2;
            else w = 2;
            const uint32_t rel = static_cast<uint32_t>(pos - 2 * w);
#pragma unroll
            for (int ww = 0; ww < 3; ++ww)
                if (ww == w) {
                    g[ww] |= f[ww] == 0u ? (rel | (c << 4)) : ((rel << 2) | (c << 6));
                    ++f[ww];
                }
        }
        uint8_t *dst = gbw + 3 * b;
        dst[0] = static_cast<uint8_t>(g[0]);
        dst[1] = static_cast<uint8_t>(g[1]);
        dst[2] = static_cast<uint8_t>(g[2]);
    }
}

// tensor-core values and metadata of a canonical 2:4 matrix from its group
// bytes (four groups per thread; k % 16 == 0)
__global__ void __launch_bounds__(256) k_gb_to_mma(const uint8_t *__restrict__ gb, Pack24Args p) {
    const uint32_t n_quads = static_cast<uint32_t>(p.n_groups >> 2);
    const uint32_t stride = gridDim.x * blockDim.x;
    for (uint32_t q = blockIdx.x * blockDim.x + threadIdx.x; q < n_quads; q += stride) {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t *>(gb) + q);
        QuadOut o;
        o.gb = w;
        o.vlo = o.vhi = o.meta = o.mask = o.band = 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t b = (w >> (8 * j)) & 0xffu;
            const uint32_t c0 = (b >> 4) & 3u, c1 = b >> 6;
            const uint32_t v = ((c0 & 2u) * 0x7eu + c0) | (((c1 & 2u) * 0x7eu + c1) << 8);
            if (j < 2) o.vlo |= v << (16 * j);
            else o.vhi |= v << (16 * (j - 2));
            o.meta |= (b & 0xfu) << (4 * j);
        }
        store_quad(p, q, o);
    }
}

cudaError_t launch_pack68(const float *W, int64_t n_out, int64_t k, float eps, float *gamma, uint8_t *gbw,
                          int8_t *vals, uint8_t *meta, uint8_t *dec, uint8_t *mask, void *ws, cudaStream_t s) {
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    uint32_t *thr = reinterpret_cast<uint32_t *>(w8 + kPackWsThrOffset);
    unsigned long long *win = reinterpret_cast<unsigned long long *>(w8 + kPackWsWinOffset);
    unsigned long long *bins = reinterpret_cast<unsigned long long *>(w8 + kPackWsBinsOffset);
    cudaError_t err = cudaMemsetAsync(ws, 0, kPackWsBytes, s);
    if (err != cudaSuccess) return err;
    const int64_t n_el = n_out * k;
    unsigned *counter = reinterpret_cast<unsigned *>(w8 + kPackWsCounterOffset);
    // gamma over the dense matrix, as for 2:4
    k_abs_sum_fast<<<grid_for(n_el / 4, 256, 4), 256, 0, s>>>(reinterpret_cast<const float4 *>(W), n_el / 4, win,
                                                             bins, counter, n_el, eps, gamma, thr);
    k_pack68<<<grid_for(n_el / 8, 256, 8), 256, 0, s>>>(reinterpret_cast<const float4 *>(W), n_el / 8, thr, gbw);
    const int64_t kw = k / 2 * 3;   // window layout width
    if (vals || meta) {
        Pack24Args a;
        a.W = nullptr;
        a.n_groups = n_out * kw / 4;
        a.gpr = kw / 4;
        a.gpr_div = make_fastdiv(static_cast<uint32_t>(kw / 4));
        a.n_out = n_out;
        a.k = kw;
        a.meta_rows = (n_out + 127) / 128 * 128;
        a.thr = nullptr;
        a.gb = nullptr;
        a.vals = reinterpret_cast<uint16_t *>(vals);
        a.meta = meta;
        a.mask = nullptr;
        k_gb_to_mma<<<grid_for(a.n_groups / 4, 256, 8), 256, 0, s>>>(gbw, a);
        if (meta && (a.meta_rows != n_out || (kw % 128) != 0))
            k_meta_pad<<<grid_for(((kw + 127) / 128) * (a.meta_rows - n_out) * 16 + n_out * 16, 256, 4), 256, 0, s>>>(
                meta, n_out, kw, a.meta_rows);
    }
    if (dec)
        k_make_dec<<<grid_for(n_out / 16 * (kw / 64) * 32, 256, 8), 256, 0, s>>>(gbw, n_out, kw,
                                                                                 reinterpret_cast<uint2 *>(dec));
    if (mask) k_mask_nm<<<grid_for(n_el / 8, 256, 8), 256, 0, s>>>(W, n_el / 8, 6, 8, mask);
    return cudaGetLastError();
}

}  // namespace bitnet
