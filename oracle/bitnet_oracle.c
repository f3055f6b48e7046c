/*
 * Plain CPU oracle for the Sparse-BitNet BitLinear hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or helper with the CUDA
 * library: it is written straight from the definitions, slow and literal.
 *
 * Sources of the definitions (cited by page title and section):
 *  [P5] "BitNet b1.58: Ternary Weights for 1.58-bit LLMs", section "The
 *       mechanism": absmean scale gamma over the whole weight matrix, divide
 *       by gamma, round, clip to {-1,0,1}; activations scaled per token to the
 *       symmetric range [-Q_b, Q_b] with no zero-point; the ternary product is
 *       signed accumulation (add, subtract or skip).
 *  [P4] "Sparse-BitNet" (gist.science technical summary), section 2
 *       "Methodologie", "Kerncomponenten": the N:M mask is chosen from the
 *       magnitudes of the master weights (before quantisation), the forward
 *       pass quantises to ternary and then applies the mask; section 2
 *       "Training Strategie": the mask is recomputed every step and the
 *       straight-through estimator passes gradients through quantiser and mask.
 *  [P4-1] same page, section 1 "Het Probleem": N:M means at most N of every M
 *       consecutive weights are non-zero (2:4: at most 2 of 4).
 *
 * Readings where the pages are silent (the equations of [P5] were lost):
 *  - gamma = fp32(fp64_rn(exact sum |W|) / n) + eps, eps passed in.
 *  - round() is round-half-to-even (rintf); codes are clipped to [-1, 1].
 *  - Q_b = 127; scale s = 127 / max(absmax, eps) in fp32; q = rint(x * s).
 *  - top-N ties go to the lower position; +0.0 and -0.0 tie.
 *  - a kept weight whose code is 0 still occupies its slot in the packing.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fopenmp -shared -fPIC.
 * -ffp-contract=off keeps every product separately rounded (no FMA).
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* threads                                                                   */
/* ------------------------------------------------------------------------ */

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Exact sum of |W|, rounded once to fp64.  [P5] "The mechanism": the scale   */
/* is the mean absolute value of the whole matrix.                           */
/*                                                                           */
/* Every finite fp32 x is an integer multiple of 2^-149:                     */
/*   |x| = m * 2^(e-1) * 2^-149, e = max(biased exponent, 1),                */
/*   m = 24-bit significand (hidden bit only for normals).                   */
/* The sum is kept as a big unsigned integer in units of 2^-149 (base-2^32   */
/* limbs), then rounded to the nearest fp64, ties to even.                   */
/* ------------------------------------------------------------------------ */

#define ORACLE_LIMBS 12   /* 384 bits: 2^253 * 2^24 * 2^64 fits with room */

static void big_add_shifted(uint32_t *big, uint64_t v, int shift) {
    /* big += v << shift */
    int limb = shift / 32, off = shift % 32;
    /* spread v << off over up to three 32-bit limbs */
    uint64_t lo = (off == 0) ? v : (v << off);
    uint64_t hi = (off == 0) ? 0 : (v >> (64 - off));
    uint32_t parts[4] = {(uint32_t)lo, (uint32_t)(lo >> 32), (uint32_t)hi, (uint32_t)(hi >> 32)};
    uint64_t carry = 0;
    for (int i = 0; limb + i < ORACLE_LIMBS; ++i) {
        uint64_t add = (i < 4) ? parts[i] : 0;
        if (i >= 4 && carry == 0) break;
        uint64_t s = (uint64_t)big[limb + i] + add + carry;
        big[limb + i] = (uint32_t)s;
        carry = s >> 32;
    }
}

static double big_to_double_rn(const uint32_t *big) {
    /* value = big * 2^-149, rounded to nearest fp64, ties to even */
    int top = -1;
    for (int i = ORACLE_LIMBS - 1; i >= 0 && top < 0; --i)
        if (big[i]) {
            for (int b = 31; b >= 0; --b)
                if ((big[i] >> b) & 1u) { top = i * 32 + b; break; }
        }
    if (top < 0) return 0.0;
#define BIT(p) ((p) < 0 ? 0u : ((big[(p) / 32] >> ((p) % 32)) & 1u))
    uint64_t mant = 0;
    int lsb = top - 52;               /* position of the last kept bit */
    for (int p = top; p >= lsb && p >= 0; --p) mant = (mant << 1) | BIT(p);
    if (lsb < 0) {                    /* fewer than 53 bits: exact */
        return ldexp((double)mant, -149);
    }
    unsigned round_bit = BIT(lsb - 1);
    unsigned sticky = 0;
    for (int p = lsb - 2; p >= 0; --p) if (BIT(p)) { sticky = 1; break; }
#undef BIT
    if (round_bit && (sticky || (mant & 1u))) {
        mant += 1;
        if (mant == (1ull << 53)) { mant >>= 1; lsb += 1; }
    }
    return ldexp((double)mant, lsb - 149);
}

double oracle_abs_sum(const float *W, int64_t n) {
    uint32_t big[ORACLE_LIMBS];
    memset(big, 0, sizeof big);
    for (int64_t i = 0; i < n; ++i) {
        uint32_t bits;
        memcpy(&bits, &W[i], 4);
        bits &= 0x7fffffffu;                       /* |x| */
        uint32_t e = bits >> 23, frac = bits & 0x7fffffu;
        uint64_t m = (e == 0) ? frac : (frac | 0x800000u);
        int shift = (e == 0 ? 1 : (int)e) - 1;
        if (m) big_add_shifted(big, m, shift);
    }
    return big_to_double_rn(big);
}

/* gamma = fp32(fp64 sum / n) + eps, the last addition in fp32. */
float oracle_gamma(const float *W, int64_t n, float eps) {
    double s = oracle_abs_sum(W, n);
    double mean = s / (double)n;
    float g = (float)mean;
    g = g + eps;
    return g;
}

/* ------------------------------------------------------------------------ */
/* N:M mask from master magnitudes.  [P4] "Kerncomponenten": the mask keeps  */
/* the N largest |W| in every group of M consecutive weights (along K), and  */
/* is taken on the masters, before quantisation.                             */
/* keep[r*k + c] = 1 for kept weights, 0 for dropped ones.                   */
/* ------------------------------------------------------------------------ */

void oracle_mask_nm(const float *W, int64_t rows, int64_t k, int n, int m, uint8_t *keep) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t g = 0; g < k / m; ++g) {
            const float *w = W + r * k + g * m;
            uint8_t *kp = keep + r * k + g * m;
            for (int p = 0; p < m; ++p) {
                /* rank of p: how many positions come before it in the order
                 * (|w| descending, position ascending) */
                float ap = fabsf(w[p]);
                int rank = 0;
                for (int q = 0; q < m; ++q) {
                    float aq = fabsf(w[q]);
                    if (aq > ap || (aq == ap && q < p)) rank++;
                }
                kp[p] = (uint8_t)(rank < n);
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Absmean ternarisation.  [P5] "The mechanism": divide by gamma, round, clip */
/* to [-1, 1].  Applied to every weight; the mask is applied afterwards      */
/* ([P4] "Forward Pass": quantise, then mask).                               */
/* ------------------------------------------------------------------------ */

void oracle_ternary(const float *W, int64_t count, float gamma, int8_t *q) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        float v = W[i] / gamma;
        float r = rintf(v);
        if (r > 1.0f) r = 1.0f;
        if (r < -1.0f) r = -1.0f;
        q[i] = (int8_t)r;
    }
}

/* Wq = keep * Wt (the masked ternary matrix, dense int8 {-1,0,1}). */
void oracle_apply_mask(const int8_t *wt, const uint8_t *keep, int64_t count, int8_t *wq) {
    for (int64_t i = 0; i < count; ++i) wq[i] = keep[i] ? wt[i] : 0;
}

/* ------------------------------------------------------------------------ */
/* Canonical 2:4 group byte (a storage format; the pages give none):         */
/*   bits 0-1 idx0, bits 2-3 idx1 (idx0 < idx1, the two kept positions),     */
/*   bits 4-5 code of idx0, bits 6-7 code of idx1; code 0 -> 00, +1 -> 01,   */
/*   -1 -> 11.                                                               */
/* ------------------------------------------------------------------------ */

static unsigned code2(int v) { return v == 0 ? 0u : (v > 0 ? 1u : 3u); }

int oracle_pack_24(const int8_t *wq, const uint8_t *keep, int64_t rows, int64_t k, uint8_t *gb) {
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t g = 0; g < k / 4; ++g) {
            const uint8_t *kp = keep + r * k + 4 * g;
            const int8_t *vp = wq + r * k + 4 * g;
            int idx[2], c = 0;
            for (int p = 0; p < 4; ++p) if (kp[p]) { if (c < 2) idx[c] = p; c++; }
            if (c != 2) return -1;                 /* not a 2:4 mask */
            gb[r * (k / 4) + g] = (uint8_t)(idx[0] | (idx[1] << 2) |
                                  (code2(vp[idx[0]]) << 4) | (code2(vp[idx[1]]) << 6));
        }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Per-token absmax int8 quantisation.  [P5] "The mechanism" (Activations):   */
/* each token scaled to [-Q_b, Q_b], symmetric, no zero-point; Q_b = 127.    */
/* a[t] = max(max_k |x|, eps); s = 127 / a[t]; q = clamp(rint(x*s), +-127).  */
/* ------------------------------------------------------------------------ */

void oracle_quant_act(const float *X, int64_t T, int64_t K, float eps, int8_t *Xq, float *a) {
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const float *x = X + t * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) { float v = fabsf(x[k]); if (v > amax) amax = v; }
        float at = amax > eps ? amax : eps;
        float s = 127.0f / at;
        for (int64_t k = 0; k < K; ++k) {
            float p = x[k] * s;
            float r = rintf(p);
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            Xq[t * K + k] = (int8_t)r;
        }
        a[t] = at;
    }
}

/* ------------------------------------------------------------------------ */
/* Integer product.  [P5] "The mechanism": with ternary weights each output  */
/* is a signed sum of activations.  acc[t, n] = sum_k Xq[t,k] * Wq[n,k],     */
/* accumulated in int64; returns -1 if any result leaves the int32 range.    */
/* ------------------------------------------------------------------------ */

int oracle_gemm_i32(const int8_t *Xq, const int8_t *Wq, int64_t T, int64_t N, int64_t K, int32_t *acc) {
    int bad = 0;
    /* every (t, n) is its own sum in k order: the threads share the outputs */
    #pragma omp parallel for collapse(2) schedule(static) reduction(|:bad)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t n = 0; n < N; ++n) {
            int64_t s = 0;
            const int8_t *x = Xq + t * K, *w = Wq + n * K;
            for (int64_t k = 0; k < K; ++k) s += (int64_t)x[k] * (int64_t)w[k];
            if (s > INT32_MAX || s < INT32_MIN) bad = 1;
            acc[t * N + n] = (int32_t)s;
        }
    return bad ? -1 : 0;
}

/* Dequantisation: y = fp32(acc) * ((gamma * a[t]) / 127), each step in fp32. */
void oracle_dequant(const int32_t *acc, const float *a, float gamma, int64_t T, int64_t N, float *Y) {
    for (int64_t t = 0; t < T; ++t) {
        float scale = (gamma * a[t]) / 127.0f;
        for (int64_t n = 0; n < N; ++n) Y[t * N + n] = (float)acc[t * N + n] * scale;
    }
}

/* ------------------------------------------------------------------------ */
/* Input gradient under the straight-through estimator.  [P4] "Training      */
/* Strategie" (dual STE): the quantiser and the mask pass the gradient       */
/* through, so dX = dY * (gamma * Wq), with Wq the masked ternary matrix.    */
/* Computed in fp64 from fp32-widened inputs.  Also returns, per output,     */
/* sum |dY * Wq| * gamma, the scale of an error bound for fp32 summation.    */
/* ------------------------------------------------------------------------ */

void oracle_dgrad(const float *dY, const int8_t *Wq, float gamma, int64_t T, int64_t N, int64_t K,
                  double *dX, double *absdX) {
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t k = 0; k < K; ++k) {
            double s = 0.0, sa = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                double v = (double)dY[t * N + n] * (double)Wq[n * K + k];
                s += v;
                sa += fabs(v);
            }
            dX[t * K + k] = s * (double)gamma;
            if (absdX) absdX[t * K + k] = sa * (double)gamma;
        }
}

/* ------------------------------------------------------------------------ */
/* Whole forward of one Sparse-BitLinear (config-sized convenience).         */
/* Masks (2:4 on this path), ternarises, applies the mask, packs, quantises  */
/* the activations, multiplies and dequantises.                              */
/* ------------------------------------------------------------------------ */

int oracle_forward(const float *W, int64_t N, int64_t K, const float *X, int64_t T,
                   float eps_w, float eps_a,
                   float *gamma_out, uint8_t *keep, int8_t *wq, uint8_t *gb,
                   int8_t *Xq, float *a, int32_t *acc, float *Y) {
    float g = oracle_gamma(W, N * K, eps_w);
    *gamma_out = g;
    oracle_mask_nm(W, N, K, 2, 4, keep);
    oracle_ternary(W, N * K, g, wq);
    oracle_apply_mask(wq, keep, N * K, wq);
    if (gb && oracle_pack_24(wq, keep, N, K, gb) != 0) return -1;
    oracle_quant_act(X, T, K, eps_a, Xq, a);
    if (oracle_gemm_i32(Xq, wq, T, N, K, acc) != 0) return -2;
    oracle_dequant(acc, a, g, T, N, Y);
    return 0;
}
