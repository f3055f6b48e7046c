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

__global__ void __launch_bounds__(256) k_abs_sum(const float4 *__restrict__ W, int64_t n4,
                                                 unsigned long long *__restrict__ win,
                                                 unsigned long long *__restrict__ bins) {
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
}

// ---------------------------------------------------------------- finaliser

// value += v * 2^shift on a little-endian array of 32-bit limbs.
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
        const uint64_t s = static_cast<uint64_t>(limb[j]) + a + carry;
        limb[j] = static_cast<uint32_t>(s);
        carry = s >> 32;
    }
}

__global__ void k_finalize_gamma(const unsigned long long *__restrict__ win,
                                 const unsigned long long *__restrict__ bins, int64_t n, float eps,
                                 float *__restrict__ gamma, uint32_t *__restrict__ thr_out) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    constexpr int NL = 12;   // 384 bits
    uint32_t limb[NL];
    for (int j = 0; j < NL; ++j) limb[j] = 0;
    // value is in units of 2^-149: a magnitude with biased exponent e and
    // significand m contributes m * 2^(max(e,1)-1); window entries were
    // pre-shifted by (e - 96), so they carry an extra 2^95.
    for (int e = 0; e < 256; ++e) {
        const uint64_t b = bins[e];
        if (b) limbs_add(limb, NL, b, (e == 0 ? 1 : e) - 1);
    }
    limbs_add(limb, NL, win[0], 95);
    limbs_add(limb, NL, win[1], 95 + 64);

    // nearest fp64: take the top 64 bits, fold everything below into a sticky
    // bit 0, and let the correctly rounded u64 -> f64 conversion round.
    int top = -1;
    for (int j = NL - 1; j >= 0; --j)
        if (limb[j]) {
            top = 32 * j + 31 - __clz(limb[j]);
            break;
        }
    double S = 0.0;
    if (top >= 0) {
        const int low = top - 63;   // bit index of bit 0 of the 64-bit window
        uint64_t w64 = 0;
        bool sticky = false;
        for (int b = 0; b < 64; ++b) {
            const int p = low + b;
            if (p >= 0 && ((limb[p >> 5] >> (p & 31)) & 1u)) w64 |= (1ull << b);
        }
        for (int p = 0; p < low; ++p)
            if ((limb[p >> 5] >> (p & 31)) & 1u) {
                sticky = true;
                break;
            }
        if (sticky) w64 |= 1ull;   // bit 0 lies below the 53-bit rounding position
        const double w = __ull2double_rn(w64);
        // scale by 2^(low - 149); |low - 149| keeps the factor a normal double
        const int ex = low - 149;
        const double scale = __longlong_as_double(static_cast<long long>(1023 + ex) << 52);
        S = w * scale;
    }
    const double mean = __ddiv_rn(S, static_cast<double>(n));
    float g = __double2float_rn(mean);
    g = __fadd_rn(g, eps);
    *gamma = g;

    // smallest t >= 0 with fp32(t / g) > 0.5
    uint32_t t = __float_as_uint(__fmul_rn(g, 0.5f));
    auto pred = [g](uint32_t x) { return __fdiv_rn(__uint_as_float(x), g) > 0.5f; };
    int it = 0;
    if (pred(t)) {
        while (t > 0u && pred(t - 1u) && it < 64) {
            --t;
            ++it;
        }
    } else {
        while (!pred(t) && it < 64) {
            ++t;
            ++it;
        }
    }
    *thr_out = t;
}

// ---------------------------------------------------------------- pass 2 (2:4)

struct Pack24Args {
    const float4 *W;
    int64_t n_groups;    // n_out * k / 4
    int64_t gpr;         // groups per row = k / 4
    int64_t n_out;
    int64_t k;
    int64_t meta_rows;   // rows of one metadata k-block = ceil(n_out/128)*128
    const uint32_t *thr;
    uint8_t *gb;         // [n_out, k/4] or null
    uint16_t *vals;      // [n_out, k/2] int8 pairs or null
    uint8_t *meta;       // blocks of 128 rows x 16 bytes or null
    uint8_t *mask;       // [n_out*k/8] or null
};

__global__ void __launch_bounds__(256) k_pack24(Pack24Args p) {
    const uint32_t thr = *p.thr;
    const int lane = threadIdx.x & 31;
    const int64_t warp_stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    // warp-aligned iteration so that every lane takes part in the shuffles
    for (int64_t base = (static_cast<int64_t>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31));
         base < p.n_groups; base += warp_stride) {
        const int64_t i = base + lane;
        const bool valid = i < p.n_groups;
        uint32_t bits[4] = {0u, 0u, 0u, 0u};
        if (valid) {
            const float4 v = __ldg(p.W + i);
            bits[0] = __float_as_uint(v.x);
            bits[1] = __float_as_uint(v.y);
            bits[2] = __float_as_uint(v.z);
            bits[3] = __float_as_uint(v.w);
        }
        uint32_t mag[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) mag[q] = bits[q] & 0x7fffffffu;   // |w| as ordered integers
        uint32_t keep = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            int before = 0;   // positions ranked ahead of q: larger, or equal and lower
#pragma unroll
            for (int r = 0; r < 4; ++r) before += (mag[r] > mag[q]) || (r < q && mag[r] == mag[q]);
            keep |= (before < 2 ? 1u : 0u) << q;
        }
        const uint32_t i0 = __ffs(keep) - 1;
        const uint32_t i1 = 31 - __clz(keep);
        const uint32_t b0 = bits[i0], b1 = bits[i1];
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
            const int64_t row = i / p.gpr, g = i - row * p.gpr;
            if (p.meta) {
                const int64_t kb = g >> 5;
                const int64_t off = ((kb * p.meta_rows + row) << 4) + ((g & 31) >> 1);
                p.meta[off] = static_cast<uint8_t>(nib | (nib_hi << 4));
            }
            if (p.mask) p.mask[(row * p.k >> 3) + (g >> 1)] = static_cast<uint8_t>(keep | (keep_hi << 4));
        }
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

int num_sms() {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    return sms;
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
    k_abs_sum<<<grid_for(n_el / 4, 256, 8), 256, 0, s>>>(reinterpret_cast<const float4 *>(W), n_el / 4, win, bins);
    k_finalize_gamma<<<1, 32, 0, s>>>(win, bins, n_el, eps, gamma, thr);
    const bool packed = gb || vals || meta || dec;
    if (packed) {
        Pack24Args a;
        a.W = reinterpret_cast<const float4 *>(W);
        a.n_groups = n_el / 4;
        a.gpr = k / 4;
        a.n_out = n_out;
        a.k = k;
        a.meta_rows = (n_out + 127) / 128 * 128;
        a.thr = thr;
        a.gb = gb;
        a.vals = reinterpret_cast<uint16_t *>(vals);
        a.meta = meta;
        a.mask = (n == 2 && m == 4) ? mask : nullptr;
        k_pack24<<<grid_for(a.n_groups, 256, 8), 256, 0, s>>>(a);
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

}  // namespace bitnet
