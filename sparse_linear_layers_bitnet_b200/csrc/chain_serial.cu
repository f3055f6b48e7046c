// Decode chain for dependent projections: quantise + sparse ternary GEMV of a
// sequence of projections in one persistent launch (sm_100a), for chains in
// which a projection waits for the one before it (its input is the previous
// output, through the caller's own steps).
//
// What each projection computes is the BitLinear forward of "BitNet b1.58:
// Ternary Weights for 1.58-bit LLMs", section "The mechanism" (per-token
// absmax int8 activations, ternary weights, integer sums, one rescale) with
// the 2:4 mask of "Sparse-BitNet" (gist.science), section 2
// "Kerncomponenten"; the numbers are those of bitnet_quant_act followed by
// bitnet_sparse_linear, bit for bit.
//
// Such a chain is bound by the latency of each projection, not by bandwidth:
// every CTA must see all of projection j - 1's output before it can quantise
// projection j's input.  So this kernel keeps the path from one projection to
// the next short: the sixteen consumer warps of every SM quantise the
// activation row together (all of them wait, read the row through L2 and
// form the codes), run their records and write their outputs, with no hand-over
// between warp roles.  Only the weight stream runs ahead:
//  * a producer warp streams the CTA's share of every projection's packed
//    weights (a contiguous byte range of the decode layout) into a ring of
//    64, 32 or 16 KB shared-memory stages with bulk asynchronous copies;
//  * sixteen consumer warps, per projection: wait until every CTA has finished
//    the previous projection (a grid-wide counter, acquire loads, bounded
//    wait), read the T activation rows from L2, form the per-token scales and
//    int8 codes in shared memory, run one m16n8k64 sparse MMA per 64-k tile
//    of each weight record in the ring, sum the partial tiles in shared
//    memory, write Y, and count themselves done (release add).
// Chains of independent projections take the pipelined kernel of chain.cu.
//
// Two instantiations per activation type: any T <= 8, and T = 1 with the token
// count folded to a constant (no per-token selects or chunk-to-token division
// in the quantisation).
//
// All waits are bounded (2 s): a stage that never fills, a counter that never
// reaches the grid size or an abort raised by another CTA ends the kernel
// with the timeout bit in the status word; outstanding copies are waited for
// (bounded) before the CTA exits.
#include "../../include/bitnet_sparse.h"
#include "common.cuh"
#include "frag.cuh"
#include "kernels.h"

namespace bitnet {
namespace serial {

constexpr int kChainConsumerWarps = 16;
constexpr int kChainConsumers = kChainConsumerWarps * 32;
constexpr int kChainThreads = kChainConsumers + 32;
constexpr int kChainMaxStages = 16;
constexpr size_t kSerialMaxSmem = 227 * 1024 - 1024;   // dynamic shared memory (static use < 1 KB)

struct ChainParams {
    ChainOpDev op[kChainMaxOps];
    int32_t n_ops, T, x_bf16, y_bf16, ns, kmax;
    uint32_t stage_bytes;   // ring stage size: 16, 32 or 64 KB (a multiple of 256)
    float eps;
    uint32_t *counters;   // [n_ops], zero at launch
    uint32_t *abort;      // grid-wide abort word, zero at launch
    uint32_t *status;
};

// Row tiles [t0, t1) of projection j for this CTA.  The CTA's share index v
// is its block index rotated by 61 j; share v is [v R / G, (v + 1) R / G).
// Share G - 1 is never empty when R >= 1.
// 32-bit arithmetic: v R < 2^31 since R <= 32 G (checked on the host) and G is
// the number of SMs.
__device__ __forceinline__ int chain_tiles(int j, int rows16, int &t0, int &t1) {
    const uint32_t G = gridDim.x;
    uint32_t v = blockIdx.x + (static_cast<uint32_t>(j) * 61u) % G;
    if (v >= G) v -= G;
    t0 = static_cast<int>((v * static_cast<uint32_t>(rows16)) / G);
    t1 = static_cast<int>(((v + 1u) * static_cast<uint32_t>(rows16)) / G);
    return static_cast<int>(v);
}

__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kChainConsumers) : "memory"); }

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Spins (bounded by limit_ns) until *ctr >= target.  On a timeout or a grid
// abort it sets the CTA's abort flag (and, on a timeout, the grid abort word
// and status).
__device__ bool wait_counter(const uint32_t *ctr, uint32_t target, const ChainParams &p, volatile int *s_abort,
                             uint64_t limit_ns = kWaitLimitNs) {
    if (ld_acquire(ctr) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        __nanosleep(32);
        if (ld_acquire(ctr) >= target) return true;
        if (*reinterpret_cast<volatile uint32_t *>(p.abort) != 0u) {
            *s_abort = 1;
            return false;
        }
        if (globaltimer_ns() - t0 > limit_ns) {
            *s_abort = 1;
            atomicOr(p.status, kStatusTimeout);
            atomicExch(p.abort, 1u);
            return false;
        }
    }
}

// Producer's wait for a free stage: the thread is suspended in the barrier
// (try_wait with a suspend-time hint) until the phase completes, instead of
// spinning and taking issue slots from the consumer warps.  Bounded like
// mbar_wait_bounded.
__device__ bool mbar_wait_sleep(uint64_t *bar, uint32_t parity, volatile int *abort, uint32_t *status) {
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
            : "memory");
        if (ok) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort = 1;
            atomicOr(status, kStatusTimeout);
            return false;
        }
    }
}

// Consumer's wait for a filled stage: suspended in the barrier (short hint)
// rather than spinning; bounded like mbar_wait_bounded.
__device__ __forceinline__ bool mbar_wait_full(uint64_t *bar, uint32_t parity, volatile int *abort, uint32_t *status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity), "r"(2000u)
            : "memory");
        if (ok) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort = 1;
            atomicOr(status, kStatusTimeout);
            return false;
        }
    }
}

// Wait that ignores the abort flag, up to a deadline (for draining copies in flight).
__device__ bool mbar_wait_until(uint64_t *bar, uint32_t parity, uint64_t deadline_ns) {
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() > deadline_ns) return false;
    }
    return true;
}

// Barrier of the consumer warps (hardware barrier 2; plain consumer barriers
// use 1) that also ORs a predicate over them, so that every consumer takes the
// same branch after it.
__device__ __forceinline__ bool consumer_sync_or(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 2, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(v ? 1u : 0u), "n"(kChainConsumers)
        : "memory");
    return r != 0;
}

// adds a row tile's partial sums (four accumulators) into the shared sums and clears them
__device__ __forceinline__ void chain_flush(int *s_acc, int tile, int lane, int (&acc)[4][4]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        atomicAdd(&s_acc[(tile * 32 + lane) * 4 + q], acc[0][q] + acc[1][q] + acc[2][q] + acc[3][q]);
        acc[0][q] = acc[1][q] = acc[2][q] = acc[3][q] = 0;
    }
}

template <bool BF16>
struct ChainChunk {
    static constexpr int kElems = BF16 ? 8 : 4;
    uint4 raw;
    __device__ __forceinline__ float get(int j) const {
        const int i = BF16 ? (j >> 1) : j;
        const uint32_t w = i == 0 ? raw.x : (i == 1 ? raw.y : (i == 2 ? raw.z : raw.w));
        if (BF16) return __uint_as_float((j & 1) ? (w & 0xffff0000u) : (w << 16));
        return __uint_as_float(w);
    }
    __device__ __forceinline__ float absmax() const {
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < kElems; ++j) m = fmaxf(m, fabsf(get(j)));
        return m;
    }
    // Codes of the chunk's elements e0 .. e0 + kElems - 1 of a token row whose
    // shared copy starts at row.  Within each 64-element k-tile the sixteen
    // 4-byte words are stored transposed (word 4 j + q at 4 q + j), so that the
    // 16 bytes lane q of a token takes as its m16n8k64 B fragment (k = 4 q + 16 j
    // + 0..3, j = 0..3) are contiguous.
    __device__ __forceinline__ void store_codes(int8_t *row, int e0, float s) const {
        int8_t *tile = row + (e0 & ~63);
        const int u0 = (e0 & 63) >> 2;   // first word within the tile
        if constexpr (BF16) {
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) v[j] = get(j);
            const uint2 q = codes8_fast(v, s);
            const int u1 = u0 + 1;
            *reinterpret_cast<uint32_t *>(tile + 4 * (4 * (u0 & 3) + (u0 >> 2))) = q.x;
            *reinterpret_cast<uint32_t *>(tile + 4 * (4 * (u1 & 3) + (u1 >> 2))) = q.y;
        } else {
            *reinterpret_cast<uint32_t *>(tile + 4 * (4 * (u0 & 3) + (u0 >> 2))) =
                codes4_fast(get(0), get(1), get(2), get(3), s);
        }
    }
};

// Row pitch of the shared int8 activations: k + 64 or k + 128, whichever is
// 64 mod 128 bytes, so that the two token rows one quarter-warp reads in a
// 16-byte-per-lane load fall in disjoint banks.
__device__ __host__ __forceinline__ int64_t chain_pitch(int64_t k) { return k + 64 + (k & 64); }

// Per-token absmax, scales and int8 codes of one projection's activations
// (same arithmetic as bitnet_quant_act) into shared memory, row pitch
// chain_pitch(k), each 64-k tile in fragment order (see store_codes).
// X is read through L2 only (ld.global.cg): it may have been written by other
// SMs earlier in this kernel.  Thread ctid takes the flattened 16-byte chunks
// c = ctid + 512 u.  The first kChainKeep of them are loaded together (all in
// flight at once) and stay in registers for the second pass; any further ones
// are loaded kChainKeep at a time in each pass.  Two is the measured best
// (decode step at T = 1: 0.533 ms against 0.550 with three and 0.557 with four
// cached chunks; T = 8: 1.03, 0.98 and 0.98 ms): a larger cache costs the
// one- and two-chunk rows of T = 1 more than it saves at T = 8.  A chunk's token is
// floor((c + 1/2) / cpr) through a float reciprocal: c / cpr <= 8 and c < 2^20,
// so the rounding error is far below the 1 / (2 cpr) margin.
// s_inv[t] = 127 / a_t and s_scale[t] = (gamma a_t) / 127 are formed once per
// token.
constexpr int kChainKeep = 2;

template <int TM>
__device__ __forceinline__ void chain_chunk_pos(int c, int cpr, float inv_cpr, int &t, int &i) {
    if (TM == 1) {   // one token: every chunk is in row 0
        t = 0;
        i = c;
        return;
    }
    t = __float2int_rz((static_cast<float>(c) + 0.5f) * inv_cpr);
    i = c - t * cpr;
}

// TM: the most tokens the instantiation handles (1, or 8 for any T <= 8).
template <bool BF16, int TM>
__device__ void chain_quantise(const uint4 *__restrict__ X, int T, int k, float eps, float gamma, int8_t *s_xq,
                               float (*s_red)[8], float *s_amax, float *s_inv, float *s_scale, int ctid) {
    using C = ChainChunk<BF16>;
    const int cpr = k / C::kElems;             // chunks per token row (>= 8)
    const int nchunk = T * cpr;
    const float inv_cpr = 1.0f / static_cast<float>(cpr);
    const int warp = ctid >> 5, lane = ctid & 31;
    float m[TM];
#pragma unroll
    for (int t = 0; t < TM; ++t) m[t] = 0.0f;
    C keep[kChainKeep];
#pragma unroll
    for (int u = 0; u < kChainKeep; ++u) {
        const int c = ctid + u * kChainConsumers;
        keep[u].raw = c < nchunk ? __ldcg(X + c) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kChainKeep; ++u) {
        const int c = ctid + u * kChainConsumers;
        if (c < nchunk) {
            int t, i;
            chain_chunk_pos<TM>(c, cpr, inv_cpr, t, i);
            const float ma = keep[u].absmax();
#pragma unroll
            for (int tt = 0; tt < TM; ++tt)
                if (tt == t) m[tt] = fmaxf(m[tt], ma);
        }
    }
    // chunks beyond the register cache (long rows of several tokens): kChainKeep loads in flight per round
    for (int c0 = ctid + kChainKeep * kChainConsumers; c0 < nchunk; c0 += kChainKeep * kChainConsumers) {
        C v[kChainKeep];
#pragma unroll
        for (int u = 0; u < kChainKeep; ++u) {
            const int c = c0 + u * kChainConsumers;
            if (c < nchunk) v[u].raw = __ldcg(X + c);
        }
#pragma unroll
        for (int u = 0; u < kChainKeep; ++u) {
            const int c = c0 + u * kChainConsumers;
            if (c < nchunk) {
                int t, i;
                chain_chunk_pos<TM>(c, cpr, inv_cpr, t, i);
                const float ma = v[u].absmax();
#pragma unroll
                for (int tt = 0; tt < TM; ++tt)
                    if (tt == t) m[tt] = fmaxf(m[tt], ma);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < TM; ++t) {
        if (t < T) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m[t] = fmaxf(m[t], __shfl_xor_sync(0xffffffffu, m[t], o));
        }
    }
    if (lane == 0) {
#pragma unroll
        for (int t = 0; t < TM; ++t) s_red[warp][t] = m[t];
    }
    consumer_sync();
    if (ctid < T) {
        float v = 0.0f;
#pragma unroll
        for (int q = 0; q < kChainConsumerWarps; ++q) v = fmaxf(v, s_red[q][ctid]);
        v = v > eps ? v : eps;
        s_amax[ctid] = v;
        s_inv[ctid] = __fdiv_rn(127.0f, v);
        s_scale[ctid] = __fdiv_rn(__fmul_rn(gamma, v), 127.0f);
    }
    consumer_sync();
    const int pitch = chain_pitch(k);
#pragma unroll
    for (int u = 0; u < kChainKeep; ++u) {
        const int c = ctid + u * kChainConsumers;
        if (c < nchunk) {
            int t, i;
            chain_chunk_pos<TM>(c, cpr, inv_cpr, t, i);
            keep[u].store_codes(s_xq + t * pitch, i * C::kElems, s_inv[t]);
        }
    }
    for (int c0 = ctid + kChainKeep * kChainConsumers; c0 < nchunk; c0 += kChainKeep * kChainConsumers) {
        C v[kChainKeep];
#pragma unroll
        for (int u = 0; u < kChainKeep; ++u) {
            const int c = c0 + u * kChainConsumers;
            if (c < nchunk) v[u].raw = __ldcg(X + c);
        }
#pragma unroll
        for (int u = 0; u < kChainKeep; ++u) {
            const int c = c0 + u * kChainConsumers;
            if (c < nchunk) {
                int t, i;
                chain_chunk_pos<TM>(c, cpr, inv_cpr, t, i);
                v[u].store_codes(s_xq + t * pitch, i * C::kElems, s_inv[t]);
            }
        }
    }
}

template <bool XBF16, int TM>
__global__ void __launch_bounds__(kChainThreads, 1) k_decode_chain_serial(const __grid_constant__ ChainParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t s_full[kChainMaxStages], s_empty[kChainMaxStages];
    __shared__ float s_red[kChainConsumerWarps][8];
    __shared__ float s_amax[8], s_inv[8], s_scale[8];
    __shared__ int s_abort;
    const int tid = threadIdx.x;
    const int ns = p.ns;
    const int T = TM == 1 ? 1 : p.T;   // a one-token instantiation folds T away
    const uint32_t G = gridDim.x;
    // dynamic shared memory: ring [ns][16 KB] | partial sums [kChainMaxTiles][32][4] int | int8 rows
    uint8_t *ring = smem;
    const uint32_t stage_bytes = p.stage_bytes;
    int *s_acc = reinterpret_cast<int *>(smem + static_cast<size_t>(ns) * stage_bytes);
    int8_t *s_xq = reinterpret_cast<int8_t *>(s_acc + kChainMaxTiles * 128);

    for (int i = tid; i < kChainMaxTiles * 128; i += kChainThreads) s_acc[i] = 0;
    if (tid == 0) {
        s_abort = 0;
        for (int s = 0; s < ns; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&s_empty[s], kChainConsumerWarps);
        }
        fence_mbar_init();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();

    if (tid >= kChainConsumers) {
        // ------------------------------------------------------------ producer
        if (tid != kChainConsumers) return;
        uint32_t it = 0, ps = 0, pph = 0;   // stages issued; slot it % ns; parity of fill round it / ns
        bool ok = true;
        for (int j = 0; j < p.n_ops && ok; ++j) {
            const ChainOpDev &op = p.op[j];
            int t0, t1;
            chain_tiles(j, op.n_out >> 4, t0, t1);
            const uint32_t tile_bytes = static_cast<uint32_t>(op.k >> 6) * 256u;
            const uint32_t bytes = static_cast<uint32_t>(t1 - t0) * tile_bytes;
            const uint8_t *src = op.dec + static_cast<size_t>(t0) * tile_bytes;
            // Warm L2 with this CTA's slice of the projection's activation rows
            // (128-byte lines b, b + G, ...).  Only a cache hint: L2 is the
            // coherence point, so a line prefetched before an earlier projection
            // writes it is updated by that write.
            {
                const size_t xbytes = static_cast<size_t>(p.T) * static_cast<size_t>(op.k) * (p.x_bf16 ? 2u : 4u);
                for (size_t l = static_cast<size_t>(blockIdx.x) * 128; l < xbytes; l += static_cast<size_t>(gridDim.x) * 128)
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(static_cast<const uint8_t *>(op.X) + l));
            }
            for (uint32_t off = 0; off < bytes; off += stage_bytes, ++it) {
                // reuse of slot ps in round r >= 1 waits for the consumers' release of round r - 1
                if (it >= static_cast<uint32_t>(ns) && !mbar_wait_sleep(&s_empty[ps], pph ^ 1u, &s_abort, p.status)) {
                    ok = false;
                    break;
                }
                const uint32_t n = (bytes - off) < stage_bytes ? (bytes - off) : stage_bytes;
                mbar_arrive_expect_tx(&s_full[ps], n);
                bulk_load(ring + static_cast<size_t>(ps) * stage_bytes, src + off, n, &s_full[ps]);
                if (++ps == static_cast<uint32_t>(ns)) {
                    ps = 0;
                    pph ^= 1u;
                }
            }
        }
        // drain: every issued stage must have landed before the CTA may exit
        // (earlier stages were consumed before their slot was reused)
        const uint32_t first = it > static_cast<uint32_t>(ns) ? it - ns : 0u;
        const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
        for (uint32_t q = first; q < it; ++q) mbar_wait_until(&s_full[q % ns], (q / ns) & 1u, deadline);
        return;
    }

    // ---------------------------------------------------------------- consumers
    // Every branch that can differ between consumer threads (an expired wait,
    // an abort) is decided through consumer_sync_or or a warp vote, so that the
    // consumer barriers never miss a thread.
    const int ctid = tid;
    const int warp = ctid >> 5, lane = ctid & 31;
    uint32_t cs = 0, cph = 0;   // ring slot of the next stage and the parity of its fill round
    for (int j = 0; j < p.n_ops; ++j) {
        const ChainOpDev &op = p.op[j];
        int t0, t1;
        const int share = chain_tiles(j, op.n_out >> 4, t0, t1);
        const int ntile = t1 - t0;
        const int ktiles = op.k >> 6;
        const uint32_t bytes = static_cast<uint32_t>(ntile) * static_cast<uint32_t>(ktiles) * 256u;
        // gamma belongs to the packed weights: read before the wait
        const float gamma = ntile > 0 ? __ldg(op.gamma) : 0.0f;
        // 1. every CTA has finished the previous projection
        if (j > 0 && op.wait_prev) {
            bool bad = false;
            if (ctid == 0) bad = !wait_counter(&p.counters[j - 1], G, p, &s_abort);
            if (consumer_sync_or(bad || s_abort != 0)) break;
        }
        if (ntile > 0) {
            // 2. int8 activations of this projection
            chain_quantise<XBF16, TM>(static_cast<const uint4 *>(op.X), T, op.k, p.eps, gamma, s_xq, s_red, s_amax, s_inv,
                                  s_scale, ctid);
            consumer_sync();
            // 3. weight records from the ring: in each stage, warp w takes the
            //    contiguous records [w n / 16, (w + 1) n / 16).  Lane l holds the
            //    B fragment of token l / 4 (zero for tokens >= T): the 16 bytes
            //    lane l % 4 needs of each 64-k tile sit contiguously in the
            //    shared row (fragment order), one 16-byte load per record.
            const int bn = lane >> 2;
            const bool has_b = bn < T;
            const uint4 *b_src =
                reinterpret_cast<const uint4 *>(s_xq + static_cast<int64_t>(has_b ? bn : 0) * chain_pitch(op.k)) +
                (lane & 3);
            int cur = -1;
            int acc[4][4] = {};   // partial sums of the current row tile, one accumulator per record slot
            bool failed = false;
            const float inv_kt = 1.0f / static_cast<float>(ktiles);
            for (uint32_t off = 0; off < bytes; off += stage_bytes) {
                const uint32_t s = cs;
                const bool ok = mbar_wait_full(&s_full[s], cph, &s_abort, p.status);
                if (++cs == static_cast<uint32_t>(ns)) {
                    cs = 0;
                    cph ^= 1u;
                }
                if (!__all_sync(0xffffffffu, ok)) {
                    failed = true;
                    break;
                }
                const int nrec = static_cast<int>(((bytes - off) < stage_bytes ? (bytes - off) : stage_bytes) >> 8);
                const int i0 = (warp * nrec) / kChainConsumerWarps, i1 = ((warp + 1) * nrec) / kChainConsumerWarps;
                if (i0 < i1) {
                    const int r0 = static_cast<int>(off >> 8) + i0;
                    // r0 / ktiles through the reciprocal (r0 < 2^24: off by at most one, corrected)
                    int tile = __float2int_rz(static_cast<float>(r0) * inv_kt);
                    int kt = r0 - tile * ktiles;
                    if (kt < 0) {
                        --tile;
                        kt += ktiles;
                    } else if (kt >= ktiles) {
                        ++tile;
                        kt -= ktiles;
                    }
                    const uint2 *rec = reinterpret_cast<const uint2 *>(ring + static_cast<size_t>(s) * stage_bytes) + lane;
                    int i = i0;
                    while (i < i1) {
                        if (tile != cur) {
                            if (cur >= 0) chain_flush(s_acc, cur, lane, acc);
                            cur = tile;
                        }
                        if (i + 4 <= i1 && kt + 4 <= ktiles) {
                            // four records of one row tile: all loads first, then the MMAs
                            uint2 w[4];
                            uint32_t bf[4][4];
#pragma unroll
                            for (int u = 0; u < 4; ++u) w[u] = rec[(i + u) * 32];
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                const uint4 v = has_b ? b_src[(kt + u) * 4] : make_uint4(0u, 0u, 0u, 0u);
                                bf[u][0] = v.x;
                                bf[u][1] = v.y;
                                bf[u][2] = v.z;
                                bf[u][3] = v.w;
                            }
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                uint32_t a4[4];
#pragma unroll
                                for (int r = 0; r < 4; ++r) a4[r] = expand_codes(w[u].x, r);
                                mma_sp_m16n8k64(acc[u], a4, bf[u], w[u].y);
                            }
                            i += 4;
                            kt += 4;
                        } else {
                            const uint2 w = rec[i * 32];
                            uint32_t bf[4], a4[4];
                            const uint4 v = has_b ? b_src[kt * 4] : make_uint4(0u, 0u, 0u, 0u);
                            bf[0] = v.x;
                            bf[1] = v.y;
                            bf[2] = v.z;
                            bf[3] = v.w;
#pragma unroll
                            for (int r = 0; r < 4; ++r) a4[r] = expand_codes(w.x, r);
                            mma_sp_m16n8k64(acc[0], a4, bf, w.y);
                            i += 1;
                            kt += 1;
                        }
                        if (kt == ktiles) {
                            kt = 0;
                            ++tile;
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_empty[s]);
            }
            if (cur >= 0) chain_flush(s_acc, cur, lane, acc);
            if (consumer_sync_or(failed || s_abort != 0)) break;
            // 4. dequantise and store this CTA's rows; clear the partial sums
            for (int e = ctid; e < ntile * 128; e += kChainConsumers) {
                const int tl = e >> 7, ln = (e >> 2) & 31, q = e & 3;
                const int t = 2 * (ln & 3) + (q & 1);
                const int acc = s_acc[e];
                s_acc[e] = 0;
                if (t >= T) continue;
                const int64_t n = static_cast<int64_t>(t0 + tl) * 16 + (ln >> 2) + 8 * (q >> 1);
                const int64_t o = static_cast<int64_t>(t) * op.n_out + n;
                const float y = __fmul_rn(__int2float_rn(acc), s_scale[t]);
                if (p.y_bf16)
                    static_cast<__nv_bfloat16 *>(op.Y)[o] = __float2bfloat16_rn(y);
                else
                    static_cast<float *>(op.Y)[o] = y;
                if (op.acc_out) op.acc_out[o] = acc;
            }
            // optional copies of the int8 activations and scales (by the CTA holding share G - 1)
            if (share == static_cast<int>(G) - 1) {
                if (op.xq_out) {
                    for (int i = ctid; i < T * op.k; i += kChainConsumers) {
                        const int t = i / op.k;
                        const int e = i - t * op.k, u = (e & 63) >> 2;   // undo the fragment order
                        op.xq_out[i] = s_xq[t * chain_pitch(op.k) + (e & ~63) + 4 * (4 * (u & 3) + (u >> 2)) + (e & 3)];
                    }
                }
                if (op.amax_out && ctid < T) op.amax_out[ctid] = s_amax[ctid];
            }
            consumer_sync();
        }
        // 5. count this CTA done with projection j, after projection j - 1 (chain order)
        bool bad = false;
        if (ctid == 0) {
            if (j > 0 && !op.wait_prev) bad = !wait_counter(&p.counters[j - 1], G, p, &s_abort);
            // release: the consumer barrier above ordered every consumer's Y stores before this add
            if (!bad) asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(&p.counters[j]), "r"(1u) : "memory");
        }
        if (j > 0 && !op.wait_prev && consumer_sync_or(bad)) break;
    }
}

size_t chain_smem_bytes(int ns, uint32_t stage_bytes, int64_t T, int64_t kmax) {
    return static_cast<size_t>(ns) * stage_bytes + static_cast<size_t>(kChainMaxTiles) * 128 * 4 +
           static_cast<size_t>(T) * static_cast<size_t>(kmax + 128);
}

// Ring geometry: the largest stage (64, 32 or 16 KB) that leaves three stages
// (64 KB) or two (smaller) next to the activation rows.  Larger stages mean
// fewer barrier waits and longer record runs per warp.  False when not even
// two 16 KB stages fit.
bool chain_ring(int64_t T, int64_t kmax, int *ns_out, uint32_t *stage_out) {
    const size_t fixed = chain_smem_bytes(0, 0, T, kmax);
    if (fixed >= kSerialMaxSmem) return false;
    const uint32_t sizes[3] = {65536u, 32768u, 16384u};
    const int need[3] = {3, 2, 2};
    for (int i = 0; i < 3; ++i) {
        size_t ns = (kSerialMaxSmem - fixed) / sizes[i];
        if (ns > static_cast<size_t>(kChainMaxStages)) ns = kChainMaxStages;
        if (static_cast<int>(ns) >= need[i]) {
            *ns_out = static_cast<int>(ns);
            *stage_out = sizes[i];
            return true;
        }
    }
    return false;
}

cudaError_t launch_chain(const ChainOpDev *ops, int n_ops, int64_t T, bool x_bf16, bool y_bf16, float eps,
                                int64_t kmax, void *ws, cudaStream_t s) {
    int ns = 0;
    uint32_t stage_bytes = 0;
    if (!chain_ring(T, kmax, &ns, &stage_bytes)) return cudaErrorInvalidValue;
    // one-token chains take the instantiation with T folded to 1
    const bool one = T == 1;
    auto kern = x_bf16 ? (one ? k_decode_chain_serial<true, 1> : k_decode_chain_serial<true, 8>)
                       : (one ? k_decode_chain_serial<false, 1> : k_decode_chain_serial<false, 8>);
    {
        cudaError_t e = smem_attr(reinterpret_cast<const void *>(kern), static_cast<int>(kSerialMaxSmem));
        if (e != cudaSuccess) return e;
    }
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    for (int base = 0; base < n_ops; base += kChainMaxOps) {
        const int n = (n_ops - base) < kChainMaxOps ? (n_ops - base) : kChainMaxOps;
        ChainParams p;
        for (int i = 0; i < n; ++i) p.op[i] = ops[base + i];
        // a later launch continues the chain: its first projection waits for the previous launch by stream order
        p.op[0].wait_prev = 0;
        p.n_ops = n;
        p.T = static_cast<int32_t>(T);
        p.x_bf16 = x_bf16 ? 1 : 0;
        p.y_bf16 = y_bf16 ? 1 : 0;
        p.ns = ns;
        p.stage_bytes = stage_bytes;
        p.kmax = static_cast<int32_t>(kmax);
        p.eps = eps;
        p.status = reinterpret_cast<uint32_t *>(w8 + kStatusOffset);
        p.abort = reinterpret_cast<uint32_t *>(w8 + kChainAbortOffset);
        p.counters = reinterpret_cast<uint32_t *>(w8 + kChainCountersOffset);
        cudaError_t e = cudaMemsetAsync(w8 + kChainAbortOffset, 0,
                                        kChainCountersOffset - kChainAbortOffset + static_cast<size_t>(n) * 4, s);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(num_sms()));
        cfg.blockDim = dim3(kChainThreads);
        cfg.dynamicSmemBytes = chain_smem_bytes(ns, stage_bytes, T, kmax);
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kern, p);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace serial

bool chain_serial_fits(int64_t T, int64_t kmax) {
    int ns = 0;
    uint32_t stage = 0;
    return serial::chain_ring(T, kmax, &ns, &stage);
}

cudaError_t launch_decode_chain_serial(const ChainOpDev *ops, int n_ops, int64_t T, bool x_bf16, bool y_bf16, float eps,
                                       int64_t kmax, void *ws, cudaStream_t s) {
    return serial::launch_chain(ops, n_ops, T, x_bf16, y_bf16, eps, kmax, ws, s);
}

}  // namespace bitnet
