// Decode chain: a sequence of quantise + sparse ternary GEMV projections in
// one persistent launch (sm_100a).
//
// What each projection computes is the BitLinear forward of "BitNet b1.58:
// Ternary Weights for 1.58-bit LLMs", section "The mechanism" (per-token
// absmax int8 activations, ternary weights, integer sums, one rescale) with
// the 2:4 mask of "Sparse-BitNet" (gist.science), section 2
// "Kerncomponenten"; the numbers are those of bitnet_quant_act followed by
// bitnet_sparse_linear, bit for bit.
//
// Why one launch: at decode sizes (T <= 8) a projection moves 1 to 10 MB of
// packed weights, under 2 us of HBM time, while each dependent kernel launch
// adds about 3 us of completion and dependency latency.  Every SM runs one CTA
// for the whole chain, split into roles that hand work to each other through
// mbarriers, so that no role waits for a CTA-wide barrier and the weight
// stream never pauses at a projection boundary:
//  * weight producer (one thread): streams the CTA's share of every
//    projection's packed weights (a contiguous byte range of the decode
//    layout), the shares of consecutive projections back to back, into a
//    ring of 32 KB (or 16 KB) shared-memory stages with bulk asynchronous
//    copies, so that every stage is full and the bytes in flight do not
//    depend on how small a share is.  Weights do not depend on activations,
//    so it runs ahead across projections, limited only by free stages;
//  * activation loader (one thread): copies each projection's T bf16/fp32
//    activation rows, one row per bulk copy, into four staging slots (one per
//    quantiser warp); the weight producer has already warmed L2 with them.
//    A projection marked wait_prev is loaded only once every CTA has counted
//    itself done with the previous projection (grid-wide counter, acquire);
//  * quantisers (four warps, one token row of one projection per warp at a
//    time): per-token absmax, scale and int8 codes from the staging slot into
//    one of up to eight int8 buffers, in the fragment order the MMA warps
//    read, so that the quantisers run ahead of the MMA warps;
//  * MMA warps (twelve): each owns one ring slot and runs every record of the
//    stages that land in it (every twelfth stage of the stream), whatever
//    projections they hold: one m16n8k64 sparse MMA per 16x64 weight record,
//    partial sums of row tiles added into the projection's shared partial-sum
//    buffer.  There is no barrier per projection: the hand-overs between the
//    roles go through monotonic counters in shared memory (rows quantised,
//    records run, projections finished by the epilogue), so a warp waits and
//    signals only for the projections it has records of, and the fixed
//    latency of a projection overlaps with other warps' work on the next one;
//  * epilogue (one warp): dequantises the CTA's outputs of a projection,
//    writes Y, clears the buffer and counts the CTA done (release add).
// So while the MMA warps run projection j, the quantisers prepare the next
// ones and the epilogue finishes the earlier ones.  Row tiles of a projection are split over the
// CTAs in balanced contiguous ranges, rotated per projection so that the
// larger shares move around.
//
// The 2-bit codes are expanded to int8 values 64 c (bits 6-7 of each byte),
// which takes two instructions per register; the int32 sums are 64 times the
// ternary ones, exactly, and the epilogue shifts them back.
//
// Two instantiations per activation type: any T <= 8, and T = 1 with the
// token count folded to a constant.
//
// All waits are bounded (2 s): a stage that never fills, a counter that never
// reaches the grid size or an abort raised by another CTA ends every role of
// the kernel with the timeout bit in the status word; outstanding copies are
// waited for (bounded) before the copy threads exit.
#include <cstring>
#include <vector>

#include "../../include/bitnet_sparse.h"
#include "common.cuh"
#include "frag.cuh"
#include "kernels.h"

namespace bitnet {

#ifndef CHAIN_MMA_WARPS
#define CHAIN_MMA_WARPS 12
#endif
constexpr int kChainMmaWarps = CHAIN_MMA_WARPS;
constexpr int kChainQuantWarps = 4;
constexpr int kChainQuantThreads = kChainQuantWarps * 32;
constexpr int kWarpQuant0 = kChainMmaWarps;                 // first quantiser warp
constexpr int kWarpEpi = kWarpQuant0 + kChainQuantWarps;    // epilogue warp
constexpr int kWarpXLoad = kWarpEpi + 1;                    // activation loader
constexpr int kWarpWLoad = kWarpXLoad + 1;                  // weight producer
constexpr int kChainThreads = (kWarpWLoad + 1) * 32;
constexpr int kChainMaxStages = kChainMmaWarps;             // ring slots: one per MMA warp
constexpr int kChainMaxNb = 8;                              // int8 activation buffers (1, 2, 4 or 8)
constexpr int kChainAccBufs = 8;                            // partial-sum buffers
constexpr int kChainScaleSlots = 16;                        // >= kChainMaxNb + kChainAccBufs: see the epilogue
static_assert(kChainScaleSlots >= kChainMaxNb + kChainAccBufs, "scale slots");

struct ChainParams {
    ChainOpDev op[kChainMaxOps];
    int32_t n_ops, T, x_bf16, y_bf16;
    int32_t ns;                // weight ring stages
    uint32_t stage_bytes;      // bytes of one ring stage: a multiple of 256, at most 32 KB
    int32_t nb;                // int8 activation buffers: 1, 2, 4 or 8
    int32_t nb_log2;
    uint32_t xs_off[kChainQuantWarps];   // dynamic shared memory offsets of the staging slots (one row each),
    uint32_t xq_off[kChainMaxNb];        // the int8 buffers (T rows each)
    uint32_t acc_off;                    // and the partial-sum buffers
    int32_t tiles_max;         // most row tiles a CTA takes of one projection
    uint32_t acc_bytes;        // one partial-sum buffer: T x tiles_max x 16 int32
    float eps;
    int32_t release;      // some projection of this launch waits for its predecessor: count CTAs done
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

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Spins (bounded by limit_ns) until *ctr >= target.  On a timeout or a grid
// abort it sets the CTA's abort flag (and, on a timeout, the grid abort word
// and status).  The clock and the abort words are read every 16th poll only:
// reading %globaltimer takes issue slots of a pipe the other warps need.
__device__ bool wait_counter(const uint32_t *ctr, uint32_t target, const ChainParams &p, volatile int *s_abort,
                             uint64_t limit_ns = kWaitLimitNs) {
    if (ld_acquire(ctr) >= target) return true;
    uint64_t t0 = 0;
    for (uint32_t i = 1;; ++i) {
        __nanosleep(32);
        if (ld_acquire(ctr) >= target) return true;
        if ((i & 15u) == 0u) {
            if (*reinterpret_cast<volatile uint32_t *>(p.abort) != 0u || *s_abort) {
                *s_abort = 1;
                return false;
            }
            const uint64_t now = globaltimer_ns();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > limit_ns) {
                *s_abort = 1;
                atomicOr(p.status, kStatusTimeout);
                atomicExch(p.abort, 1u);
                return false;
            }
        }
    }
}

// Wait for a phase.  The waiting warp is suspended in try_wait until the
// phase completes (or about kSuspendNs pass), so that waiting roles take no
// issue slots from the working ones; between suspensions it reads the
// CTA's abort flag and, every 16th round, the clock.  Gives up when the
// abort flag is raised or after kWaitLimitNs (then it raises the flag and
// the status bit).
constexpr uint32_t kSuspendNs = 20000;
__device__ __forceinline__ bool mbar_wait_cta(uint64_t *bar, uint32_t parity, volatile int *abort, uint32_t *status) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = 0;
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait_suspend(bar, parity, kSuspendNs)) return true;
        if (*abort) return false;
        if ((i & 15u) == 0u) {
            const uint64_t now = globaltimer_ns();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > kWaitLimitNs) {
                *abort = 1;
                atomicOr(status, kStatusTimeout);
                return false;
            }
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

// Monotonic shared-memory counters of the hand-overs between the roles (see
// the MMA warps): an acquire load, a release add, and a bounded wait for a
// count to reach a target.  A count only grows, so a wait can never mistake
// an earlier round for its own.
__device__ __forceinline__ uint32_t ld_acquire_cta(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}
__device__ __forceinline__ void red_release_cta(uint32_t *p, uint32_t v) {
    asm volatile("red.release.cta.shared::cta.add.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
__device__ bool wait_count(const uint32_t *ctr, uint32_t target, volatile int *abort, uint32_t *status) {
    if (ld_acquire_cta(ctr) >= target) return true;
    uint64_t t0 = 0;
    for (uint32_t i = 1;; ++i) {
        __nanosleep(256);   // a waiting warp leaves the issue slots to the others (quantisers at T > 1)
        if (ld_acquire_cta(ctr) >= target) return true;
        if ((i & 15u) == 0u) {
            if (*abort) return false;
            const uint64_t now = globaltimer_ns();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > kWaitLimitNs) {
                *abort = 1;
                atomicOr(status, kStatusTimeout);
                return false;
            }
        }
    }
}

// Adds bytes to the transaction count of the barrier's current phase (no arrival).
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// Barrier of the quantiser warps (hardware barrier 1), used once, after
// they have loaded every projection's gamma into shared memory.
__device__ __forceinline__ void quant_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kChainQuantThreads) : "memory"); }

// Row pitch of the shared int8 activations: k + 64 or k + 128, whichever is
// 64 mod 128 bytes, so that the two token rows one quarter-warp reads in a
// 16-byte-per-lane load fall in disjoint banks.
__device__ __host__ __forceinline__ int64_t chain_pitch(int64_t k) { return k + 64 + (k & 64); }

// |x| bits of a 16-byte chunk folded into one word whose unsigned order is the
// order of the largest magnitude: for bf16 a u16x2 max of the magnitude bits
// (sign cleared); for fp32 the u32 max of the magnitude bits.  Non-negative
// floats order like their bit patterns.
template <bool BF16>
__device__ __forceinline__ uint32_t chunk_absbits(const uint4 v) {
    if constexpr (BF16) {
        const uint32_t m = 0x7fff7fffu;
        return vmax_u16x2(vmax_u16x2(v.x & m, v.y & m), vmax_u16x2(v.z & m, v.w & m));
    } else {
        const uint32_t m = 0x7fffffffu;
        return max(max(v.x & m, v.y & m), max(v.z & m, v.w & m));
    }
}
// the fp32 bits of a folded magnitude word
template <bool BF16>
__device__ __forceinline__ uint32_t absbits_to_f32(uint32_t m) {
    if constexpr (BF16) return max(m & 0xffffu, m >> 16) << 16;
    return m;
}

// Codes of one 16-byte chunk (elements e0 .. e0 + 7 for bf16, e0 .. e0 + 3 for
// fp32 of a token row whose shared int8 copy starts at row).  Within each
// 64-element k-tile the sixteen 4-byte words are stored transposed (word
// 4 j + q at 4 q + j), so that the 16 bytes lane q of a token takes as its
// m16n8k64 B fragment (k = 4 q + 16 j + 0..3, j = 0..3) are contiguous.
template <bool BF16>
__device__ __forceinline__ uint2 chunk_store_codes(const uint4 v, int8_t *row, int e0, float s) {
    int8_t *tile = row + (e0 & ~63);
    const int u0 = (e0 & 63) >> 2;   // first word within the tile
    if constexpr (BF16) {
        float f[8];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
        const uint2 q = codes8_fast(f, s);
        const int u1 = u0 + 1;
        *reinterpret_cast<uint32_t *>(tile + 4 * (4 * (u0 & 3) + (u0 >> 2))) = q.x;
        *reinterpret_cast<uint32_t *>(tile + 4 * (4 * (u1 & 3) + (u1 >> 2))) = q.y;
        return q;
    } else {
        const uint32_t q =
            codes4_fast(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z), __uint_as_float(v.w), s);
        *reinterpret_cast<uint32_t *>(tile + 4 * (4 * (u0 & 3) + (u0 >> 2))) = q;
        return make_uint2(q, 0u);
    }
}

// Adds a row tile's partial sums (four accumulators) into the shared sums,
// layout [token][tile][row of 16], and clears them.  Lane l's value q belongs
// to row l / 4 + 8 (q / 2) and token 2 (l % 4) + q % 2 of the m16n8 tile.
template <int TM>
__device__ __forceinline__ void chain_flush(int *acc_buf, int tiles_max, int tile, int lane, int T, int (&acc)[4][4]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int t = 2 * (lane & 3) + (q & 1);
        const int row = (lane >> 2) + 8 * (q >> 1);
        const int v = acc[0][q] + acc[1][q] + acc[2][q] + acc[3][q];
        const bool real = TM == 1 ? t == 0 : t < T;
        if (real) atomicAdd(&acc_buf[(t * tiles_max + tile) * 16 + row], v);
        acc[0][q] = acc[1][q] = acc[2][q] = acc[3][q] = 0;
    }
}

template <bool XBF16, int TM>
__global__ void __launch_bounds__(kChainThreads, 1) k_decode_chain(const __grid_constant__ ChainParams p) {
    constexpr int kNacc = kChainAccBufs;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t s_full[kChainMaxStages], s_empty[kChainMaxStages];
    __shared__ __align__(8) uint64_t s_xs_full[kChainQuantWarps], s_xs_empty[kChainQuantWarps];
    // hand-over counters (monotonic): rows quantised into each int8 buffer, records run against each int8 and
    // each partial-sum buffer, projections the epilogue has finished per partial-sum buffer
    __shared__ uint32_t s_rows_q[kChainMaxNb], s_recs_x[kChainMaxNb];
    __shared__ uint32_t s_recs_a[kChainAccBufs], s_freed[kChainAccBufs];
    __shared__ float s_gamma[kChainMaxOps];
    __shared__ int2 s_tiles[kChainMaxOps];    // this CTA's row tiles [x, y) of every projection
    __shared__ int s_share[kChainMaxOps];     // and its share index
    __shared__ uint32_t s_ustart[kChainMaxOps + 1];   // stream offset of each use (projection with rows here), and the end
    __shared__ uint8_t s_uj[kChainMaxOps];            // the projection of each use
    __shared__ int2 s_uk[kChainMaxOps];               // and its k and 1 / (k / 64) (fp32 bits)
    __shared__ int s_nuses;
    __shared__ uint32_t s_cumx[kChainMaxOps];         // records of the earlier uses of the same int8 buffer
    __shared__ uint32_t s_cuma[kChainMaxOps];         // and of the same partial-sum buffer
    __shared__ float s_scale[kChainScaleSlots][8];
    __shared__ float s_amax[kChainScaleSlots][8];
    __shared__ int s_abort;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int ns = p.ns;
    const int T = TM == 1 ? 1 : p.T;   // a one-token instantiation folds T away
    const uint32_t G = gridDim.x;
    // dynamic shared memory: weight ring | staging slots | int8 buffers | partial-sum buffers, each slot and
    // buffer sized by the host for the rows it receives
    uint8_t *ring = smem;
    const uint32_t stage_bytes = p.stage_bytes;
    int *sacc = reinterpret_cast<int *>(smem + p.acc_off);
    const int acc_words = static_cast<int>(p.acc_bytes >> 2);

    for (int i = tid; i < kNacc * acc_words; i += kChainThreads) sacc[i] = 0;
    // every projection's share of this CTA, once (each role reads the table instead of dividing)
    for (int i = tid; i < p.n_ops; i += kChainThreads) {
        int t0, t1;
        s_share[i] = chain_tiles(i, p.op[i].n_out >> 4, t0, t1);
        s_tiles[i] = make_int2(t0, t1);
    }
    if (tid == 0) {
        s_abort = 0;
        for (int s = 0; s < ns; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&s_empty[s], 1);   // the slot's MMA warp
        }
        for (int s = 0; s < kChainQuantWarps; ++s) {
            mbar_init(&s_xs_full[s], 1);
            mbar_init(&s_xs_empty[s], 1);
        }
        for (int s = 0; s < kChainMaxNb; ++s) s_rows_q[s] = s_recs_x[s] = 0;
        for (int s = 0; s < kChainAccBufs; ++s) s_recs_a[s] = s_freed[s] = 0;
        fence_mbar_init();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncthreads();
    if (warp == 0) {
        // the uses and their offsets in this CTA's weight stream: lane l scans projections 4 l .. 4 l + 3
        uint32_t cnt = 0, bytes = 0, b[4];
        bool has[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int j = 4 * lane + e;
            const int nt = j < p.n_ops ? s_tiles[j].y - s_tiles[j].x : 0;
            has[e] = nt > 0;
            b[e] = has[e] ? static_cast<uint32_t>(nt) * static_cast<uint32_t>(p.op[j].k >> 6) * 256u : 0u;
            cnt += has[e] ? 1u : 0u;
            bytes += b[e];
        }
        uint32_t c_ex = cnt, b_ex = bytes;   // inclusive scans, then made exclusive
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t c = __shfl_up_sync(0xffffffffu, c_ex, d), bb = __shfl_up_sync(0xffffffffu, b_ex, d);
            if (lane >= d) {
                c_ex += c;
                b_ex += bb;
            }
        }
        c_ex -= cnt;
        b_ex -= bytes;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (has[e]) {
                s_uj[c_ex] = static_cast<uint8_t>(4 * lane + e);
                s_uk[c_ex] = make_int2(p.op[4 * lane + e].k, p.op[4 * lane + e].pad);
                s_ustart[c_ex] = b_ex;
                ++c_ex;
                b_ex += b[e];
            }
        }
        if (lane == 31) {
            s_nuses = static_cast<int>(c_ex);
            s_ustart[c_ex] = b_ex;
        }
    }
    __syncthreads();
    // hand-over targets: per use, the records of the earlier uses that share its int8 buffer (u mod nb) and its
    // partial-sum buffer (u mod kNacc)
    for (int i = tid; i < s_nuses; i += kChainThreads) {
        uint32_t cx = 0, ca = 0;
        for (int v = i - p.nb; v >= 0; v -= p.nb) cx += (s_ustart[v + 1] - s_ustart[v]) >> 8;
        for (int v = i - kNacc; v >= 0; v -= kNacc) ca += (s_ustart[v + 1] - s_ustart[v]) >> 8;
        s_cumx[i] = cx;
        s_cuma[i] = ca;
    }
    __syncthreads();

    if (warp == kWarpWLoad) {
        // ------------------------------------------------------------ weight producer
        if (lane != 0) return;
        // The CTA's shares of all projections go back to back into the ring:
        // stage k holds stream bytes [k S, (k + 1) S), one bulk copy per piece of
        // a projection in it; the stage's single arrival comes when it is full
        // (or the stream ends), so its phase completes only once every piece of
        // it has landed.
        uint32_t it = 0, ps = 0, pph = 0;   // stages opened; slot it % ns; parity of fill round it / ns
        uint32_t fill = 0;                  // bytes placed in the open stage
        bool open = false, ok = true;
        for (int j = 0; j < p.n_ops && ok; ++j) {
            const ChainOpDev &op = p.op[j];
            const int t0 = s_tiles[j].x, t1 = s_tiles[j].y;
            const uint32_t tile_bytes = static_cast<uint32_t>(op.k >> 6) * 256u;
            const uint32_t bytes = static_cast<uint32_t>(t1 - t0) * tile_bytes;
            const uint8_t *src = op.dec + static_cast<size_t>(t0) * tile_bytes;
            // Warm L2 with this CTA's slice of the projection's activation rows
            // (128-byte lines b, b + G, ...), so that the loader's copy, issued
            // later, does not queue behind the weight stream in HBM.  Only a
            // cache hint: L2 is the coherence point, so a line prefetched before
            // an earlier projection writes it is updated by that write.
            {
                const size_t xbytes = static_cast<size_t>(T) * static_cast<size_t>(op.k) * (XBF16 ? 2u : 4u);
                for (size_t l = static_cast<size_t>(blockIdx.x) * 128; l < xbytes; l += static_cast<size_t>(G) * 128)
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(static_cast<const uint8_t *>(op.X) + l));
            }
            for (uint32_t off = 0; off < bytes;) {
                if (!open) {
                    // reuse of slot ps in round r >= 1 waits for the MMA warps' release of round r - 1
                    if (it >= static_cast<uint32_t>(ns) && !mbar_wait_cta(&s_empty[ps], pph ^ 1u, &s_abort, p.status)) {
                        ok = false;
                        break;
                    }
                    open = true;
                    fill = 0;
                }
                const uint32_t n = (bytes - off) < (stage_bytes - fill) ? (bytes - off) : (stage_bytes - fill);
                mbar_expect_tx(&s_full[ps], n);
                bulk_load(ring + static_cast<size_t>(ps) * stage_bytes + fill, src + off, n, &s_full[ps]);
                fill += n;
                off += n;
                if (fill == stage_bytes) {
                    mbar_arrive(&s_full[ps]);
                    open = false;
                    ++it;
                    if (++ps == static_cast<uint32_t>(ns)) {
                        ps = 0;
                        pph ^= 1u;
                    }
                }
            }
        }
        if (open && ok) {   // the stream's last, partly filled stage
            mbar_arrive(&s_full[ps]);
            ++it;
        }
        // drain: every issued stage must have landed before the thread exits
        // (earlier stages were consumed before their slot was reused)
        const uint32_t first = it > static_cast<uint32_t>(ns) ? it - ns : 0u;
        const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
        for (uint32_t q = first; q < it; ++q) mbar_wait_until(&s_full[q % ns], (q / ns) & 1u, deadline);
        return;
    }

    if (warp == kWarpXLoad) {
        // ------------------------------------------------------------ activation loader
        if (lane != 0) return;
        // one bulk copy per activation row: row item (counting the rows of every
        // projection with rows here) goes to staging slot item % 4, which belongs
        // to quantiser warp item % 4
        uint32_t item = 0;
        bool ok = true;
        for (int j = 0; j < p.n_ops && ok; ++j) {
            const ChainOpDev &op = p.op[j];
            const int t0 = s_tiles[j].x, t1 = s_tiles[j].y;
            if (t1 == t0) continue;   // no rows here: the activations are not needed
            if (j > 0 && op.wait_prev) {
                // every CTA has finished projection j - 1 (and, in chain order, all before it)
                if (!wait_counter(&p.counters[j - 1], G, p, &s_abort)) {
                    ok = false;
                    break;
                }
                // the activations were written by other SMs' generic stores, made visible by the
                // acquire above; order that before the bulk copy's async-proxy reads
                asm volatile("fence.proxy.async.global;" ::: "memory");
            }
            const uint32_t row_bytes = static_cast<uint32_t>(op.k) * (XBF16 ? 2u : 4u);
            for (int t = 0; t < T; ++t, ++item) {
                const uint32_t slot = item % kChainQuantWarps, round = item / kChainQuantWarps;
                if (round >= 1u && !mbar_wait_cta(&s_xs_empty[slot], (round - 1u) & 1u, &s_abort, p.status)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&s_xs_full[slot], row_bytes);
                bulk_load(smem + p.xs_off[slot],
                          static_cast<const uint8_t *>(op.X) + static_cast<size_t>(t) * row_bytes, row_bytes,
                          &s_xs_full[slot]);
            }
        }
        const uint32_t first = item > kChainQuantWarps ? item - kChainQuantWarps : 0u;
        const uint64_t deadline = globaltimer_ns() + kWaitLimitNs;
        for (uint32_t q = first; q < item; ++q)
            mbar_wait_until(&s_xs_full[q % kChainQuantWarps], (q / kChainQuantWarps) & 1u, deadline);
        return;
    }

    if (warp >= kWarpQuant0 && warp < kWarpEpi) {
        // ------------------------------------------------------------ quantisers
        // Work item = one token row of one projection, in chain order; item i
        // belongs to quantiser warp i % 4 and arrives in staging slot i % 4, so
        // that several projections (T = 1) or several rows (T > 1) are
        // quantised at once and no barrier joins the quantiser warps.  A row:
        // absmax of the lane's 16-byte chunks (bit patterns), one warp
        // reduction, the scale, then the codes into the int8 buffer in
        // fragment order.
        // The staging slot is waited on by parity, which sees only the last
        // two phases of a barrier: it is this warp's own and its rows arrive
        // in consecutive rounds.  The int8 buffers are handed over through
        // the monotonic counters (records run against a buffer, rows
        // quantised into it).
        const int qw = warp - kWarpQuant0;
        const int qt = tid - kWarpQuant0 * 32;
        for (int i = qt; i < p.n_ops; i += kChainQuantThreads) s_gamma[i] = __ldg(p.op[i].gamma);
        quant_sync();   // gamma of every projection in shared memory (no load on the per-row path)
        constexpr int kElems = XBF16 ? 8 : 4;
        const uint32_t nbu = static_cast<uint32_t>(p.nb);
        uint32_t uq = 0, item = 0;   // projections and rows passed so far
        bool failed = false;
        for (int j = 0; j < p.n_ops && !failed; ++j) {
            const ChainOpDev &op = p.op[j];
            const int t0 = s_tiles[j].x, t1 = s_tiles[j].y;
            const int share = s_share[j];
            if (t1 == t0) continue;
            const int xb = static_cast<int>(uq & (nbu - 1u));
            const uint32_t xround = uq >> p.nb_log2;
            const int sc = static_cast<int>(uq % kChainScaleSlots);
            const int k = op.k;
            const int pitch = static_cast<int>(chain_pitch(k));
            const int cpr = k / kElems;   // 16-byte chunks per row
            const bool copy_out = share == static_cast<int>(G) - 1;
            const bool xq_vec = op.xq_out && (reinterpret_cast<uintptr_t>(op.xq_out) & 7u) == 0u;
            bool waited = false;
            for (int t = 0; t < T; ++t, ++item) {
                if (item % kChainQuantWarps != static_cast<uint32_t>(qw)) continue;
                // every record of this buffer's earlier projections has been run
                bool ok = waited || xround == 0u || wait_count(&s_recs_x[xb], s_cumx[uq], &s_abort, p.status);
                waited = true;
                // this warp's own staging slot: its rows arrive there in consecutive rounds
                ok = ok && mbar_wait_cta(&s_xs_full[qw], (item / kChainQuantWarps) & 1u, &s_abort, p.status);
                if (!__all_sync(0xffffffffu, ok)) {
                    failed = true;
                    break;
                }
                const uint4 *src = reinterpret_cast<const uint4 *>(smem + p.xs_off[qw]);
                // pass 1: absmax of the row
                uint32_t m = 0u;
                for (int c = lane; c < cpr; c += 32) {
                    const uint32_t a = chunk_absbits<XBF16>(src[c]);
                    m = XBF16 ? vmax_u16x2(m, a) : max(m, a);
                }
                float a = __uint_as_float(__reduce_max_sync(0xffffffffu, absbits_to_f32<XBF16>(m)));
                a = a > p.eps ? a : p.eps;
                const float s_inv = __fdiv_rn(127.0f, a);
                if (lane == 0) {
                    s_scale[sc][t] = __fdiv_rn(__fmul_rn(s_gamma[j], a), 127.0f);
                    s_amax[sc][t] = a;
                    if (copy_out && op.amax_out) op.amax_out[t] = a;
                }
                // pass 2: codes (and, on one CTA, their copy in natural order)
                int8_t *row = reinterpret_cast<int8_t *>(smem + p.xq_off[xb]) + static_cast<size_t>(t) * pitch;
                for (int c = lane; c < cpr; c += 32) {
                    const uint2 q = chunk_store_codes<XBF16>(src[c], row, c * kElems, s_inv);
                    if (copy_out && op.xq_out) {
                        int8_t *dst = op.xq_out + static_cast<size_t>(t) * k + static_cast<size_t>(c) * kElems;
                        if (xq_vec && XBF16) {
                            *reinterpret_cast<uint2 *>(dst) = q;
                        } else if (xq_vec) {
                            *reinterpret_cast<uint32_t *>(dst) = q.x;
                        } else {
#pragma unroll
                            for (int e = 0; e < kElems; ++e)
                                dst[e] = static_cast<int8_t>(((e < 4 ? q.x : q.y) >> (8 * (e & 3))) & 0xffu);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) {
                    red_release_cta(&s_rows_q[xb], 1u);   // T rows per projection
                    mbar_arrive(&s_xs_empty[qw]);
                }
            }
            ++uq;
        }
        return;
    }

    if (warp == kWarpEpi) {
        // ------------------------------------------------------------ epilogue
        uint32_t ua = 0;   // projections finished (partial-sum buffer ua % kNacc, scale slot ua % kChainScaleSlots)
        for (int j = 0; j < p.n_ops; ++j) {
            const ChainOpDev &op = p.op[j];
            const int t0 = s_tiles[j].x, t1 = s_tiles[j].y;
            const int ntile = t1 - t0;
            if (ntile > 0) {
                const int ab = static_cast<int>(ua % kNacc);
                // every record of this projection (and of the buffer's earlier ones) has been run and flushed
                const bool ok = wait_count(&s_recs_a[ab], s_cuma[ua] + static_cast<uint32_t>(ntile * (op.k >> 6)),
                                           &s_abort, p.status);
                if (!__all_sync(0xffffffffu, ok)) break;
                // Scale slot ua % (kChainMaxNb + kChainAccBufs) was written by
                // the quantisers after the MMA warps released int8 buffer use
                // ua - nb, which they do only after taking partial-sum buffer
                // use ua - nb, i.e. after this warp finished projection use
                // ua - nb - kNacc >= ua - kChainMaxNb - kChainAccBufs.
                const int sc = static_cast<int>(ua % kChainScaleSlots);
                int *acc_buf = sacc + ab * acc_words;
                const int per_t = ntile * 16;
                for (int e = lane; e < T * per_t; e += 32) {
                    const int t = TM == 1 ? 0 : e / per_t;
                    const int rem = e - t * per_t;
                    const int idx = (t * p.tiles_max + (rem >> 4)) * 16 + (rem & 15);
                    const int v = acc_buf[idx] >> 6;   // the products were 64 times the ternary ones
                    acc_buf[idx] = 0;
                    const int64_t o = static_cast<int64_t>(t) * op.n_out + static_cast<int64_t>(t0) * 16 + rem;
                    const float y = __fmul_rn(__int2float_rn(v), s_scale[sc][t]);
                    if (p.y_bf16)
                        static_cast<__nv_bfloat16 *>(op.Y)[o] = __float2bfloat16_rn(y);
                    else
                        static_cast<float *>(op.Y)[o] = y;
                    if (op.acc_out) op.acc_out[o] = v;
                }
                __syncwarp();
                if (lane == 0) red_release_cta(&s_freed[ab], 1u);   // the buffer is clear for its next projection
                ++ua;
            }
            // count this CTA done with projection j (and, by program order, with every
            // earlier one): the warp barrier orders every lane's Y stores before the
            // release.  A release waits until those stores have reached L2, about a
            // microsecond, so it is issued only when a later projection of the launch
            // waits for it (the end of the launch orders everything for what follows).
            __syncwarp();
            if (p.release && lane == 0)
                asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(&p.counters[j]), "r"(1u) : "memory");
        }
        return;
    }

    // ---------------------------------------------------------------- MMA warps
    // The ring carries this CTA's shares of all projections back to back, in
    // stages of S bytes; with W MMA warps, stage s sits in ring slot s % W, and
    // MMA warp w owns slot w: it runs every record of the stages w, w + W, ...
    // (whatever projections they belong to) and alone releases them.  The
    // hand-overs go through monotonic counters, so a warp deals only with the
    // uses (projections with rows here) it has records of: it opens use u
    // when it meets u's records (u's partial-sum buffer has been cleared by
    // the epilogue for u's round, all T rows of u are quantised), runs them,
    // and closes u as soon as it knows it has no more records of it (its stage
    // reaches u's end, or its next stage starts at or after it): it flushes
    // its partial sums and adds its record count to both buffers' counters.
    // The epilogue takes u once every record of u has been counted; the
    // quantisers refill u's int8 buffer once every record of it has been.
    const int n_uses = s_nuses;
    const uint32_t total = s_ustart[n_uses];
    int u = 0;                  // cursor: the use holding the current stream position (or an earlier one)
    bool opened = false;        // use u is open
    uint32_t mine = 0;          // records of the open use run by this warp
    bool failed = false;
    // state of the open use
    int ab = 0, xb = 0, ktiles = 1, cur = -1;
    uint32_t ustart = 0, uend = 0;
    float inv_kt = 1.0f;
    int *acc_buf = sacc;
    const uint4 *b_src = nullptr;
    int acc[4][4] = {};   // partial sums of the current row tile, one accumulator per record slot
    // Lane l holds the B fragment of token l / 4 (zero for tokens >= T): the
    // 16 bytes lane l % 4 needs of each 64-k tile sit contiguously in the
    // shared row (fragment order), one 16-byte load per record.
    const int bn = lane >> 2;
    const bool has_b = bn < T;
    auto open_use = [&]() -> bool {
        const int2 uk = s_uk[u];   // k, and 1 / ktiles formed on the host
        ab = u % kNacc;
        xb = u & (p.nb - 1);
        bool ok = wait_count(&s_freed[ab], static_cast<uint32_t>(u / kNacc), &s_abort, p.status);
        ok = ok && wait_count(&s_rows_q[xb], static_cast<uint32_t>(T) * ((static_cast<uint32_t>(u) >> p.nb_log2) + 1u),
                              &s_abort, p.status);
        if (!__all_sync(0xffffffffu, ok)) return false;
        acc_buf = sacc + ab * acc_words;
        b_src = reinterpret_cast<const uint4 *>(smem + p.xq_off[xb] +
                                                static_cast<int64_t>(has_b ? bn : 0) * chain_pitch(uk.x)) +
                (lane & 3);
        ktiles = uk.x >> 6;
        inv_kt = __int_as_float(uk.y);
        ustart = s_ustart[u];
        uend = s_ustart[u + 1];
        cur = -1;
        mine = 0;
        opened = true;
        return true;
    };
    auto close_use = [&]() {
        if (cur >= 0) chain_flush<TM>(acc_buf, p.tiles_max, cur, lane, T, acc);
        // every lane's shared atomics (and shared loads of the int8 buffer) are
        // ordered before the release of the counts
        __syncwarp();
        if (lane == 0) {
            red_release_cta(&s_recs_a[ab], mine);
            red_release_cta(&s_recs_x[xb], mine);
        }
        opened = false;
        ++u;
    };
    const uint32_t ring_step = stage_bytes * static_cast<uint32_t>(kChainMmaWarps);
    uint8_t *slot = ring + static_cast<size_t>(warp) * stage_bytes;
    uint32_t round = 0;
    for (uint32_t a = static_cast<uint32_t>(warp) * stage_bytes; a < total; a += ring_step, ++round) {
        const uint32_t b = total - a < stage_bytes ? total : a + stage_bytes;
        // the open use, if it ended before this stage (it was closed then), and other warps' uses
        while (u < n_uses && s_ustart[u + 1] <= a) ++u;
        const bool okf = mbar_wait_cta(&s_full[warp], round & 1u, &s_abort, p.status);
        if (!__all_sync(0xffffffffu, okf)) {
            failed = true;
            break;
        }
        for (uint32_t pos = a; pos < b && !failed;) {
            if (!opened && !open_use()) {
                failed = true;
                break;
            }
            const uint32_t seg_end = b < uend ? b : uend;
            // records [pos, seg_end) of the open use; r0 = the first one's index in the CTA's share
            const int r0 = static_cast<int>((pos - ustart) >> 8);
            const int cnt = static_cast<int>((seg_end - pos) >> 8);
            mine += static_cast<uint32_t>(cnt);
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
            const uint2 *rec = reinterpret_cast<const uint2 *>(slot + (pos - a)) + lane;
            int i = 0;
            while (i < cnt) {
                if (tile != cur) {
                    if (cur >= 0) chain_flush<TM>(acc_buf, p.tiles_max, cur, lane, T, acc);
                    cur = tile;
                }
                if (i + 4 <= cnt && kt + 4 <= ktiles) {
                    // four records of one row tile: all loads first, then the MMAs
                    uint2 w[4];
                    uint32_t bf[4][4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) w[e] = rec[(i + e) * 32];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint4 v = has_b ? b_src[(kt + e) * 4] : make_uint4(0u, 0u, 0u, 0u);
                        bf[e][0] = v.x;
                        bf[e][1] = v.y;
                        bf[e][2] = v.z;
                        bf[e][3] = v.w;
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        uint32_t a4[4];
#pragma unroll
                        for (int r = 0; r < 4; ++r) a4[r] = expand_codes_x64(w[e].x, r);
                        mma_sp_m16n8k64(acc[e], a4, bf[e], w[e].y);
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
                    for (int r = 0; r < 4; ++r) a4[r] = expand_codes_x64(w.x, r);
                    mma_sp_m16n8k64(acc[0], a4, bf, w.y);
                    i += 1;
                    kt += 1;
                }
                if (kt == ktiles) {
                    kt = 0;
                    ++tile;
                }
            }
            pos = seg_end;
            if (pos == uend) close_use();
        }
        if (failed) break;
        // release the stage to the producer
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[warp]);
        // the open use, if it ends before this warp's next stage
        const uint32_t na = a + ring_step < total ? a + ring_step : total;
        if (opened && uend <= na) close_use();
    }
    if (!failed && opened) close_use();
}

// ---------------------------------------------------------------- host side

static size_t round128(size_t x) { return (x + 127) / 128 * 128; }

// Shared-memory layout: the weight ring (one slot per MMA warp), four
// staging slots (slot s holds the activation rows i = s mod 4 of the chain,
// xs_slot[s] bytes), int8 buffers (buffer b holds the uses u = b mod nb,
// xq_use[u] bytes each) and eight partial-sum buffers.  The ring takes what
// is left, in stages of a multiple of 256 bytes (one record) up to 32 KB, in
// this order of preference: eight int8 buffers (the quantisers run further
// ahead) with stages of at least 8 KB; four or two buffers with 8 KB; down to
// one buffer (T >= 4) with 2 KB.  For T < 4 the buffers are four or eight
// (see the quantisers).  Every size is a multiple of 128 bytes.  False when
// even the last form does not fit.
static bool chain_layout_sized(int64_t T, const size_t xs_slot[kChainQuantWarps], const size_t *xq_use, int n_uses,
                               int tiles_max, ChainLayout *L) {
    if (T < 1 || T > 8 || n_uses < 1 || tiles_max < 1 || tiles_max > kChainMaxTiles) return false;
    const size_t acc = round128(static_cast<size_t>(T) * static_cast<size_t>(tiles_max) * 16 * 4);
    size_t xs_total = 0;
    for (int q = 0; q < kChainQuantWarps; ++q) xs_total += xs_slot[q];
    constexpr int kPasses = 3;
    const size_t min_stage[kPasses] = {8192, 8192, 2048};
    const int max_nb[kPasses] = {8, 4, 4};
    const int min_nb[kPasses] = {8, 2, 1};
    for (int pass = 0; pass < kPasses; ++pass) {
        for (int nb = max_nb[pass]; nb >= min_nb[pass]; nb >>= 1) {
            if (T < 4 && nb % 4 != 0) continue;
            size_t xq_size[kChainMaxNb] = {};
            size_t xq_total = 0;
            for (int u = 0; u < n_uses; ++u)
                xq_size[u % nb] = xq_use[u] > xq_size[u % nb] ? xq_use[u] : xq_size[u % nb];
            for (int b = 0; b < nb; ++b) xq_total += xq_size[b];
            const size_t fixed = kChainAccBufs * acc + xq_total + xs_total;
            if (fixed >= kChainMaxSmem) continue;
            size_t stage = (kChainMaxSmem - fixed) / kChainMaxStages / 256 * 256;
            if (stage > 32768) stage = 32768;
            if (stage < min_stage[pass]) continue;
            L->ns = kChainMaxStages;
            L->stage_bytes = static_cast<uint32_t>(stage);
            L->nb = nb;
            size_t off = kChainMaxStages * stage;
            for (int q = 0; q < kChainQuantWarps; ++q) {
                L->xs_off[q] = static_cast<uint32_t>(off);
                off += xs_slot[q];
            }
            for (int b = 0; b < kChainMaxNb; ++b) {
                L->xq_off[b] = static_cast<uint32_t>(off);
                if (b < nb) off += xq_size[b];
            }
            L->acc_off = static_cast<uint32_t>(off);
            L->tiles_max = tiles_max;
            L->acc_bytes = static_cast<uint32_t>(acc);
            L->smem = off + kChainAccBufs * acc;
            return true;
        }
    }
    return false;
}

bool chain_layout(int64_t T, int64_t kmax, bool x_bf16, int tiles_max, ChainLayout *L) {
    if (kmax < 64) return false;
    const size_t xs = round128(static_cast<size_t>(kmax) * (x_bf16 ? 2 : 4));
    const size_t xs_slot[kChainQuantWarps] = {xs, xs, xs, xs};
    size_t xq_use[kChainMaxNb];
    for (int b = 0; b < kChainMaxNb; ++b)
        xq_use[b] = round128(static_cast<size_t>(T) * static_cast<size_t>(chain_pitch(kmax)));
    return chain_layout_sized(T, xs_slot, xq_use, kChainMaxNb, tiles_max, L);
}

// The layout of one launch over ops[0, n).  When every projection has at
// least one row tile on every CTA (n_out / 16 >= G), the k-th
// projection with rows on a CTA is projection k on every CTA, so each slot and
// buffer can be sized for the rows it actually receives; otherwise every one
// holds rows of kmax.
static bool chain_layout_for(const ChainOpDev *ops, int n, int64_t T, bool x_bf16, int64_t kmax, int G, int tiles_max,
                             ChainLayout *L) {
    bool every_cta = true;
    for (int i = 0; i < n; ++i) every_cta = every_cta && (ops[i].n_out >> 4) >= G;
    if (!every_cta) return chain_layout(T, kmax, x_bf16, tiles_max, L);
    size_t xs_slot[kChainQuantWarps] = {};
    std::vector<size_t> xq_use(static_cast<size_t>(n));
    for (int i = 0; i < n; ++i) {
        const size_t row = round128(static_cast<size_t>(ops[i].k) * (x_bf16 ? 2 : 4));
        for (int64_t t = 0; t < T; ++t) {
            const int q = static_cast<int>((static_cast<int64_t>(i) * T + t) % kChainQuantWarps);
            xs_slot[q] = row > xs_slot[q] ? row : xs_slot[q];
        }
        xq_use[static_cast<size_t>(i)] = round128(static_cast<size_t>(T) * static_cast<size_t>(chain_pitch(ops[i].k)));
    }
    return chain_layout_sized(T, xs_slot, xq_use.data(), n, tiles_max, L);
}

cudaError_t launch_decode_chain(const ChainOpDev *ops, int n_ops, int64_t T, bool x_bf16, bool y_bf16, float eps,
                                int64_t kmax, void *ws, cudaStream_t s) {
    // A projection that waits for its predecessor makes the chain latency-bound:
    // such chains take the kernel of chain_serial.cu, whose path from one
    // projection to the next has no hand-over between warp roles.
    for (int i = 1; i < n_ops; ++i)
        if (ops[i].wait_prev) return launch_decode_chain_serial(ops, n_ops, T, x_bf16, y_bf16, eps, kmax, ws, s);
    const int G = num_sms();
    int tiles_max = 1;
    for (int i = 0; i < n_ops; ++i) {
        const int rows16 = ops[i].n_out >> 4;
        const int t = (rows16 + G - 1) / G;
        tiles_max = t > tiles_max ? t : tiles_max;
    }
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    for (int base = 0; base < n_ops; base += kChainMaxOps) {
        const int n = (n_ops - base) < kChainMaxOps ? (n_ops - base) : kChainMaxOps;
        ChainLayout L;
        if (!chain_layout_for(ops + base, n, T, x_bf16, kmax, G, tiles_max, &L)) return cudaErrorInvalidValue;
        // one-token chains take the instantiation with T folded to 1
        const bool one = T == 1;
        auto kern = x_bf16 ? (one ? k_decode_chain<true, 1> : k_decode_chain<true, 8>)
                           : (one ? k_decode_chain<false, 1> : k_decode_chain<false, 8>);
        {
            cudaError_t e = smem_attr(reinterpret_cast<const void *>(kern), static_cast<int>(kChainMaxSmem));
            if (e != cudaSuccess) return e;
        }
        ChainParams p;
        for (int i = 0; i < n; ++i) {
            p.op[i] = ops[base + i];
            // 1 / (k / 64) for the record-to-tile division on the device (r / ktiles via a float
            // product, corrected there); formed here in IEEE fp32
            const float inv_kt = 1.0f / static_cast<float>(p.op[i].k >> 6);
            std::memcpy(&p.op[i].pad, &inv_kt, 4);
        }
        // a later launch continues the chain: its first projection waits for the previous launch by stream order
        p.op[0].wait_prev = 0;
        p.n_ops = n;
        p.release = 0;
        for (int i = 1; i < n; ++i) p.release |= p.op[i].wait_prev != 0 ? 1 : 0;
        p.T = static_cast<int32_t>(T);
        p.x_bf16 = x_bf16 ? 1 : 0;
        p.y_bf16 = y_bf16 ? 1 : 0;
        p.ns = L.ns;
        p.stage_bytes = L.stage_bytes;
        p.nb = L.nb;
        p.nb_log2 = L.nb == 8 ? 3 : (L.nb == 4 ? 2 : (L.nb == 2 ? 1 : 0));
        for (int q = 0; q < kChainQuantWarps; ++q) p.xs_off[q] = L.xs_off[q];
        for (int b = 0; b < kChainMaxNb; ++b) p.xq_off[b] = L.xq_off[b];
        p.acc_off = L.acc_off;
        p.tiles_max = L.tiles_max;
        p.acc_bytes = L.acc_bytes;
        p.eps = eps;
        p.status = reinterpret_cast<uint32_t *>(w8 + kStatusOffset);
        p.abort = reinterpret_cast<uint32_t *>(w8 + kChainAbortOffset);
        p.counters = reinterpret_cast<uint32_t *>(w8 + kChainCountersOffset);
        cudaError_t e = cudaMemsetAsync(w8 + kChainAbortOffset, 0,
                                        kChainCountersOffset - kChainAbortOffset + static_cast<size_t>(n) * 4, s);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(G));
        cfg.blockDim = dim3(kChainThreads);
        cfg.dynamicSmemBytes = L.smem;
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

// ---------------------------------------------------------------- health check of the bounded waits
//
// Runs the two kinds of bounded wait the kernels use on events that never
// happen, with a short limit: warp 0 waits on an mbarrier nobody arrives at
// (mbar_wait_bounded, the wait of the GEMM and pack pipelines), warp 1 on a
// grid counter nobody increments (wait_counter, the decode chain's wait).
// Both give up after limit_ns, set the timeout bit of the status word and
// return; the kernel ends normally and the context stays usable.
__global__ void k_wait_selftest(uint32_t *status, uint32_t *abort_word, const uint32_t *counter, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int s_abort_mbar, s_abort_ctr;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        s_abort_mbar = 0;
        s_abort_ctr = 0;
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, &s_abort_mbar, status, limit_ns);
    if (threadIdx.x == 32) {
        ChainParams p;
        p.status = status;
        p.abort = abort_word;
        p.counters = nullptr;
        wait_counter(counter, 1u, p, &s_abort_ctr, limit_ns);
    }
}

cudaError_t launch_wait_selftest(void *ws, uint64_t limit_ns, cudaStream_t s) {
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    cudaError_t e = cudaMemsetAsync(ws, 0, kChainCountersOffset + 4, s);
    if (e != cudaSuccess) return e;
    k_wait_selftest<<<1, 64, 0, s>>>(reinterpret_cast<uint32_t *>(w8 + kStatusOffset),
                                     reinterpret_cast<uint32_t *>(w8 + kChainAbortOffset),
                                     reinterpret_cast<const uint32_t *>(w8 + kChainCountersOffset), limit_ns);
    return cudaGetLastError();
}

}  // namespace bitnet
