// Host-side launchers of the kernels behind the C ABI (internal header).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace bitnet {

// Workspace layout shared by the entry points: the device status word is
// always the first 4 bytes.
constexpr size_t kStatusOffset = 0;
// pack: threshold bits, 128-bit window sum, 256 exponent bins
constexpr size_t kPackWsCounterOffset = 4;
constexpr size_t kPackWsThrOffset = 8;
constexpr size_t kPackWsModeOffset = 12;
constexpr size_t kPackWsWinOffset = 16;
constexpr size_t kPackWsListCountOffset = 32;
constexpr size_t kPackWsBandOffset = 40;
constexpr size_t kPackWsBinsOffset = 256;
constexpr size_t kPackWsBytes = 256 + 256 * 8;
// linear: status word only
constexpr size_t kLinearWsBytes = 256;
// dgrad: status word, then the bf16 [k, n_out] expansion of Wq^T
constexpr size_t kDgradWsHeader = 256;

int num_sms();
// Raises func's dynamic shared-memory limit on the current device (once per device and function).
cudaError_t smem_attr(const void *func, int bytes);

// Sets the message bitnet_last_error() returns on this thread.
void set_last_error(const char *msg);

cudaError_t launch_pack(const float *W, int64_t n_out, int64_t k, int n, int m, float eps, float *gamma,
                        uint8_t *gb, int8_t *vals, uint8_t *meta, uint8_t *dec, uint8_t *mask, void *ws,
                        cudaStream_t s);

cudaError_t launch_pack_update(const float *W, int64_t n_out, int64_t k, float eps, float *gamma, uint8_t *gb,
                               int8_t *vals, uint8_t *meta, uint8_t *dec, uint8_t *mask, void *ws, size_t ws_bytes,
                               cudaStream_t s);

// Band-list bytes of the per-step pack of one matrix: room for 1/256 of the
// groups (Gaussian masters put ~0.06% of the weights within 2^-10 of the
// threshold), at least 16384 entries.
inline size_t update_list_bytes(int64_t n_out, int64_t k) {
    const size_t groups = static_cast<size_t>(n_out) * static_cast<size_t>(k) / 4;
    size_t cap = groups / 256;
    if (cap < 16384) cap = 16384;
    return cap * 4;
}

// Batched per-step pack: one matrix as the host describes it.
struct PackBatchItemHost {
    const void *W;   // fp32 or bf16 masters (w_bf16)
    int64_t n_out, k;
    float *gamma;
    uint8_t *gb;
    int8_t *vals;
    uint8_t *meta;
    uint8_t *dec;
    uint8_t *mask;
    bool w_bf16;
    bool gamma_known;   // *gamma is already the exact gamma of W (from the optimiser step)
};
constexpr int kPackBatchMax = 64;   // matrices per launch (kernel parameter space)
size_t pack_batch_ws_bytes(const int64_t *n_out, const int64_t *k, int n_items);
cudaError_t launch_pack_update_batch(const PackBatchItemHost *items, int n_items, float eps, void *ws, cudaStream_t s);

cudaError_t launch_quant_act(const void *X, bool bf16, int64_t T, int64_t K, float eps, int8_t *Xq, float *amax,
                             cudaStream_t s);

// 6:8 weights through three 2:4 windows per block of 8 (pack.cu, quant.cu)
cudaError_t launch_pack68(const float *W, int64_t n_out, int64_t k, float eps, float *gamma, uint8_t *gbw,
                          int8_t *vals, uint8_t *meta, uint8_t *dec, uint8_t *mask, void *ws, cudaStream_t s);
cudaError_t launch_quant_lift68(const void *X, bool bf16, int64_t T, int64_t K, float eps, int8_t *Xl, float *amax,
                                cudaStream_t s);

// AdamW step of fp32 masters that also emits the exact absmean gamma of the result (pack.cu)
cudaError_t launch_adamw_gamma(float *W, const float *G, float *M, float *V, int64_t n, float lr, float b1, float b2,
                               float eps, float wd, float c1, float c2, float eps_gamma, float *gamma, void *ws,
                               cudaStream_t s);

// Tensor-core instruction throughput ceiling (peak.cu); *ops = dense-equivalent operations of the launch
cudaError_t launch_tensor_peak(int kind, int64_t iters, uint32_t *status, double *ops, cudaStream_t s);

// Health check of the bounded waits (chain.cu): both kinds of wait run out on events that never happen
cudaError_t launch_wait_selftest(void *ws, uint64_t limit_ns, cudaStream_t s);

// The AdamW step with gamma over a list of matrices (pack.cu)
struct AdamWItemHost {
    float *W;
    const float *G;
    float *M, *V;
    int64_t n;
    float *gamma;
};
constexpr int kAdamWBatchMax = 64;   // matrices per launch (kernel parameter space)
cudaError_t launch_adamw_gamma_batch(const AdamWItemHost *items, int n_items, float lr, float b1, float b2, float eps,
                                     float wd, float c1, float c2, float eps_gamma, void *ws, cudaStream_t s);

// Weight gradient (gemm2.cu)
cudaError_t launch_gemm_wgrad_pair(const void *dY, const void *X, int64_t T, int64_t n_out, int64_t k, float *dW,
                                   bool accumulate, uint32_t *status, cudaStream_t s);

// Block epilogues fused into quantisation (block_quant.cu)
constexpr size_t kSwigluMaxSmem = 200 * 1024;   // h of one token row in fp32
size_t swiglu_smem_bytes(int64_t F);
cudaError_t launch_rmsnorm_quant(const void *X, const float *w, int64_t T, int64_t K, float eps_n, float eps_a,
                                 int8_t *Xq, float *amax, float *rinv, cudaStream_t s);
cudaError_t launch_swiglu_quant(const void *G, const void *U, int64_t ld, int64_t T, int64_t F, float eps_a,
                                int8_t *Xq, float *amax, cudaStream_t s);

cudaError_t launch_gemv_dec(const int8_t *Xq, const float *amax, const float *gamma, const uint8_t *dec,
                            int64_t T, int64_t n_out, int64_t k, void *Y, bool y_bf16, int32_t *acc,
                            cudaStream_t s);

// Decode chain (chain.cu): one projection as the kernel sees it.
struct ChainOpDev {
    const void *X;
    const uint8_t *dec;
    const float *gamma;
    void *Y;
    int32_t *acc_out;
    int8_t *xq_out;
    float *amax_out;
    int32_t n_out, k, wait_prev, pad;
};
constexpr int kChainMaxOps = 128;                  // projections per launch (kernel parameter space)
constexpr int kChainMaxTiles = 32;                 // 16-row tiles per CTA per projection
constexpr int kChainMaxK = 1 << 17;                // 64 * 127 * k / 2 stays inside int32 (codes expanded x64)
constexpr size_t kChainMaxSmem = 227 * 1024 - 6144;   // dynamic shared memory (static use < 6 KB)
constexpr size_t kChainAbortOffset = 4;            // workspace: grid abort word
constexpr size_t kChainCountersOffset = 256;       // workspace: one counter per projection
// Shared-memory layout of one chain launch (chain.cu).
struct ChainLayout {
    int ns;               // weight ring stages
    uint32_t stage_bytes; // bytes of one stage
    int nb;               // int8 activation buffers
    int tiles_max;        // most row tiles one CTA takes of one projection
    uint32_t xs_off[4];   // byte offsets in dynamic shared memory: activation staging slots,
    uint32_t xq_off[8];   // int8 buffers
    uint32_t acc_off;     // and the partial-sum buffers
    uint32_t acc_bytes;   // one partial-sum buffer
    size_t smem;          // dynamic shared memory of the launch
};
// A layout in which every staging slot and int8 buffer holds rows of kmax
// (the launch may size them tighter, for the rows they actually receive).
bool chain_layout(int64_t T, int64_t kmax, bool x_bf16, int tiles_max, ChainLayout *L);
// The latency-oriented chain for projections that wait for their predecessor (chain_serial.cu).
bool chain_serial_fits(int64_t T, int64_t kmax);
cudaError_t launch_decode_chain_serial(const ChainOpDev *ops, int n_ops, int64_t T, bool x_bf16, bool y_bf16, float eps,
                                       int64_t kmax, void *ws, cudaStream_t s);
cudaError_t launch_decode_chain(const ChainOpDev *ops, int n_ops, int64_t T, bool x_bf16, bool y_bf16, float eps,
                                int64_t kmax, void *ws, cudaStream_t s);

cudaError_t launch_gemv_gb(const int8_t *Xq, const float *amax, const float *gamma, const uint8_t *gb,
                           int64_t T, int64_t n_out, int64_t k, void *Y, bool y_bf16, int32_t *acc,
                           cudaStream_t s);

cudaError_t launch_gemm_sp(const int8_t *Xq, const float *amax, const float *gamma, const int8_t *vals,
                           const uint8_t *meta, int64_t T, int64_t n_out, int64_t k, void *Y, bool y_bf16,
                           int32_t *acc, uint32_t *status, cudaStream_t s);

cudaError_t launch_gemm_sp_pair(const int8_t *Xq, const float *amax, const float *gamma, const int8_t *vals,
                                const uint8_t *meta, int64_t T, int64_t n_out, int64_t k, void *Y, bool y_bf16,
                                int32_t *acc, uint32_t *status, cudaStream_t s);

cudaError_t launch_gemm_bf16_pair(const void *dY, const __nv_bfloat16 *w, const float *gamma, int64_t T,
                                  int64_t n_out, int64_t k, void *dX, bool dx_bf16, uint32_t *status, cudaStream_t s);

cudaError_t launch_dgrad(const void *dY, const float *gamma, const uint8_t *gb, int64_t T, int64_t n_out,
                         int64_t k, void *dX, bool dx_bf16, void *ws, cudaStream_t s);

}  // namespace bitnet
