// C ABI of the sparse ternary BitLinear library: host-side argument checks,
// shape dispatch and launches.  Declarations and semantics: bitnet_sparse.h.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include <vector>

#include "../../include/bitnet_sparse.h"
#include "kernels.h"

namespace {

thread_local char g_err[512] = "";

bitnet_status fail(bitnet_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return s;
}

bitnet_status cuda_status(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return BITNET_OK;
    return fail(BITNET_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace

namespace bitnet {
void set_last_error(const char *msg) { snprintf(g_err, sizeof g_err, "%s", msg); }
}  // namespace bitnet

extern "C" {

int bitnet_abi_version(void) { return 1; }

const char *bitnet_last_error(void) { return g_err; }

const char *bitnet_status_string(bitnet_status s) {
    switch (s) {
        case BITNET_OK: return "ok";
        case BITNET_ERR_INVALID_ARG: return "invalid argument";
        case BITNET_ERR_UNSUPPORTED: return "unsupported configuration";
        case BITNET_ERR_WORKSPACE: return "workspace missing or too small";
        case BITNET_ERR_CUDA: return "CUDA error";
        case BITNET_ERR_TIMEOUT: return "device-side wait timed out";
    }
    return "unknown status";
}

size_t bitnet_mma_meta_bytes(int64_t n_out, int64_t k) {
    if (n_out <= 0 || k <= 0) return 0;
    return static_cast<size_t>(ceil_div(k, 128) * ceil_div(n_out, 128) * 2048);
}

size_t bitnet_dec_bytes(int64_t n_out, int64_t k) {
    if (n_out <= 0 || k <= 0 || n_out % 16 || k % 64) return 0;
    return static_cast<size_t>(n_out / 16) * static_cast<size_t>(k / 64) * 256;
}

size_t bitnet_pack_workspace_size(int64_t, int64_t) { return bitnet::kPackWsBytes; }
size_t bitnet_linear_workspace_size(void) { return bitnet::kLinearWsBytes; }
size_t bitnet_dgrad_workspace_size(int64_t n_out, int64_t k) {
    if (n_out <= 0 || k <= 0) return bitnet::kDgradWsHeader;
    return bitnet::kDgradWsHeader + static_cast<size_t>(n_out) * static_cast<size_t>(k) * 2;
}

bitnet_status bitnet_pack_nm(const float *W, bitnet_packed_w *out, float eps, uint8_t *mask_bits, void *ws,
                             size_t ws_bytes, bitnet_stream_t stream) {
    if (!W || !out || !out->gamma) return fail(BITNET_ERR_INVALID_ARG, "pack: W, out and out->gamma are required");
    if (!ws) return fail(BITNET_ERR_WORKSPACE, "pack: workspace is required");
    if (ws_bytes < bitnet::kPackWsBytes) return fail(BITNET_ERR_WORKSPACE, "pack: workspace needs %zu bytes", bitnet::kPackWsBytes);
    const int64_t n_out = out->n_out, k = out->k;
    const int n = out->n, m = out->m;
    if (n_out <= 0 || k <= 0) return fail(BITNET_ERR_INVALID_ARG, "pack: n_out and k must be positive");
    if (!(m == 4 || m == 8) || n < 1 || n >= m) return fail(BITNET_ERR_UNSUPPORTED, "pack: N:M must have m in {4,8}, 1 <= n < m");
    if (k % 8 != 0) return fail(BITNET_ERR_INVALID_ARG, "pack: k must be a multiple of 8");
    if (!(eps >= 0.0f)) return fail(BITNET_ERR_INVALID_ARG, "pack: eps must be >= 0");
    if (!aligned(W, 16) || !aligned(ws, 16)) return fail(BITNET_ERR_INVALID_ARG, "pack: W and ws must be 16-byte aligned");
    if (static_cast<double>(n_out) * static_cast<double>(k) / 4.0 > 4294967295.0)
        return fail(BITNET_ERR_UNSUPPORTED, "pack: more than 2^32 groups of 4 in one matrix");
    const bool packed = out->group_bytes || out->mma_vals || out->mma_meta || out->dec_codes;
    if (packed && !(n == 2 && m == 4)) return fail(BITNET_ERR_UNSUPPORTED, "pack: packed layouts exist for 2:4 only");
    if ((out->mma_vals == nullptr) != (out->mma_meta == nullptr))
        return fail(BITNET_ERR_INVALID_ARG, "pack: mma_vals and mma_meta go together");
    if (out->mma_vals && (!aligned(out->mma_vals, 16) || !aligned(out->mma_meta, 16)))
        return fail(BITNET_ERR_INVALID_ARG, "pack: mma layouts must be 16-byte aligned");
    if (out->dec_codes) {
        if (!out->group_bytes) return fail(BITNET_ERR_INVALID_ARG, "pack: dec_codes are derived from group_bytes");
        if (n_out % 16 || k % 64) return fail(BITNET_ERR_UNSUPPORTED, "pack: dec_codes need n_out %% 16 == 0, k %% 64 == 0");
        if (!aligned(out->dec_codes, 16)) return fail(BITNET_ERR_INVALID_ARG, "pack: dec_codes must be 16-byte aligned");
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return cuda_status(bitnet::launch_pack(W, n_out, k, n, m, eps, out->gamma, out->group_bytes, out->mma_vals,
                                           out->mma_meta, out->dec_codes, mask_bits, ws, s),
                       "pack");
}

size_t bitnet_pack_update_workspace_size(int64_t n_out, int64_t k) {
    if (n_out <= 0 || k <= 0) return bitnet::kPackWsBytes;
    return bitnet::kPackWsBytes + bitnet::update_list_bytes(n_out, k);
}

bitnet_status bitnet_pack_nm_update(const float *W, bitnet_packed_w *out, float eps, uint8_t *mask_bits, void *ws,
                                    size_t ws_bytes, bitnet_stream_t stream) {
    if (!W || !out || !out->gamma) return fail(BITNET_ERR_INVALID_ARG, "pack_update: W, out and out->gamma are required");
    if (!ws) return fail(BITNET_ERR_WORKSPACE, "pack_update: workspace is required");
    const int64_t n_out = out->n_out, k = out->k;
    if (n_out <= 0 || k <= 0 || k % 8) return fail(BITNET_ERR_INVALID_ARG, "pack_update: bad sizes (k %% 8 == 0)");
    if (!(out->n == 2 && out->m == 4)) return fail(BITNET_ERR_UNSUPPORTED, "pack_update: 2:4 only");
    if (ws_bytes < bitnet::kPackWsBytes + 4) return fail(BITNET_ERR_WORKSPACE, "pack_update: workspace needs >= %zu bytes", bitnet::kPackWsBytes + 4);
    if (!(eps >= 0.0f)) return fail(BITNET_ERR_INVALID_ARG, "pack_update: eps must be >= 0");
    if (!aligned(W, 16) || !aligned(ws, 16)) return fail(BITNET_ERR_INVALID_ARG, "pack_update: W and ws must be 16-byte aligned");
    if ((out->mma_vals == nullptr) != (out->mma_meta == nullptr))
        return fail(BITNET_ERR_INVALID_ARG, "pack_update: mma_vals and mma_meta go together");
    if (out->dec_codes && (!out->group_bytes || n_out % 16 || k % 64))
        return fail(BITNET_ERR_INVALID_ARG, "pack_update: dec_codes need group_bytes, n_out %% 16 == 0, k %% 64 == 0");
    if (static_cast<double>(n_out) * static_cast<double>(k) / 4.0 > 4294967295.0)
        return fail(BITNET_ERR_UNSUPPORTED, "pack_update: more than 2^32 groups");
    return cuda_status(bitnet::launch_pack_update(W, n_out, k, eps, out->gamma, out->group_bytes, out->mma_vals,
                                                  out->mma_meta, out->dec_codes, mask_bits, ws, ws_bytes,
                                                  reinterpret_cast<cudaStream_t>(stream)),
                       "pack_update");
}

size_t bitnet_pack_update_batch_workspace_size(const bitnet_pack_item *items, int32_t n_items) {
    if (!items || n_items <= 0) return 256;
    std::vector<int64_t> n_out(static_cast<size_t>(n_items)), k(static_cast<size_t>(n_items));
    for (int32_t i = 0; i < n_items; ++i) {
        const bitnet_packed_w *o = items[i].out;
        n_out[static_cast<size_t>(i)] = (o && o->n_out > 0) ? o->n_out : 0;
        k[static_cast<size_t>(i)] = (o && o->k > 0) ? o->k : 0;
    }
    return bitnet::pack_batch_ws_bytes(n_out.data(), k.data(), n_items);
}

bitnet_status bitnet_pack_nm_update_batch(const bitnet_pack_item *items, int32_t n_items, float eps, void *ws,
                                          size_t ws_bytes, bitnet_stream_t stream) {
    if (n_items < 0) return fail(BITNET_ERR_INVALID_ARG, "pack_update_batch: n_items < 0");
    if (n_items == 0) return BITNET_OK;
    if (!items) return fail(BITNET_ERR_INVALID_ARG, "pack_update_batch: null items");
    if (!(eps >= 0.0f)) return fail(BITNET_ERR_INVALID_ARG, "pack_update_batch: eps must be >= 0");
    if (!ws) return fail(BITNET_ERR_WORKSPACE, "pack_update_batch: workspace is required");
    if (!aligned(ws, 16)) return fail(BITNET_ERR_INVALID_ARG, "pack_update_batch: ws must be 16-byte aligned");
    std::vector<bitnet::PackBatchItemHost> h(static_cast<size_t>(n_items));
    for (int32_t i = 0; i < n_items; ++i) {
        const bitnet_pack_item &it = items[i];
        const bitnet_packed_w *out = it.out;
        if (!it.W || !out || !out->gamma)
            return fail(BITNET_ERR_INVALID_ARG, "pack_update_batch: item %d: W, out and out->gamma are required", i);
        const int64_t n_out = out->n_out, k = out->k;
        if (n_out <= 0 || k <= 0 || k % 8) return fail(BITNET_ERR_INVALID_ARG, "pack_update_batch: item %d: bad sizes", i);
        if (!(out->n == 2 && out->m == 4)) return fail(BITNET_ERR_UNSUPPORTED, "pack_update_batch: item %d: 2:4 only", i);
        if (k % 16) return fail(BITNET_ERR_UNSUPPORTED, "pack_update_batch: item %d: k %% 16 != 0", i);
        if (it.w_dtype != BITNET_F32 && it.w_dtype != BITNET_BF16)
            return fail(BITNET_ERR_INVALID_ARG, "pack_update_batch: item %d: bad w_dtype", i);
        if (!aligned(it.W, 16)) return fail(BITNET_ERR_INVALID_ARG, "pack_update_batch: item %d: W must be 16-byte aligned", i);
        if ((out->mma_vals == nullptr) != (out->mma_meta == nullptr))
            return fail(BITNET_ERR_INVALID_ARG, "pack_update_batch: item %d: mma_vals and mma_meta go together", i);
        if (out->dec_codes && (!out->group_bytes || n_out % 16 || k % 64))
            return fail(BITNET_ERR_INVALID_ARG,
                        "pack_update_batch: item %d: dec_codes need group_bytes, n_out %% 16 == 0, k %% 64 == 0", i);
        if (static_cast<double>(n_out) * static_cast<double>(k) / 4.0 > 4294967295.0)
            return fail(BITNET_ERR_UNSUPPORTED, "pack_update_batch: item %d: more than 2^32 groups", i);
        h[static_cast<size_t>(i)] = {it.W, n_out, k, out->gamma, out->group_bytes, out->mma_vals, out->mma_meta,
                                     out->dec_codes, it.mask_bits, it.w_dtype == BITNET_BF16, it.gamma_known != 0};
    }
    const size_t need = bitnet_pack_update_batch_workspace_size(items, n_items);
    if (ws_bytes < need) return fail(BITNET_ERR_WORKSPACE, "pack_update_batch: workspace needs %zu bytes", need);
    double total_chunks = 0.0;
    for (const auto &x : h) total_chunks += std::ceil(static_cast<double>(x.n_out) * static_cast<double>(x.k) / 8192.0);
    if (total_chunks > 4294967295.0) return fail(BITNET_ERR_UNSUPPORTED, "pack_update_batch: too many weights in one call");
    return cuda_status(bitnet::launch_pack_update_batch(h.data(), n_items, eps, ws,
                                                        reinterpret_cast<cudaStream_t>(stream)),
                       "pack_update_batch");
}

bitnet_status bitnet_pack_6of8_windows(const float *W, int64_t k, float eps, bitnet_packed_w *out, uint8_t *mask_bits,
                                       void *ws, size_t ws_bytes, bitnet_stream_t stream) {
    if (!W || !out || !out->gamma || !out->group_bytes)
        return fail(BITNET_ERR_INVALID_ARG, "pack_6of8: W, out, out->gamma and out->group_bytes are required");
    if (!ws) return fail(BITNET_ERR_WORKSPACE, "pack_6of8: workspace is required");
    const int64_t n_out = out->n_out;
    if (n_out <= 0 || k <= 0) return fail(BITNET_ERR_INVALID_ARG, "pack_6of8: bad sizes");
    if (k % 64) return fail(BITNET_ERR_UNSUPPORTED, "pack_6of8: k %% 64 != 0");
    if (out->k != k / 2 * 3 || !(out->n == 2 && out->m == 4))
        return fail(BITNET_ERR_INVALID_ARG, "pack_6of8: out must describe the 2:4 window layout (k = k/2*3, n = 2, m = 4)");
    if (ws_bytes < bitnet::kPackWsBytes) return fail(BITNET_ERR_WORKSPACE, "pack_6of8: workspace needs >= %zu bytes", bitnet::kPackWsBytes);
    if (!(eps >= 0.0f)) return fail(BITNET_ERR_INVALID_ARG, "pack_6of8: eps must be >= 0");
    if (!aligned(W, 16) || !aligned(ws, 16) || !aligned(out->group_bytes, 4))
        return fail(BITNET_ERR_INVALID_ARG, "pack_6of8: W and ws 16-byte, group_bytes 4-byte aligned");
    if ((out->mma_vals == nullptr) != (out->mma_meta == nullptr))
        return fail(BITNET_ERR_INVALID_ARG, "pack_6of8: mma_vals and mma_meta go together");
    if (out->dec_codes && (n_out % 16 || k % 128))
        return fail(BITNET_ERR_INVALID_ARG, "pack_6of8: dec_codes need n_out %% 16 == 0 and k %% 128 == 0");
    if (static_cast<double>(n_out) * static_cast<double>(k) / 8.0 * 3.0 > 4294967295.0)
        return fail(BITNET_ERR_UNSUPPORTED, "pack_6of8: more than 2^32 window groups");
    return cuda_status(bitnet::launch_pack68(W, n_out, k, eps, out->gamma, out->group_bytes, out->mma_vals,
                                             out->mma_meta, out->dec_codes, mask_bits, ws,
                                             reinterpret_cast<cudaStream_t>(stream)),
                       "pack_6of8");
}

bitnet_status bitnet_quant_act_lift_6of8(const void *X, bitnet_dtype x_dtype, int64_t T, int64_t K, float eps,
                                         int8_t *Xl, float *absmax, bitnet_stream_t stream) {
    if (T < 0 || K <= 0 || K % 8) return fail(BITNET_ERR_INVALID_ARG, "quant_lift: need T >= 0, K > 0, K %% 8 == 0");
    if (T == 0) return BITNET_OK;
    if (!X || !Xl || !absmax) return fail(BITNET_ERR_INVALID_ARG, "quant_lift: null pointer");
    if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return fail(BITNET_ERR_INVALID_ARG, "quant_lift: bad dtype");
    if (!aligned(X, 16) || !aligned(Xl, 16)) return fail(BITNET_ERR_INVALID_ARG, "quant_lift: X and Xl must be 16-byte aligned");
    if (!(eps > 0.0f)) return fail(BITNET_ERR_INVALID_ARG, "quant_lift: eps must be > 0");
    if (T > 2147483647LL) return fail(BITNET_ERR_UNSUPPORTED, "quant_lift: T too large");
    return cuda_status(bitnet::launch_quant_lift68(X, x_dtype == BITNET_BF16, T, K, eps, Xl, absmax,
                                                   reinterpret_cast<cudaStream_t>(stream)),
                       "quant_lift");
}

bitnet_status bitnet_quant_act(const void *X, bitnet_dtype x_dtype, int64_t T, int64_t K, float eps, int8_t *Xq,
                               float *absmax, bitnet_stream_t stream) {
    if (T < 0 || K <= 0 || K % 8) return fail(BITNET_ERR_INVALID_ARG, "quant_act: need T >= 0, K > 0, K %% 8 == 0");
    if (T == 0) return BITNET_OK;   // an empty batch needs no buffers
    if (!X || !Xq || !absmax) return fail(BITNET_ERR_INVALID_ARG, "quant_act: null pointer");
    if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return fail(BITNET_ERR_INVALID_ARG, "quant_act: bad dtype");
    if (!aligned(X, 16) || !aligned(Xq, 16)) return fail(BITNET_ERR_INVALID_ARG, "quant_act: X and Xq must be 16-byte aligned");
    if (!(eps > 0.0f)) return fail(BITNET_ERR_INVALID_ARG, "quant_act: eps must be > 0");
    if (T > 2147483647LL) return fail(BITNET_ERR_UNSUPPORTED, "quant_act: T too large");
    return cuda_status(bitnet::launch_quant_act(X, x_dtype == BITNET_BF16, T, K, eps, Xq, absmax,
                                                reinterpret_cast<cudaStream_t>(stream)),
                       "quant_act");
}

size_t bitnet_wgrad_workspace_size(void) { return bitnet::kDgradWsHeader; }

bitnet_status bitnet_wgrad(const void *dY, const void *X, int64_t T, int64_t n_out, int64_t k, float *dW,
                           int32_t accumulate, void *ws, size_t ws_bytes, bitnet_stream_t stream) {
    if (T < 0 || n_out <= 0 || k <= 0 || n_out % 8 || k % 8)
        return fail(BITNET_ERR_INVALID_ARG, "wgrad: need T >= 0, n_out and k positive multiples of 8");
    if (!dW) return fail(BITNET_ERR_INVALID_ARG, "wgrad: null dW");
    if (!ws) return fail(BITNET_ERR_WORKSPACE, "wgrad: workspace is required");
    if (ws_bytes < bitnet_wgrad_workspace_size()) return fail(BITNET_ERR_WORKSPACE, "wgrad: workspace needs %zu bytes", bitnet_wgrad_workspace_size());
    if (!aligned(dW, 16) || !aligned(ws, 16)) return fail(BITNET_ERR_INVALID_ARG, "wgrad: dW and ws must be 16-byte aligned");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (T == 0) {   // an empty sum: dW = 0, or unchanged when accumulating
        if (accumulate) return BITNET_OK;
        return cuda_status(cudaMemsetAsync(dW, 0, static_cast<size_t>(n_out) * static_cast<size_t>(k) * 4, s), "wgrad");
    }
    if (!dY || !X) return fail(BITNET_ERR_INVALID_ARG, "wgrad: null dY or X");
    if (!aligned(dY, 16) || !aligned(X, 16)) return fail(BITNET_ERR_INVALID_ARG, "wgrad: dY and X must be 16-byte aligned");
    if (T > 2147483647LL) return fail(BITNET_ERR_UNSUPPORTED, "wgrad: T too large");
    return cuda_status(bitnet::launch_gemm_wgrad_pair(dY, X, T, n_out, k, dW, accumulate != 0,
                                                      reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + bitnet::kStatusOffset), s),
                       "wgrad");
}

size_t bitnet_adamw_workspace_size(void) { return bitnet::kPackWsBytes; }

bitnet_status bitnet_adamw_step(float *W, const float *dW, float *m, float *v, int64_t n,
                                const bitnet_adamw_hparams *h, float eps_gamma, float *gamma_out, void *ws,
                                size_t ws_bytes, bitnet_stream_t stream) {
    if (!h) return fail(BITNET_ERR_INVALID_ARG, "adamw: null hyper-parameters");
    if (n <= 0 || n % 4) return fail(BITNET_ERR_INVALID_ARG, "adamw: n must be a positive multiple of 4");
    if (!W || !dW || !m || !v || !gamma_out) return fail(BITNET_ERR_INVALID_ARG, "adamw: null pointer");
    if (!ws) return fail(BITNET_ERR_WORKSPACE, "adamw: workspace is required");
    if (ws_bytes < bitnet_adamw_workspace_size()) return fail(BITNET_ERR_WORKSPACE, "adamw: workspace needs %zu bytes", bitnet_adamw_workspace_size());
    if (!aligned(W, 16) || !aligned(dW, 16) || !aligned(m, 16) || !aligned(v, 16) || !aligned(ws, 16))
        return fail(BITNET_ERR_INVALID_ARG, "adamw: W, dW, m, v and ws must be 16-byte aligned");
    if (!(h->lr >= 0.0f) || !(h->beta1 >= 0.0f && h->beta1 < 1.0f) || !(h->beta2 >= 0.0f && h->beta2 < 1.0f) ||
        !(h->eps > 0.0f) || !(h->weight_decay >= 0.0f) || !(h->bias_correction1 > 0.0f) ||
        !(h->bias_correction2 > 0.0f) || !(eps_gamma >= 0.0f))
        return fail(BITNET_ERR_INVALID_ARG, "adamw: hyper-parameters out of range");
    return cuda_status(bitnet::launch_adamw_gamma(W, dW, m, v, n, h->lr, h->beta1, h->beta2, h->eps, h->weight_decay,
                                                  h->bias_correction1, h->bias_correction2, eps_gamma, gamma_out, ws,
                                                  reinterpret_cast<cudaStream_t>(stream)),
                       "adamw");
}

size_t bitnet_adamw_batch_workspace_size(int32_t n_items) {
    return n_items > 0 ? static_cast<size_t>(n_items) * bitnet::kPackWsBytes : 0;
}

bitnet_status bitnet_adamw_step_batch(const bitnet_adamw_item *items, int32_t n_items, const bitnet_adamw_hparams *h,
                                      float eps_gamma, void *ws, size_t ws_bytes, bitnet_stream_t stream) {
    if (n_items < 0) return fail(BITNET_ERR_INVALID_ARG, "adamw_batch: n_items < 0");
    if (n_items == 0) return BITNET_OK;
    if (!items || !h) return fail(BITNET_ERR_INVALID_ARG, "adamw_batch: null items or hyper-parameters");
    if (!(h->lr >= 0.0f) || !(h->beta1 >= 0.0f && h->beta1 < 1.0f) || !(h->beta2 >= 0.0f && h->beta2 < 1.0f) ||
        !(h->eps > 0.0f) || !(h->weight_decay >= 0.0f) || !(h->bias_correction1 > 0.0f) ||
        !(h->bias_correction2 > 0.0f) || !(eps_gamma >= 0.0f))
        return fail(BITNET_ERR_INVALID_ARG, "adamw_batch: hyper-parameters out of range");
    if (!ws) return fail(BITNET_ERR_WORKSPACE, "adamw_batch: workspace is required");
    if (ws_bytes < bitnet_adamw_batch_workspace_size(n_items))
        return fail(BITNET_ERR_WORKSPACE, "adamw_batch: workspace needs %zu bytes", bitnet_adamw_batch_workspace_size(n_items));
    if (!aligned(ws, 16)) return fail(BITNET_ERR_INVALID_ARG, "adamw_batch: ws must be 16-byte aligned");
    std::vector<bitnet::AdamWItemHost> hv(static_cast<size_t>(n_items));
    double total_chunks = 0.0;
    for (int32_t i = 0; i < n_items; ++i) {
        const bitnet_adamw_item &it = items[i];
        if (it.n <= 0 || it.n % 4) return fail(BITNET_ERR_INVALID_ARG, "adamw_batch: item %d: n must be a positive multiple of 4", i);
        if (!it.W || !it.dW || !it.m || !it.v || !it.gamma_out)
            return fail(BITNET_ERR_INVALID_ARG, "adamw_batch: item %d: null pointer", i);
        if (!aligned(it.W, 16) || !aligned(it.dW, 16) || !aligned(it.m, 16) || !aligned(it.v, 16))
            return fail(BITNET_ERR_INVALID_ARG, "adamw_batch: item %d: W, dW, m, v must be 16-byte aligned", i);
        total_chunks += std::ceil(static_cast<double>(it.n) / 8192.0);
        hv[static_cast<size_t>(i)] = {it.W, it.dW, it.m, it.v, it.n, it.gamma_out};
    }
    if (total_chunks > 4294967295.0) return fail(BITNET_ERR_UNSUPPORTED, "adamw_batch: too many weights in one call");
    return cuda_status(bitnet::launch_adamw_gamma_batch(hv.data(), n_items, h->lr, h->beta1, h->beta2, h->eps,
                                                        h->weight_decay, h->bias_correction1, h->bias_correction2,
                                                        eps_gamma, ws, reinterpret_cast<cudaStream_t>(stream)),
                       "adamw_batch");
}

bitnet_status bitnet_rmsnorm_quant(const void *X, const float *w, int64_t T, int64_t K, float eps_norm,
                                   float eps_act, int8_t *Xq, float *absmax, float *rinv, bitnet_stream_t stream) {
    if (T < 0 || K <= 0 || K % 8 || K > 65536) return fail(BITNET_ERR_INVALID_ARG, "rmsnorm_quant: need T >= 0, 0 < K <= 65536, K %% 8 == 0");
    if (!(eps_norm > 0.0f) || !(eps_act > 0.0f)) return fail(BITNET_ERR_INVALID_ARG, "rmsnorm_quant: eps must be > 0");
    if (T == 0) return BITNET_OK;
    if (!X || !Xq || !absmax) return fail(BITNET_ERR_INVALID_ARG, "rmsnorm_quant: null pointer");
    if (!aligned(X, 16) || !aligned(Xq, 16)) return fail(BITNET_ERR_INVALID_ARG, "rmsnorm_quant: X and Xq must be 16-byte aligned");
    if (w && !aligned(w, 4)) return fail(BITNET_ERR_INVALID_ARG, "rmsnorm_quant: w must be 4-byte aligned");
    if (T > 2147483647LL) return fail(BITNET_ERR_UNSUPPORTED, "rmsnorm_quant: T too large");
    return cuda_status(bitnet::launch_rmsnorm_quant(X, w, T, K, eps_norm, eps_act, Xq, absmax, rinv,
                                                    reinterpret_cast<cudaStream_t>(stream)),
                       "rmsnorm_quant");
}

bitnet_status bitnet_swiglu_quant(const void *G, const void *U, int64_t ld, int64_t T, int64_t F, float eps_act,
                                  int8_t *Xq, float *absmax, bitnet_stream_t stream) {
    if (T < 0 || F <= 0 || F % 8 || ld < F) return fail(BITNET_ERR_INVALID_ARG, "swiglu_quant: need T >= 0, F > 0, F %% 8 == 0, ld >= F");
    if (bitnet::swiglu_smem_bytes(F) > bitnet::kSwigluMaxSmem) return fail(BITNET_ERR_INVALID_ARG, "swiglu_quant: F too large");
    if (!(eps_act > 0.0f)) return fail(BITNET_ERR_INVALID_ARG, "swiglu_quant: eps must be > 0");
    if (T == 0) return BITNET_OK;
    if (!G || !U || !Xq || !absmax) return fail(BITNET_ERR_INVALID_ARG, "swiglu_quant: null pointer");
    if (!aligned(G, 2) || !aligned(U, 2) || !aligned(Xq, 16)) return fail(BITNET_ERR_INVALID_ARG, "swiglu_quant: alignment");
    if (T > 2147483647LL) return fail(BITNET_ERR_UNSUPPORTED, "swiglu_quant: T too large");
    return cuda_status(bitnet::launch_swiglu_quant(G, U, ld, T, F, eps_act, Xq, absmax,
                                                   reinterpret_cast<cudaStream_t>(stream)),
                       "swiglu_quant");
}

bitnet_status bitnet_sparse_linear(const int8_t *Xq, const float *absmax, const bitnet_packed_w *W, int64_t T,
                                   void *Y, bitnet_dtype y_dtype, int32_t *acc_out, void *ws, size_t ws_bytes,
                                   bitnet_stream_t stream) {
    if (!W || !W->gamma) return fail(BITNET_ERR_INVALID_ARG, "sparse_linear: null W or gamma");
    if (T != 0 && (!Xq || !absmax || !Y)) return fail(BITNET_ERR_INVALID_ARG, "sparse_linear: null pointer");
    if (!ws) return fail(BITNET_ERR_WORKSPACE, "sparse_linear: workspace is required");
    if (ws_bytes < bitnet::kLinearWsBytes) return fail(BITNET_ERR_WORKSPACE, "sparse_linear: workspace needs %zu bytes", bitnet::kLinearWsBytes);
    if (y_dtype != BITNET_F32 && y_dtype != BITNET_BF16) return fail(BITNET_ERR_INVALID_ARG, "sparse_linear: bad dtype");
    const int64_t n_out = W->n_out, k = W->k;
    if (T < 0 || n_out <= 0 || k <= 0 || k % 8) return fail(BITNET_ERR_INVALID_ARG, "sparse_linear: bad sizes");
    if (!(W->n == 2 && W->m == 4)) return fail(BITNET_ERR_UNSUPPORTED, "sparse_linear: 2:4 only");
    if (T == 0) return BITNET_OK;   // an empty batch needs no buffers
    if (!aligned(Xq, 16) || !aligned(ws, 16)) return fail(BITNET_ERR_INVALID_ARG, "sparse_linear: Xq and ws must be 16-byte aligned");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool bf16 = y_dtype == BITNET_BF16;
    if (T <= 8) {
        if (W->dec_codes && n_out % 16 == 0 && k % 64 == 0) {
            if (!aligned(W->dec_codes, 16)) return fail(BITNET_ERR_INVALID_ARG, "sparse_linear: dec_codes alignment");
            return cuda_status(bitnet::launch_gemv_dec(Xq, absmax, W->gamma, W->dec_codes, T, n_out, k, Y, bf16,
                                                       acc_out, s),
                               "sparse_linear (decode GEMV)");
        }
        if (W->group_bytes)
            return cuda_status(bitnet::launch_gemv_gb(Xq, absmax, W->gamma, W->group_bytes, T, n_out, k, Y, bf16,
                                                      acc_out, s),
                               "sparse_linear (group-byte GEMV)");
        if (!W->mma_vals) return fail(BITNET_ERR_INVALID_ARG, "sparse_linear: no packed layout for T <= 8");
    }
    if (!W->mma_vals || !W->mma_meta) return fail(BITNET_ERR_INVALID_ARG, "sparse_linear: T > 8 needs mma_vals and mma_meta");
    if (k % 32) return fail(BITNET_ERR_UNSUPPORTED, "sparse_linear: the tensor-core path needs k %% 32 == 0");
    if (!aligned(W->mma_vals, 16) || !aligned(W->mma_meta, 16)) return fail(BITNET_ERR_INVALID_ARG, "sparse_linear: mma layouts must be 16-byte aligned");
    if (n_out > 2147483647LL / 2 || T > 65535LL * 256) return fail(BITNET_ERR_UNSUPPORTED, "sparse_linear: sizes too large");
    uint32_t *status = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + bitnet::kStatusOffset);
    return cuda_status(bitnet::launch_gemm_sp(Xq, absmax, W->gamma, W->mma_vals, W->mma_meta, T, n_out, k, Y, bf16,
                                              acc_out, status, s),
                       "sparse_linear (tensor-core GEMM)");
}

static size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// The decode chain's shared memory holds the activations of one projection
// (T rows of k), the weight ring and the partial sums of the CTA's row tiles.
static bool chain_fits(int64_t T, int64_t kmax, bool x_bf16, int64_t n_out_max) {
    const int64_t G = bitnet::num_sms();
    const int64_t tiles = (n_out_max / 16 + G - 1) / G;
    if (tiles > bitnet::kChainMaxTiles) return false;
    bitnet::ChainLayout L;
    return bitnet::chain_layout(T, kmax, x_bf16, static_cast<int>(tiles < 1 ? 1 : tiles), &L);
}

size_t bitnet_quant_linear_workspace_size(int64_t T, int64_t K) {
    if (T <= 0 || K <= 0) return bitnet::kLinearWsBytes;
    return bitnet::kLinearWsBytes + align256(static_cast<size_t>(T) * static_cast<size_t>(K)) +
           align256(static_cast<size_t>(T) * 4);
}

bitnet_status bitnet_quant_linear(const void *X, bitnet_dtype x_dtype, float eps, const bitnet_packed_w *W,
                                  int64_t T, void *Y, bitnet_dtype y_dtype, int32_t *acc_out, int8_t *xq_out,
                                  float *absmax_out, void *ws, size_t ws_bytes, bitnet_stream_t stream) {
    if (!W || !W->gamma) return fail(BITNET_ERR_INVALID_ARG, "quant_linear: null W or gamma");
    if (T < 0) return fail(BITNET_ERR_INVALID_ARG, "quant_linear: T < 0");
    if (T != 0 && (!X || !Y)) return fail(BITNET_ERR_INVALID_ARG, "quant_linear: null pointer");
    if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return fail(BITNET_ERR_INVALID_ARG, "quant_linear: bad x dtype");
    if (y_dtype != BITNET_F32 && y_dtype != BITNET_BF16) return fail(BITNET_ERR_INVALID_ARG, "quant_linear: bad y dtype");
    if (!(eps > 0.0f)) return fail(BITNET_ERR_INVALID_ARG, "quant_linear: eps must be > 0");
    const int64_t n_out = W->n_out, k = W->k;
    if (n_out <= 0 || k <= 0 || k % 8) return fail(BITNET_ERR_INVALID_ARG, "quant_linear: bad sizes");
    if (!(W->n == 2 && W->m == 4)) return fail(BITNET_ERR_UNSUPPORTED, "quant_linear: 2:4 only");
    if (!ws) return fail(BITNET_ERR_WORKSPACE, "quant_linear: workspace is required");
    if (ws_bytes < bitnet_quant_linear_workspace_size(T, k))
        return fail(BITNET_ERR_WORKSPACE, "quant_linear: workspace needs %zu bytes", bitnet_quant_linear_workspace_size(T, k));
    if (T == 0) return BITNET_OK;   // an empty batch needs no buffers
    if (!aligned(X, 16) || !aligned(ws, 16)) return fail(BITNET_ERR_INVALID_ARG, "quant_linear: X and ws must be 16-byte aligned");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool xb = x_dtype == BITNET_BF16, yb = y_dtype == BITNET_BF16;
    if (T <= 8 && W->dec_codes && n_out % 16 == 0 && k % 64 == 0 && k <= bitnet::kChainMaxK &&
        n_out / 16 <= bitnet::kChainMaxTiles * bitnet::num_sms() && chain_fits(T, k, xb, n_out) &&
        ws_bytes >= bitnet_decode_chain_workspace_size(1)) {
        if (!aligned(W->dec_codes, 16)) return fail(BITNET_ERR_INVALID_ARG, "quant_linear: dec_codes alignment");
        bitnet::ChainOpDev op = {X, W->dec_codes, W->gamma, Y, acc_out, xq_out, absmax_out,
                                 static_cast<int32_t>(n_out), static_cast<int32_t>(k), 0, 0};
        return cuda_status(bitnet::launch_decode_chain(&op, 1, T, xb, yb, eps, k, ws, s),
                           "quant_linear (decode chain of one projection)");
    }
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    int8_t *xq = reinterpret_cast<int8_t *>(w8 + bitnet::kLinearWsBytes);
    float *am = reinterpret_cast<float *>(w8 + bitnet::kLinearWsBytes + align256(static_cast<size_t>(T) * k));
    bitnet_status st = bitnet_quant_act(X, x_dtype, T, k, eps, xq, am, stream);
    if (st != BITNET_OK) return st;
    st = bitnet_sparse_linear(xq, am, W, T, Y, y_dtype, acc_out, ws, ws_bytes, stream);
    if (st != BITNET_OK) return st;
    if (xq_out) {
        cudaError_t e = cudaMemcpyAsync(xq_out, xq, static_cast<size_t>(T) * k, cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return cuda_status(e, "quant_linear copy");
    }
    if (absmax_out) {
        cudaError_t e = cudaMemcpyAsync(absmax_out, am, static_cast<size_t>(T) * 4, cudaMemcpyDeviceToDevice, s);
        if (e != cudaSuccess) return cuda_status(e, "quant_linear copy");
    }
    return BITNET_OK;
}

size_t bitnet_decode_chain_workspace_size(int32_t n_ops) {
    const size_t n = n_ops > 0 ? static_cast<size_t>(n_ops) : 0;
    return bitnet::kChainCountersOffset + align256(4 * n);
}

bitnet_status bitnet_decode_chain(const bitnet_chain_op *ops, int32_t n_ops, int64_t T, bitnet_dtype x_dtype,
                                  bitnet_dtype y_dtype, float eps, void *ws, size_t ws_bytes, bitnet_stream_t stream) {
    if (n_ops < 0) return fail(BITNET_ERR_INVALID_ARG, "decode_chain: n_ops < 0");
    if (T < 0 || T > 8) return fail(BITNET_ERR_INVALID_ARG, "decode_chain: T must be in 0..8");
    if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return fail(BITNET_ERR_INVALID_ARG, "decode_chain: bad x dtype");
    if (y_dtype != BITNET_F32 && y_dtype != BITNET_BF16) return fail(BITNET_ERR_INVALID_ARG, "decode_chain: bad y dtype");
    if (!(eps > 0.0f)) return fail(BITNET_ERR_INVALID_ARG, "decode_chain: eps must be > 0");
    if (n_ops == 0 || T == 0) return BITNET_OK;
    if (!ops) return fail(BITNET_ERR_INVALID_ARG, "decode_chain: null ops");
    if (!ws) return fail(BITNET_ERR_WORKSPACE, "decode_chain: workspace is required");
    if (ws_bytes < bitnet_decode_chain_workspace_size(n_ops))
        return fail(BITNET_ERR_WORKSPACE, "decode_chain: workspace needs %zu bytes",
                    bitnet_decode_chain_workspace_size(n_ops));
    if (!aligned(ws, 16)) return fail(BITNET_ERR_INVALID_ARG, "decode_chain: ws must be 16-byte aligned");
    const int64_t max_tiles = static_cast<int64_t>(bitnet::kChainMaxTiles) * bitnet::num_sms();
    std::vector<bitnet::ChainOpDev> dev(static_cast<size_t>(n_ops));
    int64_t kmax = 0, nmax = 0;
    for (int32_t i = 0; i < n_ops; ++i) {
        const bitnet_chain_op &o = ops[i];
        const bitnet_packed_w *W = o.W;
        if (!W || !W->gamma || !W->dec_codes) return fail(BITNET_ERR_INVALID_ARG, "decode_chain: op %d: null W, gamma or dec_codes", i);
        if (!(W->n == 2 && W->m == 4)) return fail(BITNET_ERR_UNSUPPORTED, "decode_chain: op %d: 2:4 only", i);
        if (W->n_out <= 0 || W->k <= 0 || W->n_out % 16 || W->k % 64)
            return fail(BITNET_ERR_UNSUPPORTED, "decode_chain: op %d: needs n_out %% 16 == 0 and k %% 64 == 0", i);
        if (W->n_out / 16 > max_tiles || W->n_out > INT32_MAX || W->k > bitnet::kChainMaxK)
            return fail(BITNET_ERR_UNSUPPORTED, "decode_chain: op %d: n_out above 512 rows per SM or k above %d", i,
                        bitnet::kChainMaxK);
        if (!o.X || !o.Y) return fail(BITNET_ERR_INVALID_ARG, "decode_chain: op %d: null X or Y", i);
        if (!aligned(o.X, 16) || !aligned(W->dec_codes, 16))
            return fail(BITNET_ERR_INVALID_ARG, "decode_chain: op %d: X and dec_codes must be 16-byte aligned", i);
        if (o.wait_prev != 0 && o.wait_prev != 1) return fail(BITNET_ERR_INVALID_ARG, "decode_chain: op %d: wait_prev must be 0 or 1", i);
        kmax = W->k > kmax ? W->k : kmax;
        nmax = W->n_out > nmax ? W->n_out : nmax;
        dev[static_cast<size_t>(i)] = {o.X, W->dec_codes, W->gamma, o.Y, o.acc_out, o.xq_out, o.absmax_out,
                                       static_cast<int32_t>(W->n_out), static_cast<int32_t>(W->k), o.wait_prev, 0};
    }
    bool any_wait = false;
    for (int32_t i = 1; i < n_ops; ++i) any_wait = any_wait || ops[i].wait_prev != 0;
    if (any_wait ? !bitnet::chain_serial_fits(T, kmax) : !chain_fits(T, kmax, x_dtype == BITNET_BF16, nmax))
        return fail(BITNET_ERR_UNSUPPORTED, "decode_chain: the activations of the largest k and two weight stages do "
                                            "not fit in shared memory");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return cuda_status(bitnet::launch_decode_chain(dev.data(), n_ops, T, x_dtype == BITNET_BF16, y_dtype == BITNET_BF16,
                                                   eps, kmax, ws, s),
                       "decode_chain");
}

bitnet_status bitnet_dgrad(const void *dY, bitnet_dtype dy_dtype, const bitnet_packed_w *W, int64_t T, void *dX,
                           bitnet_dtype dx_dtype, void *ws, size_t ws_bytes, bitnet_stream_t stream) {
    if (!W || !W->gamma) return fail(BITNET_ERR_INVALID_ARG, "dgrad: null W or gamma");
    if (T != 0 && (!dY || !dX)) return fail(BITNET_ERR_INVALID_ARG, "dgrad: null pointer");
    if (!W->group_bytes) return fail(BITNET_ERR_INVALID_ARG, "dgrad: needs W->group_bytes");
    if (dy_dtype != BITNET_BF16) return fail(BITNET_ERR_UNSUPPORTED, "dgrad: dY must be bf16");
    if (dx_dtype != BITNET_F32 && dx_dtype != BITNET_BF16) return fail(BITNET_ERR_INVALID_ARG, "dgrad: bad dX dtype");
    const int64_t n_out = W->n_out, k = W->k;
    if (T < 0 || n_out <= 0 || k <= 0 || k % 8 || n_out % 8) return fail(BITNET_ERR_INVALID_ARG, "dgrad: bad sizes (k, n_out multiples of 8)");
    if (!(W->n == 2 && W->m == 4)) return fail(BITNET_ERR_UNSUPPORTED, "dgrad: 2:4 only");
    if (!ws) return fail(BITNET_ERR_WORKSPACE, "dgrad: workspace is required");
    if (ws_bytes < bitnet_dgrad_workspace_size(n_out, k)) return fail(BITNET_ERR_WORKSPACE, "dgrad: workspace needs %zu bytes", bitnet_dgrad_workspace_size(n_out, k));
    if (T == 0) return BITNET_OK;   // an empty batch needs no buffers
    if (!aligned(dY, 16) || !aligned(dX, 16) || !aligned(ws, 128)) return fail(BITNET_ERR_INVALID_ARG, "dgrad: dY, dX 16-byte and ws 128-byte alignment");
    if (T > 65535LL * 128) return fail(BITNET_ERR_UNSUPPORTED, "dgrad: T too large");
    return cuda_status(bitnet::launch_dgrad(dY, W->gamma, W->group_bytes, T, n_out, k, dX,
                                            dx_dtype == BITNET_BF16, ws, reinterpret_cast<cudaStream_t>(stream)),
                       "dgrad");
}

bitnet_status bitnet_wait_selftest(void *ws, size_t ws_bytes, int32_t limit_us, bitnet_stream_t stream) {
    if (!ws) return fail(BITNET_ERR_WORKSPACE, "wait_selftest: workspace is required");
    if (ws_bytes < bitnet_decode_chain_workspace_size(1))
        return fail(BITNET_ERR_WORKSPACE, "wait_selftest: workspace needs %zu bytes", bitnet_decode_chain_workspace_size(1));
    if (!aligned(ws, 16)) return fail(BITNET_ERR_INVALID_ARG, "wait_selftest: ws must be 16-byte aligned");
    if (limit_us <= 0 || limit_us > 2000000) return fail(BITNET_ERR_INVALID_ARG, "wait_selftest: limit_us must be in [1, 2e6]");
    return cuda_status(bitnet::launch_wait_selftest(ws, static_cast<uint64_t>(limit_us) * 1000ull,
                                                    reinterpret_cast<cudaStream_t>(stream)),
                       "wait_selftest");
}

bitnet_status bitnet_tensor_peak(int32_t kind, int64_t iters, double *ops, void *ws, size_t ws_bytes,
                                 bitnet_stream_t stream) {
    if (kind < 0 || kind > 4) return fail(BITNET_ERR_INVALID_ARG, "tensor_peak: kind must be 0 .. 4");
    if (iters < 1 || iters > (int64_t(1) << 40)) return fail(BITNET_ERR_INVALID_ARG, "tensor_peak: iters must be in [1, 2^40]");
    if (!ops) return fail(BITNET_ERR_INVALID_ARG, "tensor_peak: ops is required");
    if (!ws) return fail(BITNET_ERR_WORKSPACE, "tensor_peak: workspace is required");
    if (ws_bytes < bitnet::kLinearWsBytes) return fail(BITNET_ERR_WORKSPACE, "tensor_peak: workspace needs %zu bytes", bitnet::kLinearWsBytes);
    if (!aligned(ws, 16)) return fail(BITNET_ERR_INVALID_ARG, "tensor_peak: ws must be 16-byte aligned");
    uint32_t *status = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + bitnet::kStatusOffset);
    return cuda_status(bitnet::launch_tensor_peak(kind, iters, status, ops, reinterpret_cast<cudaStream_t>(stream)),
                       "tensor_peak");
}

bitnet_status bitnet_read_device_status(void *ws, bitnet_stream_t stream) {
    if (!ws) return fail(BITNET_ERR_INVALID_ARG, "read_device_status: null workspace");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, static_cast<uint8_t *>(ws) + bitnet::kStatusOffset, sizeof word,
                                    cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_status(e, "read_device_status");
    if (word) {
        const uint32_t zero = 0;
        e = cudaMemcpyAsync(static_cast<uint8_t *>(ws) + bitnet::kStatusOffset, &zero, sizeof zero,
                            cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return cuda_status(e, "read_device_status");
        return fail(BITNET_ERR_TIMEOUT, "a device-side bounded wait gave up (status word 0x%x)", word);
    }
    return BITNET_OK;
}

}  // extern "C"
