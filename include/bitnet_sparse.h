/*
 * bitnet_sparse.h - C ABI of the sparse ternary BitLinear hot path (sm_100a).
 *
 * The library implements the forward of one Sparse-BitLinear layer and its
 * straight-through input gradient:
 *   pack   : W (fp32 masters) -> 2:4 mask, absmean ternary codes, packed layouts
 *   quant  : X -> per-token int8 codes and absmax scales
 *   linear : Y = dequant(Xq . Wq^T)   (int8 x ternary, int32 accumulation)
 *   dgrad  : dX = gamma * dY . Wq     (straight-through estimator)
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *     allocates no memory, never frees, and never synchronises a stream unless
 *     the entry point says so (bitnet_read_device_status).
 *   - Every call is asynchronous on `stream` and returns after enqueueing.
 *   - Arguments are validated on the host before any launch; a failed check
 *     returns an error status and enqueues nothing.
 *   - Matrices are row-major with the last index contiguous.
 *   - No C++ exception crosses this boundary.
 *   - A call with T == 0 (empty batch) validates its sizes, launches nothing,
 *     and accepts NULL activation / output buffers.
 *   - bitnet_last_error() returns a human-readable detail of the last failure
 *     on the calling thread.
 */
#ifndef BITNET_SPARSE_H
#define BITNET_SPARSE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream; NULL is the legacy default stream. */
typedef struct CUstream_st *bitnet_stream_t;

typedef enum {
    BITNET_OK = 0,
    BITNET_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bad alignment */
    BITNET_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. N:M other than 2:4 for packing) */
    BITNET_ERR_WORKSPACE = 3,     /* workspace missing or smaller than *_workspace_size() */
    BITNET_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    BITNET_ERR_TIMEOUT = 5        /* a device-side bounded wait gave up (see bitnet_read_device_status) */
} bitnet_status;

typedef enum { BITNET_F32 = 0, BITNET_BF16 = 1 } bitnet_dtype;

/*
 * Packed weights of one layer, W in R^{n_out x k}.  Filled by bitnet_pack_nm and
 * read by bitnet_sparse_linear / bitnet_dgrad.  Every pointer is a device
 * buffer of the size given below, allocated by the caller; a NULL layout
 * pointer means "not produced / not available".
 *
 *   n, m         N:M pattern; the packed layouts exist for n = 2, m = 4.
 *   gamma        1 float: the absmean scale (required).
 *   group_bytes  [n_out, k/4] bytes, canonical 2:4 group byte per 4 weights:
 *                bits 0-1 idx0, bits 2-3 idx1 (idx0 < idx1: the two kept
 *                positions), bits 4-5 code(idx0), bits 6-7 code(idx1); code
 *                00 = 0, 01 = +1, 11 = -1.  Needs k % 4 == 0.
 *   mma_vals     [n_out, k/2] int8: the two kept codes of every group, in k
 *                order (the compressed sparse operand of the tensor-core GEMM).
 *   mma_meta     bitnet_mma_meta_bytes(n_out, k) bytes: the 2:4 metadata in
 *                blocks of 128 rows x 128 k (16 bytes per row, one 4-bit
 *                nibble idx0 | idx1 << 2 per group, low nibble first), block
 *                (kb, rb) at byte offset (kb * ceil(n_out/128) + rb) * 2048.
 *                Rows >= n_out and k >= k of the padded blocks hold idx (0,1).
 *   dec_codes    bitnet_dec_bytes(n_out, k) bytes: decode (GEMV) layout.  For
 *                every 16-row x 64-k tile, 32 lanes x 8 bytes: a 32-bit word
 *                of 16 two-bit codes and a 32-bit word of 8 metadata nibbles,
 *                in the register order of the warp-level sparse MMA.  Needs
 *                n_out % 16 == 0 and k % 64 == 0.
 */
typedef struct {
    int64_t n_out;
    int64_t k;
    int32_t n;
    int32_t m;
    float *gamma;
    uint8_t *group_bytes;
    int8_t *mma_vals;
    uint8_t *mma_meta;
    uint8_t *dec_codes;
} bitnet_packed_w;

/* Buffer sizes of the layouts above (bytes). */
size_t bitnet_mma_meta_bytes(int64_t n_out, int64_t k);
size_t bitnet_dec_bytes(int64_t n_out, int64_t k);

/* ------------------------------------------------------------------------
 * bitnet_pack_nm - per-step mask + ternarise + pack.
 *
 * Follows "Sparse-BitNet" (gist.science technical summary), section 2
 * "Kerncomponenten": the N:M mask is chosen from the magnitudes of the master
 * weights (top-N of every M consecutive weights along k, ties to the lower
 * position); the forward quantises to ternary and then applies the mask;
 * "Training Strategie": the mask is recomputed every step.  The quantiser is
 * the absmean one of "BitNet b1.58: Ternary Weights for 1.58-bit LLMs",
 * section "The mechanism":
 *   gamma = fp32(fp64_rn(exact sum |W|) / (n_out*k)) + eps   (fp32 add)
 *   code  = clip(rint_half_even(fp32(W / gamma)), -1, 1) for kept weights, 0 else.
 * gamma is bit-exact and independent of summation order.
 *
 *   W         [n_out, k] fp32, 16-byte aligned, k % m == 0.
 *   out       layouts to fill: out->gamma required; each of group_bytes,
 *             mma_vals + mma_meta (together), dec_codes is written when
 *             non-NULL (these need n == 2, m == 4).
 *   eps       added to the mean (>= 0).
 *   mask_bits [n_out, k/8] bytes or NULL: bit (c % 8) of byte (r*k + c)/8 is 1
 *             when weight (r, c) is kept.  Supports any 1 <= n < m, m in {4, 8}.
 *   ws        device workspace of >= bitnet_pack_workspace_size() bytes,
 *             16-byte aligned; contents on entry are ignored.
 * Errors: INVALID_ARG (null W / gamma / ws, bad sizes or alignment),
 *         UNSUPPORTED (packed layouts requested with n:m != 2:4),
 *         WORKSPACE (ws_bytes too small), CUDA (launch failure).
 * ------------------------------------------------------------------------ */
size_t bitnet_pack_workspace_size(int64_t n_out, int64_t k);
bitnet_status bitnet_pack_nm(const float *W, bitnet_packed_w *out, float eps,
                             uint8_t *mask_bits, void *ws, size_t ws_bytes,
                             bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_pack_nm_update - the per-step pack of a matrix that was packed before.
 *
 * "Sparse-BitNet" (gist.science), section 2 "Training Strategie": the mask
 * and codes are recomputed every step from masters that move by one optimizer
 * step.  Results are bit-identical to bitnet_pack_nm (2:4 only).  On entry
 * out->gamma must hold the gamma of this matrix's previous pack (as written
 * by bitnet_pack_nm / _update), or 0 when there is none.  With that hint the
 * call reads W ONCE: it sums |W| exactly and writes every layout with the
 * hint's threshold, listing the kept weights within a relative 2^-10 of that
 * threshold; if the new threshold falls inside that band only the listed
 * groups are rewritten, otherwise (or without a hint, or when the list is
 * full) a second full pass runs.  The choice is made on the device.
 *
 *   W, out, eps, mask_bits  as in bitnet_pack_nm (n = 2, m = 4).
 *   ws   >= bitnet_pack_update_workspace_size(n_out, k) bytes: the pack
 *        scratch plus the list of near-threshold groups.
 * Errors: as bitnet_pack_nm.
 * ------------------------------------------------------------------------ */
size_t bitnet_pack_update_workspace_size(int64_t n_out, int64_t k);
bitnet_status bitnet_pack_nm_update(const float *W, bitnet_packed_w *out, float eps,
                                    uint8_t *mask_bits, void *ws, size_t ws_bytes,
                                    bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_pack_nm_update_batch - bitnet_pack_nm_update of many matrices at once.
 *
 * "Sparse-BitNet" (gist.science), section 2 "Training Strategie": every step
 * re-derives the mask and codes of every layer from its masters.  Each item
 * gets exactly what bitnet_pack_nm_update(items[i].W, items[i].out, eps,
 * items[i].mask_bits, ...) gives it, bit for bit, including the use of
 * out->gamma as the previous gamma.  The whole list runs in two kernel
 * launches per 64 matrices (plus one per matrix that asks for dec_codes)
 * instead of three or four per matrix, so the fixed cost of a launch, a
 * workspace clear and a gamma finalisation is paid once per list.
 *
 *   items    host array of n_items descriptors (read during the call only):
 *              W          [n_out x k] masters of w_dtype, 16-byte aligned
 *                         (device).  BITNET_BF16 masters ("Sparse-BitNet"
 *                         (gist.science), section 2 "Kerncomponenten": the
 *                         master weights are kept in BF16) are widened exactly
 *                         to fp32, so the result is that of their fp32 values;
 *              w_dtype    BITNET_F32 or BITNET_BF16;
 *              out        host struct as for bitnet_pack_nm_update (n = 2,
 *                         m = 4, k % 16 == 0); out->gamma holds the hint;
 *              mask_bits  [n_out * k / 8] or NULL.
 *            The items' output buffers must not overlap one another.
 *   n_items  >= 0.
 *   eps      >= 0.
 *   ws       >= bitnet_pack_update_batch_workspace_size(items, n_items) bytes,
 *            16-byte aligned: one scratch header per item, then the band lists.
 * Errors: as bitnet_pack_nm_update; UNSUPPORTED when k % 16 != 0.
 * ------------------------------------------------------------------------ */
typedef struct {
    const void *W;
    bitnet_packed_w *out;
    uint8_t *mask_bits;
    int32_t w_dtype;       /* bitnet_dtype of W */
    int32_t gamma_known;   /* nonzero: out->gamma already is the exact gamma of W
                              (as bitnet_adamw_step writes it); the pack then
                              reads W once, forms no sum and keeps out->gamma */
} bitnet_pack_item;

size_t bitnet_pack_update_batch_workspace_size(const bitnet_pack_item *items, int32_t n_items);
bitnet_status bitnet_pack_nm_update_batch(const bitnet_pack_item *items, int32_t n_items, float eps,
                                          void *ws, size_t ws_bytes, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_pack_6of8_windows - 6:8 masked ternary weights as 2:4 windows.
 *
 * "Sparse-BitNet" (gist.science), section 4 "Resultaten": the method trains
 * at 6:8 (top-6 |W| of every 8 consecutive weights of a row).  "Is 2:4
 * Sparsity Still Worth It? ..." (thelatestinai.com), its SlideSparse entry:
 * a 6:8 block is rewritten without loss as three overlapping 4-wide windows
 * (at positions 0, 2 and 4 of the block), each 2:4-compliant, so the 2:4
 * tensor cores can run it.  Kept positions go, in increasing order, to the
 * leftmost window that covers them and has a free slot (this always places
 * all six).  gamma is the absmean of the dense W as for 2:4; ties in the mask
 * go to the lower position.
 *
 *   W          [n_out x k] fp32 masters, 16-byte aligned, k % 64 == 0.
 *   k          columns of W (the 6:8 width).
 *   out        window-layout packed weights: out->n_out rows, out->k == k/2*3,
 *              n = 2, m = 4.  group_bytes required; mma_vals + mma_meta and
 *              dec_codes (n_out % 16 == 0 and k % 128 == 0) optional; they are
 *              exactly the layouts bitnet_pack_nm writes for a 2:4 matrix of
 *              width k/2*3.
 *   mask_bits  [n_out * k / 8] or NULL: the 6:8 keep bits over the original k.
 *   ws         >= bitnet_pack_workspace_size(n_out, k) bytes.
 * bitnet_sparse_linear(Xl, absmax, out, ...) with Xl from
 * bitnet_quant_act_lift_6of8 then computes the 6:8 product exactly.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 * ------------------------------------------------------------------------ */
bitnet_status bitnet_pack_6of8_windows(const float *W, int64_t k, float eps, bitnet_packed_w *out,
                                       uint8_t *mask_bits, void *ws, size_t ws_bytes, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_quant_act_lift_6of8 - per-token int8 quantisation with the
 * activation layout of bitnet_pack_6of8_windows.
 *
 * Same scale and codes as bitnet_quant_act ("BitNet b1.58 ...", section "The
 * mechanism"); every block of 8 codes q[8b .. 8b+7] is written as the 12
 * codes of its three windows: q[8b .. 8b+3], q[8b+2 .. 8b+5], q[8b+4 .. 8b+7].
 *
 *   X       [T, K] fp32 or bf16, 16-byte aligned, K % 8 == 0.
 *   Xl      [T, K/2*3] int8 out, 16-byte aligned.   absmax [T] fp32 out.
 * Errors: INVALID_ARG, CUDA.
 * ------------------------------------------------------------------------ */
bitnet_status bitnet_quant_act_lift_6of8(const void *X, bitnet_dtype x_dtype, int64_t T, int64_t K, float eps,
                                         int8_t *Xl, float *absmax, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_quant_act - per-token absmax int8 activation quantisation.
 *
 * "BitNet b1.58: Ternary Weights for 1.58-bit LLMs", section "The mechanism"
 * (Activations): each token is scaled to [-Q_b, Q_b], symmetric, with no
 * zero-point; Q_b = 127:
 *   a[t] = max(max_k |X[t,k]|, eps);  s = 127 / a[t] (fp32);
 *   Xq[t,k] = clamp(rint_half_even(fp32(X[t,k] * s)), -127, 127).
 *
 *   X       [T, K] fp32 or bf16 (x_dtype), 16-byte aligned, K % 8 == 0.
 *   Xq      [T, K] int8 out, 16-byte aligned.   absmax  [T] fp32 out (= a[t]).
 * Errors: INVALID_ARG, CUDA.
 * ------------------------------------------------------------------------ */
bitnet_status bitnet_quant_act(const void *X, bitnet_dtype x_dtype, int64_t T, int64_t K,
                               float eps, int8_t *Xq, float *absmax, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_wgrad - weight gradient dW = dY^T . X (dense, every master).
 *
 * "Sparse-BitNet" (gist.science), section 2 "Training Strategie": the
 * gradient passes straight through the quantiser and the 2:4 mask to all
 * master weights, masked ones included; with both quantisers taken as the
 * identity in the backward pass, dW[n, k] = sum_t dY[t, n] X[t, k], where X
 * is the layer input (bf16) and dY the output gradient (bf16).
 *   dY         [T, n_out] bf16, 16-byte aligned.   X  [T, k] bf16, 16-byte aligned.
 *   n_out, k   positive multiples of 8; T >= 0.
 *   dW         [n_out, k] fp32 out, 16-byte aligned; accumulate != 0 adds
 *              the product to dW (gradient accumulation), else overwrites it
 *              (T = 0: zeros).
 *   ws         >= bitnet_wgrad_workspace_size() bytes (device status word).
 * Products of bf16 values are exact in fp32; the sum is an fp32 tensor-core
 * accumulation (order unspecified).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 * ------------------------------------------------------------------------ */
size_t bitnet_wgrad_workspace_size(void);
bitnet_status bitnet_wgrad(const void *dY, const void *X, int64_t T, int64_t n_out, int64_t k, float *dW,
                           int32_t accumulate, void *ws, size_t ws_bytes, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_adamw_step - AdamW update of fp32 masters that also emits the exact
 * absmean gamma of the updated matrix for the next pack.
 *
 * The pages keep latent fp32 masters and re-pack them every step ("BitNet
 * b1.58 ...", section "What this paper explains"; "Sparse-BitNet"
 * (gist.science), section 2 "Training Strategie"); they name no optimiser.
 * Per element, each step one IEEE fp32 operation in this order:
 *   m = b1 m + (1 - b1) g;   v = b2 v + (1 - b2) (g g);
 *   u = (m / c1) / (sqrt(v / c2) + eps);   w = w - lr (u + wd w)
 * with c1 = bias_correction1 = 1 - b1^t and c2 = 1 - b2^t supplied by the
 * caller.  Then gamma_out = fp32(fp32(exact sum |w| / n) + eps_gamma), as
 * bitnet_pack_nm forms it, so a pack item with gamma_known reads W once.
 *   W, m, v    [n] fp32 in/out;  dW [n] fp32;  all 16-byte aligned; n % 4 == 0.
 *   gamma_out  device fp32 scalar (normally the packed matrix's out->gamma).
 *   ws         >= bitnet_adamw_workspace_size() bytes, 16-byte aligned.
 * Errors: INVALID_ARG, WORKSPACE, CUDA.
 * ------------------------------------------------------------------------ */
typedef struct {
    float lr, beta1, beta2, eps, weight_decay;
    float bias_correction1, bias_correction2;   /* 1 - beta1^t, 1 - beta2^t */
} bitnet_adamw_hparams;

size_t bitnet_adamw_workspace_size(void);
bitnet_status bitnet_adamw_step(float *W, const float *dW, float *m, float *v, int64_t n,
                                const bitnet_adamw_hparams *h, float eps_gamma, float *gamma_out, void *ws,
                                size_t ws_bytes, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_adamw_step_batch - bitnet_adamw_step over a list of matrices in one
 * launch (per 64 matrices): the same update and the same gamma_out, bit for
 * bit, as one call per matrix.
 *   items   host array of n_items descriptors (read during the call only):
 *             W, dW, m, v  [n] fp32 device arrays, 16-byte aligned, n % 4 == 0;
 *             gamma_out    device fp32 scalar of that matrix.
 *           The items' arrays must not overlap one another.
 *   h, eps_gamma   as bitnet_adamw_step (one set for the whole list).
 *   ws      >= bitnet_adamw_batch_workspace_size(n_items) bytes, 16-byte aligned.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 * ------------------------------------------------------------------------ */
typedef struct {
    float *W;
    const float *dW;
    float *m;
    float *v;
    int64_t n;
    float *gamma_out;
} bitnet_adamw_item;

size_t bitnet_adamw_batch_workspace_size(int32_t n_items);
bitnet_status bitnet_adamw_step_batch(const bitnet_adamw_item *items, int32_t n_items, const bitnet_adamw_hparams *h,
                                      float eps_gamma, void *ws, size_t ws_bytes, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_rmsnorm_quant - RMSNorm fused into the per-token quantisation.
 *
 * "BitNet b1.58 ...", section "What this paper explains": the blocks around
 * BitLinear are LLaMA-alike (RMSNorm, SwiGLU); section "The mechanism": the
 * BitLinear input is quantised per token to [-127, 127].  Per token t:
 *   S    = sum_k X[t,k]^2, exact, rounded once to fp64;
 *   ms   = fp32(S / K);   r = fp32(1 / fp32(sqrt(fp32(ms + eps_norm))));
 *   x_k  = fp32(X[t,k] * r), then fp32(x_k * w[k]) when w is given;
 *   a[t] = max(max_k |x_k|, eps_act);  s = fp32(127 / a[t]);
 *   Xq[t,k] = clamp(rint_half_even(fp32(x_k * s)), -127, 127).
 * Every step is one IEEE fp32/fp64 operation in this order: the codes are the
 * same bit for bit on any conforming implementation.
 *
 *   X        [T, K] bf16, 16-byte aligned, K % 8 == 0, K <= 65536.
 *   w        [K] fp32 norm weight or NULL (no weight).
 *   eps_norm > 0 (added to the mean square);  eps_act > 0 (absmax floor).
 *   Xq       [T, K] int8 out, 16-byte aligned.  absmax [T] fp32 out (= a[t]).
 *   rinv     [T] fp32 out (= r) or NULL.
 * Errors: INVALID_ARG, UNSUPPORTED (T >= 2^31), CUDA.
 * ------------------------------------------------------------------------ */
bitnet_status bitnet_rmsnorm_quant(const void *X, const float *w, int64_t T, int64_t K, float eps_norm,
                                   float eps_act, int8_t *Xq, float *absmax, float *rinv, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_swiglu_quant - SwiGLU gate fused into the per-token quantisation.
 *
 * Same pages and sections as bitnet_rmsnorm_quant.  Per token t and column f:
 *   silu(g) = fp32(g / fp32(1 + exp32(-g)));   h = fp32(silu(g) * u);
 * exp32(x): x clamped to [-87, 88]; n = rint(fp32(x * log2 e));
 * r = fp32(fp32(x - fp32(n * C1)) - fp32(n * C2)) with ln 2 = C1 + C2
 * (C1 = 0x3f317200, C2 = 0x35bfbe8e as fp32 bit patterns, log2 e =
 * 0x3fb8aa3b); p = Horner form of the degree-6 Taylor polynomial of e^r with
 * coefficients 1/720, 1/120, 1/24, 1/6 (0x3ab60b61, 0x3c088889, 0x3d2aaaab,
 * 0x3e2aaaab), 1/2, 1, 1, one rounded multiply and one rounded add a step;
 * exp32 = fp32(p * 2^n).  Then the codes of h exactly as bitnet_quant_act.
 *
 *   G, U     bf16, row t at G + t*ld and U + t*ld, F columns each (the gate
 *            and up halves of one [T, 2F] buffer: U = G + F, ld = 2F).
 *   F        % 8 == 0, F <= 51200;  ld >= F.   eps_act > 0.
 *   Xq       [T, F] int8 out, 16-byte aligned.  absmax [T] fp32 out.
 * Errors: INVALID_ARG, UNSUPPORTED (T >= 2^31), CUDA.
 * ------------------------------------------------------------------------ */
bitnet_status bitnet_swiglu_quant(const void *G, const void *U, int64_t ld, int64_t T, int64_t F, float eps_act,
                                  int8_t *Xq, float *absmax, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_sparse_linear - Y = dequant(Xq . Wq^T).
 *
 * "BitNet b1.58 ...", section "The mechanism": with ternary weights each
 * output is a signed sum of activations; "Sparse-BitNet" section 2: the masked
 * ternary weights are used in the forward pass.
 *   acc[t,n] = sum_k Xq[t,k] * Wq[n,k]      (int32, exact)
 *   Y[t,n]   = fp32(acc) * ((gamma * absmax[t]) / 127)   -> fp32 or bf16
 *
 *   Xq      [T, K] int8 (from bitnet_quant_act), 16-byte aligned.
 *   absmax  [T] fp32.
 *   W       packed weights with K == W->k.  T <= 8 runs the decode GEMV and
 *           needs W->dec_codes (or W->group_bytes); T > 8 runs the tensor-core
 *           GEMM and needs W->mma_vals + W->mma_meta, with k % 32 == 0.
 *   Y       [T, n_out] of y_dtype.
 *   acc_out [T, n_out] int32 or NULL: raw accumulators (for checking).
 *   ws      >= bitnet_linear_workspace_size() bytes of device memory, holding
 *           the device status word of the bounded waits.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 * ------------------------------------------------------------------------ */
size_t bitnet_linear_workspace_size(void);
bitnet_status bitnet_sparse_linear(const int8_t *Xq, const float *absmax,
                                   const bitnet_packed_w *W, int64_t T,
                                   void *Y, bitnet_dtype y_dtype, int32_t *acc_out,
                                   void *ws, size_t ws_bytes, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_quant_linear - per-token quantisation fused with the sparse linear.
 *
 * Same result as bitnet_quant_act followed by bitnet_sparse_linear (bit for
 * bit): "BitNet b1.58 ...", section "The mechanism" (per-token symmetric
 * 8-bit activations; ternary product as signed sums).  For T <= 8 with the
 * decode layout it is the decode chain below with one projection (one
 * kernel, quantisation fused); otherwise, and for shapes the chain does not
 * take, it runs the quantisation into the workspace and the GEMV or GEMM.
 *
 *   X        [T, K] fp32 or bf16 (x_dtype), 16-byte aligned, K == W->k.
 *   eps      activation eps (> 0).
 *   W        packed weights (dec_codes for T <= 8; mma layouts for T > 8).
 *   Y        [T, n_out] of y_dtype.   acc_out  [T, n_out] int32 or NULL.
 *   xq_out   [T, K] int8 or NULL; absmax_out [T] fp32 or NULL: copies of the
 *            activation codes and scales (for checking).
 *   ws       >= bitnet_quant_linear_workspace_size(T, K) bytes.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 * ------------------------------------------------------------------------ */
size_t bitnet_quant_linear_workspace_size(int64_t T, int64_t K);
bitnet_status bitnet_quant_linear(const void *X, bitnet_dtype x_dtype, float eps,
                                  const bitnet_packed_w *W, int64_t T, void *Y, bitnet_dtype y_dtype,
                                  int32_t *acc_out, int8_t *xq_out, float *absmax_out,
                                  void *ws, size_t ws_bytes, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_decode_chain - a sequence of decode projections in one launch.
 *
 * Each op computes exactly bitnet_quant_linear(op.X, ...) for its own packed
 * weights ("BitNet b1.58 ...", section "The mechanism"; "Sparse-BitNet"
 * (gist.science), section 2 "Kerncomponenten"), for the T <= 8 tokens of a
 * decode step.  The ops run in order inside one persistent kernel (one CTA
 * per SM): ops[i] with wait_prev = 1 reads its X only after every CTA has
 * finished ops[0..i-1], so ops[i].X may be the Y of an earlier op (a chain of
 * layers); wait_prev = 0 lets an op whose X is ready start before the
 * previous op has finished (for example Q, K and V read the same X).  Packed
 * weights are streamed into shared memory ahead of use and must not be
 * written while the call runs.
 *
 *   ops      host array of n_ops descriptors (read during the call only):
 *              X        [T, W->k] of x_dtype, 16-byte aligned (device);
 *              W        host struct; needs dec_codes (16-byte aligned),
 *                       n = 2, m = 4, n_out % 16 == 0, k % 64 == 0 and
 *                       n_out / 16 <= 32 x (number of SMs);
 *              Y        [T, W->n_out] of y_dtype (device);
 *              acc_out  [T, n_out] int32 or NULL (raw accumulators);
 *              xq_out   [T, k] int8 or NULL; absmax_out [T] fp32 or NULL;
 *              wait_prev  0 or 1 (ignored for ops[0]).
 *            Y of one op must not overlap X, Y or the weights of another op
 *            that may run at the same time.
 *   n_ops    >= 0; more than 128 ops are split into launches of 128.
 *   T        1..8 tokens (0: nothing to do).
 *   eps      activation eps (> 0).
 *   ws       >= bitnet_decode_chain_workspace_size(n_ops) bytes: status word,
 *            abort word and one completion counter per op (cleared by the call).
 * Kernels: a chain with no wait_prev runs on the pipelined kernel (warp roles
 * joined by barriers and shared-memory counters); a chain with any wait_prev
 * on the latency-oriented one.  Shared memory holds the activation rows (one
 * staging row per quantiser warp, the int8 rows of several projections) and
 * the weight ring: the call returns UNSUPPORTED when they do not fit beside
 * weight stages of at least 2 KB per MMA warp (pipelined) or two 16 KB stages
 * (with waits).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA; a wait that runs out
 * inside the kernel sets the TIMEOUT bit of the device status word.
 * ------------------------------------------------------------------------ */
typedef struct {
    const void *X;
    const bitnet_packed_w *W;
    void *Y;
    int32_t *acc_out;
    int8_t *xq_out;
    float *absmax_out;
    int32_t wait_prev;
} bitnet_chain_op;

size_t bitnet_decode_chain_workspace_size(int32_t n_ops);
bitnet_status bitnet_decode_chain(const bitnet_chain_op *ops, int32_t n_ops, int64_t T,
                                  bitnet_dtype x_dtype, bitnet_dtype y_dtype, float eps,
                                  void *ws, size_t ws_bytes, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_dgrad - straight-through input gradient dX = gamma * dY . Wq.
 *
 * "Sparse-BitNet" (gist.science technical summary), section 2 "Training
 * Strategie": both the quantiser and the top-N selection pass the gradient
 * straight through (dual STE), so the input gradient flows through the
 * masked ternary weights.  Dense in the contraction over n_out (the 2:4
 * structure lies along k), bf16 operands, fp32 accumulation.
 *
 *   dY      [T, n_out] bf16 (dy_dtype must be BITNET_BF16), 16-byte aligned,
 *           n_out % 8 == 0.
 *   W       packed weights with group_bytes.
 *   dX      [T, k] fp32 or bf16 (dx_dtype).
 *   ws      >= bitnet_dgrad_workspace_size(W) bytes (holds the expanded bf16
 *           transpose of gamma-free Wq and the status word).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 * ------------------------------------------------------------------------ */
size_t bitnet_dgrad_workspace_size(int64_t n_out, int64_t k);
bitnet_status bitnet_dgrad(const void *dY, bitnet_dtype dy_dtype, const bitnet_packed_w *W,
                           int64_t T, void *dX, bitnet_dtype dx_dtype,
                           void *ws, size_t ws_bytes, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_pack_nm_noalloc - bitnet_pack_nm for callers that cannot allocate.
 *
 * No counterpart in the paper: this is a library convenience.  Some callers
 * cannot allocate device memory where they pack (an optimizer step inside a
 * fixed memory pool, an embedded runtime whose allocator the call site cannot
 * reach, a latency-critical path that must not call cudaMalloc).  This entry
 * point needs no workspace: the pack's scratch lives in a fixed device array of
 * bitnet_pack_workspace_size() bytes (2304) inside the library, present on every
 * GPU that loads the library until the process exits.  Everything else is as
 * in bitnet_pack_nm, with bit-identical results.
 *
 *   Limit: n_out * k <= 2^34 weights (2^32 groups of 4, the bound of the
 *          pack's group indexing); larger matrices are rejected with
 *          BITNET_ERR_UNSUPPORTED before any pointer is touched.
 *   First call on a device looks up the array's device address with
 *          cudaGetSymbolAddress (once per device, with that device current);
 *          make that first call before any stream capture.  The address is
 *          kept with the identity of the device's context: after a
 *          cudaDeviceReset the next call looks it up again (make that call
 *          outside stream capture too).
 *   Sharing: every call reuses the same array and clears it first; calls whose
 *          kernels overlap on the GPU (other streams, other host threads on the
 *          same device) race on it - serialise them on one stream.
 *   Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * Errors: as bitnet_pack_nm (no WORKSPACE error), plus UNSUPPORTED above the limit.
 * ------------------------------------------------------------------------ */
bitnet_status bitnet_pack_nm_noalloc(const float *W, bitnet_packed_w *out, float eps,
                                     uint8_t *mask_bits, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_wait_selftest - exercises the error path of the bounded waits.
 *
 * Every wait of the kernels (mbarrier phases of the GEMM and pack pipelines,
 * the decode chain's grid counters) gives up after a time limit, sets the
 * timeout bit of the workspace status word and lets the kernel end, so the
 * CUDA context stays usable.  This call runs one wait of each kind on an
 * event that never happens, with the limit limit_us (1 .. 2e6 microseconds),
 * on the given stream; afterwards bitnet_read_device_status(ws) returns
 * BITNET_ERR_TIMEOUT.  It faults nothing and hangs nothing: it is the health
 * check of the timeout path.
 *   ws   >= bitnet_decode_chain_workspace_size(1) bytes, 16-byte aligned
 *        (cleared by the call).
 * Errors: INVALID_ARG, WORKSPACE, CUDA.
 * ------------------------------------------------------------------------ */
bitnet_status bitnet_wait_selftest(void *ws, size_t ws_bytes, int32_t limit_us, bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * bitnet_tensor_peak - throughput ceiling of a tensor-core instruction form.
 *
 * No counterpart in the paper: it measures the denominator of the GEMMs'
 * roofline on the GPU that runs them.  "Is 2:4 Sparsity Still Worth It?"
 * (SlideSparse entry) bounds the gain of 2:4 by twice the dense rate, which a
 * given device need not deliver for a given instruction; this call measures
 * what it delivers.  One CTA pair per two SMs issues MMAs back to back on
 * operands resident in shared memory (no loads, no epilogue):
 *   kind 0  tcgen05.mma.sp.cta_group::2.kind::i8, M 256, N 224, K 64 (the
 *           2:4-sparse int8 instruction of the prefill GEMM);
 *   kind 1  tcgen05.mma.cta_group::2.kind::i8, M 256, N 256, K 32 (dense int8);
 *   kind 2  tcgen05.mma.cta_group::2.kind::f16 (bf16), M 256, N 256, K 16;
 *   kind 3  kind 0 with each stage's 2:4 metadata copied into TMEM
 *           (tcgen05.cp) right before the stage's two MMAs, two slots;
 *   kind 4  kind 3 with every copy issued four stages ahead, eight slots.
 *   iters   MMAs per CTA pair (rounded up to a whole stage), >= 1.
 *   ops     host pointer; receives the dense-equivalent operations of the
 *           launch, 2 M N K per MMA summed over the pairs (time the launch on
 *           the stream with events; ops / seconds is the ceiling).
 *   ws      >= bitnet_linear_workspace_size() bytes, 16-byte aligned: status
 *           word of the bounded wait for the tensor pipe to drain.
 * Errors: INVALID_ARG, WORKSPACE, CUDA.
 * ------------------------------------------------------------------------ */
bitnet_status bitnet_tensor_peak(int32_t kind, int64_t iters, double *ops, void *ws, size_t ws_bytes,
                                 bitnet_stream_t stream);

/* ------------------------------------------------------------------------
 * Status helpers.
 * bitnet_read_device_status synchronises `stream`, reads the status word that
 * the kernels of the last call on `ws` left (BITNET_OK or BITNET_ERR_TIMEOUT
 * when a bounded wait gave up) and clears it.
 * ------------------------------------------------------------------------ */
bitnet_status bitnet_read_device_status(void *ws, bitnet_stream_t stream);
const char *bitnet_status_string(bitnet_status s);
const char *bitnet_last_error(void);
int bitnet_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* BITNET_SPARSE_H */
