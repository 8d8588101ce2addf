/*
 * awq.h -- C ABI of the B200 (sm_100a) AWQ per-layer scale search.
 *
 * The operation: for one linear layer with fp16 weights W[N,K] and calibration
 * activations X[T,K], take the per-input-channel activation magnitudes
 * a_j = mean_t |X[t,j]|; for every alpha of a grid form s_j = a_j^alpha, quantize
 * W*diag(s) group-wise along K with round-to-nearest, dequantize and divide by
 * s, score the output error ||(W_hat - W) X^T||^2, keep the best alpha, and
 * emit packed low-bit codes with fp16 scales and zero points.
 *
 * Sources (web pages; cited by title and section):
 *   [QAS-QA]   "Как работает quantization-aware scaling в AWQ для защиты важных
 *              весов?" -- §5 mechanism, §6 objective (MSE), §9 quant_config
 *              {zero_point, q_group_size, w_bit}
 *   [AWQ-note] "AWQ: Activation-Aware Weight Quantization For On-Device LLM
 *              Compression AND Acceleration" -- section "Measures"
 *   [GPTQ-AWQ] "GPTQ与AWQ" -- section "量化方法" (W is (out_features,
 *              in_features), X is (batch, in_features))
 *   [AWQ-wiki] "AWQ" (French encyclopedia page) -- "Fondements techniques"
 *
 * Conventions shared by every entry point
 *   - Pointers are DEVICE pointers owned by the caller unless stated; the
 *     library never allocates, frees or retains them.  fp16 data is IEEE
 *     binary16 passed as `const void*`.  Every pointer must be 16-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *     are stream-ordered and asynchronous; the returned status covers argument
 *     validation and launch errors only.  Errors raised while kernels run
 *     (a bounded wait that ran out) are reported by awq_get_status().
 *   - Matrices are row-major.  W rows are contiguous (row stride K); X rows
 *     have stride ldx >= K elements, ldx a multiple of 8.
 *   - Sizes: 1 <= N, T <= 2^31 - 1; K a multiple of group_size.
 *   - Invalid arguments return AWQ_ERR_INVALID_ARG before anything is launched.
 *   - Calls are thread-safe.  What persists between calls: the device error
 *     word (read and cleared by awq_get_status()); the wait limit, one value
 *     for the process (awq_set_wait_timeout_ms); the event pair armed by
 *     awq_profile_next_search, per host thread and used by that thread's next
 *     search only; the per-device setup done once (shared-memory limits of the
 *     kernels, the device properties, the scratch address of
 *     awq_search_layer_noalloc).  No result of one call feeds another.
 */
#ifndef AWQ_B200_AWQ_H
#define AWQ_B200_AWQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define AWQ_API __attribute__((visibility("default")))
#else
#define AWQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    AWQ_OK = 0,
    AWQ_ERR_INVALID_ARG = 1,   /* bad pointer, size, alignment or config        */
    AWQ_ERR_UNSUPPORTED = 2,   /* no sm_100 device, or a config not implemented  */
    AWQ_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed           */
    AWQ_ERR_TIMEOUT = 4,       /* a kernel's bounded wait ran out (device flag)  */
    AWQ_ERR_WORKSPACE = 5      /* workspace missing or smaller than required     */
} awq_status;

/* Quantizer configuration ([QAS-QA] §9 quant_config):
 *   bits        w_bit, one of 2, 3, 4  (codes 0 .. 2^bits - 1)
 *   group_size  q_group_size along K, one of 64, 128
 *   zero_point  1: asymmetric groups with a zero point
 *                  (scale = (max w' - min w') / qmax, z = round(-min w' / scale), the
 *                  codes clamped to [0, qmax] but not z: a group that does not span
 *                  zero has z outside [0, qmax])
 *               0: symmetric absmax groups ([AWQ-note] "Measures": the INT3
 *                  grid of step max|w| / (2^(b-1) - 1)): scale = max|w'| / (2^(bits-1) - 1)
 *                  and the zero fixed at the middle code 2^(bits-1), stored in
 *                  `zeros` like any zero point, so every consumer of the packed
 *                  format treats both alike.                                    */
typedef struct {
    int32_t bits;
    int32_t group_size;
    int32_t zero_point;
} awq_qcfg;

/* Step a1 -- activation statistics ([AWQ-note] "Measures": average absolute
 * activation per input channel; [GPTQ-AWQ] "量化方法": X.abs().mean(dim=0)).
 *   X   fp16 [T, ldx] (only the first K columns are read)
 *   a   float [K] output: a_j = RN32(RN64(sum_t |X[t,j]|) / T).  The column
 *       sum is accumulated exactly (binary64 holds every partial sum while
 *       T * max|x| < 2^29), so the result is independent of summation order.
 * Requires K % 8 == 0. */
AWQ_API awq_status awq_act_stats(const void *X, int64_t T, int64_t K, int64_t ldx,
                         float *a, void *stream);

/* Step a2 -- the search space s = a^alpha ([AWQ-note] "Measures": for each
 * candidate alpha compute a^alpha).
 *   a       float [K]
 *   alphas  float [n_alpha], every value in [0, 1]  (device pointer)
 *   s       float [n_alpha, K] output: s[i,j] = RN32(pow(max(a_j, FLT_MIN), alpha_i))
 *           evaluated in binary64 (alpha = 0 gives exactly 1).
 * 1 <= n_alpha <= 64.  An alpha outside [0, 1] raises AWQ_ERR_INVALID_ARG
 * through awq_get_status(). */
AWQ_API awq_status awq_alpha_scales(const float *a, int64_t K, const float *alphas, int32_t n_alpha,
                            float *s, void *stream);

/* Steps a3/a4 standalone -- scale, group-wise round-to-nearest,
 * dequantize, unscale ([QAS-QA] §5; [AWQ-wiki] "Fondements techniques": the
 * inverse scaling is applied after dequantization).  For one scale vector s:
 *   per row n and group G of group_size columns:
 *     w'    = RN32(w * s)
 *     scale = RN32(RN32(max w' - min w') / qmax),  sh = RN16(clamp(scale, 2^-24, 65504))
 *     r     = RN32(1 / sh),  z = RN16(sat(rint(-min w' * r)))
 *             (z saturated to +-65504 and rounded to fp16, the format `zeros`
 *             stores; that stored z is the one used below, and -0 is stored as +0)
 *     q     = clamp(rint(w' * r) + z, 0, qmax)
 *     w_hat = RN16(RN32(RN32((q - z) * sh) * RN32(1 / s)))
 *   (the products inside rint are exact: rint is their only rounding)
 *   (zero_point = 0: scale = RN32(max(-min w', max w') / (2^(bits-1) - 1)), z = 2^(bits-1))
 *   W      fp16 [N, K];  s  float [K];  W_hat  fp16 [N, K] output.
 * This is the exact per-element function the search evaluates for every
 * alpha; it never runs inside the search (the search keeps W_hat on chip). */
AWQ_API awq_status awq_quant_dequant(const void *W, int64_t N, int64_t K, const float *s,
                             awq_qcfg q, void *W_hat, void *stream);

/* The same with channels held in fp16 ([AWQ-note] "Measures": keeping 1% of
 * the input channels in FP16 is the experiment that motivates the method).
 *   mask  uint8 [K] (device) or NULL: mask[k] != 0 keeps channel k in fp16 --
 *         it takes no part in its group's min and max, and W_hat[:, k] = W[:, k].
 *         A group whose channels are all kept has min = max = 0.
 * Mixed fp16/low-bit storage is not a packed format of this library: the
 * mask serves the baselines' loss (awq_search_scales) and this W_hat. */
AWQ_API awq_status awq_quant_dequant_masked(const void *W, int64_t N, int64_t K, const float *s,
                                            awq_qcfg q, const uint8_t *mask, void *W_hat, void *stream);

/* Bytes of device workspace awq_search_layer needs for these sizes. */
AWQ_API size_t awq_search_workspace_bytes(int64_t N, int64_t K, int64_t T, awq_qcfg q,
                                  int32_t n_alpha);

/* Steps a2-a6 -- the grid search ([AWQ-note] "Measures": collect X, take
 * a = mean|x|, compute a^alpha for each candidate alpha and measure the error;
 * Δy = (W_hat - W) x; [QAS-QA] §6: minimise the MSE between the outputs of the
 * original and the quantized layer on calibration data).
 *   W           fp16 [N, K]
 *   X           fp16 [T, ldx]
 *   a           float [K]  (awq_act_stats output, or any positive statistics)
 *   alphas      float [n_alpha] in [0, 1]
 *   losses      float [n_alpha] output: MSE_i = ||(W_hat_i - W) X^T||_F^2 / (N T)
 *   row_losses  float [n_alpha, N] output or NULL: per-row sums
 *               sum_t ((W_hat_i - W) X^T)[n, t]^2 (unnormalised)
 *   ws          device workspace of ws_bytes >= awq_search_workspace_bytes(...)
 * Requires K % 64 == 0 and 1 <= n_alpha <= 64.  The error matrix is never
 * written to memory: a tensor-core kernel forms (W_hat - W) X^T tile by tile in
 * tensor memory and reduces its squares on chip. */
AWQ_API awq_status awq_search_layer(const void *W, int64_t N, int64_t K,
                            const void *X, int64_t T, int64_t ldx,
                            const float *a, awq_qcfg q,
                            const float *alphas, int32_t n_alpha,
                            float *losses, float *row_losses,
                            void *ws, size_t ws_bytes, void *stream);

/* Steps a2-a6 for one part of a layer whose rows are split among several
 * callers -- typically one process per GPU, each holding rows [r0, r0 + N) of
 * the layer's W ([AWQ-note] "Measures": the error is a sum over the layer's
 * output rows, so the parts' errors add up).  Identical to awq_search_layer
 * except that the losses are normalised by the layer's row count:
 *   losses[i] = sum over these N rows of ||((W_hat_i - W) X^T)[n, :]||^2 / (rows_total T)
 * so that summing `losses` over the parts (e.g. one all-reduce of n_alpha
 * floats) gives the layer's MSE, after which every part takes the same argmin
 * (awq_pack on the summed losses) and packs its own rows.
 *   rows_total  the layer's row count, N <= rows_total < 2^31
 * Other arguments, the workspace and the errors are those of awq_search_layer
 * (sized by awq_search_workspace_bytes for this part's N). */
AWQ_API awq_status awq_search_layer_part(const void *W, int64_t N, int64_t rows_total, int64_t K,
                                         const void *X, int64_t T, int64_t ldx, const float *a, awq_qcfg q,
                                         const float *alphas, int32_t n_alpha, float *losses,
                                         float *row_losses, void *ws, size_t ws_bytes, void *stream);

/* Size of the scratch array built into the library for
 * awq_search_layer_noalloc: 32 MiB of device memory. */
#define AWQ_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/* awq_search_layer without a caller-provided workspace.  (The pages have no
 * counterpart: this is a property of the library's interface, not of AWQ.)
 *
 * For callers that cannot allocate device memory when they call the search:
 * plugin or callback code that runs inside another runtime's execution step
 * (where allocating, and the device synchronisation cudaMalloc may imply, is
 * not allowed), programs that reserved their whole device-memory budget at
 * start-up, and latency-critical paths that must not wait on an allocator.
 *
 * Arguments and results are exactly those of awq_search_layer minus `ws` and
 * `ws_bytes`; the caller still provides W, X, a, alphas, losses and
 * row_losses.  The scratch is a file-scope device array of
 * AWQ_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads the
 * library's kernels holds until the process exits.  This call allocates
 * nothing (no cudaMalloc, cudaFree or allocating library routine).
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it; make
 *     that first call before any stream capture on that device.  The cached
 *     address belongs to the device's current primary context: after
 *     cudaDeviceReset (or anything else that destroys that context) it is no
 *     longer valid, so do not call this entry point on that device again in
 *     the same process.
 *   - Layers whose awq_search_workspace_bytes(...) exceeds
 *     AWQ_NOALLOC_SCRATCH_BYTES are rejected with AWQ_ERR_WORKSPACE before
 *     anything is launched.  (The 4096 x 4096, T = 4096, 20-alpha layer needs
 *     about 24 MiB.)
 *   - Every call shares the one array and it keeps the last call's contents.
 *     Nothing in it has to start at zero: each call writes every byte it later
 *     reads.  Calls whose kernels overlap on the GPU (different streams, or
 *     threads without ordering between their streams) race on the array and
 *     corrupt each other's results: order them, e.g. on one stream. */
AWQ_API awq_status awq_search_layer_noalloc(const void *W, int64_t N, int64_t K,
                                            const void *X, int64_t T, int64_t ldx,
                                            const float *a, awq_qcfg q,
                                            const float *alphas, int32_t n_alpha,
                                            float *losses, float *row_losses, void *stream);

/* Search over caller-given scale vectors instead of a^alpha: the baselines
 * and variants the pages measure against AWQ ([AWQ-note] "Measures": plain
 * RTN is s = 1; scaling only the salient 1% of channels by a fixed 2; keeping
 * 1% of the channels in FP16, chosen by activation or by weight magnitude).
 *   s_table  float [n_s, K] (device), every value positive and finite
 *            (otherwise awq_get_status reports AWQ_ERR_INVALID_ARG)
 *   mask     uint8 [K] (device) or NULL: channels held in fp16, as in
 *            awq_quant_dequant_masked; they contribute no output error
 *   losses, row_losses, ws: as awq_search_layer, one entry per scale vector;
 *            ws >= awq_search_scales_workspace_bytes(N, K, T, q, n_s, mask != NULL)
 * 1 <= n_s <= 64.  Everything else as awq_search_layer: with the table's rows
 * equal to a^alpha_i the losses are awq_search_layer's. */
AWQ_API size_t awq_search_scales_workspace_bytes(int64_t N, int64_t K, int64_t T, awq_qcfg q,
                                                 int32_t n_s, int32_t masked);
AWQ_API awq_status awq_search_scales(const void *W, int64_t N, int64_t K, const void *X, int64_t T,
                                     int64_t ldx, awq_qcfg q, const float *s_table, int32_t n_s,
                                     const uint8_t *mask, float *losses, float *row_losses,
                                     void *ws, size_t ws_bytes, void *stream);

/* Channel selection for the FP16-protection baselines: mask[j] = 1 for the k
 * channels with the largest stat[j], 0 for the rest; ties go to the lower
 * index and NaN ranks below every number.  stat is a statistic per input
 * channel: awq_act_stats of X (activation magnitude) or of W read as [N, K]
 * rows (mean |w| per input channel, the weight-magnitude criterion).
 *   stat  float [K] (device);  mask  uint8 [K] output (device);  0 <= k <= K. */
AWQ_API awq_status awq_channel_topk(const float *stat, int64_t K, int64_t k, uint8_t *mask,
                                    void *stream);

/* s[k] = factor where mask[k] != 0, else 1: the scale vector of the variant
 * that scales only the salient channels by a fixed factor ([AWQ-note]
 * "Measures": scaling the 1% salient channels by 2); factor 1 gives plain RTN.
 *   mask  uint8 [K] (device);  s  float [K] output (device);  factor > 0, finite. */
AWQ_API awq_status awq_salient_scales(const uint8_t *mask, int64_t K, float factor, float *s,
                                      void *stream);

/* Output error of any quantized weights W_hat (fp16 [N, K], e.g. from GPTQ):
 *   loss = ||(W_hat - W) X^T||^2 / (N T), row_losses[n] = sum_t ((W_hat - W) X^T)[n, t]^2
 * with (W_hat - W) rounded to fp16 and contracted on the tensor cores as in
 * awq_search_layer.  ws >= awq_output_error_workspace_bytes(N, K, T), 256-byte
 * aligned.  K % 64 == 0. */
AWQ_API size_t awq_output_error_workspace_bytes(int64_t N, int64_t K, int64_t T);
AWQ_API awq_status awq_output_error(const void *W, const void *W_hat, int64_t N, int64_t K,
                                    const void *X, int64_t T, int64_t ldx, float *loss,
                                    float *row_losses, void *ws, size_t ws_bytes, void *stream);

/* AWQ followed by GPTQ error compensation ([AWQ-note] "Measures": AWQ and GPTQ
 * are complementary, AWQ+GPTQ at INT2; [Notes-52] §4: round one column at a time
 * and push its error into the weights not yet quantized, weighted by
 * second-order statistics of the real input; [GPTQ-AWQ] "GPTQ": a column sweep
 * with a Cholesky factor prepared once).  Three steps, all binary32:
 *
 * awq_gptq_hessian: H = 2 X'^T X' with x' = RN32(x RN32(1/s)) -- the input the
 *   scaled layer sees (s = 1 for GPTQ alone, s_best for AWQ+GPTQ).
 *   X fp16 [T, ldx];  s float [K];  H float [K, K] output (full, symmetric).
 *
 * awq_gptq_factor: U, the upper triangular factor with (H + damp mean(diag H) I)^-1
 *   = U^T U (below the diagonal: 0).  Blocked Cholesky of the order-reversed
 *   damped matrix and a blocked triangular inverse.  damp = 0.01 is the usual
 *   choice.  A pivot that is not positive sets a device flag reported by
 *   awq_get_status as AWQ_ERR_INVALID_ARG.  ws >= awq_gptq_factor_workspace_bytes(K).
 *
 * awq_gptq_quantize: per row of w = RN32(W s), for k = 0 .. K-1: at a group's
 *   first column the group parameters of the quantizer of awq_quant_dequant from
 *   the group's current weights; q_k = clamp(rint(w_k r) + z, 0, qmax);
 *   wq = RN32((q_k - z) sh);  e = RN32(RN32(w_k - wq) / U_kk);
 *   w_j = fmaf(-e, U_kj, w_j) for j > k.  Outputs the codes, scales and zeros
 *   in awq_pack's layout (s is the layer's s: s_best for AWQ+GPTQ) and
 *   W_hat = RN16(RN32(wq RN32(1/s))), fp16 [N, K].
 *
 * K % 64 == 0 and K <= 8192 (each row of W stays in shared memory during its
 * sweep); larger K returns AWQ_ERR_INVALID_ARG. */
AWQ_API awq_status awq_gptq_hessian(const void *X, int64_t T, int64_t K, int64_t ldx, const float *s,
                                    float *H, void *stream);
/* The same H on the tensor cores (tcgen05): x' is split into three bf16 pieces
 * whose sum is x' exactly, so every product is exact and only the binary32
 * additions (in the tensor core's order, not token order) round; H is exactly
 * symmetric.  ws >= awq_gptq_hessian_workspace_bytes(T, K) (the pieces, bf16
 * [3][K][T rounded up to 64]), 256-byte aligned; overwritten by every call. */
AWQ_API size_t awq_gptq_hessian_workspace_bytes(int64_t T, int64_t K);
AWQ_API awq_status awq_gptq_hessian_tc(const void *X, int64_t T, int64_t K, int64_t ldx, const float *s,
                                       float *H, void *ws, size_t ws_bytes, void *stream);
AWQ_API size_t awq_gptq_factor_workspace_bytes(int64_t K);
AWQ_API awq_status awq_gptq_factor(const float *H, int64_t K, float damp, float *U, void *ws,
                                   size_t ws_bytes, void *stream);
AWQ_API awq_status awq_gptq_quantize(const void *W, int64_t N, int64_t K, const float *s,
                                     const float *U, awq_qcfg q, uint32_t *codes, void *scales,
                                     void *zeros, void *W_hat, void *stream);

/* Steps a7-a8 -- argmin over the grid and packing ([AWQ-note] "Measures":
 * scale by the best alpha's s, group-quantize, keep the quantized weights and
 * the necessary metadata).
 *   best_idx  int32 [1] output: first index of the smallest loss (NaN = +inf)
 *   s_best    float [K] output: s at the best alpha
 *   codes     uint32 [N, K*c/32] output, c = 4 for bits 3/4 (8 codes per word),
 *             c = 2 for bits 2 (16 per word); code of column k at bit c*(k mod 32/c)
 *             of word k/(32/c) (least significant first)
 *   scales    fp16 [N, K/group_size] output: sh per group
 *   zeros     fp16 [N, K/group_size] output: z per group, an integer (outside
 *             [0, 2^bits - 1] for a group that does not span zero)
 * The argmin runs on the device; nothing is read back to the host.
 * Dequantization: w_hat = RN16(RN32(RN32((code - zero) * scale) * RN32(1/s_best))). */
AWQ_API awq_status awq_pack(const void *W, int64_t N, int64_t K, const float *a, awq_qcfg q,
                    const float *alphas, const float *losses, int32_t n_alpha,
                    int32_t *best_idx, float *s_best, uint32_t *codes,
                    void *scales, void *zeros, void *stream);

/* Step a8 alone for a given scale vector s (float [K], device): the codes,
 * scales and zeros of W diag(s) with the layout of awq_pack (a baseline's
 * packed layer, or a scale chosen elsewhere). */
AWQ_API awq_status awq_pack_scales(const void *W, int64_t N, int64_t K, const float *s, awq_qcfg q,
                                   uint32_t *codes, void *scales, void *zeros, void *stream);

/* Synchronises `stream`, then reports (and clears) errors raised on the device
 * since the last call: AWQ_ERR_TIMEOUT if a kernel's bounded wait ran out,
 * AWQ_ERR_INVALID_ARG if a kernel saw an alpha outside [0, 1], a given scale
 * that is not positive and finite, or a Hessian that is not positive definite,
 * AWQ_ERR_CUDA for
 * a pending CUDA error.  AWQ_OK otherwise. */
AWQ_API awq_status awq_get_status(void *stream);

/* Consumer of the packed format: the quantized linear layer for a few tokens
 * (decode), computed straight from the codes ([AWQ-note] "Tiny Chat": the
 * weights are dequantized inside the kernel and never written back as fp16;
 * [QAS-QA] §5: the layer's input is divided by s).
 *   Y[t, n] = sum_k x'[t, k] * (q[n, k] - z[n, k/g]) * sh[n, k/g],
 *   x'[t, k] = RN32(x[t, k] * RN32(1 / s_best[k])),
 * accumulated in binary32 (summation order unspecified).
 *   codes, scales, zeros, s_best  awq_pack's outputs for W [N, K]
 *   X   fp16 [T, ldx] (the layer's input, not yet divided by s)
 *   Y   float [T, N] output, row-major
 *   ws  device workspace of ws_bytes >= awq_qlinear_workspace_bytes(T, K, N),
 *       256-byte aligned (x' as binary32, partial sums of row blocks split
 *       across thread blocks, arrival counters); overwritten by every call
 * Requires K % 64 == 0.  Built for small T (decode), where streaming the
 * packed codes from HBM is the cost.  awq_qlinear runs awq_qlinear_cc for one
 * token and awq_qlinear_tc from 2 tokens on; either may be called directly.
 * Calls that share a workspace must be ordered (one stream). */
AWQ_API size_t awq_qlinear_workspace_bytes(int64_t T, int64_t K, int64_t N);
/* The kernel awq_qlinear runs for T tokens: 0 the CUDA-core kernel
 * (awq_qlinear_cc), 1 the tensor-core kernel (awq_qlinear_tc).  Host only. */
AWQ_API int32_t awq_qlinear_path(int64_t T);
AWQ_API awq_status awq_qlinear(const uint32_t *codes, const void *scales, const void *zeros,
                               const float *s_best, int64_t N, int64_t K, awq_qcfg q,
                               const void *X, int64_t T, int64_t ldx, float *Y,
                               void *ws, size_t ws_bytes, void *stream);

/* The product on the CUDA cores: binary32 multiply-adds, one, two or four
 * tokens a pass (two for 2-bit codes), each pass re-reading the codes.  The
 * summation order depends on the device's SM count, not on timing: repeated
 * calls on one device give identical Y. */
AWQ_API awq_status awq_qlinear_cc(const uint32_t *codes, const void *scales, const void *zeros,
                                  const float *s_best, int64_t N, int64_t K, awq_qcfg q,
                                  const void *X, int64_t T, int64_t ldx, float *Y,
                                  void *ws, size_t ws_bytes, void *stream);

/* The same product on the tensor cores (tcgen05), for any T.  Identical
 * arguments, workspace (awq_qlinear_workspace_bytes covers both) and result
 * definition as awq_qlinear, evaluated as
 *   Y[t, n] = sum_g sh[n, g] (D_g[n, t] - z[n, g] S_g[t]),
 *   D_g = sum_{k in g} q[n, k] x'[t, k]   (bf16 operands, fp32 accumulation:
 *         q is exact in bf16 and x' is split into three bf16 pieces whose sum
 *         is x' exactly, so every product is exact),
 *   S_g = RN32(sum_{k in g} x'[t, k]) in binary64.
 * Only the binary32 additions round, so the error of a group scales with
 * sh (sum |q x'| + |z S_g|) where the CUDA-core form's scales with
 * sum |x' (q - z)| sh; the two agree closely when a group's codes lie on both
 * sides of z.  Passes of up to 5, 10 or 16 tokens each read the codes once.  The units (128
 * rows x 256 columns) are dealt to the SMs in contiguous ranges; a row block
 * split between two ranges is summed by the last to arrive, in range order, so
 * repeated calls on one device give identical Y.  Calls that share a workspace
 * must be ordered. */
AWQ_API awq_status awq_qlinear_tc(const uint32_t *codes, const void *scales, const void *zeros,
                                  const float *s_best, int64_t N, int64_t K, awq_qcfg q,
                                  const void *X, int64_t T, int64_t ldx, float *Y,
                                  void *ws, size_t ws_bytes, void *stream);

/* Self-test of device-side failure detection (no counterpart on the pages: it
 * checks the library, not the method).  Launches one warp that waits on a
 * barrier nothing ever completes, with the same bounded wait every role of the
 * search kernel uses.  Expected: the launch returns AWQ_OK, the kernel ends by
 * itself after the wait limit (awq_set_wait_timeout_ms), and the next
 * awq_get_status(stream) reports AWQ_ERR_TIMEOUT and clears it; the context
 * stays usable.  Never traps, never faults. */
AWQ_API awq_status awq_selftest_bounded_wait(void *stream);

/* Upper bound, in milliseconds, on any single wait inside the library's
 * kernels (default 4000).  Applies to launches made after the call. */
AWQ_API void awq_set_wait_timeout_ms(uint32_t ms);

/* Profiling hook.  The next awq_search_layer call made by the calling thread
 * records `ev_begin` immediately before and `ev_end` immediately after the
 * launch of its tensor-core search kernel, on that call's stream, so a caller
 * can time that kernel alone with cudaEventElapsedTime.  Both are cudaEvent_t
 * created by the caller; NULL clears the request.  The request is consumed by
 * that one call. */
AWQ_API void awq_profile_next_search(void *ev_begin, void *ev_end);

/* A static, human-readable name for a status code. */
AWQ_API const char *awq_status_string(awq_status s);

#ifdef __cplusplus
}
#endif

#endif /* AWQ_B200_AWQ_H */
