/*
 * sq.h -- C ABI of libsq, the SmoothQuant W8A8 linear layer on NVIDIA B200
 * (sm_100a).
 *
 * The layer computes Y = X W^T with X [T x K] (tokens x input channels) and
 * W [N x K] (output x input channels), summing over K ("One outlier"
 * quantization notes, "Which scales factor out, and why"). SmoothQuant divides
 * activation channel j by s_j and multiplies weight input column j by s_j, an
 * exact rewrite X W^T = (X diag(s)^-1)(W diag(s))^T ("SmoothQuant Explained",
 * "The transform"), then runs both operands through symmetric int8 and an
 * integer GEMM whose epilogue applies one scale per token and one per output
 * channel ("Why do activation outliers break INT8 W8A8 on LLMs...", "A strong
 * answer").
 *
 * Conventions for every call
 *  - Matrices are row-major with leading dimension equal to their column
 *    count, and start on a 16-byte boundary. K (the column count of X and W)
 *    must be a multiple of 16.
 *  - Unless a call says otherwise, pointers are CUDA device memory owned by
 *    the caller. The library never frees or keeps them.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *    default stream). A status of SQ_OK means the arguments were accepted and
 *    the work was enqueued; a kernel-side failure (a bounded wait that ran
 *    out) is reported later by sq_get_status().
 *  - Calls allocate no device memory. sq_w8a8_gemm and sq_linear take a
 *    caller-provided workspace sized by their *_workspace_size function.
 *  - Outputs must not alias inputs.
 *  - There is no CPU fallback: every step runs in this library's kernels.
 *
 * Rounding: round to nearest, ties to even, everywhere a value is rounded.
 * int8 codes use the symmetric range [-127, 127] ("One outlier" notes, "The
 * four operations").
 */
#ifndef SQ_H_
#define SQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
/* Same type as cudaStream_t. */
typedef struct CUstream_st* sq_stream_t;

typedef enum sq_status {
    SQ_OK = 0,
    SQ_ERR_INVALID_ARG = 1,  /* NULL pointer, negative size, alpha outside [0,1], eps < 0,
                                workspace too small */
    SQ_ERR_UNSUPPORTED = 2,  /* K not a multiple of 16, misaligned pointer, unsupported dtype
                                or size */
    SQ_ERR_CUDA = 3,         /* a CUDA runtime call failed; see sq_last_error_string() */
    SQ_ERR_TIMEOUT = 4,      /* a kernel's bounded wait ran out (reported by sq_get_status) */
    SQ_ERR_BOUNDS = 5        /* debug builds only (-DSQ_DEBUG): a kernel's index check found a store
                                outside its buffer and skipped it (reported by sq_get_status) */
} sq_status;

typedef enum sq_dtype {
    SQ_F32 = 0,   /* IEEE binary32 */
    SQ_BF16 = 1,  /* bfloat16 (top half of a binary32) */
    SQ_I32 = 2    /* int32: raw GEMM accumulators (output only) */
} sq_dtype;

/* Library version (major * 10000 + minor * 100 + patch). */
int sq_version(void);

/* ---------------------------------------------------------------- step a1
 * Per-input-channel absolute maximum (calibration).
 *   absmax[j] = max(absmax[j], max_r |x[r, j]|)
 * Defined by the numerator and denominator maxima of the smoothing factor:
 * max_t |X_tj| over tokens and max_n |W_nj| over output channels
 * ("Why do activation outliers break INT8 W8A8...", "A strong answer"; "One
 * outlier" notes, "Route it, or move it": amax over dim 0). Applied to X it
 * calibrates activations; applied to W [N x K] it gives the weight maxima.
 *   x       [rows x cols], dtype dt (SQ_F32 or SQ_BF16), device.
 *   absmax  [cols] float, device, in/out: a running maximum. The caller sets it
 *           to +0 before the first batch; repeated calls over calibration
 *           batches accumulate (the pages warn that the calibration set must
 *           contain the outlier channels' true maxima).
 * cols must be a multiple of 16. rows == 0 is a no-op. NaN inputs are not
 * supported. Exact (max is order-independent). */
sq_status sq_calibrate_absmax(const void* x, sq_dtype dt, int64_t rows, int64_t cols,
                              float* absmax, sq_stream_t stream);

/* ---------------------------------------------------------------- step a2
 * Smoothing factors
 *   s_j = max(xmax_j, eps)^alpha / max(wmax_j, eps)^(1 - alpha)
 * ("SmoothQuant Explained", "Alpha: how much difficulty to move"; the eps
 * clamp of both maxima follows "One outlier" notes, "Route it, or move it").
 * Evaluated in fp64 and rounded once to fp32. For alpha in {0, 1/4, 1/2, 3/4, 1}
 * the powers are exact compositions of correctly rounded sqrt, so the result
 * is reproducible bit for bit; other alphas use pow() (within 1 fp32 ulp of
 * the exact value).
 *   xmax, wmax [K] float, device.   s [K] float, device, out.
 *   alpha in [0, 1], eps >= 0 (1e-8 in the pages). */
sq_status sq_smooth_factors(const float* xmax, const float* wmax, int64_t K, float alpha,
                            float eps, float* s, sq_stream_t stream);

/* ---------------------------------------------------------------- step a3
 * Fold s into the weights and quantize per output channel.
 *   What_nj   = W_nj * s_j                              (fp32)
 *   w_scale_n = max_j |What_nj| / 127                   (1.0 for an all-zero row)
 *   wq_nj     = clamp(round(What_nj / w_scale_n), -127, 127)
 * ("Why do activation outliers break INT8 W8A8...", "A strong answer": the
 * weight columns absorb s_j before quantization, per-output-channel scales;
 * "One outlier" notes, "The four operations" for the quantizer and the
 * zero-range case.)
 *   w        [N x K], dtype dt (SQ_F32 or SQ_BF16), device.
 *   s        [K] float, device.
 *   wq       [N x K] int8, device, out.
 *   w_scale  [N] float, device, out. */
sq_status sq_fold_quant_weights(const void* w, sq_dtype dt, int64_t N, int64_t K,
                                const float* s, int8_t* wq, float* w_scale,
                                sq_stream_t stream);

/* ---------------------------------------------------------------- step a4
 * Smooth the activations and quantize per token (dynamic scale).
 *   Xhat_tj   = X_tj / s_j                              (fp32 division)
 *   x_scale_t = max_j |Xhat_tj| / 127                   (1.0 for an all-zero row)
 *   xq_tj     = clamp(round(Xhat_tj / x_scale_t), -127, 127)
 * ("SmoothQuant Explained", "The transform" and O1 per-token dynamic
 * quantization in "Where it fits"; "Why are activations harder to quantize...",
 * "Dynamic scaling".)
 *   x        [T x K], dtype dt (SQ_F32 or SQ_BF16), device.
 *   s        [K] float, device.
 *   xq       [T x K] int8, device, out.
 *   x_scale  [T] float, device, out. */
sq_status sq_smooth_quant_act(const void* x, sq_dtype dt, int64_t T, int64_t K,
                              const float* s, int8_t* xq, float* x_scale,
                              sq_stream_t stream);

/* ---------------------------------------------------------------- both calibrations in one launch
 * sq_calibrate_absmax_pair: step a1 on the activations x [T x K] into xmax and
 * on the weights w [N x K] into wmax (both running maxima, as
 * sq_calibrate_absmax), in one launch whose blocks are shared between the two
 * tensors, so neither waits for the tail of the other. Same results as the two
 * separate calls, bit for bit. Same dtype for both. */
sq_status sq_calibrate_absmax_pair(const void* x, int64_t T, const void* w, int64_t N, sq_dtype dt,
                                   int64_t K, float* xmax, float* wmax, sq_stream_t stream);

/* ---------------------------------------------------------------- both quantizations in one launch
 * sq_fold_smooth_quant_pair: step a3 on the weights w [N x K] (into wq,
 * w_scale) and step a4 on the activations x [T x K] (into xq, x_scale) with the
 * same smoothing factors s, in one launch where the library's streamed row
 * kernel takes both tensors (bf16 inputs and K within its range), else as the
 * two calls one after the other. Same results as sq_fold_quant_weights
 * followed by sq_smooth_quant_act, bit for bit; same arguments and layouts as
 * those two calls. Same dtype for both inputs. */
sq_status sq_fold_smooth_quant_pair(const void* w, int64_t N, const void* x, int64_t T, sq_dtype dt, int64_t K,
                                    const float* s, int8_t* wq, float* w_scale, int8_t* xq, float* x_scale,
                                    sq_stream_t stream);

/* ---------------------------------------------------------------- per-tensor scales (O2, O3)
 * One activation scale for the whole tensor instead of one per token: the
 * per-tensor dynamic (O2) and per-tensor static (O3) levels of "SmoothQuant
 * Explained", "Where it fits, and where it does not". Static scales are
 * frozen at calibration and clip any later input beyond them; dynamic scales
 * cost a reduction over the tensor before every quantized matmul ("Why are
 * activations harder to quantize than weights in a transformer?", "Static
 * scaling" / "Dynamic scaling").
 *
 * sq_tensor_absmax: running per-tensor range of the smoothed activations,
 *   amax[0] = max(amax[0], max_{r,j} |RN(x[r, j] / s_j)|)
 *   x     [rows x cols], dtype dt (SQ_F32 or SQ_BF16), device.
 *   s     [cols] float, device, every s_j positive and finite; or NULL for the
 *         unsmoothed tensor (the maximum of |x|).
 *   amax  [1] float, device, in/out; the caller sets it to +0 for a fresh
 *         range. On the batch about to be quantized it gives the O2 range;
 *         accumulated over calibration batches (or applied once to the [1 x K]
 *         calibration maxima xmax) it gives the O3 range.
 *   Exact: the division is monotone, so each column's maximum is divided once.
 *
 * sq_quant_act_per_tensor: codes with one scale,
 *   scale   = amax[0] / 127                                  (1.0 if amax[0] == 0)
 *   xq_tj   = clamp(round(RN(x_tj / s_j) / scale), -127, 127)
 *   x_scale_t = scale for every t, so sq_w8a8_gemm applies it unchanged.
 *   x [T x K] (SQ_F32 or SQ_BF16), s [K] or NULL, amax [1] float (read on the
 *   device), xq [T x K] int8 out, x_scale [T] float out: all device.
 *   Values beyond the range clamp to +-127 (the static-scale clipping). */
sq_status sq_tensor_absmax(const void* x, sq_dtype dt, int64_t rows, int64_t cols,
                           const float* s, float* amax, sq_stream_t stream);
sq_status sq_quant_act_per_tensor(const void* x, sq_dtype dt, int64_t T, int64_t K,
                                  const float* s, const float* amax, int8_t* xq,
                                  float* x_scale, sq_stream_t stream);

/* ---------------------------------------------------------------- RMSNorm with the folded gain
 * The deployed form of step a4: diag(s)^-1 folded offline into the gain of
 * the RMSNorm that feeds the layer, so the norm itself emits the smoothed
 * activations ("SmoothQuant Explained", "Why the rescaling is free at
 * runtime"; "Why do activation outliers break INT8 W8A8...", "A strong
 * answer": the 1/s_j folds into the preceding RMSNorm gain).
 *
 * sq_fold_norm_gain (offline):  gain_folded_j = RN(gain_j / s_j)
 *   gain [K] dtype dt (SQ_F32 or SQ_BF16), s [K] float, gain_folded [K] float out.
 *
 * sq_rmsnorm_quant_act: per token row t
 *   r_t     = RN32(1 / sqrt(sum_j x_tj^2 / K + eps))   (fp64 sum and 1/sqrt)
 *   v_tj    = RN(RN(x_tj * r_t) * gain_folded_j)       (the norm output, fp32)
 *   x_scale_t = max_j |v_tj| / 127 (1.0 for an all-zero row),
 *   xq_tj   = clamp(round(v_tj / x_scale_t), -127, 127)
 *   x [T x K] (SQ_F32 or SQ_BF16), gain_folded [K] float, xq [T x K] int8 out,
 *   x_scale [T] float out, inv_rms [T] float out (r_t) or NULL: all device.
 *   eps > 0 (the norm's epsilon). K <= 32768 for SQ_BF16 input, K <= 16384 for
 *   SQ_F32 (the row is held in registers); larger K returns SQ_ERR_UNSUPPORTED.
 *   The norm output is quantized from fp32; it is never rounded to bf16.
 *   The sum of squares is exact per term but its fp64 rounding order is the
 *   kernel's, so r_t may differ from an index-order evaluation in the last
 *   fp32 bit in rare cases; everything after r_t is exact. */
sq_status sq_fold_norm_gain(const void* gain, sq_dtype dt, int64_t K, const float* s,
                            float* gain_folded, sq_stream_t stream);
sq_status sq_rmsnorm_quant_act(const void* x, sq_dtype dt, int64_t T, int64_t K,
                               const float* gain_folded, float eps, int8_t* xq,
                               float* x_scale, float* inv_rms, sq_stream_t stream);

/* ---------------------------------------------------------------- step a5
 * int8 x int8 -> int32 GEMM with the dequantizing epilogue.
 *   acc_tn = sum_k xq_tk * wq_nk                        (exact int32)
 *   y_tn   = (float(acc_tn) * x_scale_t) * w_scale_n    (two fp32 roundings)
 * ("Activation Outlier Channels and Mixed-Precision Decomposition",
 * "Decomposition": integer matmul, float epilogue; "One outlier" notes, "Which
 * scales factor out, and why": per-token and per-output-channel scales leave
 * the integer sum untouched.)
 *   xq [M x K] int8, x_scale [M] float, wq [N x K] int8, w_scale [N] float: device.
 *   y  [M x N], out_dt = SQ_BF16 (fp32 value rounded to nearest even), SQ_F32, or
 *      SQ_I32 (the raw accumulators; scales ignored and may be NULL).
 *   workspace: device, ws_bytes >= sq_w8a8_gemm_workspace_size(M, N, K). When the
 *      required size is non-zero (small M, the split-K weight-streaming path) the
 *      workspace must be zero-filled before its first use; every call that
 *      completes leaves it zero-filled again. Calls that share a workspace must
 *      not overlap on the GPU.
 * |acc| <= 127 * 127 * K, which fits int32 for every K <= 133,144; larger K is
 * rejected (SQ_ERR_UNSUPPORTED). */
size_t sq_w8a8_gemm_workspace_size(int64_t M, int64_t N, int64_t K);
sq_status sq_w8a8_gemm(const int8_t* xq, const float* x_scale, const int8_t* wq,
                       const float* w_scale, int64_t M, int64_t N, int64_t K, void* y,
                       sq_dtype out_dt, void* workspace, size_t ws_bytes,
                       sq_stream_t stream);

/* ---------------------------------------------------------------- mixed-precision decomposition
 * The LLM.int8()-style alternative to smoothing: a static set of outlier
 * input channels keeps full precision and the rest of the contraction runs
 * in int8. The sum over K splits exactly,
 *   Y = X_bulk W_bulk^T + X_out W_out^T,
 * so the only error is that of the bulk quantization, whose scales no longer
 * have to cover the outliers ("Activation Outlier Channels and Mixed-Precision
 * Decomposition", "Decomposition: keep the outliers in high precision"; "One
 * outlier" notes, "Route it, or move it"). The set is chosen once from
 * calibration maxima, so the kernels can specialize on it (same page: a set
 * determined once from calibration and stored with the checkpoint).
 *
 * sq_outlier_split: channel j is an outlier when xmax[j] >= threshold.
 *   xmax [K] float (from sq_calibrate_absmax); keep [K] float out (0 for an
 *   outlier, 1 otherwise); idx [K] int32 out (capacity K), the outlier channels
 *   in ascending order; count [1] int32 out, their number. All device.
 *
 * sq_quant_bulk: per-row int8 of the bulk channels,
 *   scale_r = max_{j: keep_j = 1} |x_rj| / 127   (1.0 if that is 0)
 *   q_rj    = clamp(round(x_rj / scale_r), -127, 127) for bulk channels, 0 for
 *             outlier channels.
 *   Rows of X give per-token scales, rows of W per-output-channel scales.
 *   x [rows x K] (SQ_F32 or SQ_BF16), keep [K] float with every entry exactly 0
 *   or 1, q [rows x K] int8 out, scale [rows] float out: all device.
 *
 * sq_gather_columns: out[r, o] = float(x[r, idx[o]]) for o < n, 0 for
 *   n <= o < ld. x [rows x K] (SQ_F32 or SQ_BF16), idx [n] int32 with entries
 *   in [0, K) (an entry outside reads nothing and gives NaN), out [rows x ld]
 *   float: device. For the outlier operands x_out and w_out below.
 *
 * sq_w8a8_gemm_split: the int8 GEMM of sq_w8a8_gemm over the full K (the
 *   outlier channels hold code 0) plus the outlier term in its epilogue,
 *     y_tn = fma chain over o = 0 .. ld-1 of x_out[t, o] * w_out[n, o],
 *            starting from (float(acc_tn) * x_scale_t) * w_scale_n,
 *   every step an fp32 fused multiply-add, then rounded to out_dt.
 *   x_out [M x ld] and w_out [N x ld] float, device, 16-byte aligned, zero
 *   beyond the real outlier count; ld a multiple of 4 in [0, 32] (ld = 0 is
 *   the plain GEMM). out_dt SQ_F32 or SQ_BF16. Workspace and every other
 *   argument as for sq_w8a8_gemm. */
sq_status sq_outlier_split(const float* xmax, int64_t K, float threshold, float* keep,
                           int32_t* idx, int32_t* count, sq_stream_t stream);
sq_status sq_quant_bulk(const void* x, sq_dtype dt, int64_t rows, int64_t K, const float* keep,
                        int8_t* q, float* scale, sq_stream_t stream);
sq_status sq_gather_columns(const void* x, sq_dtype dt, int64_t rows, int64_t K,
                            const int32_t* idx, int64_t n, int64_t ld, float* out,
                            sq_stream_t stream);
sq_status sq_w8a8_gemm_split(const int8_t* xq, const float* x_scale, const int8_t* wq,
                             const float* w_scale, int64_t M, int64_t N, int64_t K,
                             const float* x_out, const float* w_out, int64_t ld, void* y,
                             sq_dtype out_dt, void* workspace, size_t ws_bytes,
                             sq_stream_t stream);

/* ---------------------------------------------------------------- no-alloc decode GEMM
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory -- a server that has reserved the GPU's
 * memory up front for weights and KV cache, a latency-bound decode loop that
 * cannot afford cudaMalloc's device-wide synchronization, or a plug-in with no
 * access to its host framework's allocator.
 * It computes exactly what sq_w8a8_gemm computes for 1 <= M <= 16 (the split-K
 * weight-streaming path), but keeps that path's scratch (partial sums and
 * completion counters) in a fixed array inside the library instead of a
 * caller workspace, and allocates nothing.
 *   Limits: 1 <= M <= 16 and M * N <= 262,144 (1 MiB + 32 KiB of scratch,
 *   held by every GPU that loads the library until the process exits); larger
 *   sizes return SQ_ERR_UNSUPPORTED with a message. M == 0 or N == 0 is a
 *   no-op.
 *   The first call on a device looks up the scratch array's device address and
 *   keeps it for the life of the process; make that first call before
 *   capturing any stream into a CUDA graph. After cudaDeviceReset on that
 *   device the kept address is stale: do not call this function on that
 *   device again in the same process.
 *   Each call clears the part of the scratch it uses (cudaMemsetAsync on
 *   `stream`) before its kernel. All calls on a device share the one array:
 *   calls that overlap on the GPU (different streams, no ordering between
 *   them) race and give wrong results; serialize them.
 *   Other arguments, layouts and errors are those of sq_w8a8_gemm. */
sq_status sq_w8a8_gemm_noalloc(const int8_t* xq, const float* x_scale, const int8_t* wq,
                               const float* w_scale, int64_t M, int64_t N, int64_t K, void* y,
                               sq_dtype out_dt, sq_stream_t stream);
/* Test hook for the entry point above: fills the current device's whole
 * scratch array with a non-zero byte pattern on `stream`, as a call that
 * stopped early (a bounded wait that ran out) would leave it, so a test can
 * check that the next call still starts from a cleared scratch. */
sq_status sq_selftest_dirty_noalloc_scratch(sq_stream_t stream);

/* ---------------------------------------------------------------- alpha search
 * Per-layer choice of the migration strength: for each candidate alpha the
 * whole path (a2 smoothing factors, a3 fold + quantize W, a4 smooth + quantize
 * X, a5 GEMM with fp32 output) runs on the calibration batch x, and its
 * relative output error
 *   err[a] = ||Yq(alpha_a) - Y||_F / ||Y||_F,   Y = X W^T
 * is returned ("Why do activation outliers break INT8 W8A8...", "A strong
 * answer": the alpha sweep and its W8A8 error column; "SmoothQuant
 * Explained", "Alpha: how much difficulty to move": the best alpha is
 * model-specific). The maxima (a1) come from x and w once. Y is computed once
 * by this library's own kernels: for bf16 operands the tcgen05 GEMM with
 * kind::f16 (every product exact in fp32, the sum accumulated in fp32 in the
 * tensor core's order), for fp32 operands a CUDA-core GEMM (a chain of fp32
 * fused multiply-adds in k order). The sums of squares are fp64.
 *   x [T x K], w [N x K]: dtype in_dt (SQ_F32 or SQ_BF16), device.
 *   alphas [n_alpha] float, HOST, each in [0, 1]; 1 <= n_alpha <= 64.
 *   eps as for sq_smooth_factors.
 *   err [n_alpha] double, HOST, out. best_alpha [1] float, HOST, out (the first
 *   alpha with the smallest error), or NULL.
 *   workspace: device, ws_bytes >= sq_alpha_search_workspace_size(T, N, K,
 *   n_alpha), zero-filled before its first use (it holds a GEMM workspace).
 * The call synchronizes `stream` before it returns (the errors are host
 * values). */
size_t sq_alpha_search_workspace_size(int64_t T, int64_t N, int64_t K, int64_t n_alpha);
sq_status sq_alpha_search(const void* x, const void* w, sq_dtype in_dt, int64_t T, int64_t N,
                          int64_t K, const float* alphas, int64_t n_alpha, float eps,
                          double* err, float* best_alpha, void* workspace, size_t ws_bytes,
                          sq_stream_t stream);

/* ---------------------------------------------------------------- FP8 E4M3 sibling
 * The same layer with FP8 E4M3 codes instead of int8: per-token activation
 * scales and per-output-channel weight scales amax / 448, each quotient
 * converted to E4M3 with round-to-nearest-even and saturation to +-448 (the
 * format has no infinities), and the GEMM on the FP8 tensor cores with fp32
 * accumulation ("Why do activation outliers break INT8 W8A8...", "A strong
 * answer": per-token FP8 activations keep about 3 mantissa bits of relative
 * precision for small values, so smoothing matters less: 3.3% error before
 * smoothing, 2.9% after, on the page's synthetic data).
 *
 * sq_fold_quant_weights_e4m3 / sq_smooth_quant_act_e4m3: as
 *   sq_fold_quant_weights / sq_smooth_quant_act (same fold and smoothing, fp32
 *   division for the quotient), codes are E4M3 bytes, scale = amax / 448 (1.0
 *   for an all-zero row). K <= 65536.
 * sq_w8a8_gemm_e4m3: acc_tn = sum_k dec(xq_tk) dec(wq_nk) accumulated by the
 *   tensor cores in fp32 (every product of two E4M3 values is exact in fp32;
 *   the order of the additions is the hardware's), y_tn = (acc_tn * x_scale_t)
 *   * w_scale_n, out_dt SQ_F32 or SQ_BF16. No workspace. */
sq_status sq_fold_quant_weights_e4m3(const void* w, sq_dtype dt, int64_t N, int64_t K, const float* s,
                                     uint8_t* wq, float* w_scale, sq_stream_t stream);
sq_status sq_smooth_quant_act_e4m3(const void* x, sq_dtype dt, int64_t T, int64_t K, const float* s,
                                   uint8_t* xq, float* x_scale, sq_stream_t stream);
/* sq_fold_smooth_quant_pair_e4m3: sq_fold_quant_weights_e4m3 on w [N x K] and
 *   sq_smooth_quant_act_e4m3 on x [T x K] with the same s, in one launch where
 *   the library's streamed row kernel takes both (bf16 rows that fill its
 *   lanes), else the two calls; same results, bit for bit. */
sq_status sq_fold_smooth_quant_pair_e4m3(const void* w, int64_t N, const void* x, int64_t T, sq_dtype dt, int64_t K,
                                         const float* s, uint8_t* wq, float* w_scale, uint8_t* xq, float* x_scale,
                                         sq_stream_t stream);
sq_status sq_w8a8_gemm_e4m3(const uint8_t* xq, const float* x_scale, const uint8_t* wq,
                            const float* w_scale, int64_t M, int64_t N, int64_t K, void* y,
                            sq_dtype out_dt, sq_stream_t stream);

/* ---------------------------------------------------------------- whole layer
 * The whole path on one batch: calibrate X and W (a1, from zero), smoothing
 * factors (a2), fold + quantize W (a3), smooth + quantize X (a4), GEMM with
 * dequant (a5).
 *   x [M x K], w [N x K]: dtype in_dt (SQ_F32 or SQ_BF16).
 *   y [M x N]: dtype out_dt (SQ_F32 or SQ_BF16).
 *   x, w and y may each be device memory or host memory (pinned host memory
 *   copies asynchronously; pageable host memory makes the copy synchronous).
 *   Host x and w are staged through the workspace by a copy stream of the
 *   library, so that one call's input copies overlap the previous call's GEMM
 *   and output copy: they wait only until the previous call through the same
 *   workspace has finished reading its staged inputs, not for other work
 *   enqueued earlier on `stream` -- the host buffers must hold the inputs when
 *   the call is made. The kernels run on `stream` after those copies. A host y
 *   is copied back on `stream`; the call returns before the copy completes, so
 *   synchronize `stream` before reading it.
 *   workspace: device, ws_bytes >= sq_linear_workspace_size(...); it holds the
 *   maxima, factors, codes, scales and (for host operands) the staged copies.
 *   Zero-fill it once before its first use (it contains the GEMM workspace). */
size_t sq_linear_workspace_size(int64_t M, int64_t N, int64_t K, sq_dtype in_dt,
                                sq_dtype out_dt);
/* Where sq_linear keeps the layer's intermediates inside its workspace, so a
 * caller can read or reuse them after the call (the int8 weights and their
 * scales, say, to run later batches through sq_w8a8_gemm alone): byte offsets
 * from the workspace base of, in this order,
 *   [0] xmax [K] float   [1] wmax [K] float   [2] s [K] float
 *   [3] xq [M x K] int8  [4] x_scale [M] float
 *   [5] wq [N x K] int8  [6] w_scale [N] float
 * (7 entries, each a multiple of 256). They hold the last call's values once
 * that call's work on its stream has completed. Host only (no CUDA call).
 * Returns SQ_ERR_INVALID_ARG for a negative size or NULL offsets, and
 * SQ_ERR_UNSUPPORTED for a dtype sq_linear does not take. */
sq_status sq_linear_workspace_offsets(int64_t M, int64_t N, int64_t K, sq_dtype in_dt,
                                      sq_dtype out_dt, size_t* offsets);
sq_status sq_linear(const void* x, const void* w, sq_dtype in_dt, int64_t M, int64_t N,
                    int64_t K, float alpha, float eps, void* y, sq_dtype out_dt,
                    void* workspace, size_t ws_bytes, sq_stream_t stream);

/* ---------------------------------------------------------------- measurement aid
 * sq_probe_tensor_int8: the int8 tensor-core rate of the current GPU, as a
 * roofline denominator for the int8 GEMM. The pages state only that integer
 * tensor cores run at roughly twice the FP16 rate ("SmoothQuant Explained",
 * "Where it fits"); this measures it. One launch on `stream`: every pair of
 * SMs issues `iters` x 4 of the prefill GEMM's instruction
 * (tcgen05.mma.cta_group::2.kind::i8, 256 x 256 x 32) on operands held in
 * shared memory, with no global-memory traffic. *ops (host, may be NULL)
 * receives the int8 operations the launch performs (2 per multiply-add); the
 * caller times the launch (for example with CUDA events on `stream`).
 * clocks (device, 2 entries, may be NULL) receives, from one SM, the SM clock
 * cycles and the nanoseconds (%globaltimer) spanning its MMAs, so that the
 * rate can be stated per cycle at the clock the launch ran at.
 * iters in [1, 10^7], else SQ_ERR_INVALID_ARG. Computes nothing else. */
sq_status sq_probe_tensor_int8(int64_t iters, double* ops, unsigned long long* clocks,
                               sq_stream_t stream);

/* ---------------------------------------------------------------- status
 * Synchronize `stream`, then return and clear the first error any kernel of
 * this library recorded on the current device since the last call (SQ_OK if
 * none). SQ_ERR_TIMEOUT means a bounded wait inside a kernel ran out; the
 * kernel stopped and the CUDA context stays usable. */
sq_status sq_get_status(sq_stream_t stream);

/* Site code of the error sq_get_status() last returned (0 if none). */
unsigned int sq_last_status_site(void);

/* Human-readable description of the last host-side error on this thread. */
const char* sq_last_error_string(void);

/* Limit, in milliseconds, for every bounded wait inside the kernels (default
 * 2000). Applies to launches made after the call, on every device. */
sq_status sq_set_wait_timeout_ms(int64_t ms);

/* Self-test of the bounded-wait machinery: launches one CTA that waits, with a
 * limit of `limit_us` microseconds, on a barrier that nothing arrives at. The
 * wait runs out, the kernel records SQ_ERR_TIMEOUT and returns. Used by tests
 * to show that a stalled wait ends with a status instead of a hang. */
sq_status sq_selftest_wait_timeout(int64_t limit_us, sq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SQ_H_ */
