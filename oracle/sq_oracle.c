/*
 * sq_oracle.c -- plain, slow, obviously-correct CPU oracle for the SmoothQuant
 * W8A8 linear layer Y = X W^T.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the benchmark's
 * CPU-baseline / reference arm load this library. The product path (the CUDA
 * library and its Python binding) never calls it, and the two share no code,
 * headers, tables or helpers.
 *
 * Sources (web pages on W8A8 post-training quantization and SmoothQuant):
 *   [KJ] "Why are activations harder to quantize than weights in a transformer?"
 *   [SQE] "SmoothQuant Explained"
 *   [II] "Why do activation outliers break INT8 W8A8 on LLMs, and how does
 *        SmoothQuant fix it by moving scale into the weights?"
 *   [MM] "Activation Outlier Channels and Mixed-Precision Decomposition"
 *   [OO] "One outlier" quantization notes (the four operations / which scales
 *        factor out / route it, or move it)
 *
 * Notation follows [OO] "Which scales factor out, and why": X is [T x K]
 * (tokens x input channels), W is [N x K] (output x input channels), and the
 * layer computes Y = X W^T, summing over K.
 *
 * Precision. Everything that decides an int8 code runs in IEEE fp32 in the
 * order written below, with FMA contraction disabled at build time
 * (-ffp-contract=off) and no fast-math, so every step is one correctly
 * rounded fp32 operation. The smoothing factor is evaluated in fp64 and
 * rounded once to fp32. The *_f64 functions are a separate double-precision
 * statement of the same method, used for the identity and error experiments.
 *
 * Every function is a direct loop over the definition: no blocking, no fusion,
 * no reordering. OpenMP only splits independent rows (or, for the column
 * maximum, independent row ranges whose maxima are combined; max is exact and
 * order-free).
 *
 * Planted mistakes. sqo_set_mutation() switches in one deliberate, plausible
 * bug at a time (wrong rounding, missing clamp, transposed operand...). It
 * exists only so the pin tests can show that each such bug fails at least one
 * pin. The default (0) is the correct oracle.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define SQO_F32 0
#define SQO_BF16 1

/* ---- planted-mistake switch (tests only) ---------------------------------- */
enum {
    MUT_NONE = 0,
    MUT_ROUND_HALF_AWAY = 1,   /* round ties away from zero instead of to even */
    MUT_RECIP_SCALE = 2,       /* multiply by 127/amax instead of dividing by amax/127 */
    MUT_NO_CLAMP = 3,          /* cast to int8 without clamping to [-127,127] */
    MUT_ALPHA_SWAPPED = 4,     /* exponents alpha and 1-alpha exchanged */
    MUT_SMOOTH_MULTIPLY = 5,   /* activations multiplied by s instead of divided */
    MUT_GEMM_TRANSPOSED_W = 6, /* W read as [K x N] instead of [N x K] */
    MUT_DEQUANT_DROP_SW = 7,   /* epilogue forgets the weight scale */
    MUT_NO_ZERO_GUARD = 8,     /* all-zero row divides by a zero scale */
    MUT_SCALE_128 = 9,         /* scale = amax/128 (asymmetric range) */
    MUT_FOLD_DIVIDES = 10,     /* weights divided by s instead of multiplied */
    MUT_COLMAX_NO_ABS = 11,    /* column max of signed values, not magnitudes */
    MUT_SMOOTH_WRONG_INDEX = 12, /* activation channel j divided by s[j+1] */
    MUT_TENSOR_MAX_UNSMOOTHED = 13, /* per-tensor maximum taken before smoothing */
    MUT_NORM_NO_EPS = 14,      /* RMSNorm without its epsilon */
    MUT_NORM_MEAN_ABS = 15,    /* RMSNorm from the mean |x| instead of the mean square */
    MUT_SPLIT_MAX_ALL = 16,    /* bulk scale taken over the outlier channels too */
    MUT_SPLIT_DROP_OUTLIERS = 17, /* decomposition forgets the floating-point term */
    MUT_E4M3_TRUNCATE = 18,    /* FP8 E4M3 conversion truncates instead of rounding */
    MUT_POW_EXPONENT = 19      /* generic alpha: pow(v, 1 - a) instead of pow(v, a) */
};
static int g_mutation = MUT_NONE;

void sqo_set_mutation(int m) { g_mutation = m; }
int sqo_get_mutation(void) { return g_mutation; }
int sqo_version(void) { return 1; }

/* ---- bf16 <-> fp32 (own definitions) -------------------------------------- */

/* A bf16 value is the top 16 bits of an fp32 value, so widening is exact. */
float sqo_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even (finite inputs; NaN kept quiet). */
uint16_t sqo_f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

static float load_elem(const void *p, int dt, int64_t i)
{
    if (dt == SQO_BF16)
        return sqo_bf16_to_f32(((const uint16_t *)p)[i]);
    return ((const float *)p)[i];
}

/* ---- the quantizer primitive ---------------------------------------------- */

/* Round to nearest integer, ties to even: the rounding of np.round and
 * torch.round used by the pages' quantizers ([II] q8; [OO] "The four
 * operations"). nearbyintf follows the default FE_TONEAREST mode. */
static float round_code(float v)
{
    if (g_mutation == MUT_ROUND_HALF_AWAY)
        return roundf(v);
    return nearbyintf(v);
}

/* q = clamp(round(v / scale), -127, 127) ([OO] "The four operations":
 * round, then clamp, so 127.6 becomes 127 and never wraps to -128). */
static int8_t code_of(float v, float scale, float amax)
{
    float r;
    if (g_mutation == MUT_RECIP_SCALE)
        r = round_code(v * (127.0f / amax));
    else
        r = round_code(v / scale);
    if (g_mutation == MUT_NO_CLAMP)
        return (int8_t)(int32_t)r; /* wraps modulo 256 */
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    return (int8_t)r;
}

/* Symmetric int8 quantization of one row with a dynamic scale:
 *   amax  = max_j |v_j|
 *   scale = amax / 127        (n = 2^(8-1) - 1 = 127, [OO] "The four operations")
 *   q_j   = clamp(round(v_j / scale), -127, 127)
 * An all-zero row is legal input and gives scale 1 with all codes 0 ([OO],
 * "Handle the zero-range case"). */
void sqo_quant_row(const float *v, int64_t K, int8_t *q, float *scale_out)
{
    float amax = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
        float a = fabsf(v[j]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0f && g_mutation != MUT_NO_ZERO_GUARD) {
        for (int64_t j = 0; j < K; ++j) q[j] = 0;
        *scale_out = 1.0f;
        return;
    }
    float scale = (g_mutation == MUT_SCALE_128) ? amax / 128.0f : amax / 127.0f;
    for (int64_t j = 0; j < K; ++j) q[j] = code_of(v[j], scale, amax);
    *scale_out = scale;
}

/* The same quantizer with a given (static) scale instead of a row maximum
 * ([OO] quantize_dequantize with an explicit clip; [KJ] "Static scaling").
 * Values beyond the grid are clamped, not represented. */
void sqo_quant_fixed(const float *v, int64_t n, float scale, int8_t *q)
{
    for (int64_t i = 0; i < n; ++i) q[i] = code_of(v[i], scale, 127.0f * scale);
}

/* ---- a1: per-input-channel absolute maximum (calibration) ----------------- */

/* absmax[j] = max(absmax[j], max_r |x[r, j]|) over rows r of a row-major
 * [rows x cols] matrix. Applied to activations X it gives max_t |X_tj|; applied
 * to weights W [N x K] it gives max_n |W_nj| ([II] smoothing-factor formula;
 * [OO] "Route it, or move it": amax over dim 0 for both act and weight).
 * The caller initialises absmax (to +0 for a fresh calibration); repeated calls
 * over calibration batches keep a running maximum. */
void sqo_col_absmax(const void *x, int dt, int64_t rows, int64_t cols, float *absmax)
{
#pragma omp parallel
    {
        float *part = (float *)calloc((size_t)cols, sizeof(float));
        int have = 0;
#pragma omp for schedule(static)
        for (int64_t r = 0; r < rows; ++r) {
            have = 1;
            for (int64_t j = 0; j < cols; ++j) {
                float v = load_elem(x, dt, r * cols + j);
                float a = (g_mutation == MUT_COLMAX_NO_ABS) ? v : fabsf(v);
                if (a > part[j]) part[j] = a;
            }
        }
#pragma omp critical
        {
            if (have)
                for (int64_t j = 0; j < cols; ++j)
                    if (part[j] > absmax[j]) absmax[j] = part[j];
        }
        free(part);
    }
}

/* ---- a2: smoothing factors ------------------------------------------------ */

/* v^a for the exponents the method uses, each an exact composition of
 * correctly rounded fp64 operations; any other exponent goes through pow(). */
static double pow_alpha(double v, double a)
{
    if (a == 0.0) return 1.0;
    if (a == 1.0) return v;
    if (a == 0.5) return sqrt(v);
    if (a == 0.25) return sqrt(sqrt(v));
    if (a == 0.75) return sqrt(v) * sqrt(sqrt(v));
    if (g_mutation == MUT_POW_EXPONENT) return pow(v, 1.0 - a);
    return pow(v, a);
}

/* s_j = max(|X_j|)^alpha / max(|W_j|)^(1-alpha)   ([SQE] "Alpha: how much
 * difficulty to move"; [II] "A strong answer"), with both maxima first clamped
 * from below by eps ([OO] "Route it, or move it": clamp_min(eps) on x_max and
 * w_max). Evaluated in fp64, rounded once to fp32. */
void sqo_smooth_factors(const float *xmax, const float *wmax, int64_t K,
                        float alpha, float eps, float *s)
{
    double a = (double)alpha;
    double b = 1.0 - a;
    if (g_mutation == MUT_ALPHA_SWAPPED) { double t = a; a = b; b = t; }
    for (int64_t j = 0; j < K; ++j) {
        float xm = xmax[j] > eps ? xmax[j] : eps;
        float wm = wmax[j] > eps ? wmax[j] : eps;
        double v = pow_alpha((double)xm, a) / pow_alpha((double)wm, b);
        s[j] = (float)v;
    }
}

/* ---- a3: fold s into the weights, then per-output-channel int8 ------------ */

/* For each output row n:  What_nj = W_nj * s_j  (fp32), then the dynamic
 * symmetric quantizer over the row gives wq[n, :] and w_scale[n].
 * Multiplying input column j of W by s_j is the weight side of
 * X W^T = (X diag(s)^-1)(W diag(s))^T ([II] "A strong answer"; [OO] "Route
 * it, or move it"). A per-output-channel scale factors out of the sum over K
 * ([OO] "Which scales factor out, and why"). */
void sqo_fold_quant_weights(const void *w, int dt, int64_t N, int64_t K, const float *s,
                            int8_t *wq, float *w_scale)
{
#pragma omp parallel
    {
        float *row = (float *)malloc((size_t)K * sizeof(float));
#pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            for (int64_t j = 0; j < K; ++j) {
                float v = load_elem(w, dt, n * K + j);
                row[j] = (g_mutation == MUT_FOLD_DIVIDES) ? v / s[j] : v * s[j];
            }
            sqo_quant_row(row, K, wq + n * K, w_scale + n);
        }
        free(row);
    }
}

/* ---- a4: smooth the activations, then per-token int8 ---------------------- */

/* For each token row t:  Xhat_tj = X_tj / s_j  (fp32 division, as written
 * "X / s" and "act / D" on the pages), then the dynamic symmetric quantizer
 * over the row gives xq[t, :] and x_scale[t] (per-token dynamic scale
 * amax/127, [II] "A strong answer"; [SQE] O1 "per-token dynamic"). */
void sqo_smooth_quant_act(const void *x, int dt, int64_t T, int64_t K, const float *s,
                          int8_t *xq, float *x_scale)
{
#pragma omp parallel
    {
        float *row = (float *)malloc((size_t)K * sizeof(float));
#pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            for (int64_t j = 0; j < K; ++j) {
                float v = load_elem(x, dt, t * K + j);
                if (g_mutation == MUT_SMOOTH_MULTIPLY)
                    row[j] = v * s[j];
                else if (g_mutation == MUT_SMOOTH_WRONG_INDEX)
                    row[j] = v / s[(j + 1) % K];
                else
                    row[j] = v / s[j];
            }
            sqo_quant_row(row, K, xq + t * K, x_scale + t);
        }
        free(row);
    }
}

/* ---- a5: int8 x int8 -> int32 GEMM and the dequantizing epilogue ---------- */

/* acc[t, n] = sum_k xq[t, k] * wq[n, k], accumulated exactly in int64 and
 * stored as int32. Returns the number of entries that do not fit in int32
 * (0 for every K below 133,144, since |acc| <= 127*127*K). ([MM] "Decomposition":
 * integer matmul, float epilogue; [OO] "Which scales factor out, and why".) */
int64_t sqo_gemm_i8(const int8_t *xq, const int8_t *wq, int64_t M, int64_t N, int64_t K,
                    int32_t *acc)
{
    int64_t overflow = 0;
#pragma omp parallel for schedule(static) reduction(+ : overflow)
    for (int64_t t = 0; t < M; ++t) {
        for (int64_t n = 0; n < N; ++n) {
            int64_t sum = 0;
            for (int64_t k = 0; k < K; ++k) {
                int64_t wv = (g_mutation == MUT_GEMM_TRANSPOSED_W) ? wq[k * N + n] : wq[n * K + k];
                sum += (int64_t)xq[t * K + k] * wv;
            }
            if (sum > INT32_MAX || sum < INT32_MIN) overflow += 1;
            acc[t * N + n] = (int32_t)sum;
        }
    }
    return overflow;
}

/* Y[t, n] = (float(acc[t, n]) * x_scale[t]) * w_scale[n]: the per-token and
 * per-output-channel scales applied once after the integer sum, each product
 * one fp32 rounding. y_f32 and/or y_bf16 may be NULL; the bf16 output is the
 * fp32 value rounded to nearest-even. */
void sqo_dequant(const int32_t *acc, const float *x_scale, const float *w_scale,
                 int64_t M, int64_t N, float *y_f32, uint16_t *y_bf16)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < M; ++t) {
        for (int64_t n = 0; n < N; ++n) {
            float y = (float)acc[t * N + n] * x_scale[t];
            if (g_mutation != MUT_DEQUANT_DROP_SW) y = y * w_scale[n];
            if (y_f32) y_f32[t * N + n] = y;
            if (y_bf16) y_bf16[t * N + n] = sqo_f32_to_bf16_rne(y);
        }
    }
}

/* ---- fp64 statement of the method (identity and error experiments) ------- */

/* Y = X W^T in fp64: Y[t, n] = sum_k X[t, k] W[n, k]. */
void sqo_matmul_xwT_f64(const double *X, const double *W, int64_t T, int64_t N, int64_t K,
                        double *Y)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t n = 0; n < N; ++n) {
            double sum = 0.0;
            for (int64_t k = 0; k < K; ++k) sum += X[t * K + k] * W[n * K + k];
            Y[t * N + n] = sum;
        }
}

void sqo_col_absmax_f64(const double *x, int64_t rows, int64_t cols, double *absmax)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < cols; ++j) {
            double v = x[r * cols + j];
            double a = (g_mutation == MUT_COLMAX_NO_ABS) ? v : fabs(v);
            if (a > absmax[j]) absmax[j] = a;
        }
}

/* s_j = max(xmax_j, eps)^alpha / max(wmax_j, eps)^(1-alpha) in fp64 (eps = 0
 * reproduces the unclamped form of [II]). */
void sqo_smooth_factors_f64(const double *xmax, const double *wmax, int64_t K,
                            double alpha, double eps, double *s)
{
    double a = alpha, b = 1.0 - alpha;
    if (g_mutation == MUT_ALPHA_SWAPPED) { double t = a; a = b; b = t; }
    for (int64_t j = 0; j < K; ++j) {
        double xm = xmax[j] > eps ? xmax[j] : eps;
        double wm = wmax[j] > eps ? wmax[j] : eps;
        s[j] = pow_alpha(xm, a) / pow_alpha(wm, b);
    }
}

/* Xs = X diag(s)^-1 and Ws = W diag(s): channel j of X divided by s_j, input
 * column j of W multiplied by s_j. */
void sqo_smooth_f64(const double *X, const double *W, const double *s, int64_t T, int64_t N,
                    int64_t K, double *Xs, double *Ws)
{
    for (int64_t t = 0; t < T; ++t)
        for (int64_t j = 0; j < K; ++j) {
            double v = X[t * K + j];
            if (g_mutation == MUT_SMOOTH_MULTIPLY)
                Xs[t * K + j] = v * s[j];
            else if (g_mutation == MUT_SMOOTH_WRONG_INDEX)
                Xs[t * K + j] = v / s[(j + 1) % K];
            else
                Xs[t * K + j] = v / s[j];
        }
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K; ++j) {
            double v = W[n * K + j];
            Ws[n * K + j] = (g_mutation == MUT_FOLD_DIVIDES) ? v / s[j] : v * s[j];
        }
}

static double round_code_f64(double v)
{
    if (g_mutation == MUT_ROUND_HALF_AWAY) return round(v);
    return nearbyint(v);
}

/* Per-row symmetric int8 in fp64: scale = amax/127, q = clamp(round(v/scale)). */
void sqo_quant_rows_f64(const double *v, int64_t rows, int64_t K, int8_t *q, double *scale)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const double *row = v + r * K;
        double amax = 0.0;
        for (int64_t j = 0; j < K; ++j) {
            double a = fabs(row[j]);
            if (a > amax) amax = a;
        }
        if (amax == 0.0 && g_mutation != MUT_NO_ZERO_GUARD) {
            for (int64_t j = 0; j < K; ++j) q[r * K + j] = 0;
            scale[r] = 1.0;
            continue;
        }
        double sc = (g_mutation == MUT_SCALE_128) ? amax / 128.0 : amax / 127.0;
        for (int64_t j = 0; j < K; ++j) {
            double c = (g_mutation == MUT_RECIP_SCALE) ? round_code_f64(row[j] * (127.0 / amax))
                                                       : round_code_f64(row[j] / sc);
            if (g_mutation == MUT_NO_CLAMP) {
                q[r * K + j] = (int8_t)(int32_t)c;
                continue;
            }
            if (c > 127.0) c = 127.0;
            if (c < -127.0) c = -127.0;
            q[r * K + j] = (int8_t)c;
        }
        scale[r] = sc;
    }
}

/* Yq[t, n] = (sum_k xq[t,k] wq[n,k]) * sa[t] * sw[n] in fp64, the integer sum
 * exact. */
void sqo_w8a8_f64(const int8_t *xq, const double *sa, const int8_t *wq, const double *sw,
                  int64_t T, int64_t N, int64_t K, double *Yq)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t n = 0; n < N; ++n) {
            int64_t sum = 0;
            for (int64_t k = 0; k < K; ++k) {
                int64_t wv = (g_mutation == MUT_GEMM_TRANSPOSED_W) ? wq[k * N + n] : wq[n * K + k];
                sum += (int64_t)xq[t * K + k] * wv;
            }
            double y = (double)sum * sa[t];
            if (g_mutation != MUT_DEQUANT_DROP_SW) y *= sw[n];
            Yq[t * N + n] = y;
        }
}

/* ||Yq - Y||_F / ||Y||_F, the W8A8 relative output error of [II]. */
double sqo_rel_frobenius_f64(const double *Yq, const double *Y, int64_t n)
{
    double num = 0.0, den = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        double d = Yq[i] - Y[i];
        num += d * d;
        den += Y[i] * Y[i];
    }
    return sqrt(num) / sqrt(den);
}

/* ======================================================================
 * Next steps on the same layer: other activation granularities, the norm
 * fold, the outlier decomposition and the FP8 sibling. Same rules as above:
 * direct loops over each definition, fp32 in the order written unless noted.
 * ====================================================================== */

/* ---- per-tensor activation scales (O2 dynamic, O3 static) ---------------- */

/* Smoothed value of one activation: RN(x / s_j), or x itself when s is NULL
 * (the unsmoothed layer). */
static float smoothed(const void *x, int dt, int64_t i, const float *s, int64_t j)
{
    float v = load_elem(x, dt, i);
    return s ? v / s[j] : v;
}

/* amax = max(amax, max_{t,j} |RN(X_tj / s_j)|) over a [rows x cols] batch: the
 * single range a per-tensor scale must cover ([KJ] "The outlier structure": a
 * symmetric per-tensor scale covers the largest absolute value present). Run
 * on the batch being quantized it gives the dynamic per-tensor range (O2);
 * accumulated over calibration batches it gives the frozen static range (O3,
 * [KJ] "Static scaling"; [SQE] "Where it fits": O2 and O3). The caller
 * initialises amax (+0 for a fresh range). */
void sqo_tensor_absmax(const void *x, int dt, int64_t rows, int64_t cols, const float *s,
                       float *amax)
{
    float m = *amax;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < cols; ++j) {
            float v = (g_mutation == MUT_TENSOR_MAX_UNSMOOTHED) ? load_elem(x, dt, r * cols + j)
                                                                : smoothed(x, dt, r * cols + j, s, j);
            float a = fabsf(v);
            if (a > m) m = a;
        }
    *amax = m;
}

/* Per-tensor symmetric int8 of the smoothed activations with a given range
 * amax: scale = amax / 127 (1 for amax = 0), q = clamp(round(RN(X/s) / scale),
 * -127, 127). With a static (calibrated) range the clamp is what happens to an
 * input beyond it ([KJ] "Static scaling": such inputs are clipped; [OO] "The
 * four operations"). Every x_scale[t] is set to the one scale, so the
 * per-token epilogue of the GEMM applies it unchanged. */
void sqo_quant_act_per_tensor(const void *x, int dt, int64_t T, int64_t K, const float *s,
                              float amax, int8_t *xq, float *x_scale)
{
    const float scale = (amax == 0.0f) ? 1.0f : amax / 127.0f;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t j = 0; j < K; ++j)
            xq[t * K + j] = (amax == 0.0f) ? 0 : code_of(smoothed(x, dt, t * K + j, s, j), scale, amax);
        x_scale[t] = scale;
    }
}

/* ---- RMSNorm with the smoothing folded into its gain ---------------------- */

/* g'_j = RN(g_j / s_j): diag(s)^-1 folded into the norm's per-channel gain
 * offline ([SQE] "Why the rescaling is free at runtime"; [II] "What
 * SmoothQuant does": the 1/s_j folds into the preceding RMSNorm gain). */
void sqo_fold_norm_gain(const void *g, int dt, int64_t K, const float *s, float *gf)
{
    for (int64_t j = 0; j < K; ++j) gf[j] = load_elem(g, dt, j) / s[j];
}

/* RMSNorm of one token row followed by the per-token quantizer:
 *   r_t   = 1 / sqrt(sum_j x_tj^2 / K + eps), in fp64 (sum in index order),
 *           rounded once to fp32
 *   xh_tj = RN(RN(x_tj * r_t) * g'_j)          (fp32, the norm's output)
 *   (xq[t, :], x_scale[t]) = dynamic symmetric int8 of xh_t
 * The norm emits the smoothed activations directly, so the separate division
 * by s disappears from the runtime ([SQE] "Why the rescaling is free at
 * runtime"). If r_in is not NULL its r_t is used instead of the computed one;
 * r_out (may be NULL) receives the r_t used. */
void sqo_rmsnorm_quant_act(const void *x, int dt, int64_t T, int64_t K, const float *gf, float eps,
                           const float *r_in, int8_t *xq, float *x_scale, float *r_out)
{
#pragma omp parallel
    {
        float *row = (float *)malloc((size_t)K * sizeof(float));
#pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            float r;
            if (r_in) {
                r = r_in[t];
            } else {
                double ss = 0.0;
                for (int64_t j = 0; j < K; ++j) {
                    double v = (double)load_elem(x, dt, t * K + j);
                    ss += (g_mutation == MUT_NORM_MEAN_ABS) ? fabs(v) : v * v;
                }
                double ms = ss / (double)K;
                if (g_mutation == MUT_NORM_MEAN_ABS) ms = ms * ms;
                if (g_mutation != MUT_NORM_NO_EPS) ms = ms + (double)eps;
                r = (float)(1.0 / sqrt(ms));
            }
            for (int64_t j = 0; j < K; ++j) {
                float v = load_elem(x, dt, t * K + j) * r;
                row[j] = v * gf[j];
            }
            sqo_quant_row(row, K, xq + t * K, x_scale + t);
            if (r_out) r_out[t] = r;
        }
        free(row);
    }
}

/* ---- mixed-precision decomposition (LLM.int8()-style) --------------------- */

/* Static outlier set from calibration maxima: channel j is an outlier when
 * xmax_j >= threshold. keep[j] = 0 for outliers, 1 otherwise; idx receives the
 * outlier channels in ascending order; returns their count ([MM]
 * "Decomposition": a set determined once from calibration and stored with the
 * checkpoint). */
int64_t sqo_outlier_split(const float *xmax, int64_t K, float threshold, float *keep, int32_t *idx)
{
    int64_t n = 0;
    for (int64_t j = 0; j < K; ++j) {
        if (xmax[j] >= threshold) {
            keep[j] = 0.0f;
            idx[n++] = (int32_t)j;
        } else {
            keep[j] = 1.0f;
        }
    }
    return n;
}

/* Per-row int8 of the bulk (non-outlier) channels: the row's scale covers the
 * bulk only and the outlier channels get code 0, so an integer GEMM over the
 * full K sums exactly the bulk terms ([MM] "Decomposition": the bulk
 * quantization uses a scale chosen for the bulk distribution; [OO] "Route it,
 * or move it"). Rows of X give per-token scales, rows of W per-output-channel
 * scales. */
void sqo_quant_bulk(const void *x, int dt, int64_t rows, int64_t K, const float *keep, int8_t *q,
                    float *scale)
{
#pragma omp parallel
    {
        float *row = (float *)malloc((size_t)K * sizeof(float));
#pragma omp for schedule(static)
        for (int64_t r = 0; r < rows; ++r) {
            for (int64_t j = 0; j < K; ++j) {
                float v = load_elem(x, dt, r * K + j);
                row[j] = (keep[j] != 0.0f || g_mutation == MUT_SPLIT_MAX_ALL) ? v : 0.0f;
            }
            sqo_quant_row(row, K, q + r * K, scale + r);
            if (g_mutation == MUT_SPLIT_MAX_ALL)
                for (int64_t j = 0; j < K; ++j)
                    if (keep[j] == 0.0f) q[r * K + j] = 0;
        }
        free(row);
    }
}

/* out[r, o] = x[r, idx[o]] as fp32 for o < n, 0 for n <= o < ld: the outlier
 * channels gathered into a dense [rows x ld] matrix. */
void sqo_gather_columns(const void *x, int dt, int64_t rows, int64_t K, const int32_t *idx, int64_t n,
                        int64_t ld, float *out)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t o = 0; o < ld; ++o)
            out[r * ld + o] = (o < n) ? load_elem(x, dt, r * K + idx[o]) : 0.0f;
}

/* Y = Y_bulk + X_out W_out^T ([OO] "Route it, or move it": the sum over K
 * splits into the int8 term and a thin floating-point term; [MM]
 * "Decomposition"): Y_bulk = (float(acc) * sa_t) * sw_n as in the plain
 * epilogue, the outlier term sum_o x_out[t,o] w_out[n,o] in fp64, their sum
 * rounded once to fp32 (and that value to bf16). mag (may be NULL) receives
 * |Y_bulk| + sum_o |x_out w_out|, the scale of the rounding error any fp32
 * evaluation order makes. */
void sqo_dequant_split(const int32_t *acc, const float *x_scale, const float *w_scale, int64_t M,
                       int64_t N, const float *x_out, const float *w_out, int64_t n, int64_t ld,
                       float *y_f32, uint16_t *y_bf16, double *mag)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < M; ++t) {
        for (int64_t c = 0; c < N; ++c) {
            float yb = ((float)acc[t * N + c] * x_scale[t]) * w_scale[c];
            double yo = 0.0, mo = 0.0;
            for (int64_t o = 0; o < n; ++o) {
                double p = (double)x_out[t * ld + o] * (double)w_out[c * ld + o];
                yo += p;
                mo += fabs(p);
            }
            if (g_mutation == MUT_SPLIT_DROP_OUTLIERS) yo = 0.0;
            float y = (float)((double)yb + yo);
            if (y_f32) y_f32[t * N + c] = y;
            if (y_bf16) y_bf16[t * N + c] = sqo_f32_to_bf16_rne(y);
            if (mag) mag[t * N + c] = fabs((double)yb) + mo;
        }
    }
}

/* ---- FP8 E4M3 sibling ------------------------------------------------------ */

/* E4M3 (the OCP "fn" variant: 4 exponent bits, bias 7, 3 mantissa bits, no
 * infinities, largest finite 448, subnormal step 2^-9). Decoding a byte: */
double sqo_e4m3_to_f64(uint8_t b)
{
    int sign = b >> 7, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Encoding with round to nearest, ties to even, saturating to +-448 (values
 * beyond the largest finite code take it; there is no infinity). The sign
 * of zero is kept. */
uint8_t sqo_e4m3_from_f64(double v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0;
    double a = fabs(v);
    double q;
    if (a >= 448.0) return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {
        q = ldexp(1.0, -9);                 /* subnormal quantum */
    } else {
        int e;
        frexp(a, &e);                       /* a = f * 2^e, f in [0.5, 1) */
        q = ldexp(1.0, e - 1 - 3);          /* 3 mantissa bits below the leading one */
    }
    double k = (g_mutation == MUT_E4M3_TRUNCATE) ? floor(a / q) : nearbyint(a / q);
    double r = k * q;                       /* exact: k < 2^5, q a power of two */
    if (r >= 448.0) return sign | 0x7E;
    if (r == 0.0) return sign;
    if (r < ldexp(1.0, -6)) return sign | (uint8_t)(r / ldexp(1.0, -9));
    int e;
    double f = frexp(r, &e);                /* r = f * 2^e */
    int exp_field = e - 1 + 7;
    int mant = (int)((f * 2.0 - 1.0) * 8.0);
    return sign | (uint8_t)(exp_field << 3) | (uint8_t)mant;
}

/* Per-row FP8 quantization: scale = amax / 448 (1 for an all-zero row),
 * code_j = E4M3(RN(v_j / scale)), the fp32 quotient encoded as above ([II]
 * "The reversal condition is the format": per-token FP8 activations; the
 * same per-row rule gives per-output-channel FP8 weights). */
void sqo_quant_row_e4m3(const float *v, int64_t K, uint8_t *q, float *scale_out)
{
    float amax = 0.0f;
    for (int64_t j = 0; j < K; ++j) {
        float a = fabsf(v[j]);
        if (a > amax) amax = a;
    }
    float scale = (amax == 0.0f) ? 1.0f : amax / 448.0f;
    for (int64_t j = 0; j < K; ++j) q[j] = sqo_e4m3_from_f64((double)(v[j] / scale));
    *scale_out = scale;
}

/* The FP8 path of the layer in fp32, in the order of the int8 path: weights
 * folded (RN(W_nj s_j)) and activations smoothed (RN(X_tj / s_j)) exactly as
 * in steps a3 and a4, then the per-row FP8 quantizer above. */
void sqo_fold_quant_weights_e4m3(const void *w, int dt, int64_t N, int64_t K, const float *s,
                                 uint8_t *wq, float *w_scale)
{
#pragma omp parallel
    {
        float *row = (float *)malloc((size_t)K * sizeof(float));
#pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            for (int64_t j = 0; j < K; ++j) row[j] = load_elem(w, dt, n * K + j) * s[j];
            sqo_quant_row_e4m3(row, K, wq + n * K, w_scale + n);
        }
        free(row);
    }
}

void sqo_smooth_quant_act_e4m3(const void *x, int dt, int64_t T, int64_t K, const float *s,
                               uint8_t *xq, float *x_scale)
{
#pragma omp parallel
    {
        float *row = (float *)malloc((size_t)K * sizeof(float));
#pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            for (int64_t j = 0; j < K; ++j) row[j] = load_elem(x, dt, t * K + j) / s[j];
            sqo_quant_row_e4m3(row, K, xq + t * K, x_scale + t);
        }
        free(row);
    }
}

/* acc[t, n] = sum_k dec(xq[t,k]) dec(wq[n,k]) in fp64 (exact: every product of
 * two E4M3 values has at most 8 significant bits between 2^-18 and 2^17.6, so
 * sums of up to 32768 of them span fewer than 53 bits), then the epilogue of
 * the int8 path on the sum rounded once to fp32:
 *   y = (RN32(acc) * x_scale[t]) * w_scale[n]. mag (may be NULL) receives
 * sum_k |dec(xq) dec(wq)| * x_scale * w_scale, the scale of accumulation error. */
void sqo_gemm_dequant_e4m3(const uint8_t *xq, const float *x_scale, const uint8_t *wq, const float *w_scale,
                           int64_t M, int64_t N, int64_t K, float *y, double *mag)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < M; ++t)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, am = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = sqo_e4m3_to_f64(xq[t * K + k]) * sqo_e4m3_to_f64(wq[n * K + k]);
                acc += p;
                am += fabs(p);
            }
            float v = ((float)acc * x_scale[t]) * w_scale[n];
            y[t * N + n] = v;
            if (mag) mag[t * N + n] = am * (double)x_scale[t] * (double)w_scale[n];
        }
}

/* The same rule in fp64 for the error experiments. */
void sqo_quant_rows_e4m3_f64(const double *v, int64_t rows, int64_t K, uint8_t *q, double *scale)
{
    for (int64_t r = 0; r < rows; ++r) {
        const double *x = v + r * K;
        double amax = 0.0;
        for (int64_t j = 0; j < K; ++j)
            if (fabs(x[j]) > amax) amax = fabs(x[j]);
        double sc = (amax == 0.0) ? 1.0 : amax / 448.0;
        for (int64_t j = 0; j < K; ++j) q[r * K + j] = sqo_e4m3_from_f64(x[j] / sc);
        scale[r] = sc;
    }
}

/* Yq[t, n] = (sum_k dec(xq[t,k]) dec(wq[n,k])) * sa[t] * sw[n] in fp64 (each
 * product of two E4M3 values is exact in fp64; the sum runs in index order). */
void sqo_w8a8_e4m3_f64(const uint8_t *xq, const double *sa, const uint8_t *wq, const double *sw,
                       int64_t T, int64_t N, int64_t K, double *Yq)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += sqo_e4m3_to_f64(xq[t * K + k]) * sqo_e4m3_to_f64(wq[n * K + k]);
            Yq[t * N + n] = acc * sa[t] * sw[n];
        }
}

/* Thread count the OpenMP regions use (reported with CPU timings). */
int sqo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void sqo_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
