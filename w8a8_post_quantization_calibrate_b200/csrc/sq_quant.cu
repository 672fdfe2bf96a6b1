// sq_quant.cu -- the HBM-bound steps of the SmoothQuant W8A8 path on sm_100a:
//   a1  per-input-channel absmax calibration     (sq_calibrate_absmax)
//   a2  smoothing factors                        (sq_smooth_factors)
//   a3  weight fold + per-output-channel int8    (sq_fold_quant_weights)
//   a4  activation smoothing + per-token int8    (sq_smooth_quant_act)
//
// Exactness. Every value that decides an int8 code is one correctly rounded
// fp32 operation in the order the method defines it (explicit __fmul_rn /
// __fdiv_rn, never contracted), rounding to nearest-even, so the codes and
// scales are reproducible bit for bit on any IEEE implementation.
#include <cstdio>
#include <cuda_runtime.h>

#include "sq_device.cuh"
#include "sq_internal.h"

namespace sq {

// ============================================================== a1: column absmax
// Block: 8 warps. Each lane owns VEC consecutive columns (one 16-byte load per
// row); a block covers 32*VEC columns and a chunk of rows, warps striding over
// the rows. Per-column maxima are combined across warps in shared memory and
// merged into the output with an integer atomicMax on the fp32 bit pattern
// (monotone for non-negative floats).
template <typename T>
struct Vec16;
template <>
struct Vec16<float> {
    static constexpr int N = 4;
    static __device__ __forceinline__ void absmax(float (&m)[4], const uint4& v) {
        m[0] = fmaxf(m[0], fabsf(__uint_as_float(v.x)));
        m[1] = fmaxf(m[1], fabsf(__uint_as_float(v.y)));
        m[2] = fmaxf(m[2], fabsf(__uint_as_float(v.z)));
        m[3] = fmaxf(m[3], fabsf(__uint_as_float(v.w)));
    }
};
template <>
struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    static __device__ __forceinline__ void absmax(float (&m)[8], const uint4& v) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            m[2 * i] = fmaxf(m[2 * i], fabsf(bf16_lo(w[i])));
            m[2 * i + 1] = fmaxf(m[2 * i + 1], fabsf(bf16_hi(w[i])));
        }
    }
};

constexpr int kAbsmaxThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kAbsmaxThreads)
col_absmax_kernel(const uint8_t* __restrict__ x, int64_t rows, int64_t cols,
                  int64_t rows_per_chunk, float* __restrict__ absmax) {
    constexpr int VEC = Vec16<T>::N;
    constexpr int TILE = 32 * VEC;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t col = (int64_t)blockIdx.x * TILE + lane * VEC;
    const int64_t r_begin = (int64_t)blockIdx.y * rows_per_chunk;
    const int64_t r_end = min(rows, r_begin + rows_per_chunk);
    const int64_t row_bytes = cols * (int64_t)sizeof(T);

    float m[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) m[i] = 0.0f;

    if (col < cols) {
        const uint8_t* p = x + col * (int64_t)sizeof(T);
        int64_t r = r_begin + warp;
        for (; r + 24 < r_end; r += 32) {
            const uint4 v0 = ld_stream_v4(p + r * row_bytes);
            const uint4 v1 = ld_stream_v4(p + (r + 8) * row_bytes);
            const uint4 v2 = ld_stream_v4(p + (r + 16) * row_bytes);
            const uint4 v3 = ld_stream_v4(p + (r + 24) * row_bytes);
            Vec16<T>::absmax(m, v0);
            Vec16<T>::absmax(m, v1);
            Vec16<T>::absmax(m, v2);
            Vec16<T>::absmax(m, v3);
        }
        for (; r < r_end; r += 8) Vec16<T>::absmax(m, ld_stream_v4(p + r * row_bytes));
    }

    __shared__ float red[8][TILE];
#pragma unroll
    for (int i = 0; i < VEC; ++i) red[warp][lane * VEC + i] = m[i];
    __syncthreads();
    for (int c = threadIdx.x; c < TILE; c += kAbsmaxThreads) {
        float v = red[0][c];
#pragma unroll
        for (int w = 1; w < 8; ++w) v = fmaxf(v, red[w][c]);
        const int64_t gc = (int64_t)blockIdx.x * TILE + c;
        if (gc < cols) atomicMax(reinterpret_cast<int*>(absmax + gc), __float_as_int(v));
    }
}

// ============================================================== a2: smoothing factors
// v^a for the exponents used in practice as exact compositions of correctly
// rounded fp64 square roots and products; other exponents use pow().
__device__ __forceinline__ double pow_alpha_dev(double v, double a) {
    if (a == 0.0) return 1.0;
    if (a == 1.0) return v;
    if (a == 0.5) return __dsqrt_rn(v);
    if (a == 0.25) return __dsqrt_rn(__dsqrt_rn(v));
    if (a == 0.75) return __dmul_rn(__dsqrt_rn(v), __dsqrt_rn(__dsqrt_rn(v)));
    return pow(v, a);
}

__global__ void smooth_factors_kernel(const float* __restrict__ xmax, const float* __restrict__ wmax,
                                      int64_t K, float alpha, float eps, float* __restrict__ s) {
    const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= K) return;
    const float xm = xmax[j] > eps ? xmax[j] : eps;
    const float wm = wmax[j] > eps ? wmax[j] : eps;
    const double a = (double)alpha;
    const double num = pow_alpha_dev((double)xm, a);
    const double den = pow_alpha_dev((double)wm, 1.0 - a);
    s[j] = __double2float_rn(__ddiv_rn(num, den));
}

// ============================================================== a3 / a4: row quantization
// One CTA quantizes one row at a time (grid-strided over rows). Thread t owns
// the 8-element chunks t, t+TPB, ... of the row (at most MAXC of them) and keeps
// the transformed values in registers between the two passes:
//   pass 1: v = in * s (fold, a3) or in / s (smooth, a4); running max |v|
//   block-wide max -> scale = amax / 127 (1 for an all-zero row)
//   pass 2: code = clamp(round_half_even(v / scale), -127, 127), 8 codes per store.
enum RowMode { kFold = 0, kSmooth = 1 };

template <typename T>
struct Chunk8;
template <>
struct Chunk8<float> {
    static __device__ __forceinline__ void load(const float* row, int64_t c, float (&v)[8]) {
        const uint4 a = ld_stream_v4(row + c * 8);
        const uint4 b = ld_stream_v4(row + c * 8 + 4);
        v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y);
        v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
        v[4] = __uint_as_float(b.x); v[5] = __uint_as_float(b.y);
        v[6] = __uint_as_float(b.z); v[7] = __uint_as_float(b.w);
    }
};
template <>
struct Chunk8<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* row, int64_t c, float (&v)[8]) {
        const uint4 a = ld_stream_v4(row + c * 8);
        v[0] = bf16_lo(a.x); v[1] = bf16_hi(a.x);
        v[2] = bf16_lo(a.y); v[3] = bf16_hi(a.y);
        v[4] = bf16_lo(a.z); v[5] = bf16_hi(a.z);
        v[6] = bf16_lo(a.w); v[7] = bf16_hi(a.w);
    }
};

__device__ __forceinline__ uint32_t code8(float v, float scale) {
    int q = __float2int_rn(__fdiv_rn(v, scale));
    q = max(-127, min(127, q));
    return static_cast<uint32_t>(q) & 0xffu;
}

template <typename T, int MODE, int TPB, int MAXC>
__global__ void __launch_bounds__(TPB)
row_quant_kernel(const T* __restrict__ in, int64_t rows, int64_t K, const float* __restrict__ s,
                 int8_t* __restrict__ q, float* __restrict__ scale_out) {
    constexpr int NW = TPB / 32;
    __shared__ float red[2][NW];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t nchunks = K >> 3;
    int parity = 0;

    for (int64_t row = blockIdx.x; row < rows; row += gridDim.x, parity ^= 1) {
        const T* rin = in + row * K;
        float v[MAXC][8];
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < MAXC; ++i) {
            const int64_t c = tid + (int64_t)i * TPB;
            if (c < nchunks) {
                float x[8];
                Chunk8<T>::load(rin, c, x);
                const float4 s0 = __ldg(reinterpret_cast<const float4*>(s + c * 8));
                const float4 s1 = __ldg(reinterpret_cast<const float4*>(s + c * 8 + 4));
                const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    v[i][e] = (MODE == kFold) ? __fmul_rn(x[e], sv[e]) : __fdiv_rn(x[e], sv[e]);
                    amax = fmaxf(amax, fabsf(v[i][e]));
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (lane == 0) red[parity][warp] = amax;
        __syncthreads();
        amax = red[parity][0];
#pragma unroll
        for (int w = 1; w < NW; ++w) amax = fmaxf(amax, red[parity][w]);

        const bool zero = (amax == 0.0f);
        const float scale = zero ? 1.0f : __fdiv_rn(amax, 127.0f);
        int8_t* rq = q + row * K;
#pragma unroll
        for (int i = 0; i < MAXC; ++i) {
            const int64_t c = tid + (int64_t)i * TPB;
            if (c < nchunks) {
                uint2 packed = make_uint2(0u, 0u);
                if (!zero) {
                    packed.x = code8(v[i][0], scale) | (code8(v[i][1], scale) << 8) |
                               (code8(v[i][2], scale) << 16) | (code8(v[i][3], scale) << 24);
                    packed.y = code8(v[i][4], scale) | (code8(v[i][5], scale) << 8) |
                               (code8(v[i][6], scale) << 16) | (code8(v[i][7], scale) << 24);
                }
                *reinterpret_cast<uint2*>(rq + c * 8) = packed;
            }
        }
        if (tid == 0) scale_out[row] = scale;
    }
}

// ============================================================== host side
namespace {

template <typename T, int MODE, int TPB, int MAXC>
sq_status launch_row_quant_inst(const void* in, int64_t rows, int64_t K, const float* s,
                                int8_t* q, float* scale, cudaStream_t st) {
    const int64_t max_blocks = (int64_t)device_info().sm_count * (2048 / TPB);
    const int grid = (int)(rows < max_blocks ? rows : max_blocks);
    row_quant_kernel<T, MODE, TPB, MAXC><<<grid, TPB, 0, st>>>(
        static_cast<const T*>(in), rows, K, s, q, scale);
    return check_launch("row_quant_kernel");
}

template <typename T, int MODE, int TPB>
sq_status launch_row_quant_tpb(int maxc, const void* in, int64_t rows, int64_t K, const float* s,
                               int8_t* q, float* scale, cudaStream_t st) {
    switch (maxc) {
        case 1: return launch_row_quant_inst<T, MODE, TPB, 1>(in, rows, K, s, q, scale, st);
        case 2: return launch_row_quant_inst<T, MODE, TPB, 2>(in, rows, K, s, q, scale, st);
        case 4: return launch_row_quant_inst<T, MODE, TPB, 4>(in, rows, K, s, q, scale, st);
        case 8: return launch_row_quant_inst<T, MODE, TPB, 8>(in, rows, K, s, q, scale, st);
    }
    set_error("internal: unsupported chunk count %d", maxc);
    return SQ_ERR_UNSUPPORTED;
}

int pow2ceil(int64_t v) {
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

template <typename T, int MODE>
sq_status launch_row_quant(const void* in, int64_t rows, int64_t K, const float* s, int8_t* q,
                           float* scale, cudaStream_t st) {
    const int64_t nchunks = K / 8;
    int64_t tpb = pow2ceil((nchunks + 3) / 4);
    if (tpb < 128) tpb = 128;
    if (tpb > 1024) tpb = 1024;
    const int64_t per = (nchunks + tpb - 1) / tpb;
    const int maxc = pow2ceil(per);
    if (maxc > 8) {
        set_error("K=%lld exceeds the row-quantization limit of 65536", (long long)K);
        return SQ_ERR_UNSUPPORTED;
    }
    switch (tpb) {
        case 128: return launch_row_quant_tpb<T, MODE, 128>(maxc, in, rows, K, s, q, scale, st);
        case 256: return launch_row_quant_tpb<T, MODE, 256>(maxc, in, rows, K, s, q, scale, st);
        case 512: return launch_row_quant_tpb<T, MODE, 512>(maxc, in, rows, K, s, q, scale, st);
        default: return launch_row_quant_tpb<T, MODE, 1024>(maxc, in, rows, K, s, q, scale, st);
    }
}

sq_status check_input_dtype(sq_dtype dt) {
    if (dt != SQ_F32 && dt != SQ_BF16) {
        set_error("input dtype must be SQ_F32 or SQ_BF16 (got %d)", (int)dt);
        return SQ_ERR_UNSUPPORTED;
    }
    return SQ_OK;
}

sq_status check_matrix(const void* p, int64_t rows, int64_t cols, const char* name) {
    if (rows < 0 || cols < 0) {
        set_error("%s: negative size (%lld x %lld)", name, (long long)rows, (long long)cols);
        return SQ_ERR_INVALID_ARG;
    }
    if (rows > 0 && cols > 0 && p == nullptr) {
        set_error("%s: NULL pointer", name);
        return SQ_ERR_INVALID_ARG;
    }
    if (cols % 16 != 0) {
        set_error("%s: column count %lld is not a multiple of 16", name, (long long)cols);
        return SQ_ERR_UNSUPPORTED;
    }
    if (p && !aligned16(p)) {
        set_error("%s: pointer is not 16-byte aligned", name);
        return SQ_ERR_UNSUPPORTED;
    }
    return SQ_OK;
}

}  // namespace

sq_status calibrate_absmax_impl(const void* x, sq_dtype dt, int64_t rows, int64_t cols,
                                float* absmax, cudaStream_t st) {
    sq_status r;
    if ((r = check_input_dtype(dt)) != SQ_OK) return r;
    if ((r = check_matrix(x, rows, cols, "x")) != SQ_OK) return r;
    if (cols > 0 && !absmax) { set_error("absmax: NULL pointer"); return SQ_ERR_INVALID_ARG; }
    if (rows == 0 || cols == 0) return SQ_OK;
    const int es = dt == SQ_F32 ? 4 : 2;
    const int64_t tile = 32 * (16 / es);
    const int64_t ct = (cols + tile - 1) / tile;
    const int64_t bytes = rows * cols * es;
    int64_t target = bytes / 65536;
    const int64_t cap = (int64_t)device_info().sm_count * 16;
    if (target > cap) target = cap;
    int64_t rc = target / ct;
    if (rc < 1) rc = 1;
    const int64_t rc_max = (rows + 7) / 8;
    if (rc > rc_max) rc = rc_max;
    if (rc > 65535) rc = 65535;
    const int64_t per = (rows + rc - 1) / rc;
    rc = (rows + per - 1) / per;
    if (ct > 2147483647LL) { set_error("cols too large"); return SQ_ERR_UNSUPPORTED; }
    dim3 grid((unsigned)ct, (unsigned)rc);
    if (dt == SQ_F32)
        col_absmax_kernel<float><<<grid, kAbsmaxThreads, 0, st>>>(
            static_cast<const uint8_t*>(x), rows, cols, per, absmax);
    else
        col_absmax_kernel<__nv_bfloat16><<<grid, kAbsmaxThreads, 0, st>>>(
            static_cast<const uint8_t*>(x), rows, cols, per, absmax);
    return check_launch("col_absmax_kernel");
}

sq_status smooth_factors_impl(const float* xmax, const float* wmax, int64_t K, float alpha,
                              float eps, float* s, cudaStream_t st) {
    if (K < 0) { set_error("K < 0"); return SQ_ERR_INVALID_ARG; }
    if (!(alpha >= 0.0f && alpha <= 1.0f)) { set_error("alpha must be in [0, 1]"); return SQ_ERR_INVALID_ARG; }
    if (!(eps >= 0.0f)) { set_error("eps must be >= 0"); return SQ_ERR_INVALID_ARG; }
    if (K == 0) return SQ_OK;
    if (!xmax || !wmax || !s) { set_error("NULL pointer"); return SQ_ERR_INVALID_ARG; }
    const int threads = 256;
    const int64_t blocks = (K + threads - 1) / threads;
    smooth_factors_kernel<<<(unsigned)blocks, threads, 0, st>>>(xmax, wmax, K, alpha, eps, s);
    return check_launch("smooth_factors_kernel");
}

static sq_status row_quant_common(int mode, const void* in, sq_dtype dt, int64_t rows, int64_t K,
                                  const float* s, int8_t* q, float* scale, cudaStream_t st) {
    sq_status r;
    if ((r = check_input_dtype(dt)) != SQ_OK) return r;
    if ((r = check_matrix(in, rows, K, "input")) != SQ_OK) return r;
    if (rows == 0) return SQ_OK;
    if (K == 0) { set_error("K must be positive"); return SQ_ERR_INVALID_ARG; }
    if (!s || !q || !scale) { set_error("NULL pointer"); return SQ_ERR_INVALID_ARG; }
    if (!aligned16(s) || !aligned16(q)) { set_error("s and codes must be 16-byte aligned"); return SQ_ERR_UNSUPPORTED; }
    if (mode == kFold)
        return dt == SQ_F32 ? launch_row_quant<float, kFold>(in, rows, K, s, q, scale, st)
                            : launch_row_quant<__nv_bfloat16, kFold>(in, rows, K, s, q, scale, st);
    return dt == SQ_F32 ? launch_row_quant<float, kSmooth>(in, rows, K, s, q, scale, st)
                        : launch_row_quant<__nv_bfloat16, kSmooth>(in, rows, K, s, q, scale, st);
}

sq_status fold_quant_weights_impl(const void* w, sq_dtype dt, int64_t N, int64_t K, const float* s,
                                  int8_t* wq, float* w_scale, cudaStream_t st) {
    return row_quant_common(kFold, w, dt, N, K, s, wq, w_scale, st);
}

sq_status smooth_quant_act_impl(const void* x, sq_dtype dt, int64_t T, int64_t K, const float* s,
                                int8_t* xq, float* x_scale, cudaStream_t st) {
    return row_quant_common(kSmooth, x, dt, T, K, s, xq, x_scale, st);
}

}  // namespace sq

extern "C" {

sq_status sq_calibrate_absmax(const void* x, sq_dtype dt, int64_t rows, int64_t cols,
                              float* absmax, sq_stream_t stream) {
    return sq::calibrate_absmax_impl(x, dt, rows, cols, absmax, (cudaStream_t)stream);
}

sq_status sq_smooth_factors(const float* xmax, const float* wmax, int64_t K, float alpha,
                            float eps, float* s, sq_stream_t stream) {
    return sq::smooth_factors_impl(xmax, wmax, K, alpha, eps, s, (cudaStream_t)stream);
}

sq_status sq_fold_quant_weights(const void* w, sq_dtype dt, int64_t N, int64_t K, const float* s,
                                int8_t* wq, float* w_scale, sq_stream_t stream) {
    return sq::fold_quant_weights_impl(w, dt, N, K, s, wq, w_scale, (cudaStream_t)stream);
}

sq_status sq_smooth_quant_act(const void* x, sq_dtype dt, int64_t T, int64_t K, const float* s,
                              int8_t* xq, float* x_scale, sq_stream_t stream) {
    return sq::smooth_quant_act_impl(x, dt, T, K, s, xq, x_scale, (cudaStream_t)stream);
}

}  // extern "C"
