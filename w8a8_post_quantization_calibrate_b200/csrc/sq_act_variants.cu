// sq_act_variants.cu -- the other ways to quantize the activations of the
// smoothed layer:
//   per-tensor scales, dynamic (O2) and static (O3)   (sq_tensor_absmax,
//                                                       sq_quant_act_per_tensor)
//   the smoothing folded into an RMSNorm gain          (sq_fold_norm_gain,
//                                                       sq_rmsnorm_quant_act)
// The per-token dynamic form (O1) is sq_smooth_quant_act in sq_quant.cu.
// Included into the library's single translation unit after sq_quant.cu,
// whose helpers it uses.
#include <cuda_runtime.h>

#include "sq_device.cuh"
#include "sq_internal.h"

namespace sq {

// ============================================================== per-tensor codes
// Same layout as the column-maximum kernel: each lane owns VEC consecutive
// columns (one 16-byte load per row), 8 warps stride over a chunk of rows in
// double-buffered batches of 4 rows per warp, about one wave of blocks. Every lane therefore
// needs the multipliers of its own VEC columns only, kept in registers.
//
// Codes. One scale for the whole tensor, so the two multipliers fold into one:
// c_j = RN(RN(1/s_j) * RN(1/scale)) and q' = RN(x * c_j). Four roundings
// separate q' from x / (s_j scale) and two separate q* = RN(RN(x / s_j) /
// scale) from it, so |q' - q*| <= 6 ulp(|q*|), below 5e-5 while |q*| <= 128.
// q' is clamped to [-127, 127] first (clamp then round = round then clamp for
// an integer bound; a |q'| >= 128 means |q*| > 127.5), then rounded with the
// 1.5 * 2^23 addition; a value within 2^-13 of a half-integer has its code
// recomputed with the two IEEE divisions. Columns whose c_j is outside
// [2^-120, 2^120], or a scale below 2^-100 (where RN(x / s_j) may be
// subnormal), take the IEEE divisions for every element.
constexpr float kPtMinScale = 7.888609052210118e-31f;   // 2^-100
constexpr float kPtMinMul = 7.52316384526264e-37f;      // 2^-120
constexpr float kPtMaxMul = 1.329227995784916e36f;      // 2^120

__device__ __noinline__ uint32_t exact_code_pt(float x, const float* s, int64_t j, float scale) {
    const float v = s ? __fdiv_rn(x, s[j]) : x;
    int qi = __float2int_rn(__fdiv_rn(v, scale));
    qi = max(-127, min(127, qi));
    return (uint32_t)qi & 0xffu;
}

template <typename T>
__global__ void __launch_bounds__(kAbsmaxThreads)
per_tensor_quant_kernel(const uint8_t* __restrict__ x, int64_t rows, int64_t cols, int64_t rows_per_chunk,
                        const float* __restrict__ s, const float* __restrict__ amax_p,
                        int8_t* __restrict__ q, float* __restrict__ x_scale) {
    constexpr int VEC = Vec16<T>::N;
    constexpr int TILE = 32 * VEC;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t col = (int64_t)blockIdx.x * TILE + lane * VEC;
    const int64_t r_begin = (int64_t)blockIdx.y * rows_per_chunk;
    const int64_t r_end = min(rows, r_begin + rows_per_chunk);

    pdl_wait();
    pdl_trigger();
    const float amax = *amax_p;
    const bool zero = !(amax > 0.0f);
    const float scale = zero ? 1.0f : __fdiv_rn(amax, 127.0f);
    if (blockIdx.x == 0 && lane == 0)
        for (int64_t r = r_begin + warp; r < r_end; r += 8) x_scale[r] = scale;
    if (col >= cols) return;

    const float rs = __frcp_rn(scale);
    bool exact = !(scale >= kPtMinScale);
    uint64_t c2[VEC / 2];
#pragma unroll
    for (int p = 0; p < VEC / 2; ++p) {
        float c[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float m = s ? __frcp_rn(__ldg(s + col + 2 * p + h)) : 1.0f;
            c[h] = __fmul_rn(m, rs);
            exact |= !(c[h] >= kPtMinMul && c[h] <= kPtMaxMul);
        }
        c2[p] = f2_pack(c[0], c[1]);
    }
    const uint64_t mag2 = f2_pack(kMagic, kMagic);
    const int64_t row_bytes = cols * (int64_t)sizeof(T);
    const uint8_t* p = x + col * (int64_t)sizeof(T);

    // Batches of kAbsmaxBatch rows per warp, double-buffered: the next batch's
    // loads are issued before the current one is converted.
    constexpr int B = kAbsmaxBatch;
    constexpr int64_t step = 8 * B;
    RawChunk<T> v[B], nxt[B];
    int64_t r = r_begin + warp;
#pragma unroll
    for (int u = 0; u < B; ++u)
        if (r + 8 * u < r_end) v[u].a = ld_stream_v4(p + (r + 8 * u) * row_bytes);   // 16 bytes: 8 bf16 or 4 fp32
    for (; r < r_end; r += step) {
#pragma unroll
        for (int u = 0; u < B; ++u)
            if (r + step + 8 * u < r_end) nxt[u].a = ld_stream_v4(p + (r + step + 8 * u) * row_bytes);
#pragma unroll
        for (int u = 0; u < B; ++u) {
            const int64_t rr = r + 8 * u;
            if (rr >= r_end) continue;
            uint32_t t[VEC];
            if (zero) {
#pragma unroll
                for (int e = 0; e < VEC; ++e) t[e] = 0u;
            } else if (exact) {
#pragma unroll
                for (int e = 0; e < VEC; ++e) t[e] = exact_code_pt(v[u].get(e), s, col + e, scale);
            } else {
                bool near_tie = false;
#pragma unroll
                for (int pp = 0; pp < VEC / 2; ++pp) {
                    float a0, a1;
                    f2_unpack(f2_mul(v[u].pair(pp), c2[pp]), a0, a1);
                    a0 = fminf(fmaxf(a0, -127.0f), 127.0f);
                    a1 = fminf(fmaxf(a1, -127.0f), 127.0f);
                    const uint64_t q2 = f2_pack(a0, a1);
                    const uint64_t t2 = f2_add(q2, mag2);
                    const uint64_t d2 = f2_sub(q2, f2_sub(t2, mag2));
                    float t0, t1, d0, d1;
                    f2_unpack(t2, t0, t1);
                    f2_unpack(d2, d0, d1);
                    t[2 * pp] = __float_as_uint(t0);
                    t[2 * pp + 1] = __float_as_uint(t1);
                    near_tie |= fabsf(d0) >= 0.5f - kTieGuard;
                    near_tie |= fabsf(d1) >= 0.5f - kTieGuard;
                }
                if (near_tie) {
#pragma unroll
                    for (int e = 0; e < VEC; ++e) {
                        float c0, c1;
                        f2_unpack(c2[e / 2], c0, c1);
                        float qv = __fmul_rn(v[u].get(e), (e & 1) ? c1 : c0);
                        qv = fminf(fmaxf(qv, -127.0f), 127.0f);
                        const float dd = __fsub_rn(qv, __fsub_rn(__fadd_rn(qv, kMagic), kMagic));
                        if (fabsf(dd) >= 0.5f - kTieGuard) t[e] = exact_code_pt(v[u].get(e), s, col + e, scale);
                    }
                }
            }
            int8_t* dst = q + rr * cols + col;
            if (VEC == 8) {
                const uint32_t lo = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410);
                const uint32_t hi = __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410);
                *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi);
            } else {
                *reinterpret_cast<uint32_t*>(dst) =
                    __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410);
            }
        }
#pragma unroll
        for (int u = 0; u < B; ++u) v[u] = nxt[u];
    }
}

// ============================================================== norm gain fold
template <typename T>
__global__ void fold_norm_gain_kernel(const T* __restrict__ g, int64_t K, const float* __restrict__ s,
                                      float* __restrict__ gf) {
    const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (j < K) gf[j] = __fdiv_rn((float)g[j], s[j]);
}

// ============================================================== host side
sq_status tensor_absmax_impl(const void* x, sq_dtype dt, int64_t rows, int64_t cols, const float* s,
                             float* amax, cudaStream_t st) {
    sq_status r;
    if ((r = check_input_dtype(dt)) != SQ_OK) return r;
    if ((r = check_matrix(x, rows, cols, "x")) != SQ_OK) return r;
    if (!amax) { set_error("amax: NULL pointer"); return SQ_ERR_INVALID_ARG; }
    if (rows == 0 || cols == 0) return SQ_OK;
    dim3 grid;
    int64_t per = 0;
    const int per_sm = dt == SQ_F32 ? column_blocks_per_sm<col_absmax_kernel<float, true>>()
                                    : column_blocks_per_sm<col_absmax_kernel<__nv_bfloat16, true>>();
    if ((r = absmax_grid(rows, cols, dt == SQ_F32 ? 4 : 2, grid, per, per_sm)) != SQ_OK) return r;
    if (dt == SQ_F32)
        return launch_pdl("col_absmax_kernel<tensor>", col_absmax_kernel<float, true>, grid, dim3(kAbsmaxThreads), 0,
                          st, 1, static_cast<const uint8_t*>(x), rows, cols, per, amax, s, AbsmaxPair{});
    return launch_pdl("col_absmax_kernel<tensor>", col_absmax_kernel<__nv_bfloat16, true>, grid, dim3(kAbsmaxThreads),
                      0, st, 1, static_cast<const uint8_t*>(x), rows, cols, per, amax, s, AbsmaxPair{});
}

sq_status quant_act_per_tensor_impl(const void* x, sq_dtype dt, int64_t T, int64_t K, const float* s,
                                    const float* amax, int8_t* xq, float* x_scale, cudaStream_t st) {
    sq_status r;
    if ((r = check_input_dtype(dt)) != SQ_OK) return r;
    if ((r = check_matrix(x, T, K, "x")) != SQ_OK) return r;
    if (T == 0) return SQ_OK;
    if (K == 0) { set_error("K must be positive"); return SQ_ERR_INVALID_ARG; }
    if (!amax || !xq || !x_scale) { set_error("NULL pointer"); return SQ_ERR_INVALID_ARG; }
    if (!aligned16(xq)) { set_error("codes must be 16-byte aligned"); return SQ_ERR_UNSUPPORTED; }
    dim3 grid;
    int64_t per = 0;
    const int per_sm = dt == SQ_F32 ? column_blocks_per_sm<per_tensor_quant_kernel<float>>()
                                    : column_blocks_per_sm<per_tensor_quant_kernel<__nv_bfloat16>>();
    if ((r = absmax_grid(T, K, dt == SQ_F32 ? 4 : 2, grid, per, per_sm)) != SQ_OK) return r;
    if (dt == SQ_F32)
        return launch_pdl("per_tensor_quant_kernel", per_tensor_quant_kernel<float>, grid, dim3(kAbsmaxThreads), 0, st,
                          1, static_cast<const uint8_t*>(x), T, K, per, s, amax, xq, x_scale);
    return launch_pdl("per_tensor_quant_kernel", per_tensor_quant_kernel<__nv_bfloat16>, grid, dim3(kAbsmaxThreads), 0,
                      st, 1, static_cast<const uint8_t*>(x), T, K, per, s, amax, xq, x_scale);
}

sq_status fold_norm_gain_impl(const void* g, sq_dtype dt, int64_t K, const float* s, float* gf,
                              cudaStream_t st) {
    sq_status r;
    if ((r = check_input_dtype(dt)) != SQ_OK) return r;
    if (K < 0) { set_error("K < 0"); return SQ_ERR_INVALID_ARG; }
    if (K == 0) return SQ_OK;
    if (!g || !s || !gf) { set_error("NULL pointer"); return SQ_ERR_INVALID_ARG; }
    const int threads = 256;
    const unsigned blocks = (unsigned)((K + threads - 1) / threads);
    if (dt == SQ_F32)
        fold_norm_gain_kernel<float><<<blocks, threads, 0, st>>>(static_cast<const float*>(g), K, s, gf);
    else
        fold_norm_gain_kernel<__nv_bfloat16><<<blocks, threads, 0, st>>>(
            static_cast<const __nv_bfloat16*>(g), K, s, gf);
    return check_launch("fold_norm_gain_kernel");
}

sq_status rmsnorm_quant_act_impl(const void* x, sq_dtype dt, int64_t T, int64_t K, const float* gf,
                                 float eps, int8_t* xq, float* x_scale, float* inv_rms, cudaStream_t st) {
    sq_status r;
    if ((r = check_input_dtype(dt)) != SQ_OK) return r;
    if ((r = check_matrix(x, T, K, "x")) != SQ_OK) return r;
    if (!(eps > 0.0f) || !(eps < 3.0e38f)) { set_error("eps must be positive and finite"); return SQ_ERR_INVALID_ARG; }
    if (T == 0) return SQ_OK;
    if (K == 0) { set_error("K must be positive"); return SQ_ERR_INVALID_ARG; }
    if (!gf || !xq || !x_scale) { set_error("NULL pointer"); return SQ_ERR_INVALID_ARG; }
    if (!aligned16(gf) || !aligned16(xq)) { set_error("gain and codes must be 16-byte aligned"); return SQ_ERR_UNSUPPORTED; }
    return dt == SQ_F32
        ? launch_row_quant<float, kNorm>(x, T, K, gf, xq, x_scale, st, eps, inv_rms)
        : launch_row_quant<__nv_bfloat16, kNorm>(x, T, K, gf, xq, x_scale, st, eps, inv_rms);
}

}  // namespace sq

extern "C" {

sq_status sq_tensor_absmax(const void* x, sq_dtype dt, int64_t rows, int64_t cols, const float* s,
                           float* amax, sq_stream_t stream) {
    return sq::tensor_absmax_impl(x, dt, rows, cols, s, amax, (cudaStream_t)stream);
}

sq_status sq_quant_act_per_tensor(const void* x, sq_dtype dt, int64_t T, int64_t K, const float* s,
                                  const float* amax, int8_t* xq, float* x_scale, sq_stream_t stream) {
    return sq::quant_act_per_tensor_impl(x, dt, T, K, s, amax, xq, x_scale, (cudaStream_t)stream);
}

sq_status sq_fold_norm_gain(const void* gain, sq_dtype dt, int64_t K, const float* s, float* gain_folded,
                            sq_stream_t stream) {
    return sq::fold_norm_gain_impl(gain, dt, K, s, gain_folded, (cudaStream_t)stream);
}

sq_status sq_rmsnorm_quant_act(const void* x, sq_dtype dt, int64_t T, int64_t K, const float* gain_folded,
                               float eps, int8_t* xq, float* x_scale, float* inv_rms, sq_stream_t stream) {
    return sq::rmsnorm_quant_act_impl(x, dt, T, K, gain_folded, eps, xq, x_scale, inv_rms,
                                      (cudaStream_t)stream);
}

}  // extern "C"
