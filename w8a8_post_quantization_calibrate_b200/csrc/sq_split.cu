// sq_split.cu -- the host of the mixed-precision decomposition (LLM.int8()
// style): a static set of outlier input channels, chosen once from the
// calibration maxima, stays in floating point while the rest of the
// contraction runs through the int8 path ("Activation Outlier Channels and
// Mixed-Precision Decomposition", "Decomposition: keep the outliers in high
// precision"; "One outlier" notes, "Route it, or move it").
//
// B200 layout. Nothing is compacted along K: the int8 operands keep their full
// [rows x K] layout with code 0 in the outlier channels, so the tensor-core
// GEMM runs unchanged over all of K (a few zero columns cost < 1% of its MACs)
// and needs no gather. Only the outlier columns themselves are gathered, into
// small dense [rows x ld] fp32 matrices that the GEMM epilogue reads
// (sq_w8a8_gemm_split in sq_gemm.cu).
#include <cuda_runtime.h>

#include "sq_device.cuh"
#include "sq_internal.h"

namespace sq {

// One CTA of 1024 threads walks the channels in order; a block-wide prefix
// count of the outlier flags places each outlier index, so idx is ascending
// and the result does not depend on scheduling.
constexpr int kSplitThreads = 1024;

__global__ void __launch_bounds__(kSplitThreads)
outlier_split_kernel(const float* __restrict__ xmax, int64_t K, float threshold, float* __restrict__ keep,
                     int32_t* __restrict__ idx, int32_t* __restrict__ count) {
    __shared__ int warp_tot[32];
    __shared__ int base_sh;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) base_sh = 0;
    __syncthreads();
    for (int64_t j0 = 0; j0 < K; j0 += kSplitThreads) {
        const int64_t j = j0 + tid;
        const bool out = j < K && xmax[j] >= threshold;
        if (j < K) keep[j] = out ? 0.0f : 1.0f;
        const unsigned ball = __ballot_sync(0xffffffffu, out);
        if (lane == 0) warp_tot[warp] = __popc(ball);
        __syncthreads();
        int before = base_sh;
        for (int w = 0; w < warp; ++w) before += warp_tot[w];
        if (out) idx[before + __popc(ball & ((1u << lane) - 1u))] = (int32_t)j;
        __syncthreads();
        if (tid == 0) {
            int tot = 0;
            for (int w = 0; w < kSplitThreads / 32; ++w) tot += warp_tot[w];
            base_sh += tot;
        }
        __syncthreads();
    }
    if (tid == 0) *count = base_sh;
}

// out[r, o] = float(x[r, idx[o]]) for o < n, 0 for n <= o < ld. An index
// outside [0, K) reads nothing and yields NaN.
template <typename T>
__global__ void gather_columns_kernel(const T* __restrict__ x, int64_t rows, int64_t K,
                                      const int32_t* __restrict__ idx, int n, int ld, float* __restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= rows * ld) return;
    const int64_t r = i / ld;
    const int o = (int)(i - r * ld);
    float v = 0.0f;
    if (o < n) {
        const int32_t j = idx[o];
        v = (j >= 0 && j < K) ? (float)x[r * K + j] : __int_as_float(0x7fc00000);
    }
    out[i] = v;
}

sq_status outlier_split_impl(const float* xmax, int64_t K, float threshold, float* keep, int32_t* idx,
                             int32_t* count, cudaStream_t st) {
    if (K < 0) { set_error("K < 0"); return SQ_ERR_INVALID_ARG; }
    if (K > 2147483647LL) { set_error("K too large"); return SQ_ERR_UNSUPPORTED; }
    if (!count || (K > 0 && (!xmax || !keep || !idx))) { set_error("NULL pointer"); return SQ_ERR_INVALID_ARG; }
    if (!(threshold == threshold)) { set_error("threshold is NaN"); return SQ_ERR_INVALID_ARG; }
    outlier_split_kernel<<<1, kSplitThreads, 0, st>>>(xmax, K, threshold, keep, idx, count);
    return check_launch("outlier_split_kernel");
}

sq_status gather_columns_impl(const void* x, sq_dtype dt, int64_t rows, int64_t K, const int32_t* idx, int64_t n,
                              int64_t ld, float* out, cudaStream_t st) {
    sq_status r;
    if ((r = check_input_dtype(dt)) != SQ_OK) return r;
    if (rows < 0 || K < 0 || n < 0 || ld < n) { set_error("need rows, K, n >= 0 and ld >= n"); return SQ_ERR_INVALID_ARG; }
    if (ld > 2147483647LL || n > K) { set_error("n must not exceed K"); return SQ_ERR_INVALID_ARG; }
    if (rows == 0 || ld == 0) return SQ_OK;
    if (!out || (n > 0 && (!x || !idx))) { set_error("NULL pointer"); return SQ_ERR_INVALID_ARG; }
    const int64_t total = rows * ld;
    const int threads = 256;
    const int64_t blocks = (total + threads - 1) / threads;
    if (blocks > 2147483647LL) { set_error("too many elements"); return SQ_ERR_UNSUPPORTED; }
    if (dt == SQ_F32)
        gather_columns_kernel<float><<<(unsigned)blocks, threads, 0, st>>>(
            static_cast<const float*>(x), rows, K, idx, (int)n, (int)ld, out);
    else
        gather_columns_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, 0, st>>>(
            static_cast<const __nv_bfloat16*>(x), rows, K, idx, (int)n, (int)ld, out);
    return check_launch("gather_columns_kernel");
}

// Per-row int8 of the bulk channels. With keep_j in {0, 1}, RN(x * keep_j) is
// x itself or a signed zero, so this is exactly the fold-and-quantize kernel
// with keep as the per-column multiplier: the outlier channels drop out of the
// row maximum and get code 0.
sq_status quant_bulk_impl(const void* x, sq_dtype dt, int64_t rows, int64_t K, const float* keep, int8_t* q,
                          float* scale, cudaStream_t st) {
    return fold_quant_weights_impl(x, dt, rows, K, keep, q, scale, st);
}

}  // namespace sq

extern "C" {

sq_status sq_outlier_split(const float* xmax, int64_t K, float threshold, float* keep, int32_t* idx,
                           int32_t* count, sq_stream_t stream) {
    return sq::outlier_split_impl(xmax, K, threshold, keep, idx, count, (cudaStream_t)stream);
}

sq_status sq_gather_columns(const void* x, sq_dtype dt, int64_t rows, int64_t K, const int32_t* idx, int64_t n,
                            int64_t ld, float* out, sq_stream_t stream) {
    return sq::gather_columns_impl(x, dt, rows, K, idx, n, ld, out, (cudaStream_t)stream);
}

sq_status sq_quant_bulk(const void* x, sq_dtype dt, int64_t rows, int64_t K, const float* keep, int8_t* q,
                        float* scale, sq_stream_t stream) {
    return sq::quant_bulk_impl(x, dt, rows, K, keep, q, scale, (cudaStream_t)stream);
}

}  // extern "C"
