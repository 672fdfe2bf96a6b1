// sq_search.cu -- per-layer search for the migration strength alpha: run the
// whole W8A8 path once per candidate alpha on a calibration batch and measure
// the relative output error ||Yq - Y||_F / ||Y||_F against the unquantized
// product Y = X W^T ("Why do activation outliers break INT8 W8A8...", "A
// strong answer": the alpha sweep and its error column; "SmoothQuant
// Explained", "Alpha: how much difficulty to move": alpha is a per-model
// tuning parameter).
//
// Y is a plain floating-point GEMM computed once by this library's kernels:
// for bf16 operands the tcgen05 GEMM with kind::f16 (exact products, fp32
// accumulation in TMEM), for fp32 operands a CUDA-core kernel (fp32 fused
// multiply-adds in k order). Each candidate then costs a2, a3, a4, the int8
// GEMM with fp32 output and one error reduction: a grid-strided pass that
// accumulates sum (Yq - Y)^2 and sum Y^2 in fp64 per block, and a one-block
// pass that adds the block sums in a fixed order (deterministic on a given
// GPU).
#include <cmath>
#include <mutex>

#include <cuda_runtime.h>

#include "sq_device.cuh"
#include "sq_internal.h"

namespace sq {

constexpr int kErrThreads = 256;
constexpr int kErrMaxBlocks = 2048;
constexpr int64_t kMaxAlphas = 64;

__global__ void __launch_bounds__(kErrThreads)
err_partial_kernel(const float* __restrict__ yq, const float* __restrict__ yr, int64_t n,
                   double* __restrict__ part) {
    double a = 0.0, b = 0.0;
    const int64_t n4 = n >> 2;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
        const float4 q = __ldcs(reinterpret_cast<const float4*>(yq) + i);
        const float4 r = __ldcs(reinterpret_cast<const float4*>(yr) + i);
        const double d0 = (double)q.x - (double)r.x, d1 = (double)q.y - (double)r.y;
        const double d2 = (double)q.z - (double)r.z, d3 = (double)q.w - (double)r.w;
        a += d0 * d0 + d1 * d1 + d2 * d2 + d3 * d3;
        b += (double)r.x * r.x + (double)r.y * r.y + (double)r.z * r.z + (double)r.w * r.w;
    }
    if (blockIdx.x == 0)
        for (int64_t i = (n4 << 2) + threadIdx.x; i < n; i += blockDim.x) {
            const double d = (double)yq[i] - (double)yr[i];
            a += d * d;
            b += (double)yr[i] * yr[i];
        }
    __shared__ double sa[kErrThreads / 32], sb[kErrThreads / 32];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        b += __shfl_xor_sync(0xffffffffu, b, o);
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) { sa[warp] = a; sb[warp] = b; }
    __syncthreads();
    if (threadIdx.x == 0) {
        double ta = 0.0, tb = 0.0;
        for (int w = 0; w < kErrThreads / 32; ++w) { ta += sa[w]; tb += sb[w]; }
        part[2 * blockIdx.x] = ta;
        part[2 * blockIdx.x + 1] = tb;
    }
}

// err = sqrt(sum a) / sqrt(sum b) over the block sums, added in a fixed order.
__global__ void __launch_bounds__(kErrThreads)
err_finalize_kernel(const double* __restrict__ part, int nblocks, double* __restrict__ err) {
    __shared__ double sa[kErrThreads], sb[kErrThreads];
    double a = 0.0, b = 0.0;
    for (int i = threadIdx.x; i < nblocks; i += kErrThreads) {
        a += part[2 * i];
        b += part[2 * i + 1];
    }
    sa[threadIdx.x] = a;
    sb[threadIdx.x] = b;
    __syncthreads();
    for (int h = kErrThreads / 2; h > 0; h >>= 1) {
        if (threadIdx.x < h) {
            sa[threadIdx.x] += sa[threadIdx.x + h];
            sb[threadIdx.x] += sb[threadIdx.x + h];
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const double num = sa[0], den = sb[0];
        *err = den > 0.0 ? sqrt(num) / sqrt(den) : (num > 0.0 ? INFINITY : 0.0);
    }
}

// The first alpha with the smallest error.
__global__ void argmin_alpha_kernel(const double* __restrict__ err, const float* __restrict__ alphas, int n,
                                    float* __restrict__ best) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int k = 0;
    for (int i = 1; i < n; ++i)
        if (err[i] < err[k]) k = i;
    *best = alphas[k];
}

namespace {

struct SearchLayout {
    size_t xmax, wmax, s, xq, xs, wq, wsc, gemm_ws, gemm_ws_bytes, yref, yq, part, err, alphas, best, total;
};

SearchLayout search_layout(int64_t T, int64_t N, int64_t K, int64_t n_alpha) {
    SearchLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += (bytes + 255) & ~size_t(255);
        return at;
    };
    L.xmax = take((size_t)K * 4);
    L.wmax = take((size_t)K * 4);
    L.s = take((size_t)K * 4);
    L.xq = take((size_t)T * K);
    L.xs = take((size_t)T * 4);
    L.wq = take((size_t)N * K);
    L.wsc = take((size_t)N * 4);
    L.gemm_ws_bytes = sq_w8a8_gemm_workspace_size(T, N, K);
    L.gemm_ws = take(L.gemm_ws_bytes);
    L.yref = take((size_t)T * N * 4);
    L.yq = take((size_t)T * N * 4);
    L.part = take((size_t)kErrMaxBlocks * 2 * sizeof(double));
    L.err = take((size_t)n_alpha * sizeof(double));
    L.alphas = take((size_t)n_alpha * sizeof(float));
    L.best = take(sizeof(float));
    L.total = off;
    return L;
}

// yref [T x N] row-major = X W^T, by this library's own kernels.
sq_status reference_gemm(const void* x, const void* w, sq_dtype dt, int64_t T, int64_t N, int64_t K, float* yref,
                         cudaStream_t st) {
    return float_gemm_xwt(x, w, dt, T, N, K, yref, st);
}

}  // namespace

size_t alpha_search_workspace_size(int64_t T, int64_t N, int64_t K, int64_t n_alpha) {
    if (T <= 0 || N <= 0 || K <= 0 || n_alpha <= 0) return 0;
    return search_layout(T, N, K, n_alpha).total;
}

sq_status alpha_search_impl(const void* x, const void* w, sq_dtype dt, int64_t T, int64_t N, int64_t K,
                            const float* alphas, int64_t n_alpha, float eps, double* err, float* best_alpha,
                            void* ws, size_t ws_bytes, cudaStream_t st) {
    if (dt != SQ_F32 && dt != SQ_BF16) { set_error("input dtype must be SQ_F32 or SQ_BF16"); return SQ_ERR_UNSUPPORTED; }
    if (T <= 0 || N <= 0 || K <= 0) { set_error("sizes must be positive"); return SQ_ERR_INVALID_ARG; }
    if (K % 16 != 0) { set_error("K must be a multiple of 16"); return SQ_ERR_UNSUPPORTED; }
    if (T > 2147483647LL || N > 2147483647LL || K > 2147483647LL) { set_error("size too large"); return SQ_ERR_UNSUPPORTED; }
    if (n_alpha <= 0 || n_alpha > kMaxAlphas) {
        set_error("between 1 and %lld alphas", (long long)kMaxAlphas);
        return SQ_ERR_INVALID_ARG;
    }
    if (!x || !w || !alphas || !err) { set_error("NULL pointer"); return SQ_ERR_INVALID_ARG; }
    for (int64_t i = 0; i < n_alpha; ++i)
        if (!(alphas[i] >= 0.0f && alphas[i] <= 1.0f)) { set_error("alpha must be in [0, 1]"); return SQ_ERR_INVALID_ARG; }
    const SearchLayout L = search_layout(T, N, K, n_alpha);
    if (!ws || ws_bytes < L.total) {
        set_error("workspace too small: %zu bytes given, %zu needed", ws_bytes, L.total);
        return SQ_ERR_INVALID_ARG;
    }
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) { set_error("workspace must be 256-byte aligned"); return SQ_ERR_UNSUPPORTED; }
    uint8_t* base = static_cast<uint8_t*>(ws);
    float* xmax = reinterpret_cast<float*>(base + L.xmax);
    float* wmax = reinterpret_cast<float*>(base + L.wmax);
    float* s = reinterpret_cast<float*>(base + L.s);
    int8_t* xq = reinterpret_cast<int8_t*>(base + L.xq);
    float* xs = reinterpret_cast<float*>(base + L.xs);
    int8_t* wq = reinterpret_cast<int8_t*>(base + L.wq);
    float* wsc = reinterpret_cast<float*>(base + L.wsc);
    float* yref = reinterpret_cast<float*>(base + L.yref);
    float* yq = reinterpret_cast<float*>(base + L.yq);
    double* part = reinterpret_cast<double*>(base + L.part);
    double* errd = reinterpret_cast<double*>(base + L.err);
    float* alphas_d = reinterpret_cast<float*>(base + L.alphas);
    float* best_d = reinterpret_cast<float*>(base + L.best);

    cudaError_t e;
    sq_status r;
    if ((e = cudaMemcpyAsync(alphas_d, alphas, (size_t)n_alpha * sizeof(float), cudaMemcpyHostToDevice, st)) != cudaSuccess)
        return cuda_fail(e, "copy alphas");
    if ((e = cudaMemsetAsync(xmax, 0, L.s - L.xmax, st)) != cudaSuccess) return cuda_fail(e, "clear maxima");
    if ((r = calibrate_absmax_pair_impl(x, T, w, N, dt, K, xmax, wmax, st)) != SQ_OK) return r;
    if ((r = reference_gemm(x, w, dt, T, N, K, yref, st)) != SQ_OK) return r;
    const int64_t nel = T * N;
    int blocks = device_info().sm_count * 4;
    if (blocks > kErrMaxBlocks) blocks = kErrMaxBlocks;
    for (int64_t a = 0; a < n_alpha; ++a) {
        if ((r = smooth_factors_impl(xmax, wmax, K, alphas[a], eps, s, st)) != SQ_OK) return r;
        if ((r = fold_smooth_quant_pair_impl(w, N, x, T, dt, K, s, wq, wsc, xq, xs, st)) != SQ_OK) return r;
        if ((r = gemm_dispatch(xq, xs, wq, wsc, T, N, K, yq, SQ_F32, base + L.gemm_ws, L.gemm_ws_bytes, st)) != SQ_OK)
            return r;
        err_partial_kernel<<<blocks, kErrThreads, 0, st>>>(yq, yref, nel, part);
        if ((r = check_launch("err_partial_kernel")) != SQ_OK) return r;
        err_finalize_kernel<<<1, kErrThreads, 0, st>>>(part, blocks, errd + a);
        if ((r = check_launch("err_finalize_kernel")) != SQ_OK) return r;
    }
    argmin_alpha_kernel<<<1, 32, 0, st>>>(errd, alphas_d, (int)n_alpha, best_d);
    if ((r = check_launch("argmin_alpha_kernel")) != SQ_OK) return r;
    if ((e = cudaMemcpyAsync(err, errd, (size_t)n_alpha * sizeof(double), cudaMemcpyDeviceToHost, st)) != cudaSuccess)
        return cuda_fail(e, "copy errors to host");
    if (best_alpha &&
        (e = cudaMemcpyAsync(best_alpha, best_d, sizeof(float), cudaMemcpyDeviceToHost, st)) != cudaSuccess)
        return cuda_fail(e, "copy best alpha to host");
    if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e, "synchronize");
    return SQ_OK;
}

}  // namespace sq

extern "C" {

size_t sq_alpha_search_workspace_size(int64_t T, int64_t N, int64_t K, int64_t n_alpha) {
    return sq::alpha_search_workspace_size(T, N, K, n_alpha);
}

sq_status sq_alpha_search(const void* x, const void* w, sq_dtype in_dt, int64_t T, int64_t N, int64_t K,
                          const float* alphas, int64_t n_alpha, float eps, double* err, float* best_alpha,
                          void* workspace, size_t ws_bytes, sq_stream_t stream) {
    return sq::alpha_search_impl(x, w, in_dt, T, N, K, alphas, n_alpha, eps, err, best_alpha, workspace, ws_bytes,
                                 (cudaStream_t)stream);
}

}  // extern "C"
