// sq_api.cu -- library-wide state and the whole-layer entry point: error
// reporting, the device status word, device facts, the bounded-wait self-test
// and sq_linear (steps a1..a5 on one batch, host or device operands).
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <map>
#include <mutex>
#include <utility>

#include <cuda_runtime.h>

#include "sq_device.cuh"
#include "sq_internal.h"

namespace sq {

namespace {
thread_local char g_err[512] = "";
thread_local unsigned int g_last_site = 0u;
std::atomic<long long> g_wait_ms{2000};

DeviceInfo g_info[64];
std::mutex g_info_mu;
}  // namespace

void set_error(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
}

sq_status cuda_fail(cudaError_t e, const char* what) {
    set_error("%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
    return SQ_ERR_CUDA;
}

const DeviceInfo& device_info() {
    int dev = 0;
    cudaGetDevice(&dev);
    dev &= 63;
    DeviceInfo& d = g_info[dev];
    if (d.device != dev) {
        std::lock_guard<std::mutex> lk(g_info_mu);
        if (d.device != dev) {
            DeviceInfo n;
            cudaDeviceGetAttribute(&n.sm_count, cudaDevAttrMultiProcessorCount, dev);
            cudaDeviceGetAttribute(&n.clock_khz, cudaDevAttrClockRate, dev);
            cudaDeviceGetAttribute(&n.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
            if (n.sm_count <= 0) n.sm_count = 148;
            if (n.clock_khz <= 0) n.clock_khz = 2000000;
            n.device = dev;
            d = n;
        }
    }
    return d;
}

long long wait_limit_cycles() {
    return g_wait_ms.load() * (long long)device_info().clock_khz;
}

// A single CTA that waits, with a bounded wait, on a barrier nothing arrives at.
__global__ void selftest_wait_kernel(long long limit) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, limit, &abort_flag, SITE_SELFTEST);
}

// ------------------------------------------------------------------ sq_linear
namespace {

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

struct LinearLayout {
    size_t xmax, wmax, s, xq, xs, wq, wsc, gemm_ws, x_stage, w_stage, y_stage, total, gemm_ws_bytes;
};

LinearLayout linear_layout(int64_t M, int64_t N, int64_t K, sq_dtype in_dt, sq_dtype out_dt) {
    const size_t ies = in_dt == SQ_F32 ? 4 : 2;
    const size_t oes = out_dt == SQ_F32 ? 4 : 2;
    LinearLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off += align256(bytes); return o; };
    L.xmax = take((size_t)K * 4);
    L.wmax = take((size_t)K * 4);
    L.s = take((size_t)K * 4);
    L.xq = take((size_t)M * K);
    L.xs = take((size_t)M * 4);
    L.wq = take((size_t)N * K);
    L.wsc = take((size_t)N * 4);
    L.gemm_ws_bytes = sq_w8a8_gemm_workspace_size(M, N, K);
    L.gemm_ws = take(L.gemm_ws_bytes);
    L.x_stage = take((size_t)M * K * ies);
    L.w_stage = take((size_t)N * K * ies);
    L.y_stage = take((size_t)M * N * oes);
    L.total = off;
    return L;
}

// Host operands are staged by a copy stream of the library (one per device),
// so that the next call's input copies overlap this call's GEMM and output
// copy. Two events per workspace order the staging: inputs_ready (the copies
// are done; the compute waits for it) and inputs_free (the last kernel that
// reads the staged inputs is done; the next call's copies wait for it).
struct CopyState {
    cudaStream_t stream = nullptr;
    cudaEvent_t inputs_ready = nullptr;
    cudaEvent_t inputs_free = nullptr;
};
std::mutex g_copy_mu;
cudaStream_t g_copy_stream[64] = {};
std::map<std::pair<int, const void*>, CopyState> g_copy_state;

sq_status copy_state(const void* ws, CopyState& out) {
    const int dev = device_info().device;
    std::lock_guard<std::mutex> lk(g_copy_mu);
    cudaError_t e;
    if (!g_copy_stream[dev & 63]) {
        if ((e = cudaStreamCreateWithFlags(&g_copy_stream[dev & 63], cudaStreamNonBlocking)) != cudaSuccess)
            return cuda_fail(e, "create the copy stream");
    }
    CopyState& c = g_copy_state[{dev, ws}];
    if (!c.inputs_ready) {
        if ((e = cudaEventCreateWithFlags(&c.inputs_ready, cudaEventDisableTiming)) != cudaSuccess)
            return cuda_fail(e, "create an event");
        if ((e = cudaEventCreateWithFlags(&c.inputs_free, cudaEventDisableTiming)) != cudaSuccess)
            return cuda_fail(e, "create an event");
    }
    c.stream = g_copy_stream[dev & 63];
    out = c;
    return SQ_OK;
}

// true if the pointer is usable by kernels (device or managed memory).
bool is_device_ptr(const void* p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

}  // namespace

sq_status calibrate_absmax_impl(const void*, sq_dtype, int64_t, int64_t, float*, cudaStream_t);
sq_status smooth_factors_impl(const float*, const float*, int64_t, float, float, float*, cudaStream_t);
sq_status fold_quant_weights_impl(const void*, sq_dtype, int64_t, int64_t, const float*, int8_t*, float*,
                                  cudaStream_t);
sq_status smooth_quant_act_impl(const void*, sq_dtype, int64_t, int64_t, const float*, int8_t*, float*,
                                cudaStream_t);
sq_status fold_smooth_quant_pair_impl(const void*, int64_t, const void*, int64_t, sq_dtype, int64_t, const float*,
                                      int8_t*, float*, int8_t*, float*, cudaStream_t);
sq_status calibrate_absmax_pair_impl(const void*, int64_t, const void*, int64_t, sq_dtype, int64_t, float*, float*,
                                     cudaStream_t);

sq_status linear_impl(const void* x, const void* w, sq_dtype in_dt, int64_t M, int64_t N, int64_t K,
                      float alpha, float eps, void* y, sq_dtype out_dt, void* ws, size_t ws_bytes,
                      cudaStream_t st) {
    if (in_dt != SQ_F32 && in_dt != SQ_BF16) { set_error("input dtype must be SQ_F32 or SQ_BF16"); return SQ_ERR_UNSUPPORTED; }
    if (out_dt != SQ_F32 && out_dt != SQ_BF16) { set_error("output dtype must be SQ_F32 or SQ_BF16"); return SQ_ERR_UNSUPPORTED; }
    if (M < 0 || N < 0 || K < 0) { set_error("negative size"); return SQ_ERR_INVALID_ARG; }
    if (M == 0 || N == 0) return SQ_OK;
    if (K == 0 || K % 16 != 0) { set_error("K must be a positive multiple of 16"); return SQ_ERR_UNSUPPORTED; }
    if (!x || !w || !y) { set_error("NULL pointer"); return SQ_ERR_INVALID_ARG; }
    const LinearLayout L = linear_layout(M, N, K, in_dt, out_dt);
    if (!ws || ws_bytes < L.total) {
        set_error("workspace too small: %zu bytes given, %zu needed", ws_bytes, L.total);
        return SQ_ERR_INVALID_ARG;
    }
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) { set_error("workspace must be 256-byte aligned"); return SQ_ERR_UNSUPPORTED; }
    uint8_t* base = static_cast<uint8_t*>(ws);
    const size_t ies = in_dt == SQ_F32 ? 4 : 2;
    const size_t oes = out_dt == SQ_F32 ? 4 : 2;

    const void* xd = x;
    const void* wd = w;
    void* yd = y;
    cudaError_t e;
    const bool x_host = !is_device_ptr(x), w_host = !is_device_ptr(w);
    CopyState cs;
    if (x_host || w_host) {
        sq_status r0 = copy_state(ws, cs);
        if (r0 != SQ_OK) return r0;
        if ((e = cudaStreamWaitEvent(cs.stream, cs.inputs_free, 0)) != cudaSuccess) return cuda_fail(e, "wait for the staging");
        if (x_host) {
            xd = base + L.x_stage;
            if ((e = cudaMemcpyAsync(const_cast<void*>(xd), x, (size_t)M * K * ies, cudaMemcpyHostToDevice, cs.stream)) != cudaSuccess)
                return cuda_fail(e, "copy x to device");
        }
        if (w_host) {
            wd = base + L.w_stage;
            if ((e = cudaMemcpyAsync(const_cast<void*>(wd), w, (size_t)N * K * ies, cudaMemcpyHostToDevice, cs.stream)) != cudaSuccess)
                return cuda_fail(e, "copy w to device");
        }
        if ((e = cudaEventRecord(cs.inputs_ready, cs.stream)) != cudaSuccess) return cuda_fail(e, "record the copies");
        if ((e = cudaStreamWaitEvent(st, cs.inputs_ready, 0)) != cudaSuccess) return cuda_fail(e, "wait for the copies");
    }
    const bool y_host = !is_device_ptr(y);
    if (y_host) yd = base + L.y_stage;

    float* xmax = reinterpret_cast<float*>(base + L.xmax);
    float* wmax = reinterpret_cast<float*>(base + L.wmax);
    float* s = reinterpret_cast<float*>(base + L.s);
    int8_t* xq = reinterpret_cast<int8_t*>(base + L.xq);
    float* xs = reinterpret_cast<float*>(base + L.xs);
    int8_t* wq = reinterpret_cast<int8_t*>(base + L.wq);
    float* wsc = reinterpret_cast<float*>(base + L.wsc);

    // xmax and wmax are adjacent: one memset starts both calibrations from +0.
    if ((e = cudaMemsetAsync(xmax, 0, L.s - L.xmax, st)) != cudaSuccess) return cuda_fail(e, "clear maxima");
    sq_status r;
    if ((r = calibrate_absmax_pair_impl(xd, M, wd, N, in_dt, K, xmax, wmax, st)) != SQ_OK) return r;
    if ((r = smooth_factors_impl(xmax, wmax, K, alpha, eps, s, st)) != SQ_OK) return r;
    if ((r = fold_smooth_quant_pair_impl(wd, N, xd, M, in_dt, K, s, wq, wsc, xq, xs, st)) != SQ_OK) return r;
    if ((x_host || w_host) && (e = cudaEventRecord(cs.inputs_free, st)) != cudaSuccess)
        return cuda_fail(e, "record the end of the staged inputs' use");
    if ((r = gemm_dispatch(xq, xs, wq, wsc, M, N, K, yd, out_dt, base + L.gemm_ws, L.gemm_ws_bytes, st)) != SQ_OK)
        return r;
    if (y_host) {
        if ((e = cudaMemcpyAsync(y, yd, (size_t)M * N * oes, cudaMemcpyDeviceToHost, st)) != cudaSuccess)
            return cuda_fail(e, "copy y to host");
    }
    return SQ_OK;
}

}  // namespace sq

extern "C" {

int sq_version(void) { return 100; }

const char* sq_last_error_string(void) { return sq::g_err; }

unsigned int sq_last_status_site(void) { return sq::g_last_site; }

sq_status sq_set_wait_timeout_ms(int64_t ms) {
    if (ms <= 0) {
        sq::set_error("wait timeout must be positive");
        return SQ_ERR_INVALID_ARG;
    }
    sq::g_wait_ms.store(ms);
    return SQ_OK;
}

sq_status sq_get_status(sq_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return sq::cuda_fail(e, "cudaStreamSynchronize");
    unsigned int code = 0, site = 0, zero = 0;
    if ((e = cudaMemcpyFromSymbol(&code, sq::g_status, sizeof code)) != cudaSuccess)
        return sq::cuda_fail(e, "read device status");
    if (code != 0) {
        cudaMemcpyFromSymbol(&site, sq::g_status_site, sizeof site);
        cudaMemcpyToSymbol(sq::g_status_site, &zero, sizeof zero);
        if ((e = cudaMemcpyToSymbol(sq::g_status, &zero, sizeof zero)) != cudaSuccess)
            return sq::cuda_fail(e, "clear device status");
        sq::g_last_site = site;
        sq::set_error("a kernel recorded status %u at site %u", code, site);
        return (sq_status)code;
    }
    sq::g_last_site = 0;
    return SQ_OK;
}

sq_status sq_selftest_wait_timeout(int64_t limit_us, sq_stream_t stream) {
    if (limit_us <= 0) {
        sq::set_error("limit must be positive");
        return SQ_ERR_INVALID_ARG;
    }
    const long long cycles = limit_us * (long long)sq::device_info().clock_khz / 1000;
    sq::selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(cycles);
    return sq::check_launch("selftest_wait_kernel");
}

size_t sq_linear_workspace_size(int64_t M, int64_t N, int64_t K, sq_dtype in_dt, sq_dtype out_dt) {
    if (M < 0 || N < 0 || K < 0) return 0;
    return sq::linear_layout(M, N, K, in_dt, out_dt).total;
}

sq_status sq_linear_workspace_offsets(int64_t M, int64_t N, int64_t K, sq_dtype in_dt, sq_dtype out_dt,
                                      size_t* offsets) {
    if (M < 0 || N < 0 || K < 0 || !offsets) {
        sq::set_error("negative size or NULL offsets");
        return SQ_ERR_INVALID_ARG;
    }
    if ((in_dt != SQ_F32 && in_dt != SQ_BF16) || (out_dt != SQ_F32 && out_dt != SQ_BF16)) {
        sq::set_error("input and output dtypes must be SQ_F32 or SQ_BF16");
        return SQ_ERR_UNSUPPORTED;
    }
    const sq::LinearLayout L = sq::linear_layout(M, N, K, in_dt, out_dt);
    offsets[0] = L.xmax;
    offsets[1] = L.wmax;
    offsets[2] = L.s;
    offsets[3] = L.xq;
    offsets[4] = L.xs;
    offsets[5] = L.wq;
    offsets[6] = L.wsc;
    return SQ_OK;
}

sq_status sq_linear(const void* x, const void* w, sq_dtype in_dt, int64_t M, int64_t N, int64_t K,
                    float alpha, float eps, void* y, sq_dtype out_dt, void* workspace, size_t ws_bytes,
                    sq_stream_t stream) {
    return sq::linear_impl(x, w, in_dt, M, N, K, alpha, eps, y, out_dt, workspace, ws_bytes,
                           (cudaStream_t)stream);
}

}  // extern "C"
