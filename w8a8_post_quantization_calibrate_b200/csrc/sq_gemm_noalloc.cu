// sq_gemm_noalloc.cu -- sq_w8a8_gemm_noalloc: the decode (M <= 16) GEMM for
// callers that cannot allocate device memory.
//
// Who needs it: a serving process that reserves nearly all of the GPU's memory
// up front (weights plus a preallocated KV cache) has no room, and often no
// permission, for transient allocations; cudaMalloc also synchronizes the
// device, which a latency-bound decode loop cannot afford; and a plug-in
// running inside a host framework may not have access to that framework's
// allocator. Such callers can pass inputs and outputs but no workspace.
//
// The weight-streaming decode kernel needs scratch for its split-K partial
// sums and completion counters. Here that scratch is a fixed array in this
// file, so the call allocates nothing. Its address is looked up once per
// device with cudaGetSymbolAddress (host code must not pass the symbol itself:
// on the host it names a host-side stand-in, not device memory).
#include <mutex>

#include <cuda_runtime.h>

#include "sq_internal.h"

namespace sq {
namespace {

// Maximum scratch: M*N int32 partial sums (at most 1 MiB, so M*N <= 262,144)
// plus 4 counters per 128-row weight tile (32 KiB would take N up to 262,144;
// since M >= 1, the M*N limit already keeps N, and so the counters, within it).
constexpr size_t kNoallocAccBytes = size_t(1) << 20;
constexpr size_t kNoallocCountBytes = size_t(32) << 10;
constexpr size_t kNoallocScratchBytes = kNoallocAccBytes + kNoallocCountBytes;

// Held by every GPU that loads this library, until the process exits. All
// calls on a device share it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

struct NoallocScratch {
    unsigned char* ptr = nullptr;
    bool ready = false;
};
NoallocScratch g_noalloc[64];
std::mutex g_noalloc_mu;

// Device address of the scratch array for the current device (set up on the
// first call per device).
sq_status noalloc_scratch(unsigned char** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 64) {
        set_error("device index %d out of range", dev);
        return SQ_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    NoallocScratch& s = g_noalloc[dev];
    if (!s.ready) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
        s.ptr = static_cast<unsigned char*>(p);
        s.ready = true;
    }
    *out = s.ptr;
    return SQ_OK;
}

}  // namespace

sq_status gemm_noalloc(const int8_t* xq, const float* x_scale, const int8_t* wq, const float* w_scale,
                       int64_t M, int64_t N, int64_t K, void* y, sq_dtype out_dt, cudaStream_t st) {
    if (M < 0 || N < 0 || K < 0) { set_error("negative size"); return SQ_ERR_INVALID_ARG; }
    if (out_dt != SQ_F32 && out_dt != SQ_BF16 && out_dt != SQ_I32) {
        set_error("output dtype must be SQ_F32, SQ_BF16 or SQ_I32");
        return SQ_ERR_UNSUPPORTED;
    }
    if (M == 0 || N == 0) return SQ_OK;
    if (M > STREAM_MAX_M) {
        set_error("sq_w8a8_gemm_noalloc: M=%lld exceeds its maximum of %d", (long long)M, STREAM_MAX_M);
        return SQ_ERR_UNSUPPORTED;
    }
    // The N test is a guard only: M >= 1 and the M*N limit already bound N.
    if (M * N > (int64_t)(kNoallocAccBytes / sizeof(int32_t)) || N > (int64_t)(kNoallocCountBytes / 16) * S_BM) {
        set_error("sq_w8a8_gemm_noalloc: M*N=%lld exceeds its scratch (M*N <= %zu)", (long long)(M * N),
                  kNoallocAccBytes / sizeof(int32_t));
        return SQ_ERR_UNSUPPORTED;
    }
    if (K == 0 || K % 16 != 0) { set_error("K=%lld must be a positive multiple of 16", (long long)K); return SQ_ERR_UNSUPPORTED; }
    if (K > 133144) { set_error("K=%lld: 127*127*K would overflow int32", (long long)K); return SQ_ERR_UNSUPPORTED; }
    if (!xq || !wq || !y) { set_error("NULL pointer"); return SQ_ERR_INVALID_ARG; }
    if (out_dt != SQ_I32 && (!x_scale || !w_scale)) { set_error("NULL scale pointer"); return SQ_ERR_INVALID_ARG; }
    if (!aligned16(xq) || !aligned16(wq) || !aligned16(y) || (w_scale && !aligned16(w_scale))) {
        set_error("xq, wq, y and w_scale must be 16-byte aligned");
        return SQ_ERR_UNSUPPORTED;
    }
    unsigned char* scratch = nullptr;
    sq_status r = noalloc_scratch(&scratch);
    if (r != SQ_OK) return r;
    const size_t used = stream_ws_bytes(M, N);
    // The kernel leaves the scratch zeroed when it completes, but a call that
    // stopped early (a bounded wait ran out) would not: clear what the kernel
    // expects to start at zero.
    cudaError_t e = cudaMemsetAsync(scratch, 0, used, st);
    if (e != cudaSuccess) return cuda_fail(e, "clear no-alloc scratch");
    CUtensorMap tw, tx;
    if ((r = make_map_i8(&tw, wq, N, K, S_BM)) != SQ_OK) return r;
    if ((r = make_map_i8(&tx, xq, M, K, S_BN)) != SQ_OK) return r;
    int32_t* acc = reinterpret_cast<int32_t*>(scratch);
    const size_t acc_al = (((size_t)M * N * 4) + 255) & ~size_t(255);
    unsigned int* counts = reinterpret_cast<unsigned int*>(scratch + acc_al);
    switch (out_dt) {
        case SQ_F32: return launch_stream<kOutF32>(tw, tx, x_scale, w_scale, y, (int)M, (int)N, (int)K, acc, counts, st);
        case SQ_BF16: return launch_stream<kOutBF16>(tw, tx, x_scale, w_scale, y, (int)M, (int)N, (int)K, acc, counts, st);
        default: return launch_stream<kOutI32>(tw, tx, x_scale, w_scale, y, (int)M, (int)N, (int)K, acc, counts, st);
    }
}

// Test hook: overwrite the whole scratch array with a non-zero byte pattern,
// as a call that stopped early would leave it.
sq_status noalloc_dirty(cudaStream_t st) {
    unsigned char* scratch = nullptr;
    sq_status r = noalloc_scratch(&scratch);
    if (r != SQ_OK) return r;
    cudaError_t e = cudaMemsetAsync(scratch, 0xA5, kNoallocScratchBytes, st);
    return e == cudaSuccess ? SQ_OK : cuda_fail(e, "dirty no-alloc scratch");
}

}  // namespace sq

extern "C" sq_status sq_selftest_dirty_noalloc_scratch(sq_stream_t stream) {
    return sq::noalloc_dirty((cudaStream_t)stream);
}

extern "C" sq_status sq_w8a8_gemm_noalloc(const int8_t* xq, const float* x_scale, const int8_t* wq,
                                          const float* w_scale, int64_t M, int64_t N, int64_t K, void* y,
                                          sq_dtype out_dt, sq_stream_t stream) {
    return sq::gemm_noalloc(xq, x_scale, wq, w_scale, M, N, K, y, out_dt, (cudaStream_t)stream);
}
