// sq_internal.h -- host-side helpers shared by the library's translation units.
#pragma once

#include <cstdint>
#include <utility>

#include <cuda_runtime.h>

#include "sq.h"

namespace sq {

// Thread-local last error message (sq_last_error_string).
void set_error(const char* fmt, ...);

// Record a CUDA runtime failure and return SQ_ERR_CUDA.
sq_status cuda_fail(cudaError_t e, const char* what);

// Check the last launch on this thread.
inline sq_status check_launch(const char* what) {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SQ_OK : cuda_fail(e, what);
}

// Device facts, cached per device.
struct DeviceInfo {
    int device = -1;
    int sm_count = 0;
    int clock_khz = 0;      // maximum SM clock
    int max_smem_optin = 0; // bytes per block
};
const DeviceInfo& device_info();

// Wait limit for bounded device waits, in SM clock cycles for the current device.
long long wait_limit_cycles();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launch with programmatic stream serialization allowed (the kernel must call
// pdl_wait() before touching global memory), optionally as clusters of
// cluster_x CTAs.
template <typename... KArgs, typename... Args>
sq_status launch_pdl(const char* what, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t st, unsigned cluster_x, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster_x > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
    if (e != cudaSuccess) return cuda_fail(e, what);
    return check_launch(what);
}

// Site codes recorded with a device-side error (sq_last_status_site).
enum Site : unsigned int {
    SITE_SELFTEST = 1,
    SITE_GEMM_PRODUCER = 10,
    SITE_GEMM_MMA_FULL = 11,
    SITE_GEMM_MMA_TMEM = 12,
    SITE_GEMM_EPILOGUE = 13,
    SITE_GEMM_DRAIN = 14,
    SITE_STREAM_PRODUCER = 20,
    SITE_STREAM_MMA_FULL = 21,
    SITE_STREAM_MMA_TMEM = 22,
    SITE_STREAM_EPILOGUE = 23,
    SITE_STREAM_DRAIN = 24,
    SITE_QUANT_WAIT = 30,
    SITE_QUANT_DRAIN = 31,
    SITE_PROBE = 40,
    SITE_DBG_RING_CODES = 50,
    SITE_DBG_RING_REPAIR = 51,
    SITE_DBG_RING_SCALE = 52,
    SITE_DBG_GEMM_VECTOR = 53,
    SITE_DBG_DECODE_OWNER = 54,
};

// Internal entry points used by sq_linear.
struct SplitTerm;
sq_status gemm_dispatch(const int8_t* xq, const float* x_scale, const int8_t* wq,
                        const float* w_scale, int64_t M, int64_t N, int64_t K, void* y,
                        sq_dtype out_dt, void* workspace, size_t ws_bytes, cudaStream_t stream,
                        const SplitTerm* split = nullptr);

}  // namespace sq
