// sq_probe.cu -- a measurement aid, not a step of the layer: the rate at which
// this GPU's tensor cores execute int8 MMAs, with nothing else in the way.
//
// The pages' only statement about speed is that integer tensor cores run at
// roughly twice the FP16 rate ("SmoothQuant Explained", "Where it fits"). A
// roofline fraction for the int8 GEMM needs the int8 rate itself, measured on
// the part at hand rather than inferred from a bf16 figure. This kernel issues
// the same instruction as the prefill GEMM -- tcgen05.mma.cta_group::2.kind::i8
// with M = 256, N = 256, K = 32, one elected thread per SM pair -- back to back
// on operand tiles that stay in shared memory, alternating between two TMEM
// accumulators, and touches no global memory. Its operations per second are
// the ceiling the GEMM's mainloop can reach at the clock it runs at.
#include <cuda_runtime.h>

#include "sq_device.cuh"
#include "sq_internal.h"

namespace sq {

constexpr int PROBE_THREADS = 64;          // warp 0 issues, warp 1 owns TMEM
constexpr uint32_t PROBE_TILE = 128 * BK;  // 16 KB: 128 rows x 128 bytes
// Enough dynamic shared memory that only one probe CTA fits on an SM (each
// allocates all 512 TMEM columns).
constexpr size_t PROBE_SMEM = 140 * 1024;
constexpr int64_t PROBE_MAX_ITERS = 10000000;

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__global__ void __launch_bounds__(PROBE_THREADS, 1)
probe_mma_i8_pair_kernel(int64_t iters, long long wait_limit, unsigned long long* __restrict__ clocks) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + PROBE_TILE;
    uint64_t* done = reinterpret_cast<uint64_t*>(smem + 2 * PROBE_TILE);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    pdl_wait();   // start only once the previous kernel in the stream has finished

    // Zero operands keep the accumulators defined; the values do not change
    // the instruction's timing.
    for (int i = threadIdx.x; i < (int)(2 * PROBE_TILE / 16); i += PROBE_THREADS)
        reinterpret_cast<uint4*>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(done), 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair<TMEM_COLS>(smem_u32(tmem_holder));
        tc_fence_before();
    }
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    const long long c0 = clock64();
    const unsigned long long t0 = global_ns();
    if (warp == 0 && lane == 0 && rank == 0) {
        const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
        for (int64_t it = 0; it < iters; ++it) {
            const uint32_t d = tmem_base + (uint32_t)((it & 1) * ACC_COLS);
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k)
                mma_i8_pair(d, make_sw128_kmajor_desc(a0 + k * UMMA_K), make_sw128_kmajor_desc(b0 + k * UMMA_K),
                            IDESC_PAIR, (it >= 2 || k > 0) ? 1u : 0u);
        }
        mma_commit_pair(smem_u32(done));   // arrives on both CTAs' barrier once every MMA is done
    }
    if (warp == 0 && lane == 0) mbar_wait(smem_u32(done), 0, wait_limit, &abort_flag, SITE_PROBE);
    if (clocks != nullptr && blockIdx.x == 0 && threadIdx.x == 0) {
        // this SM's clock over the MMAs: cycles and nanoseconds
        clocks[0] = (unsigned long long)(clock64() - c0);
        clocks[1] = global_ns() - t0;
    }
    __syncwarp();
    tc_fence_before();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair<TMEM_COLS>(tmem_base);
    }
}

sq_status probe_tensor_int8(int64_t iters, double* ops, unsigned long long* clocks, cudaStream_t st) {
    if (iters < 1 || iters > PROBE_MAX_ITERS) {
        set_error("iters=%lld must be in [1, %lld]", (long long)iters, (long long)PROBE_MAX_ITERS);
        return SQ_ERR_INVALID_ARG;
    }
    static bool attr_done[64] = {};
    const DeviceInfo& di = device_info();
    sq_status r = ensure_smem_attr(probe_mma_i8_pair_kernel, PROBE_SMEM, attr_done[di.device & 63]);
    if (r != SQ_OK) return r;
    const int pairs = di.sm_count / 2;
    // the MMAs of one launch, plus a margin, within the bounded wait
    const long long limit = wait_limit_cycles() + iters * 4 * 2000LL;
    r = launch_pdl("probe_mma_i8_pair_kernel", probe_mma_i8_pair_kernel, dim3(2 * pairs), dim3(PROBE_THREADS),
                   PROBE_SMEM, st, 2, iters, limit, clocks);
    if (r != SQ_OK) return r;
    if (ops) *ops = 2.0 * 256.0 * 256.0 * (double)UMMA_K * (BK / UMMA_K) * (double)iters * (double)pairs;
    return SQ_OK;
}

}  // namespace sq

extern "C" sq_status sq_probe_tensor_int8(int64_t iters, double* ops, unsigned long long* clocks,
                                          sq_stream_t stream) {
    return sq::probe_tensor_int8(iters, ops, clocks, (cudaStream_t)stream);
}
