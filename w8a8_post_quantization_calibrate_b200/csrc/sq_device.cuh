// sq_device.cuh -- device-side building blocks shared by the sm_100a kernels:
// bf16 handling, the device status word, bounded mbarrier waits, TMA tile
// loads and the tcgen05 (5th-generation tensor core / tensor memory) wrappers.
//
// Every spin-wait here is bounded: it gives up after a clock64() budget,
// records SQ_ERR_TIMEOUT (and the site) in the device status word, raises the
// CTA's abort flag so the other warp roles stop too, and returns false. No
// wait can hang the GPU.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "sq_internal.h"

namespace sq {

// ---------------------------------------------------------------- status word
// g_status holds the first error any kernel recorded (0 = none); g_status_site
// says where. Read and cleared by sq_get_status(). The library is a single
// translation unit, so this header (and these definitions) appear once.
__device__ unsigned int g_status = 0u;
__device__ unsigned int g_status_site = 0u;

__device__ __forceinline__ void record_status(unsigned int code, unsigned int site) {
    if (atomicCAS(&g_status, 0u, code) == 0u) atomicExch(&g_status_site, site);
}

// ---------------------------------------------------------------- debug index checks
// A build with -DSQ_DEBUG checks, before the global stores whose indices the
// kernels do not otherwise guard (rows that fill every lane, rare-path
// repairs, vector stores, cluster ranks), that the access is inside its
// buffer; a failed check records SQ_ERR_BOUNDS with the store's site in the
// status word (sq_get_status reports it) and the store is skipped. Nothing
// traps. Without SQ_DEBUG every check is the constant true.
#ifdef SQ_DEBUG
__device__ __forceinline__ bool dchk(bool ok, unsigned int site) {
    if (!ok) record_status(SQ_ERR_BOUNDS, site);
    return ok;
}
#else
__device__ __forceinline__ bool dchk(bool, unsigned int) { return true; }
#endif

// ---------------------------------------------------------------- bf16 / misc
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}"
                 :: "r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
                 :: "r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}

// Wait for the phase of `bar` with the given parity to complete. Gives up
// after `limit` SM clock cycles, or as soon as another role raised *abort.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, long long limit,
                                          volatile int* abort, unsigned int site) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (clock64() - t0 > limit) {
            *abort = 1;
            record_status(SQ_ERR_TIMEOUT, site);
            return false;
        }
    }
}

// The same bounded wait for threads with nothing else to do: each try_wait
// may suspend the thread (up to 0.2 ms) until the phase completes, instead of
// returning at once, so that waiting warps do not take issue slots from the
// warps that compute.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity), "r"(200000u) : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_sleep(uint32_t bar, uint32_t parity, long long limit,
                                                volatile int* abort, unsigned int site) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity)) return true;
        if (*abort) return false;
        if (clock64() - t0 > limit) {
            *abort = 1;
            record_status(SQ_ERR_TIMEOUT, site);
            return false;
        }
    }
}

// ---------------------------------------------------------------- thread-block clusters
// Rank of this CTA in its cluster, the cluster's size, a barrier of all the
// cluster's threads, and the cluster-scope pieces of an exchange between CTAs:
// the shared::cluster address of an offset in another CTA, an integer atomic
// add there, a remote arrive that releases this thread's earlier writes, and a
// bounded wait that acquires them.
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t mapa_rank(uint32_t local_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void red_add_cluster(uint32_t cluster_addr, int32_t v) {
    asm volatile("red.relaxed.cluster.shared::cluster.add.s32 [%0], %1;" :: "r"(cluster_addr), "r"(v) : "memory");
}
__device__ __forceinline__ void arrive_remote_release(uint32_t cluster_bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" :: "r"(cluster_bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_acq_cluster(uint32_t bar, uint32_t parity, long long limit,
                                                      volatile int* abort, unsigned int site) {
    if (mbar_try_wait_acq_cluster(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait_acq_cluster(bar, parity)) return true;
        if (*abort) return false;
        if (clock64() - t0 > limit) {
            *abort = 1;
            record_status(SQ_ERR_TIMEOUT, site);
            return false;
        }
    }
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

// ---------------------------------------------------------------- programmatic dependent launch
// The library's kernels are launched with programmatic stream serialization:
// a kernel may be scheduled while the previous kernel in the stream is still
// finishing. Every kernel calls pdl_wait() before its first access to global
// memory (it returns once the previous grid has completed and its writes are
// visible; immediately if there is no such grid), then pdl_trigger() so that
// the next kernel can be scheduled in turn. Only shared-memory and TMEM set-up
// may come before pdl_wait().
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- TMA
// 2-D tiled bulk tensor load global -> shared, completion signalled on `bar`
// (complete_tx). No multicast. x is the innermost (contiguous) coordinate.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, uint32_t bar,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];"
        :: "r"(dst), "l"(tmap), "r"(bar), "r"(x), "r"(y) : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" :: "l"(tmap) : "memory");
}

// ---------------------------------------------------------------- tcgen05
template <int NCOLS>
__device__ __forceinline__ void tmem_alloc(uint32_t holder_smem) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(holder_smem), "n"(NCOLS) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

template <int NCOLS>
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                 :: "r"(taddr), "n"(NCOLS) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, int8 x int8 -> int32, one CTA.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// The same for FP8: kind::f8f6f4 with E4M3 A and B (both operands one type), fp32 D.
__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// The same for bf16: kind::f16 with bf16 A and B, fp32 D.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// Arrive once on `bar` when every tcgen05 op this thread issued so far is done.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(bar) : "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile stored by TMA with
// 128-byte swizzle: rows of 128 bytes, 8-row atoms 1024 bytes apart (stride
// byte offset), leading byte offset unused (encoded 1), descriptor version 1,
// layout type 2 (128B swizzle). The tile base must be 1024-byte aligned;
// advancing along K inside the atom moves the start address by 32 bytes.
__device__ __forceinline__ uint64_t make_sw128_kmajor_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);        // start address   [0,14)
    d |= (uint64_t)1 << 16;                               // LBO (unused)    [16,30)
    d |= (uint64_t)(1024u >> 4) << 32;                    // SBO = 1024 B    [32,46)
    d |= (uint64_t)1 << 46;                               // version         [46,48)
    d |= (uint64_t)2 << 61;                               // 128B swizzle    [61,64)
    return d;
}

// Instruction descriptor, kind::i8: signed int8 A and B, int32 D, both
// operands K-major, shape M x N.
__host__ __device__ constexpr uint32_t make_idesc_i8(int M, int N) {
    return (2u << 4)                          // D format: s32
         | (1u << 7)                          // A format: signed 8-bit
         | (1u << 10)                         // B format: signed 8-bit
         | ((uint32_t)(N >> 3) << 17)         // N / 8
         | ((uint32_t)(M >> 4) << 24);        // M / 16
}

// Instruction descriptor, kind::f8f6f4: E4M3 A and B (format code 0), fp32 D
// (format code 1), both operands K-major, shape M x N.
__host__ __device__ constexpr uint32_t make_idesc_e4m3(int M, int N) {
    return (1u << 4)                          // D format: f32
         | (0u << 7)                          // A format: E4M3
         | (0u << 10)                         // B format: E4M3
         | ((uint32_t)(N >> 3) << 17)         // N / 8
         | ((uint32_t)(M >> 4) << 24);        // M / 16
}

// Instruction descriptor, kind::f16 with bf16 A and B (format code 1) and fp32
// D (format code 1), both operands K-major, shape M x N.
__host__ __device__ constexpr uint32_t make_idesc_bf16(int M, int N) {
    return (1u << 4)                          // D format: f32
         | (1u << 7)                          // A format: bf16
         | (1u << 10)                         // B format: bf16
         | ((uint32_t)(N >> 3) << 17)         // N / 8
         | ((uint32_t)(M >> 4) << 24);        // M / 16
}

// 32 lanes x 32 columns of 32-bit TMEM -> 32 registers per thread (thread i
// of the warp reads lane base+i).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32"
        " {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
          "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
          "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]),
          "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32"
        " {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
          "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
          "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- epilogue math
// y = (float(acc) * sa) * sw, each step one round-to-nearest fp32 operation
// (explicit intrinsics: never contracted into an FMA).
__device__ __forceinline__ float dequant(int32_t acc, float sa, float sw) {
    return __fmul_rn(__fmul_rn(__int2float_rn(acc), sa), sw);
}
// The epilogue value of a raw 32-bit accumulator: int32 (int8 operands) or fp32 (FP8).
template <bool F8>
__device__ __forceinline__ float dequant_raw(uint32_t acc, float sa, float sw) {
    if (F8) return __fmul_rn(__fmul_rn(__uint_as_float(acc), sa), sw);
    return dequant((int32_t)acc, sa, sw);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace sq
