// sq_gemm.cu -- step a5: int8 x int8 -> int32 GEMM with the dequantizing
// epilogue, on the sm_100a tensor cores (tcgen05.mma kind::i8, TMEM int32
// accumulators, TMA-fed 128B-swizzled shared-memory tiles).
//
//   acc[t, n] = sum_k xq[t, k] * wq[n, k]
//   y[t, n]   = (float(acc[t, n]) * x_scale[t]) * w_scale[n]
//
// Per-token and per-output-channel scales are constant along K, so they leave
// the integer sum untouched and are applied once, after it ("One outlier"
// notes, "Which scales factor out, and why"; "Activation Outlier Channels and
// Mixed-Precision Decomposition", "Decomposition": integer matmul, float
// epilogue).
//
// Two kernels:
//  * gemm_tiled_kernel (prefill, M > 16): persistent CTAs, one per SM, over
//    128 x 256 output tiles. Warp 0 streams A/B k-blocks with TMA into a
//    4-stage ring; one thread of warp 1 issues tcgen05.mma (M=128, N=256,
//    K=32) into one of two TMEM accumulators; warps 2-5 drain the other
//    accumulator (tcgen05.ld), apply the scales and store Y, overlapping the
//    next tile's main loop.
//  * gemm_stream_kernel (decode, M <= 16): the product is computed transposed,
//    Y^T = Wq Xq^T, so the weight rows fill the 128-row MMA side and the few
//    tokens are the N=16 side. The weight matrix is streamed once from HBM,
//    split over all SMs along (row tile, k-block) work units; partial int32
//    sums of a row tile meet in a global workspace (exact integer atomics) and
//    the CTA that completes a tile applies the epilogue and re-zeroes it.
#include <cstdio>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "sq_device.cuh"
#include "sq_internal.h"

namespace sq {

// ------------------------------------------------------------------ shapes
constexpr int BM = 128;          // output rows per tile (tokens)
constexpr int BN = 256;          // output columns per tile (output channels)
constexpr int BK = 128;          // k-block: 128 int8 = one 128-byte swizzle row
constexpr int UMMA_K = 32;       // K of one kind::i8 MMA
constexpr int STAGES = 4;
constexpr uint32_t A_STAGE = BM * BK;           // 16 KB
constexpr uint32_t B_STAGE = BN * BK;           // 32 KB
constexpr int ACC_COLS = BN;                    // int32 columns per accumulator
constexpr int TMEM_COLS = 2 * ACC_COLS;         // double-buffered: 512 columns
constexpr int GEMM_THREADS = 192;               // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr uint32_t IDESC_TILED = make_idesc_i8(BM, BN);
constexpr uint32_t IDESC_TILED_E4M3 = make_idesc_e4m3(BM, BN);
constexpr uint32_t IDESC_TILED_BF16 = make_idesc_bf16(BM, BN);

// Operand kinds of the 1-CTA kernel: int8 codes (the layer's GEMM), FP8 E4M3
// codes, or bf16 values (the plain floating-point product of the alpha
// search, fp32 accumulation, raw fp32 output).
enum OperandKind { kAkI8 = 0, kAkE4M3 = 1, kAkBF16 = 2 };
// Elements of one 128-byte k-block row.
__host__ __device__ constexpr int bk_elems(int ak) { return ak == kAkBF16 ? 64 : 128; }

constexpr int S_BM = 128;        // weight rows per tile (MMA M)
constexpr int S_BN = 16;         // tokens (MMA N)
constexpr int S_STAGES = 8;
constexpr uint32_t S_A_STAGE = S_BM * BK;       // 16 KB
constexpr uint32_t S_B_STAGE = S_BN * BK;       // 2 KB
constexpr int S_TMEM_COLS = 32;                 // 2 x 16 columns
constexpr uint32_t IDESC_STREAM = make_idesc_i8(S_BM, S_BN);
constexpr int STREAM_MAX_M = 16;

enum OutKind { kOutF32 = 0, kOutBF16 = 1, kOutI32 = 2 };
constexpr int kMaxSplitLd = 32;  // outlier channels the decomposed epilogue takes
constexpr size_t kSplitSmem = (size_t)BN * kMaxSplitLd * sizeof(float);   // w_out^T of one tile: 32 KB

constexpr size_t tiled_smem_bytes() {
    return 1024 /*alignment slack*/ + STAGES * (A_STAGE + B_STAGE) + 256 /*barriers etc*/;
}
constexpr size_t stream_smem_bytes() {
    return 1024 + S_STAGES * (S_A_STAGE + S_B_STAGE) + 256;
}

// One MMA of the 1-CTA kernel (32 bytes of K): int8, FP8 E4M3 or bf16 operands.
template <int AK>
__device__ __forceinline__ void mma_tiled(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    if (AK == kAkE4M3) mma_f8(d_tmem, adesc, bdesc, IDESC_TILED_E4M3, accumulate);
    else if (AK == kAkBF16) mma_bf16(d_tmem, adesc, bdesc, IDESC_TILED_BF16, accumulate);
    else mma_i8(d_tmem, adesc, bdesc, IDESC_TILED, accumulate);
}

// Tile order: groups of 16 row tiles, column tiles outermost inside a group, so
// the CTAs in flight at one time share few A and B panels (L2 reuse).
__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int& mb, int& nb) {
    constexpr int GROUP = 16;
    const int group = tile / (GROUP * num_n);
    const int first_m = group * GROUP;
    const int gm = min(num_m - first_m, GROUP);
    const int idx = tile - group * GROUP * num_n;
    mb = first_m + idx % gm;
    nb = idx / gm;
}

// The floating-point term of the mixed-precision decomposition ("Activation
// Outlier Channels and Mixed-Precision Decomposition", "Decomposition"; "One
// outlier" notes, "Route it, or move it"): the few outlier input channels,
// gathered into x_out [M x ld] and w_out [N x ld] (fp32, zero-padded to ld, a
// multiple of 4), are added to the dequantized int8 term in the epilogue as a
// chain of fp32 fused multiply-adds in channel order:
//   y = fma(x_out[ld-1], w_out[ld-1], ... fma(x_out[0], w_out[0], y_bulk)).
struct SplitTerm {
    const float* x_out = nullptr;
    const float* w_out = nullptr;
    int ld = 0;
};

// The prefill kernels stage w_out of the tile's BN columns in shared memory,
// transposed to [ld][BN], before each tile's epilogue (the four epilogue
// warps together); every lane then reads the same float4 of four columns at
// once (a broadcast). Two mbarriers with bounded waits order the staging:
// SFULL (all four warps have written the tile) and SEMPTY (all four have
// finished reading the previous one), so a warp that leaves early on an error
// cannot strand the others.

// Called by the four epilogue warps (threads 64..191) for their it-th tile.
// Returns false if a wait gave up (the caller leaves its tile loop).
__device__ __forceinline__ bool stage_split(float* w_s, const SplitTerm& sp, int nb, int N, uint32_t it,
                                            uint32_t sfull, uint32_t sempty, long long limit,
                                            volatile int* abort_flag) {
    if (it > 0 && !mbar_wait(sempty, (it - 1) & 1, limit, abort_flag, SITE_GEMM_EPILOGUE)) return false;
    const int n0 = nb * BN;
    for (int i = (int)threadIdx.x - 64; i < BN * sp.ld; i += 128) {
        const int o = i / BN, c = i - o * BN;
        const int col = n0 + c;
        w_s[o * BN + c] = col < N ? __ldg(sp.w_out + (int64_t)col * sp.ld + o) : 0.0f;
    }
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(sfull);
    return mbar_wait(sfull, it & 1, limit, abort_flag, SITE_GEMM_EPILOGUE);
}

// v[i] += sum_o x_out[row, o] * w_out[col0 + i, o] for 32 columns of a row;
// xr = x_out + row * ld, ws_col = the staged w_out^T at column col0.
__device__ __forceinline__ void add_split32(float (&v)[32], const float* __restrict__ xr, const float* ws_col,
                                            int ld) {
#pragma unroll 1
    for (int o4 = 0; o4 < ld; o4 += 4) {
        const float4 xo = __ldg(reinterpret_cast<const float4*>(xr + o4));
        const float xv[4] = {xo.x, xo.y, xo.z, xo.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float* wrow = ws_col + (o4 + k) * BN;
#pragma unroll
            for (int i4 = 0; i4 < 8; ++i4) {
                const float4 w4 = *reinterpret_cast<const float4*>(wrow + 4 * i4);
                v[4 * i4] = fmaf(xv[k], w4.x, v[4 * i4]);
                v[4 * i4 + 1] = fmaf(xv[k], w4.y, v[4 * i4 + 1]);
                v[4 * i4 + 2] = fmaf(xv[k], w4.z, v[4 * i4 + 2]);
                v[4 * i4 + 3] = fmaf(xv[k], w4.w, v[4 * i4 + 3]);
            }
        }
    }
}

// The same sum for one output element (token t, output channel n).
__device__ __forceinline__ float add_split1(float v, int64_t t, int64_t n, const SplitTerm& sp) {
    const float* xr = sp.x_out + t * (int64_t)sp.ld;
    const float* wr = sp.w_out + n * (int64_t)sp.ld;
#pragma unroll 1
    for (int o = 0; o < sp.ld; o += 4) {
        const float4 xo = __ldg(reinterpret_cast<const float4*>(xr + o));
        const float4 wo = __ldg(reinterpret_cast<const float4*>(wr + o));
        v = fmaf(xo.x, wo.x, v);
        v = fmaf(xo.y, wo.y, v);
        v = fmaf(xo.z, wo.z, v);
        v = fmaf(xo.w, wo.w, v);
    }
    return v;
}

// Stores 32 consecutive outputs of one row (row-major y, row stride N). For
// bf16 operands (AK == kAkBF16) the outputs are the raw fp32 accumulators.
// SW_SMEM: w_scale points into a shared-memory copy (read with plain loads).
template <int OUT, bool SPLIT, int AK = kAkI8, bool SW_SMEM = false>
__device__ __forceinline__ void store_row32(void* y, int64_t row, int col0, int N, const uint32_t (&r)[32],
                                            float sa, const float* __restrict__ w_scale, const float* xr,
                                            const float* ws_col, int ld) {
    const int64_t base = row * (int64_t)N + col0;
    const bool full = (col0 + 32 <= N);
    if (OUT == kOutI32) {
        int32_t* yp = static_cast<int32_t*>(y) + base;
        if (full && (N & 3) == 0) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<int4*>(yp + i) = make_int4((int)r[i], (int)r[i + 1], (int)r[i + 2], (int)r[i + 3]);
        } else {
            for (int i = 0; i < 32; ++i)
                if (col0 + i < N) yp[i] = (int32_t)r[i];
        }
        return;
    }
    constexpr bool F8 = AK == kAkE4M3;
    float v[32];
    if (AK == kAkBF16) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
    } else if (full) {
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
            const float4 sw = SW_SMEM ? *reinterpret_cast<const float4*>(w_scale + col0 + i)
                                      : __ldg(reinterpret_cast<const float4*>(w_scale + col0 + i));
            v[i] = dequant_raw<F8>(r[i], sa, sw.x);
            v[i + 1] = dequant_raw<F8>(r[i + 1], sa, sw.y);
            v[i + 2] = dequant_raw<F8>(r[i + 2], sa, sw.z);
            v[i + 3] = dequant_raw<F8>(r[i + 3], sa, sw.w);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            v[i] = (col0 + i < N) ? dequant_raw<F8>(r[i], sa, SW_SMEM ? w_scale[col0 + i] : __ldg(w_scale + col0 + i))
                                  : 0.0f;
    }
    if (SPLIT) add_split32(v, xr, ws_col, ld);
    if (OUT == kOutF32) {
        float* yp = static_cast<float*>(y) + base;
        if (full && (N & 3) == 0) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                if (dchk((reinterpret_cast<uintptr_t>(yp + i) & 15u) == 0, SITE_DBG_GEMM_VECTOR))
                    *reinterpret_cast<float4*>(yp + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        } else {
            for (int i = 0; i < 32; ++i)
                if (col0 + i < N) yp[i] = v[i];
        }
    } else {
        __nv_bfloat16* yp = static_cast<__nv_bfloat16*>(y) + base;
        if (full && (N & 7) == 0) {
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
                uint4 pk;
                pk.x = pack_bf16x2(v[i], v[i + 1]);
                pk.y = pack_bf16x2(v[i + 2], v[i + 3]);
                pk.z = pack_bf16x2(v[i + 4], v[i + 5]);
                pk.w = pack_bf16x2(v[i + 6], v[i + 7]);
                if (dchk((reinterpret_cast<uintptr_t>(yp + i) & 15u) == 0, SITE_DBG_GEMM_VECTOR))
                    *reinterpret_cast<uint4*>(yp + i) = pk;
            }
        } else {
            for (int i = 0; i < 32; ++i)
                if (col0 + i < N) yp[i] = __float2bfloat16_rn(v[i]);
        }
    }
}

// ================================================================== prefill
template <int OUT, bool SPLIT, int AK = kAkI8>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
gemm_tiled_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const float* __restrict__ x_scale, const float* __restrict__ w_scale,
                  void* __restrict__ y, int M, int N, int K, const SplitTerm sp, long long wait_limit) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * A_STAGE;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * B_STAGE);
    // bars: full[STAGES] | empty[STAGES] | tfull[2] | tempty[2] | drain
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    __shared__ int no_abort;  // always 0: drain waits must not be cut short by the abort flag

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_m = (M + BM - 1) / BM, num_n = (N + BN - 1) / BN;
    const int num_tiles = num_m * num_n;
    constexpr int BKE = bk_elems(AK);   // elements per k-block
    const int num_kb = (K + BKE - 1) / BKE;

    auto bar = [&](int i) { return smem_u32(bars + i); };
    const int FULL = 0, EMPTY = STAGES, TFULL = 2 * STAGES, TEMPTY = 2 * STAGES + 2, DRAIN = 2 * STAGES + 4;
    // entry 2 * STAGES + 5 holds the TMEM address and the abort flag
    const int SFULL = 2 * STAGES + 6, SEMPTY = 2 * STAGES + 7;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar(FULL + s), 1);
            mbar_init(bar(EMPTY + s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(bar(TFULL + a), 1);
            mbar_init(bar(TEMPTY + a), 4);
        }
        mbar_init(bar(DRAIN), 1);
        if (SPLIT) {
            mbar_init(bar(SFULL), 4);
            mbar_init(bar(SEMPTY), 4);
        }
        *abort_flag = 0;
        no_abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc<TMEM_COLS>(smem_u32(tmem_holder));
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        // ---------------------------------------------------- TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                int mb, nb;
                tile_coords(tile, num_m, num_n, mb, nb);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(bar(EMPTY + stage), phase ^ 1, wait_limit, abort_flag, SITE_GEMM_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(bar(FULL + stage), A_STAGE + B_STAGE);
                    tma_load_2d(smem_u32(sA + stage * A_STAGE), &tmA, bar(FULL + stage), kb * BKE, mb * BM);
                    tma_load_2d(smem_u32(sB + stage * B_STAGE), &tmB, bar(FULL + stage), kb * BKE, nb * BN);
                    ++issued;
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok || *abort_flag) {
                // Every bulk copy this CTA started must land before the CTA exits.
                for (int s = 0; s < STAGES; ++s) {
                    const long long cnt = issued / STAGES + (s < issued % STAGES ? 1 : 0);
                    if (cnt > 0)
                        mbar_wait(bar(FULL + s), (uint32_t)((cnt - 1) & 1), wait_limit, &no_abort, SITE_GEMM_DRAIN);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                if (!mbar_wait(bar(TEMPTY + acc), acc_phase ^ 1, wait_limit, abort_flag, SITE_GEMM_MMA_TMEM)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * ACC_COLS);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(bar(FULL + stage), phase, wait_limit, abort_flag, SITE_GEMM_MMA_FULL)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + stage * A_STAGE);
                    const uint32_t b0 = smem_u32(sB + stage * B_STAGE);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k)
                        mma_tiled<AK>(d_tmem, make_sw128_kmajor_desc(a0 + k * UMMA_K),
                               make_sw128_kmajor_desc(b0 + k * UMMA_K),
                               (kb | k) != 0 ? 1u : 0u);
                    mma_commit(bar(EMPTY + stage));
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit(bar(TFULL + acc));
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
            // All issued MMAs must finish before TMEM is released.
            mma_commit(bar(DRAIN));
            mbar_wait(bar(DRAIN), 0, wait_limit, &no_abort, SITE_GEMM_DRAIN);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------- epilogue (warps 2..5)
        const int quarter = warp & 3;  // TMEM lanes this warp may read: 32*quarter ..
        int acc = 0;
        uint32_t acc_phase = 0;
        float* w_s = reinterpret_cast<float*>(smem + STAGES * (A_STAGE + B_STAGE) + 256);
        uint32_t it = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
            int mb, nb;
            tile_coords(tile, num_m, num_n, mb, nb);
            if (SPLIT && !stage_split(w_s, sp, nb, N, it, bar(SFULL), bar(SEMPTY), wait_limit, abort_flag)) break;
            if (!mbar_wait(bar(TFULL + acc), acc_phase, wait_limit, abort_flag, SITE_GEMM_EPILOGUE)) break;
            tc_fence_after();
            const int64_t row = (int64_t)mb * BM + quarter * 32 + lane;
            const bool row_ok = row < M;
            const float sa = (OUT != kOutI32 && AK != kAkBF16 && row_ok) ? __ldg(x_scale + row) : 0.0f;
            const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * ACC_COLS);
#pragma unroll 1
            for (int c = 0; c < BN / 32; c += 2) {
                uint32_t r0[32], r1[32];
                tmem_ld_32x32b_x32(taddr + c * 32, r0);
                tmem_ld_32x32b_x32(taddr + (c + 1) * 32, r1);
                tmem_wait_ld();
                const int col0 = nb * BN + c * 32;
                const float* xr = SPLIT && row_ok ? sp.x_out + row * sp.ld : nullptr;
                if (row_ok && col0 < N)
                    store_row32<OUT, SPLIT, AK>(y, row, col0, N, r0, sa, w_scale, xr, w_s + c * 32, sp.ld);
                if (row_ok && col0 + 32 < N)
                    store_row32<OUT, SPLIT, AK>(y, row, col0 + 32, N, r1, sa, w_scale, xr, w_s + (c + 1) * 32, sp.ld);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bar(TEMPTY + acc));
                if (SPLIT) mbar_arrive(bar(SEMPTY));   // this warp has read the staged tile
            }
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc<TMEM_COLS>(tmem_base);
    }
}

// ================================================================== prefill, paired SMs
// A cluster of two CTAs on a pair of SMs computes 256 x 256 output tiles with
// tcgen05.mma.cta_group::2 (M=256, N=256, K=32), issued by CTA 0. Each CTA
// loads only its own halves -- 128 rows of A (its rows of the tile) and 128
// rows of B (half of the tile's columns) -- into a 6-stage ring; the MMA reads
// the B half of the other CTA directly. Both CTAs' loads signal CTA 0's "full"
// barrier (one arrival, 64 KB of transactions); CTA 0's commits arrive on the
// "empty" and "accumulator full" barriers of both CTAs (commit multicast, a
// barrier arrival -- no data multicast). Each CTA's TMEM holds its 128 rows x
// 256 columns of the accumulator (double-buffered); its epilogue warps drain
// it and arrive on CTA 0's "accumulator empty" barrier.
//
// Wide tiles (NT = 512 columns, for long K): each CTA loads two 128-row boxes
// of B per stage (its halves of the tile's two 256-column blocks), CTA 0 issues
// two N = 256 MMAs per k-step into TMEM columns 0..255 and 256..511, and the
// single accumulator fills all 512 columns, so the epilogue of a tile is not
// overlapped with the next tile's MMAs. Per k-step a pair moves 96 KB for
// 256 x 512 outputs instead of 64 KB for 256 x 256: a quarter less operand
// traffic per product through L2 and shared memory, and half as many tiles
// re-reading the same panels from DRAM.
constexpr uint32_t P_A_STAGE = 128 * BK;        // 16 KB: this CTA's 128 rows of A
constexpr uint32_t IDESC_PAIR = make_idesc_i8(256, 256);
__host__ __device__ constexpr int pair_stages(int nt) { return nt == 512 ? 4 : 6; }
__host__ __device__ constexpr uint32_t pair_b_stage(int nt) { return (uint32_t)(nt / 2) * BK; }   // this CTA's rows of B
__host__ __device__ constexpr int pair_accs(int nt) { return nt == 512 ? 1 : 2; }   // TMEM accumulators of nt columns

constexpr size_t pair_smem_bytes(int nt) {
    return 1024 + (size_t)pair_stages(nt) * (P_A_STAGE + pair_b_stage(nt)) + 256;
}
// Beyond the ring: the outlier term's staging (SPLIT), or else one copy per
// epilogue warp of the tile's output-channel scales and two 2 KB buffers per
// epilogue warp for bf16 output blocks (32 rows x 32 columns) on their way to
// global memory by bulk tensor stores.
constexpr uint32_t kOutBlockBytes = 32 * 32 * 2;
constexpr size_t pair_epilogue_smem_bytes(int nt, bool split) {
    return split ? kSplitSmem : 4 * (size_t)nt * sizeof(float) + 4 * 2 * (size_t)kOutBlockBytes;
}

__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void* tmap, uint32_t bar_cta0, int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];"
        :: "r"(dst), "l"(tmap), "r"(bar_cta0), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void mma_i8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}
__device__ __forceinline__ void mma_f8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}
constexpr uint32_t IDESC_PAIR_E4M3 = make_idesc_e4m3(256, 256);
// One MMA of the pair: int8 or FP8 E4M3 operands.
template <bool F8>
__device__ __forceinline__ void mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    if (F8) mma_f8_pair(d_tmem, adesc, bdesc, IDESC_PAIR_E4M3, accumulate);
    else mma_i8_pair(d_tmem, adesc, bdesc, IDESC_PAIR, accumulate);
}

// Arrive once on `bar` in both CTAs of the pair when the MMAs issued so far are done.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 :: "r"(bar), "h"((uint16_t)3) : "memory");
}
// shared::cluster address of the same shared-memory offset in CTA 0 of the cluster.
__device__ __forceinline__ uint32_t cta0_addr(uint32_t local_addr) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(r) : "r"(local_addr));
    return r;
}
// Arrive once on `bar` of CTA 0 only when the MMAs issued so far are done.
__device__ __forceinline__ void mma_commit_cta0(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 :: "r"(bar), "h"((uint16_t)1) : "memory");
}
__device__ __forceinline__ void arrive_on_cta0(uint32_t local_bar) {
    asm volatile("{\n\t.reg .b32 ra;\n\t"
                 "mapa.shared::cluster.u32 ra, %0, 0;\n\t"
                 "mbarrier.arrive.release.cluster.shared::cluster.b64 _, [ra];\n\t}"
                 :: "r"(local_bar) : "memory");
}
// Bulk tensor stores from shared memory (no multicast): issue, group, and wait
// until a group no longer reads its source (or has completed).
__device__ __forceinline__ void tma_store_2d(const void* tmap, uint32_t src, int32_t x, int32_t y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
                 :: "l"(tmap), "r"(src), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_le1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

template <int NCOLS>
__device__ __forceinline__ void tmem_alloc_pair(uint32_t holder_smem) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(holder_smem), "n"(NCOLS) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
template <int NCOLS>
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" :: "r"(taddr), "n"(NCOLS) : "memory");
}

template <int OUT, bool SPLIT, bool F8 = false, int NT = 256>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const float* __restrict__ x_scale, const float* __restrict__ w_scale,
                 void* __restrict__ y, int M, int N, int K, const SplitTerm sp, long long wait_limit,
                 const __grid_constant__ CUtensorMap tmY, int tstore) {
    static_assert(NT == 256 || NT == 512, "256- or 512-column tiles");
    static_assert(NT == 256 || !SPLIT, "the outlier term's staging is sized for 256 columns");
    constexpr int P_STAGES = pair_stages(NT);
    constexpr uint32_t P_B_STAGE = pair_b_stage(NT);
    constexpr uint32_t P_TX_BYTES = 2 * (P_A_STAGE + P_B_STAGE);   // both CTAs, per stage
    constexpr int ACCS = pair_accs(NT);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + P_STAGES * P_A_STAGE;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sB + P_STAGES * P_B_STAGE);
    // bars: full[P_STAGES] | empty[P_STAGES] | tfull[2] | tempty[2] | drain
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * P_STAGES + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    __shared__ int no_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int num_m = (M + 255) / 256, num_n = (N + NT - 1) / NT;
    const int num_tiles = num_m * num_n;
    const int num_kb = (K + BK - 1) / BK;

    auto bar = [&](int i) { return smem_u32(bars + i); };
    const int FULL = 0, EMPTY = P_STAGES, TFULL = 2 * P_STAGES, TEMPTY = 2 * P_STAGES + 2, DRAIN = 2 * P_STAGES + 4;
    // the next accumulator and the parity of its barriers
    auto next_acc = [](int& acc, uint32_t& acc_phase) {
        if (ACCS == 2) {
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
        } else {
            acc_phase ^= 1;
        }
    };
    // entry 2 * P_STAGES + 5 holds the TMEM address and the abort flag
    const int SFULL = 2 * P_STAGES + 6, SEMPTY = 2 * P_STAGES + 7;   // this CTA's own staging

    if (threadIdx.x == 0) {
        for (int s = 0; s < P_STAGES; ++s) {
            mbar_init(bar(FULL + s), 1);
            mbar_init(bar(EMPTY + s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(bar(TFULL + a), 1);
            mbar_init(bar(TEMPTY + a), 8);   // 4 epilogue warps in each CTA
        }
        mbar_init(bar(DRAIN), 1);
        if (SPLIT) {
            mbar_init(bar(SFULL), 4);
            mbar_init(bar(SEMPTY), 4);
        }
        *abort_flag = 0;
        no_abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc_pair<TMEM_COLS>(smem_u32(tmem_holder));
        tc_fence_before();
    }
    // barriers of both CTAs initialised before either uses the other's
    __syncwarp();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        // ---------------------------------------------------- TMA producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
                int mb, nb;
                tile_coords(tile, num_m, num_n, mb, nb);
                const int arow = mb * 256 + (int)rank * 128;
                const int brow = nb * NT + (int)rank * 128;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(bar(EMPTY + stage), phase ^ 1, wait_limit, abort_flag, SITE_GEMM_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    const uint32_t full0 = cta0_addr(bar(FULL + stage));
                    if (rank == 0) mbar_arrive_expect_tx(bar(FULL + stage), P_TX_BYTES);
                    tma_load_2d_pair(smem_u32(sA + stage * P_A_STAGE), &tmA, full0, kb * BK, arow);
                    tma_load_2d_pair(smem_u32(sB + stage * P_B_STAGE), &tmB, full0, kb * BK, brow);
                    if (NT == 512)   // this CTA's half of the second 256-column block
                        tma_load_2d_pair(smem_u32(sB + stage * P_B_STAGE + 128 * BK), &tmB, full0, kb * BK, brow + 256);
                    ++issued;
                    if (++stage == P_STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok || *abort_flag) {
                // Copies in flight must land before the pair exits. CTA 0 can see
                // its full barriers complete; both CTAs also wait a bounded grace time.
                if (rank == 0) {
                    for (int s = 0; s < P_STAGES; ++s) {
                        const long long cnt = issued / P_STAGES + (s < issued % P_STAGES ? 1 : 0);
                        if (cnt > 0)
                            mbar_wait(bar(FULL + s), (uint32_t)((cnt - 1) & 1), wait_limit, &no_abort, SITE_GEMM_DRAIN);
                    }
                }
                const long long t0 = clock64();
                while (clock64() - t0 < 2000000) { }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer (CTA 0)
        if (lane == 0 && rank == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
                if (!mbar_wait(bar(TEMPTY + acc), acc_phase ^ 1, wait_limit, abort_flag, SITE_GEMM_MMA_TMEM)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * NT);
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(bar(FULL + stage), phase, wait_limit, abort_flag, SITE_GEMM_MMA_FULL)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + stage * P_A_STAGE);
                    const uint32_t b0 = smem_u32(sB + stage * P_B_STAGE);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        const uint64_t ad = make_sw128_kmajor_desc(a0 + k * UMMA_K);
                        mma_pair<F8>(d_tmem, ad, make_sw128_kmajor_desc(b0 + k * UMMA_K), (kb | k) != 0 ? 1u : 0u);
                        if (NT == 512)
                            mma_pair<F8>(d_tmem + 256, ad, make_sw128_kmajor_desc(b0 + 128 * BK + k * UMMA_K),
                                         (kb | k) != 0 ? 1u : 0u);
                    }
                    mma_commit_pair(bar(EMPTY + stage));
                    if (++stage == P_STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit_pair(bar(TFULL + acc));
                next_acc(acc, acc_phase);
            }
            mma_commit_cta0(bar(DRAIN));
            mbar_wait(bar(DRAIN), 0, wait_limit, &no_abort, SITE_GEMM_DRAIN);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------- epilogue (warps 2..5, both CTAs)
        const int quarter = warp & 3;
        int acc = 0;
        uint32_t acc_phase = 0;
        float* w_s = reinterpret_cast<float*>(smem + P_STAGES * (P_A_STAGE + P_B_STAGE) + 256);
        // without the outlier term: this warp's copy of the tile's output-channel
        // scales, loaded while the tile's main loop runs (the warp is done with
        // the previous tile), so the epilogue reads them from shared memory
        float* scl = w_s + (warp - 2) * NT;
        // bf16 output by bulk tensor stores (tstore): the warp writes each 32 x 32
        // block of its rows into one of its two buffers, and one lane stores it;
        // the TMEM accumulator is released as soon as it has been read, and the
        // stores drain while the next tile's MMAs run
        const bool tma_out = OUT == kOutBF16 && !SPLIT && tstore != 0;
        uint8_t* obuf = reinterpret_cast<uint8_t*>(w_s + 4 * NT) + (size_t)(warp - 2) * 2 * kOutBlockBytes;
        uint32_t nblk = 0;
        uint32_t it = 0;
        for (int tile = pair; tile < num_tiles; tile += npairs, ++it) {
            int mb, nb;
            tile_coords(tile, num_m, num_n, mb, nb);
            if (!SPLIT && OUT != kOutI32) {
#pragma unroll
                for (int i = lane * 4; i < NT; i += 128) {
                    const int col = nb * NT + i;
                    float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    if (col + 3 < N) {
                        v = __ldg(reinterpret_cast<const float4*>(w_scale + col));
                    } else {
                        if (col < N) v.x = __ldg(w_scale + col);
                        if (col + 1 < N) v.y = __ldg(w_scale + col + 1);
                        if (col + 2 < N) v.z = __ldg(w_scale + col + 2);
                    }
                    *reinterpret_cast<float4*>(scl + i) = v;
                }
                __syncwarp();
            }
            if (SPLIT && !stage_split(w_s, sp, nb, N, it, bar(SFULL), bar(SEMPTY), wait_limit, abort_flag)) break;
            if (!mbar_wait(bar(TFULL + acc), acc_phase, wait_limit, abort_flag, SITE_GEMM_EPILOGUE)) break;
            tc_fence_after();
            const int64_t row = (int64_t)mb * 256 + rank * 128 + quarter * 32 + lane;
            const bool row_ok = row < M;
            const float sa = (OUT != kOutI32 && row_ok) ? __ldg(x_scale + row) : 0.0f;
            const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * NT);
#pragma unroll 1
            for (int c = 0; c < NT / 32; c += 2) {
                uint32_t r0[32], r1[32];
                tmem_ld_32x32b_x32(taddr + c * 32, r0);
                tmem_ld_32x32b_x32(taddr + (c + 1) * 32, r1);
                tmem_wait_ld();
                const int col0 = nb * NT + c * 32;
                if (tma_out) {
                    const int row_w = mb * 256 + (int)rank * 128 + quarter * 32;   // the warp's first row
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const uint32_t* rr = j ? r1 : r0;
                        const int cc = col0 + 32 * j;
                        uint8_t* buf = obuf + (nblk & 1u) * kOutBlockBytes;
                        if (lane == 0) bulk_wait_read_le1();   // this buffer's last store has read it
                        __syncwarp();
                        const float* sw = scl + (cc - nb * NT);   // zero past N
                        uint32_t pk[16];
#pragma unroll
                        for (int i = 0; i < 32; i += 2)
                            pk[i / 2] = pack_bf16x2(dequant_raw<F8>(rr[i], sa, sw[i]),
                                                    dequant_raw<F8>(rr[i + 1], sa, sw[i + 1]));
                        uint4* dst = reinterpret_cast<uint4*>(buf + lane * 64);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0 && cc < N && row_w < M) {
                            tma_store_2d(&tmY, smem_u32(buf), cc, row_w);   // rows past M, columns past N clipped
                            bulk_commit_group();
                        }
                        ++nblk;
                    }
                    continue;
                }
                const float* xr = SPLIT && row_ok ? sp.x_out + row * sp.ld : nullptr;
                // scales indexed by absolute column: this warp's copy, or global memory
                const float* sw_base = SPLIT ? w_scale : scl - nb * NT;
                if (row_ok && col0 < N)
                    store_row32<OUT, SPLIT, F8 ? kAkE4M3 : kAkI8, !SPLIT>(y, row, col0, N, r0, sa, sw_base, xr,
                                                                          w_s + c * 32, sp.ld);
                if (row_ok && col0 + 32 < N)
                    store_row32<OUT, SPLIT, F8 ? kAkE4M3 : kAkI8, !SPLIT>(y, row, col0 + 32, N, r1, sa, sw_base, xr,
                                                                          w_s + (c + 1) * 32, sp.ld);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (rank == 0) mbar_arrive(bar(TEMPTY + acc));
                else arrive_on_cta0(bar(TEMPTY + acc));
                if (SPLIT) mbar_arrive(bar(SEMPTY));   // this warp has read the staged tile
            }
            next_acc(acc, acc_phase);
        }
        if (tma_out && lane == 0) bulk_wait_all();   // every output block written
    }

    // neither CTA leaves while the other may still touch its shared memory or TMEM
    __syncwarp();
    tc_fence_before();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair<TMEM_COLS>(tmem_base);
    }
}

// ================================================================== decode
// Work unit = (row tile of W, k-block). CTA c owns units [c*U/G, (c+1)*U/G);
// a maximal run of its units inside one row tile is a segment, accumulated in
// TMEM and added into ws_acc[t * N + n] with integer atomics. tile_count[tile]
// (one counter per 32-row quarter of the tile) counts k-blocks merged so far;
// the warp that brings it to num_kb writes those rows of Y and leaves ws_acc /
// tile_count zero again.
template <int OUT, bool SPLIT>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
gemm_stream_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                   const float* __restrict__ x_scale, const float* __restrict__ w_scale,
                   void* __restrict__ y, int M, int N, int K,
                   int32_t* __restrict__ ws_acc, unsigned int* __restrict__ tile_count,
                   const SplitTerm sp, long long wait_limit) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + S_STAGES * S_A_STAGE;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sB + S_STAGES * S_B_STAGE);
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * S_STAGES + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    __shared__ int no_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_tiles = (N + S_BM - 1) / S_BM;
    const int num_kb = (K + BK - 1) / BK;
    const long long units = (long long)num_tiles * num_kb;
    const long long u_begin = units * blockIdx.x / gridDim.x;
    const long long u_end = units * (blockIdx.x + 1) / gridDim.x;

    auto bar = [&](int i) { return smem_u32(bars + i); };
    const int FULL = 0, EMPTY = S_STAGES, TFULL = 2 * S_STAGES, TEMPTY = 2 * S_STAGES + 2, DRAIN = 2 * S_STAGES + 4;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S_STAGES; ++s) {
            mbar_init(bar(FULL + s), 1);
            mbar_init(bar(EMPTY + s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(bar(TFULL + a), 1);
            mbar_init(bar(TEMPTY + a), 4);
        }
        mbar_init(bar(DRAIN), 1);
        *abort_flag = 0;
        no_abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        tmem_alloc<S_TMEM_COLS>(smem_u32(tmem_holder));
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (long long u = u_begin; u < u_end && ok; ++u) {
                const int tile = (int)(u / num_kb), kb = (int)(u % num_kb);
                if (!mbar_wait(bar(EMPTY + stage), phase ^ 1, wait_limit, abort_flag, SITE_STREAM_PRODUCER)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(bar(FULL + stage), S_A_STAGE + S_B_STAGE);
                tma_load_2d(smem_u32(sA + stage * S_A_STAGE), &tmW, bar(FULL + stage), kb * BK, tile * S_BM);
                tma_load_2d(smem_u32(sB + stage * S_B_STAGE), &tmX, bar(FULL + stage), kb * BK, 0);
                ++issued;
                if (++stage == S_STAGES) { stage = 0; phase ^= 1; }
            }
            if (!ok || *abort_flag) {
                for (int s = 0; s < S_STAGES; ++s) {
                    const long long cnt = issued / S_STAGES + (s < issued % S_STAGES ? 1 : 0);
                    if (cnt > 0)
                        mbar_wait(bar(FULL + s), (uint32_t)((cnt - 1) & 1), wait_limit, &no_abort, SITE_STREAM_DRAIN);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            long long u = u_begin;
            while (u < u_end && ok) {
                const int tile = (int)(u / num_kb);
                const long long seg_end = min(u_end, (long long)(tile + 1) * num_kb);
                if (!mbar_wait(bar(TEMPTY + acc), acc_phase ^ 1, wait_limit, abort_flag, SITE_STREAM_MMA_TMEM)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * S_BN);
                bool first = true;
                for (; u < seg_end; ++u) {
                    if (!mbar_wait(bar(FULL + stage), phase, wait_limit, abort_flag, SITE_STREAM_MMA_FULL)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + stage * S_A_STAGE);
                    const uint32_t b0 = smem_u32(sB + stage * S_B_STAGE);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        mma_i8(d_tmem, make_sw128_kmajor_desc(a0 + k * UMMA_K),
                               make_sw128_kmajor_desc(b0 + k * UMMA_K), IDESC_STREAM,
                               (first && k == 0) ? 0u : 1u);
                    }
                    first = false;
                    mma_commit(bar(EMPTY + stage));
                    if (++stage == S_STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit(bar(TFULL + acc));
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
            mma_commit(bar(DRAIN));
            mbar_wait(bar(DRAIN), 0, wait_limit, &no_abort, SITE_STREAM_DRAIN);
        }
        __syncwarp();
    } else {
        // Each epilogue warp owns 32 weight rows of the tile (its TMEM lane
        // quarter) and its own completion counter, so no cross-warp barrier is
        // needed and an aborted wait cannot strand the other warps.
        const int quarter = warp & 3;
        int acc = 0;
        uint32_t acc_phase = 0;
        long long u = u_begin;
        while (u < u_end) {
            const int tile = (int)(u / num_kb);
            const long long seg_end = min(u_end, (long long)(tile + 1) * num_kb);
            const unsigned int seg_len = (unsigned int)(seg_end - u);
            u = seg_end;
            if (!mbar_wait(bar(TFULL + acc), acc_phase, wait_limit, abort_flag, SITE_STREAM_EPILOGUE)) break;
            tc_fence_after();
            uint32_t r[16];
            tmem_ld_32x32b_x16(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * S_BN), r);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(TEMPTY + acc));
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;

            const int n = tile * S_BM + quarter * 32 + lane;
            if (n < N) {
#pragma unroll
                for (int t = 0; t < S_BN; ++t)
                    if (t < M) atomicAdd(ws_acc + (int64_t)t * N + n, (int32_t)r[t]);
            }
            __threadfence();
            __syncwarp();
            unsigned int* cnt = tile_count + tile * 4 + quarter;
            unsigned int prev = 0;
            if (lane == 0) prev = atomicAdd(cnt, seg_len);
            prev = __shfl_sync(0xffffffffu, prev, 0);
            if (prev + seg_len == (unsigned int)num_kb) {
                // Last contributor of these 32 rows: every other CTA's partial
                // sums are in ws_acc. Write Y and leave the workspace zeroed.
                __threadfence();
                if (n < N) {
                    // all partial sums (and scales) are loaded before any is used
                    const float sw = (OUT != kOutI32) ? __ldg(w_scale + n) : 0.0f;
                    int32_t a[S_BN];
                    float sa[S_BN];
#pragma unroll
                    for (int t = 0; t < S_BN; ++t) {
                        a[t] = t < M ? __ldcg(ws_acc + (int64_t)t * N + n) : 0;
                        sa[t] = (OUT != kOutI32 && t < M) ? __ldg(x_scale + t) : 0.0f;
                    }
#pragma unroll
                    for (int t = 0; t < S_BN; ++t) {
                        if (t < M) {
                            const int64_t o = (int64_t)t * N + n;
                            ws_acc[o] = 0;
                            if (OUT == kOutI32) {
                                static_cast<int32_t*>(y)[o] = a[t];
                            } else {
                                float v = dequant(a[t], sa[t], sw);
                                if (SPLIT) v = add_split1(v, t, n, sp);
                                if (OUT == kOutF32) static_cast<float*>(y)[o] = v;
                                else static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(v);
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) *cnt = 0u;
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc<S_TMEM_COLS>(tmem_base);
    }
}

// ================================================================== decode, clusters
// The same swap-AB product (weight rows on the MMA's 128-row side, the tokens
// as N = 16), with the split-K partial sums merged inside thread-block
// clusters instead of through global memory.
//
// Work split: the 128-row weight tiles are dealt to the clusters in contiguous
// runs of whole tiles; inside a cluster, the (tile, k-block) units of its tiles
// are split evenly between its CTAs in contiguous ranges. A CTA accumulates
// each run of its units inside one tile (a segment) in TMEM. The CTA holding a
// tile's first k-block owns the tile and writes its rows of Y. Every other CTA
// holding units of that tile -- for a given CTA this can only be its first
// segment, and an owner can receive only into its last segment -- adds its
// partial sums into the owner's receive buffer in shared memory with
// distributed-shared-memory integer atomics (exact and order-free) and then
// arrives, with release semantics at cluster scope, on the owner's receive
// barrier. The owner's epilogue waits (bounded, acquire at cluster scope) for
// the arrivals it expects, adds the buffer to its own TMEM partial sums and
// applies the epilogue. Nothing is written to global memory but Y.
//
// Segment bookkeeping is pure arithmetic on the static split, identical in
// every CTA of the cluster.
struct DecodeSplit {
    int rank, csize;          // this CTA's rank in the cluster, the cluster size
    long long units;          // units of the cluster's tiles
    int tile0;                // the cluster's first tile
    int num_kb;
    __device__ long long begin(int r) const { return units * r / csize; }
    // rank holding local unit u (u < units)
    __device__ int holder(long long u) const {
        int r = (int)((u * csize) / units);
        while (r + 1 < csize && begin(r + 1) <= u) ++r;
        while (r > 0 && begin(r) > u) --r;
        return r;
    }
};


constexpr size_t DC_RECV_BYTES = (size_t)S_BN * S_BM * sizeof(int32_t);   // 8 KB: [token][row] int32
constexpr size_t decode_cluster_smem_bytes() {
    return 1024 + S_STAGES * (S_A_STAGE + S_B_STAGE) + DC_RECV_BYTES + 256;
}

template <int OUT>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
gemm_decode_cluster_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                           const float* __restrict__ x_scale, const float* __restrict__ w_scale,
                           void* __restrict__ y, int M, int N, int K, long long wait_limit) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + S_STAGES * S_A_STAGE;
    int32_t* recv = reinterpret_cast<int32_t*>(sB + S_STAGES * S_B_STAGE);
    uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(recv) + DC_RECV_BYTES);
    // bars: full[S_STAGES] | empty[S_STAGES] | tfull[2] | tempty[2] | drain | recv
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * S_STAGES + 6);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    __shared__ int no_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_tiles = (N + S_BM - 1) / S_BM;
    const int num_kb = (K + BK - 1) / BK;
    DecodeSplit sp;
    sp.csize = (int)cluster_nctarank();
    sp.rank = (int)cluster_rank();
    const int cl = blockIdx.x / sp.csize, ncl = gridDim.x / sp.csize;
    sp.tile0 = (int)((long long)num_tiles * cl / ncl);
    const int tile1 = (int)((long long)num_tiles * (cl + 1) / ncl);
    sp.num_kb = num_kb;
    sp.units = (long long)(tile1 - sp.tile0) * num_kb;
    const long long u_begin = sp.begin(sp.rank), u_end = sp.begin(sp.rank + 1);

    auto bar = [&](int i) { return smem_u32(bars + i); };
    const int FULL = 0, EMPTY = S_STAGES, TFULL = 2 * S_STAGES, TEMPTY = 2 * S_STAGES + 2, DRAIN = 2 * S_STAGES + 4,
              RECV = 2 * S_STAGES + 5;

    // Contributors to this CTA's last segment (if it is owned and the tile
    // continues past this CTA's range): the CTAs holding the rest of the tile.
    int n_contrib = 0;
    if (u_end > u_begin) {
        const long long last_lo = max(u_begin, ((u_end - 1) / num_kb) * num_kb);
        const long long tile_end = ((u_end - 1) / num_kb + 1) * num_kb;
        if (last_lo % num_kb == 0 && u_end < tile_end) {
            const int last = sp.holder(tile_end - 1);
            for (int q = sp.rank + 1; q <= last; ++q) n_contrib += sp.begin(q) < sp.begin(q + 1) ? 1 : 0;
        }
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < S_STAGES; ++s) {
            mbar_init(bar(FULL + s), 1);
            mbar_init(bar(EMPTY + s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(bar(TFULL + a), 1);
            mbar_init(bar(TEMPTY + a), 4);
        }
        mbar_init(bar(DRAIN), 1);
        mbar_init(bar(RECV), n_contrib > 0 ? (uint32_t)(128 * n_contrib) : 1u);
        *abort_flag = 0;
        no_abort = 0;
        fence_barrier_init();
    }
    for (int i = threadIdx.x; i < (int)(DC_RECV_BYTES / 16); i += GEMM_THREADS)
        reinterpret_cast<uint4*>(recv)[i] = make_uint4(0u, 0u, 0u, 0u);
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        tmem_alloc<S_TMEM_COLS>(smem_u32(tmem_holder));
        tc_fence_before();
    }
    // every CTA's barriers and receive buffer are ready before any remote access
    __syncwarp();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (long long u = u_begin; u < u_end && ok; ++u) {
                const int tile = sp.tile0 + (int)(u / num_kb), kb = (int)(u % num_kb);
                if (!mbar_wait(bar(EMPTY + stage), phase ^ 1, wait_limit, abort_flag, SITE_STREAM_PRODUCER)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(bar(FULL + stage), S_A_STAGE + S_B_STAGE);
                tma_load_2d(smem_u32(sA + stage * S_A_STAGE), &tmW, bar(FULL + stage), kb * BK, tile * S_BM);
                tma_load_2d(smem_u32(sB + stage * S_B_STAGE), &tmX, bar(FULL + stage), kb * BK, 0);
                ++issued;
                if (++stage == S_STAGES) { stage = 0; phase ^= 1; }
            }
            if (!ok || *abort_flag) {
                for (int s = 0; s < S_STAGES; ++s) {
                    const long long cnt = issued / S_STAGES + (s < issued % S_STAGES ? 1 : 0);
                    if (cnt > 0)
                        mbar_wait(bar(FULL + s), (uint32_t)((cnt - 1) & 1), wait_limit, &no_abort, SITE_STREAM_DRAIN);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            long long u = u_begin;
            while (u < u_end && ok) {
                const long long seg_end = min(u_end, (u / num_kb + 1) * num_kb);
                if (!mbar_wait(bar(TEMPTY + acc), acc_phase ^ 1, wait_limit, abort_flag, SITE_STREAM_MMA_TMEM)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * S_BN);
                bool first = true;
                for (; u < seg_end; ++u) {
                    if (!mbar_wait(bar(FULL + stage), phase, wait_limit, abort_flag, SITE_STREAM_MMA_FULL)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + stage * S_A_STAGE);
                    const uint32_t b0 = smem_u32(sB + stage * S_B_STAGE);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k)
                        mma_i8(d_tmem, make_sw128_kmajor_desc(a0 + k * UMMA_K),
                               make_sw128_kmajor_desc(b0 + k * UMMA_K), IDESC_STREAM, (first && k == 0) ? 0u : 1u);
                    first = false;
                    mma_commit(bar(EMPTY + stage));
                    if (++stage == S_STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit(bar(TFULL + acc));
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
            mma_commit(bar(DRAIN));
            mbar_wait(bar(DRAIN), 0, wait_limit, &no_abort, SITE_STREAM_DRAIN);
        }
        __syncwarp();
    } else {
        // Epilogue: warp `quarter` owns weight rows quarter*32 .. +32 of each
        // tile (its TMEM lane quarter); lane l holds row quarter*32 + l.
        const int quarter = warp & 3;
        const int row_in_tile = quarter * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        long long u = u_begin;
        while (u < u_end) {
            const long long seg_lo = u;
            const long long seg_hi = min(u_end, (u / num_kb + 1) * num_kb);
            const int tile = sp.tile0 + (int)(seg_lo / num_kb);
            u = seg_hi;
            if (!mbar_wait(bar(TFULL + acc), acc_phase, wait_limit, abort_flag, SITE_STREAM_EPILOGUE)) break;
            tc_fence_after();
            uint32_t r[16];
            tmem_ld_32x32b_x16(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * S_BN), r);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(TEMPTY + acc));
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;

            if (seg_lo % num_kb != 0) {
                // a contribution to the tile's owner
                const int owner = sp.holder((seg_lo / num_kb) * num_kb);
                // the owner holds the tile's first unit, before this CTA's range
                if (!dchk(owner >= 0 && owner < sp.rank, SITE_DBG_DECODE_OWNER)) continue;
                const uint32_t rbase = mapa_rank(smem_u32(recv), (uint32_t)owner);
#pragma unroll
                for (int t = 0; t < S_BN; ++t)
                    if (t < M) red_add_cluster(rbase + (uint32_t)((t * S_BM + row_in_tile) * 4), (int32_t)r[t]);
                arrive_remote_release(mapa_rank(bar(RECV), (uint32_t)owner));
                continue;
            }
            if (seg_hi % num_kb != 0 && n_contrib > 0) {
                // owned, and the rest of the tile comes from the next CTAs
                if (!mbar_wait_acq_cluster(bar(RECV), 0, wait_limit, abort_flag, SITE_STREAM_EPILOGUE)) break;
#pragma unroll
                for (int t = 0; t < S_BN; ++t)
                    if (t < M) r[t] = (uint32_t)((int32_t)r[t] + recv[t * S_BM + row_in_tile]);
            }
            const int n = tile * S_BM + row_in_tile;
            if (n < N) {
                const float sw = (OUT != kOutI32) ? __ldg(w_scale + n) : 0.0f;
#pragma unroll
                for (int t = 0; t < S_BN; ++t) {
                    if (t < M) {
                        const int64_t o = (int64_t)t * N + n;
                        if (OUT == kOutI32) {
                            static_cast<int32_t*>(y)[o] = (int32_t)r[t];
                        } else {
                            const float v = dequant((int32_t)r[t], __ldg(x_scale + t), sw);
                            if (OUT == kOutF32) static_cast<float*>(y)[o] = v;
                            else static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(v);
                        }
                    }
                }
            }
        }
    }

    // no CTA leaves while another may still add into its shared memory
    __syncwarp();
    tc_fence_before();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc<S_TMEM_COLS>(tmem_base);
    }
}

// ================================================================== host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

sq_status get_encoder() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode) {
        set_error("cuTensorMapEncodeTiled is not available from the driver");
        return SQ_ERR_CUDA;
    }
    return SQ_OK;
}

// Row-major int8 matrix [rows x K] as a 2-D tensor map with 128B swizzle and a
// (128 bytes of K) x box_rows box. Out-of-range rows/columns read as zero.
sq_status make_map_i8(CUtensorMap* map, const void* base, int64_t rows, int64_t K, uint32_t box_rows) {
    sq_status r = get_encoder();
    if (r != SQ_OK) return r;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K};
    cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult cr = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed (%d) for a %lld x %lld int8 matrix", (int)cr,
                  (long long)rows, (long long)K);
        return SQ_ERR_CUDA;
    }
    return SQ_OK;
}

// Row-major bf16 output Y [M x N] as a 2-D tensor map for bulk stores of 32 x 32
// blocks (no swizzle; out-of-range rows and columns are not written). N * 2
// must be a multiple of 16 bytes.
sq_status make_map_out_bf16(CUtensorMap* map, void* base, int64_t M, int64_t N) {
    sq_status r = get_encoder();
    if (r != SQ_OK) return r;
    cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)N * 2};
    cuuint32_t box[2] = {32u, 32u};
    cuuint32_t estr[2] = {1, 1};
    CUresult cr = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed (%d) for a %lld x %lld bf16 output", (int)cr, (long long)M,
                  (long long)N);
        return SQ_ERR_CUDA;
    }
    return SQ_OK;
}

// Row-major bf16 matrix [rows x K] as a 2-D tensor map with 128B swizzle and a
// (64 elements = 128 bytes of K) x box_rows box.
sq_status make_map_bf16(CUtensorMap* map, const void* base, int64_t rows, int64_t K, uint32_t box_rows) {
    sq_status r = get_encoder();
    if (r != SQ_OK) return r;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {64u, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult cr = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed (%d) for a %lld x %lld bf16 matrix", (int)cr,
                  (long long)rows, (long long)K);
        return SQ_ERR_CUDA;
    }
    return SQ_OK;
}

template <typename Kern>
sq_status ensure_smem_attr(Kern k, size_t bytes, bool& done) {
    // Per device: the attribute is a property of the function on the current device.
    static thread_local int last_dev = -1;
    (void)last_dev;
    if (done) return SQ_OK;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(max dynamic shared memory)");
    done = true;
    return SQ_OK;
}

template <int OUT, bool SPLIT = false, int AK = kAkI8>
sq_status launch_tiled(const CUtensorMap& ta, const CUtensorMap& tb, const float* xs, const float* wsc, void* y,
                       int M, int N, int K, cudaStream_t st, const SplitTerm& sp = SplitTerm{}) {
    static bool attr_done[64] = {};
    const DeviceInfo& di = device_info();
    const size_t smem = tiled_smem_bytes() + (SPLIT ? kSplitSmem : 0);
    sq_status r = ensure_smem_attr(gemm_tiled_kernel<OUT, SPLIT, AK>, smem, attr_done[di.device & 63]);
    if (r != SQ_OK) return r;
    const int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    const int grid = tiles < di.sm_count ? tiles : di.sm_count;
    return launch_pdl("gemm_tiled_kernel", gemm_tiled_kernel<OUT, SPLIT, AK>, dim3(grid), dim3(GEMM_THREADS), smem, st, 1,
                      ta, tb, xs, wsc, y, M, N, K, sp, wait_limit_cycles());
}

template <int OUT, bool SPLIT, bool F8, int NT>
sq_status launch_pair_nt(const CUtensorMap& ta, const CUtensorMap& tb, const float* xs, const float* wsc, void* y,
                         int M, int N, int K, cudaStream_t st, const SplitTerm& sp) {
    // bf16 output through bulk tensor stores where the row stride allows a map
    CUtensorMap ty;
    std::memset(&ty, 0, sizeof(ty));
    int tstore = 0;
    if (OUT == kOutBF16 && !SPLIT && (N % 8) == 0) {
        sq_status rm = make_map_out_bf16(&ty, y, M, N);
        if (rm != SQ_OK) return rm;
        tstore = 1;
    }
    static bool attr_done[64] = {};
    const DeviceInfo& di = device_info();
    const size_t smem = pair_smem_bytes(NT) + pair_epilogue_smem_bytes(NT, SPLIT);
    sq_status r = ensure_smem_attr(gemm_pair_kernel<OUT, SPLIT, F8, NT>, smem, attr_done[di.device & 63]);
    if (r != SQ_OK) return r;
    const int tiles = ((M + 255) / 256) * ((N + NT - 1) / NT);
    const int max_pairs = di.sm_count / 2;
    const int pairs = tiles < max_pairs ? tiles : max_pairs;
    return launch_pdl("gemm_pair_kernel", gemm_pair_kernel<OUT, SPLIT, F8, NT>, dim3(2 * pairs), dim3(GEMM_THREADS),
                      smem, st, 2, ta, tb, xs, wsc, y, M, N, K, sp, wait_limit_cycles(), ty, tstore);
}

// Wide (512-column) tiles for long K, where a tile's main loop dwarfs its
// unoverlapped epilogue; 256-column tiles otherwise and for the outlier term.
constexpr int kWidePairMinK = 16384;

template <int OUT, bool SPLIT = false, bool F8 = false>
sq_status launch_pair(const CUtensorMap& ta, const CUtensorMap& tb, const float* xs, const float* wsc, void* y,
                      int M, int N, int K, cudaStream_t st, const SplitTerm& sp = SplitTerm{}) {
    if constexpr (!SPLIT) {
        if (K >= kWidePairMinK) return launch_pair_nt<OUT, SPLIT, F8, 512>(ta, tb, xs, wsc, y, M, N, K, st, sp);
    }
    return launch_pair_nt<OUT, SPLIT, F8, 256>(ta, tb, xs, wsc, y, M, N, K, st, sp);
}

template <int OUT, bool SPLIT = false>
sq_status launch_stream(const CUtensorMap& tw, const CUtensorMap& tx, const float* xs, const float* wsc, void* y,
                        int M, int N, int K, int32_t* ws_acc, unsigned int* counts, cudaStream_t st,
                        const SplitTerm& sp = SplitTerm{}) {
    static bool attr_done[64] = {};
    const DeviceInfo& di = device_info();
    const size_t smem = stream_smem_bytes();
    sq_status r = ensure_smem_attr(gemm_stream_kernel<OUT, SPLIT>, smem, attr_done[di.device & 63]);
    if (r != SQ_OK) return r;
    const long long units = (long long)((N + S_BM - 1) / S_BM) * ((K + BK - 1) / BK);
    const int grid = units < di.sm_count ? (int)units : di.sm_count;
    return launch_pdl("gemm_stream_kernel", gemm_stream_kernel<OUT, SPLIT>, dim3(grid), dim3(GEMM_THREADS), smem, st,
                      1, tw, tx, xs, wsc, y, M, N, K, ws_acc, counts, sp, wait_limit_cycles());
}

// Cluster sizes the decode kernel may use, and how many clusters of each can
// be resident at once on the current device (queried once per device).
constexpr int kDecodeClusterSizes[4] = {2, 4, 8, 16};

struct DecodeClusterInfo {
    bool ready = false;
    int max_clusters[4] = {0, 0, 0, 0};
};
DecodeClusterInfo g_dc_info[64];
std::mutex g_dc_mu;

sq_status decode_cluster_info(DecodeClusterInfo& out) {
    const DeviceInfo& di = device_info();
    std::lock_guard<std::mutex> lk(g_dc_mu);
    DecodeClusterInfo& d = g_dc_info[di.device & 63];
    if (!d.ready) {
        const size_t smem = decode_cluster_smem_bytes();
        auto kern = gemm_decode_cluster_kernel<kOutBF16>;
        cudaError_t e;
        const void* fns[3] = {(const void*)gemm_decode_cluster_kernel<kOutF32>,
                              (const void*)gemm_decode_cluster_kernel<kOutBF16>,
                              (const void*)gemm_decode_cluster_kernel<kOutI32>};
        for (const void* f : fns) {
            if ((e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
                return cuda_fail(e, "cudaFuncSetAttribute(max dynamic shared memory)");
            if ((e = cudaFuncSetAttribute(f, cudaFuncAttributeNonPortableClusterSizeAllowed, 1)) != cudaSuccess)
                return cuda_fail(e, "cudaFuncSetAttribute(non-portable cluster size)");
        }
        for (int i = 0; i < 4; ++i) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(kDecodeClusterSizes[i] * 8);
            cfg.blockDim = dim3(GEMM_THREADS);
            cfg.dynamicSmemBytes = smem;
            cudaLaunchAttribute attr;
            attr.id = cudaLaunchAttributeClusterDimension;
            attr.val.clusterDim.x = kDecodeClusterSizes[i];
            attr.val.clusterDim.y = 1;
            attr.val.clusterDim.z = 1;
            cfg.attrs = &attr;
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
                cudaGetLastError();
                n = 0;
            }
            d.max_clusters[i] = n;
        }
        d.ready = true;
    }
    out = d;
    return SQ_OK;
}

// The cluster size with the fewest units on the busiest CTA (ties: the
// smaller size); 0 if no cluster size can be launched.
int pick_decode_cluster(const DecodeClusterInfo& info, int num_tiles, int num_kb, int& ncl_out) {
    long long best = -1;
    int best_c = 0;
    for (int i = 0; i < 4; ++i) {
        const int c = kDecodeClusterSizes[i];
        const int ncl = std::min(info.max_clusters[i], num_tiles);
        if (ncl <= 0) continue;
        const long long tiles = (num_tiles + ncl - 1) / ncl;
        const long long busiest = (tiles * num_kb + c - 1) / c;
        if (best < 0 || busiest < best) {
            best = busiest;
            best_c = c;
            ncl_out = ncl;
        }
    }
    return best_c;
}

template <int OUT>
sq_status launch_decode_cluster(const CUtensorMap& tw, const CUtensorMap& tx, const float* xs, const float* wsc,
                                void* y, int M, int N, int K, int csize, int ncl, cudaStream_t st) {
    return launch_pdl("gemm_decode_cluster_kernel", gemm_decode_cluster_kernel<OUT>, dim3(csize * ncl),
                      dim3(GEMM_THREADS), decode_cluster_smem_bytes(), st, (unsigned)csize, tw, tx, xs, wsc, y, M, N,
                      K, wait_limit_cycles());
}

size_t stream_ws_bytes(int64_t M, int64_t N) {
    const size_t acc = (size_t)M * (size_t)N * sizeof(int32_t);
    const size_t acc_al = (acc + 255) & ~size_t(255);
    const size_t cnt = (size_t)((N + S_BM - 1) / S_BM) * 4 * sizeof(unsigned int);
    return acc_al + ((cnt + 255) & ~size_t(255));
}

}  // namespace

size_t gemm_workspace_size(int64_t M, int64_t N, int64_t K) {
    (void)K;
    if (M <= 0 || N <= 0) return 0;
    return M <= STREAM_MAX_M ? stream_ws_bytes(M, N) : 0;
}

sq_status gemm_dispatch(const int8_t* xq, const float* x_scale, const int8_t* wq, const float* w_scale,
                        int64_t M, int64_t N, int64_t K, void* y, sq_dtype out_dt, void* workspace,
                        size_t ws_bytes, cudaStream_t st, const SplitTerm* split) {
    if (M < 0 || N < 0 || K < 0) { set_error("negative size"); return SQ_ERR_INVALID_ARG; }
    if (out_dt != SQ_F32 && out_dt != SQ_BF16 && out_dt != SQ_I32) {
        set_error("output dtype must be SQ_F32, SQ_BF16 or SQ_I32");
        return SQ_ERR_UNSUPPORTED;
    }
    if (M == 0 || N == 0) return SQ_OK;
    if (K == 0 || K % 16 != 0) { set_error("K=%lld must be a positive multiple of 16", (long long)K); return SQ_ERR_UNSUPPORTED; }
    if (K > 133144) { set_error("K=%lld: 127*127*K would overflow int32", (long long)K); return SQ_ERR_UNSUPPORTED; }
    if (M > 2147483647LL || N > 2147483647LL) { set_error("size too large"); return SQ_ERR_UNSUPPORTED; }
    if (!xq || !wq || !y) { set_error("NULL pointer"); return SQ_ERR_INVALID_ARG; }
    if (out_dt != SQ_I32 && (!x_scale || !w_scale)) { set_error("NULL scale pointer"); return SQ_ERR_INVALID_ARG; }
    if (!aligned16(xq) || !aligned16(wq) || !aligned16(y) || (w_scale && !aligned16(w_scale))) {
        set_error("xq, wq, y and w_scale must be 16-byte aligned");
        return SQ_ERR_UNSUPPORTED;
    }
    const int out = out_dt == SQ_F32 ? kOutF32 : (out_dt == SQ_BF16 ? kOutBF16 : kOutI32);
    sq_status r;
    const bool sp_on = split != nullptr && split->ld > 0;
    const SplitTerm sp = sp_on ? *split : SplitTerm{};
    if (M <= STREAM_MAX_M) {
        const size_t need = stream_ws_bytes(M, N);
        if (!workspace || ws_bytes < need) {
            set_error("workspace too small: %zu bytes given, %zu needed", ws_bytes, need);
            return SQ_ERR_INVALID_ARG;
        }
        if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) {
            set_error("workspace must be 256-byte aligned");
            return SQ_ERR_UNSUPPORTED;
        }
        CUtensorMap tw, tx;
        if ((r = make_map_i8(&tw, wq, N, K, S_BM)) != SQ_OK) return r;
        if ((r = make_map_i8(&tx, xq, M, K, S_BN)) != SQ_OK) return r;
        if (!sp_on) {
            // the cluster kernel merges its partial sums on chip and needs no
            // workspace; the workspace serves the decomposed path's kernel
            DecodeClusterInfo info;
            if ((r = decode_cluster_info(info)) != SQ_OK) return r;
            int ncl = 0;
            const int csize = pick_decode_cluster(info, (int)((N + S_BM - 1) / S_BM), (int)((K + BK - 1) / BK), ncl);
            if (csize > 0) {
                switch (out) {
                    case kOutF32: return launch_decode_cluster<kOutF32>(tw, tx, x_scale, w_scale, y, (int)M, (int)N, (int)K, csize, ncl, st);
                    case kOutBF16: return launch_decode_cluster<kOutBF16>(tw, tx, x_scale, w_scale, y, (int)M, (int)N, (int)K, csize, ncl, st);
                    default: return launch_decode_cluster<kOutI32>(tw, tx, x_scale, w_scale, y, (int)M, (int)N, (int)K, csize, ncl, st);
                }
            }
        }
        int32_t* ws_acc = static_cast<int32_t*>(workspace);
        const size_t acc_al = (((size_t)M * N * 4) + 255) & ~size_t(255);
        unsigned int* counts = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(workspace) + acc_al);
        if (sp_on)
            return out == kOutF32
                ? launch_stream<kOutF32, true>(tw, tx, x_scale, w_scale, y, (int)M, (int)N, (int)K, ws_acc, counts, st, sp)
                : launch_stream<kOutBF16, true>(tw, tx, x_scale, w_scale, y, (int)M, (int)N, (int)K, ws_acc, counts, st, sp);
        switch (out) {
            case kOutF32: return launch_stream<kOutF32>(tw, tx, x_scale, w_scale, y, (int)M, (int)N, (int)K, ws_acc, counts, st);
            case kOutBF16: return launch_stream<kOutBF16>(tw, tx, x_scale, w_scale, y, (int)M, (int)N, (int)K, ws_acc, counts, st);
            default: return launch_stream<kOutI32>(tw, tx, x_scale, w_scale, y, (int)M, (int)N, (int)K, ws_acc, counts, st);
        }
    }
    CUtensorMap ta, tb;
    if (M > 128) {
        // paired SMs: each CTA loads 128-row boxes of A and of B
        if ((r = make_map_i8(&ta, xq, M, K, 128)) != SQ_OK) return r;
        if ((r = make_map_i8(&tb, wq, N, K, 128)) != SQ_OK) return r;
        if (sp_on)
            return out == kOutF32
                ? launch_pair<kOutF32, true>(ta, tb, x_scale, w_scale, y, (int)M, (int)N, (int)K, st, sp)
                : launch_pair<kOutBF16, true>(ta, tb, x_scale, w_scale, y, (int)M, (int)N, (int)K, st, sp);
        switch (out) {
            case kOutF32: return launch_pair<kOutF32>(ta, tb, x_scale, w_scale, y, (int)M, (int)N, (int)K, st);
            case kOutBF16: return launch_pair<kOutBF16>(ta, tb, x_scale, w_scale, y, (int)M, (int)N, (int)K, st);
            default: return launch_pair<kOutI32>(ta, tb, x_scale, w_scale, y, (int)M, (int)N, (int)K, st);
        }
    }
    if ((r = make_map_i8(&ta, xq, M, K, BM)) != SQ_OK) return r;
    if ((r = make_map_i8(&tb, wq, N, K, BN)) != SQ_OK) return r;
    if (sp_on)
        return out == kOutF32
            ? launch_tiled<kOutF32, true>(ta, tb, x_scale, w_scale, y, (int)M, (int)N, (int)K, st, sp)
            : launch_tiled<kOutBF16, true>(ta, tb, x_scale, w_scale, y, (int)M, (int)N, (int)K, st, sp);
    switch (out) {
        case kOutF32: return launch_tiled<kOutF32>(ta, tb, x_scale, w_scale, y, (int)M, (int)N, (int)K, st);
        case kOutBF16: return launch_tiled<kOutBF16>(ta, tb, x_scale, w_scale, y, (int)M, (int)N, (int)K, st);
        default: return launch_tiled<kOutI32>(ta, tb, x_scale, w_scale, y, (int)M, (int)N, (int)K, st);
    }
}

// FP8 E4M3 operands, fp32 accumulation in TMEM: the paired-SM kernel for
// M > 128, the 1-CTA kernel otherwise (no split-K path: fp32 partial sums
// merged by atomics would depend on their order).
sq_status gemm_e4m3_impl(const uint8_t* xq, const float* x_scale, const uint8_t* wq, const float* w_scale, int64_t M,
                         int64_t N, int64_t K, void* y, sq_dtype out_dt, cudaStream_t st) {
    if (M < 0 || N < 0 || K < 0) { set_error("negative size"); return SQ_ERR_INVALID_ARG; }
    if (out_dt != SQ_F32 && out_dt != SQ_BF16) { set_error("output dtype must be SQ_F32 or SQ_BF16"); return SQ_ERR_UNSUPPORTED; }
    if (M == 0 || N == 0) return SQ_OK;
    if (K == 0 || K % 16 != 0) { set_error("K=%lld must be a positive multiple of 16", (long long)K); return SQ_ERR_UNSUPPORTED; }
    if (M > 2147483647LL || N > 2147483647LL || K > 2147483647LL) { set_error("size too large"); return SQ_ERR_UNSUPPORTED; }
    if (!xq || !wq || !y || !x_scale || !w_scale) { set_error("NULL pointer"); return SQ_ERR_INVALID_ARG; }
    if (!aligned16(xq) || !aligned16(wq) || !aligned16(y) || !aligned16(w_scale)) {
        set_error("xq, wq, y and w_scale must be 16-byte aligned");
        return SQ_ERR_UNSUPPORTED;
    }
    sq_status r;
    CUtensorMap ta, tb;
    const SplitTerm none;
    if (M > 128) {
        if ((r = make_map_i8(&ta, xq, M, K, 128)) != SQ_OK) return r;
        if ((r = make_map_i8(&tb, wq, N, K, 128)) != SQ_OK) return r;
        return out_dt == SQ_F32
            ? launch_pair<kOutF32, false, true>(ta, tb, x_scale, w_scale, y, (int)M, (int)N, (int)K, st, none)
            : launch_pair<kOutBF16, false, true>(ta, tb, x_scale, w_scale, y, (int)M, (int)N, (int)K, st, none);
    }
    if ((r = make_map_i8(&ta, xq, M, K, BM)) != SQ_OK) return r;
    if ((r = make_map_i8(&tb, wq, N, K, BN)) != SQ_OK) return r;
    return out_dt == SQ_F32
        ? launch_tiled<kOutF32, false, kAkE4M3>(ta, tb, x_scale, w_scale, y, (int)M, (int)N, (int)K, st, none)
        : launch_tiled<kOutBF16, false, kAkE4M3>(ta, tb, x_scale, w_scale, y, (int)M, (int)N, (int)K, st, none);
}

// ------------------------------------------------------------------ plain floating-point products
// y [M x N] fp32 = x [M x K] . w [N x K]^T, the reference product of the alpha
// search. bf16 operands: the 1-CTA tcgen05 kernel with kind::f16 (every
// product exact in fp32, the sum accumulated in fp32 in TMEM, its order the
// tensor core's). fp32 operands: a CUDA-core kernel, each output a chain of
// fp32 fused multiply-adds in k order.
constexpr int SG_TM = 64, SG_TN = 64, SG_TK = 16, SG_THREADS = 256;

__global__ void __launch_bounds__(SG_THREADS)
sgemm_xwt_kernel(const float* __restrict__ x, const float* __restrict__ w, float* __restrict__ y, int M, int N,
                 int K) {
    __shared__ float xs[SG_TK][SG_TM + 4];
    __shared__ float ws[SG_TK][SG_TN + 4];
    pdl_wait();
    pdl_trigger();
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;   // 16 x 16 threads, 4 x 4 outputs each
    const int m0 = blockIdx.y * SG_TM, n0 = blockIdx.x * SG_TN;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += SG_TK) {
        for (int i = threadIdx.x; i < SG_TM * SG_TK; i += SG_THREADS) {
            const int r = i / SG_TK, c = i % SG_TK;
            const int gm = m0 + r, gn = n0 + r, gk = k0 + c;
            xs[c][r] = (gm < M && gk < K) ? __ldg(x + (int64_t)gm * K + gk) : 0.0f;
            ws[c][r] = (gn < N && gk < K) ? __ldg(w + (int64_t)gn * K + gk) : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < SG_TK; ++c) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = xs[c][ty * 4 + i];
                b[i] = ws[c][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int gm = m0 + ty * 4 + i, gn = n0 + tx * 4 + j;
            if (gm < M && gn < N) y[(int64_t)gm * N + gn] = acc[i][j];
        }
}

sq_status float_gemm_xwt(const void* x, const void* w, sq_dtype dt, int64_t M, int64_t N, int64_t K, float* y,
                         cudaStream_t st) {
    if (M <= 0 || N <= 0) return SQ_OK;
    if (M > 2147483647LL || N > 2147483647LL || K > 2147483647LL) { set_error("size too large"); return SQ_ERR_UNSUPPORTED; }
    if (dt == SQ_BF16) {
        if (K % 8 != 0) { set_error("K must be a multiple of 8 for bf16 operands"); return SQ_ERR_UNSUPPORTED; }
        CUtensorMap ta, tb;
        sq_status r;
        if ((r = make_map_bf16(&ta, x, M, K, BM)) != SQ_OK) return r;
        if ((r = make_map_bf16(&tb, w, N, K, BN)) != SQ_OK) return r;
        return launch_tiled<kOutF32, false, kAkBF16>(ta, tb, nullptr, nullptr, y, (int)M, (int)N, (int)K, st);
    }
    const dim3 grid((unsigned)((N + SG_TN - 1) / SG_TN), (unsigned)((M + SG_TM - 1) / SG_TM));
    return launch_pdl("sgemm_xwt_kernel", sgemm_xwt_kernel, grid, dim3(SG_THREADS), 0, st, 1,
                      static_cast<const float*>(x), static_cast<const float*>(w), y, (int)M, (int)N, (int)K);
}

sq_status gemm_split_impl(const int8_t* xq, const float* x_scale, const int8_t* wq, const float* w_scale,
                          int64_t M, int64_t N, int64_t K, const float* x_out, const float* w_out, int64_t ld,
                          void* y, sq_dtype out_dt, void* workspace, size_t ws_bytes, cudaStream_t st) {
    if (out_dt != SQ_F32 && out_dt != SQ_BF16) {
        set_error("the decomposed GEMM writes SQ_F32 or SQ_BF16 outputs");
        return SQ_ERR_UNSUPPORTED;
    }
    if (ld < 0 || ld % 4 != 0 || ld > kMaxSplitLd) {
        set_error("ld=%lld must be a multiple of 4 in [0, %d]", (long long)ld, kMaxSplitLd);
        return SQ_ERR_UNSUPPORTED;
    }
    if (ld > 0 && M > 0 && N > 0) {
        if (!x_out || !w_out) { set_error("NULL outlier operand"); return SQ_ERR_INVALID_ARG; }
        if (!aligned16(x_out) || !aligned16(w_out)) {
            set_error("x_out and w_out must be 16-byte aligned");
            return SQ_ERR_UNSUPPORTED;
        }
    }
    SplitTerm sp;
    sp.x_out = x_out;
    sp.w_out = w_out;
    sp.ld = (int)ld;
    return gemm_dispatch(xq, x_scale, wq, w_scale, M, N, K, y, out_dt, workspace, ws_bytes, st, &sp);
}

}  // namespace sq

extern "C" {

size_t sq_w8a8_gemm_workspace_size(int64_t M, int64_t N, int64_t K) {
    return sq::gemm_workspace_size(M, N, K);
}

sq_status sq_w8a8_gemm(const int8_t* xq, const float* x_scale, const int8_t* wq, const float* w_scale,
                       int64_t M, int64_t N, int64_t K, void* y, sq_dtype out_dt, void* workspace,
                       size_t ws_bytes, sq_stream_t stream) {
    return sq::gemm_dispatch(xq, x_scale, wq, w_scale, M, N, K, y, out_dt, workspace, ws_bytes,
                             (cudaStream_t)stream, nullptr);
}

sq_status sq_w8a8_gemm_e4m3(const uint8_t* xq, const float* x_scale, const uint8_t* wq, const float* w_scale,
                            int64_t M, int64_t N, int64_t K, void* y, sq_dtype out_dt, sq_stream_t stream) {
    return sq::gemm_e4m3_impl(xq, x_scale, wq, w_scale, M, N, K, y, out_dt, (cudaStream_t)stream);
}

sq_status sq_w8a8_gemm_split(const int8_t* xq, const float* x_scale, const int8_t* wq, const float* w_scale,
                             int64_t M, int64_t N, int64_t K, const float* x_out, const float* w_out,
                             int64_t ld, void* y, sq_dtype out_dt, void* workspace, size_t ws_bytes,
                             sq_stream_t stream) {
    return sq::gemm_split_impl(xq, x_scale, wq, w_scale, M, N, K, x_out, w_out, ld, y, out_dt, workspace,
                               ws_bytes, (cudaStream_t)stream);
}

}  // extern "C"
