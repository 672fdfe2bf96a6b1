// sq_quant.cu -- the HBM-bound steps of the SmoothQuant W8A8 path on sm_100a:
//   a1  per-input-channel absmax calibration     (sq_calibrate_absmax)
//   a2  smoothing factors                        (sq_smooth_factors)
//   a3  weight fold + per-output-channel int8    (sq_fold_quant_weights)
//   a4  activation smoothing + per-token int8    (sq_smooth_quant_act)
//   RMSNorm with the folded gain + per-token int8 (sq_rmsnorm_quant_act)
//
// Exactness. Every value that decides an int8 code is one correctly rounded
// fp32 operation in the order the method defines it (explicit __fmul_rn /
// __fdiv_rn, never contracted), rounding to nearest-even, so the codes and
// scales are reproducible bit for bit on any IEEE implementation.
#include <cstdio>
#include <cuda_fp8.h>
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
constexpr int kAbsmaxRowsInFlight = 8;   // per warp (two batches); blocks cover multiples of 64 rows
constexpr int kAbsmaxBatch = 4;          // rows per warp per batch

// Two tensors in one launch (the activations and the weights of a layer share
// K): row-chunk blocks [0, rc1) read the first, the others the second.
struct AbsmaxPair {
    const uint8_t* x2 = nullptr;
    int64_t rows2 = 0, per2 = 0;
    float* absmax2 = nullptr;
    int rc1 = 0;   // 0: one tensor
};

// TENSOR = true: the per-tensor variant. Each column maximum is first divided
// by s_j (RN(max|x| / s_j) = max |RN(x / s_j)| for s_j > 0, because rounding
// is monotone), the block's columns are reduced to one value, and that value
// is merged into absmax[0].
template <typename T, bool TENSOR>
__global__ void __launch_bounds__(kAbsmaxThreads)
col_absmax_kernel(const uint8_t* __restrict__ x, int64_t rows, int64_t cols,
                  int64_t rows_per_chunk, float* __restrict__ absmax, const float* __restrict__ s,
                  const AbsmaxPair pair) {
    constexpr int VEC = Vec16<T>::N;
    constexpr int TILE = 32 * VEC;
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int64_t chunk = blockIdx.y;
    if (pair.rc1 > 0 && (int)blockIdx.y >= pair.rc1) {
        x = pair.x2;
        rows = pair.rows2;
        rows_per_chunk = pair.per2;
        absmax = pair.absmax2;
        chunk -= pair.rc1;
    }
    const int64_t col = (int64_t)blockIdx.x * TILE + lane * VEC;
    const int64_t r_begin = chunk * rows_per_chunk;
    const int64_t r_end = min(rows, r_begin + rows_per_chunk);
    const int64_t row_bytes = cols * (int64_t)sizeof(T);

    float m[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) m[i] = 0.0f;

    if (col < cols) {
        const uint8_t* p = x + col * (int64_t)sizeof(T);
        // Batches of kAbsmaxBatch rows per warp, double-buffered: the next
        // batch's loads are issued before the current one is reduced, so a
        // warp always has rows in flight.
        constexpr int B = kAbsmaxBatch;
        constexpr int64_t step = 8 * B;
        uint4 cur[B], nxt[B];
        int64_t r = r_begin + warp;
#pragma unroll
        for (int u = 0; u < B; ++u) {
            const int64_t rr = r + 8 * u;
            cur[u] = rr < r_end ? ld_stream_v4(p + rr * row_bytes) : make_uint4(0u, 0u, 0u, 0u);
        }
        for (; r < r_end; r += step) {
            const int64_t rn = r + step;
#pragma unroll
            for (int u = 0; u < B; ++u) {
                const int64_t rr = rn + 8 * u;
                nxt[u] = rr < r_end ? ld_stream_v4(p + rr * row_bytes) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < B; ++u) Vec16<T>::absmax(m, cur[u]);
#pragma unroll
            for (int u = 0; u < B; ++u) cur[u] = nxt[u];
        }
    }

    __shared__ float red[8][TILE];
#pragma unroll
    for (int i = 0; i < VEC; ++i) red[warp][lane * VEC + i] = m[i];
    __syncthreads();
    float bm = 0.0f;
    for (int c = threadIdx.x; c < TILE; c += kAbsmaxThreads) {
        float v = red[0][c];
#pragma unroll
        for (int w = 1; w < 8; ++w) v = fmaxf(v, red[w][c]);
        const int64_t gc = (int64_t)blockIdx.x * TILE + c;
        if (gc < cols) {
            if (TENSOR) bm = fmaxf(bm, s ? __fdiv_rn(v, s[gc]) : v);
            else atomicMax(reinterpret_cast<int*>(absmax + gc), __float_as_int(v));
        }
    }
    if (TENSOR) {
        __shared__ float bred[8];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
        if (lane == 0) bred[warp] = bm;
        __syncthreads();
        if (threadIdx.x == 0) {
            float v = bred[0];
#pragma unroll
            for (int w = 1; w < 8; ++w) v = fmaxf(v, bred[w]);
            atomicMax(reinterpret_cast<int*>(absmax), __float_as_int(v));
        }
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
    pdl_wait();
    pdl_trigger();
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
enum RowMode { kFold = 0, kSmooth = 1, kNorm = 2 };

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

// Code formats of the row quantizer: symmetric int8 ([-127, 127], scale =
// amax / 127) or FP8 E4M3 (scale = amax / 448, the quotient converted with
// round-to-nearest-even and saturation to +-448).
enum CodeFormat { kInt8 = 0, kE4M3 = 1 };

template <int FMT>
__device__ __forceinline__ uint32_t code8(float v, float scale) {
    if (FMT == kE4M3)
        return (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(v, scale), __NV_SATFINITE, __NV_E4M3);
    int q = __float2int_rn(__fdiv_rn(v, scale));
    q = max(-127, min(127, q));
    return static_cast<uint32_t>(q) & 0xffu;
}

template <typename T, int MODE, int TPB, int MAXC, int FMT>
__global__ void __launch_bounds__(TPB)
row_quant_kernel(const T* __restrict__ in, int64_t rows, int64_t K, const float* __restrict__ s,
                 int8_t* __restrict__ q, float* __restrict__ scale_out) {
    constexpr int NW = TPB / 32;
    __shared__ float red[2][NW];
    pdl_wait();
    pdl_trigger();
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
        const float scale = zero ? 1.0f : __fdiv_rn(amax, FMT == kE4M3 ? 448.0f : 127.0f);
        int8_t* rq = q + row * K;
#pragma unroll
        for (int i = 0; i < MAXC; ++i) {
            const int64_t c = tid + (int64_t)i * TPB;
            if (c < nchunks) {
                uint2 packed = make_uint2(0u, 0u);
                if (!zero) {
                    packed.x = code8<FMT>(v[i][0], scale) | (code8<FMT>(v[i][1], scale) << 8) |
                               (code8<FMT>(v[i][2], scale) << 16) | (code8<FMT>(v[i][3], scale) << 24);
                    packed.y = code8<FMT>(v[i][4], scale) | (code8<FMT>(v[i][5], scale) << 8) |
                               (code8<FMT>(v[i][6], scale) << 16) | (code8<FMT>(v[i][7], scale) << 24);
                }
                *reinterpret_cast<uint2*>(rq + c * 8) = packed;
            }
        }
        if (tid == 0) scale_out[row] = scale;
    }
}

// ============================================================== a3 / a4: fast exact path
// The same codes and scales as row_quant_kernel (bit for bit), with the
// per-element IEEE divisions replaced by cheaper arithmetic wherever that
// provably cannot change a result.
//
// Layout. One row is handled by a group of R warps (R = 1..16, chosen from K);
// a CTA holds several groups. Lane l of a group owns the 8-element chunks
// l, l + 32R, ... (at most CPL of them), kept in registers between the passes.
// Per CTA, the per-column multipliers m_j -- s_j (fold) or RN(1/s_j) (smooth,
// __frcp_rn) -- are staged once in shared memory as fp32 (two arrays holding
// elements 0-3 and 4-7 of every chunk, so 16-byte loads are contiguous across
// a warp) and, for bf16 inputs, rounded to bf16 pairs.
//
// Row maximum. Pass 1 approximates |v_j| (v_j = RN(x_j * s_j) or
// RN(x_j / s_j)): bf16x2 products x_j * bf16(m_j) reduced with a packed
// absolute max (relative error < 2^-7.9), or fp32 products for fp32 inputs.
// The group maximum m' of these bounds the exact maximum a within that error,
// so only elements of chunks whose approximate maximum is >= m'(1 - 2^-6) can
// attain a; their exact values (normally one chunk per row) reduced over the
// group give a exactly.
//
// Codes. With r = RN(1/scale), q' = RN(RN(x * m_j) * r) differs from
// q* = RN(v / scale) by less than 7 ulp of 127 (< 5.3e-5), so
// round-half-even(q') = round-half-even(q*) unless q' lies within that
// distance of a half-integer; a chunk with any q' within 2^-13 of one has
// those codes recomputed exactly. Rounding adds 1.5*2^23: the int8 code is the
// low byte of the sum's bits. |q'| < 127.5, so no code leaves [-127, 127].
// Pass 2 runs on packed fp32 pairs (mul/add/sub .f32x2).
//
// The error bounds are relative and need normal numbers: a row whose
// approximate maximum is below 2^-90 (this includes all-zero rows) is
// quantized entirely with exact divisions.
//
// kNorm (RMSNorm with the smoothing folded into its gain, m_j = g'_j): the
// row's factor r = RN32(1 / sqrt(sum x^2 / K + eps)) comes first, the sum of
// squares in fp64 (every square exact) reduced over the group, then
// 1/sqrt in correctly rounded fp64 operations. The norm output
// v_j = RN(RN(x_j * r) * g'_j) is an exact product chain, so the candidates
// and codes follow the fold argument with r as a common positive factor
// (pass 2 forms q' = RN(v_j * RN(1/scale)), within 4 ulp of q*).
constexpr float kMagic = 12582912.0f;            // 1.5 * 2^23
constexpr float kTieGuard = 1.0f / 8192.0f;      // >> 5.3e-5, the bound on |q' - q*|
constexpr float kCandidate = 1.0f - 1.0f / 64.0f;
constexpr float kSmallRow = 8.077935669463161e-28f;  // 2^-90
constexpr int kFastMaxThreads = 512;
constexpr int64_t kFastMaxK = 32768;             // multipliers in shared memory: 6 bytes per column
// Chunks of 8 elements each lane keeps in registers: 8 for bf16 (32 registers), 4 for fp32.
template <typename T> struct RowFastCPL { static constexpr int value = 8; };
template <> struct RowFastCPL<float> { static constexpr int value = 4; };

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
    return d;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint32_t bf2_mul(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
// Packed max of magnitudes (the sign bits of the result are not used).
__device__ __forceinline__ uint32_t bf2_maxabs(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

template <typename T>
struct RawChunk;
template <>
struct RawChunk<__nv_bfloat16> {
    uint4 a;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { a = ld_stream_v4(p); }
    __device__ __forceinline__ uint32_t word(int w) const { return w == 0 ? a.x : w == 1 ? a.y : w == 2 ? a.z : a.w; }
    __device__ __forceinline__ float get(int e) const {
        const uint32_t w = word(e >> 1);
        return (e & 1) ? bf16_hi(w) : bf16_lo(w);
    }
    // elements (2p, 2p+1) as an fp32 pair
    __device__ __forceinline__ uint64_t pair(int p) const {
        const uint32_t w = word(p);
        return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
    // approximate max |x_e * m_e| over the chunk (bf16 arithmetic)
    __device__ __forceinline__ float approx_max(const uint4& m16, const float (&)[8]) const {
        const uint32_t p = bf2_maxabs(bf2_maxabs(bf2_mul(a.x, m16.x), bf2_mul(a.y, m16.y)),
                                      bf2_maxabs(bf2_mul(a.z, m16.z), bf2_mul(a.w, m16.w)));
        return fmaxf(fabsf(bf16_lo(p)), fabsf(bf16_hi(p)));
    }
};
template <>
struct RawChunk<float> {
    uint4 a, b;
    __device__ __forceinline__ void load(const float* p) {
        a = ld_stream_v4(p);
        b = ld_stream_v4(p + 4);
    }
    __device__ __forceinline__ float get(int e) const {
        const uint32_t w = e == 0 ? a.x : e == 1 ? a.y : e == 2 ? a.z : e == 3 ? a.w
                         : e == 4 ? b.x : e == 5 ? b.y : e == 6 ? b.z : b.w;
        return __uint_as_float(w);
    }
    __device__ __forceinline__ uint64_t pair(int p) const { return f2_pack(get(2 * p), get(2 * p + 1)); }
    __device__ __forceinline__ float approx_max(const uint4&, const float (&mv)[8]) const {
        float v = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) v = fmaxf(v, fabsf(__fmul_rn(get(e), mv[e])));
        return v;
    }
};

// Exact code of one element, x the raw input: clamp(round_half_even(RN(v /
// scale)), -127, 127) with v = RN(x * s_j) (fold) or RN(x / s_j) (smooth).
// Out of line: these run only on the rare near-tie and small-row paths.
template <int MODE>
__device__ __forceinline__ float exact_value(float x, float m_j, float r) {
    if (MODE == kFold) return __fmul_rn(x, m_j);
    if (MODE == kSmooth) return __fdiv_rn(x, m_j);
    return __fmul_rn(__fmul_rn(x, r), m_j);
}

template <int MODE>
__device__ __noinline__ uint32_t exact_code(float x, float s_j, float scale, float r) {
    const float v = exact_value<MODE>(x, s_j, r);
    int qi = __float2int_rn(__fdiv_rn(v, scale));
    qi = max(-127, min(127, qi));
    return (uint32_t)qi & 0xffu;
}

// The int8 code clamp(round_half_even(RN(v / scale)), -127, 127) of an exact
// value v whose true quotient Q = v / scale lies within 2^-12 of the
// half-integer h = floor(p) + 1/2, p an approximate quotient, without a
// division. (The callers pass p = RN(v * RN(1 / scale)), within 1.6e-5 of Q,
// for elements whose fast quotient their near-tie test put within 2^-13 of h;
// that fast quotient is within 3.8e-5 of Q, so |Q - h| <= 1.6e-4 < 2^-12.)
// Then v - h * scale is a multiple of 2^(e - 25) (e the exponent of scale; h a
// multiple of 1/2, v no finer) below 2^(e - 11) in magnitude: exact in one
// fused multiply-add, and its sign places Q against h. RN(Q) = h exactly when
// |Q - h| <= ulp(h) / 2, i.e.
// when |v - h * scale| <= scale * ulp(h) / 2 (a product with a power of two,
// exact); the equal case belongs to h because h, a multiple of 1/2 below 2^23,
// has an even significand. A quotient that rounds to h takes h's even
// neighbour (round half to even); any other lies strictly between h and the
// integer on Q's side, which is its code. Requires scale >= 2^-100 (the
// kernels send rows with smaller maxima to the exact path).
__device__ __forceinline__ uint32_t near_tie_code(float v, float scale, float p) {
    const int lo = __float2int_rd(p);
    const float h = __fadd_rn((float)lo, 0.5f);
    const float res = __fmaf_rn(-h, scale, v);
    const uint32_t eh = (__float_as_uint(h) >> 23) & 0xffu;         // |h| >= 1/2: a normal number
    const float bound = __fmul_rn(scale, __uint_as_float((eh - 24u) << 23));   // scale * ulp(h) / 2
    int code = fabsf(res) <= bound ? lo + (lo & 1) : (res > 0.0f ? lo + 1 : lo);
    code = max(-127, min(127, code));
    return (uint32_t)code & 0xffu;
}

// The code of one element in either format (int8: as exact_code; E4M3: the
// IEEE quotient converted with round-to-nearest-even and saturation).
template <int MODE, int FMT>
__device__ __noinline__ uint32_t exact_code_fmt(float x, float s_j, float scale, float r) {
    return code8<FMT>(exact_value<MODE>(x, s_j, r), scale);
}

// |v| of one element, exactly (v as above).
template <int MODE>
__device__ __noinline__ float exact_abs(float x, float s_j, float r) {
    return fabsf(exact_value<MODE>(x, s_j, r));
}

// Sum over the R warps of a group, in fp64 (same slot scheme as group_max).
template <int R>
__device__ __forceinline__ double group_sum(double v, double* red, int grp, int wig, int lane, int bank) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (R == 1) return v;
    double* slot = red + (grp * 2 + bank) * R;
    if (lane == 0) slot[wig] = v;
    asm volatile("bar.sync %0, %1;" :: "r"(1 + grp), "r"(32 * R) : "memory");
    v = slot[0];
#pragma unroll
    for (int w = 1; w < R; ++w) v += slot[w];
    return v;
}

// Maximum over the R <= 32 warps of a group. Every value is non-negative and
// not NaN (maxima of |v| started from +0 with NaN-dropping max), so the bit
// patterns order as the values do and integer warp reductions give the
// maximum: one per warp, one slot per warp in shared memory, a named barrier,
// one over the R slots.
template <int R>
__device__ __forceinline__ float group_max(float v, float* red, int grp, int wig, int lane, int bank) {
    static_assert(R >= 1 && R <= 32, "one slot per lane");
    uint32_t u = __reduce_max_sync(0xffffffffu, __float_as_uint(v));
    if (R == 1) return __uint_as_float(u);
    uint32_t* slot = reinterpret_cast<uint32_t*>(red) + (grp * 2 + bank) * R;
    if (lane == 0) slot[wig] = u;
    asm volatile("bar.sync %0, %1;" :: "r"(1 + grp), "r"(32 * R) : "memory");
    u = lane < R ? slot[lane] : 0u;
    return __uint_as_float(__reduce_max_sync(0xffffffffu, u));
}

// The rarely taken paths of the row kernel. Kernels that keep one row in
// registers call them out of line (the hot loop stays small in the
// instruction cache); kernels that also hold the next row (PF) inline them, as
// a call would make the live prefetch registers spill. A chunk is passed by value.

// max_e |v_e| of one chunk, every value exact.
template <typename T, int MODE>
__device__ __forceinline__ float exact_chunk_max_in(const RawChunk<T>& ch, const float* __restrict__ s8, float rn) {
    float ex = 0.0f;
#pragma unroll
    for (int e = 0; e < 8; ++e) ex = fmaxf(ex, exact_abs<MODE>(ch.get(e), __ldg(s8 + e), rn));
    return ex;
}
template <typename T, int MODE>
__device__ __noinline__ float exact_chunk_max_out(const RawChunk<T> ch, const float* __restrict__ s8, float rn) {
    return exact_chunk_max_in<T, MODE>(ch, s8, rn);
}

// Exact codes of one chunk, packed 8 per uint2 (zero codes for a zero scale).
template <typename T, int MODE>
__device__ __forceinline__ uint2 exact_chunk_codes_in(const RawChunk<T>& ch, const float* __restrict__ s8, float scale,
                                                      float rn, bool zero) {
    uint32_t b[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) b[e] = zero ? 0u : exact_code<MODE>(ch.get(e), __ldg(s8 + e), scale, rn);
    return make_uint2(b[0] | b[1] << 8 | b[2] << 16 | b[3] << 24, b[4] | b[5] << 8 | b[6] << 16 | b[7] << 24);
}
template <typename T, int MODE>
__device__ __noinline__ uint2 exact_chunk_codes_out(const RawChunk<T> ch, const float* __restrict__ s8, float scale,
                                                    float rn, bool zero) {
    return exact_chunk_codes_in<T, MODE>(ch, s8, scale, rn, zero);
}

// Near-tie repair of one chunk's packed codes: every element whose fast
// quotient lies within the guard of a half-integer gets its exact code.
template <typename T, int MODE>
__device__ __forceinline__ uint2 fix_near_ties_in(const RawChunk<T>& ch, uint2 codes, const float* __restrict__ m_lo,
                                                  const float* __restrict__ m_hi, const float* __restrict__ s8, float r,
                                                  float rn, float scale) {
    const float4 a = *reinterpret_cast<const float4*>(m_lo);
    const float4 b = *reinterpret_cast<const float4*>(m_hi);
    const float mv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float xe = MODE == kNorm ? __fmul_rn(ch.get(e), rn) : ch.get(e);
        const float ve = __fmul_rn(xe, mv[e]);   // exact v for fold and norm
        const float qv = __fmul_rn(ve, r);
        const float d = __fsub_rn(qv, __fsub_rn(__fadd_rn(qv, kMagic), kMagic));
        if (fabsf(d) >= 0.5f - kTieGuard) {
            // smooth: the exact value takes a division; its quotient stays
            // within 2^-12 of the same half-step (v' is within 3 * 2^-24 |v| of v)
            const float vx = MODE == kSmooth ? __fdiv_rn(ch.get(e), __ldg(s8 + e)) : ve;
            const uint32_t code = near_tie_code(vx, scale, MODE == kSmooth ? __fmul_rn(vx, r) : qv);
            const int sh = 8 * (e & 3);
            uint32_t& w = (e < 4) ? codes.x : codes.y;
            w = (w & ~(0xffu << sh)) | (code << sh);
        }
    }
    return codes;
}
template <typename T, int MODE>
__device__ __noinline__ uint2 fix_near_ties_out(const RawChunk<T> ch, uint2 codes, const float* __restrict__ m_lo,
                                                const float* __restrict__ m_hi, const float* __restrict__ s8, float r,
                                                float rn, float scale) {
    return fix_near_ties_in<T, MODE>(ch, codes, m_lo, m_hi, s8, r, rn, scale);
}

template <typename T, int MODE, bool OUT>
__device__ __forceinline__ float exact_chunk_max(const RawChunk<T>& ch, const float* s8, float rn) {
    if constexpr (OUT) return exact_chunk_max_out<T, MODE>(ch, s8, rn);
    else return exact_chunk_max_in<T, MODE>(ch, s8, rn);
}
template <typename T, int MODE, bool OUT>
__device__ __forceinline__ uint2 exact_chunk_codes(const RawChunk<T>& ch, const float* s8, float scale, float rn,
                                                   bool zero) {
    if constexpr (OUT) return exact_chunk_codes_out<T, MODE>(ch, s8, scale, rn, zero);
    else return exact_chunk_codes_in<T, MODE>(ch, s8, scale, rn, zero);
}
template <typename T, int MODE, bool OUT>
__device__ __forceinline__ uint2 fix_near_ties(const RawChunk<T>& ch, uint2 codes, const float* m_lo, const float* m_hi,
                                               const float* s8, float r, float rn, float scale) {
    if constexpr (OUT) return fix_near_ties_out<T, MODE>(ch, codes, m_lo, m_hi, s8, r, rn, scale);
    else return fix_near_ties_in<T, MODE>(ch, codes, m_lo, m_hi, s8, r, rn, scale);
}

template <int R>
constexpr int row_fast_threads() { return 32 * R > 256 ? 32 * R : 256; }

// PF: double-buffer the row in registers (the next row's loads are issued
// before the current row is processed).
template <typename T, int MODE, int R, int CPL, bool PF>
__global__ void __launch_bounds__(row_fast_threads<R>(), R >= 16 ? 1 : (R >= 8 ? 2 : 4))
row_quant_fast_kernel(const T* __restrict__ in, int64_t rows, int64_t K, const float* __restrict__ s,
                      int8_t* __restrict__ q, float* __restrict__ scale_out, float eps,
                      float* __restrict__ r_out) {
    extern __shared__ float smem[];
    const int64_t nchunks = K >> 3;
    float* mul_lo = smem;                                                // [nchunks][4] fp32, elements 0..3
    float* mul_hi = smem + nchunks * 4;                                  // [nchunks][4] fp32, elements 4..7
    uint32_t* mul16 = reinterpret_cast<uint32_t*>(smem + nchunks * 8);   // [nchunks][4] bf16 pairs
    float* red = smem + nchunks * 12;                                    // [groups][2][R]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int groups = blockDim.x / (32 * R);
    double* red64 = reinterpret_cast<double*>(red + groups * 2 * R);     // [groups][2][R] (kNorm)
    const int grp = warp / R, wig = warp % R;
    const int gl = wig * 32 + lane;          // lane index inside the group

    pdl_wait();
    pdl_trigger();
    for (int64_t c = threadIdx.x; c < nchunks; c += blockDim.x) {
        float4 a = __ldg(reinterpret_cast<const float4*>(s + c * 8));
        float4 b = __ldg(reinterpret_cast<const float4*>(s + c * 8 + 4));
        if (MODE == kSmooth) {
            a = make_float4(__frcp_rn(a.x), __frcp_rn(a.y), __frcp_rn(a.z), __frcp_rn(a.w));
            b = make_float4(__frcp_rn(b.x), __frcp_rn(b.y), __frcp_rn(b.z), __frcp_rn(b.w));
        }
        *reinterpret_cast<float4*>(mul_lo + c * 4) = a;
        *reinterpret_cast<float4*>(mul_hi + c * 4) = b;
        *reinterpret_cast<uint4*>(mul16 + c * 4) =
            make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
    }
    __syncthreads();

    const uint64_t mag2 = f2_pack(kMagic, kMagic);
    int bank = 0, bank64 = 0;
    constexpr bool kPrefetch = PF;
    const int64_t stride = (int64_t)gridDim.x * groups;
    RawChunk<T> nxt[CPL];
    if (kPrefetch) {
        const int64_t row = (int64_t)blockIdx.x * groups + grp;
        if (row < rows) {
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const int64_t c = gl + (int64_t)i * 32 * R;
                if (c < nchunks) nxt[i].load(in + row * K + c * 8);
            }
        }
    }
    for (int64_t row = (int64_t)blockIdx.x * groups + grp; row < rows; row += stride) {
        const T* rin = in + row * K;
        RawChunk<T> raw[CPL];
        if (kPrefetch) {
#pragma unroll
            for (int i = 0; i < CPL; ++i) raw[i] = nxt[i];
            if (row + stride < rows) {
#pragma unroll
                for (int i = 0; i < CPL; ++i) {
                    const int64_t c = gl + (int64_t)i * 32 * R;
                    if (c < nchunks) nxt[i].load(in + (row + stride) * K + c * 8);
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const int64_t c = gl + (int64_t)i * 32 * R;
                if (c < nchunks) raw[i].load(rin + c * 8);
            }
        }

        // ---- RMSNorm factor of the row
        float rn = 1.0f;
        if (MODE == kNorm) {
            double ss = 0.0;
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const int64_t c = gl + (int64_t)i * 32 * R;
                if (c < nchunks) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const double v = (double)raw[i].get(e);
                        ss = __fma_rn(v, v, ss);
                    }
                }
            }
            ss = group_sum<R>(ss, red64, grp, wig, lane, bank64);
            bank64 ^= 1;
            rn = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(ss, (double)K), (double)eps))));
            if (r_out != nullptr && gl == 0) r_out[row] = rn;
        }

        // ---- pass 1: approximate chunk maxima
        float cm[CPL];
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int64_t c = gl + (int64_t)i * 32 * R;
            cm[i] = 0.0f;
            if (c < nchunks) {
                float mv[8];
                if (sizeof(T) == 4) {
                    const float4 a = *reinterpret_cast<const float4*>(mul_lo + c * 4);
                    const float4 b = *reinterpret_cast<const float4*>(mul_hi + c * 4);
                    mv[0] = a.x; mv[1] = a.y; mv[2] = a.z; mv[3] = a.w;
                    mv[4] = b.x; mv[5] = b.y; mv[6] = b.z; mv[7] = b.w;
                }
                const uint4 m16 = sizeof(T) == 2 ? *reinterpret_cast<const uint4*>(mul16 + c * 4) : make_uint4(0u, 0u, 0u, 0u);
                cm[i] = raw[i].approx_max(m16, mv);
                m = fmaxf(m, cm[i]);
            }
        }
        const float mrow = group_max<R>(m, red, grp, wig, lane, bank);
        bank ^= 1;
        int8_t* rq = q + row * K;

        if (!((MODE == kNorm ? __fmul_rn(mrow, rn) : mrow) >= kSmallRow)) {
            // zero, tiny or near-underflow row: exact maximum and codes
            float ex = 0.0f;
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const int64_t c = gl + (int64_t)i * 32 * R;
                if (c < nchunks) ex = fmaxf(ex, exact_chunk_max<T, MODE, !PF>(raw[i], s + c * 8, rn));
            }
            const float a = group_max<R>(ex, red, grp, wig, lane, bank);
            bank ^= 1;
            const float scale = a == 0.0f ? 1.0f : __fdiv_rn(a, 127.0f);
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const int64_t c = gl + (int64_t)i * 32 * R;
                if (c < nchunks)
                    *reinterpret_cast<uint2*>(rq + c * 8) = exact_chunk_codes<T, MODE, !PF>(raw[i], s + c * 8, scale, rn,
                                                                                     a == 0.0f);
            }
            if (gl == 0) scale_out[row] = scale;
            continue;
        }

        // exact values of the candidates (normally one chunk per row)
        const float tau = __fmul_rn(mrow, kCandidate);
        float ex = 0.0f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            if (cm[i] >= tau) {
                const int64_t c = gl + (int64_t)i * 32 * R;
                ex = fmaxf(ex, exact_chunk_max<T, MODE, !PF>(raw[i], s + c * 8, rn));
            }
        }
        const float amax = group_max<R>(ex, red, grp, wig, lane, bank);
        bank ^= 1;

        // ---- pass 2: codes
        const float scale = __fdiv_rn(amax, 127.0f);
        const float r = __frcp_rn(scale);
        const uint64_t r2 = f2_pack(r, r);
        const uint64_t rn2 = f2_pack(rn, rn);
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int64_t c = gl + (int64_t)i * 32 * R;
            if (c < nchunks) {
                const float4 a = *reinterpret_cast<const float4*>(mul_lo + c * 4);
                const float4 b = *reinterpret_cast<const float4*>(mul_hi + c * 4);
                const uint64_t mp[4] = {f2_pack(a.x, a.y), f2_pack(a.z, a.w), f2_pack(b.x, b.y), f2_pack(b.z, b.w)};
                uint32_t t[8];
                bool near_tie = false;
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const uint64_t x2 = MODE == kNorm ? f2_mul(raw[i].pair(p), rn2) : raw[i].pair(p);
                    const uint64_t q2 = f2_mul(f2_mul(x2, mp[p]), r2);
                    const uint64_t t2 = f2_add(q2, mag2);
                    const uint64_t d2 = f2_sub(q2, f2_sub(t2, mag2));
                    float t0, t1, d0, d1;
                    f2_unpack(t2, t0, t1);
                    f2_unpack(d2, d0, d1);
                    t[2 * p] = __float_as_uint(t0);
                    t[2 * p + 1] = __float_as_uint(t1);
                    near_tie |= fabsf(d0) >= 0.5f - kTieGuard;
                    near_tie |= fabsf(d1) >= 0.5f - kTieGuard;
                }
                uint2 codes;
                codes.x = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410);
                codes.y = __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410);
                if (near_tie)
                    codes = fix_near_ties<T, MODE, !PF>(raw[i], codes, mul_lo + c * 4, mul_hi + c * 4, s + c * 8, r, rn, scale);
                *reinterpret_cast<uint2*>(rq + c * 8) = codes;
            }
        }
        if (gl == 0) scale_out[row] = scale;
    }
}

// ============================================================== the streamed row kernel (bf16)
// bf16 rows of 2064 to 28672 elements. One CTA of 16 warps per SM, in groups
// of R warps; a group quantizes one row at a time, lane l of the group owning
// the 8-element chunks l, l + 32R, ... (CPL of them: the row is padded with
// zeros to 32 R CPL chunks, so the unrolled loops need no bounds checks and
// only the stores are predicated). Rows reach shared memory through a ring of
// ns slots per group (two in practice), each filled by one bulk copy
// (cp.async.bulk, its bytes counted on the slot's mbarrier) that the group's
// first lane issues ns - 1 rows ahead. DRAM latency is hidden without a second
// row in registers, and the registers hold the row's values instead:
//   fold   v_j = RN(x_j * s_j)                  exact
//   norm   v_j = RN(RN(x_j * r_t) * g'_j)       exact
//   smooth v'_j = RN(x_j * RN(1/s_j))           within 3 * 2^-24 |v_j| of v_j = RN(x_j / s_j)
// formed once (pass 1) as fp32 pairs. The row maximum is therefore exact for
// fold and norm. For smooth, the elements with |v'_j| >= m'(1 - 2^-20) (m' the
// maximum of the |v'|) get their exact value from an IEEE division; the true
// maximum is always among them, since m' <= a(1 + 3 * 2^-24) and the element
// attaining a has |v'| >= a(1 - 3 * 2^-24). (Resolving candidates against
// each lane's own maximum instead saves the second group reduction but puts an
// IEEE division in every lane: measured slower, 20.5 -> 22.5 us at K = 4096;
// against each warp's own maximum, one division per warp, it measured no
// faster at K = 28672: fewer barrier waits, 15% more instructions.)
//
// Codes (pass 2): with r = RN(1/scale), t = RN(v * r + 1.5 * 2^23) holds
// k = round-half-even(v * r) in its low mantissa bits, and d = RN(v * r - k)
// is the distance to it. v * r (one rounding, inside the fused multiply-add)
// is within 1.2e-5 of q* = RN(v / scale) for exact v and within 3.5e-5 for
// smooth's v', so k is the code of q* unless |d| >= 0.5 - 2^-13. Such elements
// (about one per 4096) get the IEEE-division code after their chunk's store,
// recomputed from the copy of the row still in shared memory; chunks needing
// exact work are collected in a bit mask, so the rare paths stay out of the
// unrolled loops. Rows whose maximum is below 2^-90 (all-zero rows included)
// are quantized entirely with exact divisions, as in the register kernel.
constexpr int kRingThreads = 512;
constexpr int kRingCPL = 8;
constexpr size_t kRingSmemMax = 231424;   // dynamic shared memory of one CTA (226 KB of the 227 KB opt-in)
constexpr float kRingCandidate = 1.0f - 1.0f / 1048576.0f;
// Near-tie guards of the streamed kernel. Its fast quotient is v' * r taken
// exactly inside the fused multiply-add (r = RN(1/scale)); against q* = RN(v /
// scale), |q| <= 127.5:
//   |v' r - q*| <= |v' - v| r + |v| |r - 1/scale| + ulp(q*) / 2
//              <= 3 * 2^-24 * 127.5 + 2^-24 * 127.5 + 2^-18 = 3.4e-5  (smooth: v' within 3 * 2^-24 |v|)
//              <= 2^-24 * 127.5 + 2^-18 = 1.2e-5                      (fold, norm: v exact)
// An element farther than the guard from a half-step has q* on the same side.
constexpr float kRingGuardExact = 1.0f / 32768.0f;    // 3.05e-5
constexpr float kRingGuardSmooth = 1.0f / 16384.0f;   // 6.1e-5

// Bring the 128-byte line holding p into L1 ahead of a load on a rare path
// (the smoothing kernel's near-tie repair reads s_j, which no shared-memory
// table holds; the same prefetch for the maximum's candidates, issued before the
// group reduction, measured slower: 190 -> 225 us at K = 28672).
__device__ __forceinline__ void prefetch_l1(const void* p) {
    asm volatile("{\n\t.reg .u64 a;\n\tcvta.to.global.u64 a, %0;\n\tprefetch.global.L1 [a];\n\t}" :: "l"(p));
}

__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :: "r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ float bf16_elem(const uint4& w, int e) {
    const uint32_t u = e < 2 ? w.x : e < 4 ? w.y : e < 6 ? w.z : w.w;
    return (e & 1) ? bf16_hi(u) : bf16_lo(u);
}

// Elements (2p, 2p+1) of a 16-byte bf16 chunk as an fp32 pair.
__device__ __forceinline__ uint64_t bf16_pair(const uint4& w, int p) {
    const uint32_t u = p == 0 ? w.x : p == 1 ? w.y : p == 2 ? w.z : w.w;
    return f2_pack(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

// The R warps of a group agree on `ok`: a named barrier with an AND reduction.
template <int R>
__device__ __forceinline__ bool group_all(bool ok, int grp) {
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
                 "bar.red.and.pred p, %2, %3, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(r) : "r"((uint32_t)ok), "r"(1 + grp), "r"(32 * R) : "memory");
    return r != 0;
}

// The second tensor of a pair launch (the activations, smoothed), quantized in
// the same launch as the weights: its rows follow the first tensor's.
struct RingPair {
    const __nv_bfloat16* in2 = nullptr;
    int64_t rows2 = 0;
    int8_t* q2 = nullptr;
    float* scale2 = nullptr;
};

template <int MODE, int R, int CPL, bool FULL, bool PAIR, int FMT>
__global__ void __launch_bounds__(kRingThreads, 1)
row_quant_ring_kernel(const __nv_bfloat16* __restrict__ in, int64_t rows, int64_t K, const float* __restrict__ s,
                      int8_t* __restrict__ q, float* __restrict__ scale_out, float eps, float* __restrict__ r_out,
                      int ns, long long wait_limit, RingPair pr) {
    static_assert(!PAIR || MODE == kFold, "the pair launch folds its first tensor and smooths its second");
    static_assert(FMT == kInt8 || MODE != kNorm, "E4M3 codes for the fold and smoothing modes");
    constexpr float kQmax = FMT == kE4M3 ? 448.0f : 127.0f;   // scale = amax / kQmax
    constexpr int G = kRingThreads / (32 * R);   // groups per CTA
    constexpr int NCP = 32 * R * CPL;            // chunks of a row padded to whole lanes
    constexpr uint32_t SLOT = NCP * 16u;         // bytes of one ring slot
    extern __shared__ __align__(128) uint8_t ring_smem[];
    const int64_t nchunks = K >> 3;
    const int nch = FULL ? NCP : (int)nchunks;   // FULL: the row fills every lane's CPL chunks
    const uint32_t row_bytes = (uint32_t)K * 2u;
    float* mul_lo = reinterpret_cast<float*>(ring_smem);         // [NCP][4]: m_j of elements 0..3
    float* mul_hi = mul_lo + NCP * 4;                            // [NCP][4]: elements 4..7
    float* mul2_lo = mul_hi + NCP * 4;                           // PAIR: RN(1/s_j) for the second tensor
    float* mul2_hi = mul2_lo + NCP * 4;
    uint8_t* slots = ring_smem + NCP * (PAIR ? 64 : 32);         // [G][ns][SLOT]
    uint64_t* bars = reinterpret_cast<uint64_t*>(slots + (size_t)G * ns * SLOT);   // [G][ns]
    float* red = reinterpret_cast<float*>(bars + G * ns);        // [G][2][R]
    double* red64 = reinterpret_cast<double*>(red + G * 2 * R);  // [G][2][R]
    __shared__ int abort_sh, never_sh;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = warp / R, wig = warp % R;
    const int gl = wig * 32 + lane;
    uint8_t* my_slots = slots + (size_t)grp * ns * SLOT;
    const uint32_t bar0 = smem_u32(bars + grp * ns);

    if (threadIdx.x == 0) {
        for (int i = 0; i < G * ns; ++i) mbar_init(smem_u32(bars + i), 1);
        abort_sh = 0;
        never_sh = 0;
        fence_barrier_init();
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();

    // rows [0, rows) of the first tensor, then (PAIR) rows [rows, total) of the second
    const int64_t total = rows + (PAIR ? pr.rows2 : 0);
    auto row_src = [&](int64_t g) {
        return (PAIR && g >= rows) ? pr.in2 + (g - rows) * K : in + g * K;
    };
    const int64_t stride = (int64_t)gridDim.x * G;
    const int64_t row0 = (int64_t)blockIdx.x * G + grp;
    int issued = 0;   // copies this group has issued (rows row0 + j * stride, j < issued)
    if (gl == 0) {
        for (int j = 0; j < ns; ++j) {
            const int64_t row = row0 + (int64_t)j * stride;
            if (row < total) {
                mbar_arrive_expect_tx(bar0 + 8u * j, row_bytes);
                bulk_copy_g2s(smem_u32(my_slots + (size_t)j * SLOT), row_src(row), row_bytes, bar0 + 8u * j);
                ++issued;
            }
        }
    }
    // multipliers, zero past the row's end; the slots' padding (never
    // written by a copy) is zeroed once, so every lane handles CPL chunks
    // without bounds checks and the padding adds nothing to any maximum
    for (int c = threadIdx.x; c < NCP; c += kRingThreads) {
        float4 a = make_float4(0.0f, 0.0f, 0.0f, 0.0f), b = a;
        if (c < nch) {
            a = __ldg(reinterpret_cast<const float4*>(s + c * 8));
            b = __ldg(reinterpret_cast<const float4*>(s + c * 8 + 4));
        }
        if (MODE == kSmooth && c < nch) {
            a = make_float4(__frcp_rn(a.x), __frcp_rn(a.y), __frcp_rn(a.z), __frcp_rn(a.w));
            b = make_float4(__frcp_rn(b.x), __frcp_rn(b.y), __frcp_rn(b.z), __frcp_rn(b.w));
        }
        *reinterpret_cast<float4*>(mul_lo + c * 4) = a;
        *reinterpret_cast<float4*>(mul_hi + c * 4) = b;
        if (PAIR) {
            if (c < nch) {
                a = make_float4(__frcp_rn(a.x), __frcp_rn(a.y), __frcp_rn(a.z), __frcp_rn(a.w));
                b = make_float4(__frcp_rn(b.x), __frcp_rn(b.y), __frcp_rn(b.z), __frcp_rn(b.w));
            }
            *reinterpret_cast<float4*>(mul2_lo + c * 4) = a;
            *reinterpret_cast<float4*>(mul2_hi + c * 4) = b;
        }
    }
    {
        const int tail = (int)((SLOT - row_bytes) / 16u);
        for (int i = threadIdx.x; i < G * ns * tail; i += kRingThreads)
            *reinterpret_cast<uint4*>(slots + (size_t)(i / tail) * SLOT + row_bytes + (size_t)(i % tail) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();

    const uint64_t mag2 = f2_pack(kMagic, kMagic);
    int bank = 0, bank64 = 0;
    int it = 0, sl = 0, ps = ns - 1;   // iteration, its slot, the previous iteration's slot
    uint32_t parity = 0;
    bool failed = false;
    // One smoothing near-tie per lane is carried to the next row: its s_j load
    // (global memory; no shared-memory table holds s_j) is issued when the tie
    // is found and consumed a row later, off the group's barrier path.
    bool pend = false;
    float pend_x = 0.0f, pend_s = 1.0f, pend_scale = 1.0f, pend_r = 1.0f;
    int8_t* pend_q = nullptr;
    auto settle = [&]() {
        if (FMT == kInt8 && pend) {
            const float vx = __fdiv_rn(pend_x, pend_s);
            *pend_q = (int8_t)near_tie_code(vx, pend_scale, __fmul_rn(vx, pend_r));
            pend = false;
        }
    };
    for (int64_t g = row0; g < total; g += stride, ++it) {
        // this row's tensor: the first (MODE), or the second (smoothed) of a pair
        const bool second = PAIR && g >= rows;
        const bool smooth = MODE == kSmooth || second;
        const int64_t row = second ? g - rows : g;
        int8_t* const qo = second ? pr.q2 : q;
        float* const so = second ? pr.scale2 : scale_out;
        const float* const mlo = second ? mul2_lo : mul_lo;
        const float* const mhi = second ? mul2_hi : mul_hi;
        const bool ok = mbar_wait_sleep(bar0 + 8u * sl, parity, wait_limit, &abort_sh, SITE_QUANT_WAIT);
        __syncwarp();   // the barrier below is warp-aligned
        if (!group_all<R>(ok, grp)) {
            failed = true;
            break;
        }
        // every warp of the group is done with the previous row's slot: refill it
        if (it > 0 && gl == 0) {
            const int64_t nr = g + (int64_t)(ns - 1) * stride;
            if (nr < total) {
                mbar_arrive_expect_tx(bar0 + 8u * ps, row_bytes);
                bulk_copy_g2s(smem_u32(my_slots + (size_t)ps * SLOT), row_src(nr), row_bytes, bar0 + 8u * ps);
                ++issued;
            }
        }
        const uint8_t* src = my_slots + (size_t)sl * SLOT;
        ps = sl;
        if (++sl == ns) {
            sl = 0;
            parity ^= 1u;
        }

        // ---- RMSNorm factor of the row (sum of squares in fp64, every square exact)
        float rn = 1.0f;
        if (MODE == kNorm) {
            double ss = 0.0;
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const int c = gl + i * 32 * R;
                const uint4 w = *reinterpret_cast<const uint4*>(src + c * 16);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const double v = (double)bf16_elem(w, e);
                    ss = __fma_rn(v, v, ss);
                }
            }
            ss = group_sum<R>(ss, red64, grp, wig, lane, bank64);
            bank64 ^= 1;
            rn = __double2float_rn(__ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(ss, (double)K), (double)eps))));
            if (r_out != nullptr && gl == 0) r_out[row] = rn;
        }
        const uint64_t rn2 = f2_pack(rn, rn);

        // ---- pass 1: the values, kept in registers, and their maximum
        uint64_t v2[CPL][4];
        float cm[CPL];
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int c = gl + i * 32 * R;
            const uint4 w = *reinterpret_cast<const uint4*>(src + c * 16);
            const float4 a = *reinterpret_cast<const float4*>(mlo + c * 4);
            const float4 b = *reinterpret_cast<const float4*>(mhi + c * 4);
            const uint64_t mp[4] = {f2_pack(a.x, a.y), f2_pack(a.z, a.w), f2_pack(b.x, b.y), f2_pack(b.z, b.w)};
            float cmax = 0.0f;
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                uint64_t x2 = bf16_pair(w, p);
                if (MODE == kNorm) x2 = f2_mul(x2, rn2);
                v2[i][p] = f2_mul(x2, mp[p]);
                float lo, hi;
                f2_unpack(v2[i][p], lo, hi);
                cmax = fmax3(cmax, fabsf(lo), fabsf(hi));
            }
            cm[i] = cmax;
            m = fmaxf(m, cmax);
        }
        settle();   // the previous row's carried repair, its load long done
        float amax = group_max<R>(m, red, grp, wig, lane, bank);
        bank ^= 1;
        int8_t* rq = qo + row * K;

        if (!(amax >= kSmallRow)) {
            // zero, tiny or near-underflow row: exact maximum and codes
            float ex = 0.0f;
#pragma unroll 1
            for (int i = 0; i < CPL; ++i) {
                const int c = gl + i * 32 * R;
                if (c < nch) {
                    RawChunk<__nv_bfloat16> ch;
                    ch.a = *reinterpret_cast<const uint4*>(src + c * 16);
                    ex = fmaxf(ex, second ? exact_chunk_max_in<__nv_bfloat16, kSmooth>(ch, s + c * 8, rn)
                                          : exact_chunk_max_in<__nv_bfloat16, MODE>(ch, s + c * 8, rn));
                }
            }
            const float a = group_max<R>(ex, red, grp, wig, lane, bank);
            bank ^= 1;
            const float scale = a == 0.0f ? 1.0f : __fdiv_rn(a, kQmax);
#pragma unroll 1
            for (int i = 0; i < CPL; ++i) {
                const int c = gl + i * 32 * R;
                if (c < nch) {
                    RawChunk<__nv_bfloat16> ch;
                    ch.a = *reinterpret_cast<const uint4*>(src + c * 16);
                    if (FMT == kInt8) {
                        *reinterpret_cast<uint2*>(rq + c * 8) =
                            second ? exact_chunk_codes_in<__nv_bfloat16, kSmooth>(ch, s + c * 8, scale, rn, a == 0.0f)
                                   : exact_chunk_codes_in<__nv_bfloat16, MODE>(ch, s + c * 8, scale, rn, a == 0.0f);
                    } else {
                        // E4M3: an all-zero row keeps the signs of its zeros (scale 1)
                        uint32_t b8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            b8[e] = second ? exact_code_fmt<kSmooth, FMT>(ch.get(e), __ldg(s + c * 8 + e), scale, rn)
                                           : exact_code_fmt<MODE, FMT>(ch.get(e), __ldg(s + c * 8 + e), scale, rn);
                        *reinterpret_cast<uint2*>(rq + c * 8) =
                            make_uint2(b8[0] | b8[1] << 8 | b8[2] << 16 | b8[3] << 24,
                                       b8[4] | b8[5] << 8 | b8[6] << 16 | b8[7] << 24);
                    }
                }
            }
            if (gl == 0) so[row] = scale;
            continue;
        }

        if (smooth) {
            // exact values of the candidates (normally the maximum alone)
            const float thr = __fmul_rn(amax, kRingCandidate);
            uint32_t cand = 0;
#pragma unroll
            for (int i = 0; i < CPL; ++i) cand |= (cm[i] >= thr ? 1u : 0u) << i;
            float ex = 0.0f;
            while (cand) {
                const int i = __ffs(cand) - 1;
                cand &= cand - 1;
                const int c = gl + i * 32 * R;
                const uint4 w = *reinterpret_cast<const uint4*>(src + c * 16);
                const float4 a = *reinterpret_cast<const float4*>(mlo + c * 4);
                const float4 b = *reinterpret_cast<const float4*>(mhi + c * 4);
                const float mv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float x = bf16_elem(w, e);
                    if (fabsf(__fmul_rn(x, mv[e])) >= thr) ex = fmaxf(ex, exact_abs<kSmooth>(x, __ldg(s + c * 8 + e), rn));
                }
            }
            amax = group_max<R>(ex, red, grp, wig, lane, bank);
            bank ^= 1;
        }

        // ---- pass 2: codes
        const float scale = __fdiv_rn(amax, kQmax);
        const float r = __frcp_rn(scale);
        const uint64_t r2 = f2_pack(r, r);
        const float guard = smooth ? kRingGuardSmooth : kRingGuardExact;
        uint32_t ntm = 0;
        uint2 codes[CPL];
        if constexpr (FMT == kInt8) {
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                uint32_t t[8];
                float dm = 0.0f;
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const uint64_t t2 = f2_fma(v2[i][p], r2, mag2);
                    const uint64_t d2 = f2_fma(v2[i][p], r2, f2_sub(mag2, t2));
                    float t0, t1, d0, d1;
                    f2_unpack(t2, t0, t1);
                    f2_unpack(d2, d0, d1);
                    t[2 * p] = __float_as_uint(t0);
                    t[2 * p + 1] = __float_as_uint(t1);
                    dm = fmax3(dm, fabsf(d0), fabsf(d1));
                }
                codes[i].x = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410);
                codes[i].y = __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410);
                const bool tie = dm >= 0.5f - guard;   // (padding: d = 0)
                if (smooth && tie) prefetch_l1(s + (gl + i * 32 * R) * 8);   // the repair divides by s_j
                ntm |= (tie ? 1u : 0u) << i;
            }
        } else {
            // E4M3: q' = RN(v r) converted at q'(1 - 2^-18) and q'(1 + 2^-18);
            // the conversion is monotone, and q* = RN(v / scale) lies within 6
            // ulps of q' (within 2^-18 |q'|), so equal codes are q*'s code
            const uint64_t lo2 = f2_pack(1.0f - 1.0f / 262144.0f, 1.0f - 1.0f / 262144.0f);
            const uint64_t hi2 = f2_pack(1.0f + 1.0f / 262144.0f, 1.0f + 1.0f / 262144.0f);
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                uint32_t c16[4];
                uint32_t diff = 0;
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const uint64_t q2 = f2_mul(v2[i][p], r2);
                    float l0, l1, h0, h1;
                    f2_unpack(f2_mul(q2, lo2), l0, l1);
                    f2_unpack(f2_mul(q2, hi2), h0, h1);
                    const uint32_t cl = __nv_cvt_float2_to_fp8x2(make_float2(l0, l1), __NV_SATFINITE, __NV_E4M3);
                    const uint32_t ch = __nv_cvt_float2_to_fp8x2(make_float2(h0, h1), __NV_SATFINITE, __NV_E4M3);
                    diff |= cl ^ ch;
                    c16[p] = cl;
                }
                codes[i] = make_uint2(c16[0] | c16[1] << 16, c16[2] | c16[3] << 16);
                ntm |= (diff != 0u ? 1u : 0u) << i;   // (padding: zeros convert alike)
            }
        }
        // the stores apart from the arithmetic, which stays free of branches
        const int64_t trows = second ? pr.rows2 : rows;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int c = gl + i * 32 * R;
            if ((FULL || c < nch) && dchk(c < nchunks && row < trows, SITE_DBG_RING_CODES))
                *reinterpret_cast<uint2*>(rq + c * 8) = codes[i];
        }
        if (gl == 0 && dchk(row < trows, SITE_DBG_RING_SCALE)) so[row] = scale;
        // near ties: the same fast quotient recomputed per element; those
        // within the guard get the IEEE-division code (same thread, later store)
        while (ntm) {
            const int i = __ffs(ntm) - 1;
            ntm &= ntm - 1;
            const int c = gl + i * 32 * R;
            const uint4 w = *reinterpret_cast<const uint4*>(src + c * 16);
            const float4 a = *reinterpret_cast<const float4*>(mlo + c * 4);
            const float4 b = *reinterpret_cast<const float4*>(mhi + c * 4);
            const float mv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float x = bf16_elem(w, e);
                const float vf = MODE == kNorm ? __fmul_rn(__fmul_rn(x, rn), mv[e]) : __fmul_rn(x, mv[e]);
                bool redo;
                if (FMT == kInt8) {
                    const float tf = __fmaf_rn(vf, r, kMagic);
                    const float df = __fmaf_rn(vf, r, __fsub_rn(kMagic, tf));
                    redo = fabsf(df) >= 0.5f - guard;
                } else {
                    const float qf = __fmul_rn(vf, r);
                    redo = __nv_cvt_float_to_fp8(__fmul_rn(qf, 1.0f - 1.0f / 262144.0f), __NV_SATFINITE, __NV_E4M3) !=
                           __nv_cvt_float_to_fp8(__fmul_rn(qf, 1.0f + 1.0f / 262144.0f), __NV_SATFINITE, __NV_E4M3);
                }
                if (redo && dchk(c < nchunks, SITE_DBG_RING_REPAIR)) {
                    uint32_t code;
                    if (FMT == kInt8) {
                        // fold and norm: vf is exact; smooth: the exact value takes a
                        // division, and its quotient stays within 2^-12 of the same
                        // half-step (v' is within 3 * 2^-24 |v| of v)
                        if (smooth && !pend) {
                            pend = true;
                            pend_x = x;
                            pend_s = __ldg(s + c * 8 + e);
                            pend_scale = scale;
                            pend_r = r;
                            pend_q = rq + c * 8 + e;
                            continue;
                        }
                        const float vx = smooth ? __fdiv_rn(x, __ldg(s + c * 8 + e)) : vf;
                        code = near_tie_code(vx, scale, __fmul_rn(vx, r));
                    } else if (second) code = exact_code_fmt<kSmooth, FMT>(x, __ldg(s + c * 8 + e), scale, rn);
                    else code = exact_code_fmt<MODE, FMT>(x, __ldg(s + c * 8 + e), scale, rn);
                    rq[c * 8 + e] = (int8_t)code;
                }
            }
        }
    }

    settle();
    if (failed && gl == 0) {
        // copies issued for rows this group will not consume: let them land
        // before the CTA exits (bounded)
        for (int j = it; j < issued; ++j)
            mbar_wait(bar0 + 8u * (j % ns), (uint32_t)(j / ns) & 1u, wait_limit, &never_sh, SITE_QUANT_DRAIN);
    }
}

// ============================================================== host side
namespace {

template <typename T, int MODE, int TPB, int MAXC, int FMT>
sq_status launch_row_quant_inst(const void* in, int64_t rows, int64_t K, const float* s,
                                int8_t* q, float* scale, cudaStream_t st) {
    const int64_t max_blocks = (int64_t)device_info().sm_count * (2048 / TPB);
    const int grid = (int)(rows < max_blocks ? rows : max_blocks);
    return launch_pdl("row_quant_kernel", row_quant_kernel<T, MODE, TPB, MAXC, FMT>, dim3(grid), dim3(TPB), 0, st, 1,
                      static_cast<const T*>(in), rows, K, s, q, scale);
}

template <typename T, int MODE, int TPB, int FMT>
sq_status launch_row_quant_tpb(int maxc, const void* in, int64_t rows, int64_t K, const float* s,
                               int8_t* q, float* scale, cudaStream_t st) {
    switch (maxc) {
        case 1: return launch_row_quant_inst<T, MODE, TPB, 1, FMT>(in, rows, K, s, q, scale, st);
        case 2: return launch_row_quant_inst<T, MODE, TPB, 2, FMT>(in, rows, K, s, q, scale, st);
        case 4: return launch_row_quant_inst<T, MODE, TPB, 4, FMT>(in, rows, K, s, q, scale, st);
        case 8: return launch_row_quant_inst<T, MODE, TPB, 8, FMT>(in, rows, K, s, q, scale, st);
    }
    set_error("internal: unsupported chunk count %d", maxc);
    return SQ_ERR_UNSUPPORTED;
}

int pow2ceil(int64_t v) {
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

// The IEEE-division kernel: one CTA per row at a time, K up to 65536.
template <typename T, int MODE, int FMT>
sq_status launch_row_quant_exact(const void* in, int64_t rows, int64_t K, const float* s, int8_t* q, float* scale,
                                 cudaStream_t st) {
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
        case 128: return launch_row_quant_tpb<T, MODE, 128, FMT>(maxc, in, rows, K, s, q, scale, st);
        case 256: return launch_row_quant_tpb<T, MODE, 256, FMT>(maxc, in, rows, K, s, q, scale, st);
        case 512: return launch_row_quant_tpb<T, MODE, 512, FMT>(maxc, in, rows, K, s, q, scale, st);
        default: return launch_row_quant_tpb<T, MODE, 1024, FMT>(maxc, in, rows, K, s, q, scale, st);
    }
}

template <typename T, int MODE, int R, int CPL = RowFastCPL<T>::value, bool PF = (R >= 8)>
sq_status launch_row_quant_fast_inst(const void* in, int64_t rows, int64_t K, const float* s, int8_t* q,
                                     float* scale, cudaStream_t st, float eps, float* r_out) {
    static bool attr_done[64] = {};
    const DeviceInfo& di = device_info();
    const int threads = 32 * R > 256 ? 32 * R : 256;
    const int groups = threads / (32 * R);
    const size_t smem = (size_t)K * 6 + (size_t)groups * 2 * R * (sizeof(float) + (MODE == kNorm ? sizeof(double) : 0));
    auto kern = row_quant_fast_kernel<T, MODE, R, CPL, PF>;
    if (!attr_done[di.device & 63]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)(kFastMaxK * 6 + 1024));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(row_quant_fast_kernel)");
        attr_done[di.device & 63] = true;
    }
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
    if (per_sm < 1) per_sm = 1;
    const int64_t need = (rows + groups - 1) / groups;
    const int64_t max_blocks = (int64_t)di.sm_count * per_sm;
    const int grid = (int)(need < max_blocks ? need : max_blocks);
    return launch_pdl("row_quant_fast_kernel", kern, dim3(grid), dim3(threads), smem, st, 1,
                      static_cast<const T*>(in), rows, K, s, q, scale, eps, r_out);
}

// The streamed kernel's shared memory: multipliers (two tables for a pair
// launch) and ns row slots per group, both padded to 32 * R * CPL chunks, the
// slots' mbarriers and the group reduction slots.
size_t ring_smem_bytes(int R, int CPL, int ns, bool pair) {
    const size_t G = (size_t)(kRingThreads / (32 * R));
    const size_t ncp = (size_t)32 * R * CPL;
    return ncp * (pair ? 64 : 32) + G * (size_t)ns * (ncp * 16 + 8) + G * 2 * (size_t)R * (4 + 8);
}

template <int MODE, int R, int CPL, bool FULL, bool PAIR, int FMT>
sq_status launch_row_quant_ring_inst(const void* in, int64_t rows, int64_t K, const float* s, int8_t* q,
                                     float* scale, cudaStream_t st, float eps, float* r_out, int ns,
                                     const RingPair& pr) {
    static bool attr_done[64] = {};
    const DeviceInfo& di = device_info();
    auto kern = row_quant_ring_kernel<MODE, R, CPL, FULL, PAIR, FMT>;
    if (!attr_done[di.device & 63]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRingSmemMax);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(row_quant_ring_kernel)");
        attr_done[di.device & 63] = true;
    }
    constexpr int G = kRingThreads / (32 * R);
    const int64_t need = (rows + (PAIR ? pr.rows2 : 0) + G - 1) / G;
    const int grid = (int)(need < di.sm_count ? need : di.sm_count);
    return launch_pdl("row_quant_ring_kernel", kern, dim3(grid), dim3(kRingThreads), ring_smem_bytes(R, CPL, ns, PAIR),
                      st, 1, static_cast<const __nv_bfloat16*>(in), rows, K, s, q, scale, eps, r_out, ns,
                      wait_limit_cycles(), pr);
}

template <int MODE, int R, bool PAIR, int FMT>
sq_status launch_row_quant_ring_r(int cpl, const void* in, int64_t rows, int64_t K, const float* s, int8_t* q,
                                  float* scale, cudaStream_t st, float eps, float* r_out, int ns,
                                  const RingPair& pr) {
    // rows that fill every lane (K = 256 R CPL) drop the stores' bounds checks;
    // E4M3 codes are instantiated for such rows only (the caller checks)
    const bool full = K / 8 == (int64_t)32 * R * cpl;
#define SQ_RING_CPL(C)                                                                                            \
    if constexpr (FMT == kInt8) {                                                                                 \
        return full ? launch_row_quant_ring_inst<MODE, R, C, true, PAIR, FMT>(in, rows, K, s, q, scale, st, eps,  \
                                                                              r_out, ns, pr)                      \
                    : launch_row_quant_ring_inst<MODE, R, C, false, PAIR, FMT>(in, rows, K, s, q, scale, st, eps, \
                                                                               r_out, ns, pr);                    \
    } else {                                                                                                      \
        return launch_row_quant_ring_inst<MODE, R, C, true, PAIR, FMT>(in, rows, K, s, q, scale, st, eps, r_out,  \
                                                                       ns, pr);                                   \
    }
    if constexpr (R == 2) {
        if (cpl == 10) { SQ_RING_CPL(10); }
    }
    switch (cpl) {
        case 5: SQ_RING_CPL(5);
        case 6: SQ_RING_CPL(6);
        case 7: SQ_RING_CPL(7);
        default: SQ_RING_CPL(8);
    }
#undef SQ_RING_CPL
}

// bf16 rows of 2064..28672 elements go to the streamed kernel: the fewest
// warps per row (R = 2, 4, 8 or 16) whose lanes hold the row in at most 8 chunks
// each (CPL = 5..8 of them, the row padded to 32 * R * CPL chunks; two warps
// with 10 chunks up to 640 chunks), and two
// ring slots per group (one row in flight while one is processed: measured
// faster than three or four). Returns false when K is outside that range or
// the padded row, its multipliers and two slots exceed the shared memory of a
// CTA (K above 28672).
template <int MODE, bool PAIR = false, int FMT = kInt8>
bool launch_row_quant_ring(const void* in, int64_t rows, int64_t K, const float* s, int8_t* q, float* scale,
                           cudaStream_t st, float eps, float* r_out, sq_status& result,
                           const RingPair& pr = RingPair{}) {
    const int64_t nchunks = K / 8;
    if (K <= 2048 || nchunks > (int64_t)32 * 16 * kRingCPL) return false;
    int R = 2;
    while ((int64_t)32 * R * kRingCPL < nchunks) R *= 2;
    int cpl = (int)((nchunks + 32 * R - 1) / (32 * R));
    if (cpl < 5) cpl = 5;
    // rows of up to 640 chunks (K <= 5120) stay on two warps with ten chunks per
    // lane: measured faster than four warps with five (13B, K = 5120: 77 against 96 us)
    if (R == 4 && nchunks <= 640) {
        R = 2;
        cpl = 10;
    }
    const int ns = 2;
    if (ring_smem_bytes(R, cpl, ns, PAIR) > kRingSmemMax) return false;
    if (FMT != kInt8 && nchunks != (int64_t)32 * R * cpl) return false;
#define SQ_RING_R(RR) launch_row_quant_ring_r<MODE, RR, PAIR, FMT>(cpl, in, rows, K, s, q, scale, st, eps, r_out, ns, pr)
    switch (R) {
        case 2: result = SQ_RING_R(2); break;
        case 4: result = SQ_RING_R(4); break;
        case 8: result = SQ_RING_R(8); break;
        default: result = SQ_RING_R(16); break;
    }
#undef SQ_RING_R
    return true;
}

template <typename T, int MODE>
sq_status launch_row_quant(const void* in, int64_t rows, int64_t K, const float* s, int8_t* q,
                           float* scale, cudaStream_t st, float eps = 0.0f, float* r_out = nullptr) {
    constexpr int CPL = RowFastCPL<T>::value;
    const int64_t nchunks = K / 8;
    if constexpr (sizeof(T) == 2) {
        sq_status res = SQ_OK;
        if (launch_row_quant_ring<MODE>(in, rows, K, s, q, scale, st, eps, r_out, res)) return res;
    }
    // the fewest warps per row whose lanes hold the row in CPL chunks each
    if (K <= kFastMaxK) {
        for (int R = 1; R <= 16; R *= 2) {
            if (nchunks <= (int64_t)32 * R * CPL) {
                switch (R) {
                    case 1: return launch_row_quant_fast_inst<T, MODE, 1>(in, rows, K, s, q, scale, st, eps, r_out);
                    case 2: return launch_row_quant_fast_inst<T, MODE, 2>(in, rows, K, s, q, scale, st, eps, r_out);
                    case 4: return launch_row_quant_fast_inst<T, MODE, 4>(in, rows, K, s, q, scale, st, eps, r_out);
                    case 8: return launch_row_quant_fast_inst<T, MODE, 8>(in, rows, K, s, q, scale, st, eps, r_out);
                    default: return launch_row_quant_fast_inst<T, MODE, 16>(in, rows, K, s, q, scale, st, eps, r_out);
                }
            }
        }
    }
    if constexpr (MODE == kNorm) {
        set_error("K=%lld exceeds the fused norm-and-quantize limit of %lld for this dtype", (long long)K,
                  (long long)(32 * 16 * 8 * RowFastCPL<T>::value));
        return SQ_ERR_UNSUPPORTED;
    } else {
    return launch_row_quant_exact<T, MODE, kInt8>(in, rows, K, s, q, scale, st);
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

// Resident 256-thread blocks per SM of a column kernel (its registers and
// static shared memory decide; looked up once per kernel).
template <auto KERN>
int column_blocks_per_sm() {
    static int cached = 0;
    if (cached == 0) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, KERN, kAbsmaxThreads, 0) != cudaSuccess || n < 1) n = 1;
        cached = n;
    }
    return cached;
}

// One full wave of 256-thread blocks (per_sm resident per SM); every block
// covers a multiple of the 64 rows it reads per iteration. Returns the grid
// and the rows per block.
sq_status absmax_grid(int64_t rows, int64_t cols, int es, dim3& grid, int64_t& per, int per_sm) {
    const int64_t tile = 32 * (16 / es);
    const int64_t ct = (cols + tile - 1) / tile;
    const int64_t step_rows = 8 * kAbsmaxRowsInFlight;
    const int64_t target = (int64_t)device_info().sm_count * per_sm;
    int64_t rc = target / ct;
    if (rc < 1) rc = 1;
    per = (rows + rc - 1) / rc;
    per = (per + step_rows - 1) / step_rows * step_rows;
    rc = (rows + per - 1) / per;
    if (rc > 65535) {
        rc = 65535;
        per = (rows + rc - 1) / rc;
        per = (per + step_rows - 1) / step_rows * step_rows;
        rc = (rows + per - 1) / per;
    }
    if (ct > 2147483647LL) { set_error("cols too large"); return SQ_ERR_UNSUPPORTED; }
    grid = dim3((unsigned)ct, (unsigned)rc);
    return SQ_OK;
}

sq_status calibrate_absmax_impl(const void* x, sq_dtype dt, int64_t rows, int64_t cols,
                                float* absmax, cudaStream_t st) {
    sq_status r;
    if ((r = check_input_dtype(dt)) != SQ_OK) return r;
    if ((r = check_matrix(x, rows, cols, "x")) != SQ_OK) return r;
    if (cols > 0 && !absmax) { set_error("absmax: NULL pointer"); return SQ_ERR_INVALID_ARG; }
    if (rows == 0 || cols == 0) return SQ_OK;
    dim3 grid;
    int64_t per = 0;
    const int per_sm = dt == SQ_F32 ? column_blocks_per_sm<col_absmax_kernel<float, false>>()
                                    : column_blocks_per_sm<col_absmax_kernel<__nv_bfloat16, false>>();
    if ((r = absmax_grid(rows, cols, dt == SQ_F32 ? 4 : 2, grid, per, per_sm)) != SQ_OK) return r;
    if (dt == SQ_F32)
        return launch_pdl("col_absmax_kernel", col_absmax_kernel<float, false>, grid, dim3(kAbsmaxThreads), 0, st, 1,
                          static_cast<const uint8_t*>(x), rows, cols, per, absmax, (const float*)nullptr,
                          AbsmaxPair{});
    return launch_pdl("col_absmax_kernel", col_absmax_kernel<__nv_bfloat16, false>, grid, dim3(kAbsmaxThreads), 0, st,
                      1, static_cast<const uint8_t*>(x), rows, cols, per, absmax, (const float*)nullptr, AbsmaxPair{});
}

// Both calibrations of a layer in one launch: one wave of blocks shared between
// the activations and the weights in proportion to their rows.
sq_status calibrate_absmax_pair_impl(const void* x, int64_t T, const void* w, int64_t N, sq_dtype dt, int64_t K,
                                     float* xmax, float* wmax, cudaStream_t st) {
    sq_status r;
    if ((r = check_input_dtype(dt)) != SQ_OK) return r;
    if ((r = check_matrix(x, T, K, "x")) != SQ_OK) return r;
    if ((r = check_matrix(w, N, K, "w")) != SQ_OK) return r;
    if (K > 0 && (!xmax || !wmax)) { set_error("absmax: NULL pointer"); return SQ_ERR_INVALID_ARG; }
    if (K == 0) return SQ_OK;
    if (T == 0) return calibrate_absmax_impl(w, dt, N, K, wmax, st);
    if (N == 0) return calibrate_absmax_impl(x, dt, T, K, xmax, st);
    const int es = dt == SQ_F32 ? 4 : 2;
    const int64_t tile = 32 * (16 / es);
    const int64_t ct = (K + tile - 1) / tile;
    if (ct > 2147483647LL) { set_error("cols too large"); return SQ_ERR_UNSUPPORTED; }
    const int64_t step_rows = 8 * kAbsmaxRowsInFlight;
    const int per_sm = dt == SQ_F32 ? column_blocks_per_sm<col_absmax_kernel<float, false>>()
                                    : column_blocks_per_sm<col_absmax_kernel<__nv_bfloat16, false>>();
    const int64_t target = (int64_t)device_info().sm_count * per_sm;
    auto chunks = [&](int64_t rows, int64_t share, int64_t& per) {
        int64_t rc = share / ct;
        if (rc < 1) rc = 1;
        per = (rows + rc - 1) / rc;
        per = (per + step_rows - 1) / step_rows * step_rows;
        return (rows + per - 1) / per;
    };
    int64_t per_x = 0, per_w = 0;
    const int64_t share_x = target * T / (T + N);
    const int64_t rc_x = chunks(T, share_x, per_x);
    const int64_t rc_w = chunks(N, target - share_x, per_w);
    if (rc_x + rc_w > 65535) {
        // very tall inputs: one launch per tensor
        if ((r = calibrate_absmax_impl(x, dt, T, K, xmax, st)) != SQ_OK) return r;
        return calibrate_absmax_impl(w, dt, N, K, wmax, st);
    }
    AbsmaxPair pair;
    pair.x2 = static_cast<const uint8_t*>(w);
    pair.rows2 = N;
    pair.per2 = per_w;
    pair.absmax2 = wmax;
    pair.rc1 = (int)rc_x;
    const dim3 grid((unsigned)ct, (unsigned)(rc_x + rc_w));
    if (dt == SQ_F32)
        return launch_pdl("col_absmax_kernel<pair>", col_absmax_kernel<float, false>, grid, dim3(kAbsmaxThreads), 0,
                          st, 1, static_cast<const uint8_t*>(x), T, K, per_x, xmax, (const float*)nullptr, pair);
    return launch_pdl("col_absmax_kernel<pair>", col_absmax_kernel<__nv_bfloat16, false>, grid, dim3(kAbsmaxThreads),
                      0, st, 1, static_cast<const uint8_t*>(x), T, K, per_x, xmax, (const float*)nullptr, pair);
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
    return launch_pdl("smooth_factors_kernel", smooth_factors_kernel, dim3((unsigned)blocks), dim3(threads), 0, st, 1,
                      xmax, wmax, K, alpha, eps, s);
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

// FP8 E4M3 codes: the same fold / smoothing, per-row scale amax / 448, every
// quotient an IEEE division (the exact kernel).
sq_status row_quant_e4m3_common(int mode, const void* in, sq_dtype dt, int64_t rows, int64_t K,
                                const float* s, uint8_t* q, float* scale, cudaStream_t st) {
    sq_status r;
    if ((r = check_input_dtype(dt)) != SQ_OK) return r;
    if ((r = check_matrix(in, rows, K, "input")) != SQ_OK) return r;
    if (rows == 0) return SQ_OK;
    if (K == 0) { set_error("K must be positive"); return SQ_ERR_INVALID_ARG; }
    if (!s || !q || !scale) { set_error("NULL pointer"); return SQ_ERR_INVALID_ARG; }
    if (!aligned16(s) || !aligned16(q)) { set_error("s and codes must be 16-byte aligned"); return SQ_ERR_UNSUPPORTED; }
    int8_t* qq = reinterpret_cast<int8_t*>(q);
    if (dt == SQ_BF16) {
        // rows that fill the streamed kernel's lanes exactly: the fast E4M3 pass
        sq_status res = SQ_OK;
        if (mode == kFold ? launch_row_quant_ring<kFold, false, kE4M3>(in, rows, K, s, qq, scale, st, 0.0f, nullptr, res)
                          : launch_row_quant_ring<kSmooth, false, kE4M3>(in, rows, K, s, qq, scale, st, 0.0f, nullptr,
                                                                         res))
            return res;
    }
    if (mode == kFold)
        return dt == SQ_F32 ? launch_row_quant_exact<float, kFold, kE4M3>(in, rows, K, s, qq, scale, st)
                            : launch_row_quant_exact<__nv_bfloat16, kFold, kE4M3>(in, rows, K, s, qq, scale, st);
    return dt == SQ_F32 ? launch_row_quant_exact<float, kSmooth, kE4M3>(in, rows, K, s, qq, scale, st)
                        : launch_row_quant_exact<__nv_bfloat16, kSmooth, kE4M3>(in, rows, K, s, qq, scale, st);
}

sq_status fold_quant_weights_impl(const void* w, sq_dtype dt, int64_t N, int64_t K, const float* s,
                                  int8_t* wq, float* w_scale, cudaStream_t st) {
    return row_quant_common(kFold, w, dt, N, K, s, wq, w_scale, st);
}

sq_status smooth_quant_act_impl(const void* x, sq_dtype dt, int64_t T, int64_t K, const float* s,
                                int8_t* xq, float* x_scale, cudaStream_t st) {
    return row_quant_common(kSmooth, x, dt, T, K, s, xq, x_scale, st);
}

// a3 and a4 in one launch where the streamed kernel takes both (bf16, and the
// two multiplier tables fit in shared memory beside the ring): the weights'
// rows, then the activations'. Elsewhere the two calls, one after the other.
sq_status fold_smooth_quant_pair_impl(const void* w, int64_t N, const void* x, int64_t T, sq_dtype dt, int64_t K,
                                      const float* s, int8_t* wq, float* w_scale, int8_t* xq, float* x_scale,
                                      cudaStream_t st) {
    sq_status r;
    if ((r = check_input_dtype(dt)) != SQ_OK) return r;
    if ((r = check_matrix(w, N, K, "w")) != SQ_OK) return r;
    if ((r = check_matrix(x, T, K, "x")) != SQ_OK) return r;
    if (N == 0) return smooth_quant_act_impl(x, dt, T, K, s, xq, x_scale, st);
    if (T == 0) return fold_quant_weights_impl(w, dt, N, K, s, wq, w_scale, st);
    if (K == 0) { set_error("K must be positive"); return SQ_ERR_INVALID_ARG; }
    if (!s || !wq || !w_scale || !xq || !x_scale) { set_error("NULL pointer"); return SQ_ERR_INVALID_ARG; }
    if (!aligned16(s) || !aligned16(wq) || !aligned16(xq)) {
        set_error("s and codes must be 16-byte aligned");
        return SQ_ERR_UNSUPPORTED;
    }
    if (dt == SQ_BF16) {
        RingPair pr;
        pr.in2 = static_cast<const __nv_bfloat16*>(x);
        pr.rows2 = T;
        pr.q2 = xq;
        pr.scale2 = x_scale;
        sq_status res = SQ_OK;
        if (launch_row_quant_ring<kFold, true>(w, N, K, s, wq, w_scale, st, 0.0f, nullptr, res, pr)) return res;
    }
    if ((r = fold_quant_weights_impl(w, dt, N, K, s, wq, w_scale, st)) != SQ_OK) return r;
    return smooth_quant_act_impl(x, dt, T, K, s, xq, x_scale, st);
}

// The same pair with FP8 E4M3 codes: one launch where the streamed kernel's
// E4M3 pass takes both (bf16 rows that fill its lanes, two multiplier tables
// beside the ring); else the two E4M3 calls.
sq_status fold_smooth_quant_pair_e4m3_impl(const void* w, int64_t N, const void* x, int64_t T, sq_dtype dt,
                                           int64_t K, const float* s, uint8_t* wq, float* w_scale, uint8_t* xq,
                                           float* x_scale, cudaStream_t st) {
    sq_status r;
    if ((r = check_input_dtype(dt)) != SQ_OK) return r;
    if ((r = check_matrix(w, N, K, "w")) != SQ_OK) return r;
    if ((r = check_matrix(x, T, K, "x")) != SQ_OK) return r;
    if (dt == SQ_BF16 && N > 0 && T > 0 && K > 0) {
        if (!s || !wq || !w_scale || !xq || !x_scale) { set_error("NULL pointer"); return SQ_ERR_INVALID_ARG; }
        if (!aligned16(s) || !aligned16(wq) || !aligned16(xq)) {
            set_error("s and codes must be 16-byte aligned");
            return SQ_ERR_UNSUPPORTED;
        }
        RingPair pr;
        pr.in2 = static_cast<const __nv_bfloat16*>(x);
        pr.rows2 = T;
        pr.q2 = reinterpret_cast<int8_t*>(xq);
        pr.scale2 = x_scale;
        sq_status res = SQ_OK;
        if (launch_row_quant_ring<kFold, true, kE4M3>(w, N, K, s, reinterpret_cast<int8_t*>(wq), w_scale, st, 0.0f,
                                                      nullptr, res, pr))
            return res;
    }
    if ((r = row_quant_e4m3_common(kFold, w, dt, N, K, s, wq, w_scale, st)) != SQ_OK) return r;
    return row_quant_e4m3_common(kSmooth, x, dt, T, K, s, xq, x_scale, st);
}

}  // namespace sq

extern "C" {

sq_status sq_fold_quant_weights_e4m3(const void* w, sq_dtype dt, int64_t N, int64_t K, const float* s, uint8_t* wq,
                                     float* w_scale, sq_stream_t stream) {
    return sq::row_quant_e4m3_common(sq::kFold, w, dt, N, K, s, wq, w_scale, (cudaStream_t)stream);
}

sq_status sq_smooth_quant_act_e4m3(const void* x, sq_dtype dt, int64_t T, int64_t K, const float* s, uint8_t* xq,
                                   float* x_scale, sq_stream_t stream) {
    return sq::row_quant_e4m3_common(sq::kSmooth, x, dt, T, K, s, xq, x_scale, (cudaStream_t)stream);
}

sq_status sq_fold_smooth_quant_pair_e4m3(const void* w, int64_t N, const void* x, int64_t T, sq_dtype dt, int64_t K,
                                         const float* s, uint8_t* wq, float* w_scale, uint8_t* xq, float* x_scale,
                                         sq_stream_t stream) {
    return sq::fold_smooth_quant_pair_e4m3_impl(w, N, x, T, dt, K, s, wq, w_scale, xq, x_scale,
                                                (cudaStream_t)stream);
}


sq_status sq_calibrate_absmax_pair(const void* x, int64_t T, const void* w, int64_t N, sq_dtype dt, int64_t K,
                                   float* xmax, float* wmax, sq_stream_t stream) {
    return sq::calibrate_absmax_pair_impl(x, T, w, N, dt, K, xmax, wmax, (cudaStream_t)stream);
}


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

sq_status sq_fold_smooth_quant_pair(const void* w, int64_t N, const void* x, int64_t T, sq_dtype dt, int64_t K,
                                    const float* s, int8_t* wq, float* w_scale, int8_t* xq, float* x_scale,
                                    sq_stream_t stream) {
    return sq::fold_smooth_quant_pair_impl(w, N, x, T, dt, K, s, wq, w_scale, xq, x_scale, (cudaStream_t)stream);
}

}  // extern "C"
