// Per-row FP8 E4M3 quantisation and the NestedFP byte-plane split.
//
// quantize: "7B on an RTX 4060 with FP8" §2.2 (dynamic activation amax,
// static weight scales) and §6.1 (448 bound); "C++ and FP8" §4.2 (per-token /
// per-channel).  split: "NestedFP dual-precision inference framework" §2.1.
//
// Both are HBM-bound elementwise passes.  quantize: one CTA per row, 128-bit
// loads, warp-shuffle max then a CTA max for the amax; rows of up to 16384
// elements are held in registers between the amax and the conversion (one
// pass over memory), longer rows are re-read from L2 for the conversion.
// Bytes per element: 4 (f32) or 2 (f16) in, 1 out.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace pgf8 {

constexpr int kQuantThreads = 256;

template <typename T> struct Vec16;   // 16 elements of T, loaded as 128-bit words

template <> struct Vec16<float> {
    float v[16];
    __device__ __forceinline__ void load(const float *p)
    {
        const float4 *q = reinterpret_cast<const float4 *>(p);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float4 t = __ldg(q + i);
            v[4 * i + 0] = t.x;
            v[4 * i + 1] = t.y;
            v[4 * i + 2] = t.z;
            v[4 * i + 3] = t.w;
        }
    }
};

template <> struct Vec16<__half> {
    float v[16];
    __device__ __forceinline__ void load(const __half *p)
    {
        const uint4 *q = reinterpret_cast<const uint4 *>(p);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            uint4 t = __ldg(q + i);
            uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                __half2 h = *reinterpret_cast<__half2 *>(&w[j]);
                float2 f = __half22float2(h);   // exact widening
                v[8 * i + 2 * j] = f.x;
                v[8 * i + 2 * j + 1] = f.y;
            }
        }
    }
};

// Maximum over the CTA's THREADS threads (red: THREADS / 32 floats).
template <int THREADS> __device__ __forceinline__ float block_max_n(float v, float *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0)
        red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < (THREADS / 32) ? red[lane] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0)
            red[0] = v;
    }
    __syncthreads();
    return red[0];
}

__device__ __forceinline__ float block_max(float v, float *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0)
        red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < (kQuantThreads / 32) ? red[lane] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0)
            red[0] = v;
    }
    __syncthreads();
    return red[0];
}

// Modes of the row quantisers.  0 dynamic: *srow = fl32(amax / 448), 1 for
// an all-zero row ("7B on an RTX 4060 with FP8" §2.2 per-token scale, §6.1
// the 448 limit); 1 static: the scale is read from *srow; 2 given amax:
// *srow holds the row's amax on input (taken over the whole row, e.g.
// reduced over tensor-parallel ranks that each hold a slice of it) and its
// scale, computed as in mode 0, on output; 3 amax only: *srow = amax, no
// codes are written.
enum : int { kQuantDynamic = 0, kQuantStatic = 1, kQuantFromAmax = 2, kQuantAmaxOnly = 3 };

// The row's scale s from this thread's partial amax (all THREADS threads
// call it).  Returns false when the row is done (mode 3).
template <int THREADS>
__device__ __forceinline__ bool row_scale(float amax, float *srow, int mode, float *red, float &s)
{
    if (mode == kQuantStatic) {
        s = *srow;
        return true;
    }
    if (mode == kQuantFromAmax) {
        amax = *srow;
        __syncthreads();   // every thread has read the amax before it is replaced by the scale
    } else {
        amax = block_max_n<THREADS>(amax, red);
        if (mode == kQuantAmaxOnly) {
            if (threadIdx.x == 0)
                *srow = amax;
            return false;
        }
    }
    s = __fdiv_rn(amax, 448.0f);
    if (s == 0.0f)
        s = 1.0f;
    if (threadIdx.x == 0)
        *srow = s;
    return true;
}

// x / s correctly rounded (binary32, nearest-even) for many x and one
// divisor s — the quotient the quantisation rounds to E4M3.
//
// Method: Markstein's FMA division (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990; "Markstein's theorem" in Muller et al., Handbook of Floating-Point
// Arithmetic).  With y = RN(1/s) (correctly rounded reciprocal, once per
// divisor) and a = |x|:
//   q0 = RN(a y)                 within (2u + u^2) |a/s|, u = 2^-24
//   r0 = RN(a - s q0)            (fma)
//   q1 = RN(q0 + r0 y)           error ~4u^2 |a/s| before rounding: faithful
//   r1 = a - s q1                exact (fma): the remainder of a faithful
//                                quotient is representable barring underflow
//   q2 = RN(q1 + r1 y) = RN(a/s) by Markstein's theorem (y within half an ulp
//                                of 1/s, q1 faithful, r1 exact)
// and the sign of x is put back (so -0 gives -0).  The steps need no
// overflow and no underflow of the remainders: that holds for
// 2^-60 <= s <= 2^96 and |x / s| <= 512 (the quantisation divides values of
// magnitude at most amax by s = RN(amax / 448)); quotients so small that
// the remainders underflow are below 2^-11 and round to a zero code either
// way.  Other divisors, and non-finite x, take the IEEE division itself.
// Checked exhaustively against __fdiv_rn over all binary32 x with
// |x| <= 512 s for a set of divisors (pgf8_selftest_row_division): equal
// quotients wherever |x / s| >= 2^-11, equal E4M3 codes everywhere.
struct RowDivisor {
    float s, y;
    bool fast;
    RowDivisor() = default;
    __device__ __forceinline__ explicit RowDivisor(float s_)
    {
        s = s_;
        y = __frcp_rn(s_);
        fast = s_ >= 0x1p-60f && s_ <= 0x1p96f;
    }
    // the FMA sequence alone (caller checked `fast` and that x is finite)
    __device__ __forceinline__ float div_fast(float x) const
    {
        const float a = fabsf(x);
        const float q0 = __fmul_rn(a, y);
        const float r0 = __fmaf_rn(-s, q0, a);
        const float q1 = __fmaf_rn(r0, y, q0);
        const float r1 = __fmaf_rn(-s, q1, a);
        const float q2 = __fmaf_rn(r1, y, q1);
        return copysignf(q2, x);
    }
    __device__ __forceinline__ float div(float x) const
    {
        if (!fast || !isfinite(x))
            return __fdiv_rn(x, s);
        return div_fast(x);
    }
};

// Converts N (8 or 16) binary32 values to N codes: E4M3(RN(v / s)),
// saturating.  One branch for the whole group (divisor in range and every
// value finite), so the N division chains interleave.
template <int N>
__device__ __forceinline__ void encode_codes(const float (&v)[N], const RowDivisor &d, uint32_t (&w)[N / 4])
{
    uint32_t inf_nan = 0;
#pragma unroll
    for (int i = 0; i < N; ++i)
        inf_nan |= static_cast<uint32_t>((__float_as_uint(v[i]) & 0x7F800000u) == 0x7F800000u);
    float q[N];
    if (d.fast && !inf_nan) {
#pragma unroll
        for (int i = 0; i < N; ++i)
            q[i] = d.div_fast(v[i]);
    } else {
#pragma unroll
        for (int i = 0; i < N; ++i)
            q[i] = d.div(v[i]);
    }
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
        const uint32_t lo = cvt_e4m3x2(q[4 * i + 0], q[4 * i + 1]);
        const uint32_t hi = cvt_e4m3x2(q[4 * i + 2], q[4 * i + 3]);
        w[i] = lo | (hi << 16);
    }
}

__device__ __forceinline__ uint4 encode16(const float (&v)[16], const RowDivisor &d)
{
    uint32_t w[4];
    encode_codes<16>(v, d, w);
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Self-test of RowDivisor: for each divisor s, every finite binary32 x with
// |x| <= 512 s (enumerated by bit pattern) is divided both ways.  Counted
// per divisor: [2i] quotients that differ where |x| >= 2^-11 s (the
// quotients the E4M3 rounding can tell apart), [2i+1] E4M3 codes that differ
// anywhere in the domain.
__global__ void __launch_bounds__(256) selftest_row_division_kernel(const float *__restrict__ divisors, int count,
                                                                    unsigned long long *__restrict__ mismatches)
{
    const int di = blockIdx.y;
    if (di >= count)
        return;
    const RowDivisor d(divisors[di]);
    const float lim = 512.0f * d.s;
    const float small = 0x1p-11f * d.s;
    unsigned long long bad_q = 0, bad_code = 0;
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
    for (uint64_t b = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < (1ull << 32); b += stride) {
        const float x = __uint_as_float(static_cast<uint32_t>(b));
        if (!(fabsf(x) <= lim))
            continue;
        const float q = d.div(x), ref = __fdiv_rn(x, d.s);
        if (fabsf(x) >= small && __float_as_uint(q) != __float_as_uint(ref))
            ++bad_q;
        if (cvt_e4m3x2(q, 0.0f) != cvt_e4m3x2(ref, 0.0f))
            ++bad_code;
    }
    if (bad_q)
        atomicAdd(&mismatches[2 * di], bad_q);
    if (bad_code)
        atomicAdd(&mismatches[2 * di + 1], bad_code);
}

// Rows of up to kRegChunks * kQuantThreads * 16 elements stay in registers
// between the amax and the conversion (one pass over global memory);
// longer rows are re-read (from L2) for the conversion.
constexpr int kRegChunks = 4;

// One row quantised by one CTA of kQuantThreads threads (every thread of
// the CTA calls it).  cols % 16 == 0; the row 16-byte aligned.  mode: see
// row_scale.
template <typename T>
__device__ __forceinline__ void quantize_one_row(const T *__restrict__ xr, int64_t cols, uint8_t *__restrict__ qr,
                                                 float *srow, int mode, float *red)
{
    const int64_t nchunk = cols / 16;

    if (nchunk <= static_cast<int64_t>(kRegChunks) * kQuantThreads) {
        Vec16<T> v[kRegChunks];
        float amax = 0.0f;
#pragma unroll
        for (int u = 0; u < kRegChunks; ++u) {
            const int64_t c = threadIdx.x + static_cast<int64_t>(u) * kQuantThreads;
            if (c < nchunk) {
                v[u].load(xr + c * 16);
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    amax = fmaxf(amax, fabsf(v[u].v[i]));
            }
        }
        float s;
        if (!row_scale<kQuantThreads>(amax, srow, mode, red, s))
            return;
        const RowDivisor d(s);
#pragma unroll
        for (int u = 0; u < kRegChunks; ++u) {
            const int64_t c = threadIdx.x + static_cast<int64_t>(u) * kQuantThreads;
            if (c < nchunk)
                *reinterpret_cast<uint4 *>(qr + c * 16) = encode16(v[u].v, d);
        }
        return;
    }

    float amax = 0.0f;
    if (mode == kQuantDynamic || mode == kQuantAmaxOnly) {
        for (int64_t c = threadIdx.x; c < nchunk; c += kQuantThreads) {
            Vec16<T> v;
            v.load(xr + c * 16);
#pragma unroll
            for (int i = 0; i < 16; ++i)
                amax = fmaxf(amax, fabsf(v.v[i]));
        }
    }
    float s;
    if (!row_scale<kQuantThreads>(amax, srow, mode, red, s))
        return;
    const RowDivisor d(s);
    for (int64_t c = threadIdx.x; c < nchunk; c += kQuantThreads) {
        Vec16<T> v;
        v.load(xr + c * 16);
        *reinterpret_cast<uint4 *>(qr + c * 16) = encode16(v.v, d);
    }
}

// One CTA per row.  cols % 16 == 0; x rows 16-byte aligned.
// flags: kQuantTriggerEarly lets a dependent launched with programmatic
// serialization start at once (used when that dependent is the library's
// own GEMM, which reads q / scales only after this grid completes);
// kQuantNoWait skips the wait for the previous kernel (used only when that
// kernel is independent of this one's inputs and signals its dependents
// after its own wait, so everything before it has completed).
constexpr int kQuantTriggerEarly = 1;
constexpr int kQuantNoWait = 2;

template <typename T>
__global__ void __launch_bounds__(kQuantThreads) quantize_rows_kernel(const T *__restrict__ x, int64_t rows,
                                                                      int64_t cols, int64_t ldx,
                                                                      uint8_t *__restrict__ q,
                                                                      float *__restrict__ scales, int mode,
                                                                      int flags)
{
    __shared__ float red[kQuantThreads / 32];
    if (flags & kQuantTriggerEarly)
        grid_launch_dependents();
    // When launched with programmatic serialization, the previous kernel in
    // the stream may still run: nothing is read or written before it ends.
    if (!(flags & kQuantNoWait))
        grid_dependency_wait();
    const int64_t row = blockIdx.x;
    if (row >= rows)
        return;
    quantize_one_row<T>(x + row * ldx, cols, q + row * cols, scales + row, mode, red);
}

// The same row quantisation with the row held in registers by a CTA of
// THREADS threads, CH 16-element chunks per thread (rows of at most
// CH * THREADS * 16 elements): the launch picks the smallest CH (and 512
// threads for the longest rows), so the CTA holds no more registers than
// its row needs and more rows are in flight per SM.  Same arithmetic as
// quantize_one_row, element by element.
template <typename T, int CH, int THREADS>
__global__ void __launch_bounds__(THREADS) quantize_rows_held_kernel(const T *__restrict__ x, int64_t rows,
                                                                     int64_t cols, int64_t ldx,
                                                                     uint8_t *__restrict__ q,
                                                                     float *__restrict__ scales, int mode,
                                                                     int flags)
{
    __shared__ float red[THREADS / 32];
    if (flags & kQuantTriggerEarly)
        grid_launch_dependents();
    if (!(flags & kQuantNoWait))
        grid_dependency_wait();
    const int64_t row = blockIdx.x;
    if (row >= rows)
        return;
    const T *xr = x + row * ldx;
    uint8_t *qr = q + row * cols;
    const int64_t nchunk = cols / 16;
    Vec16<T> v[CH];
    float amax = 0.0f;
#pragma unroll
    for (int u = 0; u < CH; ++u) {
        const int64_t c = threadIdx.x + static_cast<int64_t>(u) * THREADS;
        if (c < nchunk) {
            v[u].load(xr + c * 16);
#pragma unroll
            for (int i = 0; i < 16; ++i)
                amax = fmaxf(amax, fabsf(v[u].v[i]));
        }
    }
    float s;
    if (!row_scale<THREADS>(amax, scales + row, mode, red, s))
        return;
    const RowDivisor d(s);
#pragma unroll
    for (int u = 0; u < CH; ++u) {
        const int64_t c = threadIdx.x + static_cast<int64_t>(u) * THREADS;
        if (c < nchunk)
            *reinterpret_cast<uint4 *>(qr + c * 16) = encode16(v[u].v, d);
    }
}

// Dynamic per-token quantisation of the activations of several independent
// layers in one launch: one CTA per row over all the layers' rows (layer l
// owns rows [row0, row0 + rows) of the grid), each row exactly as
// quantize_rows_kernel computes it.
constexpr int kQuantGroupMaxLayers = 64;

struct QuantGroupLayer {
    const void *x;       // [rows, cols] f32 or f16, row stride ldx elements
    int64_t ldx, cols, row0, rows;
    uint8_t *q;          // [rows, cols] codes
    float *scales;       // [rows]
    int xdt;             // 0 f32, 1 f16
};

struct QuantGroupParams {
    QuantGroupLayer L[kQuantGroupMaxLayers];
    int nlayers;
};

__global__ void __launch_bounds__(kQuantThreads) quantize_group_kernel(const __grid_constant__ QuantGroupParams p)
{
    __shared__ float red[kQuantThreads / 32];
    grid_launch_dependents();   // the dependent is the library's grouped GEMM
    grid_dependency_wait();
    const int64_t row = blockIdx.x;
    int l = 0;
    while (l + 1 < p.nlayers && p.L[l + 1].row0 <= row)
        ++l;
    const QuantGroupLayer &g = p.L[l];
    const int64_t r = row - g.row0;
    if (r < 0 || r >= g.rows)
        return;
    if (g.xdt == 0)
        quantize_one_row<float>(static_cast<const float *>(g.x) + r * g.ldx, g.cols, g.q + r * g.cols,
                                g.scales + r, 0, red);
    else
        quantize_one_row<__half>(static_cast<const __half *>(g.x) + r * g.ldx, g.cols, g.q + r * g.cols,
                                 g.scales + r, 0, red);
}

// ------------------------------------------------------------------ per-tensor scaling
// "C++ and FP8" §5.1 (MINMAX calibration: the scale follows the largest
// magnitude over calibration data) and "7B on an RTX 4060 with FP8" §6.1
// (delayed scaling over an amax history of length >= 1024, scale below
// 448).  amax = max |x| over the tensor (NaN ignored, as the per-row
// quantisation); scale = RN(amax / 448), 1 when 0.  A delayed step
// quantises with the scale carried from the previous step: RN(max of the
// last H amaxes / 448).

// Device layout of pgf8_delayed_state (16 bytes).
struct DelayedState {
    float initial_scale;   // the scale of step 0
    unsigned pending[3];   // amax of step t accumulates in pending[t % 3] (bits of a non-negative float)
};

__device__ __forceinline__ float per_tensor_scale(float amax)
{
    const float s = __fdiv_rn(amax, 448.0f);
    return s == 0.0f ? 1.0f : s;
}

// *amax = max(*amax, max |x|): grid-stride over 16-element chunks, warp max,
// one atomic max per warp on the bits (non-negative floats, +0 start).
template <typename T>
__global__ void __launch_bounds__(kQuantThreads) amax_accumulate_kernel(const T *__restrict__ x, int64_t rows,
                                                                        int64_t cols, int64_t ldx,
                                                                        unsigned *__restrict__ amax_bits)
{
    const int64_t nch = cols / 16, total = rows * nch;
    float m = 0.0f;
    for (int64_t c = blockIdx.x * static_cast<int64_t>(kQuantThreads) + threadIdx.x; c < total;
         c += static_cast<int64_t>(gridDim.x) * kQuantThreads) {
        const int64_t r = c / nch, k = (c - r * nch) * 16;
        Vec16<T> v;
        v.load(x + r * ldx + k);
#pragma unroll
        for (int i = 0; i < 16; ++i)
            m = fmaxf(m, fabsf(v.v[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0 && m > 0.0f)
        atomicMax(amax_bits, __float_as_uint(m));
}

// Quantises one row with a per-tensor scale that get_scale() produces (a
// read of device state, possibly a CTA-wide reduction); returns the row's
// amax (block-wide, valid in every thread).  Rows of up to kRegChunks x 256
// chunks are loaded into registers before get_scale() runs, so the row's
// load latency overlaps the scale's; longer rows are streamed after it.
template <typename T, typename GetScale>
__device__ __forceinline__ float quantize_row_scaled(const T *xr, int64_t cols, uint8_t *qr, float *red,
                                                     GetScale get_scale, float &s_out)
{
    const int64_t nchunk = cols / 16;
    float a = 0.0f;
    if (nchunk <= static_cast<int64_t>(kRegChunks) * kQuantThreads) {
        Vec16<T> v[kRegChunks];
#pragma unroll
        for (int u = 0; u < kRegChunks; ++u) {
            const int64_t c = threadIdx.x + static_cast<int64_t>(u) * kQuantThreads;
            if (c < nchunk)
                v[u].load(xr + c * 16);
        }
        const float s = get_scale();
        s_out = s;
        const RowDivisor d(s);
#pragma unroll
        for (int u = 0; u < kRegChunks; ++u) {
            const int64_t c = threadIdx.x + static_cast<int64_t>(u) * kQuantThreads;
            if (c < nchunk) {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    a = fmaxf(a, fabsf(v[u].v[i]));
                *reinterpret_cast<uint4 *>(qr + c * 16) = encode16(v[u].v, d);
            }
        }
    } else {
        const float s = get_scale();
        s_out = s;
        const RowDivisor d(s);
        for (int64_t c = threadIdx.x; c < nchunk; c += kQuantThreads) {
            Vec16<T> v;
            v.load(xr + c * 16);
#pragma unroll
            for (int i = 0; i < 16; ++i)
                a = fmaxf(a, fabsf(v.v[i]));
            *reinterpret_cast<uint4 *>(qr + c * 16) = encode16(v.v, d);
        }
    }
    return block_max(a, red);
}

// Static per-tensor quantisation with the scale of a calibrated amax; one
// CTA per row.
template <typename T>
__global__ void __launch_bounds__(kQuantThreads) quantize_tensor_kernel(const T *__restrict__ x, int64_t cols,
                                                                        int64_t ldx, const float *__restrict__ amax,
                                                                        uint8_t *__restrict__ q,
                                                                        float *__restrict__ scales)
{
    __shared__ float red[kQuantThreads / 32];
    // a dependent GEMM launched with programmatic serialization may load its
    // weights now; it reads q / scales only after this grid has completed
    grid_launch_dependents();
    // launched with programmatic serialization, the previous kernel may still
    // run: nothing is read or written before it has completed
    grid_dependency_wait();
    const int64_t row = blockIdx.x;
    float s;
    (void)quantize_row_scaled(x + row * ldx, cols, q + row * cols, red, [&] { return per_tensor_scale(*amax); }, s);
    if (scales && threadIdx.x == 0)
        scales[row] = s;
}

// Step t of delayed scaling; one CTA per row.  The scale of step t is the
// scale carried out of step t-1: max over the last H amaxes (steps t-H ..
// t-1) / 448.  The history ring holds the amaxes up to step t-2; step t-1's
// amax is still pending (accumulated by its CTAs), so every CTA takes
//   max(history without slot (t-1) mod H, pending[(t-1) % 3])
// (that slot held step t-1-H, which leaves the window), and CTA 0 files the
// pending amax into the slot and clears the buffer step t+1 accumulates
// into.  Each CTA then quantises its row and folds the row amax into
// pending[t % 3].  Nothing waits on another CTA and nothing runs after the
// quantisation; step t = 0 uses the initial scale.
template <typename T>
__global__ void __launch_bounds__(kQuantThreads) quantize_delayed_kernel(const T *__restrict__ x, int64_t cols,
                                                                         int64_t ldx, uint8_t *__restrict__ q,
                                                                         float *__restrict__ scales,
                                                                         float *__restrict__ history, int H,
                                                                         DelayedState *st, int64_t t)
{
    __shared__ float red[kQuantThreads / 32];
    grid_launch_dependents();   // as in quantize_tensor_kernel
    grid_dependency_wait();
    const int64_t row = blockIdx.x;
    auto carried_scale = [&]() -> float {
        if (t == 0)
            return st->initial_scale;
        const int slot = static_cast<int>((t - 1) % H);
        const float prev = __uint_as_float(st->pending[(t - 1) % 3]);
        float m = prev;
        for (int i = threadIdx.x; i < H; i += kQuantThreads)
            if (i != slot)
                m = fmaxf(m, history[i]);
        const float sc = per_tensor_scale(block_max(m, red));
        __syncthreads();   // red is reused by the row's amax
        if (blockIdx.x == 0 && threadIdx.x == 0)
            history[slot] = prev;
        return sc;
    };
    if (blockIdx.x == 0 && threadIdx.x == 0)
        st->pending[(t + 1) % 3] = 0u;
    float s;
    const float m = quantize_row_scaled(x + row * ldx, cols, q + row * cols, red, carried_scale, s);
    if (threadIdx.x == 0) {
        if (scales)
            scales[row] = s;
        if (m > 0.0f)
            atomicMax(&st->pending[t % 3], __float_as_uint(m));
    }
}

// Fresh delayed-scaling state: history zero, nothing pending, step 0 at the
// given scale.
__global__ void __launch_bounds__(kQuantThreads) delayed_init_kernel(float *__restrict__ history, int H,
                                                                     DelayedState *st, float initial_scale)
{
    for (int i = blockIdx.x * kQuantThreads + threadIdx.x; i < H; i += gridDim.x * kQuantThreads)
        history[i] = 0.0f;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        st->initial_scale = initial_scale;
        st->pending[0] = st->pending[1] = st->pending[2] = 0u;
    }
}

// ------------------------------------------------------------------ norm / gate + quantisation
// "7B on an RTX 4060 with FP8", computation graph §2.1: LayerNorm fused with
// the QKV projection's input.  Here the normalisation (LayerNorm, or
// RMSNorm for the Llama shapes) runs in the quantisation kernel that feeds
// the projection, and the SiLU gate in the one that feeds the down
// projection, so neither intermediate goes to memory:
//   LayerNorm y = (x - mean) * rsqrt(var + eps) * gamma + beta  (biased var)
//   RMSNorm   y = x * rsqrt(mean(x^2) + eps) * gamma
//   gate      h = g / (1 + exp(-g)) * u
// in binary32, then per-token E4M3 as quantize_rows (amax, RN(amax/448),
// RN(y/s) saturating).

template <> struct Vec16<__nv_bfloat16> {
    float v[16];
    __device__ __forceinline__ void load(const __nv_bfloat16 *p)
    {
        const uint4 *q = reinterpret_cast<const uint4 *>(p);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            uint4 t = __ldg(q + i);
            uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                // bf16 -> f32 is exact: the bf16 bits are the f32's upper half
                v[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
                v[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
            }
        }
    }
};

__device__ __forceinline__ float block_sum(float v, float *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();   // red may still be read by a previous reduction
    if (lane == 0)
        red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < (kQuantThreads / 32) ? red[lane] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0)
            red[0] = v;
    }
    __syncthreads();
    return red[0];
}

// Encodes the row held in registers (y values), writes codes and the scale.
__device__ __forceinline__ void quantize_held_row(Vec16<float> (&y)[kRegChunks], int64_t nchunk, uint8_t *qr,
                                                  float *scale_out, float *red)
{
    float a = 0.0f;
#pragma unroll
    for (int u = 0; u < kRegChunks; ++u) {
        const int64_t c = threadIdx.x + static_cast<int64_t>(u) * kQuantThreads;
        if (c < nchunk) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                a = fmaxf(a, fabsf(y[u].v[i]));
        }
    }
    __syncthreads();   // red may still be read by a previous reduction
    a = block_max(a, red);
    float s = __fdiv_rn(a, 448.0f);
    if (s == 0.0f)
        s = 1.0f;
    const RowDivisor d(s);
#pragma unroll
    for (int u = 0; u < kRegChunks; ++u) {
        const int64_t c = threadIdx.x + static_cast<int64_t>(u) * kQuantThreads;
        if (c < nchunk)
            *reinterpret_cast<uint4 *>(qr + c * 16) = encode16(y[u].v, d);
    }
    if (threadIdx.x == 0)
        *scale_out = s;
}

// One CTA per row; rows of up to kRegChunks x 256 x 16 elements (held in
// registers).  beta == nullptr: RMSNorm.
template <typename T>
__global__ void __launch_bounds__(kQuantThreads) norm_quantize_kernel(const T *__restrict__ x, int64_t cols,
                                                                      int64_t ldx, const float *__restrict__ gamma,
                                                                      const float *__restrict__ beta, float eps,
                                                                      uint8_t *__restrict__ q,
                                                                      float *__restrict__ scales)
{
    __shared__ float red[kQuantThreads / 32];
    grid_launch_dependents();   // a dependent GEMM reads q / scales only after this grid completes
    grid_dependency_wait();
    const int64_t row = blockIdx.x;
    const T *xr = x + row * ldx;
    const int64_t nchunk = cols / 16;
    Vec16<float> v[kRegChunks];
#pragma unroll
    for (int u = 0; u < kRegChunks; ++u) {
        const int64_t c = threadIdx.x + static_cast<int64_t>(u) * kQuantThreads;
        if (c < nchunk) {
            Vec16<T> t;
            t.load(xr + c * 16);
#pragma unroll
            for (int i = 0; i < 16; ++i)
                v[u].v[i] = t.v[i];
        }
    }
    const float inv_n = 1.0f / static_cast<float>(cols);
    float mean = 0.0f;
    if (beta) {
        float sum = 0.0f;
#pragma unroll
        for (int u = 0; u < kRegChunks; ++u) {
            const int64_t c = threadIdx.x + static_cast<int64_t>(u) * kQuantThreads;
            if (c < nchunk) {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    sum += v[u].v[i];
            }
        }
        mean = block_sum(sum, red) * inv_n;
    }
    float ss = 0.0f;
#pragma unroll
    for (int u = 0; u < kRegChunks; ++u) {
        const int64_t c = threadIdx.x + static_cast<int64_t>(u) * kQuantThreads;
        if (c < nchunk) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float d = v[u].v[i] - mean;
                ss = fmaf(d, d, ss);
            }
        }
    }
    const float rstd = __frsqrt_rn(block_sum(ss, red) * inv_n + eps);
#pragma unroll
    for (int u = 0; u < kRegChunks; ++u) {
        const int64_t c = threadIdx.x + static_cast<int64_t>(u) * kQuantThreads;
        if (c < nchunk) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int64_t k = c * 16 + i;
                float y = (v[u].v[i] - mean) * rstd * __ldg(gamma + k);
                if (beta)
                    y += __ldg(beta + k);
                v[u].v[i] = y;
            }
        }
    }
    quantize_held_row(v, nchunk, q + row * cols, scales + row, red);
}

__device__ __forceinline__ float silu_mul(float g, float u)
{
    return __fdiv_rn(g, 1.0f + expf(-g)) * u;
}

// One CTA per row of the gate+up output gu [rows, 2I] (gate = columns
// [0, I), up = [I, 2I)); h [rows, I] is quantised.  Rows of up to
// kRegChunks x 256 x 16 elements are held in registers; longer rows are
// computed twice (amax pass, then the codes), identically.
template <typename T>
__global__ void __launch_bounds__(kQuantThreads) silu_mul_quantize_kernel(const T *__restrict__ gu, int64_t inter,
                                                                          int64_t ldg, uint8_t *__restrict__ q,
                                                                          float *__restrict__ scales)
{
    __shared__ float red[kQuantThreads / 32];
    grid_launch_dependents();
    grid_dependency_wait();
    const int64_t row = blockIdx.x;
    const T *gr = gu + row * ldg;
    const T *ur = gr + inter;
    uint8_t *qr = q + row * inter;
    const int64_t nchunk = inter / 16;
    if (nchunk <= static_cast<int64_t>(kRegChunks) * kQuantThreads) {
        Vec16<float> h[kRegChunks];
#pragma unroll
        for (int u = 0; u < kRegChunks; ++u) {
            const int64_t c = threadIdx.x + static_cast<int64_t>(u) * kQuantThreads;
            if (c < nchunk) {
                Vec16<T> g, up;
                g.load(gr + c * 16);
                up.load(ur + c * 16);
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    h[u].v[i] = silu_mul(g.v[i], up.v[i]);
            }
        }
        quantize_held_row(h, nchunk, qr, scales + row, red);
        return;
    }
    float a = 0.0f;
    for (int64_t c = threadIdx.x; c < nchunk; c += kQuantThreads) {
        Vec16<T> g, up;
        g.load(gr + c * 16);
        up.load(ur + c * 16);
#pragma unroll
        for (int i = 0; i < 16; ++i)
            a = fmaxf(a, fabsf(silu_mul(g.v[i], up.v[i])));
    }
    a = block_max(a, red);
    float s = __fdiv_rn(a, 448.0f);
    if (s == 0.0f)
        s = 1.0f;
    const RowDivisor d(s);
    for (int64_t c = threadIdx.x; c < nchunk; c += kQuantThreads) {
        Vec16<T> g, up;
        g.load(gr + c * 16);
        up.load(ur + c * 16);
        float hv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            hv[i] = silu_mul(g.v[i], up.v[i]);
        *reinterpret_cast<uint4 *>(qr + c * 16) = encode16(hv, d);
    }
    if (threadIdx.x == 0)
        scales[row] = s;
}

// NestedFP split: 8 FP16 bit patterns per thread per step (16 bytes in, 8 + 8 out).
// y = bf16_rn(x), 8 elements per step (the final rounding of a
// tensor-parallel layer's f32 sum).
__global__ void __launch_bounds__(256) round_bf16_kernel(const float4 *__restrict__ x, int64_t n8,
                                                         uint4 *__restrict__ y)
{
    grid_dependency_wait();
    for (int64_t i = blockIdx.x * 256ll + threadIdx.x; i < n8; i += static_cast<int64_t>(gridDim.x) * 256) {
        const float4 a = x[2 * i], b = x[2 * i + 1];
        const __nv_bfloat162 p0 = __floats2bfloat162_rn(a.x, a.y), p1 = __floats2bfloat162_rn(a.z, a.w);
        const __nv_bfloat162 p2 = __floats2bfloat162_rn(b.x, b.y), p3 = __floats2bfloat162_rn(b.z, b.w);
        y[i] = make_uint4(*reinterpret_cast<const uint32_t *>(&p0), *reinterpret_cast<const uint32_t *>(&p1),
                          *reinterpret_cast<const uint32_t *>(&p2), *reinterpret_cast<const uint32_t *>(&p3));
    }
}

__global__ void __launch_bounds__(256) nestedfp_split_kernel(const uint4 *__restrict__ w, int64_t n8,
                                                             uint2 *__restrict__ hi, uint2 *__restrict__ lo)
{
    for (int64_t i = blockIdx.x * 256ll + threadIdx.x; i < n8; i += static_cast<int64_t>(gridDim.x) * 256) {
        const uint4 t = __ldg(w + i);
        // bytes of the 8 halves, little endian: half e = bytes (2e: low, 2e+1: high)
        uint2 h, l;
        h.x = __byte_perm(t.x, t.y, 0x7531);
        h.y = __byte_perm(t.z, t.w, 0x7531);
        l.x = __byte_perm(t.x, t.y, 0x6420);
        l.y = __byte_perm(t.z, t.w, 0x6420);
        hi[i] = h;
        lo[i] = l;
    }
}

} // namespace pgf8
