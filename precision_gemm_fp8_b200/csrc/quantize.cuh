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

// Converts 16 binary32 values (already divided by the scale) to 16 codes.
__device__ __forceinline__ uint4 encode16(const float (&v)[16], float s)
{
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t lo = cvt_e4m3x2(__fdiv_rn(v[4 * i + 0], s), __fdiv_rn(v[4 * i + 1], s));
        const uint32_t hi = cvt_e4m3x2(__fdiv_rn(v[4 * i + 2], s), __fdiv_rn(v[4 * i + 3], s));
        w[i] = lo | (hi << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Rows of up to kRegChunks * kQuantThreads * 16 elements stay in registers
// between the amax and the conversion (one pass over global memory);
// longer rows are re-read (from L2) for the conversion.
constexpr int kRegChunks = 4;

// One CTA per row.  cols % 16 == 0; x rows 16-byte aligned.
// trigger_early: let a dependent kernel launched with programmatic stream
// serialization be scheduled at once (used only when that dependent is the
// library's own GEMM, which reads q/scales after this grid completes).
template <typename T>
__global__ void __launch_bounds__(kQuantThreads) quantize_rows_kernel(const T *__restrict__ x, int64_t rows,
                                                                      int64_t cols, int64_t ldx,
                                                                      uint8_t *__restrict__ q,
                                                                      float *__restrict__ scales, int mode,
                                                                      int trigger_early)
{
    __shared__ float red[kQuantThreads / 32];
    if (trigger_early)
        grid_launch_dependents();
    // When launched with programmatic serialization, the previous kernel in
    // the stream may still run: nothing is read or written before it ends.
    grid_dependency_wait();
    const int64_t row = blockIdx.x;
    if (row >= rows)
        return;
    const T *xr = x + row * ldx;
    uint8_t *qr = q + row * cols;
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
        if (mode == 0) {
            amax = block_max(amax, red);
            s = __fdiv_rn(amax, 448.0f);
            if (s == 0.0f)
                s = 1.0f;
            if (threadIdx.x == 0)
                scales[row] = s;
        } else {
            s = scales[row];
        }
#pragma unroll
        for (int u = 0; u < kRegChunks; ++u) {
            const int64_t c = threadIdx.x + static_cast<int64_t>(u) * kQuantThreads;
            if (c < nchunk)
                *reinterpret_cast<uint4 *>(qr + c * 16) = encode16(v[u].v, s);
        }
        return;
    }

    float s;
    if (mode == 0) {
        float amax = 0.0f;
        for (int64_t c = threadIdx.x; c < nchunk; c += kQuantThreads) {
            Vec16<T> v;
            v.load(xr + c * 16);
#pragma unroll
            for (int i = 0; i < 16; ++i)
                amax = fmaxf(amax, fabsf(v.v[i]));
        }
        amax = block_max(amax, red);
        s = __fdiv_rn(amax, 448.0f);
        if (s == 0.0f)
            s = 1.0f;
        if (threadIdx.x == 0)
            scales[row] = s;
    } else {
        s = scales[row];
    }
    for (int64_t c = threadIdx.x; c < nchunk; c += kQuantThreads) {
        Vec16<T> v;
        v.load(xr + c * 16);
        *reinterpret_cast<uint4 *>(qr + c * 16) = encode16(v.v, s);
    }
}

// NestedFP split: 8 FP16 bit patterns per thread per step (16 bytes in, 8 + 8 out).
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
