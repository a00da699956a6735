// Decode attention over the FP8 (E4M3) paged KV cache.
//
// "7B on an RTX 4060 with FP8": K/V held in FP8, dequantised on use;
// "C++ and FP8" §3.2 (paged cache of 16-token blocks kept in FP8) and §3.3
// (attention in the FP8 dataflow).  This library's reading: one query row
// per sequence (the token being generated, at position ctx - 1, which sees
// every cached position 0 .. ctx - 1), grouped query heads (query head h
// reads KV head h / (Hq / Hkv)), scores q.k * s_k / sqrt(D), softmax over
// the context, output sum p * v * s_v.
//
// HBM-bound: a decoded token costs 2·D bytes of K and V codes against about
// 4·G·D flops for the G query heads that share its KV head.  The first
// kernel streams the cache with 128-bit (K) and coalesced (V) loads on the
// CUDA cores, which keep up with HBM for one or two heads per KV head; the
// second (attn_decode_mma_kernel, on request) puts both products on the
// tensor cores with the heads as the MMA's N dimension, for larger groups.
// The context is split into chunks ("flash-decoding"): one CTA per
// (chunk, KV head, group of GT query heads, sequence) keeps each SM busy
// when the batch is small.  Each CTA reduces its chunk to a running maximum
// m, a sum l and an unnormalised output o per query head (online softmax,
// base-2 exponent with log2(e) folded into the query scale); a second
// kernel merges the chunks in chunk order, so results do not depend on
// scheduling.  With one chunk the first kernel writes the output itself.
//
// Warp step: 16 positions of one block (block_size is a multiple of 16).
// Lanes 2t and 2t+1 take position t for the scores, each half of the
// 16-byte pieces of its K row (interleaved, so the two halves read
// different shared-memory banks of q); every lane then owns D/32 adjacent
// dims of the output and reads them from each V row (one coalesced
// 32 x D/32-byte row per position).  Positions at or past the context end
// are neither scored nor read from V.  A block-table entry outside
// [0, num_blocks) is counted into *errors and its 16 positions skipped;
// nothing outside the cache is read.
#pragma once

#include <cuda_fp8.h>

#include "quantize.cuh"

namespace pgf8 {

constexpr int kAttnWarps = 4;
constexpr int kAttnThreads = 32 * kAttnWarps;
constexpr int kAttnStep = 16;   // positions per warp step

struct AttnDecodeArgs {
    const void *q;        // [seqs][Hq][D], sequence stride ldq elements
    int64_t ldq;
    int qdt;              // 0 f32, 1 f16, 2 bf16
    const uint8_t *kc;    // [num_blocks][Hkv][B][D] E4M3 codes
    const uint8_t *vc;
    const float *sk;      // [Hkv]
    const float *sv;
    const int32_t *tables;   // [seqs][table_stride]
    int64_t table_stride;
    const int32_t *ctx_lens; // [seqs]
    int64_t num_blocks, Hkv, Hq, B;
    int64_t max_ctx;      // every context is clamped to it (and counted when longer)
    int64_t chunk;        // positions per split, a multiple of 16
    int nsplit;
    int groups;           // CTAs (groups of GT query heads) per KV head
    float qscale;         // log2(e) / sqrt(D)
    void *out;            // [seqs][Hq][D], sequence stride ldo elements
    int64_t ldo;
    int odt;
    float *part;          // [seqs][Hq][nsplit][D + 2]: o[D], m, l (nsplit > 1)
    int32_t *errors;
};

__device__ __forceinline__ float load_elem(const void *p, int64_t i, int dt)
{
    if (dt == 0)
        return static_cast<const float *>(p)[i];
    if (dt == 1)
        return __half2float(static_cast<const __half *>(p)[i]);
    return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
}

__device__ __forceinline__ void store_elem(void *p, int64_t i, int dt, float v)
{
    if (dt == 0)
        static_cast<float *>(p)[i] = v;
    else if (dt == 1)
        static_cast<__half *>(p)[i] = __float2half_rn(v);
    else
        static_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(v);
}

// Two E4M3 codes (low byte first) -> two binary32 values.  Exact: every
// E4M3 value is a binary16 value and every binary16 value a binary32 one.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t two)
{
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xFFFFu), __NV_E4M3);
    return __half22float2(__half2(h));
}

// N (2, 4 or 8) adjacent E4M3 codes of one row, loaded as one word.
template <int N> struct CodesN;
template <> struct CodesN<2> {
    uint32_t w;
    __device__ __forceinline__ void load(const uint8_t *p) { w = *reinterpret_cast<const uint16_t *>(p); }
    __device__ __forceinline__ void zero() { w = 0; }
    __device__ __forceinline__ void decode(float (&f)[2]) const
    {
        const float2 a = e4m3x2_to_float2(w);
        f[0] = a.x;
        f[1] = a.y;
    }
};
template <> struct CodesN<4> {
    uint32_t w;
    __device__ __forceinline__ void load(const uint8_t *p) { w = __ldg(reinterpret_cast<const unsigned int *>(p)); }
    __device__ __forceinline__ void zero() { w = 0; }
    __device__ __forceinline__ void decode(float (&f)[4]) const
    {
        const float2 a = e4m3x2_to_float2(w), b = e4m3x2_to_float2(w >> 16);
        f[0] = a.x;
        f[1] = a.y;
        f[2] = b.x;
        f[3] = b.y;
    }
};
template <> struct CodesN<8> {
    uint2 w;
    __device__ __forceinline__ void load(const uint8_t *p) { w = __ldg(reinterpret_cast<const uint2 *>(p)); }
    __device__ __forceinline__ void zero() { w = make_uint2(0, 0); }
    __device__ __forceinline__ void decode(float (&f)[8]) const
    {
        const float2 a = e4m3x2_to_float2(w.x), b = e4m3x2_to_float2(w.x >> 16);
        const float2 c = e4m3x2_to_float2(w.y), d = e4m3x2_to_float2(w.y >> 16);
        f[0] = a.x;
        f[1] = a.y;
        f[2] = b.x;
        f[3] = b.y;
        f[4] = c.x;
        f[5] = c.y;
        f[6] = d.x;
        f[7] = d.y;
    }
};

// 16 codes of one 128-bit word -> 16 binary32 values.
__device__ __forceinline__ void decode16(const uint4 &c, float (&f)[16])
{
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 a = e4m3x2_to_float2(w[i]), b = e4m3x2_to_float2(w[i] >> 16);
        f[4 * i + 0] = a.x;
        f[4 * i + 1] = a.y;
        f[4 * i + 2] = b.x;
        f[4 * i + 3] = b.y;
    }
}

template <int D, int GT>
__global__ void __launch_bounds__(kAttnThreads) attn_decode_paged_kernel(const AttnDecodeArgs a)
{
    static_assert(D == 64 || D == 128 || D == 256, "head_dim 64, 128 or 256");
    static_assert(GT == 1 || GT == 2 || GT == 4 || GT == 8, "query heads per CTA");
    constexpr int KW = D / 32;    // 16-byte K pieces per lane (half a row)
    constexpr int DPL = D / 32;   // output dims (and V codes) per lane

    __shared__ __align__(16) float qs[GT][D];
    __shared__ __align__(16) float ps[kAttnWarps][kAttnStep][GT];
    __shared__ float red_m[kAttnWarps][GT], red_l[kAttnWarps][GT];
    __shared__ __align__(16) float red_o[kAttnWarps][GT][D];

    grid_launch_dependents();
    grid_dependency_wait();   // q from the QKV projection, the cache from its writer

    const int sp = blockIdx.x;
    const int64_t hk = blockIdx.y / a.groups;
    const int64_t h0 = hk * (a.Hq / a.Hkv) + static_cast<int64_t>(blockIdx.y % a.groups) * GT;
    const int64_t s = blockIdx.z;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const float c = a.sk[hk] * a.qscale;
    for (int i = threadIdx.x; i < GT * D; i += kAttnThreads)
        qs[i / D][i % D] = load_elem(a.q, s * a.ldq + (h0 + i / D) * D + i % D, a.qdt) * c;

    int64_t ctx = a.ctx_lens[s];
    if (ctx < 0 || ctx > a.max_ctx) {
        if (a.errors && threadIdx.x == 0 && sp == 0 && blockIdx.y == 0)
            atomicAdd(a.errors, 1);
        ctx = ctx < 0 ? 0 : a.max_ctx;
    }
    const int64_t t_begin = static_cast<int64_t>(sp) * a.chunk;
    const int64_t t_end = t_begin + a.chunk < ctx ? t_begin + a.chunk : ctx;
    __syncthreads();

    float m[GT], l[GT], o[GT][DPL];
#pragma unroll
    for (int g = 0; g < GT; ++g) {
        m[g] = -INFINITY;
        l[g] = 0.0f;
#pragma unroll
        for (int i = 0; i < DPL; ++i)
            o[g][i] = 0.0f;
    }

    const int tq = lane >> 1, hf = lane & 1;
    for (int64_t base = t_begin + kAttnStep * w; base < t_end; base += kAttnStep * kAttnWarps) {
        const int nvalid = t_end - base < kAttnStep ? static_cast<int>(t_end - base) : kAttnStep;
        const int64_t blk = a.tables[s * a.table_stride + base / a.B];
        if (blk < 0 || blk >= a.num_blocks) {   // warp-uniform
            if (a.errors && lane == 0 && blockIdx.y == 0)
                atomicAdd(a.errors, 1);
            continue;
        }
        const int64_t row0 = (blk * a.Hkv + hk) * a.B + base % a.B;   // cache row of position `base`
        const uint8_t *krow = a.kc + (row0 + tq) * D;
        const uint8_t *vrow = a.vc + row0 * D + lane * DPL;

        // issue every load of the step before any arithmetic
        const bool kval = tq < nvalid;
        uint4 kw[KW];
#pragma unroll
        for (int i = 0; i < KW; ++i)
            kw[i] = kval ? __ldg(reinterpret_cast<const uint4 *>(krow + 16 * (2 * i + hf))) : make_uint4(0, 0, 0, 0);
        CodesN<DPL> vw[kAttnStep];
#pragma unroll
        for (int t = 0; t < kAttnStep; ++t) {
            if (t < nvalid)
                vw[t].load(vrow + static_cast<int64_t>(t) * D);
            else
                vw[t].zero();
        }

        // scores: this lane's half of q . k for each query head
        float dot[GT];
#pragma unroll
        for (int g = 0; g < GT; ++g)
            dot[g] = 0.0f;
#pragma unroll
        for (int i = 0; i < KW; ++i) {
            float kf[16];
            decode16(kw[i], kf);
            const int d0 = 16 * (2 * i + hf);
#pragma unroll
            for (int g = 0; g < GT; ++g) {
                const float4 *qv = reinterpret_cast<const float4 *>(&qs[g][d0]);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float4 qq = qv[j];
                    dot[g] = fmaf(qq.x, kf[4 * j + 0], dot[g]);
                    dot[g] = fmaf(qq.y, kf[4 * j + 1], dot[g]);
                    dot[g] = fmaf(qq.z, kf[4 * j + 2], dot[g]);
                    dot[g] = fmaf(qq.w, kf[4 * j + 3], dot[g]);
                }
            }
        }

        // online softmax over the step's positions (base-2 units)
#pragma unroll
        for (int g = 0; g < GT; ++g) {
            const float full = dot[g] + __shfl_xor_sync(0xffffffffu, dot[g], 1);
            const float sc = kval ? full : -INFINITY;
            float mx = sc;
#pragma unroll
            for (int off = 2; off < 32; off <<= 1)
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float mn = fmaxf(m[g], mx);   // finite: position `base` is valid
            const float alpha = m[g] == -INFINITY ? 0.0f : exp2f(m[g] - mn);
            const float p = kval ? exp2f(sc - mn) : 0.0f;
            float psum = p;
#pragma unroll
            for (int off = 2; off < 32; off <<= 1)
                psum += __shfl_xor_sync(0xffffffffu, psum, off);
            l[g] = l[g] * alpha + psum;
            m[g] = mn;
#pragma unroll
            for (int i = 0; i < DPL; ++i)
                o[g][i] *= alpha;
            if (hf == 0)
                ps[w][tq][g] = p;
        }
        __syncwarp();

        // o += p . v over the valid positions
#pragma unroll
        for (int t = 0; t < kAttnStep; ++t) {
            if (t < nvalid) {
                float vf[DPL];
                vw[t].decode(vf);
#pragma unroll
                for (int g = 0; g < GT; ++g) {
                    const float p = ps[w][t][g];
#pragma unroll
                    for (int i = 0; i < DPL; ++i)
                        o[g][i] = fmaf(p, vf[i], o[g][i]);
                }
            }
        }
        __syncwarp();   // ps is rewritten by the next step
    }

    // merge the warps' partial softmax states
#pragma unroll
    for (int g = 0; g < GT; ++g) {
        if (lane == 0) {
            red_m[w][g] = m[g];
            red_l[w][g] = l[g];
        }
#pragma unroll
        for (int i = 0; i < DPL; ++i)
            red_o[w][g][lane * DPL + i] = o[g][i];
    }
    __syncthreads();

    const float vscale = a.sv[hk];
    for (int e = threadIdx.x; e < GT * D; e += kAttnThreads) {
        const int g = e / D, d = e % D;
        float M = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < kAttnWarps; ++ww)
            M = fmaxf(M, red_m[ww][g]);
        float L = 0.0f, O = 0.0f;
#pragma unroll
        for (int ww = 0; ww < kAttnWarps; ++ww) {
            if (red_m[ww][g] != -INFINITY) {
                const float f = exp2f(red_m[ww][g] - M);
                L = fmaf(red_l[ww][g], f, L);
                O = fmaf(red_o[ww][g][d], f, O);
            }
        }
        const int64_t h = h0 + g;
        if (a.nsplit == 1) {
            store_elem(a.out, s * a.ldo + h * D + d, a.odt, L > 0.0f ? O / L * vscale : 0.0f);
        } else {
            float *pp = a.part + ((s * a.Hq + h) * a.nsplit + sp) * (D + 2);
            pp[d] = O;
            if (d == 0) {
                pp[D] = M;
                pp[D + 1] = L;
            }
        }
    }
}

// Merges the nsplit chunk states of one (sequence, query head) per CTA, in
// chunk order; thread d writes output dim d.
template <int D>
__global__ void __launch_bounds__(D) attn_decode_combine_kernel(const float *__restrict__ part, int nsplit, int64_t Hq,
                                                                 int64_t Hkv, const float *__restrict__ sv, void *out,
                                                                 int64_t ldo, int odt)
{
    grid_launch_dependents();
    grid_dependency_wait();   // the chunk states of the kernel before
    const int64_t sh = blockIdx.x;   // s * Hq + h
    const int64_t s = sh / Hq, h = sh % Hq;
    const int d = threadIdx.x;
    const float *pp = part + sh * nsplit * (D + 2);
    float M = -INFINITY;
    for (int i = 0; i < nsplit; ++i)
        M = fmaxf(M, pp[i * (D + 2) + D]);
    float L = 0.0f, O = 0.0f;
    for (int i = 0; i < nsplit; ++i) {
        const float mi = pp[i * (D + 2) + D];
        if (mi != -INFINITY) {
            const float f = exp2f(mi - M);
            L = fmaf(pp[i * (D + 2) + D + 1], f, L);
            O = fmaf(pp[i * (D + 2) + d], f, O);
        }
    }
    store_elem(out, s * ldo + h * D + d, odt, L > 0.0f ? O / L * sv[h / (Hq / Hkv)] : 0.0f);
}

// ---------------------------------------------------------------------------
// The same decode attention with both products on the tensor cores
// (mma.sync m16n8k16, binary16 operands, binary32 accumulation), for query
// heads that share a KV head: the up to 8 heads of a CTA are the MMA's N
// dimension, so one K / V load serves all of them in one instruction.
//   scores^T [16 positions x 8 heads] = K [16 x D] . Q^T [D x 8]
//   O^T [D x 8 heads] += V^T [D x 16 positions] . P^T [16 x 8]
// K and V codes widen exactly to binary16 (cvt from E4M3 pairs); q and the
// probabilities are rounded to binary16.  The contraction index of each
// product is permuted (the sum does not depend on its order) so that every
// thread loads whole 16-byte pieces of the rows it needs: for QK, thread
// (g = lane / 4, t4 = lane % 4) holds bytes [D/4 t4, D/4 t4 + D/4) of
// positions g and g + 8, k-step j taking bytes 4j .. 4j + 3 of that piece;
// for PV it holds bytes [D/8 g, D/8 g + D/8) of positions 4 t4 .. 4 t4 + 3,
// output block b taking dims D/8 g + 2b (MMA row g) and D/8 g + 2b + 1
// (row g + 8).  The probabilities move from the score layout (positions
// g, g + 8; heads 2 t4, 2 t4 + 1) to the operand layout (heads g;
// positions 4 t4 .. 4 t4 + 3) through 256 bytes of shared memory per warp.
// Grid, chunks, masks, merge and outputs as attn_decode_paged_kernel.

__device__ __forceinline__ uint32_t e4m3x2_to_h2bits(uint32_t two)
{
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xFFFFu), __NV_E4M3);
    return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

__device__ __forceinline__ uint32_t f32x2_to_h2bits(float lo, float hi)
{
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// D(16x8, f32) += A(16x16, f16, row) . B(16x8, f16, col)
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                 "{%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// N / 4 32-bit words of one row piece, loaded as 16-byte (or 8-byte) words.
template <int NBYTES> struct RowPiece {
    static constexpr int kWords = NBYTES / 4;
    uint32_t w[kWords];
    __device__ __forceinline__ void load(const uint8_t *p)
    {
        if constexpr (NBYTES == 8) {
            const uint2 t = __ldg(reinterpret_cast<const uint2 *>(p));
            w[0] = t.x;
            w[1] = t.y;
        } else {
#pragma unroll
            for (int i = 0; i < NBYTES / 16; ++i) {
                const uint4 t = __ldg(reinterpret_cast<const uint4 *>(p) + i);
                w[4 * i + 0] = t.x;
                w[4 * i + 1] = t.y;
                w[4 * i + 2] = t.z;
                w[4 * i + 3] = t.w;
            }
        }
    }
    __device__ __forceinline__ void zero()
    {
#pragma unroll
        for (int i = 0; i < kWords; ++i)
            w[i] = 0u;
    }
};

template <int D>
__global__ void __launch_bounds__(kAttnThreads) attn_decode_mma_kernel(const AttnDecodeArgs a)
{
    static_assert(D == 64 || D == 128 || D == 256, "head_dim 64, 128 or 256");
    constexpr int KSTEPS = D / 16;   // k-steps of the QK product
    constexpr int KSEG = D / 4;      // bytes of a K row per thread
    constexpr int VSEG = D / 8;      // bytes of a V row per thread
    constexpr int DB = D / 16;       // 16-row blocks of the PV product

    __shared__ __align__(16) __half ps[kAttnWarps][8][kAttnStep];   // probabilities [head][position]
    __shared__ float red_m[kAttnWarps][8], red_l[kAttnWarps][8];
    __shared__ __align__(16) float red_o[kAttnWarps][8][D];

    grid_launch_dependents();
    grid_dependency_wait();   // q from the QKV projection, the cache from its writer

    const int sp = blockIdx.x;
    const int G = static_cast<int>(a.Hq / a.Hkv);
    const int64_t hk = blockIdx.y / a.groups;
    const int gi = static_cast<int>(blockIdx.y % a.groups);
    const int nh = G - gi * 8 < 8 ? G - gi * 8 : 8;   // query heads of this CTA
    const int64_t h0 = hk * G + gi * 8;
    const int64_t s = blockIdx.z;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t4 = lane & 3;

    // Q^T operand of every k-step: head g (zero for the padding heads).  The
    // operand is binary16, so a head whose largest |q| reaches 2^14 is
    // scaled by 2^-e first (exact; q stays below 2^15 < 65504) and its scores
    // by 2^e after the product.
    float qmax = 0.0f;
    if (g < nh) {
#pragma unroll
        for (int j = 0; j < KSTEPS; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                qmax = fmaxf(qmax, fabsf(load_elem(a.q, s * a.ldq + (h0 + g) * D + KSEG * t4 + 4 * j + i, a.qdt)));
    }
    qmax = fmaxf(qmax, __shfl_xor_sync(0xffffffffu, qmax, 1));
    qmax = fmaxf(qmax, __shfl_xor_sync(0xffffffffu, qmax, 2));   // the 4 lanes of head g
    const int qexp = qmax >= 16384.0f && qmax <= 3.4e38f ? ilogbf(qmax) - 14 : 0;
    const float qpre = ldexpf(1.0f, -qexp);
    uint32_t qb[KSTEPS][2];
#pragma unroll
    for (int j = 0; j < KSTEPS; ++j) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int d = KSEG * t4 + 4 * j + 2 * e;
            float x0 = 0.0f, x1 = 0.0f;
            if (g < nh) {
                const int64_t base = s * a.ldq + (h0 + g) * D + d;
                x0 = load_elem(a.q, base, a.qdt) * qpre;
                x1 = load_elem(a.q, base + 1, a.qdt) * qpre;
            }
            qb[j][e] = f32x2_to_h2bits(x0, x1);
        }
    }

    int64_t ctx = a.ctx_lens[s];
    if (ctx < 0 || ctx > a.max_ctx) {
        if (a.errors && threadIdx.x == 0 && sp == 0 && blockIdx.y == 0)
            atomicAdd(a.errors, 1);
        ctx = ctx < 0 ? 0 : a.max_ctx;
    }
    const int64_t t_begin = static_cast<int64_t>(sp) * a.chunk;
    const int64_t t_end = t_begin + a.chunk < ctx ? t_begin + a.chunk : ctx;
    // base-2 units; the scores of heads 2 t4 and 2 t4 + 1 undo their pre-scale
    const float scale = a.sk[hk] * a.qscale;
    const float hscale[2] = {scale * ldexpf(1.0f, __shfl_sync(0xffffffffu, qexp, 8 * t4)),
                             scale * ldexpf(1.0f, __shfl_sync(0xffffffffu, qexp, 8 * t4 + 4))};

    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.0f, 0.0f};   // heads 2 t4, 2 t4 + 1
    float o[DB][4];
#pragma unroll
    for (int b = 0; b < DB; ++b)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            o[b][i] = 0.0f;

    for (int64_t base = t_begin + kAttnStep * w; base < t_end; base += kAttnStep * kAttnWarps) {
        const int nvalid = t_end - base < kAttnStep ? static_cast<int>(t_end - base) : kAttnStep;
        const int64_t blk = a.tables[s * a.table_stride + base / a.B];
        if (blk < 0 || blk >= a.num_blocks) {   // warp-uniform
            if (a.errors && lane == 0 && blockIdx.y == 0)
                atomicAdd(a.errors, 1);
            continue;
        }
        const int64_t row0 = (blk * a.Hkv + hk) * a.B + base % a.B;

        // every load of the step first; rows past the context read as zeros
        RowPiece<KSEG> k0, k1;
        if (g < nvalid)
            k0.load(a.kc + (row0 + g) * D + KSEG * t4);
        else
            k0.zero();
        if (g + 8 < nvalid)
            k1.load(a.kc + (row0 + g + 8) * D + KSEG * t4);
        else
            k1.zero();
        RowPiece<VSEG> v[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            if (4 * t4 + r < nvalid)
                v[r].load(a.vc + (row0 + 4 * t4 + r) * D + VSEG * g);
            else
                v[r].zero();
        }

        // scores^T = K . Q^T
        float c[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int j = 0; j < KSTEPS; ++j)
            mma_16816(c, e4m3x2_to_h2bits(k0.w[j]), e4m3x2_to_h2bits(k1.w[j]), e4m3x2_to_h2bits(k0.w[j] >> 16),
                      e4m3x2_to_h2bits(k1.w[j] >> 16), qb[j][0], qb[j][1]);

        // online softmax; c[0], c[1]: position g, heads 2 t4, 2 t4 + 1; c[2], c[3]: position g + 8
        const bool v0 = g < nvalid, v1 = g + 8 < nvalid;
        float pr[4];
        float alpha[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const float s0 = v0 ? c[hh] * hscale[hh] : -INFINITY;
            const float s1 = v1 ? c[2 + hh] * hscale[hh] : -INFINITY;
            float mx = fmaxf(s0, s1);
#pragma unroll
            for (int off = 4; off < 32; off <<= 1)
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float mn = fmaxf(m[hh], mx);   // finite: position `base` is valid
            alpha[hh] = m[hh] == -INFINITY ? 0.0f : exp2f(m[hh] - mn);
            pr[hh] = v0 ? exp2f(s0 - mn) : 0.0f;
            pr[2 + hh] = v1 ? exp2f(s1 - mn) : 0.0f;
            float psum = pr[hh] + pr[2 + hh];
#pragma unroll
            for (int off = 4; off < 32; off <<= 1)
                psum += __shfl_xor_sync(0xffffffffu, psum, off);
            l[hh] = l[hh] * alpha[hh] + psum;
            m[hh] = mn;
        }
#pragma unroll
        for (int b = 0; b < DB; ++b) {
            o[b][0] *= alpha[0];
            o[b][1] *= alpha[1];
            o[b][2] *= alpha[0];
            o[b][3] *= alpha[1];
        }
        ps[w][2 * t4][g] = __float2half_rn(pr[0]);
        ps[w][2 * t4 + 1][g] = __float2half_rn(pr[1]);
        ps[w][2 * t4][g + 8] = __float2half_rn(pr[2]);
        ps[w][2 * t4 + 1][g + 8] = __float2half_rn(pr[3]);
        __syncwarp();
        const uint2 pb = *reinterpret_cast<const uint2 *>(&ps[w][g][4 * t4]);   // positions 4 t4 .. 4 t4 + 3

        // O^T += V^T . P^T
#pragma unroll
        for (int b = 0; b < DB; ++b) {
            const int wi = b >> 1, sh = 2 * (b & 1);
            // bytes (row r byte sh, row r+1 byte sh, row r byte sh+1, row r+1 byte sh+1)
            const uint32_t sel = static_cast<uint32_t>(sh | ((4 + sh) << 4) | ((sh + 1) << 8) | ((5 + sh) << 12));
            const uint32_t x01 = __byte_perm(v[0].w[wi], v[1].w[wi], sel);
            const uint32_t x23 = __byte_perm(v[2].w[wi], v[3].w[wi], sel);
            mma_16816(o[b], e4m3x2_to_h2bits(x01), e4m3x2_to_h2bits(x01 >> 16), e4m3x2_to_h2bits(x23),
                      e4m3x2_to_h2bits(x23 >> 16), pb.x, pb.y);
        }
        __syncwarp();   // ps is rewritten by the next step
    }

    // merge the warps' partial softmax states
    if (g == 0) {
        red_m[w][2 * t4] = m[0];
        red_m[w][2 * t4 + 1] = m[1];
        red_l[w][2 * t4] = l[0];
        red_l[w][2 * t4 + 1] = l[1];
    }
#pragma unroll
    for (int b = 0; b < DB; ++b) {
        const int d = VSEG * g + 2 * b;
        red_o[w][2 * t4][d] = o[b][0];
        red_o[w][2 * t4 + 1][d] = o[b][1];
        red_o[w][2 * t4][d + 1] = o[b][2];
        red_o[w][2 * t4 + 1][d + 1] = o[b][3];
    }
    __syncthreads();

    const float vscale = a.sv[hk];
    for (int e = threadIdx.x; e < nh * D; e += kAttnThreads) {
        const int hh = e / D, d = e % D;
        float M = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < kAttnWarps; ++ww)
            M = fmaxf(M, red_m[ww][hh]);
        float L = 0.0f, O = 0.0f;
#pragma unroll
        for (int ww = 0; ww < kAttnWarps; ++ww) {
            if (red_m[ww][hh] != -INFINITY) {
                const float f = exp2f(red_m[ww][hh] - M);
                L = fmaf(red_l[ww][hh], f, L);
                O = fmaf(red_o[ww][hh][d], f, O);
            }
        }
        const int64_t h = h0 + hh;
        if (a.nsplit == 1) {
            store_elem(a.out, s * a.ldo + h * D + d, a.odt, L > 0.0f ? O / L * vscale : 0.0f);
        } else {
            float *pp = a.part + ((s * a.Hq + h) * a.nsplit + sp) * (D + 2);
            pp[d] = O;
            if (d == 0) {
                pp[D] = M;
                pp[D + 1] = L;
            }
        }
    }
}

} // namespace pgf8
