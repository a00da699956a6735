// tcgen05 GEMM for the FP8 linear layer and the NestedFP linear layer.
//
//   y[m,n] = epilogue( sum_k X[m,k] * W[n,k] )
//
// X: activations [M,K], W: weights [N,K], both K-contiguous ("C++ and FP8"
// §3.3, the "tn" E4M3 x E4M3 -> f32 GEMM with bf16 output).  One kernel
// template covers the three operand kinds:
//   kE4M3     X E4M3, W E4M3, y = bf16(acc * sa[m] * sw[n])           (FP8 linear)
//   kNested8  X E4M3, W = hi plane read as E5M2, y = f16(acc * sa[m])  (NestedFP FP8 mode)
//   kNested16 X FP16, W = (hi << 8) | lo rebuilt in shared memory, y = f16(acc)
//             (NestedFP FP16 mode; "NestedFP" §2.1-2.2)
// and two orientations:
//   SWAP = false ("tiled"):  MMA A = 128 token rows,  MMA B = BN weight rows,
//                            accumulator lane = token, column = output channel;
//   SWAP = true  ("skinny"): MMA A = 128 weight rows, MMA B = BN token rows
//                            (BN >= M, zero-filled), lane = output channel,
//                            column = token.  Used for decode-sized M, where the
//                            layer streams weights from HBM.
//
// Structure (one output tile per CTA, 192 threads):
//   warp 0      TMA producer: STAGES-deep ring of (A tile, B tile), 128 bytes
//               of K per stage, 128-byte swizzle, mbarrier completion.
//   warp 1      allocates the tensor-memory accumulator and issues
//               tcgen05.mma (one thread), committing each stage back to the
//               producer and the finished tile to the epilogue.
//   warps 2-5   kNested16 only: rebuild the FP16 weight tile in place from the
//               hi/lo byte planes (byte permutes into the swizzled K-major
//               FP16 layout), then hand it to the MMA thread.
//               All kinds: epilogue — tcgen05.ld of the accumulator, scaling,
//               rounding, 16- or 2-byte stores.
// Quantised activations (XQ, skinny FP8 kinds, M <= BN <= 32, the CTA's
// activation slice small enough for registers): the kernel reads the f32 /
// f16 activations itself instead of E4M3 codes made by a separate pass
// ("7B on an RTX 4060 with FP8" §2.2 dynamic per-token scale, computed
// here).  Warps 2-5 load the CTA's K-slice of the M rows into registers and
// take each token's amax over it; the CTAs of a split-K cluster combine
// their partial maxima through distributed shared memory; the registers are
// then converted (x / s rounded to E4M3, saturating, exactly as the
// quantisation kernel does) and written into the B tiles of the weight
// stages, which the MMA thread waits for like a TMA load.  The weights need
// no dependency wait, so with programmatic launch they stream while the
// previous kernel finishes.  CTAs of weight tile 0 also write the codes (and
// one CTA the scales) to global memory, so the caller sees the same side
// outputs as with the separate pass.
// Split-K: with SPLIT, the CTAs of one thread-block cluster (along z) each
// accumulate a slice of K; partial tiles are exchanged through distributed
// shared memory and summed in cluster-rank order (deterministic), each CTA
// finishing an equal share of the tile.
//
// Every wait is bounded (kWaitLimitNs).  A thread that gives up raises the
// CTA's abort flag and the device error word; the other roles stop at their
// next wait, in-flight copies and MMAs are drained (bounded again), the
// accumulator is freed and the CTA exits through the same barriers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "quantize.cuh"
#include "sm100_ptx.cuh"

namespace pgf8 {

enum OpKind : int { kE4M3 = 0, kNested8 = 1, kNested16 = 2 };

constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;   // 1 s
constexpr unsigned kErrTimeout = 1u;

__device__ unsigned int g_device_error;

struct GemmParams {
    int M, N, K;         // elements
    int kblocks;         // ceil(K * elem_bytes / 128)
    int splits;          // CTAs per cluster along z (1 = no split)
    int prefetch_w;      // 1: weight tiles may be loaded before the grid dependency resolves
    const float *sa;     // [M] (kE4M3, kNested8)
    const float *sw;     // [N] (kE4M3)
    void *y;             // [M, N] bf16 (kE4M3) or f16; f32 when out_f32
    int out_f32;         // pair kernel, kE4M3: y is f32, the scaled sum before rounding
    // XQ kernels only
    const void *x;       // activations [M, K] f32 or f16, row stride ldx elements
    int64_t ldx;
    uint8_t *q_out;      // [M, K] E4M3 codes written by the CTAs of weight tile 0, or null
    float *sa_out;       // [M] scales written by one CTA, or null
};

// 16 consecutive activations of one row as loaded (XQ = 1: f32, 2: f16).
template <int XQ> struct XRaw;
template <> struct XRaw<1> {
    static constexpr int kElemBytes = 4;
    uint4 w[4];
    __device__ __forceinline__ void load(const uint8_t *p)
    {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            w[i] = __ldg(reinterpret_cast<const uint4 *>(p) + i);
    }
    __device__ __forceinline__ void to_float(float (&v)[16]) const
    {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[4 * i + 0] = __uint_as_float(w[i].x);
            v[4 * i + 1] = __uint_as_float(w[i].y);
            v[4 * i + 2] = __uint_as_float(w[i].z);
            v[4 * i + 3] = __uint_as_float(w[i].w);
        }
    }
};
template <> struct XRaw<2> {
    static constexpr int kElemBytes = 2;
    uint4 w[2];
    __device__ __forceinline__ void load(const uint8_t *p)
    {
#pragma unroll
        for (int i = 0; i < 2; ++i)
            w[i] = __ldg(reinterpret_cast<const uint4 *>(p) + i);
    }
    __device__ __forceinline__ void to_float(float (&v)[16]) const
    {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const uint32_t t[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&t[j]));   // exact
                v[8 * i + 2 * j] = f.x;
                v[8 * i + 2 * j + 1] = f.y;
            }
        }
    }
};

template <bool SWAP_, int BN_, int STAGES_, int KIND_, bool SPLIT_, int XQ_ = 0> struct GemmCfg {
    static constexpr bool SWAP = SWAP_;
    static constexpr int XQ = XQ_;   // 0: X read as E4M3 codes by TMA; 1 / 2: f32 / f16 activations quantised in the kernel
    static constexpr int BN = BN_;
    static constexpr int STAGES = STAGES_;
    static constexpr int KIND = KIND_;
    static constexpr bool SPLIT = SPLIT_;
    static constexpr int kThreads = 192;
    static constexpr int kTileA = 128 * 128;                  // 128 rows x 128 bytes
    static constexpr int kTileB = BN * 128;
    static constexpr int kStage = kTileA + kTileB;
    static constexpr int kRowsW = SWAP ? 128 : BN;            // weight rows per tile
    static constexpr int kRowsX = SWAP ? BN : 128;            // token rows per tile
    static constexpr int kTmemCols = BN < 32 ? 32 : BN;
    // split-K partial tile in shared memory (reuses the stage ring):
    //   SWAP: column-major [BN][128] f32;  tiled: row-major [128][BN + 4] f32
    static constexpr int kRedBytes = SWAP ? BN * 128 * 4 : 128 * (BN + 4) * 4;
    static constexpr int kRingBytes = STAGES * kStage;
    static constexpr int kDataBytes = kRingBytes > kRedBytes ? kRingBytes : kRedBytes;
    static constexpr int kBarOffset = kDataBytes;
    static constexpr int kSmemBytes = kDataBytes + 1024 /*control block*/ + 1024 /*alignment slack*/;
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M=128 must be a multiple of 16 in [16,256]");
    static_assert((BN & (BN - 1)) == 0 || BN % 32 == 0, "BN");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
    static_assert(XQ == 0 || (SWAP && KIND != kNested16 && BN <= 32), "in-kernel quantisation: skinny FP8, M <= 32");
    static_assert(STAGES <= 8 && kStage % 1024 == 0, "ring");
};

struct SharedCtl {
    uint64_t full[8];
    uint64_t empty[8];
    uint64_t conv[8];
    uint64_t tmem_full;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    float sa_s[128];        // per-token scales of the tile's tokens, loaded at kernel start
};

// Bounded wait on an mbarrier phase.  Returns false (and raises the abort
// flag and the device error word) after limit_ns, or when another role of
// the CTA has already raised the abort flag.
__device__ __forceinline__ bool wait_bounded_for(uint64_t *bar, uint32_t parity, volatile int *abort,
                                                 uint64_t limit_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t spin = 1;; ++spin) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((spin & 63u) == 0) {
            if (*abort)
                return false;
            if (global_timer_ns() - t0 > limit_ns) {
                *abort = 1;
                atomicOr(&g_device_error, kErrTimeout);
                return false;
            }
        }
    }
}

__device__ __forceinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort)
{
    return wait_bounded_for(bar, parity, abort, kWaitLimitNs);
}

// Self-test of the bounded wait: one thread waits on a barrier phase that
// nothing ever completes; the wait gives up after limit_ns, raises the
// device error word, and the kernel returns normally.
__global__ void selftest_bounded_wait_kernel(uint64_t limit_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0)
        (void)wait_bounded_for(&bar, 0, &abort, limit_ns);
}

// Wait used only while draining after an abort: bounded, never raises.
__device__ __forceinline__ void wait_drain(uint64_t *bar, uint32_t parity)
{
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > kWaitLimitNs)
            return;
    }
}

// Rebuild FP16 weights in place: the stage region holds the hi plane
// [rows][64 B] followed by the lo plane [rows][64 B] (no swizzle); it is
// rewritten as FP16 [rows][128 B] in the 128-byte-swizzled K-major layout
// (16-byte chunk j of row r stored at chunk j ^ (r % 8)).  Half e of a chunk
// is (hi[e] << 8) | lo[e]; in little-endian bytes: lo[e], hi[e].
template <int ROWS>
__device__ __forceinline__ void rebuild_fp16_tile(uint8_t *tile, int tid /*0..127*/)
{
    constexpr int kItems = ROWS * 8 / 128;   // 16-byte output chunks per thread
    uint2 h[kItems], l[kItems];
#pragma unroll
    for (int u = 0; u < kItems; ++u) {
        const int i = tid + 128 * u;         // chunk index: row i/8, chunk i%8
        h[u] = *reinterpret_cast<const uint2 *>(tile + i * 8);
        l[u] = *reinterpret_cast<const uint2 *>(tile + ROWS * 64 + i * 8);
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll
    for (int u = 0; u < kItems; ++u) {
        const int i = tid + 128 * u;
        const int r = i >> 3, j = i & 7;
        uint4 o;
        o.x = __byte_perm(l[u].x, h[u].x, 0x5140);
        o.y = __byte_perm(l[u].x, h[u].x, 0x7362);
        o.z = __byte_perm(l[u].y, h[u].y, 0x5140);
        o.w = __byte_perm(l[u].y, h[u].y, 0x7362);
        *reinterpret_cast<uint4 *>(tile + r * 128 + ((j ^ (r & 7)) << 4)) = o;
    }
}

template <int KIND> __device__ __forceinline__ void store_out(void *y, int64_t idx, float v);
template <> __device__ __forceinline__ void store_out<kE4M3>(void *y, int64_t idx, float v)
{
    reinterpret_cast<__nv_bfloat16 *>(y)[idx] = __float2bfloat16_rn(v);
}
template <> __device__ __forceinline__ void store_out<kNested8>(void *y, int64_t idx, float v)
{
    reinterpret_cast<__half *>(y)[idx] = __float2half_rn(v);
}
template <> __device__ __forceinline__ void store_out<kNested16>(void *y, int64_t idx, float v)
{
    reinterpret_cast<__half *>(y)[idx] = __float2half_rn(v);
}

// Pack two floats into two 16-bit outputs (low half = a).
template <int KIND> __device__ __forceinline__ uint32_t pack2(float a, float b)
{
    if constexpr (KIND == kE4M3) {
        __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&t);
    } else {
        __half2 t = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&t);
    }
}

// XQ helpers.
// Partial amax of one batch of 16-element chunks (row[u] < 0: no chunk):
// f32 max of |x| (NaN ignored, as the quantisation kernel), segmented warp
// max, shared atomic max on the bits (non-negative floats order like their
// bit patterns).
template <int XQ, int U>
__device__ __forceinline__ void xq_batch_amax(const XRaw<XQ> (&raw)[U], const int (&row)[U], uint32_t *xq_amax,
                                              int lane)
{
#pragma unroll
    for (int u = 0; u < U; ++u) {
        float mx = 0.0f;
        if (row[u] >= 0) {
            float v[16];
            raw[u].to_float(v);
#pragma unroll
            for (int i = 0; i < 16; ++i)
                mx = fmaxf(mx, fabsf(v[i]));
        }
        const unsigned grp = __match_any_sync(0xffffffffu, row[u]);
        const unsigned mb = __reduce_max_sync(grp, __float_as_uint(mx));
        if (row[u] >= 0 && lane == __ffs(grp) - 1)
            atomicMax(&xq_amax[row[u]], mb);
    }
}

// Per-token scales from the slice maxima: with split-K the cluster barrier
// publishes every CTA's maxima and each CTA reads all of them, so all derive
// the same s = amax / 448 (1 when the row is zero) — the "7B on an RTX 4060
// with FP8" §2.2 / §6.1 dynamic scale — into ctl->sa_s (and, from one CTA,
// p.sa_out).  Called by all 128 threads of warps 2-5.
template <class C>
__device__ __forceinline__ void xq_scales(const GemmParams &p, SharedCtl *ctl, uint32_t *xq_amax, int et, int tile_a,
                                          int split)
{
    if constexpr (C::SPLIT) {
        cluster_arrive_release();
        cluster_wait_acquire();
    } else {
        bar_sync_warps2to5();
    }
    if (et < p.M) {
        uint32_t b = xq_amax[et];
        if constexpr (C::SPLIT) {
            const uint32_t a = smem_u32(&xq_amax[et]);
            for (int z = 0; z < p.splits; ++z) {
                const uint32_t o = ld_shared_cluster_u32(map_shared_rank(a, static_cast<uint32_t>(z)));
                b = o > b ? o : b;
            }
        }
        float sc = __fdiv_rn(__uint_as_float(b), 448.0f);
        if (sc == 0.0f)
            sc = 1.0f;
        ctl->sa_s[et] = sc;
        if (p.sa_out && tile_a == 0 && split == 0)
            p.sa_out[et] = sc;
    }
    bar_sync_warps2to5();
}

// XQ: warps 2-5 quantise the CTA's activation slice (M rows x k-blocks
// [kb0, kb1)), which fits one batch of the amax pass (at most 128 x U chunks
// of 16 elements) and so stays in registers: amax, scales, then the chunks are converted to codes
// in registers and written into the B tiles of the weight stages as they
// free up.  No activation is loaded after pass 1.  The B tiles are zeroed
// once (rows >= M are never written); in a ragged last k-block the chunks
// past K are zeroed again.  Loop exits are agreed by all 128 threads
// (barrier with AND).
template <class C>
__device__ __forceinline__ void quantize_x_resident(const GemmParams &p, uint8_t *smem, SharedCtl *ctl,
                                                    uint32_t *xq_amax, volatile int *abort_flag, int kb0, int kb1,
                                                    int tile_a, int split)
{
    constexpr int XQ = C::XQ;
    constexpr int EB = XRaw<XQ>::kElemBytes;
    constexpr int U = XQ == 1 ? 4 : 8;
    const int et = static_cast<int>(threadIdx.x) - 64;   // 0..127
    const int lane = et & 31;
    const uint8_t *xb = static_cast<const uint8_t *>(p.x);
    const int64_t row_bytes = p.ldx * EB;

    // B tiles start zero (rows >= M are never written)
    for (int i = et; i < C::STAGES * C::kTileB / 16; i += 128) {
        const int st = i / (C::kTileB / 16), rest = i % (C::kTileB / 16);
        *reinterpret_cast<uint4 *>(smem + st * C::kStage + C::kTileA + rest * 16) = make_uint4(0u, 0u, 0u, 0u);
    }

    // nothing of x may be read before the kernel that writes it has completed
    grid_dependency_wait();

    // ---- 1. the slice, one batch: chunk it = u * 128 + et -> row m, chunk c
    const int kbeg = kb0 * 128;
    const int kend = (kb1 * 128 < p.K) ? kb1 * 128 : p.K;
    const int nch = (kend - kbeg) >> 4;
    const int items = p.M * nch;            // <= 128 * U (checked by the host)
    XRaw<XQ> raw[U];
    int row[U], chunk[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int it = u * 128 + et;
        row[u] = -1;
        chunk[u] = 0;
        if (it < items) {
            const int m = it / nch;
            const int c = it - m * nch;
            row[u] = m;
            chunk[u] = c;
            raw[u].load(xb + m * row_bytes + static_cast<int64_t>(kbeg + c * 16) * EB);
        }
    }
    xq_batch_amax<XQ, U>(raw, row, xq_amax, lane);

    // ---- 2. scales
    xq_scales<C>(p, ctl, xq_amax, et, tile_a, split);

    // ---- 3. codes in registers, then into the weight stages
    uint4 code[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        code[u] = make_uint4(0u, 0u, 0u, 0u);
        if (row[u] >= 0) {
            float v[16];
            raw[u].to_float(v);
            code[u] = encode16(v, RowDivisor(ctl->sa_s[row[u]]));
        }
    }
    const bool write_codes = p.q_out != nullptr && tile_a == 0;
    int s = 0;
    uint32_t ph = 0;
    for (int kb = kb0; kb < kb1; ++kb) {
        const int n = kb - kb0;
        bool ok = true;
        if (n >= C::STAGES)
            ok = wait_bounded(&ctl->empty[s], ph ^ 1u, abort_flag);
        if (!bar_and_warps2to5(ok))
            break;
        uint8_t *bt = smem + s * C::kStage + C::kTileA;
        if (kb == kb1 - 1 && kend < kb1 * 128) {
            // ragged K: the stage's chunks past K still hold an earlier
            // k-block's codes; zero them (a stale NaN code times a zero-filled
            // weight would poison the accumulator)
            for (int i = et; i < p.M * 8; i += 128) {
                const int r = i >> 3, j = i & 7;
                if (kb * 128 + 16 * j >= kend)
                    *reinterpret_cast<uint4 *>(bt + r * 128 + ((j ^ (r & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (row[u] >= 0 && (chunk[u] >> 3) == n) {
                const int r = row[u], j = chunk[u] & 7;
                if (write_codes)
                    *reinterpret_cast<uint4 *>(p.q_out + static_cast<int64_t>(r) * p.K + kbeg + chunk[u] * 16) =
                        code[u];
                *reinterpret_cast<uint4 *>(bt + r * 128 + ((j ^ (r & 7)) << 4)) = code[u];
            }
        }
        fence_proxy_async_smem();   // each writer, before the MMA (async proxy) reads
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&ctl->conv[s]);
        if (++s == C::STAGES) {
            s = 0;
            ph ^= 1u;
        }
    }
}

template <class C>
__global__ void __launch_bounds__(192, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                const __grid_constant__ CUtensorMap tmW2, const GemmParams p)
{
    constexpr bool SWAP = C::SWAP;
    constexpr int BN = C::BN;
    constexpr int STAGES = C::STAGES;
    constexpr int KIND = C::KIND;
    constexpr bool NEST16 = (KIND == kNested16);
    constexpr int XQ = C::XQ;
    constexpr uint32_t kIdesc =
        make_idesc(128, BN, /*A fmt*/ (SWAP && KIND == kNested8) ? 1 : 0, /*B fmt*/ (!SWAP && KIND == kNested8) ? 1 : 0);
    constexpr int kXStep = NEST16 ? 64 : 128;   // K elements per stage

    // A dependent kernel launched with programmatic serialization (the next
    // layer) may be scheduled into free SM slots now; it reads nothing this
    // grid writes before this grid has completed.
    grid_launch_dependents();

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    SharedCtl *ctl = reinterpret_cast<SharedCtl *>(smem + C::kBarOffset);
    volatile int *abort_flag = &ctl->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tile_a = blockIdx.x;   // A-side tile (128 rows)
    const int tile_b = blockIdx.y;   // B-side tile (BN rows)
    const int split = C::SPLIT ? static_cast<int>(blockIdx.z) : 0;
    const int kb0 = C::SPLIT ? (split * p.kblocks) / p.splits : 0;
    const int kb1 = C::SPLIT ? ((split + 1) * p.kblocks) / p.splits : p.kblocks;
    const int row0_w = SWAP ? tile_a * 128 : tile_b * BN;   // first weight row of the tile
    const int row0_x = SWAP ? tile_b * BN : tile_a * 128;   // first token row of the tile
    __shared__ uint32_t xq_amax[XQ ? 32 : 1];   // XQ: bits of the per-token amax (non-negative floats)

    // Producer state (thread 0): the first pass of the ring is issued before
    // the CTA-wide synchronisation, so its loads overlap the set-up.
    int ps = 0;
    uint32_t pph = 0;
    uint32_t issued_mask = 0, issued_ph = 0;   // per stage: loaded at least once / parity of last load
    int pending = 0;                            // stages with weights but no activations yet
    bool waited = false;
    int pkb = kb0;
    uint64_t pol_w = 0, pol_x = 0;

    auto issue_w = [&](int kb, int st_idx) {
        uint8_t *st = smem + st_idx * C::kStage;
        uint8_t *w_tile = SWAP ? st : st + C::kTileA;
        mbar_arrive_expect_tx(&ctl->full[st_idx], XQ ? C::kTileA : C::kStage);
        if constexpr (NEST16) {
            // hi and lo planes, 64 bytes (= 64 weights) of K each
            tma_load_2d_hint(w_tile, &tmW, &ctl->full[st_idx], kb * 64, row0_w, pol_w);
            tma_load_2d_hint(w_tile + C::kRowsW * 64, &tmW2, &ctl->full[st_idx], kb * 64, row0_w, pol_w);
        } else {
            tma_load_2d_hint(w_tile, &tmW, &ctl->full[st_idx], kb * 128, row0_w, pol_w);
        }
    };
    auto issue_x = [&](int kb, int st_idx) {
        uint8_t *st = smem + st_idx * C::kStage;
        uint8_t *x_tile = SWAP ? st + C::kTileA : st;
        tma_load_2d_hint(x_tile, &tmX, &ctl->full[st_idx], kb * kXStep, row0_x, pol_x);
    };
    // activations of the `pending` stages issued last (ending at k-block
    // kb_end - 1, stage s_end - 1), once the grid dependency has resolved
    auto flush_pending = [&](int kb_end, int s_end) {
        grid_dependency_wait();
        waited = true;
        for (int j = 0; j < pending; ++j)
            issue_x(kb_end - pending + j, (s_end - pending + j + STAGES) % STAGES);
        pending = 0;
    };
    // one k-block into stage ps (its empty barrier already passed)
    auto issue_stage = [&](int kb) {
        issue_w(kb, ps);
        issued_mask |= 1u << ps;
        issued_ph = (issued_ph & ~(1u << ps)) | (pph << ps);
        if (++ps == STAGES) {
            ps = 0;
            pph ^= 1u;
        }
        if constexpr (!XQ) {   // XQ: warps 2-5 load and convert the activations
            if (waited) {
                issue_x(kb, (ps + STAGES - 1) % STAGES);
            } else if (++pending == STAGES) {
                flush_pending(kb + 1, ps);
            }
        }
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
            mbar_init(&ctl->conv[s], 4);    // one arrival per warp of warps 2-5
        }
        mbar_init(&ctl->tmem_full, 1);
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        if constexpr (XQ) {
            for (int m = 0; m < 32; ++m)
                xq_amax[m] = 0u;
        }
        fence_mbar_init();
        if (!XQ)
            tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmW);
        if (NEST16)
            tma_prefetch_desc(&tmW2);
        // weights are streamed once in the skinny orientation (evict first);
        // activation tiles are re-read by every CTA (evict last)
        pol_w = SWAP ? policy_evict_first() : policy_evict_last();
        pol_x = policy_evict_last();
        if (!p.prefetch_w) {
            grid_dependency_wait();
            waited = true;
        }
        const int pre = (kb1 - kb0) < STAGES ? (kb1 - kb0) : STAGES;
        for (int j = 0; j < pre; ++j)     // fresh ring: no empty-barrier waits
            issue_stage(kb0 + j);
        pkb = kb0 + pre;
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    if (warp >= 2 && !XQ) {
        // scales of this tile's tokens, read once (after the dependency, as
        // they may come from the previous kernel)
        grid_dependency_wait();
        const int et = static_cast<int>(threadIdx.x) - 64;
        if constexpr (SWAP && KIND != kNested16) {
            if (et < BN)
                ctl->sa_s[et] = (row0_x + et < p.M) ? p.sa[row0_x + et] : 0.0f;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    // XQ with split-K: every thread of the cluster takes part in one barrier
    // phase that publishes the partial maxima; the producer and MMA warps
    // arrive now and wait after their loops
    if constexpr (XQ && C::SPLIT) {
        if (warp < 2)
            cluster_arrive_relaxed();
    }

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            for (int kb = pkb; kb < kb1; ++kb) {
                if (!wait_bounded(&ctl->empty[ps], pph ^ 1u, abort_flag))
                    break;
                issue_stage(kb);
            }
            if (pending > 0)
                flush_pending(kb1, ps);
            if (!waited)
                grid_dependency_wait();
            if (*abort_flag) {
                // drain: the last load of every used stage lands (bounded) before
                // the CTA may exit; older loads were consumed already
                for (int j = 0; j < STAGES; ++j)
                    if (issued_mask & (1u << j))
                        wait_drain(&ctl->full[j], (issued_ph >> j) & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        grid_dependency_wait();
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int kb = kb0; kb < kb1; ++kb) {
                if (!wait_bounded(&ctl->full[s], ph, abort_flag)) {
                    ok = false;
                    break;
                }
                if constexpr (NEST16 || XQ) {
                    if (!wait_bounded(&ctl->conv[s], ph, abort_flag)) {
                        ok = false;
                        break;
                    }
                }
                tc_fence_after();
                const uint32_t a_addr = smem_u32(smem + s * C::kStage);
                const uint32_t b_addr = a_addr + C::kTileA;
#pragma unroll
                for (int k = 0; k < 4; ++k) {   // 4 MMAs x 32 bytes of K
                    const uint64_t ad = sdesc_sw128(a_addr + k * 32);
                    const uint64_t bd = sdesc_sw128(b_addr + k * 32);
                    const uint32_t acc = (kb > kb0 || k > 0) ? 1u : 0u;
                    if constexpr (NEST16)
                        umma_f16(tmem, ad, bd, kIdesc, acc);
                    else
                        umma_f8f6f4(tmem, ad, bd, kIdesc, acc);
                }
                umma_commit(&ctl->empty[s]);
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            if (ok) {
                umma_commit(&ctl->tmem_full);
            } else {
                umma_commit(&ctl->drain);
                wait_drain(&ctl->drain, 0);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ FP16 rebuild
        if constexpr (NEST16) {
            const int tt = static_cast<int>(threadIdx.x) - 64;   // 0..127
            int s = 0;
            uint32_t ph = 0;
            for (int kb = kb0; kb < kb1; ++kb) {
                if (!wait_bounded(&ctl->full[s], ph, abort_flag))
                    break;
                uint8_t *tile = smem + s * C::kStage + (SWAP ? 0 : C::kTileA);
                rebuild_fp16_tile<C::kRowsW>(tile, tt);
                fence_proxy_async_smem();   // each writer, before the MMA (async proxy) reads
                __syncwarp();
                if ((threadIdx.x & 31) == 0)
                    mbar_arrive(&ctl->conv[s]);
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        } else if constexpr (XQ) {
            quantize_x_resident<C>(p, smem, ctl, xq_amax, abort_flag, kb0, kb1, tile_a, split);
        }
    }
    if constexpr (XQ && C::SPLIT) {
        if (warp < 2)
            cluster_wait_acquire();
    }

    // ---------------------------------------------------------------- epilogue
    // All 6 warps reach this point; warps 2-5 own the accumulator rows.
    const bool epi = warp >= 2;
    bool have_acc = false;
    if (epi) {
        have_acc = wait_bounded(&ctl->tmem_full, 0, abort_flag);
        have_acc = __all_sync(0xffffffffu, have_acc);
        tc_fence_after();
    }
    const int et = static_cast<int>(threadIdx.x) - 64;   // epilogue thread index 0..127
    const int q = warp & 3;                     // TMEM lane quadrant of this warp
    const int r = q * 32 + lane;                // accumulator row (lane)
    const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16);

    // skinny output of one accumulator row: channel n, tokens row0_x + j
    auto store_skinny_row = [&](const float *a, int ncols) {
        const int n = row0_w + r;
        if (n >= p.N)
            return;
        float swn = 1.0f;
        if constexpr (KIND == kE4M3)
            swn = p.sw[n];
        for (int j = 0; j < ncols; ++j) {
            const int m = row0_x + j;
            if (m < p.M) {
                float v = a[j];
                if constexpr (KIND != kNested16)
                    v = v * ctl->sa_s[j];
                if constexpr (KIND == kE4M3)
                    v = v * swn;
                store_out<KIND>(p.y, static_cast<int64_t>(m) * p.N + n, v);
            }
        }
    };

    if constexpr (!C::SPLIT) {
        if (epi && have_acc) {
            if constexpr (SWAP) {
                // lane = output channel n, column = token m
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 16) {
                    if (row0_x + c0 >= p.M)
                        break;                  // warp-uniform
                    uint32_t v[16];
                    tmem_ld_32x32b_x16(t_row + c0, v);
                    tmem_ld_wait();
                    float a[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        a[j] = __uint_as_float(v[j]);
                    const int n = row0_w + r;
                    if (n < p.N) {
                        float swn = 1.0f;
                        if constexpr (KIND == kE4M3)
                            swn = p.sw[n];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int m = row0_x + c0 + j;
                            if (m < p.M) {
                                float x = a[j];
                                if constexpr (KIND != kNested16)
                                    x = x * ctl->sa_s[c0 + j];
                                if constexpr (KIND == kE4M3)
                                    x = x * swn;
                                store_out<KIND>(p.y, static_cast<int64_t>(m) * p.N + n, x);
                            }
                        }
                    }
                }
            } else {
                // lane = token m, column = output channel n
                const int m = row0_x + r;
                float sam = 1.0f;
                if constexpr (KIND != kNested16)
                    sam = (m < p.M) ? p.sa[m] : 0.0f;
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 16) {
                    const int n0 = row0_w + c0;
                    if (n0 >= p.N)
                        break;                  // warp-uniform; N % 16 == 0
                    uint32_t v[16];
                    tmem_ld_32x32b_x16(t_row + c0, v);
                    tmem_ld_wait();
                    if (m < p.M) {
                        uint32_t o[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            float a0 = __uint_as_float(v[2 * j]), a1 = __uint_as_float(v[2 * j + 1]);
                            if constexpr (KIND != kNested16) {
                                a0 = a0 * sam;
                                a1 = a1 * sam;
                            }
                            if constexpr (KIND == kE4M3) {
                                a0 = a0 * __ldg(p.sw + n0 + 2 * j);
                                a1 = a1 * __ldg(p.sw + n0 + 2 * j + 1);
                            }
                            o[j] = pack2<KIND>(a0, a1);
                        }
                        uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(p.y) +
                                                               static_cast<int64_t>(m) * p.N + n0);
                        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
                        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------------------ split-K, symmetric
        // 1. each CTA stores its partial tile into its own (now idle) ring
        float *red = reinterpret_cast<float *>(smem);
        if (epi) {
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 16) {
                uint32_t v[16];
                if (have_acc) {
                    tmem_ld_32x32b_x16(t_row + c0, v);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        v[j] = 0u;
                }
                if constexpr (SWAP) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        red[(c0 + j) * 128 + r] = __uint_as_float(v[j]);
                } else {
                    float4 *dst = reinterpret_cast<float4 *>(red + r * (BN + 4) + c0);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                             __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
                }
            }
        }
        __syncwarp();
        cluster_sync_all();
        // 2. each CTA finishes 1/splits of the tile, summing the partials of
        //    all CTAs of the cluster in rank order
        const uint32_t red_addr = smem_u32(red);
        const int S = p.splits;
        const int rank = static_cast<int>(cluster_ctarank());
        if (epi) {
            // groups of 4 consecutive floats: SWAP: (token c, channels r..r+3);
            // tiled: (token r, channels c..c+3)
            constexpr int kGroups = 128 * BN / 4;
            const int g0 = (rank * kGroups) / S, g1 = ((rank + 1) * kGroups) / S;
            for (int g = g0 + et; g < g1; g += 128) {
                int m, n;
                uint32_t off;
                if constexpr (SWAP) {
                    const int c = g / 32, rr = (g % 32) * 4;
                    m = row0_x + c;
                    n = row0_w + rr;
                    off = static_cast<uint32_t>((c * 128 + rr) * 4);
                } else {
                    const int rr = g / (BN / 4), c = (g % (BN / 4)) * 4;
                    m = row0_x + rr;
                    n = row0_w + c;
                    off = static_cast<uint32_t>((rr * (BN + 4) + c) * 4);
                }
                if (m >= p.M || n >= p.N)
                    continue;
                // all partials are requested before any is added (the remote
                // loads overlap); the sum runs in rank order
                float4 t[8];
#pragma unroll
                for (int z = 0; z < 8; ++z)
                    if (z < S)
                        t[z] = ld_shared_cluster_v4_relaxed(map_shared_rank(red_addr + off, static_cast<uint32_t>(z)));
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int z = 0; z < 8; ++z) {
                    if (z < S) {
                        acc.x += t[z].x;
                        acc.y += t[z].y;
                        acc.z += t[z].z;
                        acc.w += t[z].w;
                    }
                }
                float a[4] = {acc.x, acc.y, acc.z, acc.w};
                float sam = 1.0f;
                if constexpr (XQ)
                    sam = ctl->sa_s[m - row0_x];
                else if constexpr (KIND != kNested16)
                    sam = p.sa[m];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if constexpr (KIND != kNested16)
                        a[j] = a[j] * sam;
                    if constexpr (KIND == kE4M3)
                        a[j] = a[j] * __ldg(p.sw + n + j);
                }
                uint2 o;
                o.x = pack2<KIND>(a[0], a[1]);
                o.y = pack2<KIND>(a[2], a[3]);
                *reinterpret_cast<uint2 *>(reinterpret_cast<uint16_t *>(p.y) + static_cast<int64_t>(m) * p.N + n) = o;
            }
        }
        __syncwarp();
        cluster_sync_all();   // no CTA leaves while its partial may still be read
    }
    (void)store_skinny_row;

    // ---------------------------------------------------------------- teardown
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

} // namespace pgf8
