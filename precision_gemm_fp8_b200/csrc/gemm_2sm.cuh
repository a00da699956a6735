// Persistent tcgen05 GEMM on CTA pairs (cta_group::2) for the tiled
// orientation of the FP8 linear layer ("C++ and FP8" §3.3) and NestedFP FP8
// mode ("NestedFP" §2.2): 256 x 256 output tiles, one tile per pair of SMs.
//
// The two CTAs of a cluster each load half of the tile's operands into their
// own shared memory (rows m0 + 128*rank of the activations, rows n0 + 128*rank
// of the weights); one thread of the even CTA issues tcgen05.mma.cta_group::2
// (M = 256, N = 256), which reads both CTAs' shared memory and accumulates
// rows m0.. into the even CTA's tensor memory and rows m0+128.. into the odd
// CTA's.  Per CTA and k-block that is 32 KB of operands for a 128 x 256 slice
// of the output, two thirds of what the one-CTA 128 x 256 tile moves, which
// leaves room for a 6-deep ring.
//
// Synchronisation (all mbarriers; every wait bounded):
//   full[s]      even CTA only: both CTAs' TMA loads complete on it (the
//                cta_group::2 form of the load addresses the even CTA's
//                barrier); the even producer posts the expected bytes of both.
//   empty[s]     per CTA: the MMA's commit arrives on the barrier at this
//                offset in both CTAs at once (tcgen05.commit with a CTA mask;
//                relaying it through a thread of the even CTA measured 2x
//                slower).
//   acc_full[b]  per CTA: the same two-CTA commit.
//   acc_empty[b] even CTA only: the 4 epilogue warps of both CTAs arrive.
//
// Wave quantisation: with T tiles on P pairs the last round of a plain
// persistent walk keeps only T mod P pairs busy.  With a stream-K region
// (sk.units > 0) the pairs walk the tiles below sk.t0 round-robin as
// above (whole tiles; neighbouring pairs on neighbouring tiles, so weight
// and activation tiles are shared in L2), and then split the remaining
// tiles' (tile, k-block) units into equal contiguous ranges, one per pair.
// sk.t0 leaves one full round plus the ragged tail to that region, so a
// tile is split between two or three pairs at most.  Fix-up as in the
// grouped kernel: a tile shared by several pairs is finished by the pair
// holding its first k-block (its last segment, accumulator kept in tensor
// memory); the following pairs store their f32 partial (each CTA its 128
// rows) into their slot at the start of their range and raise a flag; the
// finishing CTA adds them in pair order after its own (deterministic),
// clears the flags and writes the tile.
#pragma once

#include "gemm.cuh"
#include "gemm_streamk.cuh"

namespace pgf8 {

template <int BN_, int STAGES_, int KIND_> struct PairCfg {
    static constexpr int BN = BN_;                 // N of the pair's tile (MMA N)
    static constexpr int STAGES = STAGES_;
    static constexpr int KIND = KIND_;
    static constexpr bool NEST16 = (KIND == kNested16);
    static constexpr int XQ = 0;   // activations arrive as E4M3 codes (FP16 mode: as f16)
    static constexpr int kThreads = NEST16 ? 320 : 192;   // FP16 mode: 4 rebuild warps
    static constexpr int kTileA = 128 * 128;      // this CTA's 128 activation rows
    static constexpr int kTileB = (BN / 2) * 128; // this CTA's BN/2 weight rows
    static constexpr int kStage = kTileA + kTileB;
    static constexpr int kRowsX = 128;
    static constexpr int kRowsW = BN / 2;
    // two accumulator buffers of BN columns, allocated as a power of two
    static constexpr int kTmemCols = (2 * BN <= 256) ? 256 : 512;
    static_assert(BN == 128 || BN == 192 || BN == 256, "pair tile width");
    static_assert((kStage % 1024) == 0, "stage alignment");
    static constexpr int kRingBytes = STAGES * kStage;
    static constexpr int kBarOffset = kRingBytes;
    static constexpr int kSmemBytes = kRingBytes + 1024 + 1024;
    static_assert(!NEST16 || BN == 256, "FP16 mode: 256-wide tiles");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

constexpr int kPairSKMaxCtas = 160;              // partial slots (two per pair) in the workspace
constexpr size_t kPairSKFlagBytes = 1024;        // 256 flag words: CTA index < kPairSKMaxCtas

__host__ __device__ constexpr size_t pair_sk_workspace_bytes(int bn)
{
    return kPairSKFlagBytes + static_cast<size_t>(kPairSKMaxCtas) * 128 * bn * 4;
}

struct PairSK {
    int t0;              // first tile of the stream-K region (tiles below: whole, round-robin)
    int64_t units;       // (tile, k-block) units of the region; 0: no stream-K region
    unsigned *flags;     // [kPairSKMaxCtas], zero between calls
    float *partials;     // [kPairSKMaxCtas][BN][128]: this CTA's 128 rows, column-major
};

// One step of a pair's walk: tile t, k-blocks [kb0, kb1).  The whole tiles
// of the round-robin part first, then the segments of the pair's range of
// the stream-K region.
struct PairWalk {
    int pair, npairs, t0, kblocks;
    int64_t units, u0, u1;
    int t_next;          // next round-robin tile
    int64_t u;           // next stream-K unit

    __device__ __forceinline__ PairWalk(int pair_, int npairs_, const PairSK &sk, int total, int kblocks_)
        : pair(pair_), npairs(npairs_), t0(sk.units > 0 ? sk.t0 : total), kblocks(kblocks_), units(sk.units)
    {
        u0 = sk.units > 0 ? (static_cast<int64_t>(pair) * sk.units) / npairs : 0;
        u1 = sk.units > 0 ? (static_cast<int64_t>(pair + 1) * sk.units) / npairs : 0;
        t_next = pair;
        u = u0;
    }
    // false when the walk is over
    __device__ __forceinline__ bool next(int &t, int &kb0, int &kb1)
    {
        if (t_next < t0) {
            t = t_next;
            kb0 = 0;
            kb1 = kblocks;
            t_next += npairs;
            return true;
        }
        if (u >= u1)
            return false;
        const int local_t = static_cast<int>(u / kblocks);
        kb0 = static_cast<int>(u % kblocks);
        const int64_t tile_end = static_cast<int64_t>(local_t + 1) * kblocks;
        const int64_t seg_end = u1 < tile_end ? u1 : tile_end;
        kb1 = static_cast<int>(seg_end - static_cast<int64_t>(local_t) * kblocks);
        t = t0 + local_t;
        u = seg_end;
        return true;
    }
};

struct PairCtl {
    uint64_t full[16];
    uint64_t empty[16];
    uint64_t conv[16];   // FP16 mode, even CTA: both CTAs' weight halves rebuilt
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint64_t fix;        // stream-K region: partial tiles copied into shared memory
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void umma_f8f6f4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_f16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive (once) on `bar` of this CTA when every cta_group::2 tcgen05
// operation issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// TMA load into this CTA's shared memory whose completion is counted on the
// even CTA's barrier at the same offset (cta_group::2 form).
__device__ __forceinline__ void tma_load_2d_pair(void *smem_dst, const CUtensorMap *tm, uint64_t *bar, int x, int y,
                                                 uint64_t policy)
{
    const uint32_t bar_even = smem_u32(bar) & 0xFEFFFFFFu;   // clear the pair-rank bit of the address
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar_even), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

// Arrive (once) on `bar` at the same offset in both CTAs of the pair when
// every cta_group::2 tcgen05 operation issued so far by this thread has
// completed.  (A completion signal sent to two CTAs' barriers; no data moves.)
__device__ __forceinline__ void umma_commit_pair_both(uint64_t *bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(static_cast<uint16_t>(3))
        : "memory");
}

// Plain arrive on the barrier at the same offset in CTA `rank` of the cluster.
__device__ __forceinline__ void mbar_arrive_remote(uint64_t *bar, uint32_t rank)
{
    asm volatile(
        "{\n\t.reg .b32 ra;\n\t"
        "mapa.shared::cluster.u32 ra, %0, %1;\n\t"
        "mbarrier.arrive.release.cluster.shared::cluster.b64 _, [ra];\n\t}\n" ::"r"(smem_u32(bar)),
        "r"(rank)
        : "memory");
}

// Bounded wait with cluster-scope acquire (for barriers arrived on from the
// other CTA of the pair).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool wait_bounded_cluster(uint64_t *bar, uint32_t parity, volatile int *abort)
{
    if (mbar_try_wait_cluster(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t spin = 1;; ++spin) {
        if (mbar_try_wait_cluster(bar, parity))
            return true;
        if ((spin & 63u) == 0) {
            if (*abort)
                return false;
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                *abort = 1;
                atomicOr(&g_device_error, kErrTimeout);
                return false;
            }
        }
    }
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const __grid_constant__ CUtensorMap tmW2, const GemmParams p, const PairSK sk)
{
    constexpr int BN = C::BN;
    constexpr int STAGES = C::STAGES;
    constexpr int KIND = C::KIND;
    constexpr bool NEST16 = C::NEST16;
    constexpr uint32_t kIdesc = make_idesc(256, BN, 0, KIND == kNested8 ? 1 : 0);
    constexpr int kXStep = NEST16 ? 64 : 128;   // activation elements per k-block

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    PairCtl *ctl = reinterpret_cast<PairCtl *>(smem + C::kBarOffset);
    volatile int *abort_flag = &ctl->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();           // 0: issues the MMA, 1: its partner
    const bool lead = (rank == 0);
    const int pair = static_cast<int>(blockIdx.x >> 1);
    const int npairs = static_cast<int>(gridDim.x >> 1);
    const int m_tiles = (p.M + 255) / 256;
    const int n_tiles = (p.N + BN - 1) / BN;
    const int total = m_tiles * n_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
            mbar_init(&ctl->conv[s], 8);        // FP16 mode: 4 rebuild warps in each CTA
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->acc_full[b], 1);
            mbar_init(&ctl->acc_empty[b], 8);   // 4 epilogue warps in each CTA
        }
        mbar_init(&ctl->drain, 1);
        mbar_init(&ctl->fix, 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmW);
        if (NEST16)
            tma_prefetch_desc(&tmW2);
    }
    if (warp == 1) {
        tmem_alloc_pair(&ctl->tmem_base, C::kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                 // both CTAs' barriers exist before any remote arrive
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    grid_dependency_wait();
    // Dependents may start only now, when everything this grid depends on
    // has completed: a dependent that does not wait itself (the next
    // independent layer's quantisation in a grouped call) then still runs
    // after every kernel before this one.
    grid_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------ producers (both CTAs)
        if (lane == 0) {
            const uint64_t pol = policy_evict_last();
            int s = 0;
            uint32_t ph = 0;
            uint32_t issued_mask = 0, issued_ph = 0;
            bool ok = true;
            PairWalk walk(pair, npairs, sk, total, p.kblocks);
            int t, kb0, kb1;
            while (ok && walk.next(t, kb0, kb1)) {
                const int row_x = (t % m_tiles) * 256 + static_cast<int>(rank) * 128;
                const int row_w = (t / m_tiles) * BN + static_cast<int>(rank) * (BN / 2);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!wait_bounded_cluster(&ctl->empty[s], ph ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    // the even CTA passes each real completion of its empty
                    // barrier on to the odd CTA's
                    uint8_t *st = smem + s * C::kStage;
                    if constexpr (NEST16) {
                        // each CTA's loads complete on its own barrier: its
                        // rebuild warps wait for them; the MMA waits for both
                        // CTAs' rebuilds instead (conv, even CTA)
                        mbar_arrive_expect_tx(&ctl->full[s], C::kStage);
                        tma_load_2d_hint(st, &tmX, &ctl->full[s], kb * kXStep, row_x, pol);
                        tma_load_2d_hint(st + C::kTileA, &tmW, &ctl->full[s], kb * 64, row_w, pol);
                        tma_load_2d_hint(st + C::kTileA + (BN / 2) * 64, &tmW2, &ctl->full[s], kb * 64, row_w, pol);
                    } else {
                        if (lead)
                            mbar_arrive_expect_tx(&ctl->full[s], 2 * C::kStage);
                        tma_load_2d_pair(st, &tmX, &ctl->full[s], kb * 128, row_x, pol);
                        tma_load_2d_pair(st + C::kTileA, &tmW, &ctl->full[s], kb * 128, row_w, pol);
                    }
                    issued_mask |= 1u << s;
                    issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (*abort_flag && (lead || NEST16)) {
                for (int j = 0; j < STAGES; ++j)
                    if (issued_mask & (1u << j))
                        wait_drain(&ctl->full[j], (issued_ph >> j) & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (even CTA)
        if (lead && lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            int i = 0;
            PairWalk walk(pair, npairs, sk, total, p.kblocks);
            int t, kb0, kb1;
            for (; ok && walk.next(t, kb0, kb1); ++i) {
                const int buf = i & 1;
                const uint32_t use = static_cast<uint32_t>(i >> 1);
                if (!wait_bounded_cluster(&ctl->acc_empty[buf], (use & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + static_cast<uint32_t>(buf * BN);
                for (int kb = kb0; kb < kb1; ++kb) {
                    const bool got = NEST16 ? wait_bounded_cluster(&ctl->conv[s], ph, abort_flag)
                                            : wait_bounded(&ctl->full[s], ph, abort_flag);
                    if (!got) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * C::kStage);
                    const uint32_t b_addr = a_addr + C::kTileA;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t ad = sdesc_sw128(a_addr + k * 32);
                        const uint64_t bd = sdesc_sw128(b_addr + k * 32);
                        if constexpr (NEST16)
                            umma_f16_pair(d, ad, bd, kIdesc, (kb > kb0 || k > 0) ? 1u : 0u);
                        else
                            umma_f8f6f4_pair(d, ad, bd, kIdesc, (kb > kb0 || k > 0) ? 1u : 0u);
                    }
                    umma_commit_pair_both(&ctl->empty[s]);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (ok)
                    umma_commit_pair_both(&ctl->acc_full[buf]);
            }
            if (!ok) {
                umma_commit_pair(&ctl->drain);
                wait_drain(&ctl->drain, 0);
            }
        }
        __syncwarp();
    } else if (warp >= 6) {
        // ------------------------------------------------------------ FP16 rebuild (both CTAs)
        if constexpr (NEST16) {
            const int tt = static_cast<int>(threadIdx.x) - 192;   // 0..127
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            PairWalk walk(pair, npairs, sk, total, p.kblocks);
            int t, kb0, kb1;
            while (ok && walk.next(t, kb0, kb1)) {
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!wait_bounded(&ctl->full[s], ph, abort_flag)) {
                        ok = false;
                        break;
                    }
                    // this CTA's 128 weight rows: (hi << 8) | lo in the swizzled K-major FP16 layout
                    rebuild_fp16_tile<128>(smem + s * C::kStage + C::kTileA, tt);
                    fence_proxy_async_smem();   // before the MMA (async proxy, issued by the even CTA) reads
                    __syncwarp();
                    if (lane == 0) {
                        if (lead)
                            mbar_arrive(&ctl->conv[s]);
                        else
                            mbar_arrive_remote(&ctl->conv[s], 0u);
                    }
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16);
        const int cta = static_cast<int>(blockIdx.x);
        // scaled, rounded outputs of accumulator columns c0 .. c0 + 15 of row r of tile t
        auto store16 = [&](int t, int c0, const float (&a)[16]) {
            const int m = (t % m_tiles) * 256 + static_cast<int>(rank) * 128 + r;
            const int n0 = (t / m_tiles) * BN + c0;
            if (m >= p.M || n0 >= p.N)
                return;
            const float sam = NEST16 ? 1.0f : p.sa[m];
            if constexpr (KIND == kE4M3) {
                if (p.out_f32) {
                    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.y) + static_cast<int64_t>(m) * p.N +
                                                             n0);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        dst[j] = make_float4(a[4 * j] * sam * __ldg(p.sw + n0 + 4 * j),
                                             a[4 * j + 1] * sam * __ldg(p.sw + n0 + 4 * j + 1),
                                             a[4 * j + 2] * sam * __ldg(p.sw + n0 + 4 * j + 2),
                                             a[4 * j + 3] * sam * __ldg(p.sw + n0 + 4 * j + 3));
                    return;
                }
            }
            uint32_t o[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float a0 = a[2 * j] * sam, a1 = a[2 * j + 1] * sam;
                if constexpr (KIND == kE4M3) {
                    a0 = a0 * __ldg(p.sw + n0 + 2 * j);
                    a1 = a1 * __ldg(p.sw + n0 + 2 * j + 1);
                }
                o[j] = pack2<KIND>(a0, a1);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(p.y) + static_cast<int64_t>(m) * p.N + n0);
            dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
            dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
        };
        auto load16 = [&](uint32_t col, float (&a)[16]) {
            uint32_t v[16];
            tmem_ld_32x32b_x16(t_row + col, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j)
                a[j] = __uint_as_float(v[j]);
        };
        auto release = [&](int buf) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (lead)
                    mbar_arrive(&ctl->acc_empty[buf]);
                else
                    mbar_arrive_remote(&ctl->acc_empty[buf], 0u);
            }
        };
        int fin_t = -1, fin_buf = 0;
        int i = 0;
        PairWalk walk(pair, npairs, sk, total, p.kblocks);
        int t, kb0, kb1;
        for (; walk.next(t, kb0, kb1); ++i) {
            const int buf = i & 1;
            const uint32_t use = static_cast<uint32_t>(i >> 1);
            bool ok = wait_bounded_cluster(&ctl->acc_full[buf], use & 1u, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok)
                break;
            tc_fence_after();
            if (kb0 == 0 && kb1 < p.kblocks) {
                // the start of a tile finished with the following pairs'
                // partials: always the last segment; kept in tensor memory
                fin_t = t;
                fin_buf = buf;
                continue;
            }
            const bool contrib = kb0 > 0;   // always the first segment of the stream-K range
            float *slot = sk.partials + static_cast<size_t>(cta) * BN * 128;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 16) {
                float a[16];
                if (contrib) {
                    load16(static_cast<uint32_t>(buf * BN + c0), a);
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        __stcg(slot + (c0 + j) * 128 + r, a[j]);
                } else {
                    if ((t / m_tiles) * BN + c0 >= p.N)
                        break;                  // warp-uniform; N % 16 == 0
                    load16(static_cast<uint32_t>(buf * BN + c0), a);
                    store16(t, c0, a);
                }
            }
            release(buf);
            if (contrib) {
                __threadfence();
                asm volatile("bar.sync 2, 128;" ::: "memory");
                if (r == 0)
                    st_release_u32(sk.flags + cta, 1u);
            }
        }
        if (fin_t >= 0) {
            // this pair's part, then the following pairs' partials in pair order
            const int64_t last = static_cast<int64_t>(fin_t - sk.t0 + 1) * p.kblocks - 1;
            const int p_last = sk_owner(last, sk.units, npairs);
            bool got = true;
            if (r == 0)
                for (int pp = pair + 1; pp <= p_last && got; ++pp)
                    got = wait_flag_sleep(sk.flags + 2 * pp + static_cast<int>(rank), abort_flag);
            got = epi_all(got);
            // the partials, one after another through the idle ring, into
            // this pair's accumulator (the slots of this rank: every other one)
            uint32_t fph = 0;
            if (got && p_last > pair)
                got = add_partials_into_tmem(t_row, static_cast<uint32_t>(fin_buf * BN), BN,
                                             sk.partials + static_cast<size_t>(rank) * BN * 128,
                                             static_cast<size_t>(2) * BN * 128, pair + 1, p_last, smem, &ctl->fix,
                                             fph, abort_flag, r);
            if (got) {
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += 16) {
                    if ((fin_t / m_tiles) * BN + c0 >= p.N)
                        break;
                    float a[16];
                    load16(static_cast<uint32_t>(fin_buf * BN + c0), a);
                    store16(fin_t, c0, a);
                }
                asm volatile("bar.sync 2, 128;" ::: "memory");
                if (r == 0)
                    for (int pp = pair + 1; pp <= p_last; ++pp)
                        sk.flags[2 * pp + rank] = 0u;
            }
            tc_fence_before();
        }
    }

    // ---------------------------------------------------------------- teardown
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();                 // no CTA leaves while its partner may still signal it
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, C::kTmemCols);
    }
}

} // namespace pgf8
