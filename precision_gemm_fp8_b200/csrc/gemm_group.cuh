// Grouped, persistent stream-K GEMM for the weight-streaming (decode-sized
// M) FP8 linear layers of one step: the E4M3 x E4M3 -> f32 -> bf16 layer of
// "C++ and FP8" §3.3 for up to kGroupMaxLayers independent layers at once.
//
// Decode linears are bound by the weight stream ("7B token speed on consumer
// GPUs" §1: bandwidth is the first bottleneck).  One launch per layer pays
// a ramp (CTAs starting, the first weight tiles in flight) and a tail
// (split-K reduction, the last CTAs finishing) on every layer; for a 4096 x
// 4096 layer (2.6 us of weights at HBM speed) those fixed costs are as long
// as the stream itself.  Here the weight tiles of all the group's layers
// form one stream: units are (layer, 128-row weight tile, 128 bytes of K),
// ordered layer by layer and tile by tile, and every CTA (one per SM) takes
// an equal contiguous range of units, so every SM streams the same number
// of weight bytes from the first microsecond to the last, with no gap at a
// layer boundary.
//
// Orientation as the skinny kernel: MMA A = 128 weight rows (K-major),
// MMA B = the layer's tokens, zero-padded to bn = 16..BNMAX rows; the
// instruction descriptor is built per layer (its N is the layer's bn).
// A CTA's range splits into segments, one per weight tile it touches; each
// segment accumulates into one of two tensor-memory buffers, so a segment's
// epilogue overlaps the next segment's main loop.  A tile shared by several
// CTAs is finished by the CTA that holds its first k-block, which is that
// CTA's last segment; the following CTAs contribute the rest as their first
// segment, storing the f32 partial into their workspace slot and raising
// their flag right at the start of their range.  The finishing CTA reaches
// the tile at the end of its range, adds the partials in CTA order after
// its own (a fixed order: deterministic for a given group and grid), clears
// the flags it consumed (the flag words are zero after every completed
// call) and applies the scales.  No CTA waits on a CTA that is waiting.
//
//   warp 0      TMA producer: STAGES-deep ring of (weight tile, token tile)
//   warp 1      tensor-memory allocation, MMA issue (one thread)
//   warps 2-5   epilogue
// Waits are bounded as in gemm.cuh.
#pragma once

#include "gemm.cuh"
#include "gemm_persistent.cuh"
#include "gemm_streamk.cuh"

namespace pgf8 {

constexpr int kGroupMaxLayers = 32;
constexpr int kGroupMaxCtas = 256;             // partial slots in the group workspace
constexpr size_t kGroupFlagBytes = 1024;       // kGroupMaxCtas 32-bit flags

template <int BNMAX_, int STAGES_, int KIND_ = kE4M3> struct GroupCfg {
    static constexpr int BNMAX = BNMAX_;
    static constexpr int STAGES = STAGES_;
    static constexpr int KIND = KIND_;
    static constexpr bool NEST16 = (KIND == kNested16);
    static constexpr int kThreads = NEST16 ? 320 : 192;   // FP16 mode: 4 rebuild warps
    static constexpr int kTileA = 128 * 128;
    static constexpr int kStage = kTileA + BNMAX * 128;
    static constexpr int kTmemCols = (2 * BNMAX) < 32 ? 32 : 2 * BNMAX;
    static constexpr int kRingBytes = STAGES * kStage;
    static constexpr int kBarOffset = kRingBytes;
    static constexpr int kSmemBytes = kRingBytes + 1024 + 1024;
    static_assert(BNMAX == 16 || BNMAX == 32 || BNMAX == 64 || BNMAX == 128 || BNMAX == 256, "token tile");
    static_assert(STAGES <= 16 && kStage % 1024 == 0, "ring");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

__host__ __device__ constexpr size_t group_workspace_bytes(int bnmax)
{
    return kGroupFlagBytes + static_cast<size_t>(kGroupMaxCtas) * bnmax * 128 * 4;
}

struct GroupLayer {
    int64_t unit0;       // first unit of the layer in the group's order
    int M, N, K;
    int kblocks;         // ceil(K bytes / 128): K / 64 k-blocks of FP16 activations in FP16 mode
    int bn;              // token rows of the MMA: M rounded up to 16 (<= BNMAX)
    const float *sa;     // [M] per-token scales (E4M3 and NestedFP FP8 mode)
    const float *sw;     // [N] per-channel scales (E4M3)
    void *y;             // [M, N] bf16 (E4M3), f16 (NestedFP), or f32 when out_f32
    int out_f32;         // 1: y is f32, the scaled sum before rounding
};

struct GroupParams {
    CUtensorMap tmW[kGroupMaxLayers];   // weights [N, K] codes (NestedFP: the hi plane), box 128 x 128;
                                        // FP16 mode: hi plane, box 64 bytes x 128, no swizzle
    CUtensorMap tmW2[kGroupMaxLayers];  // FP16 mode: lo plane, as tmW
    CUtensorMap tmX[kGroupMaxLayers];   // activation codes [M, K], box 128 x bn (FP16 mode: f16, box 64 x bn)
    GroupLayer L[kGroupMaxLayers];
    int nlayers;
    int prefetch_w;      // weights may be read before the grid dependency resolves
    int64_t units;       // total units of the group
    unsigned *flags;     // [kGroupMaxCtas], zero between calls
    float *partials;     // [kGroupMaxCtas][BNMAX][128]
};

// The segment of the range [u, u1) that starts at unit u: layer l (found
// from the hint upwards), weight tile t, k-blocks [kb0, kb1) of that tile.
struct GroupSeg {
    int l, t, kb0, kb1;
};

__device__ __forceinline__ GroupSeg group_seg(const GroupParams &p, int64_t u, int64_t u1, int l_hint)
{
    int l = l_hint;
    while (l + 1 < p.nlayers && p.L[l + 1].unit0 <= u)
        ++l;
    const GroupLayer &g = p.L[l];
    const int64_t local = u - g.unit0;
    GroupSeg s;
    s.l = l;
    s.t = static_cast<int>(local / g.kblocks);
    s.kb0 = static_cast<int>(local % g.kblocks);
    const int64_t tile_end = g.unit0 + static_cast<int64_t>(s.t + 1) * g.kblocks;
    s.kb1 = static_cast<int>((u1 < tile_end ? u1 : tile_end) - g.unit0 - static_cast<int64_t>(s.t) * g.kblocks);
    return s;
}

__device__ __forceinline__ int64_t group_seg_end(const GroupParams &p, const GroupSeg &s)
{
    return p.L[s.l].unit0 + static_cast<int64_t>(s.t) * p.L[s.l].kblocks + s.kb1;
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1) gemm_group_kernel(const __grid_constant__ GroupParams p)
{
    constexpr int BNMAX = C::BNMAX;
    constexpr int STAGES = C::STAGES;
    constexpr int KIND = C::KIND;
    constexpr bool NEST16 = C::NEST16;
    constexpr int kXStep = NEST16 ? 64 : 128;   // activation elements per k-block

    grid_launch_dependents();

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    PersistCtl *ctl = reinterpret_cast<PersistCtl *>(smem + C::kBarOffset);
    volatile int *abort_flag = &ctl->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = static_cast<int>(gridDim.x);
    const int c = static_cast<int>(blockIdx.x);
    const int64_t u0 = sk_unit_begin(c, p.units, G);
    const int64_t u1 = sk_unit_begin(c + 1, p.units, G);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
            mbar_init(&ctl->conv[s], 4);    // FP16 mode: one arrival per rebuild warp
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->acc_full[b], 1);
            mbar_init(&ctl->acc_empty[b], 4);
        }
        mbar_init(&ctl->drain, 1);
        mbar_init(&ctl->fix, 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_x = policy_evict_last();
            bool waited = false;
            if (!p.prefetch_w) {
                grid_dependency_wait();
                waited = true;
            }
            int s = 0;
            uint32_t ph = 0;
            uint32_t issued_mask = 0, issued_ph = 0;
            // stages whose token tile waits for the grid dependency: (layer, kb)
            int pend_l[STAGES], pend_kb[STAGES], pend_s[STAGES];
            int pending = 0;
            int l_hint = 0;
            bool stop = false;
            for (int64_t u = u0; u < u1 && !stop;) {
                const GroupSeg sg = group_seg(p, u, u1, l_hint);
                l_hint = sg.l;
                const GroupLayer &g = p.L[sg.l];
                const uint32_t bytes = static_cast<uint32_t>(C::kTileA + g.bn * 128);
                for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
                    if (!wait_bounded(&ctl->empty[s], ph ^ 1u, abort_flag)) {
                        stop = true;
                        break;
                    }
                    uint8_t *st = smem + s * C::kStage;
                    mbar_arrive_expect_tx(&ctl->full[s], bytes);
                    if constexpr (NEST16) {
                        // hi and lo planes, 64 bytes (= 64 weights) of K each
                        tma_load_2d_hint(st, &p.tmW[sg.l], &ctl->full[s], kb * 64, sg.t * 128, pol_w);
                        tma_load_2d_hint(st + 128 * 64, &p.tmW2[sg.l], &ctl->full[s], kb * 64, sg.t * 128, pol_w);
                    } else {
                        tma_load_2d_hint(st, &p.tmW[sg.l], &ctl->full[s], kb * 128, sg.t * 128, pol_w);
                    }
                    issued_mask |= 1u << s;
                    issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
                    if (waited) {
                        tma_load_2d_hint(st + C::kTileA, &p.tmX[sg.l], &ctl->full[s], kb * kXStep, 0, pol_x);
                    } else {
                        pend_l[pending] = sg.l;
                        pend_kb[pending] = kb;
                        pend_s[pending] = s;
                        if (++pending == STAGES) {
                            // the first ring pass of weights went out before the
                            // grid dependency resolved; token tiles only after it
                            grid_dependency_wait();
                            waited = true;
                            for (int j = 0; j < pending; ++j)
                                tma_load_2d_hint(smem + pend_s[j] * C::kStage + C::kTileA, &p.tmX[pend_l[j]],
                                                 &ctl->full[pend_s[j]], pend_kb[j] * kXStep, 0, pol_x);
                            pending = 0;
                        }
                    }
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                u = group_seg_end(p, sg);
            }
            if (!waited)
                grid_dependency_wait();
            for (int j = 0; j < pending; ++j)
                tma_load_2d_hint(smem + pend_s[j] * C::kStage + C::kTileA, &p.tmX[pend_l[j]], &ctl->full[pend_s[j]],
                                 pend_kb[j] * kXStep, 0, pol_x);
            if (*abort_flag) {
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
            int i = 0;
            int l_hint = 0;
            for (int64_t u = u0; ok && u < u1; ++i) {
                const GroupSeg sg = group_seg(p, u, u1, l_hint);
                l_hint = sg.l;
                // weights are operand A: E5M2 in NestedFP FP8 mode; FP16 in FP16 mode (kind::f16)
                const uint32_t idesc = make_idesc(128, p.L[sg.l].bn, KIND == kNested8 ? 1 : 0, 0);
                const int buf = i & 1;
                const uint32_t use = static_cast<uint32_t>(i >> 1);
                if (!wait_bounded(&ctl->acc_empty[buf], (use & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + static_cast<uint32_t>(buf * BNMAX);
                for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
                    if (!wait_bounded(&ctl->full[s], ph, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if constexpr (NEST16) {
                        if (!wait_bounded(&ctl->conv[s], ph, abort_flag)) {
                            ok = false;
                            break;
                        }
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * C::kStage);
                    const uint32_t b_addr = a_addr + C::kTileA;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint32_t acc = (kb > sg.kb0 || k > 0) ? 1u : 0u;
                        if constexpr (NEST16)
                            umma_f16(d, sdesc_sw128(a_addr + k * 32), sdesc_sw128(b_addr + k * 32), idesc, acc);
                        else
                            umma_f8f6f4(d, sdesc_sw128(a_addr + k * 32), sdesc_sw128(b_addr + k * 32), idesc, acc);
                    }
                    umma_commit(&ctl->empty[s]);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (ok)
                    umma_commit(&ctl->acc_full[buf]);
                u = group_seg_end(p, sg);
            }
            if (!ok) {
                umma_commit(&ctl->drain);
                wait_drain(&ctl->drain, 0);
            }
        }
        __syncwarp();
    } else if (warp >= 6) {
        // ------------------------------------------------------------ FP16 rebuild (FP16 mode)
        if constexpr (NEST16) {
            const int tt = static_cast<int>(threadIdx.x) - 192;   // 0..127
            int s = 0;
            uint32_t ph = 0;
            int l_hint = 0;
            bool ok = true;
            for (int64_t u = u0; ok && u < u1;) {
                const GroupSeg sg = group_seg(p, u, u1, l_hint);
                l_hint = sg.l;
                for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
                    if (!wait_bounded(&ctl->full[s], ph, abort_flag)) {
                        ok = false;
                        break;
                    }
                    rebuild_fp16_tile<128>(smem + s * C::kStage, tt);
                    fence_proxy_async_smem();   // each writer, before the MMA (async proxy) reads
                    __syncwarp();
                    if ((threadIdx.x & 31) == 0)
                        mbar_arrive(&ctl->conv[s]);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                u = group_seg_end(p, sg);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        grid_dependency_wait();   // per-token scales come from the kernel before
        const int qd = warp & 3;
        const int r = qd * 32 + lane;
        const uint32_t t_row = tmem + (static_cast<uint32_t>(qd * 32) << 16);
        // outputs of tokens c0 .. c0 + 15 of accumulator row r (channel n of
        // tile t of layer g)
        auto store16 = [&](const GroupLayer &g, int t, int c0, const float (&a)[16]) {
            const int n = t * 128 + r;
            if (n >= g.N)
                return;
            if constexpr (KIND == kE4M3) {
                const float swn = g.sw[n];
                if (g.out_f32) {
                    float *y = static_cast<float *>(g.y);
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (c0 + j < g.M)
                            y[static_cast<int64_t>(c0 + j) * g.N + n] = a[j] * __ldg(g.sa + c0 + j) * swn;
                    return;
                }
                __nv_bfloat16 *y = static_cast<__nv_bfloat16 *>(g.y);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (c0 + j < g.M)
                        y[static_cast<int64_t>(c0 + j) * g.N + n] =
                            __float2bfloat16_rn(a[j] * __ldg(g.sa + c0 + j) * swn);
            } else {
                // NestedFP: f16 out; FP8 mode scales by the per-token scale
                __half *y = static_cast<__half *>(g.y);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    if (c0 + j < g.M) {
                        float v = a[j];
                        if constexpr (KIND == kNested8)
                            v = v * __ldg(g.sa + c0 + j);
                        y[static_cast<int64_t>(c0 + j) * g.N + n] = __float2half_rn(v);
                    }
                }
            }
        };
        auto load16 = [&](uint32_t col, float (&a)[16]) {
            uint32_t v[16];
            tmem_ld_32x32b_x16(t_row + col, v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j)
                a[j] = __uint_as_float(v[j]);
        };
        int fin_l = -1, fin_t = -1, fin_buf = 0;
        int i = 0;
        int l_hint = 0;
        for (int64_t u = u0; u < u1; ++i) {
            const GroupSeg sg = group_seg(p, u, u1, l_hint);
            l_hint = sg.l;
            u = group_seg_end(p, sg);
            const GroupLayer &g = p.L[sg.l];
            const int buf = i & 1;
            const uint32_t use = static_cast<uint32_t>(i >> 1);
            bool ok = wait_bounded(&ctl->acc_full[buf], use & 1u, abort_flag);
            if (!epi_all(ok))
                break;
            tc_fence_after();
            const bool contrib = sg.kb0 > 0;   // the rest of a tile begun by a preceding CTA
            if (!contrib && sg.kb1 < g.kblocks) {
                // the start of a tile finished with the following CTAs'
                // partials: always this CTA's last segment; its accumulator
                // stays in tensor memory until the partials are added
                fin_l = sg.l;
                fin_t = sg.t;
                fin_buf = buf;
                continue;
            }
            float *slot = p.partials + static_cast<size_t>(c) * BNMAX * 128;
#pragma unroll 1
            for (int c0 = 0; c0 < g.bn; c0 += 16) {
                float a[16];
                load16(static_cast<uint32_t>(buf * BNMAX + c0), a);
                if (contrib) {
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        __stcg(slot + (c0 + j) * 128 + r, a[j]);
                } else {
                    store16(g, sg.t, c0, a);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&ctl->acc_empty[buf]);   // the accumulator buffer is free again
            if (contrib) {
                // always this CTA's first segment: published at once
                __threadfence();
                asm volatile("bar.sync 2, 128;" ::: "memory");
                if (r == 0)
                    st_release_u32(p.flags + c, 1u);
            }
        }
        if (fin_l >= 0) {
            // this CTA's own part first, then the following CTAs' partials in
            // CTA order
            const GroupLayer &g = p.L[fin_l];
            const int64_t last = g.unit0 + static_cast<int64_t>(fin_t + 1) * g.kblocks - 1;
            const int c_last = sk_owner(last, p.units, G);
            bool got = true;
            if (r == 0)
                for (int cc = c + 1; cc <= c_last && got; ++cc)
                    got = wait_flag_sleep(p.flags + cc, abort_flag);
            got = epi_all(got);
            // the partials, one after another through the idle ring, into
            // this CTA's accumulator
            uint32_t fph = 0;
            if (got && c_last > c)
                got = add_partials_into_tmem(t_row, static_cast<uint32_t>(fin_buf * BNMAX), g.bn, p.partials,
                                             static_cast<size_t>(BNMAX) * 128, c + 1, c_last, smem, &ctl->fix, fph,
                                             abort_flag, r);
            if (got) {
#pragma unroll 1
                for (int c0 = 0; c0 < g.bn; c0 += 16) {
                    float a[16];
                    load16(static_cast<uint32_t>(fin_buf * BNMAX + c0), a);
                    store16(g, fin_t, c0, a);
                }
                asm volatile("bar.sync 2, 128;" ::: "memory");
                if (r == 0)
                    for (int cc = c + 1; cc <= c_last; ++cc)
                        p.flags[cc] = 0u;
            }
            tc_fence_before();
        }
    }

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
