// Stream-K skinny tcgen05 GEMM for decode-sized M (M <= 32): the weight-
// streaming form of the FP8 linear layer ("C++ and FP8" §3.3) and of both
// NestedFP modes ("NestedFP" §2.2).
//
// The 128-row weight tiles are the MMA A operand, the (zero-padded) tokens
// the BN-row B operand.  The work — units of (weight tile, 128 bytes of K) —
// is cut into gridDim.x equal contiguous ranges, one per CTA, ordered tile
// by tile, so every CTA streams the same number of weight bytes and the grid
// (one CTA per SM, ~110 KB of shared memory) leaves room on every SM for the
// next layer's CTAs to load their first weight tiles before this layer ends.
//
// A CTA's range splits into segments, one per weight tile it touches; each
// segment accumulates into one of two tensor-memory buffers (the epilogue of
// a segment overlaps the next segment's main loop).  A segment that covers
// its whole tile is written out directly.  A tile shared by several CTAs is
// finished by the CTA that holds its last k-block: the other CTAs (always
// the preceding ones, each contributing its last segment) store their f32
// partial tile into their slot of the workspace and raise their flag; the
// finishing CTA waits for those flags (bounded), adds the partials in CTA
// order and then its own (a fixed order: deterministic), applies the scales
// and clears the flags it consumed, which leaves the flag words zero after
// every completed call.
#pragma once

#include "gemm.cuh"
#include "gemm_persistent.cuh"

namespace pgf8 {

constexpr int kStreamKMaxCtas = 256;           // partial slots in the workspace
constexpr size_t kStreamKFlagBytes = 1024;     // kStreamKMaxCtas 32-bit flags

template <int BN_, int STAGES_, int KIND_> struct StreamKCfg {
    static constexpr int BN = BN_;
    static constexpr int STAGES = STAGES_;
    static constexpr int KIND = KIND_;
    static constexpr int XQ = 0;   // activations arrive as E4M3 codes
    static constexpr bool SWAP = true;
    static constexpr bool NEST16 = (KIND == kNested16);
    static constexpr int kThreads = NEST16 ? 320 : 192;
    static constexpr int kTileA = 128 * 128;
    static constexpr int kTileB = BN * 128;
    static constexpr int kStage = kTileA + kTileB;
    static constexpr int kRowsW = 128;
    static constexpr int kRowsX = BN;
    static constexpr int kTmemCols = (2 * BN) < 32 ? 32 : 2 * BN;
    static constexpr int kRingBytes = STAGES * kStage;
    static constexpr int kBarOffset = kRingBytes;
    static constexpr int kSmemBytes = kRingBytes + 1024 + 1024;
    static_assert(BN == 16 || BN == 32, "stream-K kernel serves M <= 32");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

__host__ __device__ constexpr size_t streamk_workspace_bytes(int bn)
{
    return kStreamKFlagBytes + static_cast<size_t>(kStreamKMaxCtas) * bn * 128 * 4;
}

struct StreamKParams {
    int64_t units;        // weight tiles x k-blocks
    unsigned *flags;      // [kStreamKMaxCtas], zero between calls
    float *partials;      // [kStreamKMaxCtas][BN][128]
};

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u32(unsigned *p, unsigned v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// All 128 epilogue threads (named barrier 2) agree on a predicate: true only
// if it is true in every one of them.  Keeps their later barriers aligned
// even when one of them gave up a bounded wait.
__device__ __forceinline__ bool epi_all(bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 2, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(v))
        : "memory");
    return r != 0;
}

// Bounded wait for a flag word to become nonzero.
__device__ __forceinline__ bool wait_flag(const unsigned *f, volatile int *abort)
{
    if (ld_acquire_u32(f) != 0u)
        return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t spin = 1;; ++spin) {
        if (ld_acquire_u32(f) != 0u)
            return true;
        if ((spin & 15u) == 0) {
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

// Bounded wait for a flag word, for ONE thread of a CTA, sleeping between
// polls (64 ns doubling to 1 us): a CTA of spinning threads would flood L2
// with loads that the TMA loads of the CTAs still computing need.  The
// caller releases the CTA's other threads with a barrier afterwards.
__device__ __forceinline__ bool wait_flag_sleep(const unsigned *f, volatile int *abort)
{
    if (ld_acquire_u32(f) != 0u)
        return true;
    const uint64_t t0 = global_timer_ns();
    unsigned ns = 64;
    for (;;) {
        __nanosleep(ns);
        if (ld_acquire_u32(f) != 0u)
            return true;
        if (ns < 1024)
            ns <<= 1;
        if (*abort)
            return false;
        if (global_timer_ns() - t0 > kWaitLimitNs) {
            *abort = 1;
            atomicOr(&g_device_error, kErrTimeout);
            return false;
        }
    }
}

// Finishing side of a tile shared by several CTAs: adds the partial tiles
// of the CTAs cfirst .. clast (slot c at parts + c * slot_floats; column j
// of accumulator row r at j * 128 + r) in that order into this CTA's
// accumulator columns [col0, col0 + ncols) of tensor memory, for the 128
// rows owned by warps 2-5 (thread r; t_row = its warp's lane quadrant).
// One partial at a time, one thread copies it whole into `stage` (idle
// shared memory of at least ncols * 512 bytes) with the bulk-copy engine;
// every thread then adds its row from shared memory into tensor memory.
// Reading the partials from global memory chunk by chunk instead costs a
// dependent L2 round trip per 16 columns.  Returns false when a wait gave
// up.  Called by all 128 threads; uses named barrier 2.
__device__ __forceinline__ bool add_partials_into_tmem(uint32_t t_row, uint32_t col0, int ncols, const float *parts,
                                                       size_t slot_floats, int cfirst, int clast, uint8_t *stage,
                                                       uint64_t *bar, uint32_t &phase, volatile int *abort, int r)
{
    const float *st = reinterpret_cast<const float *>(stage);
    for (int c = cfirst; c <= clast; ++c) {
        if (r == 0) {
            fence_proxy_async_smem();   // earlier generic reads of `stage` before the copy overwrites it
            mbar_arrive_expect_tx(bar, static_cast<uint32_t>(ncols) * 512u);
            bulk_copy_g2s(stage, parts + static_cast<size_t>(c) * slot_floats, static_cast<uint32_t>(ncols) * 512u,
                          bar);
        }
        bool ok = wait_bounded(bar, phase, abort);
        phase ^= 1u;
        if (!epi_all(ok)) {
            if (r == 0)
                wait_drain(bar, phase ^ 1u);   // the copy in flight lands before the CTA may exit
            return false;
        }
#pragma unroll 1
        for (int c0 = 0; c0 < ncols; c0 += 16) {
            uint32_t v[16];
            tmem_ld_32x32b_x16(t_row + col0 + static_cast<uint32_t>(c0), v);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j)
                v[j] = __float_as_uint(__uint_as_float(v[j]) + st[(c0 + j) * 128 + r]);
            tmem_st_32x32b_x16(t_row + col0 + static_cast<uint32_t>(c0), v);
        }
        tmem_st_wait();
        asm volatile("bar.sync 2, 128;" ::: "memory");   // every row read before the next copy
    }
    return true;
}

__device__ __forceinline__ int64_t sk_unit_begin(int c, int64_t units, int G)
{
    return (static_cast<int64_t>(c) * units) / G;
}

// The CTA whose range holds unit u.
__device__ __forceinline__ int sk_owner(int64_t u, int64_t units, int G)
{
    int c = static_cast<int>((u * G) / units);
    while (c + 1 < G && sk_unit_begin(c + 1, units, G) <= u)
        ++c;
    while (c > 0 && sk_unit_begin(c, units, G) > u)
        --c;
    return c;
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1)
    gemm_streamk_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                        const __grid_constant__ CUtensorMap tmW2, const GemmParams p, const StreamKParams q)
{
    constexpr int BN = C::BN;
    constexpr int STAGES = C::STAGES;
    constexpr int KIND = C::KIND;
    constexpr bool NEST16 = C::NEST16;
    constexpr uint32_t kIdesc = make_idesc(128, BN, KIND == kNested8 ? 1 : 0, 0);
    constexpr int kXStep = NEST16 ? 64 : 128;

    grid_launch_dependents();

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    PersistCtl *ctl = reinterpret_cast<PersistCtl *>(smem + C::kBarOffset);
    volatile int *abort_flag = &ctl->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = static_cast<int>(gridDim.x);
    const int c = static_cast<int>(blockIdx.x);
    const int kbt = p.kblocks;
    const int64_t u0 = sk_unit_begin(c, q.units, G);
    const int64_t u1 = sk_unit_begin(c + 1, q.units, G);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
            mbar_init(&ctl->conv[s], 4);    // one arrival per rebuild warp
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->acc_full[b], 1);
            mbar_init(&ctl->acc_empty[b], 4);
        }
        mbar_init(&ctl->drain, 1);
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
            int pending = 0;
            for (int64_t u = u0; u < u1; ++u) {
                const int t = static_cast<int>(u / kbt);
                const int kb = static_cast<int>(u % kbt);
                if (!wait_bounded(&ctl->empty[s], ph ^ 1u, abort_flag))
                    break;
                uint8_t *st = smem + s * C::kStage;
                mbar_arrive_expect_tx(&ctl->full[s], C::kStage);
                if constexpr (NEST16) {
                    tma_load_2d_hint(st, &tmW, &ctl->full[s], kb * 64, t * 128, pol_w);
                    tma_load_2d_hint(st + 128 * 64, &tmW2, &ctl->full[s], kb * 64, t * 128, pol_w);
                } else {
                    tma_load_2d_hint(st, &tmW, &ctl->full[s], kb * 128, t * 128, pol_w);
                }
                issued_mask |= 1u << s;
                issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
                if (waited) {
                    tma_load_2d_hint(st + C::kTileA, &tmX, &ctl->full[s], kb * kXStep, 0, pol_x);
                } else if (++pending == STAGES || u + 1 == u1) {
                    // weights of the first pass went out before the grid
                    // dependency resolved; activations only after it
                    grid_dependency_wait();
                    waited = true;
                    for (int j = 0; j < pending; ++j) {
                        const int64_t uj = u - pending + 1 + j;
                        const int sj = (s - pending + 1 + j + STAGES) % STAGES;
                        tma_load_2d_hint(smem + sj * C::kStage + C::kTileA, &tmX, &ctl->full[sj],
                                         static_cast<int>(uj % kbt) * kXStep, 0, pol_x);
                    }
                    pending = 0;
                }
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            if (!waited)
                grid_dependency_wait();
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
            for (int64_t u = u0; ok && u < u1; ++i) {
                const int t = static_cast<int>(u / kbt);
                const int64_t seg_end = min(u1, static_cast<int64_t>(t + 1) * kbt);
                const int buf = i & 1;
                const uint32_t use = static_cast<uint32_t>(i >> 1);
                if (!wait_bounded(&ctl->acc_empty[buf], (use & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + static_cast<uint32_t>(buf * BN);
                for (int64_t v = u; v < seg_end; ++v) {
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
                        const uint64_t ad = sdesc_sw128(a_addr + k * 32);
                        const uint64_t bd = sdesc_sw128(b_addr + k * 32);
                        const uint32_t acc = (v > u || k > 0) ? 1u : 0u;
                        if constexpr (NEST16)
                            umma_f16(d, ad, bd, kIdesc, acc);
                        else
                            umma_f8f6f4(d, ad, bd, kIdesc, acc);
                    }
                    umma_commit(&ctl->empty[s]);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (ok)
                    umma_commit(&ctl->acc_full[buf]);
                u = seg_end;
            }
            if (!ok) {
                umma_commit(&ctl->drain);
                wait_drain(&ctl->drain, 0);
            }
        }
        __syncwarp();
    } else if (warp < 6) {
        // ------------------------------------------------------------ epilogue
        grid_dependency_wait();
        const int qd = warp & 3;
        const int r = qd * 32 + lane;
        const uint32_t t_row = tmem + (static_cast<uint32_t>(qd * 32) << 16);
        // Output of one accumulator row of tile t (this thread: channel n).
        auto store_row = [&](int t, const float (&a)[BN]) {
            const int n = t * 128 + r;
            if (n < p.N) {
                float swn = 1.0f;
                if constexpr (KIND == kE4M3)
                    swn = p.sw[n];
#pragma unroll
                for (int j = 0; j < BN; ++j) {
                    if (j < p.M) {
                        float v = a[j];
                        if constexpr (KIND != kNested16)
                            v = v * p.sa[j];
                        if constexpr (KIND == kE4M3)
                            v = v * swn;
                        store_out<KIND>(p.y, static_cast<int64_t>(j) * p.N + n, v);
                    }
                }
            }
        };
        // The first segment may finish a tile started by preceding CTAs; its
        // values wait in registers until the end, so that this CTA publishes
        // its own partial (its last segment) first and no CTA ever waits on a
        // CTA that is itself waiting.
        float first[BN];
        int deferred_tile = -1;
        int i = 0;
        for (int64_t u = u0; u < u1; ++i) {
            const int t = static_cast<int>(u / kbt);
            const int kb_first = static_cast<int>(u % kbt);
            const int64_t seg_end = min(u1, static_cast<int64_t>(t + 1) * kbt);
            const bool tile_done = (seg_end == static_cast<int64_t>(t + 1) * kbt);   // holds the tile's last k-block
            const int buf = i & 1;
            const uint32_t use = static_cast<uint32_t>(i >> 1);
            bool ok = wait_bounded(&ctl->acc_full[buf], use & 1u, abort_flag);
            if (!epi_all(ok))
                break;
            tc_fence_after();
            float a[BN];
#pragma unroll
            for (int c0 = 0; c0 < BN; c0 += 16) {
                uint32_t v[16];
                tmem_ld_32x32b_x16(t_row + static_cast<uint32_t>(buf * BN + c0), v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    a[c0 + j] = __uint_as_float(v[j]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&ctl->acc_empty[buf]);   // accumulator values are in registers now

            if (!tile_done) {
                // a partial of a shared tile: always this CTA's last segment
                float *slot = q.partials + static_cast<size_t>(c) * BN * 128;
#pragma unroll
                for (int j = 0; j < BN; ++j)
                    __stcg(slot + j * 128 + r, a[j]);
                __threadfence();
                asm volatile("bar.sync 2, 128;" ::: "memory");
                if (r == 0)
                    st_release_u32(q.flags + c, 1u);
            } else if (kb_first > 0) {
                // finishes a shared tile: always this CTA's first segment
#pragma unroll
                for (int j = 0; j < BN; ++j)
                    first[j] = a[j];
                deferred_tile = t;
            } else {
                store_row(t, a);
            }
            u = seg_end;
        }
        if (deferred_tile >= 0) {
            // add the preceding CTAs' partials in CTA order, then this CTA's own
            const int t = deferred_tile;
            const int c_first = sk_owner(static_cast<int64_t>(t) * kbt, q.units, G);
            float sum[BN];
#pragma unroll
            for (int j = 0; j < BN; ++j)
                sum[j] = 0.0f;
            bool got = true;
            if (r == 0)
                for (int cc = c_first; cc < c && got; ++cc)
                    got = wait_flag_sleep(q.flags + cc, abort_flag);
            got = epi_all(got);
            for (int cc = c_first; got && cc < c; ++cc) {
                const float *slot = q.partials + static_cast<size_t>(cc) * BN * 128;
#pragma unroll
                for (int j = 0; j < BN; ++j)
                    sum[j] += __ldcg(slot + j * 128 + r);
            }
#pragma unroll
            for (int j = 0; j < BN; ++j)
                sum[j] = sum[j] + first[j];
            asm volatile("bar.sync 2, 128;" ::: "memory");
            if (got && r == 0)
                for (int cc = c_first; cc < c; ++cc)
                    q.flags[cc] = 0u;
            store_row(t, sum);
        }
    } else {
        // ------------------------------------------------------------ FP16 rebuild
        if constexpr (NEST16) {
            grid_dependency_wait();
            const int tt = static_cast<int>(threadIdx.x) - 192;
            int s = 0;
            uint32_t ph = 0;
            for (int64_t u = u0; u < u1; ++u) {
                if (!wait_bounded(&ctl->full[s], ph, abort_flag))
                    break;
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
