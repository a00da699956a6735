// Persistent tcgen05 GEMM for the tiled orientation (tokens are the 128-row
// MMA operand): the prefill-sized layers of "C++ and FP8" §3.3 (E4M3 x E4M3,
// f32 accumulate, bf16 out) and both NestedFP modes ("NestedFP" §2.2).
//
// One CTA per SM walks the output tiles t = blockIdx.x, + gridDim.x, ...
// (tile t covers tokens (t % m_tiles) * 128 and channels (t / m_tiles) * BN,
// so the CTAs working at the same time share weight tiles in L2).  The
// accumulator is double-buffered in tensor memory (2 x BN columns), so the
// epilogue of one tile overlaps the main loop of the next:
//   warp 0      TMA producer, running ahead across tiles through the ring;
//   warp 1      MMA issuer: waits for a free accumulator buffer, K loop,
//               commits the buffer to the epilogue;
//   warps 2-5   epilogue: tcgen05.ld, scaling, rounding, 32-byte stores,
//               then hand the buffer back;
//   warps 6-9   (NestedFP FP16 mode only) rebuild FP16 weight tiles from the
//               hi/lo planes in shared memory.
// Waits are bounded as in gemm.cuh.
#pragma once

#include "gemm.cuh"

namespace pgf8 {

template <int BN_, int STAGES_, int KIND_> struct PersistCfg {
    static constexpr int BN = BN_;
    static constexpr int STAGES = STAGES_;
    static constexpr int KIND = KIND_;
    static constexpr int XQ = 0;   // activations arrive as E4M3 codes
    static constexpr bool SWAP = false;
    static constexpr bool NEST16 = (KIND == kNested16);
    static constexpr int kThreads = NEST16 ? 320 : 192;
    static constexpr int kTileA = 128 * 128;
    static constexpr int kTileB = BN * 128;
    static constexpr int kStage = kTileA + kTileB;
    static constexpr int kRowsW = BN;
    static constexpr int kRowsX = 128;
    static constexpr int kTmemCols = 2 * BN;
    static constexpr int kRingBytes = STAGES * kStage;
    static constexpr int kBarOffset = kRingBytes;
    static constexpr int kSmemBytes = kRingBytes + 1024 + 1024;
    static_assert(BN % 16 == 0 && BN >= 64 && BN <= 256, "BN");
    static_assert(kTmemCols <= 512, "tensor memory");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
    static_assert(STAGES <= 16, "stages");
};

struct PersistCtl {
    uint64_t full[16];
    uint64_t empty[16];
    uint64_t conv[16];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint64_t fix;        // stream-K kernels: partial tiles copied into shared memory
    uint32_t tmem_base;
    int abort;
};

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1)
    gemm_persistent_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                           const __grid_constant__ CUtensorMap tmW2, const GemmParams p)
{
    constexpr int BN = C::BN;
    constexpr int STAGES = C::STAGES;
    constexpr int KIND = C::KIND;
    constexpr bool NEST16 = C::NEST16;
    constexpr uint32_t kIdesc = make_idesc(128, BN, 0, KIND == kNested8 ? 1 : 0);
    constexpr int kXStep = NEST16 ? 64 : 128;   // K elements per stage

    grid_launch_dependents();

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    PersistCtl *ctl = reinterpret_cast<PersistCtl *>(smem + C::kBarOffset);
    volatile int *abort_flag = &ctl->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int m_tiles = (p.M + 127) / 128;
    const int n_tiles = (p.N + BN - 1) / BN;
    const int total = m_tiles * n_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
            mbar_init(&ctl->conv[s], 4);    // one arrival per rebuild warp
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->acc_full[b], 1);
            mbar_init(&ctl->acc_empty[b], 4);   // one arrival per epilogue warp
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
    grid_dependency_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = policy_evict_last();
            int s = 0;
            uint32_t ph = 0;
            uint32_t issued_mask = 0, issued_ph = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
                const int row0_x = (t % m_tiles) * 128;
                const int row0_w = (t / m_tiles) * BN;
                for (int kb = 0; kb < p.kblocks; ++kb) {
                    if (!wait_bounded(&ctl->empty[s], ph ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = smem + s * C::kStage;
                    mbar_arrive_expect_tx(&ctl->full[s], C::kStage);
                    if constexpr (NEST16) {
                        tma_load_2d_hint(st + C::kTileA, &tmW, &ctl->full[s], kb * 64, row0_w, pol);
                        tma_load_2d_hint(st + C::kTileA + BN * 64, &tmW2, &ctl->full[s], kb * 64, row0_w, pol);
                    } else {
                        tma_load_2d_hint(st + C::kTileA, &tmW, &ctl->full[s], kb * 128, row0_w, pol);
                    }
                    tma_load_2d_hint(st, &tmX, &ctl->full[s], kb * kXStep, row0_x, pol);
                    issued_mask |= 1u << s;
                    issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (*abort_flag) {
                for (int j = 0; j < STAGES; ++j)
                    if (issued_mask & (1u << j))
                        wait_drain(&ctl->full[j], (issued_ph >> j) & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            int i = 0;
            for (int t = blockIdx.x; ok && t < total; t += gridDim.x, ++i) {
                const int buf = i & 1;
                const uint32_t use = static_cast<uint32_t>(i >> 1);
                if (!wait_bounded(&ctl->acc_empty[buf], (use & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + static_cast<uint32_t>(buf * BN);
                for (int kb = 0; kb < p.kblocks; ++kb) {
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
                        const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
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
            }
            if (!ok) {
                umma_commit(&ctl->drain);
                wait_drain(&ctl->drain, 0);
            }
        }
        __syncwarp();
    } else if (warp < 6) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                 // tensor-memory lane quadrant
        const int r = q * 32 + lane;
        const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16);
        int i = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++i) {
            const int buf = i & 1;
            const uint32_t use = static_cast<uint32_t>(i >> 1);
            bool ok = wait_bounded(&ctl->acc_full[buf], use & 1u, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok)
                break;
            tc_fence_after();
            const int m = (t % m_tiles) * 128 + r;
            const int n_base = (t / m_tiles) * BN;
            float sam = 1.0f;
            if constexpr (KIND != kNested16)
                sam = (m < p.M) ? p.sa[m] : 0.0f;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 16) {
                const int n0 = n_base + c0;
                if (n0 >= p.N)
                    break;                      // warp-uniform; N % 16 == 0
                uint32_t v[16];
                tmem_ld_32x32b_x16(t_row + static_cast<uint32_t>(buf * BN + c0), v);
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
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&ctl->acc_empty[buf]);
        }
    } else {
        // ------------------------------------------------------------ FP16 rebuild
        if constexpr (NEST16) {
            const int tt = static_cast<int>(threadIdx.x) - 192;   // 0..127
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
                for (int kb = 0; kb < p.kblocks; ++kb) {
                    if (!wait_bounded(&ctl->full[s], ph, abort_flag)) {
                        ok = false;
                        break;
                    }
                    rebuild_fp16_tile<BN>(smem + s * C::kStage + C::kTileA, tt);
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
