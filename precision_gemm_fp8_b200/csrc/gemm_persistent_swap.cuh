// NestedFP FP16 mode ("NestedFP" §2.1-2.2: the FP16 weight rebuilt as
// (hi << 8) | lo inside the GEMM) for large M, in the swapped orientation:
// the rebuilt weights are the 128-row MMA A operand and the tokens the
// BN-row B operand, so each k-step rebuilds a 128-row weight tile (16 KB)
// instead of a BN-row one.  Per 64 elements of K and 128 x 256 outputs the
// shared memory moves about 128 KB (TMA 48, rebuild 16 + 16, MMA 48)
// against 160 KB when the tokens are the A operand; the FP16-mode GEMM is
// bound by that traffic.
//
// One CTA per SM walks the output tiles t = blockIdx.x, + gridDim.x, ...:
// tile t covers tokens (t % m_tiles) * BN and weight rows (t / m_tiles) * 128
// (the CTAs working at the same time share weight tiles in L2).  The
// accumulator (128 weight rows x BN tokens) is double-buffered in tensor
// memory.  Roles as gemm_persistent_kernel: warp 0 TMA producer, warp 1 MMA
// issuer, warps 2-5 epilogue (each thread one weight row: 16 tokens per
// tensor-memory load, one FP16 store per token, a warp's stores 64
// contiguous bytes of a token's row), warps 6-9 rebuild.  Waits are bounded
// as in gemm.cuh.
#pragma once

#include "gemm_persistent.cuh"

namespace pgf8 {

template <int BN_, int STAGES_> struct PersistSwapCfg {
    static constexpr int BN = BN_;                 // tokens per tile (MMA N)
    static constexpr int STAGES = STAGES_;
    static constexpr int KIND = kNested16;
    static constexpr int XQ = 0;
    static constexpr bool SWAP = true;
    static constexpr bool NEST16 = true;
    static constexpr int kThreads = 320;
    static constexpr int kTileA = 128 * 128;       // 128 weight rows x 64 FP16 (rebuilt from 2 x 8 KB planes)
    static constexpr int kTileB = BN * 128;        // BN token rows x 64 FP16
    static constexpr int kStage = kTileA + kTileB;
    static constexpr int kRowsW = 128;
    static constexpr int kRowsX = BN;
    static constexpr int kTmemCols = 2 * BN;
    static constexpr int kRingBytes = STAGES * kStage;
    static constexpr int kBarOffset = kRingBytes;
    static constexpr int kSmemBytes = kRingBytes + 1024 + 1024;
    static_assert(BN % 16 == 0 && BN >= 64 && BN <= 256, "BN");
    static_assert(kTmemCols <= 512, "tensor memory");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
    static_assert(STAGES <= 16, "stages");
};

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1)
    gemm_persistent_swap_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                                const __grid_constant__ CUtensorMap tmW2, const GemmParams p)
{
    constexpr int BN = C::BN;
    constexpr int STAGES = C::STAGES;
    constexpr uint32_t kIdesc = make_idesc(128, BN, 0, 0);   // f16 x f16 -> f32, M = 128 weights, N = BN tokens

    grid_launch_dependents();

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    PersistCtl *ctl = reinterpret_cast<PersistCtl *>(smem + C::kBarOffset);
    volatile int *abort_flag = &ctl->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int m_tiles = (p.M + BN - 1) / BN;
    const int n_tiles = (p.N + 127) / 128;
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
                const int row0_x = (t % m_tiles) * BN;
                const int row0_w = (t / m_tiles) * 128;
                for (int kb = 0; kb < p.kblocks; ++kb) {
                    if (!wait_bounded(&ctl->empty[s], ph ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = smem + s * C::kStage;
                    mbar_arrive_expect_tx(&ctl->full[s], C::kStage);
                    tma_load_2d_hint(st, &tmW, &ctl->full[s], kb * 64, row0_w, pol);
                    tma_load_2d_hint(st + 128 * 64, &tmW2, &ctl->full[s], kb * 64, row0_w, pol);
                    tma_load_2d_hint(st + C::kTileA, &tmX, &ctl->full[s], kb * 64, row0_x, pol);
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
                    if (!wait_bounded(&ctl->full[s], ph, abort_flag) || !wait_bounded(&ctl->conv[s], ph, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * C::kStage);   // rebuilt weights
                    const uint32_t b_addr = a_addr + C::kTileA;                // tokens
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        umma_f16(d, sdesc_sw128(a_addr + k * 32), sdesc_sw128(b_addr + k * 32), kIdesc,
                                 (kb > 0 || k > 0) ? 1u : 0u);
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
        // ------------------------------------------------------------ epilogue: one weight row per thread
        const int q = warp & 3;                 // tensor-memory lane quadrant
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
            const int n = (t / m_tiles) * 128 + q * 32 + lane;
            const int m_base = (t % m_tiles) * BN;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 16) {
                if (m_base + c0 >= p.M)
                    break;                      // warp-uniform
                uint32_t v[16];
                tmem_ld_32x32b_x16(t_row + static_cast<uint32_t>(buf * BN + c0), v);
                tmem_ld_wait();
                if (n < p.N) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int m = m_base + c0 + j;
                        if (m < p.M)
                            store_out<kNested16>(p.y, static_cast<int64_t>(m) * p.N + n, __uint_as_float(v[j]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&ctl->acc_empty[buf]);
        }
    } else {
        // ------------------------------------------------------------ FP16 rebuild of the 128 weight rows
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
