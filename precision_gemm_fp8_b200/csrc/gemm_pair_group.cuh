// The tiled FP8 linear layer ("C++ and FP8" §3.3: E4M3 x E4M3 -> f32 ->
// bf16) for several independent layers in one persistent launch on CTA
// pairs (cta_group::2): the 256 x 256 output tiles of every layer form one
// list, layer after layer, and the pairs walk it round-robin as the
// single-layer pair kernel walks one layer's tiles.  A layer whose tiles
// fill only part of a round (few tiles, or the ragged last round) no longer
// leaves SMs idle: the next layer's tiles fill in, and the launch pays its
// start and end once for all the layers.
//
// Roles, ring, barriers and the epilogue are those of gemm_pair_kernel
// (gemm_2sm.cuh), FP8 operands only: every tile reads its layer's tensor
// maps, token count, weight-row count, k-block count, scales and output.
// Every walk visits tiles in increasing order, so each role finds a tile's
// layer by moving a hint forward.
#pragma once

#include "gemm_2sm.cuh"

namespace pgf8 {

constexpr int kPairGroupMaxLayers = 32;

struct PairGroupLayer {
    int M, N, kblocks;
    int m_tiles;          // 256-row token tiles of the layer
    int tile0;            // the layer's first tile in the launch's list
    const float *sa, *sw; // [M], [N]
    void *y;              // [M, N] bf16
};

struct PairGroupParams {
    CUtensorMap tmX[kPairGroupMaxLayers];   // activation codes [M, K], box 128 x 128, 128-byte swizzle
    CUtensorMap tmW[kPairGroupMaxLayers];   // weight codes [N, K], box 128 x 128, 128-byte swizzle
    PairGroupLayer L[kPairGroupMaxLayers];
    int nlayers;
    int total;            // tiles of all the layers
};

__device__ __forceinline__ int pair_group_layer(const PairGroupParams &p, int t, int hint)
{
    int l = hint;
    while (l + 1 < p.nlayers && p.L[l + 1].tile0 <= t)
        ++l;
    return l;
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, 1) gemm_pair_group_kernel(const __grid_constant__ PairGroupParams p)
{
    constexpr int BN = C::BN;
    constexpr int STAGES = C::STAGES;
    static_assert(C::KIND == kE4M3 && BN == 256, "FP8 operands, 256 x 256 tiles");
    constexpr uint32_t kIdesc = make_idesc(256, BN, 0, 0);

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

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->acc_full[b], 1);
            mbar_init(&ctl->acc_empty[b], 8);   // 4 epilogue warps in each CTA
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        for (int l = 0; l < p.nlayers; ++l) {
            tma_prefetch_desc(&p.tmX[l]);
            tma_prefetch_desc(&p.tmW[l]);
        }
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
    grid_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------ producers (both CTAs)
        if (lane == 0) {
            const uint64_t pol = policy_evict_last();
            int s = 0;
            uint32_t ph = 0;
            uint32_t issued_mask = 0, issued_ph = 0;
            bool ok = true;
            int l = 0;
            for (int t = pair; ok && t < p.total; t += npairs) {
                l = pair_group_layer(p, t, l);
                const PairGroupLayer &g = p.L[l];
                const int lt = t - g.tile0;
                const int row_x = (lt % g.m_tiles) * 256 + static_cast<int>(rank) * 128;
                const int row_w = (lt / g.m_tiles) * BN + static_cast<int>(rank) * (BN / 2);
                for (int kb = 0; kb < g.kblocks; ++kb) {
                    if (!wait_bounded_cluster(&ctl->empty[s], ph ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = smem + s * C::kStage;
                    if (lead)
                        mbar_arrive_expect_tx(&ctl->full[s], 2 * C::kStage);
                    tma_load_2d_pair(st, &p.tmX[l], &ctl->full[s], kb * 128, row_x, pol);
                    tma_load_2d_pair(st + C::kTileA, &p.tmW[l], &ctl->full[s], kb * 128, row_w, pol);
                    issued_mask |= 1u << s;
                    issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (*abort_flag && lead) {
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
            int i = 0, l = 0;
            for (int t = pair; ok && t < p.total; t += npairs, ++i) {
                l = pair_group_layer(p, t, l);
                const int kblocks = p.L[l].kblocks;
                const int buf = i & 1;
                const uint32_t use = static_cast<uint32_t>(i >> 1);
                if (!wait_bounded_cluster(&ctl->acc_empty[buf], (use & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + static_cast<uint32_t>(buf * BN);
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!wait_bounded(&ctl->full[s], ph, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * C::kStage);
                    const uint32_t b_addr = a_addr + C::kTileA;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        umma_f8f6f4_pair(d, sdesc_sw128(a_addr + k * 32), sdesc_sw128(b_addr + k * 32), kIdesc,
                                         (kb > 0 || k > 0) ? 1u : 0u);
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
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16);
        int i = 0, l = 0;
        for (int t = pair; t < p.total; t += npairs, ++i) {
            l = pair_group_layer(p, t, l);
            const PairGroupLayer &g = p.L[l];
            const int buf = i & 1;
            const uint32_t use = static_cast<uint32_t>(i >> 1);
            bool ok = wait_bounded_cluster(&ctl->acc_full[buf], use & 1u, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok)
                break;
            tc_fence_after();
            const int lt = t - g.tile0;
            const int m = (lt % g.m_tiles) * 256 + static_cast<int>(rank) * 128 + r;
            const int n_base = (lt / g.m_tiles) * BN;
            const float sam = m < g.M ? g.sa[m] : 0.0f;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 16) {
                const int n0 = n_base + c0;
                if (n0 >= g.N)
                    break;                      // warp-uniform; N % 16 == 0
                uint32_t v[16];
                tmem_ld_32x32b_x16(t_row + static_cast<uint32_t>(buf * BN + c0), v);
                tmem_ld_wait();
                if (m < g.M) {
                    uint32_t o[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        o[j] = pack2<kE4M3>(__uint_as_float(v[2 * j]) * sam * __ldg(g.sw + n0 + 2 * j),
                                            __uint_as_float(v[2 * j + 1]) * sam * __ldg(g.sw + n0 + 2 * j + 1));
                    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(g.y) + static_cast<int64_t>(m) * g.N +
                                                           n0);
                    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
                    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (lead)
                    mbar_arrive(&ctl->acc_empty[buf]);
                else
                    mbar_arrive_remote(&ctl->acc_empty[buf], 0u);
            }
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
