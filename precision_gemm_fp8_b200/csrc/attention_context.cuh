// Context (prefill) attention over the FP8 (E4M3) paged KV cache on the
// 5th-generation tensor cores.
//
// "C++ and FP8" §3.3: the context attention runs in the FP8 dataflow; §3.2:
// the K / V cache is paged in blocks of 16 tokens kept in FP8.  This
// library's reading: the queries of a sequence are its last q_len positions
// ctx - q_len .. ctx - 1 (a prompt, or a prompt continued after a cached
// prefix), query i sees positions 0 .. ctx - q_len + i (causal), grouped
// query heads.  Both products are E4M3 x E4M3 -> f32 on the tensor cores:
//   S = Q_codes . K_codes^T              (Q quantised per (token, head) row
//                                         beforehand by the row quantiser)
//   P = E4M3(2^8 . exp2(S . sq . sk . log2(e)/sqrt(D) - m))   (online softmax)
//   O = P . V_codes . sv / l
// l sums the unrounded probabilities times 2^8 (the code scale cancels in
// O; scaling by a power of two leaves the sum's rounding unchanged).
// head_dim 128.
//
// One CTA per (128-query tile, query head, sequence), heaviest tiles first, 320 threads:
//   warp 0      TMA: the Q tile once, then per 128-key tile eight 16-row
//               pieces of K and of V straight from the paged cache (a piece
//               past the context, or of an out-of-range block, is read at a
//               row past the cache's end and arrives as zeros);
//   warp 1      TMEM (512 columns: S double buffer, PV double buffer) and
//               the MMA issue: S_j = Q K_j^T, then PV_{j-1} = P_{j-1} V_{j-1}
//               (V as an MN-major operand: the cache rows are d-contiguous);
//   warps 2-9   two threads per query row (kCtxParts): warp w takes keys
//               (and head-dim columns) 64 * ((w - 2) / 4) .. + 63 of TMEM
//               lane quadrant w % 4: scores from TMEM (two passes), causal
//               and validity masks (skipped for key tiles wholly below the
//               query tile with every piece present), online softmax in
//               base 2 (the parts' maxima exchanged through shared memory at
//               a named barrier), P codes written into shared memory in the
//               128-byte-swizzled K-major layout, PV_{j-1} added into
//               registers one tile late (so the PV MMA overlaps the next
//               softmax), final 1/l and scales.  Every barrier of these
//               warps also ANDs their wait results, so they leave the loop
//               together when one of them gives up.  (Four threads per row
//               measured slower on B200: 61 M against 42 M instructions for
//               the 7B 2048-token prompt, 124 against 117 us.)
// Every wait is bounded: a wait that gives up raises the CTA's abort flag
// and the device error word; in-flight copies and MMAs are drained before
// the CTA frees its TMEM and exits.
#pragma once

#include "attention.cuh"
#include "gemm.cuh"

namespace pgf8 {

constexpr int kCtxStages = 3;                   // K / V ring depth (128 keys per stage)
constexpr int kCtxTile = 16384;                  // 128 rows x 128 bytes
constexpr int kCtxQ = 0;
constexpr int kCtxK = kCtxQ + kCtxTile;
constexpr int kCtxV = kCtxK + kCtxStages * kCtxTile;
constexpr int kCtxP = kCtxV + kCtxStages * kCtxTile;
constexpr int kCtxCtl = kCtxP + 2 * kCtxTile;
constexpr int kCtxParts = 2;                     // softmax threads per query row (64 columns each)
constexpr int kCtxCols = 128 / kCtxParts;
constexpr int kCtxRed = kCtxCtl + 1024;         // [2 parities][parts][128 rows] f32: row-max exchange
constexpr int kCtxSmemBytes = kCtxRed + 2 * kCtxParts * 128 * 4 + 1024 /*alignment slack*/;
constexpr int kCtxSoftmaxThreads = 128 * kCtxParts;
constexpr int kCtxThreads = 64 + kCtxSoftmaxThreads;   // producer, MMA, softmax warps
constexpr uint32_t kCtxTmemCols = 512;
static_assert(kCtxSmemBytes <= 227 * 1024, "shared memory");

struct AttnCtxCtl {
    uint64_t q_full;
    uint64_t kv_full[kCtxStages];
    uint64_t kv_empty[kCtxStages];
    uint64_t s_full[2], s_free[2];   // S buffer b: MMA -> softmax, softmax -> MMA
    uint64_t p_full[2];              // P buffer b written (softmax -> MMA)
    uint64_t o_full[2], o_free[2];   // PV buffer b: MMA -> softmax, softmax -> MMA
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(AttnCtxCtl) <= 1024, "control block");

struct AttnCtxParams {
    const float *q_scales;       // [total_q * Hq]: row (token, head) = token * Hq + head
    const int32_t *q_start;      // [seqs + 1] first query token of each sequence
    const int32_t *ctx_lens;     // [seqs]
    const int32_t *tables;       // [seqs][table_stride]
    int64_t table_stride;
    const float *sk, *sv;        // [Hkv]
    int Hq, Hkv, B;
    int64_t num_blocks;
    int cache_rows;              // num_blocks * Hkv * B: a row coordinate past the cache (zeros)
    int max_ctx;
    int total_q;                 // query tokens in the batch: q_start must stay within it
    void *out;                   // [total_q][Hq][128], token stride ldo elements
    int64_t ldo;
    int odt;
    int vec_out;                 // out and its token stride allow 16-byte stores
    int32_t *errors;
};

// N values of one query row of the output (scaled by f) into out[base ..]:
// 16-byte stores when allowed, else element by element.
template <int N>
__device__ __forceinline__ void store_row(void *out, int64_t base, int odt, bool vec, const float (&o)[N], float f)
{
    if (!vec) {
#pragma unroll
        for (int d = 0; d < N; ++d)
            store_elem(out, base + d, odt, o[d] * f);
        return;
    }
    if (odt == 0) {
        float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(out) + base);
#pragma unroll
        for (int i = 0; i < N / 4; ++i)
            dst[i] = make_float4(o[4 * i] * f, o[4 * i + 1] * f, o[4 * i + 2] * f, o[4 * i + 3] * f);
        return;
    }
    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(out) + base);
#pragma unroll
    for (int i = 0; i < N / 8; ++i) {
        uint32_t w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float lo = o[8 * i + 2 * u] * f, hi = o[8 * i + 2 * u + 1] * f;
            if (odt == 1) {
                const __half2 hv = __floats2half2_rn(lo, hi);
                w[u] = *reinterpret_cast<const uint32_t *>(&hv);
            } else {
                const __nv_bfloat162 bv = __floats2bfloat162_rn(lo, hi);
                w[u] = *reinterpret_cast<const uint32_t *>(&bv);
            }
        }
        dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// Shared-memory descriptor of an MN-major operand tile in the 128-byte
// swizzled canonical layout: rows of 128 bytes along MN (one swizzle atom
// wide: MN = 128 for 8-bit types), K rows at 128 bytes, 8-row groups at
// 1024 bytes (stride byte offset).  The leading byte offset (distance
// between 128-element MN atoms) is not applied with a single atom; it is
// set to the same 1024 bytes, so that no reading of the two fields can
// address past the tile.
__device__ __forceinline__ uint64_t sdesc_sw128_mn(uint32_t saddr)
{
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
    d |= static_cast<uint64_t>(1024 >> 4) << 16;
    d |= static_cast<uint64_t>(1024 >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

// Cache row of the 16-position piece starting at `key` for KV head hk, or
// cache_rows (a zero piece) when the piece lies past the context or its
// block-table entry is out of range.
__device__ __forceinline__ int ctx_piece_row(const AttnCtxParams &p, int64_t s, int hk, int key, int ctx)
{
    if (key >= ctx)
        return p.cache_rows;
    const int64_t blk = p.tables[s * p.table_stride + key / p.B];
    if (blk < 0 || blk >= p.num_blocks)
        return p.cache_rows;
    return static_cast<int>((blk * p.Hkv + hk) * p.B + key % p.B);
}

// 2^x by the special-function unit (ex2.approx.ftz: a relative error of a
// few binary32 ulps, far below the E4M3 rounding of the probabilities that
// follows; -inf -> 0).
__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// AND of v over the softmax warps (named barrier 1): also the barrier at
// which they exchange row maxima through shared memory.
__device__ __forceinline__ bool ctx_softmax_all(bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(v)), "n"(kCtxSoftmaxThreads)
        : "memory");
    return r != 0;
}

__global__ void __launch_bounds__(kCtxThreads, 1) attn_context_kernel(const __grid_constant__ CUtensorMap tmQ,
                                                              const __grid_constant__ CUtensorMap tmK,
                                                              const __grid_constant__ CUtensorMap tmV,
                                                              const AttnCtxParams p)
{
    constexpr uint32_t kIdescS = make_idesc(128, 128, 0, 0);                  // Q (K-major) x K (K-major)
    constexpr uint32_t kIdescPV = make_idesc(128, 128, 0, 0) | (1u << 16);    // P (K-major) x V (MN-major)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // grid.x = query tiles x heads, heaviest (last) tiles of every head
    // first: causal tiles differ in length, and the short ones fill in last
    const int nqt = static_cast<int>(gridDim.x) / p.Hq;
    const int h = static_cast<int>(blockIdx.x) % p.Hq;
    const int qt = nqt - 1 - static_cast<int>(blockIdx.x) / p.Hq;
    const int64_t s = blockIdx.z;
    const int hk = h / (p.Hq / p.Hkv);
    const int q0 = p.q_start[s];
    const int q_len = p.q_start[s + 1] - q0;
    const int ctx = p.ctx_lens[s];
    if (q_len < 0 || q0 < 0 || q0 + q_len > p.total_q || ctx < q_len || ctx > p.max_ctx) {
        if (threadIdx.x == 0 && qt == 0 && h == 0 && p.errors)
            atomicAdd(p.errors, 1);
        return;                                          // an invalid sequence is not written
    }
    if (q_len <= qt * 128)
        return;                                          // CTA-uniform: no tile here
    if (qt == 0 && h == 0 && threadIdx.x == 0 && p.errors && q_len > nqt * 128)
        atomicAdd(p.errors, 1);                          // longer than the grid covers: the tail is not written
    const int nrows = q_len - qt * 128 < 128 ? q_len - qt * 128 : 128;
    const int pos0 = ctx - q_len + qt * 128;            // position of the tile's first query
    const int nkt = (pos0 + nrows - 1) / 128 + 1;        // key tiles 0 .. nkt - 1

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    AttnCtxCtl *ctl = reinterpret_cast<AttnCtxCtl *>(smem + kCtxCtl);
    volatile int *abort_flag = &ctl->abort;

    if (threadIdx.x == 0) {
        mbar_init(&ctl->q_full, 1);
        for (int i = 0; i < kCtxStages; ++i) {
            mbar_init(&ctl->kv_full[i], 1);
            mbar_init(&ctl->kv_empty[i], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->s_full[b], 1);
            mbar_init(&ctl->s_free[b], kCtxSoftmaxThreads / 32);   // one arrival per softmax warp
            mbar_init(&ctl->p_full[b], kCtxSoftmaxThreads / 32);
            mbar_init(&ctl->o_full[b], 1);
            mbar_init(&ctl->o_free[b], kCtxSoftmaxThreads / 32);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, kCtxTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            uint32_t issued_mask = 0, issued_ph = 0;   // per stage: loaded at least once / parity of last load
            mbar_arrive_expect_tx(&ctl->q_full, kCtxTile);
            tma_load_2d(smem + kCtxQ, &tmQ, &ctl->q_full, h * 128, q0 + qt * 128);
            for (int j = 0; j < nkt; ++j) {
                const int st = j % kCtxStages;
                const uint32_t ph = static_cast<uint32_t>(j / kCtxStages) & 1u;
                if (!wait_bounded(&ctl->kv_empty[st], ph ^ 1u, abort_flag))
                    break;
                mbar_arrive_expect_tx(&ctl->kv_full[st], 2 * kCtxTile);
                for (int i = 0; i < 8; ++i) {
                    const int row = ctx_piece_row(p, s, hk, j * 128 + i * 16, ctx);
                    tma_load_2d(smem + kCtxK + st * kCtxTile + i * 2048, &tmK, &ctl->kv_full[st], 0, row);
                    tma_load_2d(smem + kCtxV + st * kCtxTile + i * 2048, &tmV, &ctl->kv_full[st], 0, row);
                }
                issued_mask |= 1u << st;
                issued_ph = (issued_ph & ~(1u << st)) | (ph << st);
            }
            if (*abort_flag) {
                wait_drain(&ctl->q_full, 0);
                for (int i = 0; i < kCtxStages; ++i)
                    if (issued_mask & (1u << i))
                        wait_drain(&ctl->kv_full[i], (issued_ph >> i) & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            bool ok = wait_bounded(&ctl->q_full, 0, abort_flag);
            const uint32_t q_addr = smem_u32(smem + kCtxQ);
            auto issue_pv = [&](int i) -> bool {
                const int b = i & 1, k = i >> 1, st = i % kCtxStages;
                if (!wait_bounded(&ctl->p_full[b], static_cast<uint32_t>(k) & 1u, abort_flag))
                    return false;
                if (k >= 1 && !wait_bounded(&ctl->o_free[b], static_cast<uint32_t>(k - 1) & 1u, abort_flag))
                    return false;
                tc_fence_after();
                const uint32_t p_addr = smem_u32(smem + kCtxP + b * kCtxTile);
                const uint32_t v_addr = smem_u32(smem + kCtxV + st * kCtxTile);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)   // 4 x 32 keys
                    umma_f8f6f4(tmem + 256 + b * 128, sdesc_sw128(p_addr + kk * 32),
                                sdesc_sw128_mn(v_addr + kk * 32 * 128), kIdescPV, kk > 0 ? 1u : 0u);
                umma_commit(&ctl->o_full[b]);
                umma_commit(&ctl->kv_empty[st]);
                return true;
            };
            for (int j = 0; ok && j < nkt; ++j) {
                const int st = j % kCtxStages, b = j & 1, k = j >> 1;
                if (!wait_bounded(&ctl->kv_full[st], static_cast<uint32_t>(j / kCtxStages) & 1u, abort_flag) ||
                    (k >= 1 && !wait_bounded(&ctl->s_free[b], static_cast<uint32_t>(k - 1) & 1u, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t k_addr = smem_u32(smem + kCtxK + st * kCtxTile);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)   // 4 x 32 bytes of head_dim
                    umma_f8f6f4(tmem + b * 128, sdesc_sw128(q_addr + kk * 32), sdesc_sw128(k_addr + kk * 32),
                                kIdescS, kk > 0 ? 1u : 0u);
                umma_commit(&ctl->s_full[b]);
                if (j >= 1 && !issue_pv(j - 1))
                    ok = false;
            }
            if (ok)
                ok = issue_pv(nkt - 1);
            if (!ok) {
                umma_commit(&ctl->drain);
                wait_drain(&ctl->drain, 0);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax (two threads per query row)
        const int qd = warp & 3;                          // TMEM lane quadrant of this warp
        const int part = (warp - 2) >> 2;                 // columns part * kCtxCols .. + kCtxCols - 1
        const int r = qd * 32 + lane;                     // query row of the tile
        const int et = static_cast<int>(threadIdx.x) - 64;   // 0 .. kCtxSoftmaxThreads - 1
        const int c_lo = part * kCtxCols;
        const bool row_ok = r < nrows;
        const int pos = pos0 + r;
        const uint32_t t_lane = tmem + (static_cast<uint32_t>(qd * 32) << 16);
        float *red = reinterpret_cast<float *>(smem + kCtxRed);   // [parity][part][row]
        const float scale = row_ok ? p.q_scales[(static_cast<int64_t>(q0) + qt * 128 + r) * p.Hq + h] * p.sk[hk] *
                                         (1.4426950408889634f * 0.08838834764831845f)   // log2(e) / sqrt(128)
                                   : 0.0f;
        float m = -INFINITY, l = 0.0f, alpha_prev = 0.0f;   // l: this part's share of the row sum
        float o[kCtxCols];                                   // head-dim columns c_lo .. c_lo + kCtxCols - 1
#pragma unroll
        for (int d = 0; d < kCtxCols; ++d)
            o[d] = 0.0f;
        bool ok = true;

        // O += PV_i (relative to the maximum after tile i), rescaling by alpha
        auto accumulate = [&](int i, float alpha) -> bool {
            const int b = i & 1, k = i >> 1;
            const bool w = ctx_softmax_all(wait_bounded(&ctl->o_full[b], static_cast<uint32_t>(k) & 1u, abort_flag));
            if (!w)
                return false;
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < kCtxCols; c0 += 16) {
                uint32_t v[16];
                tmem_ld_32x32b_x16(t_lane + 256 + b * 128 + c_lo + c0, v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    o[c0 + e] = fmaf(o[c0 + e], alpha, __uint_as_float(v[e]));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&ctl->o_free[b]);
            return true;
        };

        for (int j = 0; j < nkt; ++j) {
            const int b = j & 1, k = j >> 1, st = j % kCtxStages;
            // validity of the tile's eight 16-key pieces (block-table entries)
            uint32_t piece_ok = 0;
            for (int i = 0; i < 8; ++i) {
                const int key = j * 128 + i * 16;
                if (key >= ctx)
                    continue;
                const int64_t blk = p.tables[s * p.table_stride + key / p.B];
                if (blk >= 0 && blk < p.num_blocks)
                    piece_ok |= 1u << i;
                else if (et == 0 && h == 0 && qt == (q_len - 1) / 128 && p.errors)
                    atomicAdd(p.errors, 1);   // once: the sequence's last query tile visits every key tile
            }
            const bool w = wait_bounded(&ctl->s_full[b], static_cast<uint32_t>(k) & 1u, abort_flag);
            const uint32_t t_s = t_lane + b * 128 + c_lo;
            // Key tiles wholly below the tile's first query and with all eight
            // pieces present need no mask (CTA-uniform).  Rows past the
            // prompt (row_ok false) are then computed unmasked as well: their
            // P and O rows are never stored, and nothing mixes rows.
            const bool unmasked = piece_ok == 0xFFu && j * 128 + 127 <= pos0;
            // pass 1: the maximum of this part's valid scores, exchanged with the other parts'
            float mx = -INFINITY;
            if (w) {
                tc_fence_after();
                if (unmasked) {
                    float vmax = -INFINITY;
#pragma unroll 1
                    for (int c0 = 0; c0 < kCtxCols; c0 += 16) {
                        uint32_t v[16];
                        tmem_ld_32x32b_x16(t_s + c0, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            vmax = fmaxf(vmax, __uint_as_float(v[e]));
                    }
                    mx = vmax * scale;   // scale >= 0: rounding is monotone, the maximum commutes
                } else {
#pragma unroll 1
                    for (int c0 = 0; c0 < kCtxCols; c0 += 16) {
                        uint32_t v[16];
                        tmem_ld_32x32b_x16(t_s + c0, v);
                        tmem_ld_wait();
                        const bool pok = (piece_ok >> ((c_lo + c0) >> 4)) & 1u;
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int key = j * 128 + c_lo + c0 + e;
                            const float sc = __uint_as_float(v[e]) * scale;
                            mx = (pok && row_ok && key <= pos) ? fmaxf(mx, sc) : mx;
                        }
                    }
                }
            }
            float *red_j = red + (j & 1) * (kCtxParts * 128);
            red_j[part * 128 + r] = mx;
            if (!ctx_softmax_all(w)) {
                ok = false;
                break;
            }
#pragma unroll
            for (int q = 0; q < kCtxParts; ++q)
                mx = fmaxf(mx, red_j[q * 128 + r]);
            const float mn = fmaxf(m, mx);
            const float alpha = m == -INFINITY ? 0.0f : ex2_approx(m - mn);
            // pass 2: the probabilities times 2^8 (the E4M3 code scale, folded
            // into the exponent), their codes into P buffer b, this part's
            // row sum (in the same units)
            const float nm8 = 8.0f - mn;
            float rs = 0.0f;
            uint8_t *prow = smem + kCtxP + b * kCtxTile + r * 128;
#pragma unroll 1
            for (int c0 = 0; c0 < kCtxCols; c0 += 16) {
                uint32_t v[16];
                tmem_ld_32x32b_x16(t_s + c0, v);
                tmem_ld_wait();
                const int cc = c_lo + c0;
                float pr[16];
                if (unmasked) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        pr[e] = ex2_approx(fmaf(__uint_as_float(v[e]), scale, nm8));
                        rs += pr[e];
                    }
                } else {
                    const bool pok = (piece_ok >> (cc >> 4)) & 1u;
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int key = j * 128 + cc + e;
                        const bool valid = pok && row_ok && key <= pos;
                        pr[e] = valid ? ex2_approx(fmaf(__uint_as_float(v[e]), scale, nm8)) : 0.0f;
                        rs += pr[e];
                    }
                }
                uint32_t wv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    wv[u] = static_cast<uint32_t>(cvt_e4m3x2(pr[4 * u], pr[4 * u + 1])) |
                            (static_cast<uint32_t>(cvt_e4m3x2(pr[4 * u + 2], pr[4 * u + 3])) << 16);
                *reinterpret_cast<uint4 *>(prow + (((cc >> 4) ^ (r & 7)) << 4)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&ctl->s_free[b]);
            // V rows past the context inside the piece that holds position ctx
            // come from the cache as they are: clear them, since a zero
            // probability times a NaN code would still be NaN
            const int cut = ctx - j * 128;
            if (cut > 0 && cut < 128 && (cut & 15) != 0 && ((piece_ok >> (cut >> 4)) & 1u)) {
                const bool wk = ctx_softmax_all(
                    wait_bounded(&ctl->kv_full[st], static_cast<uint32_t>(j / kCtxStages) & 1u, abort_flag));
                if (!wk) {
                    ok = false;
                    break;
                }
                const int row = cut + (et >> 3);          // 16 rows x 8 chunks cover the rest of the piece
                if (et < 128 && row < ((cut >> 4) + 1) * 16)
                    *reinterpret_cast<uint4 *>(smem + kCtxV + st * kCtxTile + row * 128 + (et & 7) * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();   // P codes (and cleared V rows) before the MMA reads them
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&ctl->p_full[b]);
            m = mn;
            l = fmaf(l, alpha, rs);
            if (j >= 1 && !accumulate(j - 1, alpha_prev)) {
                ok = false;
                break;
            }
            alpha_prev = alpha;
        }
        if (ok)
            ok = accumulate(nkt - 1, alpha_prev);
        if (ok) {
            // the row sum: both halves add the two shares in the same order
            float *red_l = red + (nkt & 1) * (kCtxParts * 128);
            red_l[part * 128 + r] = l;
            ctx_softmax_all(true);
            float lsum = 0.0f;
#pragma unroll
            for (int q = 0; q < kCtxParts; ++q)   // the same order in every part
                lsum += red_l[q * 128 + r];
            if (row_ok) {
                const float f = lsum > 0.0f ? p.sv[hk] / lsum : 0.0f;   // P and l both carry the 2^8
                const int64_t base =
                    (static_cast<int64_t>(q0) + qt * 128 + r) * p.ldo + static_cast<int64_t>(h) * 128 + c_lo;
                store_row<kCtxCols>(p.out, base, p.odt, p.vec_out != 0, o, f);
            }
        }
    }

    // -------------------------------------------------------------------- teardown
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kCtxTmemCols);
    }
}

} // namespace pgf8
