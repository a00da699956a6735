/*
 * pgf8 — FP8 (E4M3) quantised linear layer and NestedFP dual-precision
 * linear layer for NVIDIA B200 (sm_100a).  C ABI.
 *
 * The layer computed here is the one the "precision_gemm_fp8" pages
 * describe:
 *   - "7B on an RTX 4060 with FP8" (intelliparadigm.com 2151670), §2.1:
 *     weights and activations in FP8 E4M3; §2.2: weights use static
 *     (offline-calibrated) scales, activations dynamic scales from a
 *     runtime amax; §6.1: scaled values must stay within 448.
 *   - "C++ and FP8 quantization for LLM inference" (tqpw.cn 201730), §3.3:
 *     an E4M3 x E4M3 GEMM with FP32 accumulation and BF16 output whose
 *     operands are both K-contiguous ("TN"); §4.2: per-channel weight and
 *     per-token activation granularity.
 *   - "NestedFP dual-precision inference framework" (intelliparadigm.com
 *     2229392), §2.1: one FP16 weight tensor stored as an upper-byte plane
 *     and a lower-byte plane; FP16 mode rebuilds (upper << 8) | lower, FP8
 *     mode feeds the upper byte alone to the compute units; §2.2: the
 *     rebuild is fused into the GEMM's shared-memory stage.
 *
 * Conventions for every entry point
 *   Memory      All pointers are DEVICE pointers owned by the caller.  The
 *               library never allocates or frees device memory; the size of
 *               any workspace is returned by the matching *_workspace_size().
 *   Workspace   A workspace must be zero-filled once, before its first use
 *               (e.g. cudaMemset); every call that completes leaves the words
 *               it synchronises on zero again, so it can be reused without
 *               clearing.  After PGF8_ERR_TIMEOUT, zero it again.  One
 *               workspace serves one call at a time (calls on different
 *               streams need different workspaces).  For M <= 32 the
 *               stream-K kernel (PGF8_PATH_STREAMK, chosen only on request)
 *               keeps its flags and partial tiles there; the kernels chosen
 *               by PGF8_PATH_AUTO need none beyond the dynamic entry points'
 *               activation codes and scales.
 *   Layout      Row-major, last index contiguous: activations x/aq [M, K],
 *               weights w/wq/hi/lo [N, K] (K contiguous, "TN"), outputs
 *               y [M, N].  Row strides equal the row length unless an
 *               ld* argument is given.
 *   Alignment   Every base pointer 16-byte aligned; K % 16 == 0 and
 *               N % 16 == 0 (the tensor-memory-access unit moves 16-byte
 *               granules); row strides in bytes a multiple of 16.
 *   Execution   Asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *               default stream) on the current device.  A return of
 *               PGF8_OK means the work was enqueued.
 *   Errors      Argument errors are reported before anything is enqueued
 *               (INVALID_ARG, ALIGNMENT, UNSUPPORTED).  A failed launch
 *               returns PGF8_ERR_CUDA (details: pgf8_last_cuda_error).  Every
 *               device-side wait is bounded; a kernel that gives up raises a
 *               device error word, reported by pgf8_device_status() as
 *               PGF8_ERR_TIMEOUT.  No C++ exception crosses this boundary.
 *   Determinism Results are bit-identical from run to run for the same
 *               inputs, shapes and options: split-K partial sums are added
 *               in a fixed order, never with floating-point atomics.
 */
#ifndef PGF8_H
#define PGF8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PGF8_OK = 0,
    PGF8_ERR_INVALID_ARG = 1,
    PGF8_ERR_ALIGNMENT = 2,
    PGF8_ERR_UNSUPPORTED = 3,
    PGF8_ERR_CUDA = 4,
    PGF8_ERR_TIMEOUT = 5,
    PGF8_ERR_TOO_LARGE = 6
} pgf8_status;

typedef enum { PGF8_F32 = 0, PGF8_F16 = 1, PGF8_BF16 = 2 } pgf8_dtype;

typedef enum { PGF8_SCALE_DYNAMIC = 0, PGF8_SCALE_STATIC = 1 } pgf8_scale_mode;

typedef enum { PGF8_NESTED_FP16 = 0, PGF8_NESTED_FP8 = 1 } pgf8_nested_mode;

/* Kernel family used by the linear entry points. */
typedef enum {
    PGF8_PATH_AUTO = 0,    /* chosen from M, N, K */
    PGF8_PATH_SKINNY = 1,  /* weight-streaming: weights are the 128-row MMA operand,
                              tokens the narrow one (M <= 128) */
    PGF8_PATH_TILED = 2,   /* tokens are the 128-row MMA operand (any M) */
    PGF8_PATH_STREAMK = 3, /* skinny, stream-K over one CTA per SM (M <= 32; needs the
                              workspace) */
    PGF8_PATH_TILED_PAIR = 4 /* tiled on SM pairs (cta_group::2), 256 x 256 tiles (FP8
                              kinds: tile_n 128 / 192 / 256; NestedFP FP16 mode: 256) */
} pgf8_path;

/* Flags of pgf8_linear_opts.flags.
 *
 * PGF8_FLAG_OVERLAP_PREVIOUS: launch the call's first kernel with
 * programmatic stream serialization, so that it and the GEMM's first weight
 * loads may run while the previous kernel in the stream is still finishing
 * (the GEMM of the previous layer, typically).  Activations are read, and
 * outputs and workspace written, only after that kernel has completed; the
 * weights (wq/sw, or hi/lo) may be read earlier.  Set it only when no kernel
 * that can still be running writes those weights (weights that are static
 * during inference satisfy this). */
#define PGF8_FLAG_OVERLAP_PREVIOUS 1

/* PGF8_FLAG_FUSED_QUANT (dynamic entry points only): quantise the
 * activations inside the GEMM instead of running the per-token quantisation
 * as its own kernel first.  Applies where a dynamic call has M <= 32 on the
 * skinny path (path AUTO or SKINNY, tile_n 0, 16 or 32) and each CTA's
 * activation slice (M rows of its K-split) fits its registers (at most 8192
 * f32 or 16384 f16 elements); elsewhere the flag changes nothing.  One
 * kernel instead of two, with the same codes, scales and outputs, bit for
 * bit.  Not the default: on B200 the two-kernel form measured faster in
 * chained decode steps (its quantisation kernel hides the GEMM's weight
 * prefetch behind the previous layer). */
#define PGF8_FLAG_FUSED_QUANT 2

/* PGF8_FLAG_ATTN_MMA (pgf8_fp8_attention_decode_paged only): run both
 * products on the tensor cores (mma.sync, binary16 operands, binary32
 * accumulation), up to 8 query heads of one KV head per CTA.  The query and
 * the probabilities are rounded to binary16 on the way (relative 2^-11);
 * K / V codes widen exactly.  Without the flag the CUDA-core kernel keeps
 * them in binary32. */
#define PGF8_FLAG_ATTN_MMA 4

/* PGF8_FLAG_STREAM_K_TAIL (FP8 linear entry points, M > 128, pair kernel):
 * the last full round of 256 x 256 tiles and the ragged tail are split in
 * equal k-block ranges over every SM pair, partial tiles summed in a fixed
 * order through the workspace (pgf8_fp8_linear_workspace_size bytes for
 * M > 128).  Off by default: measured on B200 it is slower than whole
 * tiles on most 7B / 70B shapes (pairs working on disjoint k-ranges no
 * longer share weight tiles in L2). */
#define PGF8_FLAG_STREAM_K_TAIL 8

/* Optional tuning of the linear entry points; a NULL pointer means all
 * defaults.  Fields set to 0 mean "choose automatically". */
typedef struct {
    int32_t path;      /* pgf8_path */
    int32_t split_k;   /* K split across a thread-block cluster, 1..8 */
    int32_t tile_n;    /* narrow MMA operand rows: 16, 32, 64, 128 (skinny) or 128, 256 (tiled) */
    int32_t flags;     /* PGF8_FLAG_* */
} pgf8_linear_opts;

/* ------------------------------------------------------------------------
 * Per-row FP8 quantisation (activations per token, weights per output
 * channel).  "7B on an RTX 4060 with FP8" §2.2 and §6.1; "C++ and FP8" §4.2.
 *
 * For each row r of x ([rows, cols], element type xdt = PGF8_F32 or
 * PGF8_F16, row stride ldx elements):
 *   DYNAMIC: amax = max_k |x[r,k]|; scales[r] = fl32(amax / 448), or 1.0
 *            when that quotient is 0 (all-zero row);
 *   STATIC:  scales[r] is read (must be positive and finite);
 *   q[r,k] = E4M3 code of fl32(x[r,k] / scales[r]), rounded to nearest even,
 *            saturated to +-448, sign of zero kept.
 * q is [rows, cols] contiguous (uint8 codes, OCP E4M3 "FN" layout).
 * Results are bit-exact with respect to that definition.  Non-finite input
 * values give unspecified codes.  rows == 0 is a no-op (pointers may then
 * be NULL).
 * ---------------------------------------------------------------------- */
pgf8_status pgf8_fp8_quantize_rows(const void *x, pgf8_dtype xdt, int64_t rows, int64_t cols,
                                   int64_t ldx, uint8_t *q, float *scales,
                                   pgf8_scale_mode mode, void *stream);

/* ------------------------------------------------------------------------
 * FP8 linear with fused dequantisation ("C++ and FP8" §3.3):
 *   y[m,n] = bf16_rn( (sum_k e4m3(aq[m,k]) * e4m3(wq[n,k])) * sa[m] * sw[n] )
 * with FP32 accumulation.  aq [M,K] uint8, sa [M] f32, wq [N,K] uint8,
 * sw [N] f32, y [M,N] bf16.  M >= 1.  workspace: see the conventions above
 * (pgf8_fp8_linear_workspace_size bytes, nonzero for M <= 32; may be NULL).
 * ---------------------------------------------------------------------- */
pgf8_status pgf8_fp8_linear(const uint8_t *aq, const float *sa, int64_t M, int64_t K,
                            const uint8_t *wq, const float *sw, int64_t N, void *y_bf16,
                            void *workspace, size_t workspace_bytes, void *stream);

pgf8_status pgf8_fp8_linear_ex(const uint8_t *aq, const float *sa, int64_t M, int64_t K,
                               const uint8_t *wq, const float *sw, int64_t N, void *y_bf16,
                               void *workspace, size_t workspace_bytes,
                               const pgf8_linear_opts *opts, void *stream);

size_t pgf8_fp8_linear_workspace_size(int64_t M, int64_t N, int64_t K);

/* ------------------------------------------------------------------------
 * FP8 paged KV cache ("7B on an RTX 4060 with FP8": K/V stored in FP8;
 * "C++ and FP8" §3.2: a paged cache of token blocks kept in FP8).
 *
 * pgf8_fp8_kv_write_paged: writes `tokens` K (or V) rows of
 *   kv [tokens, heads, head_dim] (f32, f16 or bf16; token stride ldkv
 *   elements, so a slice of the QKV projection's output can be passed as
 *   it is) at positions first_pos .. first_pos + tokens - 1 into
 *   cache [num_blocks, heads, block_size, head_dim] (E4M3 codes): position
 *   p goes to block block_table[p / block_size], slot p % block_size.
 *   Codes E4M3(RN(x / scales[h])), saturating (scales [heads] f32, one per
 *   KV head, > 0).  The block table (device int32 [table_len]) must cover
 *   the positions (else PGF8_ERR_INVALID_ARG before any launch); entries
 *   outside [0, num_blocks) are skipped and counted per token into
 *   *bad_blocks (device int32, may be NULL): nothing is written outside the
 *   cache.  head_dim % 16 == 0; kv, cache 16-byte aligned.  flags:
 *   PGF8_FLAG_OVERLAP_PREVIOUS as for the quantisation calls.
 * ---------------------------------------------------------------------- */
pgf8_status pgf8_fp8_kv_write_paged(const void *kv, pgf8_dtype dt, int64_t tokens, int64_t heads, int64_t head_dim,
                                    int64_t ldkv, const float *scales, int64_t first_pos, int64_t block_size,
                                    const int32_t *block_table, int64_t table_len, int64_t num_blocks,
                                    uint8_t *cache, int32_t *bad_blocks, int32_t flags, void *stream);

/* ------------------------------------------------------------------------
 * Decode attention over the FP8 paged KV cache ("7B on an RTX 4060 with
 * FP8": K/V held in FP8 and dequantised on use; "C++ and FP8" §3.2 paged
 * cache of 16-token blocks, §3.3 attention in the FP8 dataflow).
 *
 * One query row per sequence: the token being generated, at position
 * ctx - 1, which sees cached positions 0 .. ctx - 1 (ctx = context_lens[s]).
 * For query head h over KV head hk = h / (q_heads / kv_heads):
 *   score_t = (q[s,h,:] . dec(K_t)) * k_scales[hk] / sqrt(head_dim)
 *   out[s,h,:] = (sum_t softmax(score)_t * dec(V_t)) * v_scales[hk]
 * with dec the E4M3 value of a code and K_t / V_t the cache rows of
 * position t: block block_tables[s * table_stride + t / block_size], slot
 * t % block_size.  Computed in binary32 (q widened, scores and softmax in
 * binary32 with exp2f, outputs rounded once to out_dt); ctx == 0 gives 0.
 *
 * q:    [seqs, q_heads, head_dim], f32 / f16 / bf16, sequence stride ldq
 *       elements (a slice of the QKV projection output can be passed).
 * cache: the K and V caches [num_blocks, kv_heads, block_size, head_dim]
 *       (as written by pgf8_fp8_kv_write_paged), their per-head scales.
 *       head_dim 64, 128 or 256; block_size a multiple of 16; q_heads a
 *       multiple of kv_heads.
 * block_tables: device int32 [seqs, table_stride]; context_lens: device
 *       int32 [seqs].  max_context (host) bounds every context length and
 *       must fit the table (max_context <= table_stride * block_size); a
 *       longer (or negative) length is clamped to it and counted.
 * out:  [seqs, q_heads, head_dim], out_dt, sequence stride ldo elements.
 * splits: 0 chooses the number of context chunks from the grid
 *       (pgf8_fp8_attention_decode_plan reports it); > 0 caps it.  With more
 *       than one chunk a second kernel merges the chunks in chunk order,
 *       through `workspace` (pgf8_fp8_attention_decode_workspace_size bytes
 *       for the same arguments, 4-byte aligned; may be NULL when that is 0).
 * errors: device int32 or NULL.  Block-table entries outside
 *       [0, num_blocks) are counted (once per 16 positions) and those
 *       positions left out; clamped context lengths are counted once per
 *       sequence.  Nothing outside the cache is read.
 * Alignment: caches 16 bytes; q and out their element size; scales, tables,
 * lengths and errors 4 bytes.  flags: PGF8_FLAG_OVERLAP_PREVIOUS,
 * PGF8_FLAG_ATTN_MMA.  seqs == 0 is a no-op.  Results do not depend on
 * scheduling.
 * ---------------------------------------------------------------------- */
typedef struct {
    const uint8_t *k_cache;   /* [num_blocks, kv_heads, block_size, head_dim] E4M3 codes */
    const uint8_t *v_cache;   /* same shape */
    const float *k_scales;    /* [kv_heads] */
    const float *v_scales;    /* [kv_heads] */
    int64_t num_blocks;
    int64_t kv_heads;
    int64_t block_size;
    int64_t head_dim;
} pgf8_paged_kv_cache;

pgf8_status pgf8_fp8_attention_decode_plan(int64_t seqs, int64_t q_heads, int64_t kv_heads, int64_t head_dim,
                                           int64_t max_context, int64_t splits, int64_t *nsplit, int64_t *chunk);

size_t pgf8_fp8_attention_decode_workspace_size(int64_t seqs, int64_t q_heads, int64_t kv_heads, int64_t head_dim,
                                                int64_t max_context, int64_t splits);

pgf8_status pgf8_fp8_attention_decode_paged(const void *q, pgf8_dtype q_dt, int64_t seqs, int64_t q_heads,
                                            int64_t ldq, const pgf8_paged_kv_cache *cache,
                                            const int32_t *block_tables, int64_t table_stride,
                                            const int32_t *context_lens, int64_t max_context, void *out,
                                            pgf8_dtype out_dt, int64_t ldo, int64_t splits, void *workspace,
                                            size_t workspace_bytes, int32_t *errors, int32_t flags, void *stream);

/* ------------------------------------------------------------------------
 * Context (prefill) attention over the FP8 paged KV cache on the tensor
 * cores ("C++ and FP8" §3.3: context attention in the FP8 dataflow; §3.2:
 * paged FP8 cache).  The queries of sequence s are the q_len(s) =
 * q_start[s+1] - q_start[s] tokens q_start[s] .. q_start[s+1] - 1 of the
 * packed query batch, at positions ctx - q_len .. ctx - 1 (ctx =
 * context_lens[s] >= q_len; the cache must already hold positions
 * 0 .. ctx - 1, the new ones included).  Query i sees positions
 * 0 .. ctx - q_len + i (causal); query head h reads KV head
 * h / (q_heads / kv_heads).
 *
 * The query enters as E4M3 codes with one scale per (token, head) row:
 * q_codes [total_q, q_heads, 128] and q_scales [total_q * q_heads], as
 * pgf8_fp8_quantize_rows (DYNAMIC) writes them for q viewed as
 * [total_q * q_heads, 128].  Both products run E4M3 x E4M3 with binary32
 * accumulation: scores S = q_codes . k_codes * sq * sk / sqrt(128); softmax
 * in binary32 (exp2f); the probabilities relative to the running row
 * maximum are rounded to E4M3 after scaling by 2^8 (the only rounding
 * beyond binary32: at most 2^-4 relative, or 2^-18 absolute below 2^-14);
 * out = (sum_t P_t . v_codes_t) * 2^-8 * sv / sum_t p_t, rounded once to
 * out_dt.
 *
 * head_dim must be 128 (else PGF8_ERR_UNSUPPORTED); block_size a multiple
 * of 16; num_blocks * kv_heads * block_size < 2^31 - 1.  max_q_len (host)
 * bounds every q_len: the grid covers it.  out [total_q, q_heads, 128],
 * token stride ldo elements.  errors (device int32 or NULL) counts
 * out-of-range block-table entries (those positions are left out), q_len
 * beyond max_q_len (the tail rows are not written) and sequences with
 * ctx < q_len, ctx > max_context or query tokens outside [0, total_q)
 * (not written).  Alignment: q_codes and
 * the caches 16 bytes; q_scales, q_start, tables, lengths, errors 4 bytes;
 * out its element size.  seqs, total_q or max_q_len == 0: no-op.
 * ---------------------------------------------------------------------- */
pgf8_status pgf8_fp8_attention_context_paged(const uint8_t *q_codes, const float *q_scales,
                                             const int32_t *q_start, int64_t seqs, int64_t total_q,
                                             int64_t max_q_len, int64_t q_heads, const pgf8_paged_kv_cache *cache,
                                             const int32_t *block_tables, int64_t table_stride,
                                             const int32_t *context_lens, int64_t max_context, void *out,
                                             pgf8_dtype out_dt, int64_t ldo, int32_t *errors, void *stream);

/* ------------------------------------------------------------------------
 * Normalisation or gate fused with the per-token quantisation ("7B on an
 * RTX 4060 with FP8", computation graph §2.1: LayerNorm fused with the QKV
 * projection's input).  The normalised / gated values never go to memory;
 * the codes and per-token scales feed pgf8_fp8_linear.  The values are
 * computed in binary32 (textbook definitions below), then quantised as in
 * pgf8_fp8_quantize_rows (DYNAMIC).  The pages print no formula and no
 * numerics for these steps; the binary32 rounding of the values depends on
 * the kernel's reduction order and on expf.
 *
 * pgf8_fp8_norm_quantize: x [rows, cols] f32 or f16 (row stride ldx),
 *   gamma [cols] f32, beta [cols] f32 or NULL.  With beta: LayerNorm
 *   y = (x - mean) * rsqrt(var + eps) * gamma + beta (biased variance);
 *   without: RMSNorm y = x * rsqrt(mean(x^2) + eps) * gamma.  eps >= 0.
 *   cols % 16 == 0 and cols <= 16384 (a row is held in registers; else
 *   PGF8_ERR_UNSUPPORTED).  q [rows, cols], scales [rows].
 * pgf8_fp8_silu_mul_quantize: gu [rows, 2*inter] bf16 or f32 (row stride
 *   ldg >= 2*inter), the gate+up projection's output: gate = columns
 *   [0, inter), up = [inter, 2*inter).  h = gate / (1 + exp(-gate)) * up is
 *   quantised into q [rows, inter], scales [rows].  inter % 16 == 0.
 * flags: PGF8_FLAG_OVERLAP_PREVIOUS as for the per-tensor calls.
 * ---------------------------------------------------------------------- */
pgf8_status pgf8_fp8_norm_quantize(const void *x, pgf8_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                                   const float *gamma, const float *beta, float eps, uint8_t *q, float *scales,
                                   int32_t flags, void *stream);
pgf8_status pgf8_fp8_silu_mul_quantize(const void *gu, pgf8_dtype gdt, int64_t rows, int64_t inter, int64_t ldg,
                                       uint8_t *q, float *scales, int32_t flags, void *stream);

/* ------------------------------------------------------------------------
 * Per-tensor activation scaling ("C++ and FP8" §5.1: MINMAX calibration,
 * the scale follows the largest magnitude seen over calibration data;
 * "7B on an RTX 4060 with FP8" §6.1: delayed scaling over an amax history
 * of length >= 1024, scale below 448).  Readings: amax = max |x| over the
 * tensor (NaN ignored); scale = RN(amax / 448) in binary32, 1 when 0; codes
 * = E4M3(RN(x / scale)), saturating.  The codes and per-row scales feed
 * pgf8_fp8_linear as they are (every row carries the tensor's scale).
 * x [rows, cols] f32 or f16, row stride ldx; q [rows, cols] contiguous;
 * alignment as for pgf8_fp8_quantize_rows; rows == 0 does nothing (except
 * for a delayed step, which needs at least one row).
 *
 * pgf8_fp8_amax_accumulate: *amax = max(*amax, amax(x)) (device scalar,
 *   start from +0.0; calibration over several batches accumulates).
 * pgf8_fp8_quantize_tensor: static per-tensor quantisation with the scale
 *   of a calibrated amax (device scalar); scales [rows] (may be NULL)
 *   receives that scale.
 * pgf8_delayed_state_init: history [history_len] (device) zeroed, the
 *   state (device, 16-byte aligned) set to quantise step 0 with
 *   initial_scale (> 0).  history_len 1..2^24 (the pages ask >= 1024).
 * pgf8_fp8_quantize_delayed: step `step` (0, 1, 2, ... : the caller counts
 *   the calls made on this state) quantises x (rows >= 1) with the scale
 *   carried out of the previous step, RN(max of the last history_len
 *   amaxes / 448) (1 when 0; step 0: initial_scale), written to scales
 *   [rows] if not NULL; x's amax is recorded for the steps that follow.
 *   One kernel, no CTA waits for another: step t derives its scale from the
 *   history ring (amaxes up to step t-2) and the amax of step t-1, which is
 *   still pending in state.pending[(t-1) % 3] (one CTA then files it into
 *   slot (t-1) mod history_len).  Steps on one state must be stream-ordered
 *   and numbered consecutively.
 * flags (quantize_tensor, quantize_delayed): PGF8_FLAG_OVERLAP_PREVIOUS
 *   launches the kernel with programmatic stream serialization, as for the
 *   linear entry points: it reads and writes nothing before the previous
 *   kernel in the stream has completed, and a GEMM launched the same way
 *   after it may start loading its weights while it runs.
 * ---------------------------------------------------------------------- */
typedef struct {
    float initial_scale;  /* the scale of step 0 */
    uint32_t pending[3];  /* amax of step t, accumulated in pending[t % 3] (bits of a float >= 0) */
} pgf8_delayed_state;

pgf8_status pgf8_fp8_amax_accumulate(const void *x, pgf8_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                                     float *amax, void *stream);
pgf8_status pgf8_fp8_quantize_tensor(const void *x, pgf8_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                                     const float *amax, uint8_t *q, float *scales, int32_t flags, void *stream);
pgf8_status pgf8_delayed_state_init(pgf8_delayed_state *state, float *history, int32_t history_len,
                                    float initial_scale, void *stream);
pgf8_status pgf8_fp8_quantize_delayed(const void *x, pgf8_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                                      uint8_t *q, float *scales, float *history, int32_t history_len,
                                      pgf8_delayed_state *state, int64_t step, int32_t flags, void *stream);

/* ------------------------------------------------------------------------
 * Dynamic-activation FP8 linear: per-token quantisation of x (as
 * pgf8_fp8_quantize_rows, DYNAMIC) followed by pgf8_fp8_linear, enqueued as
 * one dependent pair so the GEMM's set-up and first weight loads overlap the
 * quantisation ("7B on an RTX 4060 with FP8" §2.2: activations quantised at
 * run time).  x [M,K] f32 or f16 with row stride ldx.  The workspace
 * (size from pgf8_fp8_linear_dynamic_workspace_size; zero-filled before its
 * first use) receives the E4M3 activation codes [M,K] at byte offset
 * pgf8_fp8_linear_dynamic_codes_offset(M, K) and the per-token scales [M] at
 * pgf8_fp8_linear_dynamic_scales_offset(M, K); the caller may read both after
 * the call completes.  Its first 1024 bytes are synchronisation words for
 * every shape, so one workspace can serve layers of different shapes.  wq must not be written by work enqueued
 * between this call's quantisation and GEMM (nothing is).
 * ---------------------------------------------------------------------- */
pgf8_status pgf8_fp8_linear_dynamic(const void *x, pgf8_dtype xdt, int64_t M, int64_t K,
                                    int64_t ldx, const uint8_t *wq, const float *sw, int64_t N,
                                    void *y_bf16, void *workspace, size_t workspace_bytes,
                                    const pgf8_linear_opts *opts, void *stream);

size_t pgf8_fp8_linear_dynamic_workspace_size(int64_t M, int64_t N, int64_t K);
size_t pgf8_fp8_linear_dynamic_codes_offset(int64_t M, int64_t K);

/* Which kernels a dynamic FP8 linear call with these arguments would run
 * (host only: nothing is enqueued, no device memory is touched).  *fused =
 * 1 when the GEMM quantises the activations itself (PGF8_FLAG_FUSED_QUANT
 * set and applicable), else 0.  *split_k = the K-split of the skinny GEMM
 * (1..8), or 0 when the call takes a tiled kernel.  Returns
 * PGF8_ERR_INVALID_ARG / ALIGNMENT / UNSUPPORTED for arguments the call
 * itself would reject on shape or dtype grounds.  The pages have no
 * counterpart: this is a query of this library's kernel choice. */
pgf8_status pgf8_fp8_linear_dynamic_plan(int64_t M, int64_t N, int64_t K, pgf8_dtype xdt,
                                         const pgf8_linear_opts *opts, int32_t *fused, int32_t *split_k);

/* One layer of pgf8_fp8_linear_dynamic_many: the arguments of
 * pgf8_fp8_linear_dynamic. */
typedef struct {
    const void *x;           /* [M, K] f32 or f16, row stride ldx */
    int32_t xdt;             /* pgf8_dtype */
    int32_t reserved;
    int64_t M, K, ldx, N;
    const uint8_t *wq;       /* [N, K] E4M3 codes */
    const float *sw;         /* [N] */
    void *y;                 /* [M, N] bf16 */
    void *workspace;         /* pgf8_fp8_linear_dynamic_workspace_size(M, N, K) bytes */
    size_t workspace_bytes;
} pgf8_fp8_layer;

/* ------------------------------------------------------------------------
 * A sequence of dynamic FP8 linear layers enqueued by one call, in order, on
 * `stream` (a decoder step's linears, say).  Every layer is checked before
 * anything is enqueued; the first invalid one makes the call return its
 * status and enqueue nothing.  Layer i+1 is launched with
 * PGF8_FLAG_OVERLAP_PREVIOUS (it may start loading its weights while layer i
 * finishes), so no layer's weights may alias another layer's x, y or
 * workspace; the first layer uses the flags given in opts.  Each layer may
 * read the previous layer's y as its x (the overlap never moves an
 * activation read ahead of the kernel that writes it).
 * ---------------------------------------------------------------------- */
pgf8_status pgf8_fp8_linear_dynamic_many(const pgf8_fp8_layer *layers, int64_t count,
                                         const pgf8_linear_opts *opts, void *stream);
size_t pgf8_fp8_linear_dynamic_scales_offset(int64_t M, int64_t K);

/* ------------------------------------------------------------------------
 * A group of INDEPENDENT dynamic FP8 linear layers (no layer reads another
 * layer's output: the linears of several sequences or of one decoder step
 * measured as a batch, the separate Q, K, V or gate and up projections)
 * enqueued by one call on `stream`.  Each layer computes exactly what
 * pgf8_fp8_linear_dynamic computes ("7B on an RTX 4060 with FP8" §2.2
 * per-token dynamic scale, §6.1 scale = amax / 448; "C++ and FP8" §3.3
 * E4M3 x E4M3 -> f32 -> bf16): its codes and scales in its own workspace
 * are bit-identical to that call's, its outputs are within the same bound
 * (the f32 summation order differs).
 *
 * Layers with M <= 128 are quantised by one launch and then streamed by one
 * persistent grouped kernel (one CTA per SM, each SM streaming an equal
 * share of all those layers' weights, up to 32 layers per launch pair).
 * Decode-sized layers are bound by their weight stream ("7B token speed on
 * consumer GPUs" §1), and one stream for the whole group pays the start and
 * the end of a launch once instead of once per layer.  The layers with
 * M > 128 are then quantised by one launch and multiplied as
 * pgf8_fp8_linear_group multiplies them (the layers with a few rounds of
 * tiles in one launch on SM pairs, so one layer's last round is filled by
 * the next layer's; larger layers one tiled launch each).  With explicit kernel options (path, tile_n or split_k set)
 * the layers with 128 < M <= 256 take a grouped launch pair of their own
 * and larger layers run one dynamic call each, with those options.
 *
 * group_workspace: pgf8_fp8_linear_group_workspace_size(max M over the
 * layers) bytes of device memory, 16-byte aligned, zero-filled once before
 * its first use; every completed call leaves its flag words zero again, so
 * it is reused without clearing.  Calls that use one group workspace must
 * not overlap on the GPU.  May be null when no layer has M <= 256.
 * Errors: any layer's own argument errors (nothing is enqueued);
 * PGF8_ERR_INVALID_ARG when an output or workspace of one layer overlaps
 * an input, output or workspace of another (or its own input), or the
 * group workspace is missing or too small; PGF8_ERR_ALIGNMENT for an
 * unaligned group workspace.  Deterministic for a fixed group of shapes on
 * a fixed device.  PGF8_FLAG_OVERLAP_PREVIOUS in opts applies to the first
 * launch.  The pages have no grouped form: this is how this library
 * streams a step's decode linears on B200.
 * ---------------------------------------------------------------------- */
pgf8_status pgf8_fp8_linear_dynamic_group(const pgf8_fp8_layer *layers, int64_t count,
                                          void *group_workspace, size_t group_workspace_bytes,
                                          const pgf8_linear_opts *opts, void *stream);
size_t pgf8_fp8_linear_group_workspace_size(int64_t max_m);

/* One layer of pgf8_fp8_linear_group: the arguments of pgf8_fp8_linear
 * (pre-quantised activations). */
typedef struct {
    const uint8_t *aq;       /* [M, K] E4M3 codes */
    const float *sa;         /* [M] */
    const uint8_t *wq;       /* [N, K] E4M3 codes */
    const float *sw;         /* [N] */
    void *y;                 /* [M, N] bf16 */
    int64_t M, K, N;
} pgf8_fp8_gemm_layer;

/* ------------------------------------------------------------------------
 * Independent FP8 GEMMs with their dequantising epilogue ("C++ and FP8"
 * §3.3: E4M3 x E4M3 -> f32 -> bf16), each exactly what pgf8_fp8_linear
 * computes (within the same bound; the f32 summation order may differ).
 * The layers with at most 296 tiles of 256 x 256 (four rounds of the
 * B200's 74 SM pairs) share one persistent launch on SM pairs over all
 * their tiles (up to 32 layers per launch); each larger layer runs its own
 * tiled launch (measured faster for those).  The tiled GEMMs of the
 * grouped dynamic call's M > 128 layers, for callers that quantise
 * themselves; any M works, but the 256-token tiles suit M > 128.
 * No workspace.  Errors: a layer's argument errors (as pgf8_fp8_linear) or
 * an output overlapping any layer's operands or another layer's output
 * (PGF8_ERR_INVALID_ARG), before anything is enqueued; opts other than the
 * automatic choice (path, tile_n, split_k) give PGF8_ERR_UNSUPPORTED.
 * The launch may start while the previous kernel in the stream finishes
 * (it reads nothing before that kernel has completed).
 * ---------------------------------------------------------------------- */
pgf8_status pgf8_fp8_linear_group(const pgf8_fp8_gemm_layer *layers, int64_t count,
                                  const pgf8_linear_opts *opts, void *stream);

/* ------------------------------------------------------------------------
 * Building blocks of a tensor-parallel FP8 linear layer ("C++ and FP8"
 * §4.2: the --tp_size deployment; §5.2: the partial results of a split
 * layer summed over NVLink).  A layer split along K (row-parallel) gives
 * each rank a slice of every token's row, but the per-token scale must
 * come from the amax over the WHOLE row ("7B on an RTX 4060 with FP8"
 * §2.2, §6.1), and the partial products must be summed before the single
 * rounding to bf16.  The sequence per rank is:
 *   pgf8_fp8_row_amax        amax of each row of this rank's slice
 *   (all-reduce MAX of the amax over the ranks)
 *   pgf8_fp8_quantize_rows_amax   codes and scales from the reduced amax:
 *                            bit-identical to pgf8_fp8_quantize_rows
 *                            (DYNAMIC) on the full rows
 *   pgf8_fp8_linear_partial  f32 partial sum of this rank's slice of K,
 *                            scaled by sa[m] * sw[n] (sw of the full rows)
 *   (all-reduce SUM of the f32 partials over the ranks)
 *   pgf8_round_bf16          one rounding of the sum to bf16
 * A layer split along N (column-parallel) needs none of this: each rank
 * quantises the whole activation rows and runs pgf8_fp8_linear_dynamic on
 * its channels.
 *
 * pgf8_fp8_row_amax: amax[r] = max_c |x[r, c]| (NaN ignored), x [rows,
 *   cols] f32 or f16 (row stride ldx elements).  Checks and alignment as
 *   pgf8_fp8_quantize_rows (no codes).
 * pgf8_fp8_quantize_rows_amax: amax_scales[r] holds the row's amax on
 *   input; on output it holds s = fl32(amax / 448) (1 for a zero amax), and
 *   q[r, c] = E4M3_satfinite_RN(fl32(x[r, c] / s)).
 * pgf8_fp8_linear_partial: y_f32[m, n] = fl32(sum_k e4m3(aq[m,k])
 *   e4m3(wq[n,k]) * sa[m] * sw[n]) with f32 accumulation and no rounding
 *   to 16 bits.  workspace: pgf8_fp8_linear_partial_workspace_size bytes,
 *   16-byte aligned, zero-filled once (the kernels leave their flag words
 *   zero).  y_f32 16-byte aligned.  Deterministic for a fixed shape.
 * pgf8_round_bf16: y[i] = bf16_RN(x[i]); n % 8 == 0, both 16-byte aligned.
 * ---------------------------------------------------------------------- */
pgf8_status pgf8_fp8_row_amax(const void *x, pgf8_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                              float *amax, void *stream);
pgf8_status pgf8_fp8_quantize_rows_amax(const void *x, pgf8_dtype xdt, int64_t rows, int64_t cols,
                                        int64_t ldx, uint8_t *q, float *amax_scales, void *stream);
pgf8_status pgf8_fp8_linear_partial(const uint8_t *aq, const float *sa, int64_t M, int64_t K,
                                    const uint8_t *wq, const float *sw, int64_t N, float *y_f32,
                                    void *workspace, size_t workspace_bytes, void *stream);
size_t pgf8_fp8_linear_partial_workspace_size(int64_t M, int64_t N, int64_t K);
pgf8_status pgf8_round_bf16(const float *x, int64_t n, void *y_bf16, void *stream);

/* ------------------------------------------------------------------------
 * NestedFP byte-plane split ("NestedFP" §2.1): for each FP16 weight bit
 * pattern b of w_f16 [N,K]: hi[n,k] = b >> 8 (sign, 5 exponent bits, top 2
 * mantissa bits), lo[n,k] = b & 0xFF.  Bit-exact; (hi << 8) | lo == b.
 * ---------------------------------------------------------------------- */
pgf8_status pgf8_nestedfp_split(const void *w_f16, int64_t N, int64_t K, uint8_t *hi,
                                uint8_t *lo, void *stream);

/* ------------------------------------------------------------------------
 * NestedFP linear ("NestedFP" §2.1-2.2).  x_f16 [M,K] FP16, y_f16 [M,N] FP16.
 *   PGF8_NESTED_FP16: y = fp16_rn( sum_k x[m,k] * fp16((hi<<8)|lo)[n,k] ),
 *     the weight rebuilt bit-exactly in shared memory inside the GEMM;
 *     FP32 accumulation.  workspace: pgf8_nestedfp_linear_workspace_size
 *     bytes (nonzero for M <= 256: flags and partial slots of the grouped
 *     kernel, zero-filled once), may be NULL above.
 *   PGF8_NESTED_FP8: x is quantised per token to E4M3 (as
 *     pgf8_fp8_quantize_rows, DYNAMIC) into the workspace, and
 *     y = fp16_rn( (sum_k e4m3(aq[m,k]) * e5m2(hi[n,k])) * sa[m] ): the upper
 *     byte is read as an E5M2 code with unit scale, which is the FP16 weight
 *     with its low 8 bits cleared.  lo is ignored and may be NULL.
 * With the automatic kernel choice, M <= 16 runs the split-K skinny
 * kernel, 16 < M <= 256 the grouped weight-streaming kernel on this one
 * layer (every SM streams an equal share of the weight planes), larger M
 * the tiled kernels (FP16 mode: the one-CTA persistent kernel; its SM-pair
 * form, PGF8_PATH_TILED_PAIR, measured slower).  Several layers of one
 * mode: pgf8_nestedfp_linear_group.
 * ---------------------------------------------------------------------- */
pgf8_status pgf8_nestedfp_linear(const void *x_f16, int64_t M, int64_t K, const uint8_t *hi,
                                 const uint8_t *lo, int64_t N, pgf8_nested_mode mode,
                                 void *y_f16, void *workspace, size_t workspace_bytes,
                                 void *stream);

pgf8_status pgf8_nestedfp_linear_ex(const void *x_f16, int64_t M, int64_t K, const uint8_t *hi,
                                    const uint8_t *lo, int64_t N, pgf8_nested_mode mode,
                                    void *y_f16, void *workspace, size_t workspace_bytes,
                                    const pgf8_linear_opts *opts, void *stream);

size_t pgf8_nestedfp_linear_workspace_size(int64_t M, int64_t N, int64_t K,
                                           pgf8_nested_mode mode);

/* One layer of pgf8_nestedfp_linear_group: the arguments of
 * pgf8_nestedfp_linear. */
typedef struct {
    const void *x_f16;       /* [M, K] FP16, rows K elements apart */
    const uint8_t *hi;       /* [N, K] upper byte plane */
    const uint8_t *lo;       /* [N, K] lower byte plane (FP16 mode; ignored in FP8 mode) */
    void *y_f16;             /* [M, N] FP16 */
    void *workspace;         /* FP8 mode: pgf8_nestedfp_linear_workspace_size(M, N, K, FP8) bytes
                                (codes and scales); FP16 mode: unused, may be NULL */
    size_t workspace_bytes;
    int64_t M, K, N;
} pgf8_nested_layer;

/* ------------------------------------------------------------------------
 * A group of INDEPENDENT NestedFP linear layers in one mode ("NestedFP"
 * §2.1-2.2; no layer reads another layer's output), enqueued by one call on
 * `stream`.  Each layer computes exactly what pgf8_nestedfp_linear computes
 * in that mode (FP8 mode: its codes and scales bit-identical; its outputs
 * within the same bound, the f32 summation order differs).
 * Layers with M <= 256 stream their weight planes through the grouped
 * weight-streaming kernel (FP8 mode: one quantisation launch first; one
 * launch for the layers with M <= 128 and one for 128 < M <= 256, up to 32
 * layers each); larger layers run one call each.
 *   group_workspace: pgf8_fp8_linear_group_workspace_size(max M of the
 *     layers with M <= 256) bytes, zero-filled once before first use and
 *     left zero by every call; may be NULL when no layer has M <= 256.
 *   Every layer is checked before anything is enqueued (as
 *   pgf8_nestedfp_linear, plus: no layer's y or workspace overlaps any
 *   layer's x or another layer's y or workspace, else INVALID_ARG).
 *   PGF8_FLAG_OVERLAP_PREVIOUS in opts applies to the first launch.
 * ---------------------------------------------------------------------- */
pgf8_status pgf8_nestedfp_linear_group(const pgf8_nested_layer *layers, int64_t count,
                                       pgf8_nested_mode mode, void *group_workspace,
                                       size_t group_workspace_bytes, const pgf8_linear_opts *opts,
                                       void *stream);

/* ------------------------------------------------------------------------
 * Allocation-free dynamic FP8 linear.  The pages have no counterpart of this
 * entry point; it exists for callers that cannot hand the library a
 * workspace: a host program that links only this C library and has no
 * device allocator of its own, or an inference runtime whose device memory
 * is planned once before serving and which must not allocate on the request
 * path.
 *
 * It computes exactly what pgf8_fp8_linear_dynamic computes (same kernels,
 * same results), but keeps the activation codes and scales in a fixed array
 * inside the library (PGF8_NOALLOC_SCRATCH_BYTES, 8 MiB, held by every GPU
 * that loads the library until the process exits).  The caller still passes
 * x, wq, sw and y.  Nothing is allocated and no allocating routine is
 * called.
 *   Limit   pgf8_fp8_linear_dynamic_workspace_size(M, N, K) must not exceed
 *           PGF8_NOALLOC_SCRATCH_BYTES, else PGF8_ERR_TOO_LARGE is returned
 *           before anything is enqueued (e.g. M = 16 allows K up to ~350k;
 *           M = 1024 allows K up to ~8k).
 *   Set-up  The first call on each device, with that device current, looks
 *           up the array's device address (cudaGetSymbolAddress); make that
 *           first call before any stream capture begins.
 *   Sharing Every call uses the same array and it keeps the last call's
 *           codes and scales.  Nothing in it needs clearing (each call
 *           writes the codes and scales before its GEMM reads them), but
 *           calls whose work overlaps on the GPU (different streams, or
 *           different host threads on one device) race on the array: order
 *           them on one stream.
 * ---------------------------------------------------------------------- */
#define PGF8_NOALLOC_SCRATCH_BYTES (8u << 20)

pgf8_status pgf8_fp8_linear_dynamic_noalloc(const void *x, pgf8_dtype xdt, int64_t M, int64_t K,
                                            int64_t ldx, const uint8_t *wq, const float *sw,
                                            int64_t N, void *y_bf16, void *stream);

/* ------------------------------------------------------------------------
 * Diagnostics.
 * pgf8_last_cuda_error: the cudaError_t of the most recent failed CUDA call
 *   made by this library on the calling thread (0 if none).
 * pgf8_device_status: synchronises `stream`, then reads and clears the
 *   device error word of the current device: PGF8_ERR_TIMEOUT if a kernel
 *   gave up a bounded wait since the last check, PGF8_ERR_CUDA if the
 *   synchronisation itself failed, else PGF8_OK.
 * pgf8_selftest_bounded_wait: enqueues a one-thread kernel that waits on a
 *   barrier phase nothing ever completes, with a bound of limit_ns
 *   (1e3..2e9) instead of the library's 1 s.  The wait gives up, raises the
 *   device error word and the kernel returns: the next pgf8_device_status()
 *   on that stream reports PGF8_ERR_TIMEOUT and clears it.  For checking the
 *   failure path without hanging or faulting the GPU.
 * pgf8_selftest_row_division: checks the division the quantisation uses
 *   (x / s rounded to nearest-even binary32, one divisor per row, by an
 *   FMA remainder correction) against the device's IEEE division over EVERY
 *   finite binary32 x with |x| <= 512 s, for each of the `count` divisors in
 *   divisors[] (device, f32, count 1..64).  mismatches[] (device, 2 * count
 *   uint64, zero-filled by the caller) receives per divisor i:
 *   [2i] quotients that differ bitwise where |x| >= 2^-11 s, and [2i+1]
 *   E4M3 codes (RN, saturating) that differ anywhere in the domain.  Below
 *   2^-11 s the quotient may differ in its last bits (subnormal remainders)
 *   while its code is zero either way.  About 2^32 divisions per divisor
 *   (milliseconds each).  The pages define the quotient only as the rounded
 *   division; this self-test has no counterpart there.
 * pgf8_status_str: static description of a status code.
 * pgf8_version: library version as major*10000 + minor*100 + patch.
 * ---------------------------------------------------------------------- */
pgf8_status pgf8_last_cuda_error(int *cuda_err);
pgf8_status pgf8_device_status(void *stream);
pgf8_status pgf8_selftest_bounded_wait(int64_t limit_ns, void *stream);
pgf8_status pgf8_selftest_row_division(const float *divisors, int32_t count,
                                       unsigned long long *mismatches, void *stream);
const char *pgf8_status_str(pgf8_status status);
int pgf8_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PGF8_H */
