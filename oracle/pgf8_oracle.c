/*
 * pgf8 CPU oracle — TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, scalar C11 restatement of what the FP8 linear layer and the
 * NestedFP dual-precision layer compute.  It exists so that tests, the
 * smoke check and the benchmark's CPU-baseline leg can check the CUDA path
 * against an independent definition.  Nothing in the product links, loads
 * or calls this file; it shares no source, header, table or constant with
 * the CUDA library, and it includes no CUDA header.
 *
 * Arithmetic rules:
 *   - every floating-point quantity that the pages leave open is carried in
 *     IEEE binary64 (double); format conversions are done on the exact value
 *     with frexp/ldexp and nearbyint() under the default round-to-nearest-
 *     even mode;
 *   - where the method itself fixes a binary32 step (the per-token scale and
 *     the scaled value that is then cast to FP8) the step is written as a
 *     plain float operation, which C11 on x86-64 evaluates as a correctly
 *     rounded IEEE binary32 division (FLT_EVAL_METHOD == 0);
 *   - no blocking, reordering, vectorisation or threading: every result is
 *     the textbook loop.
 *
 * Sources (pages of the "precision_gemm_fp8" subject):
 *   [FP8-4060]  "7B on an RTX 4060 with FP8" (intelliparadigm.com 2151670):
 *               §2.1 E4M3 format; §2.2 static weight / dynamic activation
 *               scaling; §6.1 scale bound 448 and exponent saturation.
 *   [CPP-FP8]   "C++ and FP8 quantization for LLM inference" (tqpw.cn 201730):
 *               §3.1 E4M3 or E5M2; §3.3 kernel e4m3 x e4m3 -> f32 accumulate
 *               -> bf16 output, TN; §4.2 per-channel / per-token flags.
 *   [NestedFP]  "NestedFP dual-precision inference framework"
 *               (intelliparadigm.com 2229392): §2.1 byte-plane split and the
 *               (upper<<8)|lower rebuild; FP8 mode uses the upper byte;
 *               §4.1 underflow handling of the E4M3 converter.
 * The E4M3 ("FN" variant: no infinities, one NaN pattern per sign, largest
 * finite 448) and E5M2 bit layouts are the public OCP 8-bit floating point
 * definitions; binary16 is IEEE 754.
 *
 * Parity status of each function is stated in its comment; every function
 * here is pinned by a CPU test (see tests/test_oracle_*.py).
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>

#define ORC_OK 0
#define ORC_ERR_NONFINITE 1
#define ORC_ERR_BADSCALE 2
#define ORC_ERR_ARG 3

/* ------------------------------------------------------------------ */
/* FP8 E4M3 (FN): sign | 4 exponent bits (bias 7) | 3 mantissa bits.   */
/* [FP8-4060] §2.1 names E4M3; §6.1 fixes 448 as the largest value.    */
/* ------------------------------------------------------------------ */

double orc_e4m3_decode(uint8_t c)
{
    int s = (c >> 7) & 1;
    int e = (c >> 3) & 0xF;
    int m = c & 0x7;
    double v;
    if (e == 15 && m == 7)
        return NAN;                         /* the only NaN patterns: 0x7F, 0xFF */
    if (e == 0)
        v = ldexp((double)m, -9);           /* subnormal: m * 2^-9 */
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* Saturating, round-to-nearest-even cast of a binary32 value to E4M3.
 * Values above 448 in magnitude (and infinities) become +-448; NaN stays
 * NaN; the sign of zero is kept.  Subnormal results are produced by
 * rounding on the 2^-9 grid ([NestedFP] §4.1 asks that underflow be
 * handled). */
uint8_t orc_e4m3_encode(float v)
{
    if (isnan(v))
        return signbit(v) ? 0xFF : 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a > 448.0)
        return sign | 0x7E;                 /* satfinite */
    if (a < ldexp(1.0, -6)) {               /* below the smallest normal */
        double k = nearbyint(a * 512.0);    /* k in [0, 8]; 8 lands on 0x08 = 2^-6 */
        return sign | (uint8_t)k;
    }
    int e;
    (void)frexp(a, &e);                     /* a = f * 2^e, f in [0.5, 1) */
    int E = e - 1;                          /* a = 1.xxx * 2^E */
    double r = nearbyint((ldexp(a, -E) - 1.0) * 8.0);
    if (r == 8.0) {                         /* mantissa carried into the exponent */
        E += 1;
        r = 0.0;
    }
    if (E > 8 || (E == 8 && r == 7.0))
        return sign | 0x7E;
    return sign | (uint8_t)(((E + 7) << 3) | (int)r);
}

/* ------------------------------------------------------------------ */
/* FP8 E5M2: sign | 5 exponent bits (bias 15) | 2 mantissa bits.       */
/* [CPP-FP8] §3.1 names it as the other FP8 layout; it is exactly the  */
/* upper byte of an IEEE binary16 value ([NestedFP] §2.1).             */
/* ------------------------------------------------------------------ */

double orc_e5m2_decode(uint8_t c)
{
    int s = (c >> 7) & 1;
    int e = (c >> 2) & 0x1F;
    int m = c & 0x3;
    double v;
    if (e == 31)
        return m == 0 ? (s ? -INFINITY : INFINITY) : NAN;
    if (e == 0)
        v = ldexp((double)m, -16);          /* subnormal: m * 2^-16 */
    else
        v = ldexp(1.0 + (double)m / 4.0, e - 15);
    return s ? -v : v;
}

/* Saturating RNE cast to E5M2 (largest finite 57344 = 0x7B). */
uint8_t orc_e5m2_encode(float v)
{
    if (isnan(v))
        return signbit(v) ? 0xFF : 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a > 57344.0)
        return sign | 0x7B;
    if (a < ldexp(1.0, -14)) {
        double k = nearbyint(a * 65536.0);  /* k in [0, 4]; 4 lands on 0x04 = 2^-14 */
        return sign | (uint8_t)k;
    }
    int e;
    (void)frexp(a, &e);
    int E = e - 1;
    double r = nearbyint((ldexp(a, -E) - 1.0) * 4.0);
    if (r == 4.0) {
        E += 1;
        r = 0.0;
    }
    if (E > 15 || (E == 15 && r == 3.0))
        return sign | 0x7B;
    return sign | (uint8_t)(((E + 15) << 2) | (int)r);
}

/* ------------------------------------------------------------------ */
/* IEEE binary16 decode from its bit pattern.                          */
/* ------------------------------------------------------------------ */

double orc_fp16_decode(uint16_t b)
{
    int s = (b >> 15) & 1;
    int e = (b >> 10) & 0x1F;
    int m = b & 0x3FF;
    double v;
    if (e == 31)
        return m == 0 ? (s ? -INFINITY : INFINITY) : NAN;
    if (e == 0)
        v = ldexp((double)m, -24);
    else
        v = ldexp(1.0 + (double)m / 1024.0, e - 15);
    return s ? -v : v;
}

/* ------------------------------------------------------------------ */
/* Per-row quantisation ([FP8-4060] §2.2 dynamic activation amax;      */
/* [CPP-FP8] §4.2 per-token / per-channel granularity; [FP8-4060] §6.1 */
/* the 448 bound applies to the scaled values).                        */
/*                                                                     */
/* For each row r (fixed order of the steps, since the pages leave it  */
/* open):                                                              */
/*   amax  = max_k |x[r,k]|                      (exact)               */
/*   s     = fl32(amax / 448)                    (binary32 division)   */
/*           s := 1 when that quotient is 0 (an all-zero row)          */
/*   q[r,k]= E4M3_satfinite_RNE( fl32(x[r,k] / s) )                    */
/* mode 0 (dynamic) writes s to scales[r]; mode 1 (static) reads it.   */
/* ------------------------------------------------------------------ */

static int quantize_one_row(const float *xr, int64_t cols, uint8_t *qr, float *s_io, int mode)
{
    float s;
    if (mode == 0) {
        float amax = 0.0f;
        for (int64_t k = 0; k < cols; ++k) {
            float a = fabsf(xr[k]);
            if (!isfinite(a))
                return ORC_ERR_NONFINITE;
            if (a > amax)
                amax = a;
        }
        s = amax / 448.0f;
        if (s == 0.0f)
            s = 1.0f;
        *s_io = s;
    } else {
        s = *s_io;
        if (!(s > 0.0f) || !isfinite(s))
            return ORC_ERR_BADSCALE;
        for (int64_t k = 0; k < cols; ++k)
            if (!isfinite(xr[k]))
                return ORC_ERR_NONFINITE;
    }
    for (int64_t k = 0; k < cols; ++k) {
        float t = xr[k] / s;                /* correctly rounded binary32 quotient */
        qr[k] = orc_e4m3_encode(t);
    }
    return ORC_OK;
}

/* x: rows x cols binary32 with row stride ldx (elements); q: rows x cols
 * contiguous codes; scales: rows. */
int orc_quantize_rows_f32(const float *x, int64_t rows, int64_t cols, int64_t ldx,
                          uint8_t *q, float *scales, int mode)
{
    if (rows < 0 || cols < 0 || ldx < cols || (mode != 0 && mode != 1))
        return ORC_ERR_ARG;
    for (int64_t r = 0; r < rows; ++r) {
        int st = quantize_one_row(x + r * ldx, cols, q + r * cols, scales + r, mode);
        if (st != ORC_OK)
            return st;
    }
    return ORC_OK;
}

/* Same for binary16 input bits: each element is widened exactly to
 * binary32 first (every binary16 value is a binary32 value). */
int orc_quantize_rows_f16(const uint16_t *x, int64_t rows, int64_t cols, int64_t ldx,
                          uint8_t *q, float *scales, int mode, float *tmp_row)
{
    if (rows < 0 || cols < 0 || ldx < cols || (mode != 0 && mode != 1))
        return ORC_ERR_ARG;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < cols; ++k)
            tmp_row[k] = (float)orc_fp16_decode(x[r * ldx + k]);
        int st = quantize_one_row(tmp_row, cols, q + r * cols, scales + r, mode);
        if (st != ORC_OK)
            return st;
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* FP8 linear ([CPP-FP8] §3.3: E4M3 x E4M3 operands, both K-contiguous */
/* ("TN"), f32 accumulation, bf16 output; scales from [FP8-4060] §2.2).*/
/*   ref[m,n] = ( sum_k dec(aq[m,k]) * dec(wq[n,k]) ) * sa[m] * sw[n]  */
/* evaluated in binary64.  Every product of two E4M3 values is exact   */
/* in binary64.                                                        */
/* ------------------------------------------------------------------ */

void orc_fp8_linear(const uint8_t *aq, const float *sa, int64_t M, int64_t K,
                    const uint8_t *wq, const float *sw, int64_t N, double *ref)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += orc_e4m3_decode(aq[m * K + k]) * orc_e4m3_decode(wq[n * K + k]);
            ref[m * N + n] = acc * (double)sa[m] * (double)sw[n];
        }
}

/* ------------------------------------------------------------------ */
/* NestedFP ([NestedFP] §2.1).                                         */
/* ------------------------------------------------------------------ */

/* Split each binary16 bit pattern b into hi = b >> 8 (sign, the five
 * exponent bits and the top two mantissa bits) and lo = b & 0xFF (the low
 * eight mantissa bits). */
void orc_nestedfp_split(const uint16_t *w, int64_t count, uint8_t *hi, uint8_t *lo)
{
    for (int64_t i = 0; i < count; ++i) {
        hi[i] = (uint8_t)(w[i] >> 8);
        lo[i] = (uint8_t)(w[i] & 0xFF);
    }
}

uint16_t orc_nestedfp_rebuild(uint8_t hi, uint8_t lo)
{
    return (uint16_t)(((unsigned)hi << 8) | (unsigned)lo);
}

/* FP16 mode: the weight is the rebuilt binary16 value.
 *   ref[m,n] = sum_k fp16(x[m,k]) * fp16((hi[n,k] << 8) | lo[n,k])   (binary64) */
void orc_nestedfp_linear_fp16(const uint16_t *x, int64_t M, int64_t K,
                              const uint8_t *hi, const uint8_t *lo, int64_t N, double *ref)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                uint16_t wb = orc_nestedfp_rebuild(hi[n * K + k], lo[n * K + k]);
                acc += orc_fp16_decode(x[m * K + k]) * orc_fp16_decode(wb);
            }
            ref[m * N + n] = acc;
        }
}

/* FP8 mode: the upper byte alone is the weight, read as an E5M2 code with
 * unit scale; activations are quantised per token to E4M3 exactly as
 * orc_quantize_rows_f16 does (dynamic mode).  aq (M x K) and sa (M) are
 * outputs, tmp_row holds K floats.
 *   ref[m,n] = ( sum_k dec_e4m3(aq[m,k]) * dec_e5m2(hi[n,k]) ) * sa[m]   */
int orc_nestedfp_linear_fp8(const uint16_t *x, int64_t M, int64_t K,
                            const uint8_t *hi, int64_t N, double *ref,
                            uint8_t *aq, float *sa, float *tmp_row)
{
    int st = orc_quantize_rows_f16(x, M, K, K, aq, sa, 0, tmp_row);
    if (st != ORC_OK)
        return st;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += orc_e4m3_decode(aq[m * K + k]) * orc_e5m2_decode(hi[n * K + k]);
            ref[m * N + n] = acc * (double)sa[m];
        }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Per-tensor scaling variants.                                        */
/*                                                                     */
/* [CPP-FP8] §5.1 names MINMAX calibration (the scale follows the      */
/* largest magnitude seen over representative calibration data);       */
/* [FP8-4060] §6.1 asks for an amax history of length >= 1024 and a    */
/* scale below 448.  Readings (the pages give no formulas):            */
/*   amax of a tensor   = max |x| over all its elements (exact);       */
/*   per-tensor scale   s = fl32(amax / 448), 1 when that is 0 (as the */
/*                      per-row rule);                                 */
/*   delayed scaling    step t quantises with the scale carried in     */
/*                      from step t-1; then history[pos] = amax(x_t),  */
/*                      pos = (pos + 1) mod H, and the carried scale   */
/*                      becomes fl32(max(history) / 448) (1 when 0).   */
/* Values above 448 s saturate to the largest finite code (satfinite). */
/* Non-finite inputs are an error here (the pages define no result).   */
/* ------------------------------------------------------------------ */

/* *amax = max(*amax, max |x|) over a rows x cols block (row stride ldx). */
int orc_amax_accumulate_f32(const float *x, int64_t rows, int64_t cols, int64_t ldx, float *amax)
{
    if (rows < 0 || cols < 0 || ldx < cols || !amax || !(*amax >= 0.0f))
        return ORC_ERR_ARG;
    float m = *amax;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t k = 0; k < cols; ++k) {
            float a = fabsf(x[r * ldx + k]);
            if (!isfinite(a))
                return ORC_ERR_NONFINITE;
            if (a > m)
                m = a;
        }
    }
    *amax = m;
    return ORC_OK;
}

/* The per-tensor scale of an amax (reading above). */
static float scale_of_amax(float amax)
{
    float s = amax / 448.0f;
    if (s == 0.0f)
        s = 1.0f;
    return s;
}

/* Static per-tensor quantisation with the scale of a calibrated amax:
 * every row uses s = scale_of_amax(amax); s is written to *s_out. */
int orc_quantize_tensor_f32(const float *x, int64_t rows, int64_t cols, int64_t ldx, float amax, uint8_t *q,
                            float *s_out)
{
    if (rows < 0 || cols < 0 || ldx < cols || !(amax >= 0.0f) || !isfinite(amax))
        return ORC_ERR_ARG;
    float s = scale_of_amax(amax);
    for (int64_t r = 0; r < rows; ++r) {
        float sr = s;
        int st = quantize_one_row(x + r * ldx, cols, q + r * cols, &sr, 1);
        if (st != ORC_OK)
            return st;
    }
    *s_out = s;
    return ORC_OK;
}

/* One step of delayed scaling (reading above).  history: H >= 1 amaxes,
 * *pos in [0, H), *scale the carried scale (> 0, finite).  q receives the
 * codes of this step; *step_scale the scale they were made with. */
int orc_delayed_step_f32(const float *x, int64_t rows, int64_t cols, int64_t ldx, uint8_t *q, float *history,
                         int32_t H, int32_t *pos, float *scale, float *step_scale)
{
    if (rows < 0 || cols < 0 || ldx < cols || H < 1 || !pos || *pos < 0 || *pos >= H || !scale)
        return ORC_ERR_ARG;
    float s = *scale;
    if (!(s > 0.0f) || !isfinite(s))
        return ORC_ERR_BADSCALE;
    for (int64_t r = 0; r < rows; ++r) {
        float sr = s;
        int st = quantize_one_row(x + r * ldx, cols, q + r * cols, &sr, 1);
        if (st != ORC_OK)
            return st;
    }
    float a = 0.0f;
    int st = orc_amax_accumulate_f32(x, rows, cols, ldx, &a);
    if (st != ORC_OK)
        return st;
    *step_scale = s;
    history[*pos] = a;
    *pos = (*pos + 1) % H;
    float hmax = 0.0f;
    for (int32_t i = 0; i < H; ++i)
        if (history[i] > hmax)
            hmax = history[i];
    *scale = scale_of_amax(hmax);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Normalisation and gated activation ahead of the quantisation.       */
/*                                                                     */
/* [FP8-4060] "computation graph restructuring" §2.1 fuses LayerNorm   */
/* with the QKV projection's input; its feature list pairs LayerNorm   */
/* with the activation.  The pages print no formula.  Readings (the    */
/* textbook definitions), evaluated in binary64:                       */
/*   LayerNorm  y = (x - mean) / sqrt(var + eps) * gamma + beta,       */
/*              mean = sum x / K, var = sum (x - mean)^2 / K;          */
/*   RMSNorm    y = x / sqrt(sum x^2 / K + eps) * gamma  (beta absent);*/
/*   SiLU gate  h = g / (1 + exp(-g)) * u.                             */
/* ------------------------------------------------------------------ */

/* y [rows, cols] binary64 from x (row stride ldx); beta == NULL selects
 * RMSNorm. */
int orc_norm_rows(const float *x, int64_t rows, int64_t cols, int64_t ldx, const float *gamma, const float *beta,
                  double eps, double *y)
{
    if (rows < 0 || cols < 1 || ldx < cols || !gamma || !(eps >= 0.0))
        return ORC_ERR_ARG;
    for (int64_t r = 0; r < rows; ++r) {
        const float *xr = x + r * ldx;
        for (int64_t k = 0; k < cols; ++k)
            if (!isfinite(xr[k]))
                return ORC_ERR_NONFINITE;
        double mean = 0.0;
        if (beta) {
            for (int64_t k = 0; k < cols; ++k)
                mean += (double)xr[k];
            mean /= (double)cols;
        }
        double ss = 0.0;
        for (int64_t k = 0; k < cols; ++k) {
            double d = (double)xr[k] - mean;
            ss += d * d;
        }
        double inv = 1.0 / sqrt(ss / (double)cols + eps);
        for (int64_t k = 0; k < cols; ++k) {
            double v = ((double)xr[k] - mean) * inv * (double)gamma[k];
            if (beta)
                v += (double)beta[k];
            y[r * cols + k] = v;
        }
    }
    return ORC_OK;
}

/* h[i] = g[i] / (1 + exp(-g[i])) * u[i] in binary64. */
void orc_silu_mul(const double *g, const double *u, int64_t count, double *h)
{
    for (int64_t i = 0; i < count; ++i)
        h[i] = g[i] / (1.0 + exp(-g[i])) * u[i];
}

/* ------------------------------------------------------------------ */
/* FP8 KV cache.                                                       */
/*                                                                     */
/* [FP8-4060] stores K/V in FP8 (half the cache: 96 -> 48 MB at 1024   */
/* tokens, ~1 % conversion cost); [CPP-FP8] §3.2 pages the cache in    */
/* blocks of 16 tokens handed out by a central allocator and keeps the */
/* blocks in FP8, §3.3 computes context attention in the FP8 dataflow  */
/* (kv_cache_dtype fp8).  No formula or scale granularity is printed.  */
/* Readings:                                                           */
/*   scales     one per KV head, MINMAX over calibration data:         */
/*              s_h = fl32(max |k[., h, .]| / 448), 1 when 0;          */
/*   codes      E4M3_satfinite_RNE(fl32(k / s_h)), as the rows above;  */
/*   layout     cache[block][kv_head][slot][d], slot = token % B, the  */
/*              block of a token from a block table (token / B -> id); */
/*   attention  per query head h (KV head h / G with G = Hq / Hkv):    */
/*              out = sum_t softmax_t(q . k_t / sqrt(D)) v_t over the  */
/*              dequantised cache, keys t <= the query's position,     */
/*              evaluated in binary64 (q unquantised).                 */
/* ------------------------------------------------------------------ */

/* s[h] for kv [T, H, D] binary32 (contiguous). */
int orc_kv_calibrate_scales(const float *kv, int64_t T, int64_t H, int64_t D, float *s)
{
    if (T < 0 || H < 1 || D < 1)
        return ORC_ERR_ARG;
    for (int64_t h = 0; h < H; ++h) {
        float amax = 0.0f;
        for (int64_t t = 0; t < T; ++t)
            for (int64_t d = 0; d < D; ++d) {
                float a = fabsf(kv[(t * H + h) * D + d]);
                if (!isfinite(a))
                    return ORC_ERR_NONFINITE;
                if (a > amax)
                    amax = a;
            }
        s[h] = scale_of_amax(amax);
    }
    return ORC_OK;
}

/* Writes tokens [t0, t0 + T) of kv [T, H, D] into the paged cache
 * [num_blocks, H, B, D] through block_table (logical block -> physical). */
int orc_kv_write_paged(const float *kv, int64_t t0, int64_t T, int64_t H, int64_t D, const float *s, int64_t B,
                       const int32_t *block_table, int64_t num_blocks, uint8_t *cache)
{
    if (t0 < 0 || T < 0 || H < 1 || D < 1 || B < 1)
        return ORC_ERR_ARG;
    for (int64_t t = 0; t < T; ++t) {
        int64_t pos = t0 + t;
        int64_t blk = block_table[pos / B];
        if (blk < 0 || blk >= num_blocks)
            return ORC_ERR_ARG;
        int64_t slot = pos % B;
        for (int64_t h = 0; h < H; ++h) {
            if (!(s[h] > 0.0f) || !isfinite(s[h]))
                return ORC_ERR_BADSCALE;
            for (int64_t d = 0; d < D; ++d) {
                float x = kv[(t * H + h) * D + d];
                if (!isfinite(x))
                    return ORC_ERR_NONFINITE;
                float q = x / s[h];
                cache[((blk * H + h) * B + slot) * D + d] = orc_e4m3_encode(q);
            }
        }
    }
    return ORC_OK;
}

/* Attention of Tq queries q [Tq, Hq, D] (binary64) at positions
 * ctx - Tq .. ctx - 1 over the first ctx tokens of the paged K / V caches
 * [num_blocks, Hkv, B, D]; causal: query i sees positions <= ctx - Tq + i.
 * out [Tq, Hq, D] binary64. */
int orc_attention_paged(const double *q, int64_t Tq, int64_t Hq, int64_t D, const uint8_t *kcache,
                        const uint8_t *vcache, const float *sk, const float *sv, int64_t Hkv, int64_t B,
                        const int32_t *block_table, int64_t num_blocks, int64_t ctx, double *out, double *scratch)
{
    if (Tq < 1 || Hq < 1 || D < 1 || Hkv < 1 || Hq % Hkv != 0 || B < 1 || ctx < Tq)
        return ORC_ERR_ARG;
    const int64_t G = Hq / Hkv;
    const double inv = 1.0 / sqrt((double)D);
    for (int64_t i = 0; i < Tq; ++i) {
        const int64_t last = ctx - Tq + i;   /* causal: keys 0 .. last */
        for (int64_t h = 0; h < Hq; ++h) {
            const int64_t hk = h / G;
            const double *qv = q + (i * Hq + h) * D;
            double mx = -INFINITY;
            for (int64_t t = 0; t <= last; ++t) {
                int64_t blk = block_table[t / B];
                if (blk < 0 || blk >= num_blocks)
                    return ORC_ERR_ARG;
                const uint8_t *kr = kcache + ((blk * Hkv + hk) * B + t % B) * D;
                double dot = 0.0;
                for (int64_t d = 0; d < D; ++d)
                    dot += qv[d] * orc_e4m3_decode(kr[d]) * (double)sk[hk];
                scratch[t] = dot * inv;
                if (scratch[t] > mx)
                    mx = scratch[t];
            }
            double den = 0.0;
            for (int64_t t = 0; t <= last; ++t) {
                scratch[t] = exp(scratch[t] - mx);
                den += scratch[t];
            }
            double *o = out + (i * Hq + h) * D;
            for (int64_t d = 0; d < D; ++d)
                o[d] = 0.0;
            for (int64_t t = 0; t <= last; ++t) {
                int64_t blk = block_table[t / B];
                const uint8_t *vr = vcache + ((blk * Hkv + hk) * B + t % B) * D;
                const double p = scratch[t] / den;
                for (int64_t d = 0; d < D; ++d)
                    o[d] += p * orc_e4m3_decode(vr[d]) * (double)sv[hk];
            }
        }
    }
    return ORC_OK;
}
