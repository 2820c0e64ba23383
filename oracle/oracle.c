/*
 * oracle.c — plain fp64 CPU oracle for the Inkling decoder attention layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or helper
 * with the CUDA library; the two meet only through seeded input arrays.
 *
 * What it computes (vLLM Recipes page "thinkingmachines/Inkling", section
 * Overview, "Architectural highlights" bullets Attention and Short
 * convolution; the bitbyai.com summary "TML Inkling on vLLM", section "What
 * makes Inkling different?"):
 *
 *   sconv   y[t,c] = bf16_rne( sum_{k=0..3} w[c,k] * x[t-k,c] )
 *           depthwise, window 4, tap 0 = current token, separate weights for
 *           keys and values; history before t=0 is zero (prefill) or the
 *           3 raw tokens held in the rolling state (decode).
 *   logits  s[i,j] = (q_i . Kc_j) / sqrt(d) + bias[h, min(i-j, D_max)]
 *           (relative-position term added to the pre-softmax logits in place
 *           of RoPE; grouped-query attention at head size 128, kv head =
 *           h / (Hq/Hkv)).
 *   mask    j allowed iff 0 <= i-j and (W == 0 or i-j < W)
 *           (sliding-window layers vs full-attention layers).
 *   softmax brute force per row: m = max s, p = exp(s-m), out = sum p Vc / sum p,
 *           lse = m + log(sum p); all in fp64, output not rounded.
 *   paging  the decode cache is [num_blocks, Hkv, 128, d]; token position j of
 *           sequence s lives in block block_table[s, j/128], slot j%128
 *           (block size 128 from the MI355X launch line of the same page).
 *
 * Every step is written out in the order above: no blocking, fusion or
 * reordering.  OpenMP only splits independent rows across host cores.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- bf16 -- */

/* bf16 bit pattern -> exact double value. */
double oracle_bf16_to_f64(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* double -> bf16 bit pattern, one rounding, to nearest with ties to even.
 * bf16 has 8 exponent bits and 7 stored mantissa bits: a normal value with
 * binary exponent e is a multiple of 2^(e-7); below 2^-126 the spacing stays
 * 2^-133 (subnormals).  The value is scaled to units of that spacing, rounded
 * with rint() (default rounding mode: nearest, ties to even), scaled back
 * (exactly), and then reinterpreted through float, which holds every bf16
 * value exactly. */
uint16_t oracle_f64_to_bf16_rne(double x)
{
    if (isnan(x)) return (uint16_t)0x7FC0;
    uint16_t sign = signbit(x) ? (uint16_t)0x8000 : (uint16_t)0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80);
    int e2;
    frexp(a, &e2);               /* a = f * 2^e2, f in [0.5, 1) */
    int e = e2 - 1;              /* a = m * 2^e,  m in [1, 2)   */
    if (e < -126) e = -126;      /* subnormal range keeps the spacing */
    int qexp = e - 7;
    double units = rint(ldexp(a, -qexp));
    double r = ldexp(units, qexp);
    if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80);  /* overflow -> inf */
    float f = (float)r;          /* exact: r is a bf16 value */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* --------------------------------------------------------------- sconv -- */

/* Causal depthwise window-4 short convolution over one batch of rows.
 *   x     [B, T, C] bf16 raw inputs
 *   hist  [B, 3, C] bf16 raw history (slot 0 = x[-3], 1 = x[-2], 2 = x[-1]),
 *         or NULL for zero history
 *   w     [C, 4] fp32, w[c,0] multiplies the current token
 *   y     [B, T, C] bf16 output, rounded once from the fp64 sum */
void oracle_sconv(const uint16_t *x, const uint16_t *hist, const float *w,
                  int64_t B, int64_t T, int64_t C, uint16_t *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t t = 0; t < T; ++t) {
            for (int64_t c = 0; c < C; ++c) {
                double acc = 0.0;
                for (int k = 0; k < 4; ++k) {
                    int64_t src = t - k;
                    double xv;
                    if (src >= 0) {
                        xv = oracle_bf16_to_f64(x[(b * T + src) * C + c]);
                    } else if (hist != NULL) {
                        xv = oracle_bf16_to_f64(hist[(b * 3 + (3 + src)) * C + c]);
                    } else {
                        xv = 0.0;
                    }
                    acc += (double)w[c * 4 + k] * xv;
                }
                y[(b * T + t) * C + c] = oracle_f64_to_bf16_rne(acc);
            }
        }
    }
}

/* Decode-side append: n_new raw tokens per sequence are convolved against the
 * rolling 3-token state, written to their slots in the paged cache, and the
 * state is replaced by the last 3 raw tokens of (state ++ new tokens).
 *   x_new       [S, n_new, Hkv, d] bf16 raw keys (or values)
 *   state       [S, 3, Hkv*d] bf16, updated in place
 *   w           [Hkv*d, 4] fp32
 *   cache       [num_blocks, Hkv, 128, d] bf16, slots written in place
 *   block_table [S, max_blocks] int32
 *   seq_lens    [S] int32: length after appending; new tokens sit at
 *               positions L-n_new .. L-1 */
void oracle_sconv_append(const uint16_t *x_new, uint16_t *state, const float *w,
                         uint16_t *cache, const int32_t *block_table,
                         const int32_t *seq_lens, int64_t S, int64_t n_new,
                         int64_t Hkv, int64_t d, int64_t max_blocks)
{
    const int64_t C = Hkv * d;
#pragma omp parallel for schedule(static)
    for (int64_t s = 0; s < S; ++s) {
        /* extended raw sequence: 3 history tokens then the new ones */
        int64_t n_ext = 3 + n_new;
        uint16_t *ext = (uint16_t *)malloc((size_t)(n_ext * C) * sizeof(uint16_t));
        for (int64_t t = 0; t < 3; ++t)
            memcpy(ext + t * C, state + (s * 3 + t) * C, (size_t)C * sizeof(uint16_t));
        for (int64_t t = 0; t < n_new; ++t)
            memcpy(ext + (3 + t) * C, x_new + (s * n_new + t) * C, (size_t)C * sizeof(uint16_t));
        int64_t L = seq_lens[s];
        for (int64_t t = 0; t < n_new; ++t) {
            int64_t pos = L - n_new + t;
            int64_t blk = block_table[s * max_blocks + pos / 128];
            int64_t slot = pos % 128;
            for (int64_t c = 0; c < C; ++c) {
                double acc = 0.0;
                for (int k = 0; k < 4; ++k)
                    acc += (double)w[c * 4 + k] * oracle_bf16_to_f64(ext[(3 + t - k) * C + c]);
                int64_t kvh = c / d, e = c % d;
                cache[((blk * Hkv + kvh) * 128 + slot) * d + e] = oracle_f64_to_bf16_rne(acc);
            }
        }
        for (int64_t t = 0; t < 3; ++t)
            memcpy(state + (s * 3 + t) * C, ext + (n_ext - 3 + t) * C, (size_t)C * sizeof(uint16_t));
        free(ext);
    }
}

/* ------------------------------------------------------------ attention -- */

/* One query row.  key_row(j) / val_row(j) give the post-sconv key and value of
 * position j for this row's kv head.  Keys are positions 0 .. n_keys-1; the
 * query sits at position i.  Returns lse; writes d fp64 outputs. */
typedef const uint16_t *(*row_fn)(const void *ctx, int64_t j);

static double attn_row(const uint16_t *q, row_fn key_row, row_fn val_row,
                       const void *ctx, int64_t i, int64_t n_keys, int64_t window,
                       int64_t d, const float *bias_h, int64_t D_max, double *out)
{
    const double scale = 1.0 / sqrt((double)d);
    int64_t lo = 0;
    if (window > 0 && i - window + 1 > lo) lo = i - window + 1;
    int64_t hi = i < n_keys - 1 ? i : n_keys - 1;      /* causal: j <= i */
    int64_t n = hi - lo + 1;
    double *s = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    /* logits */
    for (int64_t j = lo; j <= hi; ++j) {
        const uint16_t *k = key_row(ctx, j);
        double dot = 0.0;
        for (int64_t e = 0; e < d; ++e)
            dot += oracle_bf16_to_f64(q[e]) * oracle_bf16_to_f64(k[e]);
        int64_t dist = i - j;
        int64_t idx = dist < D_max ? dist : D_max;
        s[j - lo] = dot * scale + (double)bias_h[idx];
    }
    /* softmax */
    double m = -INFINITY;
    for (int64_t t = 0; t < n; ++t)
        if (s[t] > m) m = s[t];
    double l = 0.0;
    for (int64_t t = 0; t < n; ++t) {
        s[t] = exp(s[t] - m);
        l += s[t];
    }
    /* weighted sum of values */
    for (int64_t e = 0; e < d; ++e) out[e] = 0.0;
    for (int64_t j = lo; j <= hi; ++j) {
        const uint16_t *v = val_row(ctx, j);
        double p = s[j - lo];
        for (int64_t e = 0; e < d; ++e) out[e] += p * oracle_bf16_to_f64(v[e]);
    }
    for (int64_t e = 0; e < d; ++e) out[e] /= l;
    free(s);
    return m + log(l);
}

/* contiguous [B, T, Hkv, d] keys/values */
typedef struct {
    const uint16_t *k, *v;
    int64_t b, kvh, T, Hkv, d;
} dense_ctx;

static const uint16_t *dense_key(const void *p, int64_t j)
{
    const dense_ctx *c = (const dense_ctx *)p;
    return c->k + ((c->b * c->T + j) * c->Hkv + c->kvh) * c->d;
}
static const uint16_t *dense_val(const void *p, int64_t j)
{
    const dense_ctx *c = (const dense_ctx *)p;
    return c->v + ((c->b * c->T + j) * c->Hkv + c->kvh) * c->d;
}

/* Attention rows over already-convolved keys and values.
 *   q      [B, T, Hq, d] bf16
 *   kc, vc [B, T, Hkv, d] bf16 (post-sconv)
 *   bias   [Hq, D_max+1] fp32
 *   rows   n_rows triples (b, h, i) of query rows to compute
 *   out    [n_rows, d] fp64; lse [n_rows] fp64 (nullable) */
void oracle_attention_rows(const uint16_t *q, const uint16_t *kc, const uint16_t *vc,
                           const float *bias, int64_t B, int64_t T, int64_t Hq,
                           int64_t Hkv, int64_t d, int64_t window, int64_t D_max,
                           const int32_t *rows, int64_t n_rows, double *out,
                           double *lse)
{
    (void)B;
    const int64_t G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
        dense_ctx ctx = {kc, vc, b, h / G, T, Hkv, d};
        double l = attn_row(q + ((b * T + i) * Hq + h) * d, dense_key, dense_val, &ctx,
                            i, T, window, d, bias + h * (D_max + 1), D_max, out + r * d);
        if (lse) lse[r] = l;
    }
}

/* Full prefill for selected rows: sconv of raw keys and values with zero
 * history (rounded to bf16), then attention rows.  kc_out / vc_out receive
 * the convolved keys and values ([B, T, Hkv, d] bf16, caller-allocated). */
void oracle_prefill_rows(const uint16_t *q, const uint16_t *k_raw, const uint16_t *v_raw,
                         const float *w_k, const float *w_v, const float *bias,
                         int64_t B, int64_t T, int64_t Hq, int64_t Hkv, int64_t d,
                         int64_t window, int64_t D_max, const int32_t *rows,
                         int64_t n_rows, double *out, double *lse,
                         uint16_t *kc_out, uint16_t *vc_out)
{
    oracle_sconv(k_raw, NULL, w_k, B, T, Hkv * d, kc_out);
    oracle_sconv(v_raw, NULL, w_v, B, T, Hkv * d, vc_out);
    oracle_attention_rows(q, kc_out, vc_out, bias, B, T, Hq, Hkv, d, window, D_max,
                          rows, n_rows, out, lse);
}

/* paged [num_blocks, Hkv, 128, d] keys/values through a block table */
typedef struct {
    const uint16_t *k, *v;
    const int32_t *bt;  /* this sequence's block-table row */
    int64_t kvh, Hkv, d;
} paged_ctx;

static const uint16_t *paged_key(const void *p, int64_t j)
{
    const paged_ctx *c = (const paged_ctx *)p;
    int64_t blk = c->bt[j / 128];
    return c->k + ((blk * c->Hkv + c->kvh) * 128 + j % 128) * c->d;
}
static const uint16_t *paged_val(const void *p, int64_t j)
{
    const paged_ctx *c = (const paged_ctx *)p;
    int64_t blk = c->bt[j / 128];
    return c->v + ((blk * c->Hkv + c->kvh) * 128 + j % 128) * c->d;
}

/* Single-token decode for selected (sequence, head) pairs: the query is at
 * position L-1 and attends to keys 0 .. L-1 of its sequence through the
 * block table (window-limited when window > 0).
 *   q           [S, Hq, d] bf16
 *   k_cache     [num_blocks, Hkv, 128, d] bf16 (post-sconv)
 *   block_table [S, max_blocks] int32;  seq_lens [S] int32
 *   pairs       n_pairs pairs (s, h); out [n_pairs, d] fp64; lse [n_pairs] */
void oracle_decode_rows(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                        const int32_t *block_table, const int32_t *seq_lens,
                        const float *bias, int64_t Hq, int64_t Hkv, int64_t d,
                        int64_t max_blocks, int64_t window, int64_t D_max,
                        const int32_t *pairs, int64_t n_pairs, double *out, double *lse)
{
    const int64_t G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_pairs; ++r) {
        int64_t s = pairs[2 * r], h = pairs[2 * r + 1];
        int64_t L = seq_lens[s];
        paged_ctx ctx = {k_cache, v_cache, block_table + s * max_blocks, h / G, Hkv, d};
        double l = attn_row(q + (s * Hq + h) * d, paged_key, paged_val, &ctx, L - 1, L,
                            window, d, bias + h * (D_max + 1), D_max, out + r * d);
        if (lse) lse[r] = l;
    }
}

/* Multi-token decode (draft tokens of speculative decoding / multi-token
 * prediction, vLLM Recipes "thinkingmachines/Inkling", Overview, MTP bullet:
 * up to 9 tokens per forward step).  A sequence of length L (the q_len new
 * tokens already appended to the cache) has queries q [S, q_len, Hq, d];
 * query qi sits at position i = L - q_len + qi and sees keys j <= i (inside
 * the window), with the bias at distance i - j.  rows holds (s, qi, h)
 * triples; out and lse are per row. */
void oracle_decode_mq_rows(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                           const int32_t *block_table, const int32_t *seq_lens,
                           const float *bias, int64_t Hq, int64_t Hkv, int64_t d,
                           int64_t max_blocks, int64_t window, int64_t D_max, int64_t q_len,
                           const int32_t *rows, int64_t n_rows, double *out, double *lse)
{
    const int64_t G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t s = rows[3 * r], qi = rows[3 * r + 1], h = rows[3 * r + 2];
        int64_t L = seq_lens[s];
        paged_ctx ctx = {k_cache, v_cache, block_table + s * max_blocks, h / G, Hkv, d};
        double l = attn_row(q + ((s * q_len + qi) * Hq + h) * d, paged_key, paged_val, &ctx,
                            L - q_len + qi, L, window, d, bias + h * (D_max + 1), D_max,
                            out + r * d);
        if (lse) lse[r] = l;
    }
}
