/*
 * MiniKV CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct CPU restatement of what the MiniKV hot path
 * computes.  Only the test suite, the smoke check and the CPU-baseline leg of the
 * benchmark may load this file's shared library.  It shares no code, header,
 * table or helper with the CUDA library and includes none of it.
 *
 * Sources (the only description of the method there is):
 *   [abstract]  "MiniKV: Pushing the Limits of LLM Inference via 2-Bit
 *               Layer-Discriminative KV Cache", paper abstract (2-bit KV cache,
 *               layer-discriminative, kernels compatible with FlashAttention).
 *   [summary]   gptget.net/papers/2411.18077, sections "方法论" (methodology) and
 *               "方法详解" (method details): sub-channel key quantization,
 *               per-token value quantization, compact layout; adaptive KV keeps
 *               tokens by importance; selective flash attention done with a
 *               second kernel.
 *   [glossary]  same page, "术语表": adaptive KV = keep KV states by importance.
 *   [table]     pre.notesum.ai 2411.18077v1, LongBench table, "MiniKV Pyramid"
 *               rows (layer-discriminative budget).
 * The pages give names, not formulas.  Every concrete choice below is the
 * plainest reading, listed with its reason in the design notes:
 *   O1  causal softmax attention, fp64                    [abstract]
 *   O2  window score = sum of softmax mass over the last W queries and the
 *       query heads that share a KV head                  [summary, 方法详解]
 *   O3  keep window + top-(keep-W) by score, ties -> lower index [glossary]
 *   O5  split: newest r tokens stay fp16 (R <= r < R+G)
 *   O6  asymmetric min/max 2-bit quantizer, fp16 scale/zero, exact fp32 steps
 *       keys: per channel over G tokens; values: per token over Gv channels
 *                                                         [summary, 方法论]
 *   O7  16 codes per little-endian 32-bit word, channel 16w+i at bits 2i..2i+1
 *   O8  dequant x^ = c*scale + zero (exact in fp64)
 *   O9  decode: attend over dequantized packed tokens + fp16 residual, fp64
 *   O10 decode-time attention mass (H2O-style accumulated score): each step
 *       adds, per cached token, its softmax probability summed over the query
 *       heads of the KV head                             [summary, 实验设计]
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared
 * (no FMA contraction, SSE2 float arithmetic, IEEE round-to-nearest-even).
 * fp16 values travel as their 16-bit patterns (uint16_t).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ fp16 */

/* IEEE binary16 bit pattern -> exact double. */
double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);              /* zero / subnormal */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);  /* (1.m) * 2^(e-15) */
    return sign ? -v : v;
}

/* float -> binary16, round to nearest, ties to even.  Works in double, where
 * every step below is exact (a float has at most 24 significant bits). */
uint16_t oracle_float_to_half(float f)
{
    uint16_t sign = signbit(f) ? 0x8000 : 0;
    double a = fabs((double)f);
    if (isnan(f)) return sign | 0x7e00;
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: units of 2^-24; rounding up to 1024 lands exactly on
         * the smallest normal, whose pattern is 0x400. */
        double q = nearbyint(ldexp(a, 24));
        return sign | (uint16_t)q;
    }
    int e;
    (void)frexp(a, &e);          /* a = f * 2^e, f in [0.5, 1) */
    e -= 1;                      /* a in [2^e, 2^(e+1)) */
    double q = nearbyint(ldexp(a, 10 - e)); /* significand in [1024, 2048] */
    if (q == 2048.0) { q = 1024.0; e += 1; }
    if (e + 15 >= 31) return sign | 0x7c00; /* overflow -> inf */
    return sign | (uint16_t)(((e + 15) << 10) | ((int)q - 1024));
}

static float h2f(uint16_t h) { return (float)oracle_half_to_double(h); }

/* ------------------------------------------------------- O5: the split */

/* N kept tokens -> n_q packed tokens (a multiple of G) and r fp16 residual
 * tokens.  The newest tokens stay fp16: R <= r <= R+G-1 once N >= R. */
void oracle_split(int N, int R, int G, int *n_q, int *r)
{
    if (N >= R) {
        *r = R + (N - R) % G;
        *n_q = N - *r;
    } else {
        *r = N;
        *n_q = 0;
    }
}

/* ------------------------------------------------ O6: quantize one group */

/* Quantize n fp16 values x[i*stride] to 2-bit codes with one fp16 scale and
 * zero (asymmetric min/max).  Every fp32 step is a single IEEE
 * round-to-nearest-even operation, in this order:
 *   mn = min x, mx = max x                (exact; a zero extreme is taken as +0)
 *   scale = half( float(mx) - float(mn) ) / 3 )
 *   zero  = mn
 *   c = 0 if scale == 0, else clamp(rint((float(x) - float(zero)) / float(scale)), 0, 3)
 */
void oracle_quantize_group(const uint16_t *x, int n, long stride,
                           uint16_t *scale_out, uint16_t *zero_out, uint8_t *codes)
{
    float mn = INFINITY, mx = -INFINITY;
    uint16_t mn_bits = 0;
    for (int i = 0; i < n; ++i) {
        float v = h2f(x[(long)i * stride]);
        if (v < mn) { mn = v; mn_bits = x[(long)i * stride]; }
        if (v > mx) mx = v;
    }
    /* -0 and +0 are one value: a zero extreme is taken as +0 */
    if (mn == 0.0f) { mn = 0.0f; mn_bits = 0; }
    if (mx == 0.0f) mx = 0.0f;
    volatile float diff = mx - mn;                 /* fp32 subtract */
    volatile float s32 = diff / 3.0f;              /* fp32 divide */
    uint16_t scale = oracle_float_to_half(s32);
    float s = h2f(scale);
    *scale_out = scale;
    *zero_out = mn_bits;
    for (int i = 0; i < n; ++i) {
        int c = 0;
        if (s != 0.0f) {
            volatile float num = h2f(x[(long)i * stride]) - mn;
            volatile float q = num / s;
            float rq = nearbyintf(q);              /* ties to even */
            c = rq < 0.0f ? 0 : (rq > 3.0f ? 3 : (int)rq);
        }
        codes[i] = (uint8_t)c;
    }
}

/* ------------------------------------------------------- O7: bit packing */

/* codes[D] (one token) -> D/16 words; channel 16w+i goes to bits 2i..2i+1 of w */
void oracle_pack_token(const uint8_t *codes, int D, uint32_t *words)
{
    for (int w = 0; w < D / 16; ++w) {
        uint32_t acc = 0;
        for (int i = 0; i < 16; ++i)
            acc |= (uint32_t)(codes[16 * w + i] & 3u) << (2 * i);
        words[w] = acc;
    }
}

static int code_at(const uint32_t *words, int c)
{
    return (int)((words[c / 16] >> (2 * (c % 16))) & 3u);
}

/* ------------------------------------- O5-O7: pack one (b, kv-head) slice */

/* k, v: [n_q, D] fp16 (the oldest n_q kept tokens; n_q a multiple of G).
 * k_codes, v_codes: [n_q, D/16]; k_scale, k_zero: [n_q/G, D];
 * v_scale, v_zero: [n_q, D/Gv].  Keys: one (scale, zero) per channel per
 * group of G consecutive tokens, groups aligned to token 0.  Values: one
 * (scale, zero) per token per block of Gv consecutive channels. */
void oracle_pack_tokens(const uint16_t *k, const uint16_t *v, int n_q, int D, int G, int Gv,
                        uint32_t *k_codes, uint16_t *k_scale, uint16_t *k_zero,
                        uint32_t *v_codes, uint16_t *v_scale, uint16_t *v_zero)
{
    uint8_t *kc = (uint8_t *)malloc((size_t)n_q * D + 1);
    uint8_t *vc = (uint8_t *)malloc((size_t)n_q * D + 1);
    uint8_t *tmp = (uint8_t *)malloc((size_t)(G > D ? G : D) + 1);
    for (int g = 0; g < n_q / G; ++g)
        for (int c = 0; c < D; ++c) {
            oracle_quantize_group(k + (long)g * G * D + c, G, D,
                                  &k_scale[(long)g * D + c], &k_zero[(long)g * D + c], tmp);
            for (int t = 0; t < G; ++t) kc[(long)(g * G + t) * D + c] = tmp[t];
        }
    for (int t = 0; t < n_q; ++t)
        for (int j = 0; j < D / Gv; ++j)
            oracle_quantize_group(v + (long)t * D + (long)j * Gv, Gv, 1,
                                  &v_scale[(long)t * (D / Gv) + j], &v_zero[(long)t * (D / Gv) + j],
                                  vc + (long)t * D + (long)j * Gv);
    for (int t = 0; t < n_q; ++t) {
        oracle_pack_token(kc + (long)t * D, D, k_codes + (long)t * (D / 16));
        oracle_pack_token(vc + (long)t * D, D, v_codes + (long)t * (D / 16));
    }
    free(kc); free(vc); free(tmp);
}

/* --------------------------------------------------- O8: dequantization */

/* Dequantize packed tokens [0, n_q) of one slice into fp64 rows [n_q, D]. */
void oracle_dequant_tokens(const uint32_t *k_codes, const uint16_t *k_scale, const uint16_t *k_zero,
                           const uint32_t *v_codes, const uint16_t *v_scale, const uint16_t *v_zero,
                           int n_q, int D, int G, int Gv, double *k_hat, double *v_hat)
{
    for (int t = 0; t < n_q; ++t) {
        const uint32_t *kw = k_codes + (long)t * (D / 16);
        const uint32_t *vw = v_codes + (long)t * (D / 16);
        for (int c = 0; c < D; ++c) {
            long ks = (long)(t / G) * D + c;
            long vs = (long)t * (D / Gv) + c / Gv;
            k_hat[(long)t * D + c] = code_at(kw, c) * oracle_half_to_double(k_scale[ks])
                                   + oracle_half_to_double(k_zero[ks]);
            v_hat[(long)t * D + c] = code_at(vw, c) * oracle_half_to_double(v_scale[vs])
                                   + oracle_half_to_double(v_zero[vs]);
        }
    }
}

/* ---------------------------------------------- O1: prefill attention */

/* One query head: q, k, v [T, D] fp16 -> o [T, D] fp64.
 * o[i] = sum_{j<=i} softmax_j(tau * q_i . k_j) v_j  (causal, no other mask). */
void oracle_prefill_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                              int T, int D, double tau, double *o)
{
    double *kd = (double *)malloc(sizeof(double) * (size_t)T * D + 8);
    double *vd = (double *)malloc(sizeof(double) * (size_t)T * D + 8);
    double *p = (double *)malloc(sizeof(double) * (size_t)T + 8);
    double *qi = (double *)malloc(sizeof(double) * (size_t)D + 8);
    for (long n = 0; n < (long)T * D; ++n) {
        kd[n] = oracle_half_to_double(k[n]);
        vd[n] = oracle_half_to_double(v[n]);
    }
    for (int i = 0; i < T; ++i) {
        for (int c = 0; c < D; ++c) qi[c] = oracle_half_to_double(q[(long)i * D + c]);
        double m = -INFINITY;
        for (int j = 0; j <= i; ++j) {
            double s = 0.0;
            for (int c = 0; c < D; ++c) s += qi[c] * kd[(long)j * D + c];
            p[j] = tau * s;
            if (p[j] > m) m = p[j];
        }
        double l = 0.0;
        for (int j = 0; j <= i; ++j) { p[j] = exp(p[j] - m); l += p[j]; }
        for (int c = 0; c < D; ++c) {
            double acc = 0.0;
            for (int j = 0; j <= i; ++j) acc += p[j] * vd[(long)j * D + c];
            o[(long)i * D + c] = acc / l;
        }
    }
    free(kd); free(vd); free(p); free(qi);
}

/* O1 for selected query rows only: rows[n] in [0, T); out [nrows, D] fp64.
 * Row i is the same computation as in oracle_prefill_attention. */
void oracle_prefill_attention_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v, int T, int D,
                                   double tau, const int32_t *rows, int nrows, double *out)
{
    double *p = (double *)malloc(sizeof(double) * (size_t)T + 8);
    double *qi = (double *)malloc(sizeof(double) * (size_t)D + 8);
    for (int n = 0; n < nrows; ++n) {
        int i = rows[n];
        for (int c = 0; c < D; ++c) qi[c] = oracle_half_to_double(q[(long)i * D + c]);
        double m = -INFINITY;
        for (int j = 0; j <= i; ++j) {
            double s = 0.0;
            for (int c = 0; c < D; ++c) s += qi[c] * oracle_half_to_double(k[(long)j * D + c]);
            p[j] = tau * s;
            if (p[j] > m) m = p[j];
        }
        double l = 0.0;
        for (int j = 0; j <= i; ++j) { p[j] = exp(p[j] - m); l += p[j]; }
        for (int c = 0; c < D; ++c) {
            double acc = 0.0;
            for (int j = 0; j <= i; ++j) acc += p[j] * oracle_half_to_double(v[(long)j * D + c]);
            out[(long)n * D + c] = acc / l;
        }
    }
    free(p); free(qi);
}

/* ------------------------------------------- O2: observation-window scores */

/* One KV head.  q: [g, T, D] fp16 (the g query heads that read this KV head),
 * k: [T, D] fp16.  s[j] = sum over those heads h and the last W query rows i
 * of the causal softmax probability P_h[i, j] (zero for j > i). */
void oracle_window_scores(const uint16_t *q, const uint16_t *k, int g, int T, int D, int W,
                          double tau, double *s)
{
    double *kd = (double *)malloc(sizeof(double) * (size_t)T * D + 8);
    double *p = (double *)malloc(sizeof(double) * (size_t)T + 8);
    double *qi = (double *)malloc(sizeof(double) * (size_t)D + 8);
    for (long n = 0; n < (long)T * D; ++n) kd[n] = oracle_half_to_double(k[n]);
    for (int j = 0; j < T; ++j) s[j] = 0.0;
    for (int h = 0; h < g; ++h)
        for (int i = T - W; i < T; ++i) {
            for (int c = 0; c < D; ++c) qi[c] = oracle_half_to_double(q[((long)h * T + i) * D + c]);
            double m = -INFINITY;
            for (int j = 0; j <= i; ++j) {
                double a = 0.0;
                for (int c = 0; c < D; ++c) a += qi[c] * kd[(long)j * D + c];
                p[j] = tau * a;
                if (p[j] > m) m = p[j];
            }
            double l = 0.0;
            for (int j = 0; j <= i; ++j) { p[j] = exp(p[j] - m); l += p[j]; }
            for (int j = 0; j <= i; ++j) s[j] += p[j] / l;
        }
    free(kd); free(p); free(qi);
}

/* ----------------------------------------------------------- O3: select */

static const double *g_sel_scores;
static int cmp_candidates(const void *a, const void *b)
{
    int i = *(const int *)a, j = *(const int *)b;
    double si = g_sel_scores[i], sj = g_sel_scores[j];
    if (si > sj) return -1;          /* higher score first */
    if (si < sj) return 1;
    return (i > j) - (i < j);        /* equal score: lower index first */
}
static int cmp_int(const void *a, const void *b)
{
    int i = *(const int *)a, j = *(const int *)b;
    return (i > j) - (i < j);
}

/* Keep `keep` of T positions.  keep >= T keeps all T.  Otherwise (W <= keep
 * required) the window [T-W, T) is always kept and the remaining keep-W are the
 * candidates j < T-W that come first in (score descending, index ascending).
 * idx receives the kept positions in ascending order.  Returns the number
 * kept, or -1 on bad arguments. */
int oracle_select(const double *s, int T, int W, int keep, int32_t *idx)
{
    if (T <= 0 || W < 0 || keep < 0) return -1;
    if (keep >= T) {
        for (int j = 0; j < T; ++j) idx[j] = j;
        return T;
    }
    if (W > keep) return -1;
    int nc = T - W;
    int *cand = (int *)malloc(sizeof(int) * (size_t)(nc > 0 ? nc : 1));
    for (int j = 0; j < nc; ++j) cand[j] = j;
    g_sel_scores = s;
    qsort(cand, (size_t)nc, sizeof(int), cmp_candidates);
    int n = 0;
    for (int j = 0; j < keep - W; ++j) idx[n++] = cand[j];
    for (int j = T - W; j < T; ++j) idx[n++] = j;
    qsort(idx, (size_t)n, sizeof(int32_t), cmp_int);
    free(cand);
    return n;
}

/* --------------------------------------------------- O9: decode attention */

/* One KV head, one step, after the new token has been appended to the
 * residual.  q: [g, D] fp16.  The cache holds n_q packed tokens (layout of
 * O5-O7) followed by the residual res_k/res_v [r, D] fp16, oldest first.
 * out[h] = sum_t softmax_t(tau * q_h . kappa_t) nu_t over all n_q + r tokens,
 * kappa/nu the dequantized (O8) packed rows and the raw residual rows; fp64.
 * If mass is not NULL, O10 as well: mass[t] = sum_h softmax_t(tau * q_h .
 * kappa_t) for t in [0, n_q + r), packed tokens first, then the residual
 * oldest first (the order in which the tokens entered the cache). */
static void decode_attention_impl(const uint16_t *q, int g,
                                  const uint32_t *k_codes, const uint16_t *k_scale, const uint16_t *k_zero,
                                  const uint32_t *v_codes, const uint16_t *v_scale, const uint16_t *v_zero,
                                  int n_q, const uint16_t *res_k, const uint16_t *res_v, int r,
                                  int D, int G, int Gv, double tau, double *out, double *mass)
{
    int n = n_q + r;
    double *kh = (double *)malloc(sizeof(double) * ((size_t)n * D + 1));
    double *vh = (double *)malloc(sizeof(double) * ((size_t)n * D + 1));
    double *p = (double *)malloc(sizeof(double) * ((size_t)n + 1));
    oracle_dequant_tokens(k_codes, k_scale, k_zero, v_codes, v_scale, v_zero, n_q, D, G, Gv, kh, vh);
    for (long e = 0; e < (long)r * D; ++e) {
        kh[(long)n_q * D + e] = oracle_half_to_double(res_k[e]);
        vh[(long)n_q * D + e] = oracle_half_to_double(res_v[e]);
    }
    if (mass)
        for (int t = 0; t < n; ++t) mass[t] = 0.0;
    for (int h = 0; h < g; ++h) {
        double m = -INFINITY;
        for (int t = 0; t < n; ++t) {
            double a = 0.0;
            for (int c = 0; c < D; ++c) a += oracle_half_to_double(q[(long)h * D + c]) * kh[(long)t * D + c];
            p[t] = tau * a;
            if (p[t] > m) m = p[t];
        }
        double l = 0.0;
        for (int t = 0; t < n; ++t) { p[t] = exp(p[t] - m); l += p[t]; }
        for (int c = 0; c < D; ++c) {
            double acc = 0.0;
            for (int t = 0; t < n; ++t) acc += p[t] * vh[(long)t * D + c];
            out[(long)h * D + c] = acc / l;
        }
        if (mass)
            for (int t = 0; t < n; ++t) mass[t] += p[t] / l;
    }
    free(kh); free(vh); free(p);
}

void oracle_decode_attention(const uint16_t *q, int g,
                             const uint32_t *k_codes, const uint16_t *k_scale, const uint16_t *k_zero,
                             const uint32_t *v_codes, const uint16_t *v_scale, const uint16_t *v_zero,
                             int n_q, const uint16_t *res_k, const uint16_t *res_v, int r,
                             int D, int G, int Gv, double tau, double *out)
{
    decode_attention_impl(q, g, k_codes, k_scale, k_zero, v_codes, v_scale, v_zero, n_q, res_k, res_v, r,
                          D, G, Gv, tau, out, NULL);
}

/* ------------------------------------------- O10: decode attention mass */

/* O9 plus this step's attention mass of every cached token (see
 * decode_attention_impl): mass [n_q + r] fp64, overwritten.  H2O, the
 * accumulated-attention eviction the summary's experiments compare against,
 * ranks tokens by the sum of these per-step masses; the caller accumulates. */
void oracle_decode_attention_mass(const uint16_t *q, int g,
                                  const uint32_t *k_codes, const uint16_t *k_scale, const uint16_t *k_zero,
                                  const uint32_t *v_codes, const uint16_t *v_scale, const uint16_t *v_zero,
                                  int n_q, const uint16_t *res_k, const uint16_t *res_v, int r,
                                  int D, int G, int Gv, double tau, double *out, double *mass)
{
    decode_attention_impl(q, g, k_codes, k_scale, k_zero, v_codes, v_scale, v_zero, n_q, res_k, res_v, r,
                          D, G, Gv, tau, out, mass);
}
