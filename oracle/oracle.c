/*
 * oracle.c -- TEST INFRASTRUCTURE ONLY.  Plain, slow, fp64 CPU statement of
 * what the prefill attention path computes.  Only the tests, the smoke check
 * and the bench's CPU-baseline leg may load this library; the product path
 * never does.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes (per sequence i of a packed batch, query row a, query head h):
 *
 *   absolute position    P  = ctx_i + a                (ctx_i = 0 unless chunked)
 *   kv head              g  = h / (n_head / n_kv_head)  (contiguous GQA groups)
 *   visible keys         j = 0 .. P                     (causal: j <= P)
 *                        j = P - W + 1 .. P (and >= 0)   (sliding window of W keys)
 *   key / value row j    = cache row (page block_table[i][j / bs], slot j % bs)
 *                          if j < ctx_i, else the input row j - ctx_i
 *   score                s_j = scale * sum_d q[d] * k_j[d]
 *   softmax (two pass)   m = max_j s_j ; w_j = exp(s_j - m) ; l = sum_j w_j
 *   output               D = sum_j (w_j / l) * v_j
 *
 * and separately the paged KV write: token t of sequence i lands in page
 * block_table[i][(ctx_i + t) / bs], slot (ctx_i + t) % bs, K half then V half.
 *
 * Sources (page address, section):
 *   hncyxsy.com/news/270449 §2.3 -- per head S = Q K^T, upper triangle
 *       masked (causal), softmax, weighted sum with V, heads concatenated.
 *   hncyxsy.com/news/270449 §3.1 -- S = Q_head K_head^T divided by
 *       sqrt(head_dim); K^T is a logical transpose.
 *   hncyxsy.com/news/270449 §3.2 -- the plain softmax scans S twice (row max,
 *       then exp sum); the weighted sum is D = softmax(S) V.
 *   hncyxsy.com/news/270449 §3.4, hncyxsy.com/news/227904 §3.2 -- GQA:
 *       several query heads share one K/V head.
 *   hncyxsy.com/news/270449 §4.2, hncyxsy.com/news/227904 §3.4 -- the KV cache
 *       is stored in fixed-size blocks reached through a page table.
 *   hncyxsy.com/news/227904 §2.1 -- chunked prefill: a chunk needs the K/V of
 *       all earlier tokens.
 *   lnwmold.com/news/496245 §1.1 -- attention_scores = Q K^T / sqrt(d_head).
 *   lnwmold.com/news/496245 §4.1 -- sliding-window attention: each token
 *       attends only to its W nearest predecessors, n*W work instead of n^2.
 *
 * Readings where the pages are silent:
 *   the scale is the caller's float, widened to fp64; disallowed keys are
 *   left out of the sum (no -inf arithmetic); GQA groups are contiguous; a
 *   chunk is aligned bottom-right (row a sits at absolute position ctx + a);
 *   the cache page is [2][block_size][n_kv_head][head_dim]; the prefix is read
 *   from the cache as it stood before the call; a window of W keys counts the
 *   token itself (row P sees keys P-W+1 .. P, so n rows cost n*W pairs once
 *   P >= W - 1), W = 0 meaning no window.
 *
 * Parity pins: every function here is checked against closed forms,
 * invariants, a brute-force loop and a library routine by the CPU tests.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_BLOCK_TABLE 2
#define ORACLE_ERR_NOMEM 3

/* bfloat16 bits -> double: the 16 bits are the top half of an IEEE binary32. */
static double bf16_bits_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

typedef struct {
    const uint16_t *q, *k, *v;
    const int32_t *cu_seqlens, *context_lens;
    int num_seqs, n_head, n_kv_head, head_dim;
    double scale;
    const uint16_t *kv_cache;
    int num_blocks;
    const int32_t *block_table;
    int max_blocks_per_seq, block_size;
    int window; /* 0: plain causal; W >= 1: keys P-W+1 .. P only */
} problem_t;

/* Sequence holding packed row t (cu_seqlens is non-decreasing). */
static int seq_of_row(const problem_t *p, int t) {
    for (int i = 0; i < p->num_seqs; ++i)
        if (t >= p->cu_seqlens[i] && t < p->cu_seqlens[i + 1]) return i;
    return -1;
}

/* Address of the K (which = 0) or V (which = 1) row for kv head g of absolute
 * key position j of sequence i; NULL if the page table entry is invalid. */
static const uint16_t *kv_row(const problem_t *p, int i, int j, int g, int which) {
    int ctx = p->context_lens ? p->context_lens[i] : 0;
    size_t G = (size_t)p->n_kv_head, d = (size_t)p->head_dim;
    if (j >= ctx) {
        size_t row = (size_t)p->cu_seqlens[i] + (size_t)(j - ctx);
        const uint16_t *base = which ? p->v : p->k;
        return base + (row * G + (size_t)g) * d;
    }
    int lp = j / p->block_size;
    if (lp >= p->max_blocks_per_seq) return NULL;
    int page = p->block_table[(size_t)i * p->max_blocks_per_seq + lp];
    if (page < 0 || page >= p->num_blocks) return NULL;
    size_t slot = (size_t)(j % p->block_size);
    size_t off = (((size_t)page * 2 + (size_t)which) * (size_t)p->block_size + slot) * G + (size_t)g;
    return p->kv_cache + off * d;
}

/* One output row: query row t (packed index), query head h.
 * w: scratch of at least (P + 1) doubles; on return w[j] = softmax weight
 * (exactly 0 for keys outside the window). */
static int attend_one(const problem_t *p, int t, int h, double *out, double *w, int *n_keys) {
    int i = seq_of_row(p, t);
    if (i < 0) return ORACLE_ERR_ARG;
    int ctx = p->context_lens ? p->context_lens[i] : 0;
    int a = t - p->cu_seqlens[i];
    int P = ctx + a;                                   /* absolute position */
    int r = p->n_head / p->n_kv_head;
    int g = h / r;                                     /* contiguous GQA group */
    int d = p->head_dim;
    const uint16_t *qrow = p->q + ((size_t)t * p->n_head + (size_t)h) * (size_t)d;

    double qd[512];
    for (int x = 0; x < d; ++x) qd[x] = bf16_bits_to_double(qrow[x]);
    /* first visible key: 0, or the start of the window ending at P */
    int j0 = 0;
    if (p->window > 0 && P - p->window + 1 > 0) j0 = P - p->window + 1;
    for (int j = 0; j < j0; ++j) w[j] = 0.0;

    /* pass 1: scores and their maximum (keys j0..P; the rest are masked out) */
    double m = -INFINITY;
    for (int j = j0; j <= P; ++j) {
        const uint16_t *krow = kv_row(p, i, j, g, 0);
        if (!krow) return ORACLE_ERR_BLOCK_TABLE;
        double dot = 0.0;
        for (int x = 0; x < d; ++x) dot += qd[x] * bf16_bits_to_double(krow[x]);
        double s = p->scale * dot;
        w[j] = s;
        if (s > m) m = s;
    }
    /* pass 2: exponentials and their sum */
    double l = 0.0;
    for (int j = j0; j <= P; ++j) {
        w[j] = exp(w[j] - m);
        l += w[j];
    }
    for (int j = j0; j <= P; ++j) w[j] /= l;
    /* weighted sum with V */
    for (int x = 0; x < d; ++x) out[x] = 0.0;
    for (int j = j0; j <= P; ++j) {
        const uint16_t *vrow = kv_row(p, i, j, g, 1);
        if (!vrow) return ORACLE_ERR_BLOCK_TABLE;
        for (int x = 0; x < d; ++x) out[x] += w[j] * bf16_bits_to_double(vrow[x]);
    }
    *n_keys = P + 1;
    return ORACLE_OK;
}

static int check_problem(const problem_t *p) {
    if (!p->q || !p->k || !p->v || !p->cu_seqlens) return ORACLE_ERR_ARG;
    if (p->num_seqs < 0 || p->n_head < 1 || p->n_kv_head < 1) return ORACLE_ERR_ARG;
    if (p->n_head % p->n_kv_head) return ORACLE_ERR_ARG;
    if (p->head_dim < 1 || p->head_dim > 512) return ORACLE_ERR_ARG;
    if (p->context_lens && (!p->kv_cache || !p->block_table || p->block_size < 1)) return ORACLE_ERR_ARG;
    if (p->window < 0) return ORACLE_ERR_ARG;
    return ORACLE_OK;
}

static int max_keys(const problem_t *p) {
    int mk = 1;
    for (int i = 0; i < p->num_seqs; ++i) {
        int n = p->cu_seqlens[i + 1] - p->cu_seqlens[i];
        int ctx = p->context_lens ? p->context_lens[i] : 0;
        if (ctx + n > mk) mk = ctx + n;
    }
    return mk;
}

#define PROBLEM_ARGS                                                                       \
    const uint16_t *q, const uint16_t *k, const uint16_t *v, const int32_t *cu_seqlens,   \
    const int32_t *context_lens, int num_seqs, int n_head, int n_kv_head, int head_dim,  \
    double scale, const uint16_t *kv_cache, int num_blocks, const int32_t *block_table,   \
    int max_blocks_per_seq, int block_size, int window

#define PROBLEM_INIT                                                                       \
    problem_t pr = {q, k, v, cu_seqlens, context_lens, num_seqs, n_head, n_kv_head,       \
                    head_dim, scale, kv_cache, num_blocks, block_table, max_blocks_per_seq, \
                    block_size, window};                                                    \
    int rc0 = check_problem(&pr);                                                          \
    if (rc0) return rc0;

/* Attention output for selected (row, head) pairs: out[n_sel][head_dim].
 * context_lens may be NULL (plain prefill: every context is 0). */
int oracle_attention_rows(PROBLEM_ARGS, const int32_t *sel_row, const int32_t *sel_head, int n_sel,
                          double *out) {
    PROBLEM_INIT
    int mk = max_keys(&pr);
    int rc = ORACLE_OK;
#pragma omp parallel
    {
        double *w = (double *)malloc(sizeof(double) * (size_t)mk);
        int local = w ? ORACLE_OK : ORACLE_ERR_NOMEM;
#pragma omp for schedule(dynamic, 1)
        for (int s = 0; s < n_sel; ++s) {
            int nk = 0;
            if (local == ORACLE_OK)
                local = attend_one(&pr, sel_row[s], sel_head[s], out + (size_t)s * head_dim, w, &nk);
        }
        free(w);
#pragma omp critical
        if (local && !rc) rc = local;
    }
    return rc;
}

/* Attention output for every row and head: out[T][n_head][head_dim]. */
int oracle_attention_all(PROBLEM_ARGS, double *out) {
    PROBLEM_INIT
    int T = num_seqs > 0 ? cu_seqlens[num_seqs] : 0;
    int mk = max_keys(&pr);
    int rc = ORACLE_OK;
    long total = (long)T * n_head;
#pragma omp parallel
    {
        double *w = (double *)malloc(sizeof(double) * (size_t)mk);
        int local = w ? ORACLE_OK : ORACLE_ERR_NOMEM;
#pragma omp for schedule(dynamic, 4)
        for (long u = 0; u < total; ++u) {
            int t = (int)(u / n_head), h = (int)(u % n_head), nk = 0;
            if (local == ORACLE_OK)
                local = attend_one(&pr, t, h, out + (size_t)u * head_dim, w, &nk);
        }
        free(w);
#pragma omp critical
        if (local && !rc) rc = local;
    }
    return rc;
}

/* Softmax weights of one (row, head): w_out[0..P], returns the key count via
 * *n_keys.  Exposed so the tests can check the normalisation directly. */
int oracle_softmax_weights(PROBLEM_ARGS, int row, int head, double *w_out, int *n_keys) {
    PROBLEM_INIT
    double o[512];
    return attend_one(&pr, row, head, o, w_out, n_keys);
}

/* Paged KV write: copy every token's K and V rows (all kv heads) into its
 * cache slot.  Bit copy; nothing else in the pool changes. */
int oracle_kv_write(const uint16_t *k, const uint16_t *v, const int32_t *cu_seqlens,
                    const int32_t *context_lens, int num_seqs, int n_kv_head, int head_dim,
                    uint16_t *kv_cache, int num_blocks, const int32_t *block_table,
                    int max_blocks_per_seq, int block_size) {
    if (!k || !v || !cu_seqlens || !kv_cache || !block_table || block_size < 1) return ORACLE_ERR_ARG;
    size_t row = (size_t)n_kv_head * (size_t)head_dim;
    for (int i = 0; i < num_seqs; ++i) {
        int ctx = context_lens ? context_lens[i] : 0;
        for (int t = cu_seqlens[i]; t < cu_seqlens[i + 1]; ++t) {
            int P = ctx + (t - cu_seqlens[i]);
            int lp = P / block_size;
            if (lp >= max_blocks_per_seq) return ORACLE_ERR_BLOCK_TABLE;
            int page = block_table[(size_t)i * max_blocks_per_seq + lp];
            if (page < 0 || page >= num_blocks) return ORACLE_ERR_BLOCK_TABLE;
            size_t slot = (size_t)(P % block_size);
            uint16_t *kd = kv_cache + (((size_t)page * 2 + 0) * (size_t)block_size + slot) * row;
            uint16_t *vd = kv_cache + (((size_t)page * 2 + 1) * (size_t)block_size + slot) * row;
            memcpy(kd, k + (size_t)t * row, row * sizeof(uint16_t));
            memcpy(vd, v + (size_t)t * row, row * sizeof(uint16_t));
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ FP8 KV cache
 * hncyxsy.com/news/227904 §2.3: the KV cache may be kept in FP8 while the
 * softmax stays at higher precision; §3.3: FP8 / INT8 (1 byte per element).
 * Readings: the format is e4m3 (1 sign, 4 exponent bits with bias 7, 3
 * mantissa bits; exponent field 0 holds the subnormals m * 2^-9; code 0x7F /
 * 0xFF is NaN, so the largest finite value is 448).  Each kv head has one
 * scale for K and one for V: the stored code is e4m3(x / scale) with the
 * quotient formed in fp32 (x is the bf16 value, scale the caller's float) and
 * rounded to the nearest code, ties to the even code, magnitudes beyond 448
 * saturating to 448; the value the attention uses is code_value * scale.
 */

/* e4m3 code of a float32 value (round to nearest even, saturate to +-448). */
uint8_t oracle_e4m3_encode(float x) {
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a != a) return (uint8_t)(sign | 0x7F);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    if (a < ldexp(1.0, -6)) {                 /* subnormal codes: m * 2^-9, m = 0 .. 8 */
        double m = nearbyint(a * 512.0);      /* default rounding: to nearest, ties to even */
        return (uint8_t)(sign | (uint8_t)m);  /* m = 8 is the smallest normal, code 0x08 */
    }
    int e;
    double f = frexp(a, &e);                  /* a = f 2^e, f in [0.5, 1) */
    int E = e - 1;                            /* a = 2^E (1 + frac) */
    double m = nearbyint((2.0 * f - 1.0) * 8.0);
    if (m == 8.0) {
        m = 0.0;
        E += 1;
    }
    return (uint8_t)(sign | (uint8_t)((E + 7) << 3) | (uint8_t)m);
}

/* Value of an e4m3 code (NaN codes give NaN). */
double oracle_e4m3_decode(uint8_t c) {
    int e = (c >> 3) & 0xF, m = c & 7;
    double v;
    if ((c & 0x7F) == 0x7F) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return (c & 0x80) ? -v : v;
}

/* Quantize n bf16 values with one scale: out[x] = e4m3(fp32(value) / scale). */
void oracle_e4m3_quantize(const uint16_t *in, size_t n, float scale, uint8_t *out) {
    for (size_t x = 0; x < n; ++x) {
        float v = (float)bf16_bits_to_double(in[x]);
        out[x] = oracle_e4m3_encode(v / scale);
    }
}

/* Paged KV write into an FP8 cache [num_blocks][2][bs][G][d] of codes:
 * token t of sequence i goes to position ctx_i + t, K with k_scale[g], V with
 * v_scale[g].  Nothing else in the pool changes. */
int oracle_kv_write_fp8(const uint16_t *k, const uint16_t *v, const int32_t *cu_seqlens,
                        const int32_t *context_lens, int num_seqs, int n_kv_head, int head_dim,
                        const float *k_scale, const float *v_scale, uint8_t *kv_cache, int num_blocks,
                        const int32_t *block_table, int max_blocks_per_seq, int block_size) {
    if (!k || !v || !cu_seqlens || !kv_cache || !block_table || !k_scale || !v_scale || block_size < 1)
        return ORACLE_ERR_ARG;
    size_t d = (size_t)head_dim, G = (size_t)n_kv_head;
    for (int i = 0; i < num_seqs; ++i) {
        int ctx = context_lens ? context_lens[i] : 0;
        for (int t = cu_seqlens[i]; t < cu_seqlens[i + 1]; ++t) {
            int P = ctx + (t - cu_seqlens[i]);
            int lp = P / block_size;
            if (lp >= max_blocks_per_seq) return ORACLE_ERR_BLOCK_TABLE;
            int page = block_table[(size_t)i * max_blocks_per_seq + lp];
            if (page < 0 || page >= num_blocks) return ORACLE_ERR_BLOCK_TABLE;
            size_t slot = (size_t)(P % block_size);
            for (size_t g = 0; g < G; ++g) {
                uint8_t *kd = kv_cache + ((((size_t)page * 2 + 0) * (size_t)block_size + slot) * G + g) * d;
                uint8_t *vd = kv_cache + ((((size_t)page * 2 + 1) * (size_t)block_size + slot) * G + g) * d;
                oracle_e4m3_quantize(k + ((size_t)t * G + g) * d, d, k_scale[g], kd);
                oracle_e4m3_quantize(v + ((size_t)t * G + g) * d, d, v_scale[g], vd);
            }
        }
    }
    return ORACLE_OK;
}

/* Decode over an FP8 cache: the new token of sequence i (q row i, k/v row i)
 * at position ctx_i attends to the dequantized cache entries 0 .. ctx_i - 1
 * and to its own K/V quantized the same way (every key the attention sees is
 * a dequantized cache value).  out[B][n_head][head_dim] in fp64. */
int oracle_decode_fp8(const uint16_t *q, const uint16_t *k, const uint16_t *v, const int32_t *context_lens,
                      int num_seqs, int n_head, int n_kv_head, int head_dim, double scale, const float *k_scale,
                      const float *v_scale, const uint8_t *kv_cache, int num_blocks, const int32_t *block_table,
                      int max_blocks_per_seq, int block_size, double *out) {
    if (!q || !k || !v || !context_lens || !kv_cache || !block_table || !k_scale || !v_scale || !out)
        return ORACLE_ERR_ARG;
    if (n_head < 1 || n_kv_head < 1 || n_head % n_kv_head || head_dim < 1 || head_dim > 512) return ORACLE_ERR_ARG;
    int r = n_head / n_kv_head, rc = ORACLE_OK;
    size_t d = (size_t)head_dim, G = (size_t)n_kv_head;
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < num_seqs * n_head; ++u) {
        int i = u / n_head, h = u % n_head, g = h / r, ctx = context_lens[i];
        int local = ORACLE_OK;
        double qd[512], kq[512], vq[512], *w = NULL, *o = out + (size_t)u * d;
        uint8_t knew[512], vnew[512];
        for (size_t x = 0; x < d; ++x) qd[x] = bf16_bits_to_double(q[((size_t)i * (size_t)n_head + (size_t)h) * d + x]);
        oracle_e4m3_quantize(k + ((size_t)i * G + (size_t)g) * d, d, k_scale[g], knew);
        oracle_e4m3_quantize(v + ((size_t)i * G + (size_t)g) * d, d, v_scale[g], vnew);
        w = (double *)malloc(sizeof(double) * (size_t)(ctx + 1));
        if (!w) local = ORACLE_ERR_NOMEM;
        /* pass 1: scores over keys 0 .. ctx (key ctx = the new token) */
        double m = -INFINITY;
        for (int j = 0; j <= ctx && local == ORACLE_OK; ++j) {
            const uint8_t *kc = knew;
            if (j < ctx) {
                int lp = j / block_size, page = lp < max_blocks_per_seq ? block_table[(size_t)i * max_blocks_per_seq + lp] : -1;
                if (page < 0 || page >= num_blocks) { local = ORACLE_ERR_BLOCK_TABLE; break; }
                kc = kv_cache + ((((size_t)page * 2 + 0) * (size_t)block_size + (size_t)(j % block_size)) * G + (size_t)g) * d;
            }
            for (size_t x = 0; x < d; ++x) kq[x] = oracle_e4m3_decode(kc[x]) * (double)k_scale[g];
            double dot = 0.0;
            for (size_t x = 0; x < d; ++x) dot += qd[x] * kq[x];
            w[j] = scale * dot;
            if (w[j] > m) m = w[j];
        }
        /* pass 2: exponentials, their sum, and the weighted sum of dequantized values */
        double l = 0.0;
        for (size_t x = 0; x < d; ++x) o[x] = 0.0;
        for (int j = 0; j <= ctx && local == ORACLE_OK; ++j) {
            w[j] = exp(w[j] - m);
            l += w[j];
        }
        for (int j = 0; j <= ctx && local == ORACLE_OK; ++j) {
            const uint8_t *vc = vnew;
            if (j < ctx) {
                int page = block_table[(size_t)i * max_blocks_per_seq + j / block_size];
                vc = kv_cache + ((((size_t)page * 2 + 1) * (size_t)block_size + (size_t)(j % block_size)) * G + (size_t)g) * d;
            }
            for (size_t x = 0; x < d; ++x) vq[x] = oracle_e4m3_decode(vc[x]) * (double)v_scale[g];
            for (size_t x = 0; x < d; ++x) o[x] += (w[j] / l) * vq[x];
        }
        free(w);
        if (local) {
#pragma omp critical
            if (!rc) rc = local;
        }
    }
    return rc;
}

/* Chunked prefill over an FP8 cache: chunk row a of sequence i (packed row
 * cu_seqlens[i] + a) sits at position ctx_i + a and attends to keys
 * 0 .. ctx_i + a.  Key j < ctx_i is the dequantized cache entry; key
 * j >= ctx_i is chunk row j - ctx_i quantized with the same per-kv-head scales
 * and dequantized, as it is then stored (every key and value the attention
 * sees is a dequantized cache value).  With one-row chunks this is
 * oracle_decode_fp8.  The chunk's codes are computed once, before any score.
 * Outputs for the selected (packed row, head) pairs, or for every pair when
 * n_sel < 0 (out[T][n_head][head_dim]), in fp64. */
int oracle_chunked_fp8(const uint16_t *q, const uint16_t *k, const uint16_t *v, const int32_t *cu_seqlens,
                       const int32_t *context_lens, int num_seqs, int n_head, int n_kv_head, int head_dim,
                       double scale, const float *k_scale, const float *v_scale, const uint8_t *kv_cache,
                       int num_blocks, const int32_t *block_table, int max_blocks_per_seq, int block_size,
                       const int32_t *sel_row, const int32_t *sel_head, int n_sel, double *out) {
    if (!q || !k || !v || !cu_seqlens || !context_lens || !kv_cache || !block_table || !k_scale || !v_scale || !out)
        return ORACLE_ERR_ARG;
    if (n_head < 1 || n_kv_head < 1 || n_head % n_kv_head || head_dim < 1 || head_dim > 512 || block_size < 1)
        return ORACLE_ERR_ARG;
    int r = n_head / n_kv_head, rc = ORACLE_OK, T = cu_seqlens[num_seqs];
    size_t d = (size_t)head_dim, G = (size_t)n_kv_head;
    /* the chunk's own codes, and the sequence of each packed row */
    uint8_t *kc8 = (uint8_t *)malloc((size_t)T * G * d + 1), *vc8 = (uint8_t *)malloc((size_t)T * G * d + 1);
    int *seq_of = (int *)malloc(sizeof(int) * ((size_t)T + 1));
    if (!kc8 || !vc8 || !seq_of) {
        free(kc8);
        free(vc8);
        free(seq_of);
        return ORACLE_ERR_NOMEM;
    }
    for (int i = 0; i < num_seqs; ++i)
        for (int t = cu_seqlens[i]; t < cu_seqlens[i + 1]; ++t) {
            seq_of[t] = i;
            for (size_t g = 0; g < G; ++g) {
                oracle_e4m3_quantize(k + ((size_t)t * G + g) * d, d, k_scale[g], kc8 + ((size_t)t * G + g) * d);
                oracle_e4m3_quantize(v + ((size_t)t * G + g) * d, d, v_scale[g], vc8 + ((size_t)t * G + g) * d);
            }
        }
    int n_pairs = n_sel >= 0 ? n_sel : T * n_head;
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < n_pairs; ++u) {
        int t = n_sel >= 0 ? sel_row[u] : u / n_head, h = n_sel >= 0 ? sel_head[u] : u % n_head;
        int local = ORACLE_OK;
        double *o = out + (size_t)u * d;
        if (t < 0 || t >= T || h < 0 || h >= n_head) {
            local = ORACLE_ERR_ARG;
        } else {
            int i = seq_of[t], g = h / r, ctx = context_lens[i], c0 = cu_seqlens[i];
            int P = ctx + (t - c0); /* absolute position of the row */
            double qd[512], kq[512], vq[512], *w = (double *)malloc(sizeof(double) * (size_t)(P + 1));
            if (!w) local = ORACLE_ERR_NOMEM;
            for (size_t x = 0; x < d; ++x) qd[x] = bf16_bits_to_double(q[((size_t)t * (size_t)n_head + (size_t)h) * d + x]);
            /* pass 1: scores over keys 0 .. P */
            double m = -INFINITY;
            for (int j = 0; j <= P && local == ORACLE_OK; ++j) {
                const uint8_t *kc;
                if (j < ctx) {
                    int lp = j / block_size;
                    int page = lp < max_blocks_per_seq ? block_table[(size_t)i * max_blocks_per_seq + lp] : -1;
                    if (page < 0 || page >= num_blocks) { local = ORACLE_ERR_BLOCK_TABLE; break; }
                    kc = kv_cache + ((((size_t)page * 2 + 0) * (size_t)block_size + (size_t)(j % block_size)) * G +
                                     (size_t)g) * d;
                } else {
                    kc = kc8 + ((size_t)(c0 + j - ctx) * G + (size_t)g) * d;
                }
                for (size_t x = 0; x < d; ++x) kq[x] = oracle_e4m3_decode(kc[x]) * (double)k_scale[g];
                double dot = 0.0;
                for (size_t x = 0; x < d; ++x) dot += qd[x] * kq[x];
                w[j] = scale * dot;
                if (w[j] > m) m = w[j];
            }
            /* pass 2: exponentials, their sum, and the weighted sum of dequantized values */
            double l = 0.0;
            for (size_t x = 0; x < d; ++x) o[x] = 0.0;
            for (int j = 0; j <= P && local == ORACLE_OK; ++j) {
                w[j] = exp(w[j] - m);
                l += w[j];
            }
            for (int j = 0; j <= P && local == ORACLE_OK; ++j) {
                const uint8_t *vc;
                if (j < ctx) {
                    int page = block_table[(size_t)i * max_blocks_per_seq + j / block_size];
                    vc = kv_cache + ((((size_t)page * 2 + 1) * (size_t)block_size + (size_t)(j % block_size)) * G +
                                     (size_t)g) * d;
                } else {
                    vc = vc8 + ((size_t)(c0 + j - ctx) * G + (size_t)g) * d;
                }
                for (size_t x = 0; x < d; ++x) vq[x] = oracle_e4m3_decode(vc[x]) * (double)v_scale[g];
                for (size_t x = 0; x < d; ++x) o[x] += (w[j] / l) * vq[x];
            }
            free(w);
        }
        if (local) {
#pragma omp critical
            if (!rc) rc = local;
        }
    }
    free(kc8);
    free(vc8);
    free(seq_of);
    return rc;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads for the parallel loops that follow (n >= 1); a timing harness sets it
 * to the cores the process may run on. */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
