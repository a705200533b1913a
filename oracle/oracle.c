/*
 * oracle.c -- plain, slow fp64 CPU definition of hybrid compressed / sparse /
 * sliding-window attention (forward pass).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark load this file.  It shares no code,
 * header, table or helper with the CUDA library, and it never reads anything
 * the CUDA library produced.
 *
 * Sources (web pages on DeepSeek-V4 hybrid attention):
 *   [V4-blog]   "deepseek-v4" (s1mplewind astro blog), section "1. hybrid attn",
 *               subsections CSA, HCA and SWA.
 *   [CSDN]      "DeepSeek-V4 CSA / HCA mechanism" code page (un.csdn.net),
 *               section 1 (HCA, block_merge) and section 2 (CSA, block_compress).
 *   [zwxr]      "DeepSeek-V4 architecture diagram" post (zwxr.cn), section 4
 *               (SWA boundary handling), 4.2 and 4.4.
 *   [CS336]     CS336 lecture notes, "Attention Heads variants" (MQA/GQA) and
 *               "Attention Alternatives" (FlashAttention, DSA lightning indexer).
 *
 * Every floating-point input arrives as raw bf16 bits (uint16) or fp32 and is
 * widened exactly to double; all arithmetic is double.  Outputs are double,
 * except the compressed caches, which are also returned rounded to bf16 (the
 * storage format of the compressed KV cache).
 *
 * Readings of points the pages leave open are listed next to the code that
 * takes them.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_INDEX (-1)
#define ORACLE_BAD_ARG (-2)

static double from_bf16(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 value, ties to even.  bf16 keeps 8
 * significant bits and fp32's exponent range; its smallest subnormal step is
 * 2^-133.  The value is scaled so that the kept bits form an integer, rounded
 * with rint() (round-half-even in the default rounding mode) and scaled back;
 * the result is exactly representable as a float, whose top 16 bits are the
 * bf16 encoding. */
static uint16_t to_bf16(double v)
{
    if (isnan(v))
        return 0x7fc0;
    int neg = signbit(v) ? 1 : 0;
    double a = fabs(v);
    uint32_t bits;
    if (isinf(a) || a >= 0x1p128) {
        bits = 0x7f800000u;
    } else if (a == 0.0) {
        bits = 0;
    } else {
        int e;
        (void)frexp(a, &e);                 /* a = f * 2^e, f in [0.5, 1) */
        int qexp = e - 8;                   /* step between neighbouring bf16 values */
        if (qexp < -133)
            qexp = -133;
        double q = ldexp(1.0, qexp);
        double r = rint(a / q) * q;         /* a / q is exact (power of two) */
        float f = (float)r;                 /* exact, or +inf on overflow */
        memcpy(&bits, &f, sizeof bits);
    }
    return (uint16_t)((bits >> 16) | (neg ? 0x8000u : 0u));
}

void oracle_round_bf16(const double *in, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = to_bf16(in[i]);
}

/* ------------------------------------------------------------------------ *
 * Stage 1: block_merge ([CSDN] section 1, block_merge; [V4-blog] CSA "4:1
 * compression", HCA "m = 128").
 *
 * The block weights W[m][dx] are turned into per-channel softmax weights over
 * the m positions of a block:  P[i][c] = exp(W[i][c]) / sum_i' exp(W[i'][c]).
 * Entry j of the compressed cache is  c[j][c] = sum_i P[i][c] * x[j*m + i][c],
 * for j < floor(L / m); a trailing partial block is not compressed.
 * The same weights serve every head (x is [B][L][H][dx]).
 * ------------------------------------------------------------------------ */
void oracle_block_merge(const uint16_t *x, int B, int L, int H, int dx, int m,
                        const float *w, double *out, uint16_t *out_bf16)
{
    int Nc = L / m;
    double *P = (double *)malloc(sizeof(double) * (size_t)m * dx);
    for (int c = 0; c < dx; ++c) {
        double den = 0.0;
        for (int i = 0; i < m; ++i)
            den += exp((double)w[(size_t)i * dx + c]);
        for (int i = 0; i < m; ++i)
            P[(size_t)i * dx + c] = exp((double)w[(size_t)i * dx + c]) / den;
    }
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b) {
        for (int j = 0; j < Nc; ++j) {
            for (int h = 0; h < H; ++h) {
                for (int c = 0; c < dx; ++c) {
                    double acc = 0.0;
                    for (int i = 0; i < m; ++i) {
                        size_t src = (((size_t)b * L + (size_t)j * m + i) * H + h) * dx + c;
                        acc += P[(size_t)i * dx + c] * from_bf16(x[src]);
                    }
                    size_t dst = (((size_t)b * Nc + j) * H + h) * dx + c;
                    if (out)
                        out[dst] = acc;
                    if (out_bf16)
                        out_bf16[dst] = to_bf16(acc);
                }
            }
        }
    }
    free(P);
}

/* Visibility of compressed entries.  Entry j summarises raw positions
 * j*m .. j*m + m - 1.  It is visible to a query at position t when its last
 * position lies before the first position of t's raw window, t - W + 1:
 *     (j + 1) * m - 1 < t - W + 1.
 * Compressed history and raw window are thus disjoint ([V4-blog] SWA: two
 * paths, recent raw KV and older compressed KV).  The number of visible
 * entries is the count of j >= 0 satisfying this, capped by the cache
 * capacity Nc. */
static int visible_count(int64_t t, int m, int W, int Nc)
{
    int64_t n = 0;
    /* smallest j that fails: (j+1)*m - 1 >= t - W + 1 */
    while (n < Nc && (n + 1) * (int64_t)m - 1 < t - W + 1)
        ++n;
    return (int)n;
}

static int is_visible(int64_t j, int64_t t, int m, int W)
{
    return (j + 1) * (int64_t)m - 1 < t - W + 1;
}

int oracle_visible_count(int64_t t, int m, int W, int Nc)
{
    return visible_count(t, m, W, Nc);
}

/* ------------------------------------------------------------------------ *
 * Stage 2a: lightning-indexer score ([CS336] "DSA ... Lightning Indexer";
 * [V4-blog] CSA "Lightning Indexer finds the top-K compressed entries most
 * relevant to the current query").  The pages name the indexer but give no
 * formula; the reading taken is a ReLU-weighted head sum with no scale:
 *     I[t][s] = sum_h w[t][h] * max(0, sum_c qi[t][h][c] * kic[s][c])
 * for every visible entry s of query t.  Invisible entries get NaN.
 *
 * rows[r] = b * Lq + t selects which query rows to score; the query's
 * absolute position is q_pos[b * Lq + t] (or t when q_pos is NULL).
 * ------------------------------------------------------------------------ */
void oracle_index_scores(const uint16_t *qi, const float *wi, const uint16_t *kic,
                         int B, int Lq, int Hi, int di, int Nc, int m, int W,
                         const int32_t *q_pos, const int64_t *rows, int nrows,
                         double *scores, int32_t *nvis_out)
{
    (void)B;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        int64_t row = rows[r];
        int64_t b = row / Lq;
        int64_t t = q_pos ? q_pos[row] : row % Lq;
        int nv = visible_count(t, m, W, Nc);
        if (nvis_out)
            nvis_out[r] = nv;
        double *out = scores + (size_t)r * Nc;
        for (int s = 0; s < Nc; ++s) {
            if (s >= nv) {
                out[s] = NAN;
                continue;
            }
            double I = 0.0;
            for (int h = 0; h < Hi; ++h) {
                double dot = 0.0;
                for (int c = 0; c < di; ++c)
                    dot += from_bf16(qi[((size_t)row * Hi + h) * di + c]) *
                           from_bf16(kic[((size_t)b * Nc + s) * di + c]);
                double relu = dot > 0.0 ? dot : 0.0;
                I += (double)wi[(size_t)row * Hi + h] * relu;
            }
            out[s] = I;
        }
    }
}

/* ------------------------------------------------------------------------ *
 * Stage 2b: exact per-query top-K ([V4-blog] CSA, "top-K compressed entries
 * for the current query").  Readings:
 *  - the ranking decision is taken on the score rounded to fp32 (the
 *    precision the scores are kept in on the device);
 *  - equal fp32 scores: the lower entry index ranks first;
 *  - with n_vis <= K every visible entry is selected;
 *  - the selected entry indices are written in ascending order, and the
 *    remaining slots hold -1.
 * ------------------------------------------------------------------------ */
typedef struct {
    float key;
    int32_t idx;
} rank_item;

static int rank_cmp(const void *pa, const void *pb)
{
    const rank_item *a = (const rank_item *)pa, *b = (const rank_item *)pb;
    if (a->key > b->key)
        return -1;
    if (a->key < b->key)
        return 1;
    return (a->idx > b->idx) - (a->idx < b->idx);
}

static int int_cmp(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

void oracle_topk(const double *scores, const int32_t *nvis, int nrows, int Nc, int K,
                 int32_t *idx_out)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        int nv = nvis[r];
        rank_item *items = (rank_item *)malloc(sizeof(rank_item) * (size_t)(nv > 0 ? nv : 1));
        for (int s = 0; s < nv; ++s) {
            items[s].key = (float)scores[(size_t)r * Nc + s];
            items[s].idx = s;
        }
        qsort(items, (size_t)nv, sizeof(rank_item), rank_cmp);
        int take = nv < K ? nv : K;
        int32_t *dst = idx_out + (size_t)r * K;
        for (int k = 0; k < take; ++k)
            dst[k] = items[k].idx;
        qsort(dst, (size_t)take, sizeof(int32_t), int_cmp);
        for (int k = take; k < K; ++k)
            dst[k] = -1;
        free(items);
    }
}

/* ------------------------------------------------------------------------ *
 * Stage 3: one attention over the union of compressed and raw keys
 * ([V4-blog] SWA: "the compressed KV and the raw KV of the window go into the
 * attention block in sequence order"; inputs are "top-k sparse CSA KV + 128
 * raw KV" for CSA and "heavily compressed dense KV + 128 KV" for HCA).
 *
 * For query row (b, t) and query head h (KV head h / (Hq / Hkv), [CS336] MQA
 * and GQA share one KV head among a group of query heads):
 *   compressed keys: the listed entries idx[row][0..topk) that are >= 0 and
 *                    visible (CSA), or every visible entry (HCA, idx NULL);
 *   raw keys:        positions p with max(0, t - W + 1) <= p <= t (window of
 *                    W tokens including t, stride 1, clipped at the sequence
 *                    start: [zwxr] 4.4), read from raw row p - kv_pos0[b]
 *                    when that row exists in the raw buffer.
 *   logits  l_k = scale * q . k_k;  weights p_k = exp(l_k - max) / sum;
 *   o = sum_k p_k v_k;  lse = max + log(sum exp(l_k - max)).
 * An empty key set (possible only when W = 0) gives o = 0 and lse = -inf.
 * One softmax spans both parts.  The scale is 1/sqrt(d) unless given.
 *
 * Optional debug outputs: n_comp/n_win per row, and for every (row, head) the
 * softmax weights p_out[.., maxkeys] with key labels keys_out[row][..]
 * (compressed entry j -> j, raw position p -> -(p + 1)).
 * ------------------------------------------------------------------------ */
int oracle_hybrid_attention(const uint16_t *q, const uint16_t *kc, const uint16_t *vc,
                            const int32_t *idx, int topk,
                            const uint16_t *k_raw, const uint16_t *v_raw,
                            int B, int Lq, int Lkv, int Hq, int Hkv, int d, int m, int W,
                            int Nc, double scale, const int32_t *q_pos, const int32_t *kv_pos0,
                            const int64_t *rows, int nrows, double *o, double *lse,
                            int32_t *n_comp, int32_t *n_win, double *p_out, int maxkeys,
                            int32_t *keys_out)
{
    (void)B;
    if (Hkv <= 0 || Hq % Hkv != 0)
        return ORACLE_BAD_ARG;
    int g = Hq / Hkv;
    int status = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        int64_t row = rows[r];
        int64_t b = row / Lq;
        int64_t t = q_pos ? q_pos[row] : row % Lq;
        int64_t kv0 = kv_pos0 ? kv_pos0[b] : 0;

        /* key list: compressed entries first, then raw window rows */
        int cap = (idx ? topk : Nc) + (W > 0 ? W : 0);
        int32_t *ckey = (int32_t *)malloc(sizeof(int32_t) * (size_t)(cap > 0 ? cap : 1));
        int64_t *rrow = (int64_t *)malloc(sizeof(int64_t) * (size_t)(cap > 0 ? cap : 1));
        int nc = 0, nw = 0;
        if (idx) {
            for (int k = 0; k < topk; ++k) {
                int32_t j = idx[(size_t)row * topk + k];
                if (j < 0)
                    continue;
                if (j >= Nc) {
#pragma omp atomic write
                    status = ORACLE_BAD_INDEX;
                    continue;
                }
                if (is_visible(j, t, m, W))
                    ckey[nc++] = j;
            }
        } else {
            int nv = visible_count(t, m, W, Nc);
            for (int j = 0; j < nv; ++j)
                ckey[nc++] = j;
        }
        int64_t p_lo = t - W + 1;
        if (p_lo < 0)
            p_lo = 0;
        for (int64_t p = p_lo; p <= t && W > 0; ++p) {
            int64_t rr = p - kv0;
            if (rr >= 0 && rr < Lkv)
                rrow[nw++] = rr;
        }
        if (n_comp)
            n_comp[r] = nc;
        if (n_win)
            n_win[r] = nw;
        if (keys_out) {
            for (int k = 0; k < maxkeys; ++k) {
                int32_t lab = 0x7fffffff;
                if (k < nc)
                    lab = ckey[k];
                else if (k < nc + nw)
                    lab = (int32_t)(-(rrow[k - nc] + kv0 + 1));
                keys_out[(size_t)r * maxkeys + k] = lab;
            }
        }

        int nk = nc + nw;
        double *logit = (double *)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
        for (int h = 0; h < Hq; ++h) {
            int kvh = h / g;
            const uint16_t *qv = q + ((size_t)row * Hq + h) * d;
            double *oo = o + ((size_t)r * Hq + h) * d;
            if (nk == 0) {
                for (int c = 0; c < d; ++c)
                    oo[c] = 0.0;
                if (lse)
                    lse[(size_t)r * Hq + h] = -INFINITY;
                continue;
            }
            double mx = -INFINITY;
            for (int k = 0; k < nk; ++k) {
                const uint16_t *kv;
                if (k < nc)
                    kv = kc + (((size_t)b * Nc + ckey[k]) * Hkv + kvh) * d;
                else
                    kv = k_raw + (((size_t)b * Lkv + rrow[k - nc]) * Hkv + kvh) * d;
                double dot = 0.0;
                for (int c = 0; c < d; ++c)
                    dot += from_bf16(qv[c]) * from_bf16(kv[c]);
                logit[k] = scale * dot;
                if (logit[k] > mx)
                    mx = logit[k];
            }
            double den = 0.0;
            for (int k = 0; k < nk; ++k)
                den += exp(logit[k] - mx);
            for (int c = 0; c < d; ++c)
                oo[c] = 0.0;
            for (int k = 0; k < nk; ++k) {
                double p = exp(logit[k] - mx) / den;
                const uint16_t *vv;
                if (k < nc)
                    vv = vc + (((size_t)b * Nc + ckey[k]) * Hkv + kvh) * d;
                else
                    vv = v_raw + (((size_t)b * Lkv + rrow[k - nc]) * Hkv + kvh) * d;
                for (int c = 0; c < d; ++c)
                    oo[c] += p * from_bf16(vv[c]);
                if (p_out && k < maxkeys)
                    p_out[((size_t)r * Hq + h) * maxkeys + k] = p;
            }
            if (lse)
                lse[(size_t)r * Hq + h] = mx + log(den);
        }
        free(logit);
        free(ckey);
        free(rrow);
    }
    return status;
}
