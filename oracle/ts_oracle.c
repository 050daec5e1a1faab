/*
 * TokenSelect decode-step oracle: plain, slow, float64 CPU definitions.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is used by the test-suite, by the
 * smoke check and by the CPU-baseline leg of the benchmark.  The product path
 * (the CUDA library) never links, loads or calls it, and it shares no code,
 * header or constant with that library.
 *
 * Sources (web pages on the method; cited by page title and section):
 *   [TS-README]  "TokenSelect: Efficient Long-Context Inference and Length
 *                Extrapolation for LLMs via Dynamic Token-Level KV Cache
 *                Selection" -- GitHub README, section "Key Takeaways":
 *                (1) per-head criticality of each cached token is the
 *                Query-Key dot product; (2) per-head soft voting: the
 *                per-head criticality is softmax-normalised and summed over
 *                heads; (3) Selection Cache: consecutive similar queries share
 *                one selection.  The same README's summary line says that a
 *                small number of critical KV tokens take part in attention.
 *   [TS-SUMMARY] GrooveSquid summary of the same paper (medium-difficulty
 *                summary): non-contiguous, token-level attention sparsity,
 *                per-head soft voting, Selection Cache, dot-product kernel.
 *   [QUEST]      Bohrium page for "Quest: Query-Aware Sparsity for Efficient
 *                Long-Context LLM Inference" (arXiv 2406.10774), Abstract and
 *                "Method Overview" (4): each KV cache page keeps the minimal
 *                and maximal key values; a page's criticality is estimated
 *                from the element-wise products of the query with them; the
 *                Top-K critical pages are loaded for attention.  Used here
 *                only for the page-level comparator at the end of the file.
 * Where the pages leave a step open, the reading used is noted at the
 * function (readings R1..R19, R21..R23).
 *
 * Conventions shared by every function:
 *   - bf16 inputs are passed as raw uint16 bit patterns and widened exactly
 *     to double (bf16 -> fp32 is a 16-bit shift; fp32 -> fp64 is exact).
 *   - K and V are one sequence's rows of a layer's cache, element
 *     (token t, kv-head g, channel c) at t*stride_tok + g*stride_head + c.
 *   - q is [h_q][d] contiguous (one decode query, all heads).
 *   - GQA: query head h reads kv head g(h) = h / (h_q / h_kv)   (R1).
 *   - Every arithmetic step is float64, in the order written, one thread.
 *
 * Parity pins for every function live in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Exact bf16 -> double widening. */
static double widen_bf16(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* Selection Cache  [TS-README, Key Takeaways (3); TS-SUMMARY]               */
/* ------------------------------------------------------------------------ */

/* Cosine similarity of two bf16 vectors of length len, in float64.
 * Reading R7: the query of one sequence is compared as one flattened
 * vector over all query heads (one decision per sequence and layer).
 * A zero vector has no direction: the cosine is reported as 0. */
double oracle_cosine(const uint16_t *a, const uint16_t *b, int64_t len)
{
    double ab = 0.0, aa = 0.0, bb = 0.0;
    for (int64_t i = 0; i < len; ++i) {
        double x = widen_bf16(a[i]);
        double y = widen_bf16(b[i]);
        ab += x * y;
        aa += x * x;
        bb += y * y;
    }
    if (aa == 0.0 || bb == 0.0)
        return 0.0;
    return ab / (sqrt(aa) * sqrt(bb));
}

/* One selection-cache decision for one sequence.
 * reuse = (not the first step) and cos(q_t, q_{t-1}) >= theta ("at or above").
 * Afterwards q_prev holds q_t (the comparison is always with the immediately
 * preceding step's query).  Returns reuse (0/1); *cos_out gets the cosine
 * (0 on the first step). */
int oracle_selcache(const uint16_t *q, uint16_t *q_prev, int64_t len,
                    int first_step, double theta, double *cos_out)
{
    double c = 0.0;
    int reuse = 0;
    if (!first_step) {
        c = oracle_cosine(q, q_prev, len);
        reuse = (c >= theta) ? 1 : 0;
    }
    memcpy(q_prev, q, (size_t)len * sizeof(uint16_t));
    if (cos_out)
        *cos_out = c;
    return reuse;
}

/* ------------------------------------------------------------------------ */
/* Per-head criticality and soft vote  [TS-README, Key Takeaways (1), (2)]  */
/* ------------------------------------------------------------------------ */

/* Criticality logits of one query head over all n cached tokens:
 *   s[i] = scale * sum_c q[h][c] * K[i][g(h)][c]
 * Reading R2: scale (1/sqrt(d) by default) is applied, so that the softmax
 * below is the head's own attention distribution. */
void oracle_head_logits(const uint16_t *k, int64_t n, int32_t h_kv, int32_t d,
                        int64_t stride_tok, int64_t stride_head,
                        const uint16_t *q, int32_t h_q, int32_t h, double scale,
                        double *s_out)
{
    int32_t group = h_q / h_kv;
    int32_t g = h / group;
    const uint16_t *qh = q + (int64_t)h * d;
    for (int64_t i = 0; i < n; ++i) {
        const uint16_t *ki = k + i * stride_tok + (int64_t)g * stride_head;
        double dot = 0.0;
        for (int32_t c = 0; c < d; ++c)
            dot += widen_bf16(qh[c]) * widen_bf16(ki[c]);
        s_out[i] = scale * dot;
    }
}

/* Softmax of one row over the token axis (reading R3: all n tokens, sink and
 * local included).  p[i] = exp(s[i] - M) / Z with M = max s, Z = sum exp(s - M).
 * Returns the log-normaliser L = M + ln Z.  n == 0 returns -inf. */
double oracle_softmax_row(const double *s, int64_t n, double *p_out)
{
    if (n <= 0)
        return -INFINITY;
    double m = s[0];
    for (int64_t i = 1; i < n; ++i)
        if (s[i] > m)
            m = s[i];
    double z = 0.0;
    for (int64_t i = 0; i < n; ++i)
        z += exp(s[i] - m);
    for (int64_t i = 0; i < n; ++i)
        p_out[i] = exp(s[i] - m) / z;
    return m + log(z);
}

/* Soft vote of one sequence: v[i] = sum over query heads h of p_h[i], where
 * p_h is head h's softmax of its criticality logits.  L_out (may be NULL)
 * receives each head's log-normaliser.  Since each p_h sums to 1, the votes
 * sum to h_q. */
void oracle_votes(const uint16_t *k, int64_t n, int32_t h_kv, int32_t d,
                  int64_t stride_tok, int64_t stride_head,
                  const uint16_t *q, int32_t h_q, double scale,
                  double *v_out, double *L_out)
{
    for (int64_t i = 0; i < n; ++i)
        v_out[i] = 0.0;
    if (n <= 0) {
        for (int32_t h = 0; h < h_q && L_out; ++h)
            L_out[h] = -INFINITY;
        return;
    }
    double *s = (double *)malloc((size_t)n * sizeof(double));
    double *p = (double *)malloc((size_t)n * sizeof(double));
    for (int32_t h = 0; h < h_q; ++h) {
        oracle_head_logits(k, n, h_kv, d, stride_tok, stride_head, q, h_q, h,
                           scale, s);
        double L = oracle_softmax_row(s, n, p);
        if (L_out)
            L_out[h] = L;
        for (int64_t i = 0; i < n; ++i)
            v_out[i] += p[i];
    }
    free(s);
    free(p);
}

/* ------------------------------------------------------------------------ */
/* Token selection: top-k by vote plus the fixed sink and local windows      */
/* ------------------------------------------------------------------------ */

typedef struct {
    double v;
    int64_t i;
} vote_entry;

/* Order: larger vote first; equal votes go to the lower token id (R5). */
static int vote_entry_cmp(const void *pa, const void *pb)
{
    const vote_entry *a = (const vote_entry *)pa;
    const vote_entry *b = (const vote_entry *)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    if (a->i < b->i) return -1;
    if (a->i > b->i) return 1;
    return 0;
}

/* Window bounds shared by select and its callers (R4):
 *   sink  = [0, s'),           s' = min(n_sink, n)
 *   local = [l0, n),           l0 = max(n - n_local, s')
 *   candidates C = [s', l0)
 * so the three parts never overlap and together cover at most n tokens. */
void oracle_windows(int64_t n, int64_t n_sink, int64_t n_local,
                    int64_t *sink_end, int64_t *local_begin)
{
    int64_t s = n_sink < n ? n_sink : n;
    int64_t l0 = n - n_local;
    if (l0 < s)
        l0 = s;
    *sink_end = s;
    *local_begin = l0;
}

/* Selected ids of one sequence, ascending (R6):
 *   T   = the first min(k, |C|) candidates in (vote desc, id asc) order,
 *   ids = sort(sink U T U local).
 * ids_out must hold k + n_sink + n_local entries; entries past the returned
 * count are set to -1.  Returns the count m = min(n, ...) of selected ids. */
int64_t oracle_select(const double *v, int64_t n, int64_t k, int64_t n_sink,
                      int64_t n_local, int32_t *ids_out)
{
    int64_t cap = k + n_sink + n_local;
    for (int64_t j = 0; j < cap; ++j)
        ids_out[j] = -1;
    if (n <= 0)
        return 0;

    int64_t s_end, l_begin;
    oracle_windows(n, n_sink, n_local, &s_end, &l_begin);
    int64_t nc = l_begin - s_end;
    int64_t take = k < nc ? k : nc;

    unsigned char *chosen = (unsigned char *)calloc((size_t)n, 1);
    for (int64_t i = 0; i < s_end; ++i)
        chosen[i] = 1;
    for (int64_t i = l_begin; i < n; ++i)
        chosen[i] = 1;
    if (take > 0) {
        vote_entry *e = (vote_entry *)malloc((size_t)nc * sizeof(vote_entry));
        for (int64_t j = 0; j < nc; ++j) {
            e[j].v = v[s_end + j];
            e[j].i = s_end + j;
        }
        qsort(e, (size_t)nc, sizeof(vote_entry), vote_entry_cmp);
        for (int64_t j = 0; j < take; ++j)
            chosen[e[j].i] = 1;
        free(e);
    }
    int64_t m = 0;
    for (int64_t i = 0; i < n; ++i)
        if (chosen[i])
            ids_out[m++] = (int32_t)i;
    free(chosen);
    return m;
}

/* Ids of a sequence that reuses its selection while its cache grows (a
 * decode loop that appends the new token's K/V before each step; TS-README
 * "Key Takeaways", Selection Cache; reading R19).  What is reused is the
 * previous step's top-k part T_prev: the ids of the previous row that lie in
 * that step's candidate range [s'_old, l0_old).  The sink and local windows
 * are those of the current length n_new, and a kept id that is no longer a
 * candidate, outside [s'_new, l0_new), is dropped:
 *   ids = sort([0, s'_new) U (T_prev n [s'_new, l0_new)) U [l0_new, n_new)).
 * With n_new == n_old this is the previous row itself (R8).
 * prev_ids: the previous row, ascending, prev_count entries valid.
 * ids_out must hold k + n_sink + n_local entries; entries past the returned
 * count are set to -1.  Returns the count. */
int64_t oracle_reuse_ids(const int32_t *prev_ids, int64_t prev_count, int64_t n_old, int64_t n_new,
                         int64_t k, int64_t n_sink, int64_t n_local, int32_t *ids_out)
{
    int64_t cap = k + n_sink + n_local;
    for (int64_t j = 0; j < cap; ++j)
        ids_out[j] = -1;
    if (n_new <= 0)
        return 0;
    int64_t s_old, l0_old, s_new, l0_new;
    oracle_windows(n_old, n_sink, n_local, &s_old, &l0_old);
    oracle_windows(n_new, n_sink, n_local, &s_new, &l0_new);
    unsigned char *chosen = (unsigned char *)calloc((size_t)n_new, 1);
    for (int64_t i = 0; i < s_new; ++i)
        chosen[i] = 1;
    for (int64_t i = l0_new; i < n_new; ++i)
        chosen[i] = 1;
    for (int64_t j = 0; j < prev_count; ++j) {
        int64_t id = prev_ids[j];
        if (id >= s_old && id < l0_old && id >= s_new && id < l0_new)
            chosen[id] = 1;
    }
    int64_t m = 0;
    for (int64_t i = 0; i < n_new && m < cap; ++i)
        if (chosen[i])
            ids_out[m++] = (int32_t)i;
    free(chosen);
    return m;
}

/* ------------------------------------------------------------------------ */
/* Attention over the selected tokens  [TS-README summary line]              */
/* ------------------------------------------------------------------------ */

/* out[h][c] = sum_j softmax_j(scale * q_h . K[ids[j]][g(h)]) * V[ids[j]][g(h)][c]
 * over the m selected ids.  m == 0 leaves out at zero (nothing to attend to). */
void oracle_sparse_attn(const uint16_t *k, const uint16_t *v, int32_t h_kv,
                        int32_t d, int64_t stride_tok, int64_t stride_head,
                        const uint16_t *q, int32_t h_q, double scale,
                        const int32_t *ids, int64_t m, double *out)
{
    int32_t group = h_q / h_kv;
    for (int64_t x = 0; x < (int64_t)h_q * d; ++x)
        out[x] = 0.0;
    if (m <= 0)
        return;
    double *s = (double *)malloc((size_t)m * sizeof(double));
    double *p = (double *)malloc((size_t)m * sizeof(double));
    for (int32_t h = 0; h < h_q; ++h) {
        int32_t g = h / group;
        const uint16_t *qh = q + (int64_t)h * d;
        for (int64_t j = 0; j < m; ++j) {
            const uint16_t *kj = k + (int64_t)ids[j] * stride_tok + (int64_t)g * stride_head;
            double dot = 0.0;
            for (int32_t c = 0; c < d; ++c)
                dot += widen_bf16(qh[c]) * widen_bf16(kj[c]);
            s[j] = scale * dot;
        }
        oracle_softmax_row(s, m, p);
        double *oh = out + (int64_t)h * d;
        for (int64_t j = 0; j < m; ++j) {
            const uint16_t *vj = v + (int64_t)ids[j] * stride_tok + (int64_t)g * stride_head;
            for (int32_t c = 0; c < d; ++c)
                oh[c] += p[j] * widen_bf16(vj[c]);
        }
    }
    free(s);
    free(p);
}

/* Dense decode attention over every cached token, written out on its own
 * (no id list): the reference that full selection must reproduce. */
void oracle_dense_attn(const uint16_t *k, const uint16_t *v, int64_t n,
                       int32_t h_kv, int32_t d, int64_t stride_tok,
                       int64_t stride_head, const uint16_t *q, int32_t h_q,
                       double scale, double *out)
{
    int32_t group = h_q / h_kv;
    for (int64_t x = 0; x < (int64_t)h_q * d; ++x)
        out[x] = 0.0;
    if (n <= 0)
        return;
    double *w = (double *)malloc((size_t)n * sizeof(double));
    for (int32_t h = 0; h < h_q; ++h) {
        int32_t g = h / group;
        const uint16_t *qh = q + (int64_t)h * d;
        double mx = -INFINITY;
        for (int64_t t = 0; t < n; ++t) {
            const uint16_t *kt = k + t * stride_tok + (int64_t)g * stride_head;
            double dot = 0.0;
            for (int32_t c = 0; c < d; ++c)
                dot += widen_bf16(qh[c]) * widen_bf16(kt[c]);
            w[t] = scale * dot;
            if (w[t] > mx)
                mx = w[t];
        }
        double den = 0.0;
        for (int64_t t = 0; t < n; ++t) {
            w[t] = exp(w[t] - mx);
            den += w[t];
        }
        double *oh = out + (int64_t)h * d;
        for (int64_t t = 0; t < n; ++t) {
            const uint16_t *vt = v + t * stride_tok + (int64_t)g * stride_head;
            double a = w[t] / den;
            for (int32_t c = 0; c < d; ++c)
                oh[c] += a * widen_bf16(vt[c]);
        }
    }
    free(w);
}

/* ------------------------------------------------------------------------ */
/* Page-level comparator: Quest's min/max page bounds  [QUEST]              */
/* ------------------------------------------------------------------------ */

/* Pages of one sequence (reading R21): page j holds the sequence's tokens
 * [j*P, min((j+1)*P, n)); there are ceil(n / P) of them, the last one
 * possibly short. */
int64_t oracle_quest_pages(int64_t n, int64_t P)
{
    return n <= 0 ? 0 : (n + P - 1) / P;
}

/* Per-page element-wise minimum and maximum of the keys, per kv head and
 * channel [QUEST, Abstract: "keeps track of the minimal and maximal Key
 * values in KV cache pages"].  Outputs are bf16 bit patterns laid out
 * [page][kv head][channel]; the extremes of bf16 values are bf16 values.
 * On equal values (+0 and -0) the earlier token's bits are kept. */
void oracle_quest_meta(const uint16_t *k, int64_t n, int32_t h_kv, int32_t d,
                       int64_t stride_tok, int64_t stride_head, int64_t P,
                       uint16_t *kmin_out, uint16_t *kmax_out)
{
    int64_t pages = oracle_quest_pages(n, P);
    for (int64_t j = 0; j < pages; ++j) {
        int64_t t0 = j * P;
        int64_t t1 = t0 + P < n ? t0 + P : n;
        for (int32_t g = 0; g < h_kv; ++g) {
            for (int32_t c = 0; c < d; ++c) {
                uint16_t lo = k[t0 * stride_tok + (int64_t)g * stride_head + c];
                uint16_t hi = lo;
                for (int64_t t = t0 + 1; t < t1; ++t) {
                    uint16_t x = k[t * stride_tok + (int64_t)g * stride_head + c];
                    if (widen_bf16(x) < widen_bf16(lo))
                        lo = x;
                    if (widen_bf16(x) > widen_bf16(hi))
                        hi = x;
                }
                int64_t o = (j * h_kv + g) * (int64_t)d + c;
                kmin_out[o] = lo;
                kmax_out[o] = hi;
            }
        }
    }
}

/* Page criticality [QUEST, Method Overview (4)]: for query head h with kv
 * head g(h) (R1), the largest value q_h . k can take over the box
 * [kmin, kmax] of the page,
 *   U_h(j) = scale * sum_c max(q_h[c] * kmin[j][g][c], q_h[c] * kmax[j][g][c]),
 * an upper bound of the scaled logit of every key in the page.  One selection
 * serves all heads of a sequence, so the page's score is the sum of the
 * per-head bounds over the h_q query heads (reading R22):
 *   score[j] = sum_h U_h(j). */
void oracle_quest_scores(const uint16_t *kmin, const uint16_t *kmax, int64_t pages,
                         int32_t h_kv, int32_t d, const uint16_t *q, int32_t h_q,
                         double scale, double *score_out)
{
    int32_t group = h_q / h_kv;
    for (int64_t j = 0; j < pages; ++j) {
        double total = 0.0;
        for (int32_t h = 0; h < h_q; ++h) {
            int32_t g = h / group;
            const uint16_t *qh = q + (int64_t)h * d;
            const uint16_t *mn = kmin + (j * h_kv + g) * (int64_t)d;
            const uint16_t *mx = kmax + (j * h_kv + g) * (int64_t)d;
            double u = 0.0;
            for (int32_t c = 0; c < d; ++c) {
                double a = widen_bf16(qh[c]) * widen_bf16(mn[c]);
                double b = widen_bf16(qh[c]) * widen_bf16(mx[c]);
                u += a > b ? a : b;
            }
            total += scale * u;
        }
        score_out[j] = total;
    }
}

/* Page selection with the token windows of R4 (reading R23): a page is a
 * candidate when it holds at least one candidate token, i.e. when
 * [max(j*P, s'), min((j+1)*P, l0)) is not empty.  The Top-K pages are the
 * first min(floor(k / P), #candidates) candidate pages in (score desc, page
 * asc) order [QUEST, Abstract: "only loading the Top-K critical KV cache
 * pages"]; their candidate tokens join the sink and local windows:
 *   ids = sort([0, s') U (tokens of the chosen pages n [s', l0)) U [l0, n)),
 * at most s' + k + (n - l0) ids.  ids_out must hold k + n_sink + n_local
 * entries; entries past the returned count are set to -1. */
int64_t oracle_quest_select(const double *score, int64_t n, int64_t P, int64_t k,
                            int64_t n_sink, int64_t n_local, int32_t *ids_out)
{
    int64_t cap = k + n_sink + n_local;
    for (int64_t j = 0; j < cap; ++j)
        ids_out[j] = -1;
    if (n <= 0)
        return 0;

    int64_t s_end, l_begin;
    oracle_windows(n, n_sink, n_local, &s_end, &l_begin);
    unsigned char *chosen = (unsigned char *)calloc((size_t)n, 1);
    for (int64_t i = 0; i < s_end; ++i)
        chosen[i] = 1;
    for (int64_t i = l_begin; i < n; ++i)
        chosen[i] = 1;

    int64_t pages = oracle_quest_pages(n, P);
    vote_entry *e = (vote_entry *)malloc((size_t)(pages > 0 ? pages : 1) * sizeof(vote_entry));
    int64_t nc = 0;
    for (int64_t j = 0; j < pages; ++j) {
        int64_t lo = j * P > s_end ? j * P : s_end;
        int64_t hi = (j + 1) * P < l_begin ? (j + 1) * P : l_begin;
        if (lo < hi) {
            e[nc].v = score[j];
            e[nc].i = j;
            ++nc;
        }
    }
    int64_t kp = k / P;
    int64_t take = kp < nc ? kp : nc;
    if (take > 0) {
        qsort(e, (size_t)nc, sizeof(vote_entry), vote_entry_cmp);
        for (int64_t x = 0; x < take; ++x) {
            int64_t j = e[x].i;
            int64_t lo = j * P > s_end ? j * P : s_end;
            int64_t hi = (j + 1) * P < l_begin ? (j + 1) * P : l_begin;
            for (int64_t i = lo; i < hi; ++i)
                chosen[i] = 1;
        }
    }
    free(e);
    int64_t m = 0;
    for (int64_t i = 0; i < n; ++i)
        if (chosen[i])
            ids_out[m++] = (int32_t)i;
    free(chosen);
    return m;
}
