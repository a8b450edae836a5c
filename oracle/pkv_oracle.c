/*
 * Paged GQA decode attention: the CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference legs use it.  It shares no code, header, table or
 * constant with the CUDA library; the two see the same inputs and nothing else.
 *
 * What it computes is the plain definition, written out in fp64 with plain
 * loops and no blocking, fusion or online rescaling:
 *
 *   for every sequence (row) i, query head hq and KV head h = floor(hq / G),
 *   with G = H_q / H_kv query heads sharing one KV head
 *     [PersistentKV: Page-Aware Decode Scheduling for Long-Context LLM Serving
 *      on Commodity GPUs (gist.science explainer), Technical summary >
 *      Methodology > 1 "Native block-table decode engine": GQA grouping],
 *   for every cached token t = 0 .. N_i - 1, read through the block table
 *     page = block_table[i][t / P], slot = t mod P
 *     [same page, Methodology 1 "Layout": run on the paged layout, no repack;
 *      "Chapter 8 - Next-generation KV cache management" (actionbridge.io),
 *      section 8.1: block table maps logical block -> physical block id;
 *      "How does paged attention manage the KV cache for concurrent local AI
 *      requests?" (zimaspace), section "PagedAttention splits KV state into
 *      fixed-size blocks": indirection changes placement, not token order],
 *     s_t = scale * sum_d q[i][hq][d] * k_t[d]
 *   out[i][hq][:] = sum_t softmax(s)_t * v_t     (two passes: max, then sums)
 *
 * A row with N_i = 0 has no tokens; its output is zero (reading of the pages,
 * which only say that an empty split writes a neutral state).
 *
 * The split/merge pair below follows Methodology 1 "Sequence splitting": each
 * disjoint token range yields a partial softmax state (max m, denominator l,
 * accumulator acc) and a merge combines the states exactly.  It exists so the
 * tests can check that splitting is exact; the oracle's decode itself never
 * splits.
 *
 * Inputs are the raw bf16 bit patterns (uint16); bf16 -> double is exact.
 * Pools are addressed by element strides (page, head, token); the head_dim
 * stride is 1.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

typedef struct {
    const uint16_t *q;         /* [B][H_q][D] */
    const uint16_t *k_pool;    /* element (page, head, slot, d) at page*s_page + head*s_head + slot*s_tok + d */
    const uint16_t *v_pool;
    int64_t s_page, s_head, s_tok;
    const int32_t *block_table; /* [B][max_pages] */
    int32_t max_pages;
    const int32_t *seq_lens;    /* [B] */
    int32_t B, H_q, H_kv, D, P;
    double scale;
} problem;

static const uint16_t *kv_row(const problem *pr, const uint16_t *pool, int row, int h, int t)
{
    int32_t page = pr->block_table[(int64_t)row * pr->max_pages + t / pr->P];
    int32_t slot = t % pr->P;
    return pool + (int64_t)page * pr->s_page + (int64_t)h * pr->s_head + (int64_t)slot * pr->s_tok;
}

/* GQA: G = H_q / H_kv consecutive query heads share one KV head */
static int kv_head_of(const problem *pr, int hq)
{
    int G = pr->H_q / pr->H_kv;
    return hq / G;
}

/* logit of token t for (row, hq) */
static double logit(const problem *pr, int row, int hq, int t)
{
    int h = kv_head_of(pr, hq);
    const uint16_t *qv = pr->q + ((int64_t)row * pr->H_q + hq) * pr->D;
    const uint16_t *kv = kv_row(pr, pr->k_pool, row, h, t);
    double dot = 0.0;
    for (int d = 0; d < pr->D; ++d)
        dot += bf16_bits_to_double(qv[d]) * bf16_bits_to_double(kv[d]);
    return pr->scale * dot;
}

/* Full softmax-weighted sum for one (row, query head).  Returns 0 on success. */
static int decode_one(const problem *pr, int row, int hq, double *out)
{
    int N = pr->seq_lens[row];
    int h = kv_head_of(pr, hq);
    for (int d = 0; d < pr->D; ++d)
        out[d] = 0.0;
    if (N <= 0)
        return 0;
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    if (!s)
        return -1;
    double M = -INFINITY;
    for (int t = 0; t < N; ++t) {
        s[t] = logit(pr, row, hq, t);
        if (s[t] > M)
            M = s[t];
    }
    double Z = 0.0;
    for (int t = 0; t < N; ++t) {
        double w = exp(s[t] - M);
        Z += w;
        const uint16_t *vv = kv_row(pr, pr->v_pool, row, h, t);
        for (int d = 0; d < pr->D; ++d)
            out[d] += w * bf16_bits_to_double(vv[d]);
    }
    for (int d = 0; d < pr->D; ++d)
        out[d] /= Z;
    free(s);
    return 0;
}

typedef struct {
    const problem *pr;
    const int32_t *pairs; /* (row, hq) list, or NULL for all B*H_q in order */
    int64_t n_pairs;
    double *out;          /* [n_pairs][D] */
    int tid, n_threads;
    int status;
} worker_arg;

static void *worker(void *p)
{
    worker_arg *a = (worker_arg *)p;
    a->status = 0;
    for (int64_t i = a->tid; i < a->n_pairs; i += a->n_threads) {
        int row, hq;
        if (a->pairs) {
            row = a->pairs[2 * i];
            hq = a->pairs[2 * i + 1];
        } else {
            row = (int)(i / a->pr->H_q);
            hq = (int)(i % a->pr->H_q);
        }
        if (decode_one(a->pr, row, hq, a->out + i * a->pr->D) != 0)
            a->status = -1;
    }
    return NULL;
}

static int run_pairs(const problem *pr, const int32_t *pairs, int64_t n_pairs, double *out, int n_threads)
{
    if (n_threads < 1)
        n_threads = 1;
    if (n_threads > 256)
        n_threads = 256;
    pthread_t th[256];
    worker_arg args[256];
    int status = 0;
    for (int i = 0; i < n_threads; ++i) {
        args[i] = (worker_arg){pr, pairs, n_pairs, out, i, n_threads, 0};
        if (i > 0 && pthread_create(&th[i], NULL, worker, &args[i]) != 0)
            return -1;
    }
    worker(&args[0]);
    for (int i = 1; i < n_threads; ++i)
        pthread_join(th[i], NULL);
    for (int i = 0; i < n_threads; ++i)
        if (args[i].status != 0)
            status = -1;
    return status;
}

static int check_problem(const problem *pr)
{
    if (pr->B < 0 || pr->H_q <= 0 || pr->H_kv <= 0 || pr->D <= 0 || pr->P <= 0)
        return -1;
    if (pr->H_q % pr->H_kv != 0)
        return -1;
    for (int i = 0; i < pr->B; ++i)
        if (pr->seq_lens[i] > (int64_t)pr->max_pages * pr->P)
            return -1;
    return 0;
}

#define PROBLEM_INIT                                                                      \
    problem pr = {q, k_pool, v_pool, s_page, s_head, s_tok, block_table, max_pages, seq_lens, \
                  B, H_q, H_kv, D, P, scale}

/* out: [B][H_q][D] doubles.  Threads split the (row, hq) pairs; every pair is
 * computed by the same sequential code, so the result does not depend on the
 * thread count. */
int oracle_paged_decode(const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                        int64_t s_page, int64_t s_head, int64_t s_tok,
                        const int32_t *block_table, int32_t max_pages, const int32_t *seq_lens,
                        int32_t B, int32_t H_q, int32_t H_kv, int32_t D, int32_t P,
                        double scale, double *out, int32_t n_threads)
{
    PROBLEM_INIT;
    if (check_problem(&pr) != 0)
        return -1;
    return run_pairs(&pr, NULL, (int64_t)B * H_q, out, n_threads);
}

/* Only the listed (row, hq) pairs: pairs is [n_pairs][2], out is [n_pairs][D]. */
int oracle_paged_decode_pairs(const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                              int64_t s_page, int64_t s_head, int64_t s_tok,
                              const int32_t *block_table, int32_t max_pages, const int32_t *seq_lens,
                              int32_t B, int32_t H_q, int32_t H_kv, int32_t D, int32_t P,
                              double scale, const int32_t *pairs, int64_t n_pairs, double *out,
                              int32_t n_threads)
{
    PROBLEM_INIT;
    if (check_problem(&pr) != 0)
        return -1;
    for (int64_t i = 0; i < n_pairs; ++i)
        if (pairs[2 * i] < 0 || pairs[2 * i] >= B || pairs[2 * i + 1] < 0 || pairs[2 * i + 1] >= H_q)
            return -1;
    return run_pairs(&pr, pairs, n_pairs, out, n_threads);
}

/* Partial softmax state of one token range [tok_begin, tok_end) of (row, hq):
 *   m = max_t s_t, l = sum_t exp(s_t - m), acc = sum_t exp(s_t - m) v_t.
 * An empty range gives the neutral state m = -inf, l = 0, acc = 0. */
int oracle_partial_state(const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                         int64_t s_page, int64_t s_head, int64_t s_tok,
                         const int32_t *block_table, int32_t max_pages, const int32_t *seq_lens,
                         int32_t B, int32_t H_q, int32_t H_kv, int32_t D, int32_t P,
                         double scale, int32_t row, int32_t hq, int32_t tok_begin, int32_t tok_end,
                         double *m_out, double *l_out, double *acc_out)
{
    PROBLEM_INIT;
    if (check_problem(&pr) != 0 || row < 0 || row >= B || hq < 0 || hq >= H_q)
        return -1;
    if (tok_begin < 0 || tok_end > seq_lens[row])
        return -1;
    int h = kv_head_of(&pr, hq);
    for (int d = 0; d < D; ++d)
        acc_out[d] = 0.0;
    *m_out = -INFINITY;
    *l_out = 0.0;
    if (tok_end <= tok_begin)
        return 0;
    double m = -INFINITY;
    for (int t = tok_begin; t < tok_end; ++t) {
        double s = logit(&pr, row, hq, t);
        if (s > m)
            m = s;
    }
    double l = 0.0;
    for (int t = tok_begin; t < tok_end; ++t) {
        double w = exp(logit(&pr, row, hq, t) - m);
        l += w;
        const uint16_t *vv = kv_row(&pr, v_pool, row, h, t);
        for (int d = 0; d < D; ++d)
            acc_out[d] += w * bf16_bits_to_double(vv[d]);
    }
    *m_out = m;
    *l_out = l;
    return 0;
}

/* Exact merge of n partial states (m[i], l[i], acc[i][0..D-1]):
 *   M = max_i m_i, w_i = exp(m_i - M) (0 for a neutral state),
 *   out = sum_i w_i acc_i / sum_i w_i l_i,  and 0 when every state is neutral. */
int oracle_merge_states(int32_t n, const double *m, const double *l, const double *acc, int32_t D,
                        double *out)
{
    double M = -INFINITY;
    for (int i = 0; i < n; ++i)
        if (m[i] > M)
            M = m[i];
    for (int d = 0; d < D; ++d)
        out[d] = 0.0;
    if (M == -INFINITY)
        return 0;
    double L = 0.0;
    for (int i = 0; i < n; ++i) {
        if (m[i] == -INFINITY)
            continue;
        double w = exp(m[i] - M);
        L += w * l[i];
        for (int d = 0; d < D; ++d)
            out[d] += w * acc[(int64_t)i * D + d];
    }
    for (int d = 0; d < D; ++d)
        out[d] /= L;
    return 0;
}
