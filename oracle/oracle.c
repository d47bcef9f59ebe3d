/*
 * oracle.c -- plain, slow, fp64 CPU reference for exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path calls this file; only the tests, the
 * smoke check and the bench's CPU-baseline leg load it.  It shares no code, header or constant
 * with the CUDA library: it widens the same bf16 input bytes to double and applies the definition.
 *
 * What it computes (the plain definition of attention; "LLM study notes", self-attention steps:
 * dot product of query and key, divide by the square root of the key dimension, softmax, weight V;
 * "Flash Attention" (myungum), section 1: Attention(Q, K, V)).  For every (b, h) and query row i,
 * with the visible key set A_i = {0 .. N-1}, or {0 .. i} when causal
 * ("FlashAttention-2 GPU work partitioning", section 4: the causal mask shows a token only itself
 * and the tokens before it):
 *
 *     s_j  = scale * sum_k Q[i,k] K[j,k]          j in A_i   (one materialised row of S)
 *     m    = max_j s_j,   e_j = exp(s_j - m),   l = sum_j e_j
 *     O[i] = (sum_j e_j V[j,:]) / l
 *     LSE  = m + ln l                             (natural log, in units of the scaled scores)
 *
 * Masked keys are left out of every sum (no -inf arithmetic).  Rows are independent, so the work
 * is split over host threads by whole rows; each row is evaluated exactly as above.
 *
 * oracle_flash_alg1 restates the tiled forward algorithm of "Flash Attention" (myungum), section 2
 * (the pseudocode): outer loop over key/value blocks, inner loop over query blocks, running row
 * max m and row sum l kept beside O "in HBM" and O renormalised at every step.  It exists to pin
 * the online-softmax algebra against the plain definition, for any block sizes.
 *
 * oracle_decode_paged gathers one sequence's keys and values through its block table (a logical
 * block k of sequence s lives in physical block block_table[s][k]; "LLM study notes", paged
 * attention) and applies the same plain row definition to the gathered rows.
 *
 * oracle_prefill_paged does the same for a chunk of Lq queries per sequence: the queries are the
 * last Lq positions of the sequence's L cached tokens ("Paged vs Flash attention": paging for the
 * cache, exact attention for the compute), so query t of the chunk sits at position L - Lq + t and,
 * when causal, sees keys 0 .. L - Lq + t; otherwise all L keys.
 *
 * oracle_tree_attention is the verification step of speculative decoding ("LLM study notes",
 * speculative decoding: the draft model proposes candidate tokens arranged as a tree, and the target
 * model scores every node of the tree in one forward pass with tree attention).  The tree's T
 * nodes are the last T of the sequence's L cached tokens; node t sees the L - T context tokens and
 * the nodes u whose bit u is set in mask[t] (its ancestors and itself, for a tree).  A row that
 * sees no key at all has O = 0 and LSE = -inf.
 *
 * oracle_attention_keyrange and oracle_merge_partials split one sequence's keys into ranges, as
 * the sequence-length parallelism of "FlashAttention-2 GPU work partitioning" (section 3: a long
 * sequence is divided among several workers) does across devices.  The partial of a key range is
 * the plain row definition over the keys of that range the query sees (O = 0 and LSE = -inf when
 * it sees none); partials of disjoint ranges are merged with the rescaling rule of "Flash
 * Attention" (myungum), section 2, steps 11-12, written for log-sum-exps:
 *     M = max_r LSE_r,  w_r = exp(LSE_r - M),  O = sum_r w_r O_r / sum_r w_r,
 *     LSE = M + ln sum_r w_r.
 *
 * oracle_attention_bwd is the backward pass: the gradients of the scalar sum_i dO[i] . O[i] with
 * respect to Q, K and V for a given dO.  The pages describe the backward only in prose ("Paged vs
 * Flash attention", training: gradients from the stored intermediate results, block by block;
 * "LLM study notes" and "Flash Attention" (myungum) section 1: the attention matrix is recomputed
 * rather than stored), so the oracle is the plain definition, the chain rule through the row
 * softmax above, evaluated one query row at a time with the row recomputed from Q and K:
 *
 *     P[i,j]  = e_j / l                       (the row above; masked keys have no entry)
 *     dV[j]  += P[i,j] dO[i]
 *     dP[i,j] = dO[i] . V[j]
 *     dS[i,j] = P[i,j] (dP[i,j] - sum_k P[i,k] dP[i,k])      (the softmax Jacobian)
 *     dQ[i]  += scale dS[i,j] K[j],   dK[j] += scale dS[i,j] Q[i]
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double widen_bf16(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* One query row against n_keys key/value rows given by row pointers.  s is scratch of n_keys. */
static void attend_row(const uint16_t *q, const uint16_t *const *krow, const uint16_t *const *vrow,
                       int64_t n_keys, int d, double scale, double *s, double *o, double *lse)
{
    double m = -INFINITY;
    for (int64_t j = 0; j < n_keys; ++j) {
        double acc = 0.0;
        for (int k = 0; k < d; ++k)
            acc += widen_bf16(q[k]) * widen_bf16(krow[j][k]);
        s[j] = scale * acc;
        if (s[j] > m)
            m = s[j];
    }
    double l = 0.0;
    for (int64_t j = 0; j < n_keys; ++j) {
        s[j] = exp(s[j] - m);
        l += s[j];
    }
    for (int c = 0; c < d; ++c)
        o[c] = 0.0;
    for (int64_t j = 0; j < n_keys; ++j)
        for (int c = 0; c < d; ++c)
            o[c] += s[j] * widen_bf16(vrow[j][c]);
    for (int c = 0; c < d; ++c)
        o[c] /= l;
    if (lse)
        *lse = m + log(l);
}

/* ------------------------------------------------------------------------------------------ */
/* contiguous [B, H, N, d] prefill: all rows, or a list of (bh, row) pairs                      */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
    const uint16_t *q, *k, *v;
    int64_t N;
    int d, causal;
    double scale;
    const int64_t *pairs; /* 2*count entries (bh, row) */
    int64_t count;
    double *o, *lse;      /* o: count x d, lse: count */
    int64_t first, last;  /* this thread's share of [0, count) */
} rows_job;

static void *rows_worker(void *arg)
{
    rows_job *jb = (rows_job *)arg;
    const int d = jb->d;
    const int64_t N = jb->N;
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    const uint16_t **kr = (const uint16_t **)malloc(sizeof(void *) * (size_t)N);
    const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (size_t)N);
    for (int64_t r = jb->first; r < jb->last; ++r) {
        int64_t bh = jb->pairs[2 * r], i = jb->pairs[2 * r + 1];
        const uint16_t *Q = jb->q + bh * N * d, *K = jb->k + bh * N * d, *V = jb->v + bh * N * d;
        int64_t n_keys = jb->causal ? i + 1 : N;
        for (int64_t j = 0; j < n_keys; ++j) {
            kr[j] = K + j * d;
            vr[j] = V + j * d;
        }
        attend_row(Q + i * d, kr, vr, n_keys, d, jb->scale, s, jb->o + r * d, jb->lse + r);
    }
    free(s);
    free(kr);
    free(vr);
    return NULL;
}

/* Rows listed in pairs[2*count] = (bh, i).  o: count x d doubles, lse: count doubles. */
int oracle_attention_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t N, int d,
                          int causal, double scale, const int64_t *pairs, int64_t count,
                          double *o, double *lse, int nthreads)
{
    if (N < 1 || d < 1 || count < 0 || nthreads < 1)
        return 1;
    if (nthreads > count)
        nthreads = count > 0 ? (int)count : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    rows_job *jobs = (rows_job *)malloc(sizeof(rows_job) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) {
        rows_job j = {q, k, v, N, d, causal, scale, pairs, count, o, lse,
                      count * t / nthreads, count * (t + 1) / nthreads};
        jobs[t] = j;
        pthread_create(&th[t], NULL, rows_worker, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t)
        pthread_join(th[t], NULL);
    free(th);
    free(jobs);
    return 0;
}

/* Every row of every head: o [B*H, N, d], lse [B*H, N]. */
int oracle_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t BH, int64_t N,
                     int d, int causal, double scale, double *o, double *lse, int nthreads)
{
    int64_t count = BH * N;
    int64_t *pairs = (int64_t *)malloc(sizeof(int64_t) * 2 * (size_t)count);
    for (int64_t bh = 0; bh < BH; ++bh)
        for (int64_t i = 0; i < N; ++i) {
            pairs[2 * (bh * N + i)] = bh;
            pairs[2 * (bh * N + i) + 1] = i;
        }
    int rc = oracle_attention_rows(q, k, v, N, d, causal, scale, pairs, count, o, lse, nthreads);
    free(pairs);
    return rc;
}

/* The full probability matrix P (N x N, masked entries 0) of one head, for row-sum checks. */
int oracle_attention_probs(const uint16_t *q, const uint16_t *k, int64_t N, int d, int causal,
                           double scale, double *P)
{
    for (int64_t i = 0; i < N; ++i) {
        double *row = P + i * N;
        int64_t n_keys = causal ? i + 1 : N;
        double m = -INFINITY;
        for (int64_t j = 0; j < n_keys; ++j) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += widen_bf16(q[i * d + c]) * widen_bf16(k[j * d + c]);
            row[j] = scale * acc;
            if (row[j] > m)
                m = row[j];
        }
        double l = 0.0;
        for (int64_t j = 0; j < n_keys; ++j) {
            row[j] = exp(row[j] - m);
            l += row[j];
        }
        for (int64_t j = 0; j < n_keys; ++j)
            row[j] /= l;
        for (int64_t j = n_keys; j < N; ++j)
            row[j] = 0.0;
    }
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* The tiled algorithm as the pseudocode states it, one head, block sizes Br x Bc              */
/* ------------------------------------------------------------------------------------------ */

/*
 * Steps, in the page's order and notation (scale folded into S; causal keys j > i excluded):
 *   init O = 0 (N x d), l = 0 (N), m = -inf (N)
 *   split Q into T_r blocks of Br rows, K and V into T_c blocks of Bc rows (last ones ragged)
 *   for each key/value block j:
 *     for each query block i:
 *       S_ij = scale * Q_i K_j^T
 *       per row r: mt = rowmax(S_ij), Pt = exp(S_ij - mt), lt = rowsum(Pt)
 *                  m_new = max(m, mt), l_new = exp(m - m_new) l + exp(mt - m_new) lt
 *                  O_r <- (l exp(m - m_new) O_r + exp(mt - m_new) (Pt V_j)_r) / l_new
 *                  l <- l_new, m <- m_new
 * A row whose keys in block j are all masked has no entries: it is left unchanged.
 * l and m are returned as well; LSE = m + ln l.
 */
int oracle_flash_alg1(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t N, int d,
                      int causal, double scale, int Br, int Bc, double *O, double *l, double *m)
{
    if (Br < 1 || Bc < 1 || N < 1 || d < 1)
        return 1;
    for (int64_t i = 0; i < N * d; ++i)
        O[i] = 0.0;
    for (int64_t i = 0; i < N; ++i) {
        l[i] = 0.0;
        m[i] = -INFINITY;
    }
    int64_t Tr = (N + Br - 1) / Br, Tc = (N + Bc - 1) / Bc;
    double *S = (double *)malloc(sizeof(double) * (size_t)Br * (size_t)Bc);
    double *PV = (double *)malloc(sizeof(double) * (size_t)d);
    for (int64_t j = 0; j < Tc; ++j) {
        int64_t k0 = j * Bc, kn = (k0 + Bc <= N) ? Bc : N - k0;
        for (int64_t i = 0; i < Tr; ++i) {
            int64_t q0 = i * Br, qn = (q0 + Br <= N) ? Br : N - q0;
            for (int64_t r = 0; r < qn; ++r) {
                int64_t qi = q0 + r;
                /* S_ij row r; visible keys of this block */
                int64_t vis = kn;
                if (causal) {
                    int64_t last = qi - k0; /* last visible column in this block */
                    if (last < 0)
                        continue; /* whole block masked for this row */
                    if (last + 1 < vis)
                        vis = last + 1;
                }
                double mt = -INFINITY;
                for (int64_t c = 0; c < vis; ++c) {
                    double acc = 0.0;
                    for (int e = 0; e < d; ++e)
                        acc += widen_bf16(q[qi * d + e]) * widen_bf16(k[(k0 + c) * d + e]);
                    S[r * Bc + c] = scale * acc;
                    if (S[r * Bc + c] > mt)
                        mt = S[r * Bc + c];
                }
                double lt = 0.0;
                for (int e = 0; e < d; ++e)
                    PV[e] = 0.0;
                for (int64_t c = 0; c < vis; ++c) {
                    double p = exp(S[r * Bc + c] - mt);
                    lt += p;
                    for (int e = 0; e < d; ++e)
                        PV[e] += p * widen_bf16(v[(k0 + c) * d + e]);
                }
                double m_new = m[qi] > mt ? m[qi] : mt;
                double a_old = exp(m[qi] - m_new); /* exp(-inf) = 0 on the first visible block */
                double a_new = exp(mt - m_new);
                double l_new = a_old * l[qi] + a_new * lt;
                for (int e = 0; e < d; ++e)
                    O[qi * d + e] = (l[qi] * a_old * O[qi * d + e] + a_new * PV[e]) / l_new;
                l[qi] = l_new;
                m[qi] = m_new;
            }
        }
    }
    free(S);
    free(PV);
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* paged decode: one query per sequence, keys/values gathered through the block table          */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
    const uint16_t *q, *kp, *vp;
    const int32_t *table, *lens;
    int max_blocks, H, d, page;
    double scale;
    double *o, *lse;
    int64_t first, last; /* range of (s, h) units */
} dec_job;

static void *dec_worker(void *arg)
{
    dec_job *jb = (dec_job *)arg;
    const int H = jb->H, d = jb->d, page = jb->page;
    int64_t maxlen = (int64_t)jb->max_blocks * page;
    double *s = (double *)malloc(sizeof(double) * (size_t)maxlen);
    const uint16_t **kr = (const uint16_t **)malloc(sizeof(void *) * (size_t)maxlen);
    const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (size_t)maxlen);
    for (int64_t u = jb->first; u < jb->last; ++u) {
        int64_t sq = u / H, h = u % H;
        int64_t L = jb->lens[sq];
        for (int64_t t = 0; t < L; ++t) {
            int64_t blk = jb->table[sq * jb->max_blocks + t / page];
            int64_t off = ((blk * H + h) * page + t % page) * d;
            kr[t] = jb->kp + off;
            vr[t] = jb->vp + off;
        }
        attend_row(jb->q + (sq * H + h) * d, kr, vr, L, d, jb->scale, s, jb->o + u * d, jb->lse + u);
    }
    free(s);
    free(kr);
    free(vr);
    return NULL;
}

/* q [S,H,d]; pools [num_blocks,H,page,d]; table [S,max_blocks]; o [S,H,d]; lse [S,H]. */
int oracle_decode_paged(const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                        const int32_t *block_table, int max_blocks, const int32_t *seq_lens, int S,
                        int H, int d, int page, double scale, double *o, double *lse, int nthreads)
{
    if (S < 1 || H < 1 || d < 1 || page < 1 || max_blocks < 1 || nthreads < 1)
        return 1;
    for (int s = 0; s < S; ++s)
        if (seq_lens[s] < 1 || seq_lens[s] > (int64_t)max_blocks * page)
            return 1;
    int64_t units = (int64_t)S * H;
    if (nthreads > units)
        nthreads = (int)units;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    dec_job *jobs = (dec_job *)malloc(sizeof(dec_job) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) {
        dec_job j = {q, k_pool, v_pool, block_table, seq_lens, max_blocks, H, d, page, scale,
                     o, lse, units * t / nthreads, units * (t + 1) / nthreads};
        jobs[t] = j;
        pthread_create(&th[t], NULL, dec_worker, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t)
        pthread_join(th[t], NULL);
    free(th);
    free(jobs);
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* chunked prefill over a paged cache: Lq queries per sequence, the last Lq of its L tokens     */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
    const uint16_t *q, *kp, *vp;
    const int32_t *table, *lens;
    int max_blocks, H, Lq, d, page, causal;
    double scale;
    double *o, *lse;
    int64_t first, last; /* range of (s, h, t) rows */
} pf_job;

static void *pf_worker(void *arg)
{
    pf_job *jb = (pf_job *)arg;
    const int H = jb->H, d = jb->d, page = jb->page, Lq = jb->Lq;
    int64_t maxlen = (int64_t)jb->max_blocks * page;
    double *s = (double *)malloc(sizeof(double) * (size_t)maxlen);
    const uint16_t **kr = (const uint16_t **)malloc(sizeof(void *) * (size_t)maxlen);
    const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (size_t)maxlen);
    for (int64_t r = jb->first; r < jb->last; ++r) {
        int64_t t = r % Lq, u = r / Lq, sq = u / H, h = u % H;
        int64_t L = jb->lens[sq];
        int64_t n_keys = jb->causal ? L - Lq + t + 1 : L;
        for (int64_t k = 0; k < n_keys; ++k) {
            int64_t blk = jb->table[sq * jb->max_blocks + k / page];
            int64_t off = ((blk * H + h) * page + k % page) * d;
            kr[k] = jb->kp + off;
            vr[k] = jb->vp + off;
        }
        attend_row(jb->q + r * d, kr, vr, n_keys, d, jb->scale, s, jb->o + r * d, jb->lse + r);
    }
    free(s);
    free(kr);
    free(vr);
    return NULL;
}

/* q [S,H,Lq,d]; pools [num_blocks,H,page,d]; table [S,max_blocks]; lens [S] (each >= Lq);
 * o [S,H,Lq,d]; lse [S,H,Lq]. */
int oracle_prefill_paged(const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                         const int32_t *block_table, int max_blocks, const int32_t *seq_lens, int S,
                         int H, int Lq, int d, int page, int causal, double scale, double *o,
                         double *lse, int nthreads)
{
    if (S < 1 || H < 1 || Lq < 1 || d < 1 || page < 1 || max_blocks < 1 || nthreads < 1)
        return 1;
    for (int s = 0; s < S; ++s)
        if (seq_lens[s] < Lq || seq_lens[s] > (int64_t)max_blocks * page)
            return 1;
    int64_t rows = (int64_t)S * H * Lq;
    if (nthreads > rows)
        nthreads = (int)rows;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    pf_job *jobs = (pf_job *)malloc(sizeof(pf_job) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) {
        pf_job j = {q, k_pool, v_pool, block_table, seq_lens, max_blocks, H, Lq, d, page, causal,
                    scale, o, lse, rows * t / nthreads, rows * (t + 1) / nthreads};
        jobs[t] = j;
        pthread_create(&th[t], NULL, pf_worker, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t)
        pthread_join(th[t], NULL);
    free(th);
    free(jobs);
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* backward: dQ, dK, dV of one head at a time (heads are independent)                          */
/* ------------------------------------------------------------------------------------------ */

/* One head: Q, K, V, dO [N, d]; dq, dk, dv [N, d] (overwritten).  p, dp: scratch of N. */
static void bwd_head(const uint16_t *Q, const uint16_t *K, const uint16_t *V, const uint16_t *dO,
                     int64_t N, int d, int causal, double scale, double *dq, double *dk,
                     double *dv, double *p, double *dp)
{
    for (int64_t e = 0; e < N * d; ++e) {
        dq[e] = 0.0;
        dk[e] = 0.0;
        dv[e] = 0.0;
    }
    for (int64_t i = 0; i < N; ++i) {
        const int64_t n_keys = causal ? i + 1 : N; /* the keys row i sees */
        const uint16_t *qi = Q + i * d, *doi = dO + i * d;
        /* the probability row, recomputed */
        double m = -INFINITY;
        for (int64_t j = 0; j < n_keys; ++j) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += widen_bf16(qi[c]) * widen_bf16(K[j * d + c]);
            p[j] = scale * acc;
            if (p[j] > m)
                m = p[j];
        }
        double l = 0.0;
        for (int64_t j = 0; j < n_keys; ++j) {
            p[j] = exp(p[j] - m);
            l += p[j];
        }
        for (int64_t j = 0; j < n_keys; ++j)
            p[j] /= l;
        /* dP row and its P-weighted mean */
        double pdp = 0.0;
        for (int64_t j = 0; j < n_keys; ++j) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c)
                acc += widen_bf16(doi[c]) * widen_bf16(V[j * d + c]);
            dp[j] = acc;
            pdp += p[j] * acc;
        }
        for (int64_t j = 0; j < n_keys; ++j) {
            double ds = p[j] * (dp[j] - pdp);
            for (int c = 0; c < d; ++c) {
                dv[j * d + c] += p[j] * widen_bf16(doi[c]);
                dq[i * d + c] += scale * ds * widen_bf16(K[j * d + c]);
                dk[j * d + c] += scale * ds * widen_bf16(qi[c]);
            }
        }
    }
}

typedef struct {
    const uint16_t *q, *k, *v, *dout;
    int64_t N;
    int d, causal;
    double scale;
    const int64_t *heads;
    double *dq, *dk, *dv; /* [nheads, N, d] */
    int64_t first, last;  /* this thread's share of the head list */
} bwd_job;

static void *bwd_worker(void *arg)
{
    bwd_job *jb = (bwd_job *)arg;
    const int64_t N = jb->N;
    const int d = jb->d;
    double *p = (double *)malloc(sizeof(double) * (size_t)N);
    double *dp = (double *)malloc(sizeof(double) * (size_t)N);
    for (int64_t t = jb->first; t < jb->last; ++t) {
        int64_t off = jb->heads[t] * N * d, out = t * N * d;
        bwd_head(jb->q + off, jb->k + off, jb->v + off, jb->dout + off, N, d, jb->causal,
                 jb->scale, jb->dq + out, jb->dk + out, jb->dv + out, p, dp);
    }
    free(p);
    free(dp);
    return NULL;
}

/* q, k, v, dout [BH, N, d]; the heads listed in heads[nheads] (indices into BH) are
 * differentiated; dq, dk, dv [nheads, N, d]. */
int oracle_attention_bwd(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         const uint16_t *dout, int64_t N, int d, int causal, double scale,
                         const int64_t *heads, int64_t nheads, double *dq, double *dk, double *dv,
                         int nthreads)
{
    if (N < 1 || d < 1 || nheads < 1 || nthreads < 1)
        return 1;
    if (nthreads > nheads)
        nthreads = (int)nheads;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    bwd_job *jobs = (bwd_job *)malloc(sizeof(bwd_job) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) {
        bwd_job j = {q, k, v, dout, N, d, causal, scale, heads, dq, dk, dv,
                     nheads * t / nthreads, nheads * (t + 1) / nthreads};
        jobs[t] = j;
        pthread_create(&th[t], NULL, bwd_worker, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t)
        pthread_join(th[t], NULL);
    free(th);
    free(jobs);
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* tree attention: T draft nodes per sequence, visibility of the tree part given by bit masks  */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
    const uint16_t *q, *kp, *vp;
    const int32_t *table, *lens;
    const uint64_t *mask;
    int max_blocks, H, T, d, page;
    double scale;
    double *o, *lse;
    int64_t first, last; /* range of (s, h, t) rows */
} tree_job;

static void *tree_worker(void *arg)
{
    tree_job *jb = (tree_job *)arg;
    const int H = jb->H, d = jb->d, page = jb->page, T = jb->T;
    int64_t maxlen = (int64_t)jb->max_blocks * page;
    double *s = (double *)malloc(sizeof(double) * (size_t)maxlen);
    const uint16_t **kr = (const uint16_t **)malloc(sizeof(void *) * (size_t)maxlen);
    const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (size_t)maxlen);
    for (int64_t r = jb->first; r < jb->last; ++r) {
        int64_t t = r % T, u = r / T, sq = u / H, h = u % H;
        int64_t L = jb->lens[sq], ctx = L - T;
        uint64_t m = jb->mask[sq * T + t];
        int64_t n_keys = 0;
        for (int64_t key = 0; key < L; ++key) {
            if (key >= ctx && !((m >> (key - ctx)) & 1u))
                continue; /* a tree node this one does not see */
            int64_t blk = jb->table[sq * jb->max_blocks + key / page];
            int64_t off = ((blk * H + h) * page + key % page) * d;
            kr[n_keys] = jb->kp + off;
            vr[n_keys] = jb->vp + off;
            ++n_keys;
        }
        if (n_keys == 0) {
            for (int c = 0; c < d; ++c)
                jb->o[r * d + c] = 0.0;
            jb->lse[r] = -INFINITY;
            continue;
        }
        const uint16_t *node_q = jb->q + r * d;
        attend_row(node_q, kr, vr, n_keys, d, jb->scale, s, jb->o + r * d, jb->lse + r);
    }
    free(s);
    free(kr);
    free(vr);
    return NULL;
}

/* q [S,H,T,d]; pools [num_blocks,H,page,d]; table [S,max_blocks]; lens [S] (each >= T);
 * mask [S,T] (bit u of mask[s*T+t]: node t sees node u; T <= 64); o [S,H,T,d]; lse [S,H,T]. */
int oracle_tree_attention(const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                          const int32_t *block_table, int max_blocks, const int32_t *seq_lens,
                          const uint64_t *mask, int S, int H, int T, int d, int page, double scale,
                          double *o, double *lse, int nthreads)
{
    if (S < 1 || H < 1 || T < 1 || T > 64 || d < 1 || page < 1 || max_blocks < 1 || nthreads < 1)
        return 1;
    for (int s = 0; s < S; ++s)
        if (seq_lens[s] < T || seq_lens[s] > (int64_t)max_blocks * page)
            return 1;
    int64_t rows = (int64_t)S * H * T;
    if (nthreads > rows)
        nthreads = (int)rows;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    tree_job *jobs = (tree_job *)malloc(sizeof(tree_job) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) {
        tree_job j = {q, k_pool, v_pool, block_table, seq_lens, mask, max_blocks, H, T, d, page,
                      scale, o, lse, rows * t / nthreads, rows * (t + 1) / nthreads};
        jobs[t] = j;
        pthread_create(&th[t], NULL, tree_worker, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t)
        pthread_join(th[t], NULL);
    free(th);
    free(jobs);
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* key-range partials and their merge                                                          */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
    const uint16_t *q, *k, *v;
    int64_t Nq, Nk, q0, k0;
    int d, causal;
    double scale;
    double *o, *lse;
    int64_t first, last; /* range of (bh, row) rows */
} kr_job;

static void *kr_worker(void *arg)
{
    kr_job *jb = (kr_job *)arg;
    const int d = jb->d;
    double *s = (double *)malloc(sizeof(double) * (size_t)(jb->Nk > 0 ? jb->Nk : 1));
    const uint16_t **kr = (const uint16_t **)malloc(sizeof(void *) * (size_t)(jb->Nk > 0 ? jb->Nk : 1));
    const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (size_t)(jb->Nk > 0 ? jb->Nk : 1));
    for (int64_t r = jb->first; r < jb->last; ++r) {
        int64_t bh = r / jb->Nq, i = r % jb->Nq;
        /* query at position q0 + i sees the range's keys at positions k0 + c <= q0 + i */
        int64_t n_keys = jb->Nk;
        if (jb->causal) {
            int64_t last = jb->q0 + i - jb->k0;
            n_keys = last < 0 ? 0 : (last + 1 < jb->Nk ? last + 1 : jb->Nk);
        }
        if (n_keys == 0) {
            for (int c = 0; c < d; ++c)
                jb->o[r * d + c] = 0.0;
            jb->lse[r] = -INFINITY;
            continue;
        }
        const uint16_t *K = jb->k + bh * jb->Nk * d, *V = jb->v + bh * jb->Nk * d;
        for (int64_t c = 0; c < n_keys; ++c) {
            kr[c] = K + c * d;
            vr[c] = V + c * d;
        }
        const uint16_t *qi = jb->q + r * d;
        attend_row(qi, kr, vr, n_keys, d, jb->scale, s, jb->o + r * d, jb->lse + r);
    }
    free(s);
    free(kr);
    free(vr);
    return NULL;
}

/* q [BH, Nq, d] (positions q0 .. q0+Nq-1), k, v [BH, Nk, d] (positions k0 .. k0+Nk-1);
 * o [BH, Nq, d], lse [BH, Nq]. */
int oracle_attention_keyrange(const uint16_t *q, const uint16_t *k, const uint16_t *v, int64_t BH,
                              int64_t Nq, int64_t Nk, int64_t q0, int64_t k0, int d, int causal,
                              double scale, double *o, double *lse, int nthreads)
{
    if (BH < 1 || Nq < 1 || Nk < 0 || d < 1 || nthreads < 1)
        return 1;
    int64_t rows = BH * Nq;
    if (nthreads > rows)
        nthreads = (int)rows;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    kr_job *jobs = (kr_job *)malloc(sizeof(kr_job) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) {
        kr_job j = {q, k, v, Nq, Nk, q0, k0, d, causal, scale, o, lse,
                    rows * t / nthreads, rows * (t + 1) / nthreads};
        jobs[t] = j;
        pthread_create(&th[t], NULL, kr_worker, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t)
        pthread_join(th[t], NULL);
    free(th);
    free(jobs);
    return 0;
}

/* o_parts [G, rows, d], lse_parts [G, rows] -> o [rows, d], lse [rows]. */
int oracle_merge_partials(const double *o_parts, const double *lse_parts, int G, int64_t rows,
                          int d, double *o, double *lse)
{
    if (G < 1 || rows < 0 || d < 1)
        return 1;
    for (int64_t r = 0; r < rows; ++r) {
        double M = -INFINITY;
        for (int g = 0; g < G; ++g)
            if (lse_parts[g * rows + r] > M)
                M = lse_parts[g * rows + r];
        for (int c = 0; c < d; ++c)
            o[r * d + c] = 0.0;
        if (M == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double wsum = 0.0;
        for (int g = 0; g < G; ++g) {
            double w = exp(lse_parts[g * rows + r] - M);
            wsum += w;
            for (int c = 0; c < d; ++c)
                o[r * d + c] += w * o_parts[(g * rows + r) * d + c];
        }
        for (int c = 0; c < d; ++c)
            o[r * d + c] /= wsum;
        lse[r] = M + log(wsum);
    }
    return 0;
}
