/*
 * moba_oracle.c -- plain fp64 CPU oracle for the MoBA causal prefill forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * helper with the CUDA library; the two meet only in the seeded input
 * generator, which holds none of the method's arithmetic.
 *
 * What it computes (MoBA: Mixture of Block Attention for Long-Context LLMs):
 *   - block partition of each sequence into contiguous blocks of B keys,
 *     the last block of a sequence possibly partial
 *     (wispaper.ai blog, "The Change": block partition; sherconan.github.io,
 *     step 1 "block partition");
 *   - one mean-pooled key per block
 *     (wispaper.ai blog, "The Change": affinity equation;
 *     sherconan.github.io step 2 "parameter-free gating");
 *   - affinity s_j = <q, Kbar_j>, unscaled, for every past block j
 *     (same passages);
 *   - hard top-k gate over the past blocks, the query's own block always
 *     selected and counted toward k, future blocks never selected, ties to
 *     the lower block index, and all blocks taken when fewer than k exist
 *     (wispaper.ai blog, "The Change": routing rule and causality rule;
 *     sherconan.github.io steps 3 and 4);
 *   - exact softmax attention with scale 1/sqrt(d) over the union I of the
 *     selected blocks, causal inside the own block
 *     (wispaper.ai blog, "Starting Point" and "The Change";
 *     globaladvisors.biz, "Underlying computational mechanism");
 *   - the log-sum-exp of the scaled logits over I (natural log);
 *   - the backward of that attention over a fixed selection (dQ, dK, dV for
 *     an output gradient dO): no gradient passes through the hard gate
 *     (wispaper.ai blog, "The Change").
 *
 * The attention is evaluated directly over I, never block by block, so the
 * GPU's block-wise online-softmax merge is checked against a result that
 * does not use it.
 *
 * Precision: inputs are bf16 bit patterns, converted exactly to double; all
 * arithmetic is IEEE double; nothing is rounded back.
 *
 * Token layout: packed [T][H][d] for q, k, v; sequences given by cu[0..nseq]
 * (cu[0] = 0, cu[nseq] = T).  A batch of b sequences of length N is the
 * special case cu = {0, N, 2N, ..., bN}.  Query head h reads kv head
 * h / (Hq / Hkv) (contiguous grouping).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_EINVAL 1
#define ORC_ENOMEM 2
#define ORC_EFUTURE 3 /* a selection names a block after the query's own */

static double bf16_bits_to_double(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Number of blocks of sequence s: ceil(len / B). */
static int64_t seq_blocks(const int64_t *cu, int s, int B)
{
    int64_t len = cu[s + 1] - cu[s];
    return (len + B - 1) / B;
}

/* Sequence holding global token t (cu ascending). */
static int seq_of(const int64_t *cu, int nseq, int64_t t)
{
    int lo = 0, hi = nseq - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (cu[mid] <= t)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

static int check_common(const int64_t *cu, int nseq, int Hq, int Hkv, int d, int B)
{
    if (!cu || nseq <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || B <= 0)
        return ORC_EINVAL;
    if (Hq % Hkv)
        return ORC_EINVAL;
    if (cu[0] != 0)
        return ORC_EINVAL;
    for (int s = 0; s < nseq; ++s)
        if (cu[s + 1] < cu[s])
            return ORC_EINVAL;
    return ORC_OK;
}

/* Total block count over all sequences, and per-sequence first block. */
int64_t oracle_total_blocks(const int64_t *cu, int nseq, int B)
{
    int64_t nb = 0;
    for (int s = 0; s < nseq; ++s)
        nb += seq_blocks(cu, s, B);
    return nb;
}

/*
 * Mean-pooled block keys.  Kbar layout [Hkv][NB][d], blocks numbered
 * sequence by sequence (block j of sequence s is global block
 * first_block(s) + j).  The mean is over the tokens present in the block.
 */
int oracle_block_means(const uint16_t *K, const int64_t *cu, int nseq, int Hkv, int d,
                       int B, double *Kbar)
{
    if (check_common(cu, nseq, Hkv, Hkv, d, B) || !K || !Kbar)
        return ORC_EINVAL;
    int64_t NB = oracle_total_blocks(cu, nseq, B);
    int64_t *first = (int64_t *)malloc(sizeof(int64_t) * (size_t)(nseq + 1));
    if (!first)
        return ORC_ENOMEM;
    first[0] = 0;
    for (int s = 0; s < nseq; ++s)
        first[s + 1] = first[s] + seq_blocks(cu, s, B);

#pragma omp parallel for schedule(dynamic)
    for (int64_t gb = 0; gb < NB * Hkv; ++gb) {
        int g = (int)(gb / NB);
        int64_t blk = gb % NB;
        int s = 0;
        while (first[s + 1] <= blk)
            ++s;
        int64_t j = blk - first[s];
        int64_t t0 = cu[s] + j * B;
        int64_t t1 = t0 + B;
        if (t1 > cu[s + 1])
            t1 = cu[s + 1];
        double *out = Kbar + ((size_t)g * NB + blk) * d;
        for (int c = 0; c < d; ++c)
            out[c] = 0.0;
        for (int64_t t = t0; t < t1; ++t) {
            const uint16_t *kr = K + ((size_t)t * Hkv + g) * d;
            for (int c = 0; c < d; ++c)
                out[c] += bf16_bits_to_double(kr[c]);
        }
        double cnt = (double)(t1 - t0);
        for (int c = 0; c < d; ++c)
            out[c] /= cnt;
    }
    free(first);
    return ORC_OK;
}

/*
 * Min / max pooled block keys, the Quest-style block representation the pages
 * name as a MoBA variant (elamur summary card, "Key points": Quest as MoBA
 * with smaller blocks and min/max pooling).  Kmax, Kmin [Hkv][NB][d]: the
 * elementwise maximum and minimum of the keys present in each block.
 */
int oracle_block_minmax(const uint16_t *K, const int64_t *cu, int nseq, int Hkv, int d, int B,
                        double *Kmax, double *Kmin)
{
    if (check_common(cu, nseq, Hkv, Hkv, d, B) || !K || !Kmax || !Kmin)
        return ORC_EINVAL;
    int64_t NB = oracle_total_blocks(cu, nseq, B);
    int64_t blk = 0;
    for (int s = 0; s < nseq; ++s) {
        int64_t nb = seq_blocks(cu, s, B);
        for (int64_t j = 0; j < nb; ++j, ++blk) {
            int64_t t0 = cu[s] + j * B;
            int64_t t1 = t0 + B;
            if (t1 > cu[s + 1])
                t1 = cu[s + 1];
            for (int g = 0; g < Hkv; ++g) {
                double *mx = Kmax + ((size_t)g * NB + blk) * d;
                double *mn = Kmin + ((size_t)g * NB + blk) * d;
                for (int c = 0; c < d; ++c) {
                    mx[c] = -INFINITY;
                    mn[c] = INFINITY;
                }
                for (int64_t t = t0; t < t1; ++t) {
                    const uint16_t *kr = K + ((size_t)t * Hkv + g) * d;
                    for (int c = 0; c < d; ++c) {
                        double x = bf16_bits_to_double(kr[c]);
                        if (x > mx[c])
                            mx[c] = x;
                        if (x < mn[c])
                            mn[c] = x;
                    }
                }
            }
        }
    }
    return ORC_OK;
}

typedef struct {
    double s;
    int64_t j;
} scored_block;

/* Order: score descending, then block index ascending. */
static int cmp_scored(const void *a, const void *b)
{
    const scored_block *x = (const scored_block *)a, *y = (const scored_block *)b;
    if (x->s > y->s)
        return -1;
    if (x->s < y->s)
        return 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

static int cmp_i32(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/*
 * Gate for a list of query rows (global token indices).
 *   sel    [nrows][Hq][k]  local block ids of the chosen blocks, ascending,
 *                          -1 padded (|sel| = min(k, i(t)+1));
 *   margin [nrows][Hq]     s_(k-1) - s_(k) over the past scores sorted by
 *                          (score desc, index asc), with s_(0) = +inf; +inf
 *                          when fewer than k past blocks exist;
 *   maxabs [nrows][Hq]     max |s_j| over the past blocks (0 if none).
 * margin and maxabs may be NULL.
 */
static int select_impl(const uint16_t *Q, const double *Kbar, const double *Kmin,
                       const int64_t *cu, int nseq, int Hq, int Hkv, int d, int B, int k,
                       const int64_t *rows, int64_t nrows, int32_t *sel, double *margin,
                       double *maxabs)
{
    if (check_common(cu, nseq, Hq, Hkv, d, B) || !Q || !Kbar || !rows || !sel || k <= 0)
        return ORC_EINVAL;
    int64_t T = cu[nseq];
    int64_t NB = oracle_total_blocks(cu, nseq, B);
    int G = Hq / Hkv;
    int err = ORC_OK;

#pragma omp parallel
    {
        scored_block *buf = (scored_block *)malloc(sizeof(scored_block) * (size_t)(NB + 1));
        int32_t *tmp = (int32_t *)malloc(sizeof(int32_t) * (size_t)(k + 1));
        double *qd = (double *)malloc(sizeof(double) * (size_t)d);
        if (!buf || !tmp || !qd) {
#pragma omp atomic write
            err = ORC_ENOMEM;
        }
#pragma omp for schedule(dynamic)
        for (int64_t rh = 0; rh < nrows * Hq; ++rh) {
            if (!buf || !tmp || !qd)
                continue;
            int64_t r = rh / Hq;
            int h = (int)(rh % Hq);
            int64_t t = rows[r];
            if (t < 0 || t >= T) {
#pragma omp atomic write
                err = ORC_EINVAL;
                continue;
            }
            int s = seq_of(cu, nseq, t);
            int64_t first = 0;
            for (int u = 0; u < s; ++u)
                first += seq_blocks(cu, u, B);
            int64_t i = (t - cu[s]) / B; /* own block */
            int g = h / G;
            const uint16_t *qr = Q + ((size_t)t * Hq + h) * d;
            for (int c = 0; c < d; ++c)
                qd[c] = bf16_bits_to_double(qr[c]);
            double mx = 0.0;
            for (int64_t j = 0; j < i; ++j) {
                const double *kb = Kbar + ((size_t)g * NB + first + j) * d;
                double acc = 0.0;
                if (!Kmin) { /* mean pooling: s_j = q . Kbar_j */
                    for (int c = 0; c < d; ++c)
                        acc += qd[c] * kb[c];
                } else { /* min/max pooling: s_j = sum_c max(q_c Kmax_jc, q_c Kmin_jc) */
                    const double *kn = Kmin + ((size_t)g * NB + first + j) * d;
                    for (int c = 0; c < d; ++c) {
                        double a = qd[c] * kb[c], b2 = qd[c] * kn[c];
                        acc += (a > b2) ? a : b2;
                    }
                }
                buf[j].s = acc;
                buf[j].j = j;
                if (fabs(acc) > mx)
                    mx = fabs(acc);
            }
            qsort(buf, (size_t)i, sizeof(scored_block), cmp_scored);
            int64_t take = (i < k - 1) ? i : (k - 1);
            int n = 0;
            for (int64_t u = 0; u < take; ++u)
                tmp[n++] = (int32_t)buf[u].j;
            tmp[n++] = (int32_t)i;
            qsort(tmp, (size_t)n, sizeof(int32_t), cmp_i32);
            int32_t *out = sel + ((size_t)r * Hq + h) * k;
            for (int u = 0; u < k; ++u)
                out[u] = (u < n) ? tmp[u] : -1;
            if (margin) {
                double mg;
                if (i < k)
                    mg = INFINITY;
                else if (k == 1)
                    mg = INFINITY; /* the only chosen block is the forced own block */
                else
                    mg = buf[k - 2].s - buf[k - 1].s;
                margin[(size_t)r * Hq + h] = mg;
            }
            if (maxabs)
                maxabs[(size_t)r * Hq + h] = mx;
        }
        free(buf);
        free(tmp);
        free(qd);
    }
    return err;
}

int oracle_select(const uint16_t *Q, const double *Kbar, const int64_t *cu, int nseq, int Hq,
                  int Hkv, int d, int B, int k, const int64_t *rows, int64_t nrows,
                  int32_t *sel, double *margin, double *maxabs)
{
    return select_impl(Q, Kbar, NULL, cu, nseq, Hq, Hkv, d, B, k, rows, nrows, sel, margin,
                       maxabs);
}

/*
 * The same gate with the min/max-pooled block representation: the score of
 * past block j is sum_c max(q_c Kmax_jc, q_c Kmin_jc), the largest q . x over
 * the box spanned by the block's keys (so at least max over the block's keys
 * of q . k; Quest's criticality bound, the scoring of the method the pages
 * frame as MoBA with min/max pooling).  Same top-k, causality and tie rules,
 * same margin / maxabs outputs.
 */
int oracle_select_minmax(const uint16_t *Q, const double *Kmax, const double *Kmin,
                         const int64_t *cu, int nseq, int Hq, int Hkv, int d, int B, int k,
                         const int64_t *rows, int64_t nrows, int32_t *sel, double *margin,
                         double *maxabs)
{
    if (!Kmin)
        return ORC_EINVAL;
    return select_impl(Q, Kmax, Kmin, cu, nseq, Hq, Hkv, d, B, k, rows, nrows, sel, margin,
                       maxabs);
}

/*
 * Attention of each listed row over the key set named by a selection.
 * sel [nrows][Hq][k] holds local block ids (-1 = unused).  A past block
 * contributes all of its tokens; the own block contributes its tokens up to
 * and including t; a block after the own block is an error.
 *   O   [nrows][Hq][d]   fp64
 *   lse [nrows][Hq]      natural-log sum of exp(scale * q.k) over I
 *   nkeys [nrows][Hq]    |I| (may be NULL)
 */
int oracle_attend(const uint16_t *Q, const uint16_t *K, const uint16_t *V, const int64_t *cu,
                  int nseq, int Hq, int Hkv, int d, int B, int k, double scale,
                  const int64_t *rows, int64_t nrows, const int32_t *sel, double *O,
                  double *lse, int64_t *nkeys)
{
    if (check_common(cu, nseq, Hq, Hkv, d, B) || !Q || !K || !V || !rows || !sel || !O ||
        !lse || k <= 0)
        return ORC_EINVAL;
    int64_t T = cu[nseq];
    int G = Hq / Hkv;
    int err = ORC_OK;

#pragma omp parallel
    {
        size_t cap = 0;
        double *z = NULL;
        int64_t *idx = NULL;
        double *qd = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic)
        for (int64_t rh = 0; rh < nrows * Hq; ++rh) {
            int64_t r = rh / Hq;
            int h = (int)(rh % Hq);
            int64_t t = rows[r];
            if (t < 0 || t >= T) {
#pragma omp atomic write
                err = ORC_EINVAL;
                continue;
            }
            int s = seq_of(cu, nseq, t);
            int64_t i = (t - cu[s]) / B;
            const int32_t *sr = sel + ((size_t)r * Hq + h) * k;
            /* collect I */
            size_t need = (size_t)k * (size_t)B + 1;
            if (need > cap) {
                free(z);
                free(idx);
                cap = need;
                z = (double *)malloc(sizeof(double) * cap);
                idx = (int64_t *)malloc(sizeof(int64_t) * cap);
            }
            if (!z || !idx || !qd) {
#pragma omp atomic write
                err = ORC_ENOMEM;
                cap = 0;
                continue;
            }
            size_t m = 0;
            int bad = 0;
            for (int u = 0; u < k; ++u) {
                int64_t j = sr[u];
                if (j < 0)
                    continue;
                if (j > i) {
                    bad = 1;
                    break;
                }
                int64_t a = cu[s] + j * B;
                int64_t e = (j == i) ? (t + 1) : (a + B);
                if (e > cu[s + 1])
                    e = cu[s + 1];
                for (int64_t u2 = a; u2 < e; ++u2)
                    idx[m++] = u2;
            }
            if (bad) {
#pragma omp atomic write
                err = ORC_EFUTURE;
                continue;
            }
            const uint16_t *qr = Q + ((size_t)t * Hq + h) * d;
            for (int c = 0; c < d; ++c)
                qd[c] = bf16_bits_to_double(qr[c]);
            int g = h / G;
            double zmax = -INFINITY;
            for (size_t u = 0; u < m; ++u) {
                const uint16_t *kr = K + ((size_t)idx[u] * Hkv + g) * d;
                double acc = 0.0;
                for (int c = 0; c < d; ++c)
                    acc += qd[c] * bf16_bits_to_double(kr[c]);
                z[u] = acc * scale;
                if (z[u] > zmax)
                    zmax = z[u];
            }
            double den = 0.0;
            for (size_t u = 0; u < m; ++u) {
                z[u] = exp(z[u] - zmax);
                den += z[u];
            }
            double *orow = O + ((size_t)r * Hq + h) * d;
            for (int c = 0; c < d; ++c)
                orow[c] = 0.0;
            for (size_t u = 0; u < m; ++u) {
                const uint16_t *vr = V + ((size_t)idx[u] * Hkv + g) * d;
                double w = z[u] / den;
                for (int c = 0; c < d; ++c)
                    orow[c] += w * bf16_bits_to_double(vr[c]);
            }
            lse[(size_t)r * Hq + h] = zmax + log(den);
            if (nkeys)
                nkeys[(size_t)r * Hq + h] = (int64_t)m;
        }
        free(z);
        free(idx);
        free(qd);
    }
    return err;
}

/*
 * Backward of oracle_attend over a fixed selection.  The top-k gate is a hard
 * choice through which no gradient flows (wispaper.ai blog, "The Change":
 * the gradient does not pass through the discrete selection), so the
 * gradient is that of exact softmax attention over each row's key set I.
 * For each listed row r and head h (kv head g), with I as in oracle_attend
 * and z_u = scale * q.k_u, lse = log sum_u exp(z_u), P_u = exp(z_u - lse),
 * O = sum_u P_u v_u, and the output gradient dO (bf16 bits):
 *   D      = dO . O
 *   dS_u   = P_u (dO . v_u - D)          (softmax Jacobian applied to dO V^T)
 *   dQ[r,h] = scale * sum_u dS_u k_u
 *   dK[u,g] += scale * dS_u q
 *   dV[u,g] += P_u dO
 * dQ [nrows][Hq][d]; dK, dV [T][Hkv][d] (zeroed here, then summed over the
 * listed rows and the q heads of each kv head).  All fp64.  Work is split by
 * kv head; rows are visited in the listed order, so sums are deterministic.
 */
int oracle_attend_backward(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                           const int64_t *cu, int nseq, int Hq, int Hkv, int d, int B, int k,
                           double scale, const int64_t *rows, int64_t nrows, const int32_t *sel,
                           const uint16_t *dO, double *dQ, double *dK, double *dV)
{
    if (check_common(cu, nseq, Hq, Hkv, d, B) || !Q || !K || !V || !rows || !sel || !dO ||
        !dQ || !dK || !dV || k <= 0)
        return ORC_EINVAL;
    int64_t T = cu[nseq];
    int G = Hq / Hkv;
    int err = ORC_OK;
    memset(dK, 0, sizeof(double) * (size_t)T * Hkv * d);
    memset(dV, 0, sizeof(double) * (size_t)T * Hkv * d);
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= T)
            return ORC_EINVAL;

#pragma omp parallel for schedule(dynamic)
    for (int g = 0; g < Hkv; ++g) {
        size_t cap = (size_t)k * (size_t)B + 1;
        double *p = (double *)malloc(sizeof(double) * cap);
        int64_t *idx = (int64_t *)malloc(sizeof(int64_t) * cap);
        double *qd = (double *)malloc(sizeof(double) * (size_t)d);
        double *od = (double *)malloc(sizeof(double) * (size_t)d);
        double *gd = (double *)malloc(sizeof(double) * (size_t)d);
        if (!p || !idx || !qd || !od || !gd) {
#pragma omp atomic write
            err = ORC_ENOMEM;
        } else {
            for (int64_t r = 0; r < nrows; ++r) {
                int64_t t = rows[r];
                int s = seq_of(cu, nseq, t);
                int64_t i = (t - cu[s]) / B;
                for (int hh = 0; hh < G; ++hh) {
                    int h = g * G + hh;
                    const int32_t *sr = sel + ((size_t)r * Hq + h) * k;
                    size_t m = 0;
                    int bad = 0;
                    for (int u = 0; u < k; ++u) {
                        int64_t j = sr[u];
                        if (j < 0)
                            continue;
                        if (j > i) {
                            bad = 1;
                            break;
                        }
                        int64_t a = cu[s] + j * B;
                        int64_t e = (j == i) ? (t + 1) : (a + B);
                        if (e > cu[s + 1])
                            e = cu[s + 1];
                        for (int64_t u2 = a; u2 < e; ++u2)
                            idx[m++] = u2;
                    }
                    if (bad) {
#pragma omp atomic write
                        err = ORC_EFUTURE;
                        continue;
                    }
                    const uint16_t *qr = Q + ((size_t)t * Hq + h) * d;
                    const uint16_t *gr = dO + ((size_t)r * Hq + h) * d;
                    for (int c = 0; c < d; ++c) {
                        qd[c] = bf16_bits_to_double(qr[c]);
                        gd[c] = bf16_bits_to_double(gr[c]);
                        od[c] = 0.0;
                    }
                    /* probabilities over I */
                    double zmax = -INFINITY;
                    for (size_t u = 0; u < m; ++u) {
                        const uint16_t *kr = K + ((size_t)idx[u] * Hkv + g) * d;
                        double acc = 0.0;
                        for (int c = 0; c < d; ++c)
                            acc += qd[c] * bf16_bits_to_double(kr[c]);
                        p[u] = acc * scale;
                        if (p[u] > zmax)
                            zmax = p[u];
                    }
                    double den = 0.0;
                    for (size_t u = 0; u < m; ++u) {
                        p[u] = exp(p[u] - zmax);
                        den += p[u];
                    }
                    for (size_t u = 0; u < m; ++u)
                        p[u] /= den;
                    /* O and D = dO . O */
                    for (size_t u = 0; u < m; ++u) {
                        const uint16_t *vr = V + ((size_t)idx[u] * Hkv + g) * d;
                        for (int c = 0; c < d; ++c)
                            od[c] += p[u] * bf16_bits_to_double(vr[c]);
                    }
                    double D = 0.0;
                    for (int c = 0; c < d; ++c)
                        D += gd[c] * od[c];
                    double *dq = dQ + ((size_t)r * Hq + h) * d;
                    for (int c = 0; c < d; ++c)
                        dq[c] = 0.0;
                    for (size_t u = 0; u < m; ++u) {
                        const uint16_t *kr = K + ((size_t)idx[u] * Hkv + g) * d;
                        const uint16_t *vr = V + ((size_t)idx[u] * Hkv + g) * d;
                        double dp = 0.0;
                        for (int c = 0; c < d; ++c)
                            dp += gd[c] * bf16_bits_to_double(vr[c]);
                        double ds = p[u] * (dp - D);
                        double *dkr = dK + ((size_t)idx[u] * Hkv + g) * d;
                        double *dvr = dV + ((size_t)idx[u] * Hkv + g) * d;
                        for (int c = 0; c < d; ++c) {
                            dq[c] += scale * ds * bf16_bits_to_double(kr[c]);
                            dkr[c] += scale * ds * qd[c];
                            dvr[c] += p[u] * gd[c];
                        }
                    }
                }
            }
        }
        free(p);
        free(idx);
        free(qd);
        free(od);
        free(gd);
    }
    return err;
}

/*
 * Dense causal attention of each listed row over every earlier token of its
 * own sequence (I = {seq start .. t}); the k = n limit of the method.
 * Written without blocks or selections.
 */
int oracle_dense_causal(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                        const int64_t *cu, int nseq, int Hq, int Hkv, int d, double scale,
                        const int64_t *rows, int64_t nrows, double *O, double *lse)
{
    if (check_common(cu, nseq, Hq, Hkv, d, 1) || !Q || !K || !V || !rows || !O || !lse)
        return ORC_EINVAL;
    int64_t T = cu[nseq];
    int G = Hq / Hkv;
    int err = ORC_OK;
#pragma omp parallel
    {
        size_t cap = 0;
        double *z = NULL;
        double *qd = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic)
        for (int64_t rh = 0; rh < nrows * Hq; ++rh) {
            int64_t r = rh / Hq;
            int h = (int)(rh % Hq);
            int64_t t = rows[r];
            if (t < 0 || t >= T) {
#pragma omp atomic write
                err = ORC_EINVAL;
                continue;
            }
            int s = seq_of(cu, nseq, t);
            int64_t a = cu[s];
            size_t m = (size_t)(t - a + 1);
            if (m > cap) {
                free(z);
                cap = m;
                z = (double *)malloc(sizeof(double) * cap);
            }
            if (!z || !qd) {
#pragma omp atomic write
                err = ORC_ENOMEM;
                cap = 0;
                continue;
            }
            const uint16_t *qr = Q + ((size_t)t * Hq + h) * d;
            for (int c = 0; c < d; ++c)
                qd[c] = bf16_bits_to_double(qr[c]);
            int g = h / G;
            double zmax = -INFINITY;
            for (size_t u = 0; u < m; ++u) {
                const uint16_t *kr = K + ((size_t)(a + u) * Hkv + g) * d;
                double acc = 0.0;
                for (int c = 0; c < d; ++c)
                    acc += qd[c] * bf16_bits_to_double(kr[c]);
                z[u] = acc * scale;
                if (z[u] > zmax)
                    zmax = z[u];
            }
            double den = 0.0;
            for (size_t u = 0; u < m; ++u) {
                z[u] = exp(z[u] - zmax);
                den += z[u];
            }
            double *orow = O + ((size_t)r * Hq + h) * d;
            for (int c = 0; c < d; ++c)
                orow[c] = 0.0;
            for (size_t u = 0; u < m; ++u) {
                const uint16_t *vr = V + ((size_t)(a + u) * Hkv + g) * d;
                double w = z[u] / den;
                for (int c = 0; c < d; ++c)
                    orow[c] += w * bf16_bits_to_double(vr[c]);
            }
            lse[(size_t)r * Hq + h] = zmax + log(den);
        }
        free(z);
        free(qd);
    }
    return err;
}
