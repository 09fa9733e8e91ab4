/*
 * oracle.c -- plain, slow, obviously correct CPU reference for training-free
 * block-sparse "sol-attn" attention (Q/K mean-pooled per block, a per-row
 * adaptive threshold or top-k over pooled block scores, exact attention over
 * the kept key blocks, centroid terms for the rest, one softmax).
 *
 * TEST INFRASTRUCTURE ONLY.  The library (the CUDA path) never links, loads or
 * calls this file; only the tests, the smoke check and the benchmark's CPU
 * baseline use it.  It shares no code, header, table or constant with the
 * CUDA path.
 *
 * Sources (web pages; cited by title and section):
 *   [DOC]  "BlockSparseAttention - ComfyUI Built-in Node Documentation"
 *          (zh and ja editions): general-inputs table (extra_tokens,
 *          sink_conditioning), "sol-attn inputs" table (tau), "sla inputs"
 *          table (keep_percent), "constraints and limitations".
 *   [STAR] "minimax-h3-chunk-star7" README, sections "SLA" and "Sol".
 *
 * Arithmetic: every sum, dot product and softmax is accumulated in double
 * (fp64); values the method stores (block means, block scores, thresholds)
 * are rounded once to fp32.  Sums run in index order; dot products use a
 * fused multiply-add per term, in channel order.
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes of the repository as well):
 *   R1  block means are arithmetic means over the block's valid tokens
 *       (a partial last block averages its own tokens);
 *   R2  block score S_ib = fl32( (q_i . k_b) / sqrt(d) );
 *   R3  tau is counted in population standard deviations (ddof 0) of the whole
 *       row of nKB scores, two-pass in double; thr = fl32(mu + tau*sigma);
 *       keep iff S > thr (strict); sigma == 0 keeps only the forced blocks;
 *       tau = -inf keeps every block, tau = +inf none;
 *   R4  forced blocks (kept in addition): sink blocks [0, sink), every block
 *       overlapping the packed prefix [0, P), and every key block whose token
 *       range meets the query block's range (one block for Q64/K64, two for
 *       Q128/K64);
 *   R5  SLA keeps k = clamp(lround(p * nKB / 100), 1, nKB) blocks, the top k by
 *       score with ties to the lower index, then ORs in the forced blocks; no
 *       centroid term;
 *   R6  extra tokens: candidates are tokens of blocks not kept; token score
 *       t_j = fl32( (qt_i . k_j) / sqrt(d) ) with qt_i the pooled query rounded
 *       to the input dtype (bf16 round-to-nearest-even); the top E by score,
 *       ties to the lower token index, returned in ascending order;
 *   R7  a block that gave e_b extra tokens keeps a centroid over its
 *       remaining n_b - e_b tokens (mean recomputed over those tokens, bias
 *       ln(n_b - e_b)); a block left with no token drops; every key is so
 *       counted exactly once;
 *   R8  the centroid logit of unselected block b is q . kbar_b / sqrt(d)
 *       + ln(n_b) with value vbar_b: n_b copies of the centroid key;
 *   R9  rows in [dense_begin, dense_end) run full dense attention over all N
 *       keys and replace the sparse result;
 *   R10 attention is bidirectional (no causal mask), scale 1/sqrt(d), base-e
 *       softmax; LSE = m + ln(sum of exp(logit - m)).
 *
 * Parity pins (tests that do not rely on this file's own formulas):
 *   block means -> numpy mean;  tau = -inf and keep_percent = 100 -> dense
 *   attention;  block-constant K/V -> dense attention for any tau (pins R8
 *   including partial blocks);  Gaussian scores -> kept fraction 1 - Phi(tau)
 *   (pins R3) and the pages' 16 / 7 / 2.7 % figures;  V == 1 -> O == 1;
 *   E >= candidates -> dense (pins R6/R7);  prefix-only selection -> dense
 *   attention over the prefix;  a separate pure-Python brute force on tiny
 *   inputs covers every step.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_BF16 0
#define ORC_F32 1

/* ---------------------------------------------------------------- access */

static double load_elem(const void *base, int dtype, int64_t idx)
{
    if (dtype == ORC_F32)
        return (double)((const float *)base)[idx];
    uint32_t bits = (uint32_t)((const uint16_t *)base)[idx] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

typedef struct {
    const void *p;
    int dtype;
    int64_t sb, sn, sh;     /* element strides; channel stride is 1 */
} tensor_view;

static double tv_at(const tensor_view *t, int b, int64_t n, int h, int c)
{
    return load_elem(t->p, t->dtype, (int64_t)b * t->sb + n * t->sn + (int64_t)h * t->sh + c);
}

static int imin(int a, int b) { return a < b ? a : b; }

/* Round a float to bf16 (round to nearest, ties to even) and back. */
static float round_to_bf16(float x)
{
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u) {          /* inf / nan: truncate */
        u &= 0xffff0000u;
    } else {
        uint32_t lsb = (u >> 16) & 1u;
        u += 0x7fffu + lsb;
        u &= 0xffff0000u;
    }
    float r;
    memcpy(&r, &u, sizeof r);
    return r;
}

/* ------------------------------------------------------- block pooling  */
/*
 * Mean of x over each block of `blk` consecutive tokens, per (b, h, channel)
 * (pooling of Q and K for routing and of K and V for the centroids:
 * [STAR] "SLA" (Q=128, K=64 blocks) and "Sol" (Q64/K64, K/V centroids); R1).
 * mean: [B, H, nb, d] fp32; count: [nb] valid tokens per block.
 */
int orc_block_means(const void *x, int dtype, int64_t sb, int64_t sn, int64_t sh,
                    int B, int N, int H, int d, int blk, float *mean, int32_t *count)
{
    if (blk <= 0 || N <= 0) return -1;
    const int nb = (N + blk - 1) / blk;
    tensor_view t = {x, dtype, sb, sn, sh};
    for (int i = 0; i < nb; i++)
        count[i] = imin(N, (i + 1) * blk) - i * blk;
#pragma omp parallel for collapse(3) schedule(static)
    for (int b = 0; b < B; b++)
        for (int h = 0; h < H; h++)
            for (int i = 0; i < nb; i++) {
                const int t0 = i * blk, t1 = imin(N, t0 + blk);
                float *out = mean + (((int64_t)b * H + h) * nb + i) * d;
                for (int c = 0; c < d; c++) {
                    double s = 0.0;
                    for (int n = t0; n < t1; n++) s += tv_at(&t, b, n, h, c);
                    out[c] = (float)(s / (double)(t1 - t0));
                }
            }
    return 0;
}

/* ------------------------------------------------------- block scores   */
/*
 * S[bh, i, j] = fl32( (qbar_i . kbar_j) / sqrt(d) )  (R2).
 */
int orc_block_scores(const float *qbar, const float *kbar, int BH, int nQB, int nKB, int d,
                     float *S)
{
    const double rs = sqrt((double)d);
#pragma omp parallel for collapse(2) schedule(static)
    for (int bh = 0; bh < BH; bh++)
        for (int i = 0; i < nQB; i++) {
            const float *q = qbar + ((int64_t)bh * nQB + i) * d;
            float *row = S + ((int64_t)bh * nQB + i) * nKB;
            for (int j = 0; j < nKB; j++) {
                const float *k = kbar + ((int64_t)bh * nKB + j) * d;
                double dot = 0.0;
                for (int c = 0; c < d; c++) dot = fma((double)q[c], (double)k[c], dot);
                row[j] = (float)(dot / rs);
            }
        }
    return 0;
}

/* ------------------------------------------------------- forced blocks  */
/*
 * Blocks kept in addition to the routed set (R4): sink blocks, the blocks of
 * the packed conditioning prefix ([DOC] sink_conditioning = exact_kv: every
 * query attends exactly to the packed rows), and the diagonal blocks
 * ([DOC] "sla inputs": sink and diagonal are kept in addition).
 */
int orc_forced_blocks(int i, int nKB, int N, int Bq, int Bk, int sink_blocks, int prefix_len,
                      int keep_diag, uint8_t *forced)
{
    memset(forced, 0, (size_t)nKB);
    for (int b = 0; b < imin(sink_blocks, nKB); b++) forced[b] = 1;
    if (prefix_len > 0) {
        const int pb = imin(nKB, (prefix_len + Bk - 1) / Bk);
        for (int b = 0; b < pb; b++) forced[b] = 1;
    }
    if (keep_diag) {
        const int q0 = i * Bq, q1 = imin(N, q0 + Bq) - 1;
        for (int b = q0 / Bk; b <= q1 / Bk && b < nKB; b++) forced[b] = 1;
    }
    return 0;
}

typedef struct { float s; int idx; } scored;

static int by_score_desc(const void *a, const void *b)
{
    const scored *x = (const scored *)a, *y = (const scored *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

/* ------------------------------------------------------- selection      */
/*
 * method 0 (Sol, [DOC] "sol-attn inputs", tau: a threshold in standard
 * deviations of the score distribution; R3), method 1 (SLA, [DOC] "sla
 * inputs", keep_percent; [STAR] "SLA" top-k routing; R5).  Rows are ordered
 * [B, H, nQB]; row r is query block r % nQB.
 * keep: [nrows, nKB] 0/1;  thr: per-row threshold (Sol) or k-th largest
 * score (SLA), used by the tests to count near-threshold blocks.
 */
int orc_select(const float *S, int64_t nrows, int nQB, int nKB, int N, int Bq, int Bk,
               int method, double tau, double keep_percent, int sink_blocks, int prefix_len,
               int keep_diag, uint8_t *keep, float *thr)
{
    if (method != 0 && method != 1) return -1;
    int kk = 0;
    if (method == 1) {
        long r = lround(keep_percent * (double)nKB / 100.0);
        if (r < 1) r = 1;
        if (r > nKB) r = nKB;
        kk = (int)r;
    }
#pragma omp parallel
    {
        uint8_t *forced = (uint8_t *)malloc((size_t)nKB);
        scored *tmp = (scored *)malloc(sizeof(scored) * (size_t)nKB);
#pragma omp for schedule(static)
        for (int64_t r = 0; r < nrows; r++) {
            const float *row = S + r * nKB;
            uint8_t *out = keep + r * nKB;
            memset(out, 0, (size_t)nKB);
            if (method == 0) {
                if (isinf(tau) && tau < 0) {
                    memset(out, 1, (size_t)nKB);
                    thr[r] = -INFINITY;
                } else {
                    double mu = 0.0;
                    for (int j = 0; j < nKB; j++) mu += (double)row[j];
                    mu /= (double)nKB;
                    double var = 0.0;
                    for (int j = 0; j < nKB; j++) {
                        const double e = (double)row[j] - mu;
                        var += e * e;
                    }
                    var /= (double)nKB;
                    const double sigma = sqrt(var);
                    if (isinf(tau)) {
                        thr[r] = INFINITY;
                    } else {
                        const float t = (float)(mu + tau * sigma);
                        thr[r] = t;
                        if (sigma > 0.0)
                            for (int j = 0; j < nKB; j++) out[j] = row[j] > t;
                    }
                }
            } else {
                for (int j = 0; j < nKB; j++) { tmp[j].s = row[j]; tmp[j].idx = j; }
                qsort(tmp, (size_t)nKB, sizeof(scored), by_score_desc);
                for (int j = 0; j < kk; j++) out[tmp[j].idx] = 1;
                thr[r] = tmp[kk - 1].s;
            }
            orc_forced_blocks((int)(r % nQB), nKB, N, Bq, Bk, sink_blocks, prefix_len, keep_diag,
                              forced);
            for (int j = 0; j < nKB; j++) out[j] |= forced[j];
        }
        free(forced);
        free(tmp);
    }
    return 0;
}

/* ------------------------------------------------------- extra tokens   */
/*
 * [DOC] general inputs, extra_tokens: every query block also attends exactly
 * to its E highest-scoring tokens outside its selected blocks (R6).
 * rows: list of row ids (b*H + h)*nQB + i to compute; extra: [nsel, E]
 * ascending token indices; cnt: [nsel].
 */
int orc_extra_tokens(const float *qbar, const void *k, int dtype, int64_t sb, int64_t sn,
                     int64_t sh, int B, int H, int N, int d, int Bq, int Bk, const uint8_t *keep,
                     int E, const int64_t *rows, int64_t nsel, int32_t *extra, int32_t *cnt)
{
    (void)B;
    const int nQB = (N + Bq - 1) / Bq, nKB = (N + Bk - 1) / Bk;
    const double rs = sqrt((double)d);
    tensor_view kt = {k, dtype, sb, sn, sh};
#pragma omp parallel
    {
        scored *cand = (scored *)malloc(sizeof(scored) * (size_t)N);
        int32_t *pick = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
        double *qt = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
        for (int64_t s = 0; s < nsel; s++) {
            const int64_t r = rows[s];
            const int h = (int)((r / nQB) % H);
            const int b = (int)(r / ((int64_t)nQB * H));
            const float *q = qbar + r * d;
            for (int c = 0; c < d; c++)
                qt[c] = dtype == ORC_BF16 ? (double)round_to_bf16(q[c]) : (double)q[c];
            int nc = 0;
            for (int blk = 0; blk < nKB; blk++) {
                if (keep[r * nKB + blk]) continue;
                for (int n = blk * Bk; n < imin(N, (blk + 1) * Bk); n++) {
                    double dot = 0.0;
                    for (int c = 0; c < d; c++) dot = fma(qt[c], tv_at(&kt, b, n, h, c), dot);
                    cand[nc].s = (float)(dot / rs);
                    cand[nc].idx = n;
                    nc++;
                }
            }
            qsort(cand, (size_t)nc, sizeof(scored), by_score_desc);
            const int take = nc < E ? nc : E;
            for (int j = 0; j < take; j++) pick[j] = cand[j].idx;
            /* ascending token order */
            for (int a = 1; a < take; a++) {
                int32_t v = pick[a];
                int p = a - 1;
                while (p >= 0 && pick[p] > v) { pick[p + 1] = pick[p]; p--; }
                pick[p + 1] = v;
            }
            for (int j = 0; j < E; j++) extra[s * E + j] = j < take ? pick[j] : -1;
            cnt[s] = take;
        }
        free(cand);
        free(pick);
        free(qt);
    }
    return 0;
}

/* ------------------------------------------------------- attention      */
/*
 * Output rows of the fine pass ([STAR] "Sol": kept K/V blocks exact,
 * unselected blocks through their K/V centroid, both merged in one softmax;
 * [DOC] sink_conditioning: exact prefix, dense rows override; R7-R10).
 *
 * keep: [B*H*nQB, nKB];  extra / ecnt: [B*H*nQB, E] ascending tokens and
 * counts (ecnt may be NULL when E == 0);  kbar / vbar: [B, H, nKB, d] block
 * means;  count: [nKB] block sizes;  tok: [m, 3] (b, h, n) query tokens;
 * out: [m, d] fp64;  lse: [m] fp64.
 */
int orc_attention_rows(const void *q, const void *k, const void *v, int dtype, int64_t sb,
                       int64_t sn, int64_t sh, int B, int H, int N, int d, int Bq, int Bk,
                       const float *kbar, const float *vbar, const int32_t *count,
                       const uint8_t *keep, const int32_t *extra, const int32_t *ecnt, int E,
                       int centroid, int dense_begin, int dense_end, const int64_t *tok,
                       int64_t m, double *out, double *lse)
{
    (void)B;
    const int nQB = (N + Bq - 1) / Bq, nKB = (N + Bk - 1) / Bk;
    const double rs = sqrt((double)d);
    tensor_view qt = {q, dtype, sb, sn, sh}, kt = {k, dtype, sb, sn, sh}, vt = {v, dtype, sb, sn, sh};
#pragma omp parallel
    {
        double *logit = (double *)malloc(sizeof(double) * (size_t)(N + nKB));
        int32_t *src = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N + nKB)); /* >=0 token, <0 -(blk+1) */
        double *qrow = (double *)malloc(sizeof(double) * (size_t)d);
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
        double *cen = (double *)malloc(sizeof(double) * (size_t)nKB * 2 * d);  /* modified k', v' */
        int32_t *eb = (int32_t *)malloc(sizeof(int32_t) * (size_t)nKB);
        uint8_t *is_extra = (uint8_t *)malloc((size_t)N);
#pragma omp for schedule(dynamic, 4)
        for (int64_t s = 0; s < m; s++) {
            const int b = (int)tok[3 * s], h = (int)tok[3 * s + 1];
            const int64_t n = tok[3 * s + 2];
            const int64_t r = ((int64_t)b * H + h) * nQB + n / Bq;
            for (int c = 0; c < d; c++) qrow[c] = tv_at(&qt, b, n, h, c);
            int L = 0;
            const int dense = n >= dense_begin && n < dense_end;
            if (dense) {
                for (int j = 0; j < N; j++) src[L++] = j;
            } else {
                const uint8_t *kr = keep + r * nKB;
                const int ne = (ecnt && E > 0) ? ecnt[r] : 0;
                const int32_t *ex = extra ? extra + r * (int64_t)E : NULL;
                memset(eb, 0, sizeof(int32_t) * (size_t)nKB);
                memset(is_extra, 0, (size_t)N);
                for (int blk = 0; blk < nKB; blk++)
                    if (kr[blk])
                        for (int j = blk * Bk; j < imin(N, (blk + 1) * Bk); j++) src[L++] = j;
                for (int e = 0; e < ne; e++) {
                    src[L++] = ex[e];
                    is_extra[ex[e]] = 1;
                    eb[ex[e] / Bk]++;
                }
                if (centroid)
                    for (int blk = 0; blk < nKB; blk++) {
                        if (kr[blk]) continue;
                        if (count[blk] - eb[blk] <= 0) continue;
                        src[L++] = -(blk + 1);
                    }
            }
            /* logits */
            double mx = -INFINITY;
            for (int a = 0; a < L; a++) {
                double dot = 0.0;
                if (src[a] >= 0) {
                    for (int c = 0; c < d; c++) dot = fma(qrow[c], tv_at(&kt, b, src[a], h, c), dot);
                    logit[a] = dot / rs;
                } else {
                    const int blk = -src[a] - 1;
                    const int nb = count[blk] - eb[blk];
                    double *kc = cen + (size_t)blk * 2 * d, *vc = kc + d;
                    const float *kb = kbar + (((int64_t)b * H + h) * nKB + blk) * d;
                    const float *vb = vbar + (((int64_t)b * H + h) * nKB + blk) * d;
                    if (eb[blk] == 0) {
                        for (int c = 0; c < d; c++) { kc[c] = kb[c]; vc[c] = vb[c]; }
                    } else {
                        for (int c = 0; c < d; c++) {
                            double sk = 0.0, sv = 0.0;
                            for (int j = blk * Bk; j < imin(N, (blk + 1) * Bk); j++) {
                                if (is_extra[j]) continue;
                                sk += tv_at(&kt, b, j, h, c);
                                sv += tv_at(&vt, b, j, h, c);
                            }
                            kc[c] = (double)(float)(sk / (double)nb);
                            vc[c] = (double)(float)(sv / (double)nb);
                        }
                    }
                    for (int c = 0; c < d; c++) dot = fma(qrow[c], kc[c], dot);
                    logit[a] = dot / rs + log((double)nb);
                }
                if (logit[a] > mx) mx = logit[a];
            }
            for (int c = 0; c < d; c++) acc[c] = 0.0;
            double den = 0.0;
            for (int a = 0; a < L; a++) {
                const double p = exp(logit[a] - mx);
                den += p;
                if (src[a] >= 0) {
                    for (int c = 0; c < d; c++) acc[c] += p * tv_at(&vt, b, src[a], h, c);
                } else {
                    const double *vc = cen + (size_t)(-src[a] - 1) * 2 * d + d;
                    for (int c = 0; c < d; c++) acc[c] += p * vc[c];
                }
            }
            for (int c = 0; c < d; c++) out[s * d + c] = L > 0 ? acc[c] / den : 0.0;
            lse[s] = L > 0 ? mx + log(den) : -INFINITY;
        }
        free(logit); free(src); free(qrow); free(acc); free(cen); free(eb); free(is_extra);
    }
    return 0;
}
