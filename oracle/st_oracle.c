/*
 * st_oracle.c -- plain, slow, fp64 CPU oracle for the Sparse Transformer's factorized causal
 * self-attention (strided and fixed patterns, per-head or merged).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg may load or call this library.  It shares no code, header, table or helper with
 * the CUDA library, and the CUDA library never calls it.
 *
 * Sources (page title, section):
 *   [R]  "Sparse Transformers（稀疏 Transformer）深度解读报告"  -- §2.1 factorized self-attention
 *        (A_i^(m) is a subset of {j : j <= i}), §2.2 the strided and fixed patterns and the
 *        worked example, §3.1 head integration (Eq.6-8), §3.4 recomputation, §3.5 kernels.
 *   [G]  "长序列为何不必让每个 token 看见全部历史？滑动窗口、块稀疏与全局 token"  -- §01
 *        S_ij = q_i.k_j / sqrt(d); §02 masked softmax over the allowed keys only, a row with no
 *        allowed key needs care; §10 verification by dense truth mask and masked-V perturbation.
 *
 * Everything is the plain definition written out: each allowed set is found by scanning
 * j = 0..i with the page predicate; scores, a two-pass softmax and the output follow; the
 * gradients are ordinary calculus of that definition (no recompute trick, no blocking, no online
 * softmax).  All arithmetic is in double precision.  Query and key rows have width d, value,
 * output and output-gradient rows width e (e = d unless the query-key projection is narrower).  Readings taken where the pages are silent or
 * garbled are listed next to each function.
 *
 * Set kinds (one per head):
 *   1 sA1  strided head 1, local band   : max(0, i-l) <= j <= i                 ([R] §2.2)
 *   2 sA2  strided head 2, stride        : j <= i and (i-j) mod l == 0            ([R] §2.2)
 *   3 sU   strided merged head           : sA1 or sA2                             ([R] §3.1 Eq.7)
 *   4 fA1  fixed head 1, same block      : j <= i and floor(j/l) == floor(i/l)    ([R] §2.2)
 *   5 fA2  fixed head 2, summary columns : j <= i and (j mod l) in [l-c-o, l-1-o] ([R] §2.2)
 *   6 fU   fixed merged head             : fA1 or fA2                             ([R] §3.1 Eq.7)
 * Readings: positions are 0-based; j <= i is imposed on every set ([R] §2.1 says every set is a
 * subset of {j <= i}); the garbled fixed range {t, ..., l} with t = l - c is read as the c
 * positions l-c .. l-1 of each block; o is the per-head sub-block offset ([R] §2.2 tuning notes:
 * several A2 heads should look at different c-wide sub-blocks), o = 0 is the page's own set.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { K_SA1 = 1, K_SA2 = 2, K_SU = 3, K_FA1 = 4, K_FA2 = 5, K_FU = 6 };

/* Membership of key j in the allowed set of query i, evaluated literally. */
int oracle_allowed(int kind, int64_t i, int64_t j, int64_t l, int64_t c, int64_t o)
{
    if (j < 0 || j > i) return 0;                       /* causal: A_i is a subset of {j <= i} */
    int in1, in2;
    switch (kind) {
    case K_SA1: return j >= (i - l > 0 ? i - l : 0);
    case K_SA2: return ((i - j) % l) == 0;
    case K_SU:
        in1 = j >= (i - l > 0 ? i - l : 0);
        in2 = ((i - j) % l) == 0;
        return in1 || in2;
    case K_FA1: return (j / l) == (i / l);
    case K_FA2: return (j % l) >= l - c - o && (j % l) <= l - 1 - o;
    case K_FU:
        in1 = (j / l) == (i / l);
        in2 = (j % l) >= l - c - o && (j % l) <= l - 1 - o;
        return in1 || in2;
    default: return 0;
    }
}

/* The allowed set of row i, found by scanning every j = 0..i.  Writes the members in increasing
 * order to out (if non-NULL) and returns how many there are. */
int64_t oracle_row_set(int kind, int64_t i, int64_t l, int64_t c, int64_t o, int64_t *out)
{
    int64_t cnt = 0;
    for (int64_t j = 0; j <= i; ++j)
        if (oracle_allowed(kind, i, j, l, c, o)) {
            if (out) out[cnt] = j;
            ++cnt;
        }
    return cnt;
}

/* |A(i)| for every i < n, by scanning. */
void oracle_set_counts(int kind, int64_t n, int64_t l, int64_t c, int64_t o, int64_t *counts)
{
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < n; ++i) counts[i] = oracle_row_set(kind, i, l, c, o, NULL);
}

/* Head integration ([R] §3.1).  family: 1 strided, 2 fixed.  head_mode: 1 per-head
 * alternating (Eq.8 with the two factorized heads interleaved), 2 merged (Eq.7), 3 every head
 * is head 1, 4 every head is head 2.
 * Reading (the pages give no formula): in alternating mode head h uses pattern head 1 when h is
 * even and pattern head 2 when h is odd; the pattern-2 heads are numbered k = 0, 1, 2, ... in
 * head order (k = h/2 in alternating mode, k = h otherwise) and fixed pattern-2 head k looks at
 * the sub-block shifted by o_k = (k * step) mod l, with step = c when step <= 0.  Merged heads
 * use the same o_k.  Returns 0 on success, -1 on bad arguments. */
int oracle_head_kinds(int family, int head_mode, int num_heads, int64_t l, int64_t c,
                      int64_t step, int *kind, int64_t *off)
{
    if (family != 1 && family != 2) return -1;
    if (head_mode < 1 || head_mode > 4 || num_heads < 1 || l < 1) return -1;
    if (step <= 0) step = c;
    for (int h = 0; h < num_heads; ++h) {
        int second;
        int64_t k;
        switch (head_mode) {
        case 1: second = h & 1; k = h / 2; break;
        case 2: second = -1; k = h; break;
        case 3: second = 0; k = h; break;
        default: second = 1; k = h; break;
        }
        if (family == 1) kind[h] = second < 0 ? K_SU : (second ? K_SA2 : K_SA1);
        else             kind[h] = second < 0 ? K_FU : (second ? K_FA2 : K_FA1);
        off[h] = (family == 2) ? (k * step) % l : 0;
    }
    return 0;
}

/* ---- forward ------------------------------------------------------------------------------ */

/* One query row of one (batch, head): S_ij = q_i.k_j / sqrt(d) over j in A(i) ([G] §01), then a
 * two-pass softmax  m = max_j S_ij, Z = sum_j exp(S_ij - m), P_ij = exp(S_ij - m) / Z, and
 * O_i = sum_j P_ij v_j, lse_i = m + ln Z ([G] §02).  Reading for a row with no allowed key
 * ([G] §02 warns such a row has no softmax): O_i = 0 and lse_i = -inf.
 * Widths: d is the width of the query and key rows (the dot product, hence the 1/sqrt(d) scale),
 * e the width of the value rows and of O.  e = d except with half-size query-key projections
 * ([R] §4.5: the CIFAR-10 model halves its QK projection, so d = e / 2 there).
 * qi is the query row; kh (n x d) and vh (n x e) point at the (batch, head) slabs.  set and s are
 * scratch of n. */
static void fwd_row(const double *qi, const double *kh, const double *vh, int64_t d, int64_t e,
                    int kind, int64_t l, int64_t c, int64_t o, int64_t i, int64_t *set, double *s,
                    double *orow, double *lse)
{
    int64_t cnt = oracle_row_set(kind, i, l, c, o, set);
    for (int64_t t = 0; t < e; ++t) orow[t] = 0.0;
    if (cnt == 0) { *lse = -INFINITY; return; }
    const double scale = 1.0 / sqrt((double)d);
    double m = -INFINITY;
    for (int64_t a = 0; a < cnt; ++a) {
        const double *kj = kh + set[a] * d;
        double acc = 0.0;
        for (int64_t t = 0; t < d; ++t) acc += qi[t] * kj[t];
        s[a] = acc * scale;
        if (s[a] > m) m = s[a];
    }
    double z = 0.0;
    for (int64_t a = 0; a < cnt; ++a) z += exp(s[a] - m);
    for (int64_t a = 0; a < cnt; ++a) {
        const double p = exp(s[a] - m) / z;
        const double *vj = vh + set[a] * e;
        for (int64_t t = 0; t < e; ++t) orow[t] += p * vj[t];
    }
    *lse = m + log(z);
}

/* Full forward.  q, k: B x H x n x d; v, o: B x H x n x e; lse: B x H x n. */
void oracle_fwd(const double *q, const double *k, const double *v, int64_t B, int64_t H, int64_t n,
                int64_t d, int64_t e, const int *kind, const int64_t *off, int64_t l, int64_t c,
                double *o, double *lse)
{
#pragma omp parallel
    {
        int64_t *set = (int64_t *)malloc(sizeof(int64_t) * (size_t)n);
        double *s = (double *)malloc(sizeof(double) * (size_t)n);
#pragma omp for schedule(dynamic, 32)
        for (int64_t r = 0; r < B * H * n; ++r) {
            const int64_t bh = r / n, i = r % n, h = bh % H;
            const size_t bq = (size_t)bh * (size_t)n * (size_t)d, bv = (size_t)bh * (size_t)n * (size_t)e;
            fwd_row(q + bq + (size_t)i * (size_t)d, k + bq, v + bv, d, e, kind[h], l, c, off[h], i,
                    set, s, o + (size_t)r * (size_t)e, lse + r);
        }
        free(set);
        free(s);
    }
}

/* Forward for a chosen list of flat rows r = (b*H + h)*n + i; o_rows is nrows x e. */
void oracle_fwd_rows(const double *q, const double *k, const double *v, int64_t B, int64_t H,
                     int64_t n, int64_t d, int64_t e, const int *kind, const int64_t *off, int64_t l,
                     int64_t c, int64_t nrows, const int64_t *rows, double *o_rows,
                     double *lse_rows)
{
    (void)B;
#pragma omp parallel
    {
        int64_t *set = (int64_t *)malloc(sizeof(int64_t) * (size_t)n);
        double *s = (double *)malloc(sizeof(double) * (size_t)n);
#pragma omp for schedule(dynamic, 1)
        for (int64_t a = 0; a < nrows; ++a) {
            const int64_t r = rows[a], bh = r / n, i = r % n, h = bh % H;
            const size_t bq = (size_t)bh * (size_t)n * (size_t)d, bv = (size_t)bh * (size_t)n * (size_t)e;
            fwd_row(q + bq + (size_t)i * (size_t)d, k + bq, v + bv, d, e, kind[h], l, c, off[h], i,
                    set, s, o_rows + (size_t)a * (size_t)e, lse_rows + a);
        }
        free(set);
        free(s);
    }
}

/* Decode step: one new query row per (batch, head) at position pos, against the cached keys and
 * values of rows 0..pos (the sampling setting of [R] §2/§3, where each generated position attends
 * to its allowed set among the positions already produced).  By the definition of A(pos) (a
 * subset of {j <= pos}) this is exactly row pos of the forward pass: the same fwd_row, with the
 * query taken from q[b, h] instead of Q[b, h, pos].  q: B x H x d; k: B x H x n x d; v:
 * B x H x n x e (rows past pos are never read); o: B x H x e; lse: B x H. */
void oracle_decode(const double *q, const double *k, const double *v, int64_t B, int64_t H, int64_t n,
                   int64_t d, int64_t e, const int *kind, const int64_t *off, int64_t l, int64_t c,
                   int64_t pos, double *o, double *lse)
{
#pragma omp parallel
    {
        int64_t *set = (int64_t *)malloc(sizeof(int64_t) * (size_t)n);
        double *s = (double *)malloc(sizeof(double) * (size_t)n);
#pragma omp for schedule(dynamic, 1)
        for (int64_t bh = 0; bh < B * H; ++bh) {
            const int64_t h = bh % H;
            const size_t bq = (size_t)bh * (size_t)n * (size_t)d, bv = (size_t)bh * (size_t)n * (size_t)e;
            fwd_row(q + (size_t)bh * (size_t)d, k + bq, v + bv, d, e, kind[h], l, c, off[h], pos, set,
                    s, o + (size_t)bh * (size_t)e, lse + bh);
        }
        free(set);
        free(s);
    }
}

/* ---- backward ----------------------------------------------------------------------------- */
/* Plain calculus of the forward for a loss L with dL/dO = dO:
 *   P_ij  = exp(S_ij - lse_i)                    (j in A(i))
 *   dV_j  = sum_{i : j in A(i)} P_ij dO_i
 *   dP_ij = dO_i . v_j
 *   D_i   = sum_{j in A(i)} P_ij dP_ij
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = sum_{j in A(i)} dS_ij k_j / sqrt(d)
 *   dK_j  = sum_{i : j in A(i)} dS_ij q_i / sqrt(d)
 * [R] §3.4 recomputes attention in the backward pass instead of storing it; that is a
 * memory/time trade with no effect on these values, so the oracle simply evaluates them. */

/* Row quantities of query i: lse_i, D_i and (if dqrow != NULL) dQ_i.  qh, kh, dqrow have rows of
 * width d; vh, doh rows of width e (see fwd_row). */
static void bwd_row(const double *qh, const double *kh, const double *vh, const double *doh,
                    int64_t d, int64_t e, int kind, int64_t l, int64_t c, int64_t o, int64_t i,
                    int64_t *set, double *s, double *dp, double *lse_out, double *D_out, double *dqrow)
{
    const double scale = 1.0 / sqrt((double)d);
    int64_t cnt = oracle_row_set(kind, i, l, c, o, set);
    if (dqrow)
        for (int64_t t = 0; t < d; ++t) dqrow[t] = 0.0;
    if (cnt == 0) { *lse_out = -INFINITY; *D_out = 0.0; return; }
    const double *qi = qh + i * d, *doi = doh + i * e;
    double m = -INFINITY;
    for (int64_t a = 0; a < cnt; ++a) {
        const double *kj = kh + set[a] * d, *vj = vh + set[a] * e;
        double acc = 0.0, accp = 0.0;
        for (int64_t t = 0; t < d; ++t) acc += qi[t] * kj[t];
        for (int64_t t = 0; t < e; ++t) accp += doi[t] * vj[t];
        s[a] = acc * scale;
        dp[a] = accp;
        if (s[a] > m) m = s[a];
    }
    double z = 0.0;
    for (int64_t a = 0; a < cnt; ++a) z += exp(s[a] - m);
    const double lse = m + log(z);
    double D = 0.0;
    for (int64_t a = 0; a < cnt; ++a) D += exp(s[a] - lse) * dp[a];
    if (dqrow)
        for (int64_t a = 0; a < cnt; ++a) {
            const double ds = exp(s[a] - lse) * (dp[a] - D);
            const double *kj = kh + set[a] * d;
            for (int64_t t = 0; t < d; ++t) dqrow[t] += ds * kj[t] * scale;
        }
    *lse_out = lse;
    *D_out = D;
}

/* Key quantities of key j given lse and D of every row of the (batch, head): dK_j (width d) and
 * dV_j (width e). */
static void bwd_key(const double *qh, const double *kh, const double *vh, const double *doh,
                    int64_t n, int64_t d, int64_t e, int kind, int64_t l, int64_t c, int64_t o,
                    int64_t j, const double *lse, const double *D, double *dkrow, double *dvrow)
{
    const double scale = 1.0 / sqrt((double)d);
    for (int64_t t = 0; t < d; ++t) dkrow[t] = 0.0;
    for (int64_t t = 0; t < e; ++t) dvrow[t] = 0.0;
    const double *kj = kh + j * d, *vj = vh + j * e;
    for (int64_t i = j; i < n; ++i) {
        if (!oracle_allowed(kind, i, j, l, c, o)) continue;
        const double *qi = qh + i * d, *doi = doh + i * e;
        double acc = 0.0, accp = 0.0;
        for (int64_t t = 0; t < d; ++t) acc += qi[t] * kj[t];
        for (int64_t t = 0; t < e; ++t) accp += doi[t] * vj[t];
        const double p = exp(acc * scale - lse[i]);
        const double ds = p * (accp - D[i]);
        for (int64_t t = 0; t < e; ++t) dvrow[t] += p * doi[t];
        for (int64_t t = 0; t < d; ++t) dkrow[t] += ds * qi[t] * scale;
    }
}

/* Full backward.  q, k, dq, dk: B x H x n x d; v, dout, dv: B x H x n x e. */
void oracle_bwd(const double *q, const double *k, const double *v, const double *dout, int64_t B,
                int64_t H, int64_t n, int64_t d, int64_t e, const int *kind, const int64_t *off,
                int64_t l, int64_t c, double *dq, double *dk, double *dv)
{
    const int64_t rows = B * H * n;
    double *lse = (double *)malloc(sizeof(double) * (size_t)rows);
    double *D = (double *)malloc(sizeof(double) * (size_t)rows);
#pragma omp parallel
    {
        int64_t *set = (int64_t *)malloc(sizeof(int64_t) * (size_t)n);
        double *s = (double *)malloc(sizeof(double) * (size_t)n);
        double *dp = (double *)malloc(sizeof(double) * (size_t)n);
#pragma omp for schedule(dynamic, 32)
        for (int64_t r = 0; r < rows; ++r) {
            const int64_t bh = r / n, i = r % n, h = bh % H;
            const size_t bq = (size_t)bh * (size_t)n * (size_t)d, bv = (size_t)bh * (size_t)n * (size_t)e;
            bwd_row(q + bq, k + bq, v + bv, dout + bv, d, e, kind[h], l, c, off[h], i, set, s, dp,
                    lse + r, D + r, dq + (size_t)r * (size_t)d);
        }
#pragma omp for schedule(dynamic, 32)
        for (int64_t r = 0; r < rows; ++r) {
            const int64_t bh = r / n, j = r % n, h = bh % H;
            const size_t bq = (size_t)bh * (size_t)n * (size_t)d, bv = (size_t)bh * (size_t)n * (size_t)e;
            bwd_key(q + bq, k + bq, v + bv, dout + bv, n, d, e, kind[h], l, c, off[h], j,
                    lse + bh * n, D + bh * n, dk + (size_t)r * (size_t)d, dv + (size_t)r * (size_t)e);
        }
        free(set);
        free(s);
        free(dp);
    }
    free(lse);
    free(D);
}

/* dQ for a chosen list of flat query rows (nrows x d); also returns each row's lse and D. */
void oracle_bwd_rows(const double *q, const double *k, const double *v, const double *dout,
                     int64_t B, int64_t H, int64_t n, int64_t d, int64_t e, const int *kind,
                     const int64_t *off, int64_t l, int64_t c, int64_t nrows, const int64_t *rows,
                     double *dq_rows, double *lse_rows, double *D_rows)
{
    (void)B;
#pragma omp parallel
    {
        int64_t *set = (int64_t *)malloc(sizeof(int64_t) * (size_t)n);
        double *s = (double *)malloc(sizeof(double) * (size_t)n);
        double *dp = (double *)malloc(sizeof(double) * (size_t)n);
#pragma omp for schedule(dynamic, 1)
        for (int64_t a = 0; a < nrows; ++a) {
            const int64_t r = rows[a], bh = r / n, i = r % n, h = bh % H;
            const size_t bq = (size_t)bh * (size_t)n * (size_t)d, bv = (size_t)bh * (size_t)n * (size_t)e;
            bwd_row(q + bq, k + bq, v + bv, dout + bv, d, e, kind[h], l, c, off[h], i, set, s, dp,
                    lse_rows + a, D_rows + a, dq_rows + (size_t)a * (size_t)d);
        }
        free(set);
        free(s);
        free(dp);
    }
}

/* dK (nkeys x d) and dV (nkeys x e) for a chosen list of flat key rows r = (b*H + h)*n + j.  Key j's
 * gradients sum over the rows i that read it (j in A(i)), using those rows' lse and D; so the
 * lse and D of exactly those rows are evaluated first (plain row formulas), found by the same
 * predicate scan as bwd_key's. */
void oracle_bwd_keys(const double *q, const double *k, const double *v, const double *dout,
                     int64_t B, int64_t H, int64_t n, int64_t d, int64_t e, const int *kind,
                     const int64_t *off, int64_t l, int64_t c, int64_t nkeys, const int64_t *keys,
                     double *dk_rows, double *dv_rows)
{
    const int64_t nbh = B * H;
    char *need = (char *)calloc((size_t)(nbh * n), 1);
    for (int64_t a = 0; a < nkeys; ++a) {
        const int64_t r = keys[a], bh = r / n, j = r % n, h = bh % H;
        for (int64_t i = j; i < n; ++i)
            if (oracle_allowed(kind[h], i, j, l, c, off[h])) need[bh * n + i] = 1;
    }
    double *lse = (double *)malloc(sizeof(double) * (size_t)(nbh * n));
    double *D = (double *)malloc(sizeof(double) * (size_t)(nbh * n));
#pragma omp parallel
    {
        int64_t *set = (int64_t *)malloc(sizeof(int64_t) * (size_t)n);
        double *s = (double *)malloc(sizeof(double) * (size_t)n);
        double *dp = (double *)malloc(sizeof(double) * (size_t)n);
#pragma omp for schedule(dynamic, 32)
        for (int64_t r = 0; r < nbh * n; ++r) {
            const int64_t bh = r / n, i = r % n, h = bh % H;
            if (!need[r]) continue;
            const size_t bq = (size_t)bh * (size_t)n * (size_t)d, bv = (size_t)bh * (size_t)n * (size_t)e;
            bwd_row(q + bq, k + bq, v + bv, dout + bv, d, e, kind[h], l, c, off[h], i, set, s, dp,
                    lse + r, D + r, NULL);
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t a = 0; a < nkeys; ++a) {
            const int64_t r = keys[a], bh = r / n, j = r % n, h = bh % H;
            const size_t bq = (size_t)bh * (size_t)n * (size_t)d, bv = (size_t)bh * (size_t)n * (size_t)e;
            bwd_key(q + bq, k + bq, v + bv, dout + bv, n, d, e, kind[h], l, c, off[h], j,
                    lse + bh * n, D + bh * n, dk_rows + (size_t)a * (size_t)d,
                    dv_rows + (size_t)a * (size_t)e);
        }
        free(set);
        free(s);
        free(dp);
    }
    free(need);
    free(lse);
    free(D);
}

/* Number of OpenMP threads the oracle runs on (for reporting). */
int oracle_num_threads(void)
{
    int t = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            t = omp_get_num_threads();
#endif
        }
    }
    return t;
}
