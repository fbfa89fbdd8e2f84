/*
 * bakron_oracle.c -- plain, slow, FP64 reference for the BaKron two-sided
 * adaptive-rounding solve.  TEST INFRASTRUCTURE ONLY: nothing in the product
 * library calls, links or includes this file; only the tests, the smoke check
 * and the benchmark's CPU-baseline leg use it.  It shares no code with the CUDA
 * path.
 *
 * Source pages: "BaKron: Efficient Quantization with Kronecker-Factored
 * Hessians" (pith.science review of arXiv 2608.06291, section "What carries the
 * argument" = Proposition 3.1, "Core claim" = Theorem 3.2, referee report on
 * Algorithm 6 and Appendix C) and the arXiv abstract ("FastKron", mlsanity.com).
 *
 * Notation (all matrices row-major, double precision):
 *   W   m x n weight matrix, row i = output channel, column j = input channel.
 *   LtA n x n unit-lower-triangular normalised Cholesky factor of A^{-1}
 *       (LtA = LA * diag(LA)^{-1}, LA LA^T = A^{-1}), input side.
 *   LtB m x m the same for B^{-1}, output side.
 *   s   per-row grid step (float, as the GPU holds it), codes in [qmin, qmax].
 *
 * Proposition 3.1: a GPTQ step on vec(W) (column-major vec, Hessian A (x) B)
 * that rounds entry (i,j) with residual D_ij subtracts the outer product
 *      LtB[:, i] * D_ij * LtA[:, j]^T
 * from the not-yet-rounded entries; it only reaches rows >= i and columns >= j.
 * Hence the "intended output" (Theorem 3.2's order-independent target):
 *      Wt_ij = W_ij - sum_{(i',j') < (i,j)} LtB[i,i'] * D_i'j' * LtA[j,j']
 * over the strict product order (i' <= i, j' <= j, not both equal), with
 *      code_ij = clamp(rint(Wt_ij / s_i)),  D_ij = Wt_ij - s_i * code_ij.
 *
 * Every routine below computes this same target in a different order.  The
 * rounding decision is taken in fp32 (the precision the GPU kernel uses):
 * x = (float)Wt / s, round half to even, clamp.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Rounding decision of the fixed per-row grid: fp32 divide, round half to
 * even (nearbyintf under the default rounding mode), clamp to [qmin, qmax]. */
static int decide(double wt, float s, int qmin, int qmax)
{
    float x = (float)wt / s;
    float r = nearbyintf(x);
    if (!(r >= (float)qmin)) r = (float)qmin; /* also maps NaN to qmin */
    if (r > (float)qmax) r = (float)qmax;
    return (int)r;
}

int bko_decide(double wt, float s, int qmin, int qmax) { return decide(wt, s, qmin, qmax); }

static int imin(int a, int b) { return a < b ? a : b; }
static int imax(int a, int b) { return a > b ? a : b; }

/* ------------------------------------------------------------------------ */
/* Anti-diagonal "pull" solver (BaKron-antidiagonal evaluated entry by entry).
 *
 * Splitting the intended-output sum by column:
 *   Wt_ij = W_ij - sum_{j'<j} R_ij' LtA[j,j'] - S_ij,
 *   S_ij  = sum_{i'<i} LtB[i,i'] D_i'j,      R_ij = S_ij + D_ij,
 * i.e. R = LtB * D column by column.  Entries on one anti-diagonal i+j=k are
 * incomparable, so they are evaluated in parallel (Theorem 3.2's anti-diagonal
 * parallelism); diagonals run in increasing k.
 *
 * forced != NULL: teacher-forced mode.  The residual uses forced[i*n+j] as the
 * code (D = Wt - s*forced), while codes[] receives the oracle's own decision
 * on its Wt.  This is how a candidate code matrix is checked entry by entry.
 * Wt_out / D_out may be NULL.
 */
void bko_pull(int m, int n, const double *W, const double *LtA, const double *LtB,
              const float *s, int qmin, int qmax, const int32_t *forced,
              int32_t *codes, double *Wt_out, double *D_out, int nthreads)
{
    double *R = (double *)calloc((size_t)m * n, sizeof(double));
    double *Dt = (double *)calloc((size_t)m * n, sizeof(double)); /* Dt[j*m+i] = D_ij */
    if (nthreads < 1) nthreads = 1;
    for (int k = 0; k <= m + n - 2; ++k) {
        int i0 = imax(0, k - (n - 1)), i1 = imin(m - 1, k);
#pragma omp parallel for num_threads(nthreads) schedule(static)
        for (int i = i0; i <= i1; ++i) {
            int j = k - i;
            const double *Rrow = R + (size_t)i * n;
            const double *Arow = LtA + (size_t)j * n;
            double u = 0.0;
#pragma omp simd reduction(+ : u)
            for (int jp = 0; jp < j; ++jp) u += Rrow[jp] * Arow[jp];
            const double *Dcol = Dt + (size_t)j * m;
            const double *Brow = LtB + (size_t)i * m;
            double sc = 0.0;
#pragma omp simd reduction(+ : sc)
            for (int ip = 0; ip < i; ++ip) sc += Brow[ip] * Dcol[ip];
            double wt = W[(size_t)i * n + j] - u - sc;
            int own = decide(wt, s[i], qmin, qmax);
            int used = forced ? forced[(size_t)i * n + j] : own;
            double d = wt - (double)s[i] * (double)used;
            Dt[(size_t)j * m + i] = d;
            R[(size_t)i * n + j] = sc + d;
            codes[(size_t)i * n + j] = own;
            if (Wt_out) Wt_out[(size_t)i * n + j] = wt;
            if (D_out) D_out[(size_t)i * n + j] = d;
        }
    }
    free(R);
    free(Dt);
}

/* Same pull recurrences, visiting entries in a caller-given order
 * (order[2t], order[2t+1]) = (i, j) of the t-th entry.  Valid for any linear
 * extension of the product order; used to show the result does not depend on
 * which one is taken (Theorem 3.2). */
void bko_pull_order(int m, int n, const double *W, const double *LtA, const double *LtB,
                    const float *s, int qmin, int qmax, const int32_t *order,
                    int32_t *codes, double *Wt_out)
{
    double *R = (double *)calloc((size_t)m * n, sizeof(double));
    double *Dt = (double *)calloc((size_t)m * n, sizeof(double));
    for (long t = 0; t < (long)m * n; ++t) {
        int i = order[2 * t], j = order[2 * t + 1];
        double u = 0.0, sc = 0.0;
        for (int jp = 0; jp < j; ++jp) u += R[(size_t)i * n + jp] * LtA[(size_t)j * n + jp];
        for (int ip = 0; ip < i; ++ip) sc += LtB[(size_t)i * m + ip] * Dt[(size_t)j * m + ip];
        double wt = W[(size_t)i * n + j] - u - sc;
        int c = decide(wt, s[i], qmin, qmax);
        double d = wt - (double)s[i] * (double)c;
        Dt[(size_t)j * m + i] = d;
        R[(size_t)i * n + j] = sc + d;
        codes[(size_t)i * n + j] = c;
        if (Wt_out) Wt_out[(size_t)i * n + j] = wt;
    }
    free(R);
    free(Dt);
}

/* ------------------------------------------------------------------------ */
/* BaKron-antidiagonal in its literal "push" form: round every entry of
 * anti-diagonal k from the current Wt, then subtract LtB * D_k * LtA^T where
 * D_k holds only diagonal k's residuals.  O(m^2 n^2) work; small inputs. */
void bko_antidiag_push(int m, int n, const double *W, const double *LtA, const double *LtB,
                       const float *s, int qmin, int qmax, int32_t *codes, double *Wt_out)
{
    double *Wt = (double *)malloc((size_t)m * n * sizeof(double));
    memcpy(Wt, W, (size_t)m * n * sizeof(double));
    for (int k = 0; k <= m + n - 2; ++k) {
        int i0 = imax(0, k - (n - 1)), i1 = imin(m - 1, k);
        for (int i = i0; i <= i1; ++i) {
            int j = k - i;
            double wt = Wt[(size_t)i * n + j];
            int c = decide(wt, s[i], qmin, qmax);
            codes[(size_t)i * n + j] = c;
            if (Wt_out) Wt_out[(size_t)i * n + j] = wt;
        }
        for (int i = i0; i <= i1; ++i) {
            int j = k - i;
            double d = Wt[(size_t)i * n + j] - (double)s[i] * codes[(size_t)i * n + j];
            /* rank-1 term of the diagonal's update, restricted to entries not yet rounded */
            for (int i2 = i; i2 < m; ++i2) {
                double b = LtB[(size_t)i2 * m + i] * d;
                if (b == 0.0) continue;
                for (int j2 = j; j2 < n; ++j2) {
                    if (i2 + j2 <= k) continue;
                    Wt[(size_t)i2 * n + j2] -= b * LtA[(size_t)j2 * n + j];
                }
            }
        }
    }
    free(Wt);
}

/* ------------------------------------------------------------------------ */
/* BaKron (Algorithm 6): divide and conquer over ranges of "diagonal keys".
 *
 * key(i,j) = i/T + j/T with T = 1 gives the pages' entry-level anti-diagonal
 * ranges; T > 1 gives ranges of T x T tile diagonals (the cut the GPU path
 * uses).  Either key is monotone in the product order, so a key range is a
 * down-closed-then-up-closed band and the recursion below is valid for both.
 *
 *   solve(k, l): if l <= leaf: process the band's entries in order of
 *                (key, i+j, i), each rounded from the current Wt and its
 *                update pushed to the later entries of the same band;
 *                else h = floor(l/2); solve(k, h);
 *                Wt[tgt] -= (LtB * (D[src] * LtA^T))[tgt]   (two matmuls)
 *                with src = keys [k, k+h), tgt = keys [k+h, k+l);
 *                solve(k+h, l-h).
 */
typedef struct {
    int m, n, T, leaf, qmin, qmax;
    const double *LtA, *LtB;
    const float *s;
    double *Wt, *D, *X;
    int32_t *codes;
    double *Wt_out;
    int32_t *ord; /* scratch for the leaf's entry list */
} rec_ctx;

static int keyof(const rec_ctx *c, int i, int j) { return i / c->T + j / c->T; }

static int cmp_entries(const void *pa, const void *pb)
{
    const int32_t *a = (const int32_t *)pa, *b = (const int32_t *)pb;
    /* a[0] = key, a[1] = i, a[2] = j */
    if (a[0] != b[0]) return a[0] - b[0];
    int da = a[1] + a[2], db = b[1] + b[2];
    if (da != db) return da - db;
    return a[1] - b[1];
}

static void rec_leaf(rec_ctx *c, int k, int l)
{
    int m = c->m, n = c->n, cnt = 0;
    for (int i = 0; i < m; ++i)
        for (int j = 0; j < n; ++j) {
            int key = keyof(c, i, j);
            if (key >= k && key < k + l) {
                c->ord[3 * cnt] = key;
                c->ord[3 * cnt + 1] = i;
                c->ord[3 * cnt + 2] = j;
                ++cnt;
            }
        }
    qsort(c->ord, (size_t)cnt, 3 * sizeof(int32_t), cmp_entries);
    for (int t = 0; t < cnt; ++t) {
        int i = c->ord[3 * t + 1], j = c->ord[3 * t + 2];
        double wt = c->Wt[(size_t)i * n + j];
        int q = decide(wt, c->s[i], c->qmin, c->qmax);
        double d = wt - (double)c->s[i] * q;
        c->codes[(size_t)i * n + j] = q;
        if (c->Wt_out) c->Wt_out[(size_t)i * n + j] = wt;
        c->D[(size_t)i * n + j] = d;
        for (int u = t + 1; u < cnt; ++u) {
            int i2 = c->ord[3 * u + 1], j2 = c->ord[3 * u + 2];
            if (i2 < i || j2 < j) continue;
            c->Wt[(size_t)i2 * n + j2] -= c->LtB[(size_t)i2 * m + i] * d * c->LtA[(size_t)j2 * n + j];
        }
    }
}

static void rec_update(rec_ctx *c, int k, int h, int l)
{
    int m = c->m, n = c->n;
    /* X = D[src] * LtA^T : X[i][j2] = sum_{j : key(i,j) in src} D[i][j] * LtA[j2][j] */
    for (int i = 0; i < m; ++i)
        for (int j2 = 0; j2 < n; ++j2) {
            double acc = 0.0;
            for (int j = 0; j <= j2; ++j) {
                int key = keyof(c, i, j);
                if (key >= k && key < k + h) acc += c->D[(size_t)i * n + j] * c->LtA[(size_t)j2 * n + j];
            }
            c->X[(size_t)i * n + j2] = acc;
        }
    /* Wt[tgt] -= LtB * X */
    for (int i2 = 0; i2 < m; ++i2)
        for (int j2 = 0; j2 < n; ++j2) {
            int key = keyof(c, i2, j2);
            if (key < k + h || key >= k + l) continue;
            double acc = 0.0;
            for (int i = 0; i <= i2; ++i) acc += c->LtB[(size_t)i2 * m + i] * c->X[(size_t)i * n + j2];
            c->Wt[(size_t)i2 * n + j2] -= acc;
        }
}

static void rec_solve(rec_ctx *c, int k, int l)
{
    if (l <= c->leaf) {
        rec_leaf(c, k, l);
        return;
    }
    int h = l / 2;
    rec_solve(c, k, h);
    rec_update(c, k, h, l);
    rec_solve(c, k + h, l - h);
}

void bko_recursive(int m, int n, const double *W, const double *LtA, const double *LtB,
                   const float *s, int qmin, int qmax, int T, int leaf,
                   int32_t *codes, double *Wt_out)
{
    rec_ctx c;
    c.m = m; c.n = n; c.T = T < 1 ? 1 : T; c.leaf = leaf < 1 ? 1 : leaf;
    c.qmin = qmin; c.qmax = qmax; c.LtA = LtA; c.LtB = LtB; c.s = s;
    c.Wt = (double *)malloc((size_t)m * n * sizeof(double));
    memcpy(c.Wt, W, (size_t)m * n * sizeof(double));
    c.D = (double *)calloc((size_t)m * n, sizeof(double));
    c.X = (double *)calloc((size_t)m * n, sizeof(double));
    c.ord = (int32_t *)malloc((size_t)m * n * 3 * sizeof(int32_t));
    c.codes = codes; c.Wt_out = Wt_out;
    int nkeys = (m - 1) / c.T + (n - 1) / c.T + 1;
    rec_solve(&c, 0, nkeys);
    free(c.Wt); free(c.D); free(c.X); free(c.ord);
}

/* ------------------------------------------------------------------------ */
/* BaKron-recursive: split the columns in half when the block is at least as
 * wide as it is tall, else the rows; solve the first half, subtract its
 * contribution from the second half with two matmuls, solve the second half.
 * (The pages give the cost recurrence F(m,n) - F(m,n1) - F(m,n2) = 2 m n1 n2
 * for this variant; here only the result matters.) */
typedef struct {
    int m, n, qmin, qmax;
    const double *LtA, *LtB;
    const float *s;
    double *Wt, *D, *X;
    int32_t *codes;
    double *Wt_out;
} rc_ctx;

static void rc_update(rc_ctx *c, int fr0, int fr1, int fc0, int fc1, int sr0, int sr1, int sc0, int sc1)
{
    int m = c->m, n = c->n;
    for (int i = fr0; i < fr1; ++i)
        for (int j2 = sc0; j2 < sc1; ++j2) {
            double acc = 0.0;
            for (int j = fc0; j < fc1; ++j) acc += c->D[(size_t)i * n + j] * c->LtA[(size_t)j2 * n + j];
            c->X[(size_t)i * n + j2] = acc;
        }
    for (int i2 = sr0; i2 < sr1; ++i2)
        for (int j2 = sc0; j2 < sc1; ++j2) {
            double acc = 0.0;
            for (int i = fr0; i < fr1; ++i) acc += c->LtB[(size_t)i2 * m + i] * c->X[(size_t)i * n + j2];
            c->Wt[(size_t)i2 * n + j2] -= acc;
        }
}

static void rc_solve(rc_ctx *c, int r0, int r1, int c0, int c1)
{
    int mr = r1 - r0, nc = c1 - c0, n = c->n;
    if (mr == 1 && nc == 1) {
        double wt = c->Wt[(size_t)r0 * n + c0];
        int q = decide(wt, c->s[r0], c->qmin, c->qmax);
        c->codes[(size_t)r0 * n + c0] = q;
        if (c->Wt_out) c->Wt_out[(size_t)r0 * n + c0] = wt;
        c->D[(size_t)r0 * n + c0] = wt - (double)c->s[r0] * q;
        return;
    }
    if (nc >= mr) {
        int cm = c0 + nc / 2;
        rc_solve(c, r0, r1, c0, cm);
        rc_update(c, r0, r1, c0, cm, r0, r1, cm, c1);
        rc_solve(c, r0, r1, cm, c1);
    } else {
        int rm = r0 + mr / 2;
        rc_solve(c, r0, rm, c0, c1);
        rc_update(c, r0, rm, c0, c1, rm, r1, c0, c1);
        rc_solve(c, rm, r1, c0, c1);
    }
}

void bko_rowcol(int m, int n, const double *W, const double *LtA, const double *LtB,
                const float *s, int qmin, int qmax, int32_t *codes, double *Wt_out)
{
    rc_ctx c;
    c.m = m; c.n = n; c.qmin = qmin; c.qmax = qmax; c.LtA = LtA; c.LtB = LtB; c.s = s;
    c.Wt = (double *)malloc((size_t)m * n * sizeof(double));
    memcpy(c.Wt, W, (size_t)m * n * sizeof(double));
    c.D = (double *)calloc((size_t)m * n, sizeof(double));
    c.X = (double *)calloc((size_t)m * n, sizeof(double));
    c.codes = codes; c.Wt_out = Wt_out;
    rc_solve(&c, 0, m, 0, n);
    free(c.Wt); free(c.D); free(c.X);
}

/* ------------------------------------------------------------------------ */
/* BaKron-naive (Algorithm 2): GPTQ/LDLQ on q = vec(W) (column-major, q = j*m+i)
 * with the lower Cholesky factor Lh of H^{-1}, H = A (x) B, given explicitly as
 * an mn x mn row-major matrix (built by the caller without using Kronecker
 * structure in the solve).  For q = 0..mn-1: v_q = Q(w_q),
 * w_{q'} -= ((w_q - v_q) / Lh[q][q]) * Lh[q'][q] for q' > q. */
void bko_naive_vec(int m, int n, const double *W, const double *Lh, const float *s,
                   int qmin, int qmax, int32_t *codes, double *Wt_out)
{
    long N = (long)m * n;
    double *w = (double *)malloc((size_t)N * sizeof(double));
    for (int j = 0; j < n; ++j)
        for (int i = 0; i < m; ++i) w[(size_t)j * m + i] = W[(size_t)i * n + j];
    for (long q = 0; q < N; ++q) {
        int i = (int)(q % m), j = (int)(q / m);
        double wq = w[q];
        int c = decide(wq, s[i], qmin, qmax);
        codes[(size_t)i * n + j] = c;
        if (Wt_out) Wt_out[(size_t)i * n + j] = wq;
        double e = (wq - (double)s[i] * c) / Lh[(size_t)q * N + q];
        for (long q2 = q + 1; q2 < N; ++q2) w[q2] -= e * Lh[(size_t)q2 * N + q];
    }
    free(w);
}

/* ------------------------------------------------------------------------ */
/* Brute force over every code matrix of a tiny problem (mn <= 8): a code
 * matrix C is consistent when, with D_{i'j'} = Wt_{i'j'} - s_i' C_{i'j'} and
 * Wt from the intended-output sum (evaluated literally as the double sum over
 * strict predecessors), every entry satisfies C_ij = decide(Wt_ij).
 * Returns the number of consistent matrices; the first is written to
 * first_codes.  Also returns, through best_loss/best_codes, the code matrix of
 * least proxy loss tr((W-V)^T B (W-V) A) over all enumerated matrices. */
long bko_brute(int m, int n, const double *W, const double *LtA, const double *LtB,
               const double *A, const double *B, const float *s, int qmin, int qmax,
               int32_t *first_codes, double *best_loss, int32_t *best_codes)
{
    int N = m * n;
    if (N > 8) return -1;
    int base = qmax - qmin + 1;
    long total = 1;
    for (int t = 0; t < N; ++t) total *= base;
    int32_t C[8];
    double Wt[8], D[8], E[8];
    long found = 0;
    *best_loss = INFINITY;
    for (long idx = 0; idx < total; ++idx) {
        long r = idx;
        for (int t = 0; t < N; ++t) { C[t] = qmin + (int)(r % base); r /= base; }
        int ok = 1;
        /* visit entries in anti-diagonal order so predecessors are known */
        for (int k = 0; k <= m + n - 2 && ok; ++k)
            for (int i = imax(0, k - (n - 1)); i <= imin(m - 1, k); ++i) {
                int j = k - i;
                double acc = 0.0;
                for (int ip = 0; ip <= i; ++ip)
                    for (int jp = 0; jp <= j; ++jp) {
                        if (ip == i && jp == j) continue;
                        acc += LtB[ip + i * m] * D[ip * n + jp] * LtA[jp + j * n];
                    }
                Wt[i * n + j] = W[i * n + j] - acc;
                D[i * n + j] = Wt[i * n + j] - (double)s[i] * C[i * n + j];
                if (decide(Wt[i * n + j], s[i], qmin, qmax) != C[i * n + j]) ok = 0;
            }
        if (ok) {
            if (found == 0) memcpy(first_codes, C, (size_t)N * sizeof(int32_t));
            ++found;
        }
        /* proxy loss of this candidate */
        for (int t = 0; t < N; ++t) E[t] = W[t] - (double)s[t / n] * C[t];
        double loss = 0.0;
        for (int i = 0; i < m; ++i)
            for (int j = 0; j < n; ++j) {
                double be = 0.0, ea = 0.0;
                for (int p = 0; p < m; ++p) be += B[i * m + p] * E[p * n + j];
                for (int p = 0; p < n; ++p) ea += E[i * n + p] * A[p * n + j];
                loss += be * ea;
            }
        if (loss < *best_loss) {
            *best_loss = loss;
            memcpy(best_codes, C, (size_t)N * sizeof(int32_t));
        }
    }
    return found;
}

int bko_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
