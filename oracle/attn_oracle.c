/*
 * Exact attention oracle, fp64, CPU.  TEST INFRASTRUCTURE ONLY.
 *
 * This file is the checker for the CUDA path, not part of it.  Only the test
 * suite, the smoke entry and the bench's CPU-baseline / reference arm may load
 * it.  It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes is the plain definition of attention that the FlashAttention
 * pages state the tiled method reproduces exactly ("Exact, not approximate",
 * vibeengines.com/paper/flash-attention; "Guarantees versus empirical results",
 * chorfi.xyz/research/papers/paper-flashattention):
 *
 *   s_ij = scale * <q_i, k_j>               (j allowed: all j, or j <= i if causal)
 *   m_i  = max_j s_ij,  l_i = sum_j e^{s_ij - m_i}
 *   P_ij = e^{s_ij - m_i} / l_i             (safe softmax, "The math, worked with
 *                                            real numbers", first formula)
 *   O_i  = sum_j P_ij v_j,  LSE_i = m_i + ln l_i
 *
 * The full score row is materialised, one row at a time (the pages'
 * "standard attention" that writes every score, "The real bottleneck").
 *
 * The backward pass is not written out on the pages (they only say that the
 * method recomputes attention in the backward pass).  It is the textbook
 * softmax / matrix-product calculus for the scalar loss L = sum(O * dO):
 *   dV_j  = sum_i P_ij dO_i
 *   dP_ij = <dO_i, v_j>
 *   D_i   = sum_j P_ij dP_ij
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale * sum_j dS_ij k_j,   dK_j = scale * sum_i dS_ij q_i
 *
 * oracle_softmax_online / oracle_attn_fwd_tiled restate the pages' online
 * softmax update rule ("The math, worked with real numbers", the three update
 * lines for m_new, l_new, O_new; final answer O / l) with an arbitrary block
 * size; they exist only to pin the "block size never changes the answer" and
 * "online softmax == naive softmax" assertions ("Solve it yourself").
 *
 * Further functions, each with its own comment: Nq queries against Nk keys
 * (oracle_attn_fwd_rect), a block mask (oracle_attn_fwd_blockmask), and
 * dropout with a Philox4x64-10 keep mask (oracle_attn_fwd_dropout /
 * oracle_attn_bwd_dropout).
 *
 * Layout: every tensor is [BH][N][d] row-major fp64 (BH = batch * heads);
 * lse is [BH][N].  Masking convention (not fixed by the pages): square,
 * top-left aligned causal mask, key j allowed iff j <= i.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Safe softmax of one row: subtract the row max, exponentiate, divide by the sum. */
void oracle_softmax_naive(const double* s, long n, double* w)
{
    double m = -INFINITY;
    for (long j = 0; j < n; ++j)
        if (s[j] > m) m = s[j];
    double l = 0.0;
    for (long j = 0; j < n; ++j) {
        w[j] = exp(s[j] - m);
        l += w[j];
    }
    for (long j = 0; j < n; ++j) w[j] /= l;
}

/*
 * Online softmax: walk the row in blocks, keep a running max m and a running
 * sum l; when a block raises the max, the old sum is multiplied by
 * e^{m_old - m_new} before the block's terms are added.  m_trace / l_trace (may
 * be NULL) receive m and l after each block.
 */
void oracle_softmax_online(const double* s, long n, long block, double* w,
                           double* m_trace, double* l_trace)
{
    double m = -INFINITY, l = 0.0;
    long nb = 0;
    for (long b0 = 0; b0 < n; b0 += block) {
        long b1 = b0 + block < n ? b0 + block : n;
        double m_blk = -INFINITY;
        for (long j = b0; j < b1; ++j)
            if (s[j] > m_blk) m_blk = s[j];
        double m_new = m > m_blk ? m : m_blk;
        double add = 0.0;
        for (long j = b0; j < b1; ++j) add += exp(s[j] - m_new);
        l = (m == -INFINITY ? 0.0 : l * exp(m - m_new)) + add;
        m = m_new;
        if (m_trace) m_trace[nb] = m;
        if (l_trace) l_trace[nb] = l;
        ++nb;
    }
    for (long j = 0; j < n; ++j) w[j] = exp(s[j] - m) / l;
}

/* Number of keys row i may attend to. */
static long n_allowed(long i, long N, int causal) { return causal ? i + 1 : N; }

static double dot(const double* a, const double* b, long d)
{
    double acc = 0.0;
    for (long t = 0; t < d; ++t) acc += a[t] * b[t];
    return acc;
}

/*
 * One query row of one head: materialise the score row into srow (length N),
 * turn it into P in place, write O_i and LSE_i.
 */
static void fwd_row_nk(const double* qi, const double* k, const double* v, double* oi,
                       double* lse_i, long nk, long d, double scale, double* srow)
{
    double m = -INFINITY;
    for (long j = 0; j < nk; ++j) {
        srow[j] = scale * dot(qi, k + j * d, d);
        if (srow[j] > m) m = srow[j];
    }
    double l = 0.0;
    for (long j = 0; j < nk; ++j) {
        srow[j] = exp(srow[j] - m);
        l += srow[j];
    }
    for (long t = 0; t < d; ++t) oi[t] = 0.0;
    for (long j = 0; j < nk; ++j) {
        double p = srow[j] / l;
        const double* vj = v + j * d;
        for (long t = 0; t < d; ++t) oi[t] += p * vj[t];
    }
    *lse_i = m + log(l);
}

/* One query row i of a square [N x N] problem. */
static void fwd_row(const double* qi, const double* k, const double* v, double* oi,
                    double* lse_i, long i, long N, long d, double scale, int causal,
                    double* srow)
{
    fwd_row_nk(qi, k, v, oi, lse_i, n_allowed(i, N, causal), d, scale, srow);
}

/* Forward over all heads and rows.  Returns 0, or -1 on bad sizes / no memory. */
int oracle_attn_fwd(const double* q, const double* k, const double* v, double* o,
                    double* lse, long BH, long N, long d, double scale, int causal)
{
    if (BH < 0 || N < 0 || d < 1) return -1;
    int err = 0;
#pragma omp parallel
    {
        double* srow = (double*)malloc((size_t)(N > 0 ? N : 1) * sizeof(double));
        if (!srow) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 16) collapse(2)
        for (long h = 0; h < BH; ++h)
            for (long i = 0; i < N; ++i) {
                if (!srow) continue;
                const long base = h * N * d;
                fwd_row(q + base + i * d, k + base, v + base, o + base + i * d,
                        lse + h * N + i, i, N, d, scale, causal, srow);
            }
        free(srow);
    }
    return err;
}

/*
 * Forward with Nq queries against Nk keys (q: [BH][Nq][d]; k, v: [BH][Nk][d];
 * o: [BH][Nq][d]; lse: [BH][Nq]), the shape of decoding against a key/value
 * cache.  Causal reading (the pages fix no convention for Nq != Nk): the
 * queries are the last Nq positions of the sequence, so query i sees keys
 * j <= Nk - Nq + i; this needs Nk >= Nq and gives the square mask when Nq = Nk.
 * Returns 0, or -1 on bad sizes / no memory.
 */
int oracle_attn_fwd_rect(const double* q, const double* k, const double* v, double* o,
                         double* lse, long BH, long Nq, long Nk, long d, double scale,
                         int causal)
{
    if (BH < 0 || Nq < 0 || Nk < 1 || d < 1 || (causal && Nk < Nq)) return -1;
    int err = 0;
#pragma omp parallel
    {
        double* srow = (double*)malloc((size_t)Nk * sizeof(double));
        if (!srow) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 16) collapse(2)
        for (long h = 0; h < BH; ++h)
            for (long i = 0; i < Nq; ++i) {
                if (!srow) continue;
                const long nk = causal ? Nk - Nq + i + 1 : Nk;
                fwd_row_nk(q + (h * Nq + i) * d, k + h * Nk * d, v + h * Nk * d, o + (h * Nq + i) * d,
                           lse + h * Nq + i, nk, d, scale, srow);
            }
        free(srow);
    }
    return err;
}

/*
 * Block-sparse forward: the square problem restricted to the (query block, key
 * block) pairs a block mask allows.  The pages name block-sparse FlashAttention
 * as the approximate extension of the method (guide, "Prerequisites"); the
 * approximation is the mask itself, and over the allowed pairs this is the
 * definition above with every other score at -inf (weight exactly 0).
 *   mask: uint8 [Hm][nqb][nkb], nqb = ceil(N / br), nkb = ceil(N / bc); the
 *   head h of row block bh uses mask + (bh % H) * mask_h_stride (stride 0: one
 *   mask for every head).  Key j is allowed for query i iff
 *   mask[(i / br) * nkb + j / bc] != 0 and, when causal, j <= i.
 * A row that no key is allowed for gets O = 0 and LSE = -inf (a reading: the
 * pages do not say).  Returns 0, or -1 on bad sizes / no memory.
 */
int oracle_attn_fwd_blockmask(const double* q, const double* k, const double* v, double* o,
                              double* lse, long BH, long H, long N, long d, double scale,
                              int causal, const unsigned char* mask, long mask_h_stride,
                              long br, long bc)
{
    if (BH < 0 || H < 1 || N < 0 || d < 1 || br < 1 || bc < 1 || mask_h_stride < 0 || !mask)
        return -1;
    const long nkb = (N + bc - 1) / bc;
    int err = 0;
#pragma omp parallel
    {
        double* srow = (double*)malloc((size_t)(N > 0 ? N : 1) * sizeof(double));
        if (!srow) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 16) collapse(2)
        for (long h = 0; h < BH; ++h)
            for (long i = 0; i < N; ++i) {
                if (!srow) continue;
                const unsigned char* mrow = mask + (h % H) * mask_h_stride + (i / br) * nkb;
                const double* qi = q + (h * N + i) * d;
                const double* kh = k + h * N * d;
                const double* vh = v + h * N * d;
                double* oi = o + (h * N + i) * d;
                double m = -INFINITY;
                for (long j = 0; j < N; ++j) {
                    const int allowed = mrow[j / bc] != 0 && (!causal || j <= i);
                    srow[j] = allowed ? scale * dot(qi, kh + j * d, d) : -INFINITY;
                    if (srow[j] > m) m = srow[j];
                }
                for (long t = 0; t < d; ++t) oi[t] = 0.0;
                if (m == -INFINITY) {
                    lse[h * N + i] = -INFINITY;
                    continue;
                }
                double l = 0.0;
                for (long j = 0; j < N; ++j) {
                    srow[j] = srow[j] == -INFINITY ? 0.0 : exp(srow[j] - m);
                    l += srow[j];
                }
                for (long j = 0; j < N; ++j) {
                    if (srow[j] == 0.0) continue;
                    const double pj = srow[j] / l;
                    for (long t = 0; t < d; ++t) oi[t] += pj * vh[j * d + t];
                }
                lse[h * N + i] = m + log(l);
            }
        free(srow);
    }
    return err;
}

/*
 * Forward for rows [i0, i1) of ONE head (q, k, v point at that head's [N][d]
 * block; o / lse receive i1 - i0 rows).  Used to check sampled rows of
 * workloads too large to run whole.
 */
int oracle_attn_fwd_rows(const double* q, const double* k, const double* v, double* o,
                         double* lse, long N, long d, long i0, long i1, double scale,
                         int causal)
{
    if (N < 1 || d < 1 || i0 < 0 || i1 > N || i0 > i1) return -1;
    int err = 0;
#pragma omp parallel
    {
        double* srow = (double*)malloc((size_t)N * sizeof(double));
        if (!srow) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 4)
        for (long i = i0; i < i1; ++i) {
            if (!srow) continue;
            fwd_row(q + i * d, k, v, o + (i - i0) * d, lse + (i - i0), i, N, d, scale,
                    causal, srow);
        }
        free(srow);
    }
    return err;
}

/*
 * The online (tiled) restatement: each row walks the keys in blocks of `block`,
 * updating m, l and the output accumulator with the same factor e^{m_old-m_new},
 * and divides by l at the end.
 */
int oracle_attn_fwd_tiled(const double* q, const double* k, const double* v, double* o,
                          double* lse, long BH, long N, long d, double scale, int causal,
                          long block)
{
    if (BH < 0 || N < 0 || d < 1 || block < 1) return -1;
    int err = 0;
#pragma omp parallel
    {
        double* sblk = (double*)malloc((size_t)block * sizeof(double));
        if (!sblk) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 16) collapse(2)
        for (long h = 0; h < BH; ++h)
            for (long i = 0; i < N; ++i) {
                if (!sblk) continue;
                const long base = h * N * d;
                const double* qi = q + base + i * d;
                double* oi = o + base + i * d;
                long nk = n_allowed(i, N, causal);
                double m = -INFINITY, l = 0.0;
                for (long t = 0; t < d; ++t) oi[t] = 0.0;
                for (long b0 = 0; b0 < nk; b0 += block) {
                    long b1 = b0 + block < nk ? b0 + block : nk;
                    double m_blk = -INFINITY;
                    for (long j = b0; j < b1; ++j) {
                        sblk[j - b0] = scale * dot(qi, k + base + j * d, d);
                        if (sblk[j - b0] > m_blk) m_blk = sblk[j - b0];
                    }
                    double m_new = m > m_blk ? m : m_blk;
                    double alpha = (m == -INFINITY) ? 0.0 : exp(m - m_new);
                    l *= alpha;
                    for (long t = 0; t < d; ++t) oi[t] *= alpha;
                    for (long j = b0; j < b1; ++j) {
                        double p = exp(sblk[j - b0] - m_new);
                        l += p;
                        const double* vj = v + base + j * d;
                        for (long t = 0; t < d; ++t) oi[t] += p * vj[t];
                    }
                    m = m_new;
                }
                for (long t = 0; t < d; ++t) oi[t] /= l;
                lse[h * N + i] = m + log(l);
            }
        free(sblk);
    }
    return err;
}

/*
 * Backward for all heads (dq, dk, dv fully written).  Parallel over heads only,
 * so each head's dK / dV sums run in one thread in row order.
 */
int oracle_attn_bwd(const double* q, const double* k, const double* v, const double* dO,
                    double* dq, double* dk, double* dv, long BH, long N, long d,
                    double scale, int causal)
{
    if (BH < 0 || N < 0 || d < 1) return -1;
    int err = 0;
#pragma omp parallel
    {
        double* prow = (double*)malloc((size_t)(N > 0 ? N : 1) * sizeof(double));
        double* dprow = (double*)malloc((size_t)(N > 0 ? N : 1) * sizeof(double));
        if (!prow || !dprow) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 1)
        for (long h = 0; h < BH; ++h) {
            if (!prow || !dprow) continue;
            const long base = h * N * d;
            const double *qh = q + base, *kh = k + base, *vh = v + base, *doh = dO + base;
            double *dqh = dq + base, *dkh = dk + base, *dvh = dv + base;
            memset(dkh, 0, (size_t)(N * d) * sizeof(double));
            memset(dvh, 0, (size_t)(N * d) * sizeof(double));
            for (long i = 0; i < N; ++i) {
                const double* qi = qh + i * d;
                const double* doi = doh + i * d;
                long nk = n_allowed(i, N, causal);
                /* P_i: the materialised, max-subtracted softmax row */
                double m = -INFINITY;
                for (long j = 0; j < nk; ++j) {
                    prow[j] = scale * dot(qi, kh + j * d, d);
                    if (prow[j] > m) m = prow[j];
                }
                double l = 0.0;
                for (long j = 0; j < nk; ++j) {
                    prow[j] = exp(prow[j] - m);
                    l += prow[j];
                }
                for (long j = 0; j < nk; ++j) prow[j] /= l;
                /* dP_i and D_i = sum_j P_ij dP_ij */
                double D = 0.0;
                for (long j = 0; j < nk; ++j) {
                    dprow[j] = dot(doi, vh + j * d, d);
                    D += prow[j] * dprow[j];
                }
                double* dqi = dqh + i * d;
                for (long t = 0; t < d; ++t) dqi[t] = 0.0;
                for (long j = 0; j < nk; ++j) {
                    double ds = prow[j] * (dprow[j] - D);
                    const double* kj = kh + j * d;
                    double* dkj = dkh + j * d;
                    double* dvj = dvh + j * d;
                    for (long t = 0; t < d; ++t) {
                        dqi[t] += ds * kj[t];
                        dkj[t] += ds * qi[t];
                        dvj[t] += prow[j] * doi[t];
                    }
                }
                for (long t = 0; t < d; ++t) dqi[t] *= scale;
            }
            for (long e = 0; e < N * d; ++e) dkh[e] *= scale;
        }
        free(prow);
        free(dprow);
    }
    return err;
}

/*
 * dQ for rows [i0, i1) of ONE head (q, k, v, dO point at that head's [N][d]
 * blocks; dq receives i1 - i0 rows).  Row i of dQ needs only row i of P and
 * dP, so sampled rows of workloads too large for the full backward stay cheap.
 * Same definition as oracle_attn_bwd.
 */
int oracle_attn_bwd_dq_rows(const double* q, const double* k, const double* v, const double* dO,
                            double* dq, long N, long d, long i0, long i1, double scale,
                            int causal)
{
    if (N < 1 || d < 1 || i0 < 0 || i1 > N || i0 > i1) return -1;
    int err = 0;
#pragma omp parallel
    {
        double* prow = (double*)malloc((size_t)N * sizeof(double));
        double* dprow = (double*)malloc((size_t)N * sizeof(double));
        if (!prow || !dprow) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 4)
        for (long i = i0; i < i1; ++i) {
            if (!prow || !dprow) continue;
            const double* qi = q + i * d;
            const double* doi = dO + i * d;
            long nk = n_allowed(i, N, causal);
            double m = -INFINITY;
            for (long j = 0; j < nk; ++j) {
                prow[j] = scale * dot(qi, k + j * d, d);
                if (prow[j] > m) m = prow[j];
            }
            double l = 0.0;
            for (long j = 0; j < nk; ++j) {
                prow[j] = exp(prow[j] - m);
                l += prow[j];
            }
            for (long j = 0; j < nk; ++j) prow[j] /= l;
            double D = 0.0;
            for (long j = 0; j < nk; ++j) {
                dprow[j] = dot(doi, v + j * d, d);
                D += prow[j] * dprow[j];
            }
            double* dqi = dq + (i - i0) * d;
            for (long t = 0; t < d; ++t) dqi[t] = 0.0;
            for (long j = 0; j < nk; ++j) {
                double ds = prow[j] * (dprow[j] - D);
                const double* kj = k + j * d;
                for (long t = 0; t < d; ++t) dqi[t] += ds * kj[t];
            }
            for (long t = 0; t < d; ++t) dqi[t] *= scale;
        }
        free(prow);
        free(dprow);
    }
    return err;
}

/*
 * dK and dV for keys [j0, j1) of ONE head (dk, dv receive j1 - j0 rows).  Every
 * query row that sees one of these keys is materialised in turn (its P row, dP
 * row and D_i), and only the columns j0..j1-1 are accumulated.  Cheap for the
 * last keys of a causal head, which few rows see.  Same definition as
 * oracle_attn_bwd.
 */
int oracle_attn_bwd_kv_rows(const double* q, const double* k, const double* v, const double* dO,
                            double* dk, double* dv, long N, long d, long j0, long j1,
                            double scale, int causal)
{
    if (N < 1 || d < 1 || j0 < 0 || j1 > N || j0 > j1) return -1;
    const long nj = j1 - j0;
    memset(dk, 0, (size_t)(nj * d) * sizeof(double));
    memset(dv, 0, (size_t)(nj * d) * sizeof(double));
    double* prow = (double*)malloc((size_t)N * sizeof(double));
    double* dprow = (double*)malloc((size_t)N * sizeof(double));
    if (!prow || !dprow) {
        free(prow);
        free(dprow);
        return -1;
    }
    for (long i = causal ? j0 : 0; i < N; ++i) {
        const double* qi = q + i * d;
        const double* doi = dO + i * d;
        long nk = n_allowed(i, N, causal);
        double m = -INFINITY;
        for (long j = 0; j < nk; ++j) {
            prow[j] = scale * dot(qi, k + j * d, d);
            if (prow[j] > m) m = prow[j];
        }
        double l = 0.0;
        for (long j = 0; j < nk; ++j) {
            prow[j] = exp(prow[j] - m);
            l += prow[j];
        }
        for (long j = 0; j < nk; ++j) prow[j] /= l;
        double D = 0.0;
        for (long j = 0; j < nk; ++j) {
            dprow[j] = dot(doi, v + j * d, d);
            D += prow[j] * dprow[j];
        }
        long jend = j1 < nk ? j1 : nk;
        for (long j = j0; j < jend; ++j) {
            double ds = prow[j] * (dprow[j] - D);
            double* dkj = dk + (j - j0) * d;
            double* dvj = dv + (j - j0) * d;
            for (long t = 0; t < d; ++t) {
                dkj[t] += ds * qi[t];
                dvj[t] += prow[j] * doi[t];
            }
        }
    }
    for (long e = 0; e < nj * d; ++e) dk[e] *= scale;
    free(prow);
    free(dprow);
    return 0;
}

/* ------------------------------------------------------------------ dropout
 *
 * The pages name dropout among the settings of the kernel benchmarks (guide,
 * "What to inspect") and give no generator.  Contract (a reading): the keep
 * decision for (head bh, query i, key j) is a byte of a counter-based
 * generator, Philox4x64-10 (J. K. Salmon, M. A. Moraes, R. O. Dror and D. E.
 * Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011), so the
 * backward pass regenerates the forward's mask from (seed, offset) alone:
 *   counter = (j / 32, i, bh, 0), key = (seed, offset)
 *   the 4 output words are 32 bytes, little-endian; key j uses byte j % 32
 *   keep iff that byte < t, t in [0, 256] (keep probability t / 256)
 *   kept weights are scaled by 256 / t.
 * Forward:  O_i = (256 / t) * sum_j P_ij Z_ij v_j, LSE_i unchanged (P is the
 * softmax of the undropped scores).
 * Backward (softmax calculus with the fixed mask Z, s = 256 / t):
 *   dV_j = s sum_i P_ij Z_ij dO_i,   dP_ij = s Z_ij <dO_i, v_j>,
 *   D_i = sum_j P_ij dP_ij (= <dO_i, O_i>),  dS = P o (dP - D),
 *   dQ = scale dS K,  dK = scale dS^T Q.
 */

/* Philox4x64-10: ten rounds of the Philox S-box on a 4-word counter, the
 * 2-word key bumped by the Weyl constants between rounds (the paper's
 * Philox-4x64 parameters). */
void oracle_philox4x64_10(const uint64_t ctr[4], const uint64_t key[2], uint64_t out[4])
{
    const uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
    const uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
    uint64_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
    uint64_t k0 = key[0], k1 = key[1];
    for (int r = 0; r < 10; ++r) {
        if (r > 0) {
            k0 += W0;
            k1 += W1;
        }
        const unsigned __int128 p0 = (unsigned __int128)M0 * x0;
        const unsigned __int128 p1 = (unsigned __int128)M1 * x2;
        const uint64_t hi0 = (uint64_t)(p0 >> 64), lo0 = (uint64_t)p0;
        const uint64_t hi1 = (uint64_t)(p1 >> 64), lo1 = (uint64_t)p1;
        const uint64_t y0 = hi1 ^ x1 ^ k0, y2 = hi0 ^ x3 ^ k1;
        x0 = y0;
        x1 = lo1;
        x2 = y2;
        x3 = lo0;
    }
    out[0] = x0;
    out[1] = x1;
    out[2] = x2;
    out[3] = x3;
}

/* Keep bit Z for (bh, i, j) under the contract above. */
static int dropout_keep(uint64_t seed, uint64_t offset, long bh, long i, long j, int t)
{
    const uint64_t ctr[4] = {(uint64_t)(j / 32), (uint64_t)i, (uint64_t)bh, 0};
    const uint64_t key[2] = {seed, offset};
    uint64_t w[4];
    oracle_philox4x64_10(ctr, key, w);
    const long b = j % 32;
    const unsigned byte = (unsigned)((w[b / 8] >> (8 * (b % 8))) & 0xFFu);
    return (int)byte < t;
}

/* The keep mask of one head: z[i * N + j] in {0, 1} for all i, j < N. */
int oracle_dropout_mask(unsigned char* z, long bh, long N, int t, uint64_t seed, uint64_t offset)
{
    if (N < 0 || t < 0 || t > 256) return -1;
    for (long i = 0; i < N; ++i)
        for (long j = 0; j < N; ++j) z[i * N + j] = (unsigned char)dropout_keep(seed, offset, bh, i, j, t);
    return 0;
}

/* Forward with dropout (definition above).  t = 256 is plain attention;
 * t = 0 drops everything (O = 0).  The heads given are heads bh0 .. bh0 + BH - 1
 * of the whole problem (their index enters the generator's counter). */
int oracle_attn_fwd_dropout(const double* q, const double* k, const double* v, double* o,
                            double* lse, long BH, long N, long d, double scale, int causal,
                            int t, uint64_t seed, uint64_t offset, long bh0)
{
    if (BH < 0 || N < 0 || d < 1 || t < 0 || t > 256) return -1;
    const double s_keep = t > 0 ? 256.0 / t : 0.0;
    int err = 0;
#pragma omp parallel
    {
        double* srow = (double*)malloc((size_t)(N > 0 ? N : 1) * sizeof(double));
        if (!srow) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 16) collapse(2)
        for (long h = 0; h < BH; ++h)
            for (long i = 0; i < N; ++i) {
                if (!srow) continue;
                const long base = h * N * d;
                const double* qi = q + base + i * d;
                double* oi = o + base + i * d;
                const long nk = n_allowed(i, N, causal);
                double m = -INFINITY;
                for (long j = 0; j < nk; ++j) {
                    srow[j] = scale * dot(qi, k + base + j * d, d);
                    if (srow[j] > m) m = srow[j];
                }
                double l = 0.0;
                for (long j = 0; j < nk; ++j) {
                    srow[j] = exp(srow[j] - m);
                    l += srow[j];
                }
                for (long t2 = 0; t2 < d; ++t2) oi[t2] = 0.0;
                for (long j = 0; j < nk; ++j) {
                    if (!dropout_keep(seed, offset, bh0 + h, i, j, t)) continue;
                    const double pj = s_keep * srow[j] / l;
                    const double* vj = v + base + j * d;
                    for (long t2 = 0; t2 < d; ++t2) oi[t2] += pj * vj[t2];
                }
                lse[h * N + i] = m + log(l);
            }
        free(srow);
    }
    return err;
}

/* Backward with dropout (definition above), the mask regenerated per element.
 * The heads given are heads bh0 .. bh0 + BH - 1 of the whole problem. */
int oracle_attn_bwd_dropout(const double* q, const double* k, const double* v, const double* dO,
                            double* dq, double* dk, double* dv, long BH, long N, long d,
                            double scale, int causal, int t, uint64_t seed, uint64_t offset, long bh0)
{
    if (BH < 0 || N < 0 || d < 1 || t < 0 || t > 256) return -1;
    const double s_keep = t > 0 ? 256.0 / t : 0.0;
    int err = 0;
#pragma omp parallel
    {
        double* prow = (double*)malloc((size_t)(N > 0 ? N : 1) * sizeof(double));
        double* dprow = (double*)malloc((size_t)(N > 0 ? N : 1) * sizeof(double));
        double* zrow = (double*)malloc((size_t)(N > 0 ? N : 1) * sizeof(double));
        if (!prow || !dprow || !zrow) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 1)
        for (long h = 0; h < BH; ++h) {
            if (!prow || !dprow || !zrow) continue;
            const long base = h * N * d;
            const double *qh = q + base, *kh = k + base, *vh = v + base, *doh = dO + base;
            double *dqh = dq + base, *dkh = dk + base, *dvh = dv + base;
            memset(dkh, 0, (size_t)(N * d) * sizeof(double));
            memset(dvh, 0, (size_t)(N * d) * sizeof(double));
            for (long i = 0; i < N; ++i) {
                const double* qi = qh + i * d;
                const double* doi = doh + i * d;
                const long nk = n_allowed(i, N, causal);
                double m = -INFINITY;
                for (long j = 0; j < nk; ++j) {
                    prow[j] = scale * dot(qi, kh + j * d, d);
                    if (prow[j] > m) m = prow[j];
                }
                double l = 0.0;
                for (long j = 0; j < nk; ++j) {
                    prow[j] = exp(prow[j] - m);
                    l += prow[j];
                }
                for (long j = 0; j < nk; ++j) {
                    prow[j] /= l;
                    zrow[j] = dropout_keep(seed, offset, bh0 + h, i, j, t) ? s_keep : 0.0;
                }
                double D = 0.0;
                for (long j = 0; j < nk; ++j) {
                    dprow[j] = zrow[j] * dot(doi, vh + j * d, d);
                    D += prow[j] * dprow[j];
                }
                double* dqi = dqh + i * d;
                for (long t2 = 0; t2 < d; ++t2) dqi[t2] = 0.0;
                for (long j = 0; j < nk; ++j) {
                    const double ds = prow[j] * (dprow[j] - D);
                    const double pz = prow[j] * zrow[j];
                    const double* kj = kh + j * d;
                    double* dkj = dkh + j * d;
                    double* dvj = dvh + j * d;
                    for (long t2 = 0; t2 < d; ++t2) {
                        dqi[t2] += ds * kj[t2];
                        dkj[t2] += ds * qi[t2];
                        dvj[t2] += pz * doi[t2];
                    }
                }
                for (long t2 = 0; t2 < d; ++t2) dqi[t2] *= scale;
            }
            for (long e = 0; e < N * d; ++e) dkh[e] *= scale;
        }
        free(prow);
        free(dprow);
        free(zrow);
    }
    return err;
}

/*
 * Backward of ONE head, with the work spread over threads, for heads too long
 * for oracle_attn_bwd's one-thread-per-head loop (N = 16384).  Same definition
 * as oracle_attn_bwd, and as oracle_attn_bwd_dropout when t < 256 (t = 256 is
 * plain attention: every key kept, factor 1); bh is the head's index b * H + h
 * in the whole problem, which only enters the dropout generator.
 *
 * Two passes, each parallel over independent outputs, so every sum still runs
 * in one thread in a fixed order:
 *   rows:  for each query i, the materialised row s_i, m_i = max s_i,
 *          l_i = sum e^{s_ij - m_i}, P_ij = e^{s_ij - m_i} / l_i, dP_ij and
 *          D_i = sum_j P_ij dP_ij, then dQ_i = scale sum_j P_ij (dP_ij - D_i) k_j
 *          (exactly the row loop of oracle_attn_bwd); m_i, l_i, D_i are kept.
 *   keys:  for each key j, every query i that sees it in row order: P_ij from the
 *          same s_ij, m_i, l_i, then dV_j = sum_i P_ij Z_ij dO_i and
 *          dK_j = scale sum_i P_ij (dP_ij - D_i) q_i.
 */
int oracle_attn_bwd_head(const double* q, const double* k, const double* v, const double* dO,
                         double* dq, double* dk, double* dv, long N, long d, double scale, int causal,
                         int t, uint64_t seed, uint64_t offset, long bh)
{
    if (N < 1 || d < 1 || t < 0 || t > 256) return -1;
    const double s_keep = t > 0 ? 256.0 / t : 0.0;
    double* rm = (double*)malloc((size_t)N * sizeof(double));
    double* rl = (double*)malloc((size_t)N * sizeof(double));
    double* rD = (double*)malloc((size_t)N * sizeof(double));
    if (!rm || !rl || !rD) {
        free(rm);
        free(rl);
        free(rD);
        return -1;
    }
    int err = 0;
#pragma omp parallel
    {
        double* prow = (double*)malloc((size_t)N * sizeof(double));
        double* dprow = (double*)malloc((size_t)N * sizeof(double));
        if (!prow || !dprow) {
#pragma omp atomic write
            err = -1;
        }
#pragma omp for schedule(dynamic, 8)
        for (long i = 0; i < N; ++i) {
            if (!prow || !dprow) continue;
            const double* qi = q + i * d;
            const double* doi = dO + i * d;
            const long nk = n_allowed(i, N, causal);
            double m = -INFINITY;
            for (long j = 0; j < nk; ++j) {
                prow[j] = scale * dot(qi, k + j * d, d);
                if (prow[j] > m) m = prow[j];
            }
            double l = 0.0;
            for (long j = 0; j < nk; ++j) {
                prow[j] = exp(prow[j] - m);
                l += prow[j];
            }
            for (long j = 0; j < nk; ++j) prow[j] /= l;
            double D = 0.0;
            for (long j = 0; j < nk; ++j) {
                const double z = (t == 256) ? 1.0 : (dropout_keep(seed, offset, bh, i, j, t) ? s_keep : 0.0);
                dprow[j] = z * dot(doi, v + j * d, d);
                D += prow[j] * dprow[j];
            }
            double* dqi = dq + i * d;
            for (long e = 0; e < d; ++e) dqi[e] = 0.0;
            for (long j = 0; j < nk; ++j) {
                const double ds = prow[j] * (dprow[j] - D);
                const double* kj = k + j * d;
                for (long e = 0; e < d; ++e) dqi[e] += ds * kj[e];
            }
            for (long e = 0; e < d; ++e) dqi[e] *= scale;
            rm[i] = m;
            rl[i] = l;
            rD[i] = D;
        }
        free(prow);
        free(dprow);
    }
    if (err) {
        free(rm);
        free(rl);
        free(rD);
        return err;
    }
#pragma omp parallel for schedule(dynamic, 8)
    for (long j = 0; j < N; ++j) {
        const double* kj = k + j * d;
        const double* vj = v + j * d;
        double* dkj = dk + j * d;
        double* dvj = dv + j * d;
        for (long e = 0; e < d; ++e) dkj[e] = dvj[e] = 0.0;
        for (long i = causal ? j : 0; i < N; ++i) {
            const double* qi = q + i * d;
            const double* doi = dO + i * d;
            const double p = exp(scale * dot(qi, kj, d) - rm[i]) / rl[i];
            const double z = (t == 256) ? 1.0 : (dropout_keep(seed, offset, bh, i, j, t) ? s_keep : 0.0);
            const double dp = z * dot(doi, vj, d);
            const double ds = p * (dp - rD[i]);
            const double pz = p * z;
            for (long e = 0; e < d; ++e) {
                dkj[e] += ds * qi[e];
                dvj[e] += pz * doi[e];
            }
        }
        for (long e = 0; e < d; ++e) dkj[e] *= scale;
    }
    free(rm);
    free(rl);
    free(rD);
    return 0;
}
