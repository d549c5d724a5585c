/*
 * fa_oracle.c -- fp64 CPU oracle for the exact attention forward and its
 * gradient (oracle_attention_bwd, at the end of this file).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The product path
 * (the CUDA library and its Python binding) never calls it, and this file
 * shares no code, header or constant with that path.
 *
 * What it computes is the plain definition of scaled-dot-product attention,
 * written out row by row in double precision, with the full score row
 * materialised:
 *
 *   s_j   = scale * sum_k q[i,k] * k[j,k]          for every visible key j
 *   m     = max_j s_j
 *   p_j   = exp(s_j - m),   l = sum_j p_j
 *   O[i]  = sum_j p_j * v[j,:] / l
 *   LSE_i = m + ln(l)
 *
 * Sources: "2.3 FlashAttention与IO感知注意力(1)" (aiknowledge.cn), section 1.1,
 * function standard_attention (S = Q K^T, masked_fill(-inf), softmax, P V);
 * "flash_attention.py" (forceinjection.github.io), function standard_attention
 * (S = Q K^T / sqrt(d), softmax over the last axis, P V).  The causal mask is
 * the lower triangle including the diagonal (key j visible from query i iff
 * j <= i); the logsumexp output is the natural-log logsumexp of the scaled
 * scores over the visible keys.  Neither of these two is printed on the pages
 * as code; both are the plainest reading of the mask hook on the aiknowledge.cn
 * page and of the causal= flag of the packed call on the intelliparadigm.com
 * page (section 5.2).
 *
 * Subtracting the row max before exp() is the usual stable evaluation of the
 * same softmax; it changes nothing but rounding.
 *
 * Layout: q, k, v are [B, H, N, d] row-major doubles (the exact values of the
 * fp16/bf16 inputs, widened).  The caller may ask for a subset of query rows
 * (rows[0..nrows-1], each in [0, N)); the same subset is taken in every
 * (b, h).  o is [B, H, nrows, d] and lse is [B, H, nrows] (lse may be NULL).
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Number of keys query row i can see. */
static int visible_keys(int i, int N, int causal)
{
    return causal ? (i + 1 < N ? i + 1 : N) : N;
}

/*
 * Scores of one query row against the first nvis keys, then the softmax
 * weights p_j = exp(s_j - m) (unnormalised) and their sum l.  Returns m.
 */
static double row_weights(const double *qrow, const double *K, int nvis, int d,
                          double scale, double *p, double *l_out)
{
    double m = -INFINITY;
    for (int j = 0; j < nvis; ++j) {
        const double *krow = K + (size_t)j * d;
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += qrow[c] * krow[c];
        p[j] = scale * dot;
        if (p[j] > m) m = p[j];
    }
    double l = 0.0;
    for (int j = 0; j < nvis; ++j) {
        p[j] = exp(p[j] - m);
        l += p[j];
    }
    *l_out = l;
    return m;
}

/* Returns 0 on success, -1 on a bad argument, -2 when out of memory. */
int oracle_attention_fwd(const double *q, const double *k, const double *v,
                         double *o, double *lse, int B, int H, int N, int d,
                         double scale, int causal, const int *rows, int nrows)
{
    if (!q || !k || !v || !o || !rows) return -1;
    if (B < 1 || H < 1 || N < 1 || d < 1 || nrows < 0) return -1;
    for (int r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= N) return -1;

    const long long total = (long long)B * H * nrows;
    int failed = 0;

#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)N);
        if (!p) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (long long t = 0; t < total; ++t) {
            if (!p) continue;
            const long long bh = t / nrows;
            const int r = (int)(t % nrows);
            const int i = rows[r];
            const double *Q = q + (size_t)bh * N * d;
            const double *K = k + (size_t)bh * N * d;
            const double *V = v + (size_t)bh * N * d;
            double *out = o + ((size_t)bh * nrows + r) * d;

            const int nvis = visible_keys(i, N, causal);
            double l;
            const double m = row_weights(Q + (size_t)i * d, K, nvis, d, scale, p, &l);
            for (int c = 0; c < d; ++c) out[c] = 0.0;
            for (int j = 0; j < nvis; ++j) {
                const double *vrow = V + (size_t)j * d;
                const double w = p[j];
                for (int c = 0; c < d; ++c) out[c] += w * vrow[c];
            }
            for (int c = 0; c < d; ++c) out[c] /= l;
            if (lse) lse[(size_t)bh * nrows + r] = m + log(l);
        }
        free(p);
    }
    return failed ? -2 : 0;
}

/*
 * The normalised weight row P[i, 0..N-1] of one (b, h) slice (q, k are that
 * slice's [N, d] matrices); weights of keys the row cannot see are written as
 * 0.  Used by the tests to check that every row of P sums to one.
 */
int oracle_attention_probs(const double *q, const double *k, int N, int d,
                           double scale, int causal, int i, double *p_out)
{
    if (!q || !k || !p_out || N < 1 || d < 1 || i < 0 || i >= N) return -1;
    const int nvis = visible_keys(i, N, causal);
    double l;
    row_weights(q + (size_t)i * d, k, nvis, d, scale, p_out, &l);
    for (int j = 0; j < nvis; ++j) p_out[j] /= l;
    for (int j = nvis; j < N; ++j) p_out[j] = 0.0;
    return 0;
}

/*
 * Forward with a local window and an ALiBi bias: the two masks the packed
 * call of "Windows下RTX 3090编译Flash Attention 2.8.3全指南" (intelliparadigm.com)
 * names as keyword arguments (window_size=(-1,-1), alibi_slopes, section
 * 5.2 and 10.1) without defining them.  The reading taken:
 *
 *   key j visible from query i  iff  (left  < 0 || j >= i - left)
 *                                 && (right < 0 || j <= i + right)
 *                                 && (!causal  || j <= i)
 *   s_ij = scale * q_i . k_j  -  slope[h] * |i - j|        (slopes may be NULL)
 *
 * then the same softmax, P V and logsumexp as oracle_attention_fwd.  The
 * visible keys of a row form one range that always contains j = i.
 * Layout and row subset as oracle_attention_fwd; slopes is [H] or NULL.
 */
int oracle_attention_fwd_masked(const double *q, const double *k, const double *v,
                                double *o, double *lse, int B, int H, int N, int d,
                                double scale, int causal, int left, int right,
                                const double *slopes, const int *rows, int nrows)
{
    if (!q || !k || !v || !o || !rows) return -1;
    if (B < 1 || H < 1 || N < 1 || d < 1 || nrows < 0) return -1;
    for (int r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= N) return -1;
    const long long total = (long long)B * H * nrows;
    int failed = 0;

#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)N);
        if (!p) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (long long t = 0; t < total; ++t) {
            if (!p) continue;
            const long long bh = t / nrows;
            const int h = (int)(bh % H);
            const int r = (int)(t % nrows);
            const int i = rows[r];
            int lo = left < 0 ? 0 : i - left;
            int hi = right < 0 ? N - 1 : i + right;
            if (lo < 0) lo = 0;
            if (hi > N - 1) hi = N - 1;
            if (causal && hi > i) hi = i;
            const double slope = slopes ? slopes[h] : 0.0;
            const double *Q = q + (size_t)bh * N * d;
            const double *K = k + (size_t)bh * N * d;
            const double *V = v + (size_t)bh * N * d;
            const double *qrow = Q + (size_t)i * d;
            double *out = o + ((size_t)bh * nrows + r) * d;
            double m = -INFINITY;
            for (int j = lo; j <= hi; ++j) {
                const double *krow = K + (size_t)j * d;
                double dot = 0.0;
                for (int c = 0; c < d; ++c) dot += qrow[c] * krow[c];
                p[j] = scale * dot - slope * fabs((double)(i - j));
                if (p[j] > m) m = p[j];
            }
            double l = 0.0;
            for (int j = lo; j <= hi; ++j) {
                p[j] = exp(p[j] - m);
                l += p[j];
            }
            for (int c = 0; c < d; ++c) out[c] = 0.0;
            for (int j = lo; j <= hi; ++j) {
                const double *vrow = V + (size_t)j * d;
                for (int c = 0; c < d; ++c) out[c] += p[j] * vrow[c];
            }
            for (int c = 0; c < d; ++c) out[c] /= l;
            if (lse) lse[(size_t)bh * nrows + r] = m + log(l);
        }
        free(p);
    }
    return failed ? -2 : 0;
}

/*
 * Gradient of the forward above with respect to q, k and v, for an upstream
 * gradient dout of O (the logsumexp output is taken as not differentiated).
 * The pages name the backward pass only by its recomputation of the score
 * tile from saved row statistics ("Windows下RTX 3090编译Flash Attention 2.8.3
 * 全指南", sections 1 and 7); what it computes is fixed by the forward
 * definition and the chain rule, written out here per (b, h):
 *
 *   P[i,j]  = exp(s_ij - LSE_i)              visible keys, 0 elsewhere
 *   dV[j]   = sum_i P[i,j] * dout[i]
 *   dP[i,j] = dout[i] . v[j]
 *   D_i     = sum_j P[i,j] * dP[i,j]
 *   dS[i,j] = P[i,j] * (dP[i,j] - D_i)        (row softmax Jacobian)
 *   dq[i]   = scale * sum_j dS[i,j] * k[j]
 *   dk[j]   = scale * sum_i dS[i,j] * q[i]
 *
 * Layout as the forward: every array [B, H, N, d] row-major doubles.
 * Returns 0 on success, -1 on a bad argument, -2 when out of memory.
 */
int oracle_attention_bwd(const double *q, const double *k, const double *v,
                         const double *dout, double *dq, double *dk, double *dv,
                         int B, int H, int N, int d, double scale, int causal)
{
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return -1;
    if (B < 1 || H < 1 || N < 1 || d < 1) return -1;
    const long long heads = (long long)B * H;
    int failed = 0;

#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)N);
        double *dp = (double *)malloc(sizeof(double) * (size_t)N);
        if (!p || !dp) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (long long bh = 0; bh < heads; ++bh) {
            if (!p || !dp) continue;
            const size_t off = (size_t)bh * N * d;
            const double *Q = q + off, *K = k + off, *V = v + off, *DO = dout + off;
            double *DQ = dq + off, *DK = dk + off, *DV = dv + off;
            memset(DQ, 0, sizeof(double) * (size_t)N * d);
            memset(DK, 0, sizeof(double) * (size_t)N * d);
            memset(DV, 0, sizeof(double) * (size_t)N * d);
            for (int i = 0; i < N; ++i) {
                const int nvis = visible_keys(i, N, causal);
                const double *qrow = Q + (size_t)i * d;
                const double *dorow = DO + (size_t)i * d;
                double l;
                row_weights(qrow, K, nvis, d, scale, p, &l);
                for (int j = 0; j < nvis; ++j) p[j] /= l;
                double D = 0.0;
                for (int j = 0; j < nvis; ++j) {
                    const double *vrow = V + (size_t)j * d;
                    double dot = 0.0;
                    for (int c = 0; c < d; ++c) dot += dorow[c] * vrow[c];
                    dp[j] = dot;
                    D += p[j] * dot;
                }
                double *dqrow = DQ + (size_t)i * d;
                for (int j = 0; j < nvis; ++j) {
                    const double ds = p[j] * (dp[j] - D);
                    const double *krow = K + (size_t)j * d;
                    double *dkrow = DK + (size_t)j * d;
                    double *dvrow = DV + (size_t)j * d;
                    for (int c = 0; c < d; ++c) {
                        dqrow[c] += scale * ds * krow[c];
                        dkrow[c] += scale * ds * qrow[c];
                        dvrow[c] += p[j] * dorow[c];
                    }
                }
            }
        }
        free(p);
        free(dp);
    }
    return failed ? -2 : 0;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
