/*
 * dc_oracle.c -- plain fp64 CPU reference for Lightweight DC attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; only the test suite, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code with the CUDA library.
 *
 * What it computes (the "Lightweight DC" paragraph of the m.aitntnews.com blog
 * post on the NanoGPT speedrun, section "第二刀-砍层内"): the layer's own Q/K
 * are reused for an extra local attention window of W (=112) tokens; each
 * head's scores over that window go through a softmax; the H per-head
 * probability maps are merged, with input-dependent weights, into one shared
 * map; that shared map is applied to every head's V with a per-head scale.
 * Written out for query token t of document [a, b) and head h:
 *
 *   window      j in [lo(t), t],  lo(t) = max(a, t - W + 1)
 *   scores      s_h(t,j) = sigma * <q_h(t), k_h(j)>
 *   softmax     p_h(t,j) = exp(s_h(t,j) - m_h(t)) / Z_h(t),
 *               m_h = max_j s_h, Z_h = sum_j exp(s_h - m_h),
 *               lse_h(t) = m_h(t) + ln Z_h(t)
 *   composition P(t,j)   = sum_h c[t,h] * p_h(t,j)          (c signed, per token)
 *   head scale  o_h(t)   = g[t,h] * sum_j P(t,j) * v_h(j)
 *
 * The backward pass is not on the page; it is the chain rule applied to the
 * definition above, for L with dL/do_h(t) = dO_h(t):
 *
 *   E_h(t,j)  = <dO_h(t), v_h(j)>
 *   dg[t,h]   = sum_j P(t,j) * E_h(t,j)
 *   dP(t,j)   = sum_h g[t,h] * E_h(t,j)
 *   dc[t,h]   = sum_j dP(t,j) * p_h(t,j)
 *   ds_h(t,j) = c[t,h] * p_h(t,j) * (dP(t,j) - dc[t,h])      (softmax Jacobian)
 *   dq_h(t)   = sigma * sum_j ds_h(t,j) * k_h(j)
 *   dk_h(j)   = sigma * sum_{t : j in window(t)} ds_h(t,j) * q_h(t)
 *   dv_h(j)   = sum_{t : j in window(t)} P(t,j) * g[t,h] * dO_h(t)
 *
 * Layouts: q, k, v, o, dO, dq, dk, dv are [N][H][d]; c, g, lse, dc, dg are
 * [N][H]; pmap is [N][W] with pmap[t][w] = P(t, t - W + 1 + w) and 0 where that
 * key is outside the window or the document.  cu_seqlens has num_docs + 1
 * entries, 0 = cu[0] <= ... <= cu[num_docs] = N.
 *
 * OpenMP only splits independent output rows across threads; every sum is
 * taken in the plain order written above.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

int dc_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Index of the document that holds token t: the last i with cu[i] <= t. */
static int doc_of(const int32_t *cu, int num_docs, int64_t t)
{
    int i = 0;
    while (i + 1 < num_docs && cu[i + 1] <= t)
        ++i;
    return i;
}

static double dot(const double *x, const double *y, int d)
{
    double s = 0.0;
    for (int e = 0; e < d; ++e)
        s += x[e] * y[e];
    return s;
}

static int check_args(int64_t N, int num_docs, const int32_t *cu, int H, int d, int W)
{
    if (N < 0 || H < 1 || d < 1 || W < 1 || num_docs < 0)
        return 1;
    if (N > 0 && num_docs < 1)
        return 1;
    if (num_docs >= 1) {
        if (cu[0] != 0 || cu[num_docs] != N)
            return 1;
        for (int i = 0; i < num_docs; ++i)
            if (cu[i + 1] < cu[i])
                return 1;
    }
    return 0;
}

/*
 * Softmax of head h for query t over its window [lo, t]:
 * p[j - lo] = p_h(t, j); returns lse_h(t).
 */
static double head_softmax(const double *q, const double *k, int H, int d, double sigma,
                           int64_t t, int64_t lo, int h, double *p)
{
    const int64_t n = t - lo + 1;
    const double *qt = q + ((size_t)t * H + h) * d;
    double m = -INFINITY;
    for (int64_t jj = 0; jj < n; ++jj) {
        const double *kj = k + ((size_t)(lo + jj) * H + h) * d;
        p[jj] = sigma * dot(qt, kj, d);
        if (p[jj] > m)
            m = p[jj];
    }
    double Z = 0.0;
    for (int64_t jj = 0; jj < n; ++jj) {
        p[jj] = exp(p[jj] - m);
        Z += p[jj];
    }
    for (int64_t jj = 0; jj < n; ++jj)
        p[jj] /= Z;
    return m + log(Z);
}

int dc_oracle_fwd(int64_t N, int num_docs, const int32_t *cu, int H, int d, int W, double sigma,
                  const double *q, const double *k, const double *v,
                  const double *c, const double *g,
                  double *o, double *lse, double *pmap)
{
    if (check_args(N, num_docs, cu, H, d, W))
        return 1;
    int fail = 0;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)H * W);   /* p[h][jj] */
        double *P = (double *)malloc(sizeof(double) * (size_t)W);
        if (!p || !P) {
#pragma omp atomic write
            fail = 1;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t t = 0; t < N; ++t) {
            if (!p || !P)
                continue;
            const int64_t a = cu[doc_of(cu, num_docs, t)];
            const int64_t lo = (t - W + 1 > a) ? t - W + 1 : a;
            const int64_t n = t - lo + 1;
            for (int h = 0; h < H; ++h) {
                double l = head_softmax(q, k, H, d, sigma, t, lo, h, p + (size_t)h * W);
                if (lse)
                    lse[(size_t)t * H + h] = l;
            }
            /* shared map: P(t, j) = sum_h c[t,h] p_h(t, j) */
            for (int64_t jj = 0; jj < n; ++jj) {
                double s = 0.0;
                for (int h = 0; h < H; ++h)
                    s += c[(size_t)t * H + h] * p[(size_t)h * W + jj];
                P[jj] = s;
            }
            /* o_h(t) = g[t,h] * sum_j P(t, j) v_h(j) */
            for (int h = 0; h < H; ++h) {
                double *ot = o + ((size_t)t * H + h) * d;
                for (int e = 0; e < d; ++e) {
                    double s = 0.0;
                    for (int64_t jj = 0; jj < n; ++jj)
                        s += P[jj] * v[((size_t)(lo + jj) * H + h) * d + e];
                    ot[e] = g[(size_t)t * H + h] * s;
                }
            }
            if (pmap) {
                double *row = pmap + (size_t)t * W;
                for (int w = 0; w < W; ++w) {
                    const int64_t j = t - W + 1 + w;
                    row[w] = (j >= lo) ? P[j - lo] : 0.0;
                }
            }
        }
        free(p);
        free(P);
    }
    return fail ? 2 : 0;
}

int dc_oracle_bwd(int64_t N, int num_docs, const int32_t *cu, int H, int d, int W, double sigma,
                  const double *q, const double *k, const double *v,
                  const double *c, const double *g, const double *dO,
                  double *dq, double *dk, double *dv, double *dc, double *dg)
{
    if (check_args(N, num_docs, cu, H, d, W))
        return 1;
    double *lse = (double *)malloc(sizeof(double) * ((size_t)N * H + 1));
    if (!lse)
        return 2;
    int fail = 0;

    /* Pass 1, one query row at a time: dg, dc, dq (and lse for pass 2). */
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (size_t)H * W);   /* p_h(t, j) */
        double *E = (double *)malloc(sizeof(double) * (size_t)H * W);   /* E_h(t, j) */
        double *P = (double *)malloc(sizeof(double) * (size_t)W);
        double *dP = (double *)malloc(sizeof(double) * (size_t)W);
        if (!p || !E || !P || !dP) {
#pragma omp atomic write
            fail = 1;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t t = 0; t < N; ++t) {
            if (!p || !E || !P || !dP)
                continue;
            const int64_t a = cu[doc_of(cu, num_docs, t)];
            const int64_t lo = (t - W + 1 > a) ? t - W + 1 : a;
            const int64_t n = t - lo + 1;
            const double *ct = c + (size_t)t * H;
            const double *gt = g + (size_t)t * H;
            for (int h = 0; h < H; ++h)
                lse[(size_t)t * H + h] = head_softmax(q, k, H, d, sigma, t, lo, h, p + (size_t)h * W);
            for (int h = 0; h < H; ++h)
                for (int64_t jj = 0; jj < n; ++jj)
                    E[(size_t)h * W + jj] = dot(dO + ((size_t)t * H + h) * d,
                                                v + ((size_t)(lo + jj) * H + h) * d, d);
            for (int64_t jj = 0; jj < n; ++jj) {
                double sP = 0.0, sdP = 0.0;
                for (int h = 0; h < H; ++h) {
                    sP += ct[h] * p[(size_t)h * W + jj];
                    sdP += gt[h] * E[(size_t)h * W + jj];
                }
                P[jj] = sP;
                dP[jj] = sdP;
            }
            for (int h = 0; h < H; ++h) {
                double sg = 0.0, sc = 0.0;
                for (int64_t jj = 0; jj < n; ++jj) {
                    sg += P[jj] * E[(size_t)h * W + jj];
                    sc += dP[jj] * p[(size_t)h * W + jj];
                }
                dg[(size_t)t * H + h] = sg;
                dc[(size_t)t * H + h] = sc;
            }
            for (int h = 0; h < H; ++h) {
                double *dqt = dq + ((size_t)t * H + h) * d;
                for (int e = 0; e < d; ++e)
                    dqt[e] = 0.0;
                for (int64_t jj = 0; jj < n; ++jj) {
                    const double ds = ct[h] * p[(size_t)h * W + jj] * (dP[jj] - dc[(size_t)t * H + h]);
                    const double *kj = k + ((size_t)(lo + jj) * H + h) * d;
                    for (int e = 0; e < d; ++e)
                        dqt[e] += sigma * ds * kj[e];
                }
            }
        }
        free(p);
        free(E);
        free(P);
        free(dP);
    }
    if (fail) {
        free(lse);
        return 2;
    }

    /* Pass 2, one key row at a time: dk, dv over the queries whose window holds j. */
#pragma omp parallel
    {
        double *ph = (double *)malloc(sizeof(double) * (size_t)H);
        if (!ph) {
#pragma omp atomic write
            fail = 1;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t j = 0; j < N; ++j) {
            if (!ph)
                continue;
            const int dj = doc_of(cu, num_docs, j);
            const int64_t b = cu[dj + 1];
            const int64_t hi = (j + W - 1 < b - 1) ? j + W - 1 : b - 1;
            for (int h = 0; h < H; ++h)
                for (int e = 0; e < d; ++e) {
                    dk[((size_t)j * H + h) * d + e] = 0.0;
                    dv[((size_t)j * H + h) * d + e] = 0.0;
                }
            for (int64_t t = j; t <= hi; ++t) {
                const double *ct = c + (size_t)t * H;
                const double *gt = g + (size_t)t * H;
                double P = 0.0, dP = 0.0;
                for (int h = 0; h < H; ++h) {
                    const double s = sigma * dot(q + ((size_t)t * H + h) * d, k + ((size_t)j * H + h) * d, d);
                    ph[h] = exp(s - lse[(size_t)t * H + h]);
                    P += ct[h] * ph[h];
                    dP += gt[h] * dot(dO + ((size_t)t * H + h) * d, v + ((size_t)j * H + h) * d, d);
                }
                for (int h = 0; h < H; ++h) {
                    const double ds = ct[h] * ph[h] * (dP - dc[(size_t)t * H + h]);
                    const double *qt = q + ((size_t)t * H + h) * d;
                    const double *dOt = dO + ((size_t)t * H + h) * d;
                    double *dkj = dk + ((size_t)j * H + h) * d;
                    double *dvj = dv + ((size_t)j * H + h) * d;
                    for (int e = 0; e < d; ++e) {
                        dkj[e] += sigma * ds * qt[e];
                        dvj[e] += P * gt[h] * dOt[e];
                    }
                }
            }
        }
        free(ph);
    }
    free(lse);
    return fail ? 2 : 0;
}
