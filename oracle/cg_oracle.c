/*
 * cg_oracle.c -- plain fp64 CPU reference for the producer of the composition
 * weights c and head scales g.
 *
 * TEST INFRASTRUCTURE ONLY, like dc_oracle.c: nothing on the product path
 * links, loads or calls it, and it shares no code with the CUDA library.
 *
 * AN ASSUMED FORM.  The pages say only that the heads' combination is decided
 * dynamically from the current input (m.aitntnews.com blog post, section
 * "第二刀-砍层内", the DCMHA paragraph); they give no formula for c or g.  The
 * plainest reading taken here: per-token linear maps of the layer's input
 * hidden state x (the same input the layer's Q/K/V projection reads), with a
 * bias, and no nonlinearity (c is signed; g is whatever the map gives):
 *
 *   c[t,h] = b[h]     + sum_k x[t,k] * w[k][h]
 *   g[t,h] = b[H + h] + sum_k x[t,k] * w[k][H + h]          (k < D, h < H)
 *
 * and, for dL/dc = dc and dL/dg = dg, the gradients of those maps:
 *
 *   dx[t,k]     = sum_h dc[t,h] * w[k][h] + dg[t,h] * w[k][H + h]
 *   dw[k][h]    = sum_t x[t,k] * dc[t,h]      dw[k][H + h] = sum_t x[t,k] * dg[t,h]
 *   db[h]       = sum_t dc[t,h]               db[H + h]    = sum_t dg[t,h]
 *
 * Layouts: x, dx [N][D]; w, dw [D][2H]; b, db [2H]; c, g, dc, dg [N][H].
 * OpenMP only splits independent outputs across threads; every sum is taken in
 * the plain order written above.
 */
#include <stdint.h>

int dc_oracle_cg_fwd(int64_t N, int D, int H, const double *x, const double *w, const double *b, double *c,
                     double *g)
{
    if (N < 0 || D < 1 || H < 1 || !x || !w || !b || !c || !g) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t) {
        for (int h = 0; h < H; ++h) {
            double sc = b[h], sg = b[H + h];
            for (int k = 0; k < D; ++k) {
                sc += x[t * D + k] * w[(int64_t)k * 2 * H + h];
                sg += x[t * D + k] * w[(int64_t)k * 2 * H + H + h];
            }
            c[t * H + h] = sc;
            g[t * H + h] = sg;
        }
    }
    return 0;
}

int dc_oracle_cg_bwd(int64_t N, int D, int H, const double *x, const double *w, const double *dc,
                     const double *dg, double *dx, double *dw, double *db)
{
    if (N < 0 || D < 1 || H < 1 || !x || !w || !dc || !dg || !dx || !dw || !db) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t) {
        for (int k = 0; k < D; ++k) {
            double s = 0.0;
            for (int h = 0; h < H; ++h)
                s += dc[t * H + h] * w[(int64_t)k * 2 * H + h] + dg[t * H + h] * w[(int64_t)k * 2 * H + H + h];
            dx[t * D + k] = s;
        }
    }
#pragma omp parallel for schedule(static)
    for (int k = 0; k < D; ++k) {
        for (int h = 0; h < H; ++h) {
            double sc = 0.0, sg = 0.0;
            for (int64_t t = 0; t < N; ++t) {
                sc += x[t * D + k] * dc[t * H + h];
                sg += x[t * D + k] * dg[t * H + h];
            }
            dw[(int64_t)k * 2 * H + h] = sc;
            dw[(int64_t)k * 2 * H + H + h] = sg;
        }
    }
    for (int h = 0; h < H; ++h) {
        double sc = 0.0, sg = 0.0;
        for (int64_t t = 0; t < N; ++t) {
            sc += dc[t * H + h];
            sg += dg[t * H + h];
        }
        db[h] = sc;
        db[H + h] = sg;
    }
    return 0;
}
