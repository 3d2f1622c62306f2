/*
 * ss2d_oracle.c -- plain, slow, fp64 CPU oracle for the 2D selective scan (SS2D).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker the CUDA library is
 * compared against.  It shares no code, header, table or constant with the
 * CUDA path, and the product path never calls it.  Only the test suite, the
 * smoke check and the benchmark's CPU-baseline leg load it.
 *
 * What is computed, and where it is defined:
 *
 *  - CrossScan / CrossMerge: "VMamba: Visual State Space Model" (blog.csdn.net
 *    translation), section "2D Selective Scan (SS2D) for visual data" and the
 *    caption of Fig. 2: the input patches are unfolded along four traversal
 *    paths, each sequence is processed by its own S6 block, and the results
 *    are merged back into a 2D map by summation.  The four paths taken here
 *    are row-major (k=0), column-major (k=1) and their reverses (k=2, k=3).
 *
 *  - Selective scan (S6): "vision mamba-yolov8" (freeymw.com), section
 *    "2. Vmamba module code", function selective_scan_ref: delta gets the bias
 *    added and goes through softplus; the state is updated as
 *    h = exp(delta*A) * h + delta * B * u starting from h = 0; the output is
 *    y = sum_n C[n] * h[n] + D * u.  B and C carry G groups and channel c uses
 *    group c / (channels / G) (the repeat "B G N L -> B (G H) N L").
 *    When a gate z is given, the output is multiplied by silu(z) = z * sigmoid(z)
 *    after the D * u term is added (the last lines of selective_scan_ref), and
 *    the state after the last step can be returned (return_last_state).
 *
 *  - Backward: the same page gives only the signature of the CUDA backward
 *    (SelectiveScanFn.backward); the gradients here are the analytic
 *    derivatives of the forward recurrence above, written out step by step.
 *
 * Everything is double precision.  Loops follow the definitions in order;
 * OpenMP only distributes independent (batch, channel) sequences over host
 * threads, it never reorders the arithmetic of one sequence.
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#define K_PATHS 4

/* ---------------------------------------------------------------- paths -- */

/* Pixel index p = h*W + w visited at step l of path k (Fig. 2 of the VMamba
 * page: four traversal paths).  k=0 row-major, k=1 column-major
 * (l = w*H + h), k=2 / k=3 the same two orders walked backwards. */
long oracle_path_pixel(int k, long l, long H, long W)
{
    long L = H * W;
    long m = (k >= 2) ? (L - 1 - l) : l;
    long h, w;
    if (k % 2 == 0) {
        h = m / W;
        w = m % W;
    } else {
        h = m % H;
        w = m / H;
    }
    return h * W + w;
}

/* xs[b, k, d, l] = x[b, d, pixel(k, l)]   x: (B, D, H, W), xs: (B, 4, D, L) */
void oracle_cross_scan(long Bn, long Dn, long H, long W, const double *x, double *xs)
{
    long L = H * W;
    for (long b = 0; b < Bn; ++b)
        for (int k = 0; k < K_PATHS; ++k)
            for (long d = 0; d < Dn; ++d)
                for (long l = 0; l < L; ++l)
                    xs[((b * K_PATHS + k) * Dn + d) * L + l] =
                        x[(b * Dn + d) * L + oracle_path_pixel(k, l, H, W)];
}

/* y[b, d, p] = (t0[p] + t2[p]) + (t1[p] + t3[p]) where t_k[pixel(k, l)] = ys[b, k, d, l].
 * ys: (B, 4, D, L), y: (B, D, H, W). */
void oracle_cross_merge(long Bn, long Dn, long H, long W, const double *ys, double *y)
{
    long L = H * W;
    double *t = (double *)malloc(sizeof(double) * (size_t)(K_PATHS * L));
    for (long b = 0; b < Bn; ++b)
        for (long d = 0; d < Dn; ++d) {
            for (int k = 0; k < K_PATHS; ++k)
                for (long l = 0; l < L; ++l)
                    t[k * L + oracle_path_pixel(k, l, H, W)] = ys[((b * K_PATHS + k) * Dn + d) * L + l];
            for (long p = 0; p < L; ++p)
                y[(b * Dn + d) * L + p] = (t[0 * L + p] + t[2 * L + p]) + (t[1 * L + p] + t[3 * L + p]);
        }
    free(t);
}

/* ------------------------------------------------------- selective scan -- */

static double softplus_d(double t)
{
    /* log(1 + e^t) evaluated without overflow */
    return (t > 0.0 ? t : 0.0) + log1p(exp(-fabs(t)));
}

static double sigmoid_d(double t)
{
    return 1.0 / (1.0 + exp(-t));
}

/* silu(z) = z * sigmoid(z), the output gate of selective_scan_ref */
static double silu_d(double z)
{
    return z * sigmoid_d(z);
}

/* d silu / dz = sigmoid(z) * (1 + z * (1 - sigmoid(z))) */
static double silu_grad_d(double z)
{
    double s = sigmoid_d(z);
    return s * (1.0 + z * (1.0 - s));
}

/* delta + bias, then softplus when asked (selective_scan_ref, first lines). */
static double step_size(double delta, const double *bias, long c, int softplus, double *t_out)
{
    double t = delta + (bias ? bias[c] : 0.0);
    if (t_out) *t_out = t;
    return softplus ? softplus_d(t) : t;
}

/*
 * Forward S6 over Bn*Ch independent sequences of length L with N states.
 *   u, delta, out : (Bn, Ch, L)
 *   A             : (Ch, N)
 *   Bm, Cm        : (Bn, G, N, L), channel c uses group c / (Ch / G)
 *   Dv, bias      : (Ch) or NULL
 *   z             : (Bn, Ch, L) or NULL -- out = (y + D u) * silu(z)
 *   last_state    : (Bn, Ch, N) or NULL -- h after the last step
 */
void oracle_selective_scan_fwd(long Bn, long Ch, long L, long N, long G,
                               const double *u, const double *delta, const double *A,
                               const double *Bm, const double *Cm, const double *Dv,
                               const double *bias, int softplus, const double *z, double *out,
                               double *last_state)
{
    long per_group = Ch / G;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (long b = 0; b < Bn; ++b)
        for (long c = 0; c < Ch; ++c) {
            long g = c / per_group;
            double *h = (double *)calloc((size_t)N, sizeof(double));
            const double *uc = u + (b * Ch + c) * L;
            const double *dc = delta + (b * Ch + c) * L;
            const double *Bg = Bm + (b * G + g) * N * L;
            const double *Cg = Cm + (b * G + g) * N * L;
            for (long l = 0; l < L; ++l) {
                double dt = step_size(dc[l], bias, c, softplus, NULL);
                for (long n = 0; n < N; ++n)
                    h[n] = exp(dt * A[c * N + n]) * h[n] + dt * Bg[n * L + l] * uc[l];
                double y = 0.0;
                for (long n = 0; n < N; ++n)
                    y += Cg[n * L + l] * h[n];
                if (Dv) y += Dv[c] * uc[l];
                if (z) y *= silu_d(z[(b * Ch + c) * L + l]);
                out[(b * Ch + c) * L + l] = y;
            }
            if (last_state)
                for (long n = 0; n < N; ++n)
                    last_state[(b * Ch + c) * N + n] = h[n];
            free(h);
        }
}

/*
 * Backward S6: given dout = dLoss/dout, returns the gradients of every input.
 * du, ddelta: (Bn, Ch, L).  dA: (Ch, N).  dB, dC: (Bn, G, N, L) summed over the
 * channels of a group.  dD, dbias: (Ch), written only when D / bias are given.
 * Gradients are written (not accumulated into the caller's buffers).
 *
 * Per sequence: recompute h_l for all l, then walk l = L-1 .. 0 with the
 * adjoint lambda_n = dLoss/dh_{l,n}:
 *   lambda_n  = C[n,l] g_l + a_{l+1,n} lambda_{l+1,n}
 *   dC[n,l]  += g_l h_{l,n}
 *   ddt_l    += lambda_n (A[c,n] a_{l,n} h_{l-1,n} + B[n,l] u_l)
 *   dA[c,n]  += lambda_n dt_l a_{l,n} h_{l-1,n}
 *   dB[n,l]  += lambda_n dt_l u_l
 *   du_l     += lambda_n dt_l B[n,l]   (+ g_l D[c])
 *   ddelta_l  = ddt_l * sigmoid(t_l) under softplus, else ddt_l
 * With a gate z (out = o * silu(z), o = y + D u): g_l = dout_l * silu(z_l) is the
 * gradient reaching o, and dz_l = dout_l * o_l * silu'(z_l), o_l rebuilt from the
 * recomputed states.  dz: (Bn, Ch, L), written only when z is given.
 */
void oracle_selective_scan_bwd(long Bn, long Ch, long L, long N, long G,
                               const double *u, const double *delta, const double *A,
                               const double *Bm, const double *Cm, const double *Dv,
                               const double *bias, int softplus, const double *z,
                               const double *dout, double *du, double *ddelta, double *dA,
                               double *dB, double *dC, double *dD, double *dbias, double *dz)
{
    long per_group = Ch / G;
    /* per-batch partials of the parameter gradients, summed in fixed order below */
    double *pA = (double *)calloc((size_t)(Bn * Ch * N), sizeof(double));
    double *pD = (double *)calloc((size_t)(Bn * Ch), sizeof(double));
    double *pbias = (double *)calloc((size_t)(Bn * Ch), sizeof(double));
    memset(dB, 0, sizeof(double) * (size_t)(Bn * G * N * L));
    memset(dC, 0, sizeof(double) * (size_t)(Bn * G * N * L));

    /* channels of one batch item write the same dB/dC rows: one thread per batch item */
#pragma omp parallel for schedule(dynamic)
    for (long b = 0; b < Bn; ++b) {
        double *hist = (double *)malloc(sizeof(double) * (size_t)(L * N));
        double *lam = (double *)malloc(sizeof(double) * (size_t)N);
        double *hh = (double *)malloc(sizeof(double) * (size_t)N);
        for (long c = 0; c < Ch; ++c) {
            long g = c / per_group;
            const double *uc = u + (b * Ch + c) * L;
            const double *dc = delta + (b * Ch + c) * L;
            const double *Bg = Bm + (b * G + g) * N * L;
            const double *Cg = Cm + (b * G + g) * N * L;
            const double *gc = dout + (b * Ch + c) * L;
            double *dBg = dB + (b * G + g) * N * L;
            double *dCg = dC + (b * G + g) * N * L;

            /* forward recompute, keeping every state */
            for (long n = 0; n < N; ++n) hh[n] = 0.0;
            for (long l = 0; l < L; ++l) {
                double dt = step_size(dc[l], bias, c, softplus, NULL);
                for (long n = 0; n < N; ++n) {
                    hh[n] = exp(dt * A[c * N + n]) * hh[n] + dt * Bg[n * L + l] * uc[l];
                    hist[l * N + n] = hh[n];
                }
            }

            /* reverse adjoint walk */
            for (long n = 0; n < N; ++n) lam[n] = 0.0;
            for (long l = L - 1; l >= 0; --l) {
                double t;
                double dt = step_size(dc[l], bias, c, softplus, &t);
                double g_l = gc[l];
                if (z) {
                    double zl = z[(b * Ch + c) * L + l];
                    double o = Dv ? Dv[c] * uc[l] : 0.0;
                    for (long n = 0; n < N; ++n) o += Cg[n * L + l] * hist[l * N + n];
                    dz[(b * Ch + c) * L + l] = g_l * o * silu_grad_d(zl);
                    g_l *= silu_d(zl);
                }
                double dul = Dv ? g_l * Dv[c] : 0.0;
                double ddt = 0.0;
                if (Dv) pD[b * Ch + c] += g_l * uc[l];
                for (long n = 0; n < N; ++n) {
                    double a = exp(dt * A[c * N + n]);
                    double hp = (l > 0) ? hist[(l - 1) * N + n] : 0.0;
                    lam[n] += Cg[n * L + l] * g_l;
                    dCg[n * L + l] += g_l * hist[l * N + n];
                    ddt += lam[n] * (A[c * N + n] * a * hp + Bg[n * L + l] * uc[l]);
                    pA[(b * Ch + c) * N + n] += lam[n] * dt * a * hp;
                    dBg[n * L + l] += lam[n] * dt * uc[l];
                    dul += lam[n] * dt * Bg[n * L + l];
                    lam[n] *= a;
                }
                double dd = softplus ? ddt * sigmoid_d(t) : ddt;
                ddelta[(b * Ch + c) * L + l] = dd;
                pbias[b * Ch + c] += dd;
                du[(b * Ch + c) * L + l] = dul;
            }
        }
        free(hist);
        free(lam);
        free(hh);
    }

    for (long c = 0; c < Ch; ++c) {
        for (long n = 0; n < N; ++n) {
            double s = 0.0;
            for (long b = 0; b < Bn; ++b) s += pA[(b * Ch + c) * N + n];
            dA[c * N + n] = s;
        }
        if (dD) {
            double s = 0.0;
            for (long b = 0; b < Bn; ++b) s += pD[b * Ch + c];
            dD[c] = s;
        }
        if (dbias) {
            double s = 0.0;
            for (long b = 0; b < Bn; ++b) s += pbias[b * Ch + c];
            dbias[c] = s;
        }
    }
    free(pA);
    free(pD);
    free(pbias);
}

/* ------------------------------------------------------------ full SS2D -- */

/*
 * SS2D forward: CrossScan -> S6 on the 4*D sequences (group k for path k)
 * -> CrossMerge.  x, y: (B, D, H, W); delta: (B, 4D, L) in path order;
 * A: (4D, N); Bm, Cm: (B, 4, N, L); Dv, bias: (4D) or NULL.
 */
void oracle_ss2d_forward(long Bn, long Dn, long H, long W, long N,
                         const double *x, const double *delta, const double *A,
                         const double *Bm, const double *Cm, const double *Dv,
                         const double *bias, int softplus, double *y)
{
    long L = H * W;
    size_t seq = (size_t)(Bn * K_PATHS * Dn * L);
    double *xs = (double *)malloc(sizeof(double) * seq);
    double *ys = (double *)malloc(sizeof(double) * seq);
    oracle_cross_scan(Bn, Dn, H, W, x, xs);
    oracle_selective_scan_fwd(Bn, K_PATHS * Dn, L, N, K_PATHS, xs, delta, A, Bm, Cm, Dv, bias,
                              softplus, NULL, ys, NULL);
    oracle_cross_merge(Bn, Dn, H, W, ys, y);
    free(xs);
    free(ys);
}

/*
 * SS2D backward through the adjoints: the adjoint of CrossMerge (a sum of
 * four permutations) is CrossScan, and the adjoint of CrossScan is CrossMerge.
 *   g  = CrossScan(dy);  S6 backward on g;  dx = CrossMerge(du_seq).
 * dx: (B, D, H, W); other gradients as in oracle_selective_scan_bwd.
 */
void oracle_ss2d_backward(long Bn, long Dn, long H, long W, long N,
                          const double *x, const double *delta, const double *A,
                          const double *Bm, const double *Cm, const double *Dv,
                          const double *bias, int softplus, const double *dy,
                          double *dx, double *ddelta, double *dA, double *dB, double *dC,
                          double *dD, double *dbias)
{
    long L = H * W;
    size_t seq = (size_t)(Bn * K_PATHS * Dn * L);
    double *xs = (double *)malloc(sizeof(double) * seq);
    double *gs = (double *)malloc(sizeof(double) * seq);
    double *dus = (double *)malloc(sizeof(double) * seq);
    oracle_cross_scan(Bn, Dn, H, W, x, xs);
    oracle_cross_scan(Bn, Dn, H, W, dy, gs);
    oracle_selective_scan_bwd(Bn, K_PATHS * Dn, L, N, K_PATHS, xs, delta, A, Bm, Cm, Dv, bias,
                              softplus, NULL, gs, dus, ddelta, dA, dB, dC, dD, dbias, NULL);
    oracle_cross_merge(Bn, Dn, H, W, dus, dx);
    free(xs);
    free(gs);
    free(dus);
}

/* ---------------------------------------------------- path sets as data -- */

/*
 * The same three steps for any four paths given as a table: table[k * L + l]
 * is the pixel visited at step l of path k (each row a permutation of 0..L-1).
 * Row-major / column-major / reversed (the VMamba page's cross scan) is one
 * such table; the diagonal scans of "Visual Mamba实战从零开始搭建图像分类模型
 * 附PyTorch代码" (section 3, _get_diagonal_indices) give another.
 */
void oracle_cross_scan_table(long Bn, long Dn, long L, const long *table, const double *x, double *xs)
{
    for (long b = 0; b < Bn; ++b)
        for (int k = 0; k < K_PATHS; ++k)
            for (long d = 0; d < Dn; ++d)
                for (long l = 0; l < L; ++l)
                    xs[((b * K_PATHS + k) * Dn + d) * L + l] = x[(b * Dn + d) * L + table[k * L + l]];
}

/* y[b, d, p] = (t0[p] + t2[p]) + (t1[p] + t3[p]) where t_k[table[k][l]] = ys[b, k, d, l] */
void oracle_cross_merge_table(long Bn, long Dn, long L, const long *table, const double *ys, double *y)
{
    double *t = (double *)malloc(sizeof(double) * (size_t)(K_PATHS * L));
    for (long b = 0; b < Bn; ++b)
        for (long d = 0; d < Dn; ++d) {
            for (int k = 0; k < K_PATHS; ++k)
                for (long l = 0; l < L; ++l)
                    t[k * L + table[k * L + l]] = ys[((b * K_PATHS + k) * Dn + d) * L + l];
            for (long p = 0; p < L; ++p)
                y[(b * Dn + d) * L + p] = (t[0 * L + p] + t[2 * L + p]) + (t[1 * L + p] + t[3 * L + p]);
        }
    free(t);
}

void oracle_ss2d_forward_table(long Bn, long Dn, long L, long N, const long *table,
                               const double *x, const double *delta, const double *A,
                               const double *Bm, const double *Cm, const double *Dv,
                               const double *bias, int softplus, double *y)
{
    size_t seq = (size_t)(Bn * K_PATHS * Dn * L);
    double *xs = (double *)malloc(sizeof(double) * seq);
    double *ys = (double *)malloc(sizeof(double) * seq);
    oracle_cross_scan_table(Bn, Dn, L, table, x, xs);
    oracle_selective_scan_fwd(Bn, K_PATHS * Dn, L, N, K_PATHS, xs, delta, A, Bm, Cm, Dv, bias,
                              softplus, NULL, ys, NULL);
    oracle_cross_merge_table(Bn, Dn, L, table, ys, y);
    free(xs);
    free(ys);
}

void oracle_ss2d_backward_table(long Bn, long Dn, long L, long N, const long *table,
                                const double *x, const double *delta, const double *A,
                                const double *Bm, const double *Cm, const double *Dv,
                                const double *bias, int softplus, const double *dy,
                                double *dx, double *ddelta, double *dA, double *dB, double *dC,
                                double *dD, double *dbias)
{
    size_t seq = (size_t)(Bn * K_PATHS * Dn * L);
    double *xs = (double *)malloc(sizeof(double) * seq);
    double *gs = (double *)malloc(sizeof(double) * seq);
    double *dus = (double *)malloc(sizeof(double) * seq);
    oracle_cross_scan_table(Bn, Dn, L, table, x, xs);
    oracle_cross_scan_table(Bn, Dn, L, table, dy, gs);
    oracle_selective_scan_bwd(Bn, K_PATHS * Dn, L, N, K_PATHS, xs, delta, A, Bm, Cm, Dv, bias,
                              softplus, NULL, gs, dus, ddelta, dA, dB, dC, dD, dbias, NULL);
    oracle_cross_merge_table(Bn, Dn, L, table, dus, dx);
    free(xs);
    free(gs);
    free(dus);
}

/* number of host threads OpenMP will use (reported by the CPU baseline) */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
