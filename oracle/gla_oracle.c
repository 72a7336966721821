/*
 * gla_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, sequential fp64 CPU statement of the key-only gated linear
 * attention (GLA) token mixer of "GTR: Gated Token Recurrence for Efficient
 * Dense Prediction" (arXiv 2609.26590), method section:
 *
 *   state recurrence   S_t = Diag(gamma_t) S_{t-1} + k_t^T v_t,  S_0 = 0
 *   readout            o_t = d_k^{-1/2} q_t S_t
 *   retention gate     gamma_t = sigma(a_t)^{1/tau}, tau = 16, elementwise;
 *                      each gate entry scales one row (one key channel) of S
 *   value-side decay   fixed to one (key-side decay only)
 *   output gate        u_t = SiLU(g_t) (.) RMSNorm(o_t)
 *   scan directions    left-to-right, right-to-left, top-to-bottom,
 *                      bottom-to-top over the 2-D patch grid; results are
 *                      written back in the original spatial order.
 *
 * Only tests/, the package's smoke() entry and bench.py's CPU-baseline and
 * reference legs may load this file's library.  It shares no code, header,
 * table or constant with the CUDA path.
 *
 * Readings taken where the page is silent:
 *  - o_t reads the state AFTER token t has been added (inclusive).
 *  - d_k^{-1/2} multiplies o_t before the RMSNorm (where the equation puts it).
 *  - RMSNorm over the d_v entries of one head: o / sqrt(mean(o^2) + eps) * w,
 *    w a per-channel weight of length d_v shared by all heads, no bias.
 *  - Scan directions run along their axis, lines visited in increasing order,
 *    the state carrying over from one line's end to the next line's start:
 *      dir 0 L->R: y = p / W, x = p % W
 *      dir 1 R->L: y = p / W, x = W-1 - p % W
 *      dir 2 T->B: x = p / H, y = p % H
 *      dir 3 B->T: x = p / H, y = H-1 - p % H
 *    spatial index s = y*W + x (row-major grid).  dir 4 means dir = b % 4.
 *  - gamma is evaluated in log space: log gamma = log sigma(a) / tau.
 *
 * Layouts (all contiguous): q, k, a: [B][L][H][d_k]; v, g, out: [B][L][H][d_v];
 * w: [d_v].  L = grid_h * grid_w.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* scan position p -> spatial row-major index, for one of the four directions */
static long oracle_spatial(int dir, long p, long gh, long gw)
{
    long x, y;
    switch (dir) {
    case 0: y = p / gw; x = p % gw; break;
    case 1: y = p / gw; x = gw - 1 - p % gw; break;
    case 2: x = p / gh; y = p % gh; break;
    default: x = p / gh; y = gh - 1 - p % gh; break;
    }
    return y * gw + x;
}

/* log(sigma(a)) without overflow for either sign of a */
static double oracle_log_sigmoid(double a)
{
    if (a >= 0.0) return -log1p(exp(-a));
    return a - log1p(exp(a));
}

/*
 * Returns 0 on success, -1 on bad arguments, -2 on allocation failure.
 * o_raw (optional, may be NULL) receives o_t before the output gate, in the
 * same layout as out.
 */
int gla_oracle_fwd(const double *q, const double *k, const double *v,
                   const double *a, const double *g, const double *w,
                   double *out, double *o_raw,
                   int B, int H, int grid_h, int grid_w, int d_k, int d_v,
                   int direction, double eps, double tau, int nthreads)
{
    if (!q || !k || !v || !a || !g || !w || !out) return -1;
    if (B <= 0 || H <= 0 || grid_h <= 0 || grid_w <= 0 || d_k <= 0 || d_v <= 0) return -1;
    if (direction < 0 || direction > 4 || tau <= 0.0) return -1;

    const long L = (long)grid_h * grid_w;
    const long n_pairs = (long)B * H;
    const double scale = 1.0 / sqrt((double)d_k);
    int failed = 0;

#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)d_k * d_v);
        double *gam = (double *)malloc(sizeof(double) * (size_t)d_k);
        double *o = (double *)malloc(sizeof(double) * (size_t)d_v);
        const int ok = S && gam && o;
        if (!ok) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            failed = 1;
        }
        {
            /* every thread reaches the work-sharing loop, allocated or not */
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
            for (long pair = 0; pair < n_pairs; ++pair) {
                if (!ok) continue;
                const long b = pair / H, h = pair % H;
                const int dir = direction == 4 ? (int)(b % 4) : direction;
                memset(S, 0, sizeof(double) * (size_t)d_k * d_v);
                for (long p = 0; p < L; ++p) {
                    const long s = oracle_spatial(dir, p, grid_h, grid_w);
                    const long rk = ((b * L + s) * H + h) * (long)d_k; /* row in q,k,a */
                    const long rv = ((b * L + s) * H + h) * (long)d_v; /* row in v,g,out */
                    /* gamma_t = sigma(a_t)^(1/tau), one entry per key channel */
                    for (int c = 0; c < d_k; ++c)
                        gam[c] = exp(oracle_log_sigmoid(a[rk + c]) / tau);
                    /* S_t = Diag(gamma_t) S_{t-1} + k_t^T v_t */
                    for (int c = 0; c < d_k; ++c) {
                        const double kc = k[rk + c];
                        double *Sc = S + (size_t)c * d_v;
                        for (int j = 0; j < d_v; ++j)
                            Sc[j] = gam[c] * Sc[j] + kc * v[rv + j];
                    }
                    /* o_t = d_k^{-1/2} q_t S_t */
                    for (int j = 0; j < d_v; ++j) o[j] = 0.0;
                    for (int c = 0; c < d_k; ++c) {
                        const double qc = q[rk + c];
                        const double *Sc = S + (size_t)c * d_v;
                        for (int j = 0; j < d_v; ++j) o[j] += qc * Sc[j];
                    }
                    for (int j = 0; j < d_v; ++j) o[j] *= scale;
                    /* u_t = SiLU(g_t) * RMSNorm(o_t) */
                    double ms = 0.0;
                    for (int j = 0; j < d_v; ++j) ms += o[j] * o[j];
                    ms /= (double)d_v;
                    const double inv_rms = 1.0 / sqrt(ms + eps);
                    for (int j = 0; j < d_v; ++j) {
                        const double gj = g[rv + j];
                        const double silu = gj / (1.0 + exp(-gj));
                        out[rv + j] = o[j] * inv_rms * w[j] * silu;
                        if (o_raw) o_raw[rv + j] = o[j];
                    }
                }
            }
        }
        free(S);
        free(gam);
        free(o);
    }
    return failed ? -2 : 0;
}

/* exported so tests can pin the direction map on its own */
long gla_oracle_spatial_index(int dir, long p, long grid_h, long grid_w)
{
    return oracle_spatial(dir, p, grid_h, grid_w);
}
