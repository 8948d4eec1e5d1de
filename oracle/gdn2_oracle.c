/*
 * gdn2_oracle.c -- fp64 CPU reference for the Gated DeltaNet-2 recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path (the CUDA library and
 * its Python binding) may include, link or call this file.  Only the tests,
 * `__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py` use it.
 *
 * What it computes (burn-gdn2 README, section "Architecture", per-token
 * recurrence on the matrix state S in R^{d_k x d_v}):
 *
 *     S_t = (I - k_t (b_t . k_t)^T) diag(alpha_t) S_{t-1} + k_t (w_t . v_t)^T
 *     o_t = S_t^T q_t
 *
 * with alpha_t = exp(log_alpha_t) per key channel, b_t the erase gate on the
 * key axis and w_t the write gate on the value axis (same README section; the
 * asapai.co.kr GDN-2 article, section on splitting the gate, places the decay
 * per channel as in KDA).  Readings taken where the pages are silent:
 *   - o_t reads the post-update state S_t;
 *   - log_alpha is a natural log;
 *   - the decay diag(alpha_t) acts before the erase, in the order the
 *     equation is written;
 *   - no query scaling is applied (q and k arrive normalised).
 *
 * The code is the definition written out token by token.  The product
 * (I - k (b.k)^T) M is evaluated as M - k ((b.k)^T M); that is the same
 * matrix product regrouped, nothing more.  Every multiply-add is in double.
 *
 * Layouts (all contiguous, row-major):
 *   q, k, log_alpha, b : [B, T, H, d_k]   (float32 values, exact upcasts of
 *   v, w               : [B, T, H, d_v]    whatever the GPU received)
 *   S0                 : [B, H, d_k, d_v] double, may be NULL (zeros)
 * Outputs are compact per requested head:
 *   o   : [n_heads, T, d_v]   double
 *   S_T : [n_heads, d_k, d_v] double, may be NULL
 * `heads` lists flat head indices bh = b*H + h; NULL means all B*H heads in
 * order.  `smax` (nullable, one double per requested head) receives the
 * largest |S_t[i][j]| seen over the run, so state growth is visible.
 *
 * Returns 0 on success, -1 on bad arguments or allocation failure.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int run_head(const float *q, const float *k, const float *v,
                    const float *la, const float *b, const float *w,
                    const double *S0, double *o, double *S_T, double *smax,
                    long T, long H, long dk, long dv)
{
    double *S = (double *)malloc(sizeof(double) * (size_t)(dk * dv));
    double *r = (double *)malloc(sizeof(double) * (size_t)dv);
    double *u = (double *)malloc(sizeof(double) * (size_t)dv);
    if (!S || !r || !u) { free(S); free(r); free(u); return -1; }
    if (S0) memcpy(S, S0, sizeof(double) * (size_t)(dk * dv));
    else    memset(S, 0, sizeof(double) * (size_t)(dk * dv));
    double big = 0.0;
    const long sk = H * dk, sv = H * dv;   /* stride between tokens */
    for (long t = 0; t < T; ++t) {
        const float *qt = q + t * sk, *kt = k + t * sk, *lat = la + t * sk,
                    *bt = b + t * sk, *vt = v + t * sv, *wt = w + t * sv;
        /* diag(alpha_t) S_{t-1} */
        for (long i = 0; i < dk; ++i) {
            const double a = exp((double)lat[i]);
            double *row = S + i * dv;
            for (long j = 0; j < dv; ++j) row[j] *= a;
        }
        /* r = (b_t . k_t)^T (decayed S) */
        for (long j = 0; j < dv; ++j) r[j] = 0.0;
        for (long i = 0; i < dk; ++i) {
            const double bk = (double)bt[i] * (double)kt[i];
            const double *row = S + i * dv;
            for (long j = 0; j < dv; ++j) r[j] += bk * row[j];
        }
        /* u = w_t . v_t - r ;  S += k_t u^T */
        for (long j = 0; j < dv; ++j) u[j] = (double)wt[j] * (double)vt[j] - r[j];
        for (long i = 0; i < dk; ++i) {
            const double ki = (double)kt[i];
            double *row = S + i * dv;
            for (long j = 0; j < dv; ++j) {
                row[j] += ki * u[j];
                const double m = fabs(row[j]);
                if (m > big) big = m;
            }
        }
        /* o_t = S_t^T q_t */
        double *ot = o + t * dv;
        for (long j = 0; j < dv; ++j) ot[j] = 0.0;
        for (long i = 0; i < dk; ++i) {
            const double qi = (double)qt[i];
            const double *row = S + i * dv;
            for (long j = 0; j < dv; ++j) ot[j] += qi * row[j];
        }
    }
    if (S_T) memcpy(S_T, S, sizeof(double) * (size_t)(dk * dv));
    if (smax) *smax = big;
    free(S); free(r); free(u);
    return 0;
}

int gdn2_oracle_forward(const float *q, const float *k, const float *v,
                        const float *log_alpha, const float *b, const float *w,
                        const double *S0, double *o, double *S_T, double *smax,
                        int B, int T, int H, int d_k, int d_v,
                        const int *heads, int n_heads, int n_threads)
{
    if (!q || !k || !v || !log_alpha || !b || !w || !o) return -1;
    if (B <= 0 || T < 0 || H <= 0 || d_k <= 0 || d_v <= 0) return -1;
    const long nh = heads ? n_heads : (long)B * H;
    if (nh < 0) return -1;
    int bad = 0;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
#endif
    for (long n = 0; n < nh; ++n) {
        const long bh = heads ? heads[n] : n;
        if (bh < 0 || bh >= (long)B * H) { bad |= 1; continue; }
        const long bi = bh / H, hi = bh % H;
        const long tok0 = bi * (long)T * H + hi;      /* (b, t=0, h) row */
        const long off_k = tok0 * d_k, off_v = tok0 * d_v;
        bad |= run_head(q + off_k, k + off_k, v + off_v, log_alpha + off_k,
                        b + off_k, w + off_v,
                        S0 ? S0 + bh * (long)d_k * d_v : NULL,
                        o + n * (long)T * d_v,
                        S_T ? S_T + n * (long)d_k * d_v : NULL,
                        smax ? smax + n : NULL, T, H, d_k, d_v) != 0;
    }
    return bad ? -1 : 0;
}

int gdn2_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
