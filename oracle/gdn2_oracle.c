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
 *
 * gdn2_oracle_forward_ex adds the two steps around the recurrence that the
 * README's "Architecture" diagram draws next to it, each optional:
 *   input prep  (the "L2-Norm" after the projections; "Configuration",
 *                allow_neg_eigval "b x 2"):
 *       q = q_raw / sqrt(sum_i q_raw_i^2 + l2_eps), k likewise (over d_k;
 *           a zero vector with l2_eps = 0 stays zero),
 *       b = sigmoid(b_raw) (times 2 with allow_neg_eigval), w = sigmoid(w_raw);
 *   output epilogue ("Gated RMS Norm <- SiLU Gate"; "Configuration",
 *                norm_eps):
 *       y_j = o_j / sqrt(mean_j o_j^2 + norm_eps) * weight_j * silu(g_j),
 *       silu(x) = x / (1 + exp(-x)), per (token, head) over d_v.
 * Readings: the L2 epsilon (not on the pages) is an argument; the RMS norm
 * is taken per head over d_v with one weight vector [d_v] for all heads.
 *
 * gdn2_oracle_forward_qed adds the second erase direction of the "Query
 * Knows What to Forget" page (mlsanity 2608.13668, abstract: a direction
 * taken from the query, orthogonal to the key, that cancels what the old
 * state holds along the query).  The page gives no formula; the reading
 * taken here is the plainest one the abstract supports:
 *     r_t = q_t - ((q_t . k_t) / (k_t . k_t)) k_t      (q_t itself when k_t = 0)
 *     u_t = r_t / sqrt(r_t . r_t + qed_eps)           (u_t . k_t = 0)
 *     S_t = (I - k_t (b_t . k_t)^T - u_t (c_t . u_t)^T) diag(alpha_t) S_{t-1}
 *           + k_t (w_t . v_t)^T
 * with c_t in [0, 1] a second erase gate on the key axis, an input like b
 * (sigmoid of a logit under the input prep, never doubled).  The two erases
 * act together on the decayed state, as one rank-2 edit.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int prep;              /* q, k, b, w are raw: L2-normalise q, k; sigmoid b, w */
    int neg_eigval;        /* with prep: b = 2 sigmoid(b_raw) */
    double l2_eps;
    const float *gate;     /* NULL: no epilogue; else [B, T, H, d_v] */
    const double *weight;  /* [d_v] */
    double norm_eps;
    const float *qed_c;    /* NULL: no second erase; else [B, T, H, d_k] */
    double qed_eps;
} fuse_t;

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* q, k, b (d_k) and w (d_v) of one token as doubles, prepared if asked */
static void token_inputs(const float *qt, const float *kt, const float *bt, const float *wt,
                         double *qd, double *kd, double *bd, double *wd, long dk, long dv,
                         const fuse_t *f)
{
    for (long i = 0; i < dk; ++i) { qd[i] = qt[i]; kd[i] = kt[i]; bd[i] = bt[i]; }
    for (long j = 0; j < dv; ++j) wd[j] = wt[j];
    if (!f->prep) return;
    double sq = 0.0, sk = 0.0;
    for (long i = 0; i < dk; ++i) { sq += qd[i] * qd[i]; sk += kd[i] * kd[i]; }
    const double nq = sqrt(sq + f->l2_eps), nk = sqrt(sk + f->l2_eps);
    /* reading: a zero vector (with l2_eps = 0) normalises to the zero vector */
    const double iq = nq > 0.0 ? 1.0 / nq : 0.0, ik = nk > 0.0 ? 1.0 / nk : 0.0;
    for (long i = 0; i < dk; ++i) {
        qd[i] *= iq;
        kd[i] *= ik;
        bd[i] = (f->neg_eigval ? 2.0 : 1.0) * sigmoid(bd[i]);
    }
    for (long j = 0; j < dv; ++j) wd[j] = sigmoid(wd[j]);
}

static int run_head(const float *q, const float *k, const float *v,
                    const float *la, const float *b, const float *w, const float *g, const float *c,
                    const double *S0, double *o, double *S_T, double *smax,
                    long T, long H, long HV, long dk, long dv, const fuse_t *f)
{
    double *S = (double *)malloc(sizeof(double) * (size_t)(dk * dv));
    double *r = (double *)malloc(sizeof(double) * (size_t)dv);
    double *u = (double *)malloc(sizeof(double) * (size_t)dv);
    double *tk = (double *)malloc(sizeof(double) * (size_t)(5 * dk + 2 * dv));
    if (!S || !r || !u || !tk) { free(S); free(r); free(u); free(tk); return -1; }
    double *qd = tk, *kd = tk + dk, *bd = tk + 2 * dk, *wd = tk + 3 * dk;
    double *ud = tk + 3 * dk + dv, *cd = tk + 4 * dk + dv, *r2 = tk + 5 * dk + dv;
    if (S0) memcpy(S, S0, sizeof(double) * (size_t)(dk * dv));
    else    memset(S, 0, sizeof(double) * (size_t)(dk * dv));
    double big = 0.0;
    const long sk = H * dk, sv = HV * dv;   /* stride between tokens */
    for (long t = 0; t < T; ++t) {
        const float *lat = la + t * sk, *vt = v + t * sv;
        token_inputs(q + t * sk, k + t * sk, b + t * sk, w + t * sv, qd, kd, bd, wd, dk, dv, f);
        /* diag(alpha_t) S_{t-1} */
        for (long i = 0; i < dk; ++i) {
            const double a = exp((double)lat[i]);
            double *row = S + i * dv;
            for (long j = 0; j < dv; ++j) row[j] *= a;
        }
        /* r = (b_t . k_t)^T (decayed S) */
        for (long j = 0; j < dv; ++j) r[j] = 0.0;
        for (long i = 0; i < dk; ++i) {
            const double bk = bd[i] * kd[i];
            const double *row = S + i * dv;
            for (long j = 0; j < dv; ++j) r[j] += bk * row[j];
        }
        /* second erase: u_t from q_t orthogonal to k_t; r2 = (c_t . u_t)^T (decayed S) */
        if (c) {
            const float *ct = c + t * sk;
            double qk = 0.0, kk = 0.0, rr = 0.0;
            for (long i = 0; i < dk; ++i) { qk += qd[i] * kd[i]; kk += kd[i] * kd[i]; }
            const double coef = kk > 0.0 ? qk / kk : 0.0;
            for (long i = 0; i < dk; ++i) { ud[i] = qd[i] - coef * kd[i]; rr += ud[i] * ud[i]; }
            const double nr = sqrt(rr + f->qed_eps);
            const double inr = nr > 0.0 ? 1.0 / nr : 0.0;
            for (long i = 0; i < dk; ++i) {
                ud[i] *= inr;
                cd[i] = f->prep ? sigmoid((double)ct[i]) : (double)ct[i];
            }
            for (long j = 0; j < dv; ++j) r2[j] = 0.0;
            for (long i = 0; i < dk; ++i) {
                const double cu = cd[i] * ud[i];
                const double *row = S + i * dv;
                for (long j = 0; j < dv; ++j) r2[j] += cu * row[j];
            }
            for (long i = 0; i < dk; ++i) {   /* S -= u_t r2^T, before the key-directed edit */
                const double ui = ud[i];
                double *row = S + i * dv;
                for (long j = 0; j < dv; ++j) row[j] -= ui * r2[j];
            }
        }
        /* u = w_t . v_t - r ;  S += k_t u^T */
        for (long j = 0; j < dv; ++j) u[j] = wd[j] * (double)vt[j] - r[j];
        for (long i = 0; i < dk; ++i) {
            const double ki = kd[i];
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
            const double qi = qd[i];
            const double *row = S + i * dv;
            for (long j = 0; j < dv; ++j) ot[j] += qi * row[j];
        }
        /* y = RMSNorm(o_t) . weight . silu(g_t) */
        if (g) {
            const float *gt = g + t * sv;
            double ms = 0.0;
            for (long j = 0; j < dv; ++j) ms += ot[j] * ot[j];
            const double inv = 1.0 / sqrt(ms / (double)dv + f->norm_eps);
            for (long j = 0; j < dv; ++j) {
                const double gj = (double)gt[j];
                ot[j] = ot[j] * inv * f->weight[j] * (gj * sigmoid(gj));
            }
        }
    }
    if (S_T) memcpy(S_T, S, sizeof(double) * (size_t)(dk * dv));
    if (smax) *smax = big;
    free(S); free(r); free(u); free(tk);
    return 0;
}

/* One recurrence per (sequence, value head).  Sequence n covers tokens
 * [cu[n], cu[n+1]) of the packed token axis when cu is given (token tensors
 * are then [1, T, H or HV, d]); otherwise B sequences of T tokens.  Value head
 * hv (of HV = G H) reads key head hv / G for q, k, log_alpha and b. */
static int forward_impl(const float *q, const float *k, const float *v,
                        const float *log_alpha, const float *b, const float *w,
                        const double *S0, double *o, double *S_T, double *smax,
                        int B, int T, int H, int HV, int d_k, int d_v, const int *cu,
                        const int *heads, int n_heads, int n_threads, const fuse_t *f)
{
    if (!q || !k || !v || !log_alpha || !b || !w || !o) return -1;
    if (B <= 0 || T < 0 || H <= 0 || HV <= 0 || d_k <= 0 || d_v <= 0) return -1;
    if (HV % H != 0) return -1;
    if (f->gate && !f->weight) return -1;
    if (f->prep && !(f->l2_eps >= 0.0)) return -1;
    if (cu) {
        if (cu[0] != 0 || cu[B] != T) return -1;
        for (int n = 0; n < B; ++n)
            if (cu[n + 1] < cu[n]) return -1;
    }
    const long G = HV / H;
    const long nh = heads ? n_heads : (long)B * HV;
    if (nh < 0) return -1;
    /* output row offset of each requested head: sequences are concatenated */
    long *orow = (long *)malloc(sizeof(long) * (size_t)(nh > 0 ? nh : 1));
    if (!orow) return -1;
    long acc = 0;
    for (long n = 0; n < nh; ++n) {
        const long bh = heads ? heads[n] : n;
        const long bi = (bh >= 0 && bh < (long)B * HV) ? bh / HV : 0;
        orow[n] = acc;
        acc += cu ? (long)(cu[bi + 1] - cu[bi]) : (long)T;
    }
    int bad = 0;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
#endif
    for (long n = 0; n < nh; ++n) {
        const long bh = heads ? heads[n] : n;
        if (bh < 0 || bh >= (long)B * HV) { bad |= 1; continue; }
        const long bi = bh / HV, hv = bh % HV, hk = hv / G;
        const long t0 = cu ? (long)cu[bi] : bi * (long)T;   /* first token of the sequence */
        const long len = cu ? (long)(cu[bi + 1] - cu[bi]) : (long)T;
        const long off_k = (t0 * H + hk) * d_k, off_v = (t0 * HV + hv) * d_v;
        bad |= run_head(q + off_k, k + off_k, v + off_v, log_alpha + off_k,
                        b + off_k, w + off_v, f->gate ? f->gate + off_v : NULL,
                        f->qed_c ? f->qed_c + off_k : NULL,
                        S0 ? S0 + bh * (long)d_k * d_v : NULL,
                        o + orow[n] * d_v,
                        S_T ? S_T + n * (long)d_k * d_v : NULL,
                        smax ? smax + n : NULL, len, H, HV, d_k, d_v, f) != 0;
    }
    free(orow);
    return bad ? -1 : 0;
}

int gdn2_oracle_forward(const float *q, const float *k, const float *v,
                        const float *log_alpha, const float *b, const float *w,
                        const double *S0, double *o, double *S_T, double *smax,
                        int B, int T, int H, int d_k, int d_v,
                        const int *heads, int n_heads, int n_threads)
{
    const fuse_t f = {0, 0, 0.0, NULL, NULL, 0.0, NULL, 0.0};
    return forward_impl(q, k, v, log_alpha, b, w, S0, o, S_T, smax, B, T, H, H, d_k, d_v, NULL,
                        heads, n_heads, n_threads, &f);
}

/* prep: 0 = inputs as given, 1 = raw q, k, b, w (see the header), 3 = raw and
 * allow_neg_eigval.  gate (nullable) switches the output epilogue on; it needs
 * weight [d_v]. */
int gdn2_oracle_forward_ex(const float *q, const float *k, const float *v,
                           const float *log_alpha, const float *b, const float *w,
                           const double *S0, double *o, double *S_T, double *smax,
                           int B, int T, int H, int HV, int d_k, int d_v, const int *cu_seqlens,
                           const int *heads, int n_heads, int n_threads,
                           int prep, double l2_eps, const float *gate, const double *weight,
                           double norm_eps)
{
    if (prep != 0 && prep != 1 && prep != 3) return -1;
    const fuse_t f = {prep & 1, (prep >> 1) & 1, l2_eps, gate, weight, norm_eps, NULL, 0.0};
    return forward_impl(q, k, v, log_alpha, b, w, S0, o, S_T, smax, B, T, H, HV, d_k, d_v, cu_seqlens,
                        heads, n_heads, n_threads, &f);
}

/* The recurrence with the second, query-derived erase (see the header);
 * c is [B, T, H, d_k]; prep as for gdn2_oracle_forward_ex (c = sigmoid(c_raw)
 * under it).  Equal-length sequences, value heads = key heads, no epilogue. */
int gdn2_oracle_forward_qed(const float *q, const float *k, const float *v,
                            const float *log_alpha, const float *b, const float *c, const float *w,
                            const double *S0, double *o, double *S_T, double *smax,
                            int B, int T, int H, int d_k, int d_v,
                            const int *heads, int n_heads, int n_threads,
                            int prep, double l2_eps, double qed_eps)
{
    if (!c || !(qed_eps >= 0.0)) return -1;
    if (prep != 0 && prep != 1 && prep != 3) return -1;
    const fuse_t f = {prep & 1, (prep >> 1) & 1, l2_eps, NULL, NULL, 0.0, c, qed_eps};
    return forward_impl(q, k, v, log_alpha, b, w, S0, o, S_T, smax, B, T, H, H, d_k, d_v, NULL,
                        heads, n_heads, n_threads, &f);
}

int gdn2_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
