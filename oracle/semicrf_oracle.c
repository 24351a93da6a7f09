/*
 * semicrf_oracle.c -- plain float64 CPU semi-CRF.  TEST INFRASTRUCTURE ONLY.
 *
 * This file is the checker for the CUDA path, not part of it.  Only the test
 * suite, the smoke check and the benchmark's CPU-baseline leg may load it.  It
 * shares no code, header, table or helper with the CUDA library.
 *
 * Model (Streaming Structured Inference with Flash-SemiCRF, abstract; technical
 * summary (gist.science) section 1): a segmentation of positions [0, L) is a list
 * of segments (s_i, d_i, c_i) with s_1 = 0, s_{i+1} = s_i + d_i, s_n + d_n = L,
 * 1 <= d_i <= K.  Its score is
 *     sum_i [ sum_{u=s_i}^{s_i+d_i-1} (x[u,c_i] - nu[c_i]) + D[d_i-1,c_i] ]
 *   + sum_{i>=2} A[c_{i-1}, c_i]
 * with nu[c] the per-sequence, per-label emission baseline (technical summary
 * section 2.C: the baseline is subtracted before the prefix sums; read here as
 * the mean of x[., c] over the valid positions).  log Z = log sum_y exp score(y).
 * The first segment takes no transition term; there are no start/end scores.
 *
 * Tiers (each a separate function; none calls another's arithmetic):
 *   oracle_prefix       centring baseline nu and prefix sums S (section 2.A/2.C)
 *   oracle_factorised   the forward/backward recursions over S in log space,
 *                       log Z, exact gradients and coverage marginals
 *   oracle_edge_direct  textbook semi-CRF over edge potentials
 *                       psi(s,d,c',c) = content(s,d,c) + D + A, content by a
 *                       direct inner sum (no prefix sums), small sizes only
 *   oracle_viterbi      the factorised recursion in (max,+), float64, with the
 *                       tie-break: smallest d, then smallest previous label,
 *                       final label smallest
 *
 * Precision: float64 throughout; log-sum-exp is two-pass (max, then sum of
 * exp).  Inputs are float64 (float32 data widens exactly).  The forward and
 * backward messages are kept relative to a per-position integer offset (an
 * exact float64 integer, the running sum of the integer parts of each
 * position's largest message), the checkpoint normalisation of technical
 * summary 2.C taken at every position: the stored values stay O(1) instead of
 * growing like log Z (~10^6 on the longest workloads, where an ulp is ~2e-10
 * and the plain sums drift by ~1e-8 over 10^5 positions), and the marginals
 * combine the offsets as exact integers.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define IDX2(i, j, n2) ((size_t)(i) * (size_t)(n2) + (size_t)(j))

static double lse(const double *v, int n)
{
    double m = -INFINITY;
    for (int i = 0; i < n; ++i)
        if (v[i] > m) m = v[i];
    if (m == -INFINITY) return -INFINITY;
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += exp(v[i] - m);
    return m + log(s);
}

static int max_threads(int requested)
{
#ifdef _OPENMP
    return requested > 0 ? requested : omp_get_max_threads();
#else
    (void)requested;
    return 1;
#endif
}

/* ---------------------------------------------------------------------------
 * Centring and prefix sums (technical summary 2.A and 2.C).
 *   nu[b,c]      = (1/L_b) sum_{t<L_b} x[b,t,c]            (0 when centre == 0)
 *   S[b,0,c]     = 0
 *   S[b,t+1,c]   = S[b,t,c] + (x[b,t,c] - nu[b,c])           for t < L_b
 *   S[b,t,c]     = S[b,L_b,c]                                for t > L_b
 * Sequential float64 sums in t.
 * ------------------------------------------------------------------------- */
int oracle_prefix(int B, int T, int C, const double *x, const int32_t *lengths,
                  int centre, double *S, double *nu)
{
    for (int b = 0; b < B; ++b) {
        int L = lengths[b];
        if (L < 1 || L > T) return 1;
        const double *xb = x + (size_t)b * T * C;
        double *Sb = S + (size_t)b * (T + 1) * C;
        for (int c = 0; c < C; ++c) {
            double m = 0.0;
            if (centre) {
                double acc = 0.0;
                for (int t = 0; t < L; ++t) acc += xb[IDX2(t, c, C)];
                m = acc / (double)L;
            }
            nu[IDX2(b, c, C)] = m;
            Sb[c] = 0.0;
            for (int t = 0; t < L; ++t)
                Sb[IDX2(t + 1, c, C)] = Sb[IDX2(t, c, C)] + (xb[IDX2(t, c, C)] - m);
            for (int t = L + 1; t <= T; ++t) Sb[IDX2(t, c, C)] = Sb[IDX2(L, c, C)];
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Factorised forward/backward for one sequence (length L), log space.
 *
 *   at[0,c] = 0                                   (alpha-tilde: a segment with
 *                                                  label c may start at s)
 *   al[t,c] = lse_{d=1..min(K,t)} ( at[t-d,c] + S[t,c] - S[t-d,c] + D[d-1,c] )
 *   at[t,c] = lse_{c'} ( al[t,c'] + A[c',c] )       1 <= t < L
 *   logZ    = lse_c al[L,c]
 *
 *   be[L,c] = 0
 *   ga[s,c] = lse_{d=1..min(K,L-s)} ( S[s+d,c] - S[s,c] + D[d-1,c] + be[s+d,c] )
 *   be[s,c']= lse_c ( A[c',c] + ga[s,c] )          1 <= s < L
 *   logZ_bwd= lse_c ga[0,c]
 *
 * Marginals (exact gradients of log Z, abstract: "preserving exact gradients"):
 *   Pseg(s,d,c)  = exp( at[s,c] + S[s+d,c] - S[s,c] + D[d-1,c] + be[s+d,c] - logZ )
 *   Ptr(s,c',c)  = exp( al[s,c'] + A[c',c] + ga[s,c] - logZ )      1 <= s < L
 *   dlogZ/dD[d-1,c] = sum_s Pseg(s,d,c);  dlogZ/dA[c',c] = sum_s Ptr(s,c',c)
 *   mu[u,c] = P(position u lies in a segment labelled c)
 *           = sum_{s<=u} sum_d Pseg(s,d,c) - sum_{s+d<=u} Pseg(s,d,c)
 *   dlogZ/dx[u,c] = mu[u,c] - (1/L) sum_{u'<L} mu[u',c]   (the second term is the
 *                   path through nu; dropped when nu is detached or not used)
 *   pstart[s] = P(a segment begins at s) = sum_c sum_d Pseg(s,d,c)   (abstract:
 *               uncertainty estimates at segment boundaries)
 * ------------------------------------------------------------------------- */
static void seq_factorised(int L, int T, int K, int C, const double *S,
                           const double *Ad, const double *Dd, int par,
                           double *logZ_out, double *logZ_bwd_out,
                           double *mu /* [T*C] */, double *pstart /* [T] or NULL */,
                           double *dA_b, double *dD_b)
{
    size_t n = (size_t)(L + 1) * C;
    double *al = calloc(n, sizeof(double));
    double *at = calloc(n, sizeof(double));
    double *be = calloc(n, sizeof(double));
    double *ga = calloc(n, sizeof(double));
    double *st = calloc(n, sizeof(double));   /* P(segment with label c starts at s) */
    double *en = calloc(n, sizeof(double));   /* P(segment with label c ends at t)   */
    /* integer offsets: al[t], at[t] hold the messages minus F[t]; ga[s], be[s]
     * hold them minus Bk[s] (F, Bk exact integers) */
    double *F = calloc((size_t)L + 1, sizeof(double));
    double *Bk = calloc((size_t)L + 1, sizeof(double));
    int nt = K > C ? K : C;

    /* forward */
    for (int c = 0; c < C; ++c) at[IDX2(0, c, C)] = 0.0;
    for (int t = 1; t <= L; ++t) {
        int dmax = t < K ? t : K;
#pragma omp parallel for if (par) schedule(static)
        for (int c = 0; c < C; ++c) {
            double tmp[nt];
            for (int d = 1; d <= dmax; ++d)
                tmp[d - 1] = at[IDX2(t - d, c, C)] + (F[t - d] - F[t - 1]) +
                             (S[IDX2(t, c, C)] - S[IDX2(t - d, c, C)]) + Dd[IDX2(d - 1, c, C)];
            al[IDX2(t, c, C)] = lse(tmp, dmax);   /* relative to F[t-1] */
        }
        double m = -INFINITY;
        for (int c = 0; c < C; ++c)
            if (al[IDX2(t, c, C)] > m) m = al[IDX2(t, c, C)];
        const double o = floor(m);
        F[t] = F[t - 1] + o;
        for (int c = 0; c < C; ++c) al[IDX2(t, c, C)] -= o;
        if (t < L) {
#pragma omp parallel for if (par) schedule(static)
            for (int c = 0; c < C; ++c) {
                double tmp[nt];
                for (int cp = 0; cp < C; ++cp) tmp[cp] = al[IDX2(t, cp, C)] + Ad[IDX2(cp, c, C)];
                at[IDX2(t, c, C)] = lse(tmp, C);
            }
        }
    }
    const double zf = lse(&al[IDX2(L, 0, C)], C);   /* log Z = F[L] + zf */
    double logZ = F[L] + zf;

    /* backward */
    for (int c = 0; c < C; ++c) be[IDX2(L, c, C)] = 0.0;
    for (int s = L - 1; s >= 0; --s) {
        int dmax = (L - s) < K ? (L - s) : K;
#pragma omp parallel for if (par) schedule(static)
        for (int c = 0; c < C; ++c) {
            double tmp[nt];
            for (int d = 1; d <= dmax; ++d)
                tmp[d - 1] = (S[IDX2(s + d, c, C)] - S[IDX2(s, c, C)]) + Dd[IDX2(d - 1, c, C)] +
                             be[IDX2(s + d, c, C)] + (Bk[s + d] - Bk[s + 1]);
            ga[IDX2(s, c, C)] = lse(tmp, dmax);   /* relative to Bk[s+1] */
        }
        double m = -INFINITY;
        for (int c = 0; c < C; ++c)
            if (ga[IDX2(s, c, C)] > m) m = ga[IDX2(s, c, C)];
        const double o = floor(m);
        Bk[s] = Bk[s + 1] + o;
        for (int c = 0; c < C; ++c) ga[IDX2(s, c, C)] -= o;
        if (s >= 1) {
#pragma omp parallel for if (par) schedule(static)
            for (int cp = 0; cp < C; ++cp) {
                double tmp[nt];
                for (int c = 0; c < C; ++c) tmp[c] = Ad[IDX2(cp, c, C)] + ga[IDX2(s, c, C)];
                be[IDX2(s, cp, C)] = lse(tmp, C);
            }
        }
    }
    double logZ_bwd = Bk[0] + lse(&ga[IDX2(0, 0, C)], C);

    /* segment marginals -> dD, start/end probabilities (parallel over labels);
     * exponents: the O(1) parts minus zf, plus the exact integer offsets */
#pragma omp parallel for if (par) schedule(static)
    for (int c = 0; c < C; ++c) {
        for (int s = 0; s < L; ++s) {
            int dmax = (L - s) < K ? (L - s) : K;
            for (int d = 1; d <= dmax; ++d) {
                double P = exp((at[IDX2(s, c, C)] + (S[IDX2(s + d, c, C)] - S[IDX2(s, c, C)]) +
                                Dd[IDX2(d - 1, c, C)] + be[IDX2(s + d, c, C)] - zf) +
                               ((F[s] - F[L]) + Bk[s + d]));
                dD_b[IDX2(d - 1, c, C)] += P;
                st[IDX2(s, c, C)] += P;
                en[IDX2(s + d, c, C)] += P;
            }
        }
    }
    /* transition marginals -> dA (parallel over the previous label) */
#pragma omp parallel for if (par) schedule(static)
    for (int cp = 0; cp < C; ++cp) {
        for (int s = 1; s < L; ++s)
            for (int c = 0; c < C; ++c)
                dA_b[IDX2(cp, c, C)] += exp((al[IDX2(s, cp, C)] + Ad[IDX2(cp, c, C)] + ga[IDX2(s, c, C)] - zf) +
                                            ((F[s] - F[L]) + Bk[s]));
    }
    /* coverage: segments started at or before u minus segments ended at or before u */
    for (int c = 0; c < C; ++c) {
        double started = 0.0, ended = 0.0;
        for (int u = 0; u < L; ++u) {
            started += st[IDX2(u, c, C)];
            ended += en[IDX2(u, c, C)];
            mu[IDX2(u, c, C)] = started - ended;
        }
        for (int u = L; u < T; ++u) mu[IDX2(u, c, C)] = 0.0;
    }
    if (pstart) {
        for (int s = 0; s < T; ++s) {
            double p = 0.0;
            if (s < L)
                for (int c = 0; c < C; ++c) p += st[IDX2(s, c, C)];
            pstart[s] = p;
        }
    }
    *logZ_out = logZ;
    *logZ_bwd_out = logZ_bwd;
    free(al); free(at); free(be); free(ga); free(st); free(en); free(F); free(Bk);
}


/* dX from coverage marginals (see seq_factorised) */
static void finish_dx(int L, int T, int C, int use_nu_path, double g, const double *mu, double *dXb)
{
    for (int c = 0; c < C; ++c) {
        double mean = 0.0;
        if (use_nu_path) {
            for (int u = 0; u < L; ++u) mean += mu[IDX2(u, c, C)];
            mean /= (double)L;
        }
        for (int u = 0; u < L; ++u) dXb[IDX2(u, c, C)] = g * (mu[IDX2(u, c, C)] - mean);
        for (int u = L; u < T; ++u) dXb[IDX2(u, c, C)] = 0.0;
    }
}

/*
 * Factorised oracle over a batch.  Outputs: logZ[B], logZ_bwd[B], dX[B,T,C],
 * dA[C,C], dD[K,C] (all float64), optional mu[B,T,C] and pstart[B,T].  grad_logZ may be NULL
 * (weights 1).  centre: subtract nu; detach_nu: drop the gradient path through nu.
 * Returns 0, or 1 on an invalid length.
 */
int oracle_factorised(int B, int T, int K, int C, const double *x, const double *A,
                      const double *D, const int32_t *lengths, int centre, int detach_nu,
                      const double *grad_logZ, double *logZ, double *logZ_bwd, double *dX,
                      double *dA, double *dD, double *mu_out, double *pstart_out, int nthreads)
{
    for (int b = 0; b < B; ++b)
        if (lengths[b] < 1 || lengths[b] > T) return 1;
    int nth = max_threads(nthreads);
    double *S = malloc(sizeof(double) * (size_t)B * (T + 1) * C);
    double *nu = malloc(sizeof(double) * (size_t)B * C);
    const double *Ad = A, *Dd = D;
    double *dA_all = calloc((size_t)B * C * C, sizeof(double));
    double *dD_all = calloc((size_t)B * K * C, sizeof(double));
    oracle_prefix(B, T, C, x, lengths, centre, S, nu);

    int outer = B >= nth || nth == 1;
#ifdef _OPENMP
    omp_set_num_threads(nth);
#endif
#pragma omp parallel for if (outer) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        double *mu = malloc(sizeof(double) * (size_t)T * C);
        double g = grad_logZ ? grad_logZ[b] : 1.0;
        seq_factorised(lengths[b], T, K, C, S + (size_t)b * (T + 1) * C, Ad, Dd, !outer,
                       &logZ[b], &logZ_bwd[b], mu, pstart_out ? pstart_out + (size_t)b * T : NULL,
                       dA_all + (size_t)b * C * C, dD_all + (size_t)b * K * C);
        finish_dx(lengths[b], T, C, centre && !detach_nu, g, mu, dX + (size_t)b * T * C);
        if (mu_out) memcpy(mu_out + (size_t)b * T * C, mu, sizeof(double) * (size_t)T * C);
        free(mu);
    }
    /* sum the per-sequence parameter gradients in sequence order */
    memset(dA, 0, sizeof(double) * (size_t)C * C);
    memset(dD, 0, sizeof(double) * (size_t)K * C);
    for (int b = 0; b < B; ++b) {
        double g = grad_logZ ? grad_logZ[b] : 1.0;
        for (size_t i = 0; i < (size_t)C * C; ++i) dA[i] += g * dA_all[(size_t)b * C * C + i];
        for (size_t i = 0; i < (size_t)K * C; ++i) dD[i] += g * dD_all[(size_t)b * K * C + i];
    }
    free(S); free(nu); free(dA_all); free(dD_all);
    return 0;
}

/*
 * Forward only (log Z), same recursion as seq_factorised; used for timing
 * bounded samples and for finite differences.
 */
int oracle_logz(int B, int T, int K, int C, const double *x, const double *A, const double *D,
                const int32_t *lengths, int centre, double *logZ, int nthreads)
{
    for (int b = 0; b < B; ++b)
        if (lengths[b] < 1 || lengths[b] > T) return 1;
    int nth = max_threads(nthreads);
    double *S = malloc(sizeof(double) * (size_t)B * (T + 1) * C);
    double *nu = malloc(sizeof(double) * (size_t)B * C);
    const double *Ad = A, *Dd = D;
    oracle_prefix(B, T, C, x, lengths, centre, S, nu);
    int outer = B >= nth || nth == 1;
    int nt = K > C ? K : C;
#ifdef _OPENMP
    omp_set_num_threads(nth);
#endif
#pragma omp parallel for if (outer) schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        int L = lengths[b];
        const double *Sb = S + (size_t)b * (T + 1) * C;
        double *al = calloc((size_t)(L + 1) * C, sizeof(double));
        double *at = calloc((size_t)(L + 1) * C, sizeof(double));
        double *F = calloc((size_t)L + 1, sizeof(double));   /* integer offsets, as in seq_factorised */
        for (int t = 1; t <= L; ++t) {
            int dmax = t < K ? t : K;
#pragma omp parallel for if (!outer) schedule(static)
            for (int c = 0; c < C; ++c) {
                double tmp[nt];
                for (int d = 1; d <= dmax; ++d)
                    tmp[d - 1] = at[IDX2(t - d, c, C)] + (F[t - d] - F[t - 1]) +
                                 (Sb[IDX2(t, c, C)] - Sb[IDX2(t - d, c, C)]) + Dd[IDX2(d - 1, c, C)];
                al[IDX2(t, c, C)] = lse(tmp, dmax);
            }
            double m = -INFINITY;
            for (int c = 0; c < C; ++c)
                if (al[IDX2(t, c, C)] > m) m = al[IDX2(t, c, C)];
            const double o = floor(m);
            F[t] = F[t - 1] + o;
            for (int c = 0; c < C; ++c) al[IDX2(t, c, C)] -= o;
            if (t < L) {
#pragma omp parallel for if (!outer) schedule(static)
                for (int c = 0; c < C; ++c) {
                    double tmp[nt];
                    for (int cp = 0; cp < C; ++cp) tmp[cp] = al[IDX2(t, cp, C)] + Ad[IDX2(cp, c, C)];
                    at[IDX2(t, c, C)] = lse(tmp, C);
                }
            }
        }
        logZ[b] = F[L] + lse(&al[IDX2(L, 0, C)], C);
        free(al); free(at); free(F);
    }
    free(S); free(nu);
    return 0;
}

/* ---------------------------------------------------------------------------
 * Edge-direct tier: the textbook semi-CRF over explicit edge potentials.
 *   content(s,d,c) = sum_{u=s}^{s+d-1} (x[u,c] - nu[c])      (direct inner sum)
 *   psi(s,d,c',c)  = content(s,d,c) + D[d-1,c] + A[c',c]      (s >= 1)
 *   psi0(d,c)      = content(0,d,c) + D[d-1,c]                (first segment)
 *   a[t,c]  = log-sum over prefixes of [0,t) whose last segment has label c
 *           = lse over d, and c' when t-d >= 1, of a[t-d,c'] + psi(t-d,d,c',c);
 *             for t-d == 0 the term is psi0(d,c)
 *   b[t,c'] = log-sum over suffixes [t,L) given the segment ending at t has c'
 *           = lse over d, c of psi(t,d,c',c) + b[t+d,c];   b[L,.] = 0
 *   P(s,d,c',c) = exp(a[s,c'] + psi(s,d,c',c) + b[s+d,c] - logZ)
 * Gradients are sums of these edge marginals; coverage loops over u directly.
 * ------------------------------------------------------------------------- */
static void seq_edge_direct(int L, int T, int K, int C, const double *xb, const double *nub,
                            const double *Ad, const double *Dd, double *logZ_out,
                            double *mu /* [T*C] */, double *dA_b, double *dD_b)
{
    /* content[s][d-1][c] */
    double *content = calloc((size_t)L * K * C, sizeof(double));
    for (int s = 0; s < L; ++s)
        for (int d = 1; d <= K && s + d <= L; ++d)
            for (int c = 0; c < C; ++c) {
                double acc = 0.0;
                for (int u = s; u < s + d; ++u) acc += (xb[IDX2(u, c, C)] - nub[c]);
                content[((size_t)s * K + (d - 1)) * C + c] = acc;
            }
#define CONTENT(s, d, c) content[((size_t)(s) * K + ((d) - 1)) * C + (c)]
    size_t n = (size_t)(L + 1) * C;
    double *a = malloc(sizeof(double) * n);
    double *bb = malloc(sizeof(double) * n);
    int ntmp = K * C + 1;
    double *tmp = malloc(sizeof(double) * ntmp);
    for (int c = 0; c < C; ++c) a[IDX2(0, c, C)] = -INFINITY;
    for (int t = 1; t <= L; ++t)
        for (int c = 0; c < C; ++c) {
            int m = 0;
            for (int d = 1; d <= K && d <= t; ++d) {
                int s = t - d;
                if (s == 0) {
                    tmp[m++] = CONTENT(0, d, c) + Dd[IDX2(d - 1, c, C)];
                } else {
                    for (int cp = 0; cp < C; ++cp)
                        tmp[m++] = a[IDX2(s, cp, C)] + CONTENT(s, d, c) + Dd[IDX2(d - 1, c, C)] +
                                   Ad[IDX2(cp, c, C)];
                }
            }
            a[IDX2(t, c, C)] = lse(tmp, m);
        }
    double logZ = lse(&a[IDX2(L, 0, C)], C);
    for (int c = 0; c < C; ++c) bb[IDX2(L, c, C)] = 0.0;
    for (int t = L - 1; t >= 1; --t)
        for (int cp = 0; cp < C; ++cp) {
            int m = 0;
            for (int d = 1; d <= K && t + d <= L; ++d)
                for (int c = 0; c < C; ++c)
                    tmp[m++] = CONTENT(t, d, c) + Dd[IDX2(d - 1, c, C)] + Ad[IDX2(cp, c, C)] +
                               bb[IDX2(t + d, c, C)];
            bb[IDX2(t, cp, C)] = lse(tmp, m);
        }
    for (size_t i = 0; i < (size_t)T * C; ++i) mu[i] = 0.0;
    for (int s = 0; s < L; ++s)
        for (int d = 1; d <= K && s + d <= L; ++d)
            for (int c = 0; c < C; ++c) {
                double Pc = 0.0;
                if (s == 0) {
                    Pc = exp(CONTENT(0, d, c) + Dd[IDX2(d - 1, c, C)] + bb[IDX2(d, c, C)] - logZ);
                } else {
                    for (int cp = 0; cp < C; ++cp) {
                        double P = exp(a[IDX2(s, cp, C)] + CONTENT(s, d, c) + Dd[IDX2(d - 1, c, C)] +
                                       Ad[IDX2(cp, c, C)] + bb[IDX2(s + d, c, C)] - logZ);
                        dA_b[IDX2(cp, c, C)] += P;
                        Pc += P;
                    }
                }
                dD_b[IDX2(d - 1, c, C)] += Pc;
                for (int u = s; u < s + d; ++u) mu[IDX2(u, c, C)] += Pc;
            }
#undef CONTENT
    *logZ_out = logZ;
    free(content); free(a); free(bb); free(tmp);
}

int oracle_edge_direct(int B, int T, int K, int C, const double *x, const double *A,
                       const double *D, const int32_t *lengths, int centre, int detach_nu,
                       const double *grad_logZ, double *logZ, double *dX, double *dA,
                       double *dD, double *mu_out, int nthreads)
{
    for (int b = 0; b < B; ++b)
        if (lengths[b] < 1 || lengths[b] > T) return 1;
    int nth = max_threads(nthreads);
    double *S = malloc(sizeof(double) * (size_t)B * (T + 1) * C);
    double *nu = malloc(sizeof(double) * (size_t)B * C);
    const double *Ad = A, *Dd = D;
    double *dA_all = calloc((size_t)B * C * C, sizeof(double));
    double *dD_all = calloc((size_t)B * K * C, sizeof(double));
    oracle_prefix(B, T, C, x, lengths, centre, S, nu);   /* only nu is used here */
#ifdef _OPENMP
    omp_set_num_threads(nth);
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        double *mu = malloc(sizeof(double) * (size_t)T * C);
        double g = grad_logZ ? grad_logZ[b] : 1.0;
        seq_edge_direct(lengths[b], T, K, C, x + (size_t)b * T * C, nu + (size_t)b * C, Ad, Dd,
                        &logZ[b], mu, dA_all + (size_t)b * C * C, dD_all + (size_t)b * K * C);
        finish_dx(lengths[b], T, C, centre && !detach_nu, g, mu, dX + (size_t)b * T * C);
        if (mu_out) memcpy(mu_out + (size_t)b * T * C, mu, sizeof(double) * (size_t)T * C);
        free(mu);
    }
    memset(dA, 0, sizeof(double) * (size_t)C * C);
    memset(dD, 0, sizeof(double) * (size_t)K * C);
    for (int b = 0; b < B; ++b) {
        double g = grad_logZ ? grad_logZ[b] : 1.0;
        for (size_t i = 0; i < (size_t)C * C; ++i) dA[i] += g * dA_all[(size_t)b * C * C + i];
        for (size_t i = 0; i < (size_t)K * C; ++i) dD[i] += g * dD_all[(size_t)b * K * C + i];
    }
    free(S); free(nu); free(dA_all); free(dD_all);
    return 0;
}

/* ---------------------------------------------------------------------------
 * Viterbi: the factorised recursion in (max,+), float64.
 *   vt[0,c] = 0
 *   v[t,c]  = max_{d=1..min(K,t)} ( (vt[t-d,c] + (S[t,c] - S[t-d,c])) + D[d-1,c] )
 *             best d: the smallest d reaching the max
 *   vt[t,c] = max_{c'} ( v[t,c'] + A[c',c] )       best c': the smallest reaching it
 *   score   = max_c v[L,c], final label the smallest reaching it
 * Backtrack: t = L, c = final; repeat: d = bd[t,c], s = t-d, label [s,t) = c,
 * seg_start[s] = 1, c = bc[s,c] if s > 0, t = s.
 * Outputs: score[B] (float64), labels[B,T] (int32, -1 beyond L_b),
 * seg_start[B,T] (uint8, 0 beyond L_b).
 * ------------------------------------------------------------------------- */
int oracle_viterbi(int B, int T, int K, int C, const double *x, const double *A, const double *D,
                   const int32_t *lengths, int centre, double *score, int32_t *labels,
                   uint8_t *seg_start, int nthreads)
{
    for (int b = 0; b < B; ++b)
        if (lengths[b] < 1 || lengths[b] > T) return 1;
    int nth = max_threads(nthreads);
    double *S = malloc(sizeof(double) * (size_t)B * (T + 1) * C);
    double *nu = malloc(sizeof(double) * (size_t)B * C);
    const double *Ad = A, *Dd = D;
    oracle_prefix(B, T, C, x, lengths, centre, S, nu);
#ifdef _OPENMP
    omp_set_num_threads(nth);
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (int b = 0; b < B; ++b) {
        int L = lengths[b];
        const double *Sb = S + (size_t)b * (T + 1) * C;
        size_t n = (size_t)(L + 1) * C;
        double *v = malloc(sizeof(double) * n);
        double *vt = malloc(sizeof(double) * n);
        int32_t *bd = malloc(sizeof(int32_t) * n);
        int32_t *bc = malloc(sizeof(int32_t) * n);
        for (int c = 0; c < C; ++c) vt[IDX2(0, c, C)] = 0.0;
        for (int t = 1; t <= L; ++t) {
            for (int c = 0; c < C; ++c) {
                double best = -INFINITY;
                int arg = 0;
                for (int d = 1; d <= K && d <= t; ++d) {
                    double cand = (vt[IDX2(t - d, c, C)] + (Sb[IDX2(t, c, C)] - Sb[IDX2(t - d, c, C)])) +
                                  Dd[IDX2(d - 1, c, C)];
                    if (cand > best) { best = cand; arg = d; }
                }
                v[IDX2(t, c, C)] = best;
                bd[IDX2(t, c, C)] = arg;
            }
            if (t < L) {
                for (int c = 0; c < C; ++c) {
                    double best = -INFINITY;
                    int arg = 0;
                    for (int cp = 0; cp < C; ++cp) {
                        double cand = v[IDX2(t, cp, C)] + Ad[IDX2(cp, c, C)];
                        if (cand > best) { best = cand; arg = cp; }
                    }
                    vt[IDX2(t, c, C)] = best;
                    bc[IDX2(t, c, C)] = arg;
                }
            }
        }
        double best = -INFINITY;
        int c = 0;
        for (int cc = 0; cc < C; ++cc)
            if (v[IDX2(L, cc, C)] > best) { best = v[IDX2(L, cc, C)]; c = cc; }
        score[b] = best;
        int32_t *lab = labels + (size_t)b * T;
        uint8_t *ss = seg_start + (size_t)b * T;
        for (int u = 0; u < T; ++u) { lab[u] = -1; ss[u] = 0; }
        int t = L;
        while (t > 0) {
            int d = bd[IDX2(t, c, C)];
            int s = t - d;
            for (int u = s; u < t; ++u) lab[u] = c;
            ss[s] = 1;
            if (s > 0) c = bc[IDX2(s, c, C)];
            t = s;
        }
        free(v); free(vt); free(bd); free(bc);
    }
    free(S); free(nu);
    return 0;
}
