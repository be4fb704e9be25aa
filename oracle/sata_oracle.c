/*
 * SATA oracle: a plain, slow, float64 CPU statement of symmetry-aware Taylor
 * attention.  TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and
 * the benchmark's CPU-baseline leg may call it; the product path never does.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * Sources (web pages on the method; cited by page and section):
 *   [CC-TAYLOR] "Self-attention at constant cost per token via symmetry-aware
 *               Taylor approximation" (blog.hotdry.top, 2026-02-05)
 *   [CC-HW]     "Constant-cost attention: hardware optimization"
 *               (blog.hotdry.top, 2026-02-05)
 *
 * Every function below is checked by the CPU tests against something other
 * than itself (closed forms, brute force, exact integer identities, the
 * softmax limit); no function here is "parity unpinned".
 *
 * Conventions (the plainest reading where the pages leave a step open):
 *   - P is the number of Taylor terms, degrees p = 0 .. P-1
 *     ([CC-TAYLOR] "Feature maps and linear attention": sum from p=0 to P-1).
 *   - alpha_p = 1 / (p! * c^p); the caller passes c (the method uses sqrt(d_K))
 *     ([CC-TAYLOR] "The Taylor approximation").
 *   - M_p: all nondecreasing index tuples (i1 <= ... <= ip) over 0..d_K-1, in
 *     lexicographic order, degrees concatenated p = 0 .. P-1; M_0 is the one
 *     empty tuple ([CC-TAYLOR] "The Taylor approximation": upper-triangular
 *     minimal basis; "Hardware optimization paths": rows nondecreasing).
 *   - C_p[r] = number of times the monomial of tuple r occurs in the full
 *     expansion of (q.k)^p = p! / prod(multiplicity!) ([CC-TAYLOR] "Feature
 *     maps and linear attention").
 *   - phi_p(x)[r] = prod_m x[M_p[r][m]] (empty product = 1) ([CC-HW] "Compute
 *     density": x[..., M].prod(dim=-1)).
 *   - States Z_p = sum_t phi_p(k_t), S_p = sum_t phi_p(k_t) v_t^T, updated with
 *     token T before reading token T's output (inclusive causal range)
 *     ([CC-TAYLOR] "Feature maps and linear attention").
 *   - y_T = sum_p alpha_p phi_p(q_T)^T C_p S_p / sum_p alpha_p <phi_p(q_T), Z_p>_C
 *     (the same section; its printed "S_T / Z_T" drops alpha_p and C_p, which
 *     the truncated-series line of the same section restores).
 *   - No epsilon and no clamping in the division.
 *
 * Layouts: row-major; q,k are [T][d_K], v is [T][d_V], y is [T][d_V];
 * S is [F][d_V], Z is [F]; M is [F][P-1] (unused slots -1, width >= 1).
 * Return value: 0 on success, -1 on an invalid argument, -2 out of memory.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

/* binomial coefficient as int64 (exact for every size used here) */
long long oracle_binom(int n, int k) {
    if (k < 0 || n < 0 || k > n) return 0;
    long long r = 1;
    for (int i = 1; i <= k; ++i) r = r * (n - k + i) / i;
    return r;
}

static long long factorial_ll(int n) {
    long long r = 1;
    for (int i = 2; i <= n; ++i) r *= i;
    return r;
}

/* Number of features of the truncated expansion: sum_{p<P} m_p, each m_p
 * counted by enumeration in oracle_basis, so this only sizes buffers. */
long long oracle_num_features(int d, int P) {
    long long F = 0;
    for (int p = 0; p < P; ++p) F += oracle_binom(d + p - 1, p);
    return F;
}

/*
 * Enumerate the minimal basis.  Writes, for each feature r (p-major, then
 * lexicographic within a degree): deg[r] = p, M[r][0..p-1] = i1 <= ... <= ip
 * (remaining slots -1), C[r] = p!/prod(mult!), and offsets[p] = first feature
 * of degree p, offsets[P] = F.  Any output pointer may be NULL.  Returns the
 * number of features written, or -1 on bad arguments.
 */
long long oracle_basis(int d, int P, int *deg, int *M, long long *C, long long *offsets) {
    if (d < 1 || P < 1 || P > 20) return -1;
    int width = P - 1 > 0 ? P - 1 : 1;
    long long r = 0;
    int idx[32];
    for (int p = 0; p < P; ++p) {
        if (offsets) offsets[p] = r;
        /* odometer over nondecreasing tuples, starting at (0,...,0) */
        for (int m = 0; m < p; ++m) idx[m] = 0;
        for (;;) {
            if (deg) deg[r] = p;
            if (M) {
                for (int m = 0; m < width; ++m) M[r * width + m] = (m < p) ? idx[m] : -1;
            }
            if (C) {
                /* multinomial p! / prod over distinct indices of (count)! */
                long long c = factorial_ll(p);
                int m = 0;
                while (m < p) {
                    int run = 1;
                    while (m + run < p && idx[m + run] == idx[m]) ++run;
                    c /= factorial_ll(run);
                    m += run;
                }
                C[r] = c;
            }
            ++r;
            /* advance: rightmost slot that can still grow */
            int pos = p - 1;
            while (pos >= 0 && idx[pos] == d - 1) --pos;
            if (pos < 0) break;
            idx[pos] += 1;
            for (int m = pos + 1; m < p; ++m) idx[m] = idx[pos];
        }
    }
    if (offsets) offsets[P] = r;
    return r;
}

/* phi for one vector x[d]: out[r] = prod of x over tuple r. */
static void features(int F, int width, const int *deg, const int *M, const double *x, double *out) {
    for (int r = 0; r < F; ++r) {
        double prod = 1.0;
        for (int m = 0; m < deg[r]; ++m) prod *= x[M[r * width + m]];
        out[r] = prod;
    }
}

typedef struct {
    int F, width;
    int *deg, *M;
    long long *C;
    double *coef; /* alpha_p * C_p[r] */
} basis_t;

static int basis_make(int d, int P, double c, basis_t *b) {
    long long F = oracle_num_features(d, P);
    b->F = (int)F;
    b->width = P - 1 > 0 ? P - 1 : 1;
    b->deg = (int *)malloc(sizeof(int) * F);
    b->M = (int *)malloc(sizeof(int) * F * b->width);
    b->C = (long long *)malloc(sizeof(long long) * F);
    b->coef = (double *)malloc(sizeof(double) * F);
    if (!b->deg || !b->M || !b->C || !b->coef) return -2;
    oracle_basis(d, P, b->deg, b->M, b->C, NULL);
    for (int r = 0; r < b->F; ++r) {
        int p = b->deg[r];
        double alpha = 1.0 / ((double)factorial_ll(p) * pow(c, (double)p));
        b->coef[r] = alpha * (double)b->C[r];
    }
    return 0;
}

static void basis_free(basis_t *b) {
    free(b->deg); free(b->M); free(b->C); free(b->coef);
}

/* phi_p(x) for all features of the truncated expansion (out has F entries). */
int oracle_features(int d, int P, const double *x, double *out) {
    if (d < 1 || P < 1 || !x || !out) return -1;
    basis_t b;
    if (basis_make(d, P, 1.0, &b)) { basis_free(&b); return -2; }
    features(b.F, b.width, b.deg, b.M, x, out);
    basis_free(&b);
    return 0;
}

/*
 * The method's recurrence, token by token, continuing from the state given in
 * S [F][d_V] and Z [F] (zero them for a fresh sequence).  For each token t:
 *   Z += phi(k_t);  S += phi(k_t) v_t^T;                       (update)
 *   num = sum_r alpha C phi(q_t)_r S[r,:];  den = sum_r alpha C phi(q_t)_r Z[r];
 *   y_t = num / den.                                           (readout)
 * A decode step is this call with T = 1.  den may be NULL.
 */
int oracle_scan(int dK, int dV, int P, double c, long long T,
                const double *q, const double *k, const double *v,
                double *S, double *Z, double *y, double *den) {
    if (dK < 1 || dV < 1 || P < 1 || T < 0 || !S || !Z) return -1;
    if (T > 0 && (!q || !k || !v || !y)) return -1;
    basis_t b;
    if (basis_make(dK, P, c, &b)) { basis_free(&b); return -2; }
    double *pk = (double *)malloc(sizeof(double) * b.F);
    double *pq = (double *)malloc(sizeof(double) * b.F);
    double *num = (double *)malloc(sizeof(double) * dV);
    if (!pk || !pq || !num) { free(pk); free(pq); free(num); basis_free(&b); return -2; }
    for (long long t = 0; t < T; ++t) {
        const double *qt = q + t * dK, *kt = k + t * dK, *vt = v + t * dV;
        features(b.F, b.width, b.deg, b.M, kt, pk);
        features(b.F, b.width, b.deg, b.M, qt, pq);
        for (int r = 0; r < b.F; ++r) {
            Z[r] += pk[r];
            double *Sr = S + (long long)r * dV;
            for (int j = 0; j < dV; ++j) Sr[j] += pk[r] * vt[j];
        }
        double dn = 0.0;
        for (int j = 0; j < dV; ++j) num[j] = 0.0;
        for (int r = 0; r < b.F; ++r) {
            double a = b.coef[r] * pq[r];
            const double *Sr = S + (long long)r * dV;
            dn += a * Z[r];
            for (int j = 0; j < dV; ++j) num[j] += a * Sr[j];
        }
        for (int j = 0; j < dV; ++j) y[t * dV + j] = num[j] / dn;
        if (den) den[t] = dn;
    }
    free(pk); free(pq); free(num);
    basis_free(&b);
    return 0;
}

/*
 * The quantity the recurrence computes, written directly: causal attention
 * with the truncated Taylor kernel w_ts = sum_{p<P} (q_t.k_s / c)^p / p!,
 *   y_t = sum_{s<=t} w_ts v_s / sum_{s<=t} w_ts.
 * ([CC-TAYLOR] "The Taylor approximation" and "Feature maps and linear
 * attention").  O(T^2).  den and kappa (sum|w| / |sum w|) may be NULL.
 */
int oracle_direct(int dK, int dV, int P, double c, long long T,
                  const double *q, const double *k, const double *v,
                  double *y, double *den, double *kappa) {
    if (dK < 1 || dV < 1 || P < 1 || T < 0) return -1;
    if (T > 0 && (!q || !k || !v || !y)) return -1;
    double *num = (double *)malloc(sizeof(double) * dV);
    if (!num) return -2;
    for (long long t = 0; t < T; ++t) {
        double dn = 0.0, absw = 0.0;
        for (int j = 0; j < dV; ++j) num[j] = 0.0;
        for (long long s = 0; s <= t; ++s) {
            double x = 0.0;
            for (int i = 0; i < dK; ++i) x += q[t * dK + i] * k[s * dK + i];
            x /= c;
            double w = 0.0, term = 1.0;
            for (int p = 0; p < P; ++p) {
                w += term;
                term = term * x / (double)(p + 1);
            }
            dn += w;
            absw += fabs(w);
            for (int j = 0; j < dV; ++j) num[j] += w * v[s * dV + j];
        }
        for (int j = 0; j < dV; ++j) y[t * dV + j] = num[j] / dn;
        if (den) den[t] = dn;
        if (kappa) kappa[t] = absw / fabs(dn);
    }
    free(num);
    return 0;
}

/*
 * The masked direct form above at a few chosen tokens only: for each of the n
 * token indices ts[i] (0 <= ts[i] < T), y[i] = sum_{s<=t} w_ts v_s / sum_{s<=t} w_ts
 * with the same weights w_ts = sum_{p<P} (q_t . k_s / c)^p / p!, summed in the
 * same order as oracle_direct; den[i] and kappa[i] as there (either may be NULL).
 * Each output costs O(t (d_K + d_V)), so outputs deep into a long sequence can be
 * checked without the whole O(T^2) table.  y is [n][d_V].
 */
int oracle_direct_at(int dK, int dV, int P, double c, long long T,
                     const double *q, const double *k, const double *v,
                     long long n, const long long *ts, double *y, double *den, double *kappa) {
    if (dK < 1 || dV < 1 || P < 1 || T < 0 || n < 0) return -1;
    if (n > 0 && (!q || !k || !v || !ts || !y)) return -1;
    double *num = (double *)malloc(sizeof(double) * dV);
    if (!num) return -2;
    for (long long i = 0; i < n; ++i) {
        const long long t = ts[i];
        if (t < 0 || t >= T) {
            free(num);
            return -1;
        }
        double dn = 0.0, absw = 0.0;
        for (int j = 0; j < dV; ++j) num[j] = 0.0;
        for (long long s = 0; s <= t; ++s) {
            double x = 0.0;
            for (int a = 0; a < dK; ++a) x += q[t * dK + a] * k[s * dK + a];
            x /= c;
            double w = 0.0, term = 1.0;
            for (int p = 0; p < P; ++p) {
                w += term;
                term = term * x / (double)(p + 1);
            }
            dn += w;
            absw += fabs(w);
            for (int j = 0; j < dV; ++j) num[j] += w * v[s * dV + j];
        }
        for (int j = 0; j < dV; ++j) y[i * dV + j] = num[j] / dn;
        if (den) den[i] = dn;
        if (kappa) kappa[i] = absw / fabs(dn);
    }
    free(num);
    return 0;
}

/*
 * Gradient of the loss L = sum_t dy_t . y_t with respect to q, k and v, for the
 * masked direct form above.  The pages define no backward pass; they expect the
 * attention to be trained inside ordinary Transformer pipelines ([CC-TAYLOR]
 * "Comparison with other methods"; end-to-end training is listed under "Future
 * directions").  The reading taken: the exact chain-rule gradient of
 *   y_t = num_t / den_t,  num_t = sum_{s<=t} w_ts v_s,  den_t = sum_{s<=t} w_ts,
 *   w_ts = T_P(x_ts) = sum_{p<P} x_ts^p / p!,  x_ts = q_t . k_s / c,
 * with the inputs taken as real numbers.  Written out:
 *   g_t = dy_t / den_t,  e_t = -(dy_t . y_t) / den_t    (through num and den)
 *   dw_ts = g_t . v_s + e_t
 *   dv_s += w_ts g_t
 *   dx_ts = dw_ts * T_{P-1}(x_ts)      (d/dx T_P = T_{P-1}; T_0 = 0)
 *   dq_t += dx_ts k_s / c,  dk_s += dx_ts q_t / c
 * over every pair s <= t.  Outputs are overwritten.  dq, dk are [T][d_K], dv is
 * [T][d_V].
 */
int oracle_direct_grad(int dK, int dV, int P, double c, long long T,
                       const double *q, const double *k, const double *v, const double *dy,
                       double *dq, double *dk, double *dv) {
    if (dK < 1 || dV < 1 || P < 1 || T < 0) return -1;
    if (T > 0 && (!q || !k || !v || !dy || !dq || !dk || !dv)) return -1;
    double *y = (double *)malloc(sizeof(double) * (T > 0 ? T * dV : 1));
    double *den = (double *)malloc(sizeof(double) * (T > 0 ? T : 1));
    double *g = (double *)malloc(sizeof(double) * dV);
    if (!y || !den || !g) {
        free(y);
        free(den);
        free(g);
        return -2;
    }
    int rc = oracle_direct(dK, dV, P, c, T, q, k, v, y, den, NULL);
    if (rc != 0) {
        free(y);
        free(den);
        free(g);
        return rc;
    }
    for (long long i = 0; i < T * dK; ++i) dq[i] = dk[i] = 0.0;
    for (long long i = 0; i < T * dV; ++i) dv[i] = 0.0;
    for (long long t = 0; t < T; ++t) {
        double e = 0.0;
        for (int j = 0; j < dV; ++j) {
            g[j] = dy[t * dV + j] / den[t];
            e -= g[j] * y[t * dV + j];
        }
        for (long long s = 0; s <= t; ++s) {
            double x = 0.0;
            for (int i = 0; i < dK; ++i) x += q[t * dK + i] * k[s * dK + i];
            x /= c;
            /* w = T_P(x) and its derivative T_{P-1}(x), summed term by term */
            double w = 0.0, dwdx = 0.0, term = 1.0;
            for (int p = 0; p < P; ++p) {
                w += term;
                if (p < P - 1) dwdx += term;
                term = term * x / (double)(p + 1);
            }
            double dw = e;
            for (int j = 0; j < dV; ++j) {
                dw += g[j] * v[s * dV + j];
                dv[s * dV + j] += w * g[j];
            }
            const double dx = dw * dwdx / c;
            for (int i = 0; i < dK; ++i) {
                dq[t * dK + i] += dx * k[s * dK + i];
                dk[s * dK + i] += dx * q[t * dK + i];
            }
        }
    }
    free(y);
    free(den);
    free(g);
    return 0;
}

/*
 * Exact causal softmax attention, the limit P -> infinity of the above
 * ([CC-TAYLOR] "The Taylor approximation": the series of exp(q.k/c)).
 * Uses the running maximum for the exponent, as any careful softmax does.
 */
int oracle_softmax(int dK, int dV, double c, long long T,
                   const double *q, const double *k, const double *v, double *y) {
    if (dK < 1 || dV < 1 || T < 0) return -1;
    if (T > 0 && (!q || !k || !v || !y)) return -1;
    double *x = (double *)malloc(sizeof(double) * (T > 0 ? T : 1));
    if (!x) return -2;
    for (long long t = 0; t < T; ++t) {
        double mx = -INFINITY;
        for (long long s = 0; s <= t; ++s) {
            double dot = 0.0;
            for (int i = 0; i < dK; ++i) dot += q[t * dK + i] * k[s * dK + i];
            x[s] = dot / c;
            if (x[s] > mx) mx = x[s];
        }
        double dn = 0.0;
        for (int j = 0; j < dV; ++j) y[t * dV + j] = 0.0;
        for (long long s = 0; s <= t; ++s) {
            double e = exp(x[s] - mx);
            dn += e;
            for (int j = 0; j < dV; ++j) y[t * dV + j] += e * v[s * dV + j];
        }
        for (int j = 0; j < dV; ++j) y[t * dV + j] /= dn;
    }
    free(x);
    return 0;
}

/* State size in values and the per-token FLOP count, summed term by term from
 * the per-term formulas of [CC-TAYLOR] "Hidden-state size and FLOPs":
 *   state_p = (d_V + 1) * m_p,  flops_p = (4 d_V + 2p + 4) * m_p,
 * with m_p counted by enumerating the basis (not by the binomial formula). */
int oracle_costs(int dK, int dV, int P, long long *state_values, long long *flops_per_token) {
    if (dK < 1 || dV < 1 || P < 1) return -1;
    long long F = oracle_num_features(dK, P);
    int *deg = (int *)malloc(sizeof(int) * F);
    if (!deg) return -2;
    oracle_basis(dK, P, deg, NULL, NULL, NULL);
    long long st = 0, fl = 0;
    for (long long r = 0; r < F; ++r) {
        st += dV + 1;
        fl += 4LL * dV + 2LL * deg[r] + 4;
    }
    free(deg);
    if (state_values) *state_values = st;
    if (flops_per_token) *flops_per_token = fl;
    return 0;
}
