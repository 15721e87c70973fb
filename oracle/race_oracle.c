/*
 * race_oracle.c -- plain fp64 CPU oracle for RACE Attention (forward and backward).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls this
 * file: it is used by the test suite, by the smoke check and by the benchmark's
 * CPU-baseline leg, and it shares no code, header or table with the CUDA library.
 *
 * What it computes, and where each step comes from ("RACE Attention: A Strictly
 * Linear-Time Attention for Long-Sequence Training", gist.science summaries of
 * arXiv 2510.04008; the Chinese page is cited as zh, the others by language):
 *
 *   sharpened angular kernel that RACE approximates:
 *       sim(q,k) = (1 - arccos(q^T k / (|q||k|)) / pi)^gamma      (es §2.1, fr §2A, zh §2.1)
 *   per-token soft bucket assignment (zh §2.2 "soft bucketization"; pt §2):
 *       x^ = x / |x|                                  (the kernel works on the cosine)
 *       p_l = W_l x^  (P Gaussian hyperplanes per table l = 0..L-1)
 *       u_l = tanh(p_l)                               (zh §2.2, pt §2, es §2.3)
 *       phi_l = softmax_r( beta * c_r . u_l ),  r = 0..R-1, R = 2^P hypercube corners
 *   bucket statistics per table (zh §2.2 "bucket aggregation"):
 *       A_l[r] = sum_j phi_l(k_j)[r],   B_l[r,:] = sum_j phi_l(k_j)[r] v_j
 *   read-out with global normalisation (zh §2.2):
 *       O_i = sum_l phi_l(q_i)^T B_l / sum_l phi_l(q_i)^T A_l
 *   Algorithm 1 (bidirectional): the sums run over every key.
 *   Algorithm 2 (causal, zh §2.3; de §3): streaming cumulative statistics, so the sums
 *   for query i run over keys j <= i.
 *
 * Readings taken where the pages leave a step open (each is listed with its reason in the
 * design notes of the repository):
 *   - beta = 1/tau multiplies the corner logits (the error bound O(P/beta + ...) of
 *     Theorem 2, zh §3, falls as beta grows); tau = 0 selects hard sign hashing,
 *     phi_l = one-hot at r* = sum_p [p_lp > 0] 2^p (the YOSO-style hash the pages
 *     contrast against, es §2.3).
 *   - corner r has sign c_rp = +1 when bit p of r is set, else -1.
 *   - A and B are kept together as one state H_l = sum_j phi_l(k_j) [v_j, 1]^T, so the
 *     last column of the read-out is the denominator.
 *   - the causal sums include the diagonal (j <= i).
 *   - |x| is floored at 1e-12; a read-out whose denominator is exactly zero (hard hashing
 *     only) returns o_i = 0 and den_i = 0.
 *   - The backward pass is the chain rule applied to the steps above (the pages state the
 *     method is differentiable end to end, es §2.3, de §2, but print no gradient).
 *
 * Layout: every sequence tensor is [BH, N, d] row-major (d fastest); W is [L, P, d].
 * Parallelism (OpenMP) runs only over quantities that are independent in the definition:
 * tokens for the feature map, and single columns (or single feature rows) of the state
 * for the scans, so every sum is accumulated in token order exactly as written.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define RACE_ORACLE_EPS 1e-12
#define RACE_ORACLE_BLOCK 2048 /* tokens whose features are formed before the scan walks them */

/* ---------------------------------------------------------------------------------------- */
/* Feature map                                                                              */
/* ---------------------------------------------------------------------------------------- */

/* Norm of x floored at eps: the x^ = x / |x| step of the kernel's cosine. */
static double row_norm(const double *x, int d)
{
    double s = 0.0;
    for (int c = 0; c < d; ++c) s += x[c] * x[c];
    s = sqrt(s);
    return s > RACE_ORACLE_EPS ? s : RACE_ORACLE_EPS;
}

/* Sign of hyperplane p at corner r: +1 when bit p of r is set. */
static double corner_sign(int r, int p) { return ((r >> p) & 1) ? 1.0 : -1.0; }

/* phi(x) in R^{L*R}: normalise, project on the L tables of P hyperplanes, squash with
 * tanh, soft-assign each table to its R = 2^P corners (softmax of beta * c_r . u).
 * hard != 0 gives the one-hot sign hash instead. */
void race_oracle_features(const double *x, int d, const double *W, int L, int P,
                          double beta, int hard, double *phi)
{
    const int R = 1 << P;
    const double n = row_norm(x, d);
    double *xh = (double *)malloc(sizeof(double) * (size_t)d);
    for (int c = 0; c < d; ++c) xh[c] = x[c] / n;
    for (int l = 0; l < L; ++l) {
        double proj[8], u[8], z[64];
        for (int p = 0; p < P; ++p) {
            const double *w = W + ((size_t)l * P + p) * d;
            double s = 0.0;
            for (int c = 0; c < d; ++c) s += w[c] * xh[c];
            proj[p] = s;
        }
        double *out = phi + (size_t)l * R;
        if (hard) {
            int rstar = 0;
            for (int p = 0; p < P; ++p)
                if (proj[p] > 0.0) rstar |= 1 << p;
            for (int r = 0; r < R; ++r) out[r] = (r == rstar) ? 1.0 : 0.0;
            continue;
        }
        for (int p = 0; p < P; ++p) u[p] = tanh(proj[p]);
        double zmax = -INFINITY;
        for (int r = 0; r < R; ++r) {
            double s = 0.0;
            for (int p = 0; p < P; ++p) s += corner_sign(r, p) * u[p];
            z[r] = beta * s;
            if (z[r] > zmax) zmax = z[r];
        }
        double tot = 0.0;
        for (int r = 0; r < R; ++r) {
            z[r] = exp(z[r] - zmax);
            tot += z[r];
        }
        for (int r = 0; r < R; ++r) out[r] = z[r] / tot;
    }
    free(xh);
}

/* Hard sign-hash bucket index of every table: idx[l] = sum_p [W_lp . x^ > 0] 2^p. */
void race_oracle_hash_indices(const double *x, int d, const double *W, int L, int P,
                              int32_t *idx)
{
    const double n = row_norm(x, d);
    for (int l = 0; l < L; ++l) {
        int r = 0;
        for (int p = 0; p < P; ++p) {
            const double *w = W + ((size_t)l * P + p) * d;
            double s = 0.0;
            for (int c = 0; c < d; ++c) s += w[c] * (x[c] / n);
            if (s > 0.0) r |= 1 << p;
        }
        idx[l] = r;
    }
}

/* Vector-Jacobian product of the feature map: given dphi = dLoss/dphi(x), return
 * dx = dLoss/dx through softmax, the corner logits, tanh, the projection and the
 * normalisation (soft hashing only); dp (optional, [L*P]) receives dLoss/dp for the
 * projections p = W_l x^, from which the gradient of W follows (dW_lp += dp_lp x^). */
static void features_vjp(const double *x, int d, const double *W, int L, int P, double beta,
                         const double *dphi, double *dx, double *dp_out)
{
    const int R = 1 << P;
    double s2 = 0.0;
    for (int c = 0; c < d; ++c) s2 += x[c] * x[c];
    const double raw = sqrt(s2);
    const double n = raw > RACE_ORACLE_EPS ? raw : RACE_ORACLE_EPS;
    double *xh = (double *)malloc(sizeof(double) * (size_t)d);
    double *dxh = (double *)calloc((size_t)d, sizeof(double));
    double *phi = (double *)malloc(sizeof(double) * (size_t)R);
    for (int c = 0; c < d; ++c) xh[c] = x[c] / n;
    for (int l = 0; l < L; ++l) {
        double proj[8], u[8], z[64], dz[64], du[8], dp[8];
        for (int p = 0; p < P; ++p) {
            const double *w = W + ((size_t)l * P + p) * d;
            double s = 0.0;
            for (int c = 0; c < d; ++c) s += w[c] * xh[c];
            proj[p] = s;
            u[p] = tanh(s);
        }
        double zmax = -INFINITY;
        for (int r = 0; r < R; ++r) {
            double s = 0.0;
            for (int p = 0; p < P; ++p) s += corner_sign(r, p) * u[p];
            z[r] = beta * s;
            if (z[r] > zmax) zmax = z[r];
        }
        double tot = 0.0;
        for (int r = 0; r < R; ++r) {
            phi[r] = exp(z[r] - zmax);
            tot += phi[r];
        }
        for (int r = 0; r < R; ++r) phi[r] /= tot;
        /* softmax: dz_r = phi_r (dphi_r - sum_s phi_s dphi_s) */
        const double *g = dphi + (size_t)l * R;
        double dot = 0.0;
        for (int r = 0; r < R; ++r) dot += phi[r] * g[r];
        for (int r = 0; r < R; ++r) dz[r] = phi[r] * (g[r] - dot);
        /* z_r = beta sum_p c_rp u_p ; u = tanh(proj) */
        for (int p = 0; p < P; ++p) {
            double s = 0.0;
            for (int r = 0; r < R; ++r) s += corner_sign(r, p) * dz[r];
            du[p] = beta * s;
            dp[p] = du[p] * (1.0 - u[p] * u[p]);
            if (dp_out) dp_out[l * P + p] = dp[p];
        }
        /* proj = W_l x^ */
        for (int p = 0; p < P; ++p) {
            const double *w = W + ((size_t)l * P + p) * d;
            for (int c = 0; c < d; ++c) dxh[c] += w[c] * dp[p];
        }
    }
    /* x^ = x / max(|x|, eps) */
    if (raw > RACE_ORACLE_EPS) {
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += xh[c] * dxh[c];
        for (int c = 0; c < d; ++c) dx[c] = (dxh[c] - xh[c] * dot) / n;
    } else {
        for (int c = 0; c < d; ++c) dx[c] = dxh[c] / n;
    }
    free(xh);
    free(dxh);
    free(phi);
}

void race_oracle_features_backward(const double *x, int d, const double *W, int L, int P,
                                   double beta, const double *dphi, double *dx)
{
    if (d < 1) return;
    features_vjp(x, d, W, L, P, beta, dphi, dx, NULL);
}

/* dW[l][p][:] += sum over the tokens t0..t0+nt-1 of dp[t][l*P+p] x^_t, x^ = x / max(|x|, eps),
 * every element summed in token order. */
static void accumulate_dw(const double *x, int64_t t0, int64_t nt, int d, int LP, const double *dp,
                          double *dW)
{
    double *inv = (double *)malloc(sizeof(double) * (size_t)(nt > 0 ? nt : 1));
    if (!inv) return;
    for (int64_t t = 0; t < nt; ++t) inv[t] = 1.0 / row_norm(x + (t0 + t) * d, d);
#pragma omp parallel for schedule(static)
    for (int e = 0; e < LP * d; ++e) {
        const int lp = e / d, c = e % d;
        double s = dW[e];
        for (int64_t t = 0; t < nt; ++t) s += dp[t * LP + lp] * x[(t0 + t) * d + c] * inv[t];
        dW[e] = s;
    }
    free(inv);
}

/* ---------------------------------------------------------------------------------------- */
/* Helpers                                                                                  */
/* ---------------------------------------------------------------------------------------- */

/* Features of tokens [t0, t0+nt) of one head into phi[nt][M]. */
static void features_block(const double *x, int64_t t0, int64_t nt, int d, const double *W,
                           int L, int P, double beta, int hard, double *phi)
{
    const int M = L << P;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < nt; ++t)
        race_oracle_features(x + (t0 + t) * d, d, W, L, P, beta, hard, phi + t * M);
}

/* Augmented value row: v~ = [v, 1]. */
static double vt_at(const double *v, int64_t j, int d, int c)
{
    return c < d ? v[j * d + c] : 1.0;
}

/* ---------------------------------------------------------------------------------------- */
/* Forward: Algorithm 1 (causal = 0) and Algorithm 2 (causal = 1)                           */
/* ---------------------------------------------------------------------------------------- */

/* One head.  rows (ascending) selects the query rows written to out/den; NULL = all rows.
 * The state is held as Ht[c][m] = sum_j phi(k_j)[m] v~_j[c]: column c of every table's
 * bucket statistics (c < d: B, c = d: A). */
static int forward_head(const double *q, const double *k, const double *v, const double *W,
                        int64_t N, int d, int L, int P, double tau, int causal,
                        int64_t nrows, const int64_t *rows, double *out, double *den)
{
    const int M = L << P, D = d + 1;
    const int hard = tau == 0.0;
    const double beta = hard ? 0.0 : 1.0 / tau;
    const int64_t NB = N < RACE_ORACLE_BLOCK ? (N > 0 ? N : 1) : RACE_ORACLE_BLOCK;
    const int64_t nout = rows ? nrows : N;
    double *Ht = (double *)calloc((size_t)M * D, sizeof(double));
    double *Y = (double *)malloc(sizeof(double) * (size_t)(nout > 0 ? nout : 1) * D);
    double *phik = (double *)malloc(sizeof(double) * (size_t)NB * M);
    double *phiq = (double *)malloc(sizeof(double) * (size_t)NB * M);
    /* map each token of the block to its output slot (-1 = not requested) */
    int64_t *slot = (int64_t *)malloc(sizeof(int64_t) * (size_t)NB);
    if (!Ht || !Y || !phik || !phiq || !slot) {
        free(Ht); free(Y); free(phik); free(phiq); free(slot);
        return 1;
    }

    if (!causal) {
        /* Algorithm 1, aggregation: every key into every table's bucket statistics. */
        for (int64_t t0 = 0; t0 < N; t0 += NB) {
            const int64_t nt = (N - t0 < NB) ? N - t0 : NB;
            features_block(k, t0, nt, d, W, L, P, beta, hard, phik);
#pragma omp parallel for schedule(static)
            for (int c = 0; c < D; ++c) {
                double *h = Ht + (size_t)c * M;
                for (int64_t t = 0; t < nt; ++t) {
                    const double a = vt_at(v, t0 + t, d, c);
                    const double *f = phik + t * M;
                    for (int m = 0; m < M; ++m) h[m] += f[m] * a;
                }
            }
        }
    }

    int64_t next = 0; /* index into rows of the next requested row */
    for (int64_t t0 = 0; t0 < N; t0 += NB) {
        const int64_t nt = (N - t0 < NB) ? N - t0 : NB;
        int any = 0;
        for (int64_t t = 0; t < nt; ++t) {
            slot[t] = -1;
            if (!rows) {
                slot[t] = t0 + t;
                any = 1;
            } else if (next < nrows && rows[next] == t0 + t) {
                slot[t] = next++;
                any = 1;
                while (next < nrows && rows[next] == t0 + t) ++next; /* duplicates */
            }
        }
        if (causal) features_block(k, t0, nt, d, W, L, P, beta, hard, phik);
        if (any) {
            /* query features only where a row is requested */
#pragma omp parallel for schedule(static)
            for (int64_t t = 0; t < nt; ++t)
                if (slot[t] >= 0)
                    race_oracle_features(q + (t0 + t) * d, d, W, L, P, beta, hard, phiq + t * M);
        }
        if (!causal && !any) continue;
#pragma omp parallel for schedule(static)
        for (int c = 0; c < D; ++c) {
            double *h = Ht + (size_t)c * M;
            for (int64_t t = 0; t < nt; ++t) {
                if (causal) {
                    /* Algorithm 2: key j = t0+t joins the cumulative statistics first,
                     * so query j reads keys 0..j. */
                    const double a = vt_at(v, t0 + t, d, c);
                    const double *f = phik + t * M;
                    for (int m = 0; m < M; ++m) h[m] += f[m] * a;
                }
                if (slot[t] >= 0) {
                    const double *f = phiq + t * M;
                    double s = 0.0;
                    for (int m = 0; m < M; ++m) s += f[m] * h[m];
                    Y[slot[t] * D + c] = s;
                }
            }
        }
    }

    /* O_i = numerator / denominator */
    for (int64_t i = 0; i < nout; ++i) {
        const double dn = Y[i * D + d];
        den[i] = dn;
        for (int c = 0; c < d; ++c) out[i * d + c] = dn != 0.0 ? Y[i * D + c] / dn : 0.0;
    }
    free(Ht); free(Y); free(phik); free(phiq); free(slot);
    return 0;
}

int race_oracle_forward(const double *q, const double *k, const double *v, const double *W,
                        int64_t BH, int64_t N, int d, int L, int P, double tau, int causal,
                        int64_t nrows, const int64_t *rows, double *out, double *den)
{
    if (BH < 0 || N < 0 || d < 1 || L < 1 || P < 1 || P > 6 || tau < 0.0) return 2;
    const int64_t nout = rows ? nrows : N;
    for (int64_t bh = 0; bh < BH; ++bh) {
        const size_t off = (size_t)bh * N * d;
        int rc = forward_head(q + off, k + off, v + off, W, N, d, L, P, tau, causal, nrows, rows,
                              out + (size_t)bh * nout * d, den + (size_t)bh * nout);
        if (rc) return rc;
    }
    return 0;
}

/* Bucket statistics of one head over all N keys, H[m][c] = sum_j phi(k_j)[m] v~_j[c]
 * (zh §2.2, A and B of every table in one [M][d+1] array, m-major): the state Algorithm 2
 * carries after token N-1, from which a streaming step continues. */
static int state_head(const double *k, const double *v, const double *W, int64_t N, int d, int L,
                      int P, double tau, double *H)
{
    const int M = L << P, D = d + 1;
    const int hard = tau == 0.0;
    const double beta = hard ? 0.0 : 1.0 / tau;
    const int64_t NB = N < RACE_ORACLE_BLOCK ? (N > 0 ? N : 1) : RACE_ORACLE_BLOCK;
    double *phik = (double *)malloc(sizeof(double) * (size_t)NB * M);
    if (!phik) return 1;
    memset(H, 0, sizeof(double) * (size_t)M * D);
    for (int64_t t0 = 0; t0 < N; t0 += NB) {
        const int64_t nt = (N - t0 < NB) ? N - t0 : NB;
        features_block(k, t0, nt, d, W, L, P, beta, hard, phik);
#pragma omp parallel for schedule(static)
        for (int m = 0; m < M; ++m)
            for (int64_t t = 0; t < nt; ++t) {
                const double f = phik[t * M + m];
                for (int c = 0; c < D; ++c) H[(size_t)m * D + c] += f * vt_at(v, t0 + t, d, c);
            }
    }
    free(phik);
    return 0;
}

int race_oracle_state(const double *k, const double *v, const double *W, int64_t BH, int64_t N,
                      int d, int L, int P, double tau, double *H)
{
    if (BH < 0 || N < 0 || d < 1 || L < 1 || P < 1 || P > 6 || tau < 0.0) return 2;
    const size_t MD = (size_t)(L << P) * (size_t)(d + 1);
    for (int64_t bh = 0; bh < BH; ++bh) {
        const size_t off = (size_t)bh * N * d;
        int rc = state_head(k + off, v + off, W, N, d, L, P, tau, H + (size_t)bh * MD);
        if (rc) return rc;
    }
    return 0;
}

/* ---------------------------------------------------------------------------------------- */
/* Backward (chain rule through the forward above; soft hashing only)                      */
/* ---------------------------------------------------------------------------------------- */
/*
 *   Y_i = sum_{j in M(i)} (phi(q_i) . phi(k_j)) v~_j,   o_i = Y_i[:d] / Y_i[d]
 *   dY_i = [ dO_i / den_i , -(dO_i . o_i) / den_i ]
 *   dphi(q_i) = H_i dY_i,            H_i = sum_{j in M(i)} phi(k_j) v~_j^T
 *   dphi(k_j) = G_j v~_j,            G_j = sum_{i : j in M(i)} phi(q_i) dY_i^T
 *   dv_j      = (G_j^T phi(k_j))[:d]
 * and dq, dk follow from the feature-map VJP.
 */
static int backward_head(const double *q, const double *k, const double *v, const double *W,
                         const double *dout, int64_t N, int d, int L, int P, double tau,
                         int causal, double *dq, double *dk, double *dv, double *dW)
{
    const int M = L << P, D = d + 1;
    const double beta = 1.0 / tau;
    const int64_t NB = N < RACE_ORACLE_BLOCK ? (N > 0 ? N : 1) : RACE_ORACLE_BLOCK;
    double *o = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1) * d);
    double *den = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
    double *dY = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1) * D);
    double *Hm = (double *)calloc((size_t)M * D, sizeof(double)); /* Hm[m][c] */
    double *Gm = (double *)calloc((size_t)M * D, sizeof(double)); /* Gm[m][c] */
    double *Gc = (double *)calloc((size_t)M * D, sizeof(double)); /* Gc[c][m] */
    double *phik = (double *)malloc(sizeof(double) * (size_t)NB * M);
    double *phiq = (double *)malloc(sizeof(double) * (size_t)NB * M);
    double *dphi = (double *)malloc(sizeof(double) * (size_t)NB * M);
    double *dpb = dW ? (double *)malloc(sizeof(double) * (size_t)NB * L * P) : NULL;
    int rc = 0;
    if (!o || !den || !dY || !Hm || !Gm || !Gc || !phik || !phiq || !dphi || (dW && !dpb)) { rc = 1; goto done; }

    rc = forward_head(q, k, v, W, N, d, L, P, tau, causal, 0, NULL, o, den);
    if (rc) goto done;
    for (int64_t i = 0; i < N; ++i) {
        double s = 0.0;
        for (int c = 0; c < d; ++c) s += dout[i * d + c] * o[i * d + c];
        for (int c = 0; c < d; ++c) dY[i * D + c] = den[i] != 0.0 ? dout[i * d + c] / den[i] : 0.0;
        dY[i * D + d] = den[i] != 0.0 ? -s / den[i] : 0.0;
    }

    /* ---- dq: prefix (causal) or total (bidirectional) state H, one feature row m per thread */
    if (!causal) {
        for (int64_t t0 = 0; t0 < N; t0 += NB) {
            const int64_t nt = (N - t0 < NB) ? N - t0 : NB;
            features_block(k, t0, nt, d, W, L, P, beta, 0, phik);
#pragma omp parallel for schedule(static)
            for (int m = 0; m < M; ++m)
                for (int64_t t = 0; t < nt; ++t)
                    for (int c = 0; c < D; ++c)
                        Hm[(size_t)m * D + c] += phik[t * M + m] * vt_at(v, t0 + t, d, c);
        }
    }
    for (int64_t t0 = 0; t0 < N; t0 += NB) {
        const int64_t nt = (N - t0 < NB) ? N - t0 : NB;
        if (causal) features_block(k, t0, nt, d, W, L, P, beta, 0, phik);
#pragma omp parallel for schedule(static)
        for (int m = 0; m < M; ++m) {
            double *h = Hm + (size_t)m * D;
            for (int64_t t = 0; t < nt; ++t) {
                const int64_t i = t0 + t;
                if (causal)
                    for (int c = 0; c < D; ++c) h[c] += phik[t * M + m] * vt_at(v, i, d, c);
                double s = 0.0;
                for (int c = 0; c < D; ++c) s += h[c] * dY[i * D + c];
                dphi[t * M + m] = s;
            }
        }
#pragma omp parallel for schedule(static)
        for (int64_t t = 0; t < nt; ++t)
            features_vjp(q + (t0 + t) * d, d, W, L, P, beta, dphi + t * M, dq + (t0 + t) * d,
                         dpb ? dpb + t * L * P : NULL);
        if (dW) accumulate_dw(q, t0, nt, d, L * P, dpb, dW);
    }

    /* ---- dk, dv: suffix (causal) or total (bidirectional) state G */
    if (!causal) {
        for (int64_t t0 = 0; t0 < N; t0 += NB) {
            const int64_t nt = (N - t0 < NB) ? N - t0 : NB;
            features_block(q, t0, nt, d, W, L, P, beta, 0, phiq);
#pragma omp parallel for schedule(static)
            for (int m = 0; m < M; ++m)
                for (int64_t t = 0; t < nt; ++t)
                    for (int c = 0; c < D; ++c) {
                        const double g = phiq[t * M + m] * dY[(t0 + t) * D + c];
                        Gm[(size_t)m * D + c] += g;
                    }
        }
        for (int m = 0; m < M; ++m)
            for (int c = 0; c < D; ++c) Gc[(size_t)c * M + m] = Gm[(size_t)m * D + c];
    }
    const int64_t nblk = (N + NB - 1) / NB;
    for (int64_t b = nblk - 1; b >= 0; --b) {
        const int64_t t0 = b * NB;
        const int64_t nt = (N - t0 < NB) ? N - t0 : NB;
        features_block(k, t0, nt, d, W, L, P, beta, 0, phik);
        if (causal) features_block(q, t0, nt, d, W, L, P, beta, 0, phiq);
        /* dphi(k_j) = G_j v~_j, one feature row per thread, walking j downwards */
#pragma omp parallel for schedule(static)
        for (int m = 0; m < M; ++m) {
            double *g = Gm + (size_t)m * D;
            for (int64_t t = nt - 1; t >= 0; --t) {
                const int64_t j = t0 + t;
                if (causal)
                    for (int c = 0; c < D; ++c) g[c] += phiq[t * M + m] * dY[j * D + c];
                double s = 0.0;
                for (int c = 0; c < D; ++c) s += g[c] * vt_at(v, j, d, c);
                dphi[t * M + m] = s;
            }
        }
        /* dv_j = (G_j^T phi(k_j))[:d], one value column per thread */
#pragma omp parallel for schedule(static)
        for (int c = 0; c < d; ++c) {
            double *g = Gc + (size_t)c * M;
            for (int64_t t = nt - 1; t >= 0; --t) {
                const int64_t j = t0 + t;
                if (causal)
                    for (int m = 0; m < M; ++m) g[m] += phiq[t * M + m] * dY[j * D + c];
                double s = 0.0;
                for (int m = 0; m < M; ++m) s += g[m] * phik[t * M + m];
                dv[j * d + c] = s;
            }
        }
#pragma omp parallel for schedule(static)
        for (int64_t t = 0; t < nt; ++t)
            features_vjp(k + (t0 + t) * d, d, W, L, P, beta, dphi + t * M, dk + (t0 + t) * d,
                         dpb ? dpb + t * L * P : NULL);
        if (dW) accumulate_dw(k, t0, nt, d, L * P, dpb, dW);
    }

done:
    free(o); free(den); free(dY); free(Hm); free(Gm); free(Gc);
    free(phik); free(phiq); free(dphi); free(dpb);
    return rc;
}

/* dW (optional, [L][P][d], zeroed here) receives the gradient with respect to the
 * hyperplanes, summed over every head (W is shared by all of them): p = W_l x^ for every
 * q and k row, so dW_lp = sum over rows of dLoss/dp_lp x^. */
int race_oracle_backward(const double *q, const double *k, const double *v, const double *W,
                         const double *dout, int64_t BH, int64_t N, int d, int L, int P,
                         double tau, int causal, double *dq, double *dk, double *dv, double *dW)
{
    if (BH < 0 || N < 0 || d < 1 || L < 1 || P < 1 || P > 6 || !(tau > 0.0)) return 2;
    if (dW) memset(dW, 0, sizeof(double) * (size_t)L * P * d);
    for (int64_t bh = 0; bh < BH; ++bh) {
        const size_t off = (size_t)bh * N * d;
        int rc = backward_head(q + off, k + off, v + off, W, dout + off, N, d, L, P, tau, causal,
                               dq + off, dk + off, dv + off, dW);
        if (rc) return rc;
    }
    return 0;
}

int race_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
