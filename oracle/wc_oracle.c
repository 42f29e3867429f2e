/*
 * wc_oracle.c — plain fp64 CPU oracle for WildCat coreset attention.
 *
 * TEST INFRASTRUCTURE ONLY (see wc_oracle.h): plain loops in the order the
 * method states them, no blocking, no fusion.  OpenMP splits a few loops over
 * independent rows; it changes no summation order inside a row.
 *
 * Readings taken where the pages are silent (each also listed in the design
 * notes of the repository):
 *   - beta is passed in; the workloads use 1/sqrt(d).
 *   - the "sample from the residual diagonal" rule is an inverse-CDF draw:
 *     t = u * sum(d), pivot = the smallest i whose running sum C_i > t, with
 *     u from Philox4x32-10 (see wco_pivot_uniform).  The strict ">" never
 *     picks an index with d_i = 0, so a chosen pivot is never drawn again.
 *   - negative residual diagonal entries (rounding) are clamped to zero and
 *     the chosen pivot's residual is set to exactly zero.
 *   - the run stops early when the drawn pivot's residual is at most
 *     eps_stop * max_i H_ii (the factor would otherwise divide by noise).
 *   - entries of a new column at earlier pivots are set to zero, so that the
 *     pivot rows of the factor form an exactly lower-triangular matrix.
 */
#include "wc_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- Philox */

/* One Philox4x32 round [Philox]: two 32x32->64 multiplications whose high
 * halves are mixed with the other two words and the round key. */
static void philox_round(uint32_t x[4], const uint32_t k[2]) {
    const uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)x[0];
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)x[2];
    const uint32_t y0 = (uint32_t)(p1 >> 32) ^ x[1] ^ k[0];
    const uint32_t y1 = (uint32_t)p1;
    const uint32_t y2 = (uint32_t)(p0 >> 32) ^ x[3] ^ k[1];
    const uint32_t y3 = (uint32_t)p0;
    x[0] = y0; x[1] = y1; x[2] = y2; x[3] = y3;
}

void wco_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
    uint32_t x[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
    uint32_t k[2] = {key[0], key[1]};
    for (int round = 0; round < 10; ++round) {
        philox_round(x, k);
        /* key schedule: Weyl sequence (golden ratio, sqrt(3) - 1) */
        k[0] += 0x9E3779B9u;
        k[1] += 0xBB67AE85u;
    }
    memcpy(out, x, sizeof x);
}

double wco_pivot_uniform(uint64_t seed, uint32_t j, uint32_t unit) {
    const uint32_t ctr[4] = {j, unit, 0u, 0u};
    const uint32_t key[2] = {(uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32)};
    uint32_t out[4];
    wco_philox4x32_10(ctr, key, out);
    return (double)out[0] * (1.0 / 4294967296.0);
}

/* ------------------------------------------------------------ helpers */

static double dot(const double* a, const double* b, int32_t d) {
    double s = 0.0;
    for (int32_t c = 0; c < d; ++c) s += a[c] * b[c];
    return s;
}

/* ------------------------------------------------------ RPCholesky [Methodik-1] */

/* The smallest i with C_i > t, C_i = d_0 + ... + d_i summed in index order.
 * Also returns the running sums through `C` (n entries). */
static int32_t inverse_cdf(int32_t n, const double* dg, double t, double* C) {
    double run = 0.0;
    int32_t found = -1;
    for (int32_t i = 0; i < n; ++i) {
        run += dg[i];
        C[i] = run;
        if (found < 0 && run > t) found = i;
    }
    if (found < 0) { /* rounding left t at the top: take the last positive entry */
        for (int32_t i = n - 1; i >= 0; --i)
            if (dg[i] > 0.0) { found = i; break; }
    }
    return found;
}

int32_t wco_inverse_cdf(int32_t n, const double* dg, double t) {
    double* C = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    if (!C) return -1;
    const int32_t s = inverse_cdf(n, dg, t, C);
    free(C);
    return s;
}

/* How far the oracle's own CDF would have to move for pivot `s_other` to be
 * drawn instead of `s_own`: the distance from t to the farthest boundary
 * C_k that separates the two intervals, relative to the total T. */
static double pivot_margin(int32_t s_own, int32_t s_other, const double* C, double t, double T) {
    if (s_other > s_own) return (C[s_other - 1] - t) / T;
    return (t - C[s_other]) / T;
}

int wco_rpcholesky(int32_t n, int32_t d, const double* K, double beta, int32_t r,
                   uint64_t seed, uint32_t unit, double eps_stop,
                   const int32_t* replay_piv, int32_t replay_rank, double window,
                   int32_t* piv, double* F, double* dsum, double* dneg,
                   wco_select_info* info) {
    if (n < 1 || d < 1 || r < 1 || r > n || !K || !piv || !F || !info) return -1;

    double* dg = (double*)malloc(sizeof(double) * (size_t)n);   /* residual diagonal */
    double* H0 = (double*)malloc(sizeof(double) * (size_t)n);   /* H_ii, for dneg */
    double* C = (double*)malloc(sizeof(double) * (size_t)n);    /* running sums */
    if (!dg || !H0 || !C) { free(dg); free(H0); free(C); return -1; }

    memset(info, 0, sizeof *info);
    info->failed_step = -1;
    for (int32_t j = 0; j < r; ++j) piv[j] = -1;
    memset(F, 0, sizeof(double) * (size_t)r * (size_t)n);
    double worst_neg = 0.0;

    /* initial residual: the diagonal of H, H_ii = exp(beta ||k_i||^2) */
    double Hmax = 0.0;
    for (int32_t i = 0; i < n; ++i) {
        dg[i] = exp(beta * dot(K + (size_t)i * d, K + (size_t)i * d, d));
        H0[i] = dg[i];
        if (dg[i] > Hmax) Hmax = dg[i];
    }

    int32_t rank = r;
    for (int32_t j = 0; j < r; ++j) {
        double T = 0.0;
        for (int32_t i = 0; i < n; ++i) T += dg[i];
        if (dsum) dsum[j] = T;

        const int replaying = replay_piv != NULL;
        const int other_stops = replaying && j >= replay_rank;
        if (T <= 0.0) {
            if (replaying && !other_stops) { info->failed_step = j; info->fail_margin = INFINITY; }
            rank = j;
            break;
        }

        /* draw: t = u * T, pivot = smallest i with C_i > t */
        const double t = wco_pivot_uniform(seed, (uint32_t)j, unit) * T;
        const int32_t s_own = inverse_cdf(n, dg, t, C);
        int32_t s = s_own;

        if (replaying && !other_stops && replay_piv[j] != s_own) {
            const int32_t s_other = replay_piv[j];
            double m = INFINITY;
            if (s_other >= 0 && s_other < n && dg[s_other] > 0.0) m = pivot_margin(s_own, s_other, C, t, T);
            if (m <= window) {
                s = s_other;
                info->n_replays++;
                if (m > info->max_margin) info->max_margin = m;
            } else {
                info->failed_step = j;
                info->fail_margin = m;
                rank = j;
                break;
            }
        }

        /* stop rule: the drawn pivot carries (numerically) no residual */
        const double thresh = eps_stop * Hmax;
        int stop = dg[s] <= thresh;
        if (replaying && stop != other_stops) {
            const double m = fabs(dg[s] - thresh) / Hmax;
            if (m <= window) {
                stop = other_stops;
                info->n_replays++;
                if (m > info->max_margin) info->max_margin = m;
            } else {
                info->failed_step = j;
                info->fail_margin = m;
                rank = j;
                break;
            }
        }
        if (stop) { rank = j; break; }

        /* column j: g_i = H_{i,s} - sum_{c<j} F_ic F_sc ;  F_ij = g_i / sqrt(d_s) */
        piv[j] = s;
        const double root = sqrt(dg[s]);
        const double* ks = K + (size_t)s * d;
        const double* Fs = F + (size_t)s * r;
        #pragma omp parallel for schedule(static) if (n >= 4096)
        for (int32_t i = 0; i < n; ++i) {
            double* Fi = F + (size_t)i * r;
            double g = exp(beta * dot(K + (size_t)i * d, ks, d));
            for (int32_t c = 0; c < j; ++c) g -= Fi[c] * Fs[c];
            Fi[j] = g / root;
        }
        for (int32_t c = 0; c < j; ++c) F[(size_t)piv[c] * r + j] = 0.0;  /* earlier pivots: exactly zero */

        /* downdate the residual diagonal */
        for (int32_t i = 0; i < n; ++i) {
            const double f = F[(size_t)i * r + j];
            const double nd = dg[i] - f * f;
            if (nd < 0.0 && nd / H0[i] < worst_neg) worst_neg = nd / H0[i];
            dg[i] = nd > 0.0 ? nd : 0.0;
        }
        dg[s] = 0.0;
    }
    if (dsum) {
        double T = 0.0;
        for (int32_t i = 0; i < n; ++i) T += dg[i];
        dsum[rank] = T;
    }
    if (dneg) *dneg = worst_neg;
    info->rank = rank;
    free(dg); free(H0); free(C);
    return 0;
}

/* --------------------------------------------------- Nystrom weights [Methodik-2] */

void wco_coreset_values(int32_t n, int32_t d, int32_t dv, const double* K, const double* V,
                        double beta, int32_t rank, const int32_t* piv, double* C1) {
    const int32_t w = dv + 1;
    #pragma omp parallel for schedule(static) if ((long long)rank * n >= 65536)
    for (int32_t a = 0; a < rank; ++a) {
        const double* ks = K + (size_t)piv[a] * d;
        double* row = C1 + (size_t)a * w;
        for (int32_t c = 0; c < w; ++c) row[c] = 0.0;
        for (int32_t i = 0; i < n; ++i) {
            const double h = exp(beta * dot(ks, K + (size_t)i * d, d));
            for (int32_t c = 0; c < dv; ++c) row[c] += h * V[(size_t)i * dv + c];
            row[dv] += h;
        }
    }
}

int wco_nystrom_weights(int32_t n, int32_t d, int32_t dv, const double* K, const double* V,
                        double beta, int32_t rank, const int32_t* piv, double* W) {
    const int32_t w = dv + 1;
    if (rank <= 0) return 0;
    double* A = (double*)malloc(sizeof(double) * (size_t)rank * rank);  /* h(K_S,K_S) */
    double* L = (double*)calloc((size_t)rank * rank, sizeof(double));
    double* Y = (double*)malloc(sizeof(double) * (size_t)rank * w);
    if (!A || !L || !Y) { free(A); free(L); free(Y); return -1; }

    wco_coreset_values(n, d, dv, K, V, beta, rank, piv, W);  /* W <- C1 */

    for (int32_t a = 0; a < rank; ++a)
        for (int32_t b = 0; b < rank; ++b)
            A[(size_t)a * rank + b] = exp(beta * dot(K + (size_t)piv[a] * d, K + (size_t)piv[b] * d, d));

    /* textbook Cholesky A = L L^T, row by row */
    int bad = 0;
    for (int32_t a = 0; a < rank && !bad; ++a) {
        for (int32_t b = 0; b <= a; ++b) {
            double s = A[(size_t)a * rank + b];
            for (int32_t c = 0; c < b; ++c) s -= L[(size_t)a * rank + c] * L[(size_t)b * rank + c];
            if (a == b) {
                if (s <= 0.0) { bad = 1; break; }
                L[(size_t)a * rank + a] = sqrt(s);
            } else {
                L[(size_t)a * rank + b] = s / L[(size_t)b * rank + b];
            }
        }
    }
    if (!bad) {
        /* forward: L Y = C1 */
        for (int32_t a = 0; a < rank; ++a)
            for (int32_t c = 0; c < w; ++c) {
                double s = W[(size_t)a * w + c];
                for (int32_t b = 0; b < a; ++b) s -= L[(size_t)a * rank + b] * Y[(size_t)b * w + c];
                Y[(size_t)a * w + c] = s / L[(size_t)a * rank + a];
            }
        /* backward: L^T W = Y */
        for (int32_t a = rank - 1; a >= 0; --a)
            for (int32_t c = 0; c < w; ++c) {
                double s = Y[(size_t)a * w + c];
                for (int32_t b = a + 1; b < rank; ++b) s -= L[(size_t)b * rank + a] * W[(size_t)b * w + c];
                W[(size_t)a * w + c] = s / L[(size_t)a * rank + a];
            }
    }
    free(A); free(L); free(Y);
    return bad ? -1 : 0;
}

/* ---------------------------------------------------- coreset attention [Abstract] */

void wco_coreset_attend(int32_t nq, int32_t d, int32_t dv, const double* Q, int32_t rank,
                        const double* Ks, const double* W, double beta, double* out) {
    const int32_t w = dv + 1;
    #pragma omp parallel for schedule(static) if ((long long)nq * rank >= 65536)
    for (int32_t q = 0; q < nq; ++q) {
        double* A = (double*)calloc((size_t)w, sizeof(double));
        const double* qv = Q + (size_t)q * d;
        for (int32_t a = 0; a < rank; ++a) {
            const double p = exp(beta * dot(qv, Ks + (size_t)a * d, d));
            for (int32_t c = 0; c < w; ++c) A[c] += p * W[(size_t)a * w + c];
        }
        for (int32_t c = 0; c < dv; ++c) out[(size_t)q * dv + c] = A[c] / A[dv];
        free(A);
    }
}

void wco_exact_attention(int32_t nq, int32_t nk, int32_t d, int32_t dv, const double* Q,
                         const double* K, const double* V, double beta, double* out) {
    #pragma omp parallel for schedule(static) if ((long long)nq * nk >= 65536)
    for (int32_t q = 0; q < nq; ++q) {
        const double* qv = Q + (size_t)q * d;
        double m = -INFINITY;
        for (int32_t i = 0; i < nk; ++i) {
            const double l = beta * dot(qv, K + (size_t)i * d, d);
            if (l > m) m = l;
        }
        double den = 0.0;
        double* o = out + (size_t)q * dv;
        for (int32_t c = 0; c < dv; ++c) o[c] = 0.0;
        for (int32_t i = 0; i < nk; ++i) {
            const double p = exp(beta * dot(qv, K + (size_t)i * d, d) - m);
            den += p;
            for (int32_t c = 0; c < dv; ++c) o[c] += p * V[(size_t)i * dv + c];
        }
        for (int32_t c = 0; c < dv; ++c) o[c] /= den;
    }
}
