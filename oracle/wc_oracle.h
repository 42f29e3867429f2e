/*
 * wc_oracle.h — plain fp64 CPU oracle for WildCat coreset attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA path in
 * coreset_attention_approximation_b200/csrc, and neither includes the other.
 *
 * Every routine works on one (batch, kv-head) unit, in fp64, on inputs that
 * the caller has widened from their storage type (bf16 / fp32) to double.
 * Matrices are dense and row-major unless stated otherwise.
 *
 * Sources (the pages are the authority on what is computed):
 *   [Methodik-1]  WildCat: Near-Linear Attention in Theory and Practice,
 *                 gist.science technical summary, "Methodik" item 1
 *                 (randomly pivoted Cholesky on H = exp(beta K K^T); the pivot
 *                 is drawn from the diagonal of the current residual matrix).
 *   [Methodik-2]  same page, "Methodik" item 2 (Nystrom weights
 *                 W = h(K_S,K_S)^+ h(K_S,K), compressed values V_S = W V).
 *   [Abstract]    same title, gptget.net page, Abstract (attend over only a
 *                 small weighted coreset; bounded inputs).
 *   [Philox]      Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
 *                 easy as 1, 2, 3", SC'11 — the Philox4x32-10 bijection.
 *
 * Pins (what checks this oracle against something other than itself) live in
 * tests/test_oracle_*.py.  Parity pinned for every function here; the only
 * reading that no page fixes (Philox draw, inverse-CDF rule, stop rule) is
 * stated beside the function that makes it.
 */
#ifndef WC_ORACLE_H
#define WC_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Philox4x32-10 [Philox]: out = bijection(ctr) under key, ten rounds. */
void wco_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);

/* The uniform that drives pivot step j of unit `unit`:
 * u = Philox4x32-10(ctr = (j, unit, 0, 0), key = (seed_lo, seed_hi)).x0 * 2^-32,
 * exact in double, in [0, 1). */
double wco_pivot_uniform(uint64_t seed, uint32_t j, uint32_t unit);

/* The pivot-draw rule on a given residual diagonal dg[0..n): the smallest i
 * with dg[0] + ... + dg[i] > t (running sums in index order), or, when
 * rounding leaves no such i, the last i with dg[i] > 0 (-1 if none). */
int32_t wco_inverse_cdf(int32_t n, const double* dg, double t);

/* Outcome of one RPCholesky run. */
typedef struct {
    int32_t rank;         /* pivots accepted (<= r) */
    int32_t n_replays;    /* steps where a replayed decision differed from the oracle's own */
    int32_t failed_step;  /* -1 when every replayed decision was within the window, else the step */
    int32_t pad;
    double  max_margin;   /* largest margin among the replayed steps (0 if none) */
    double  fail_margin;  /* margin of the refused step (0 if none) */
} wco_select_info;

/*
 * Randomly pivoted Cholesky on H_ik = exp(beta <k_i, k_k>)  [Methodik-1].
 *
 * K        n x d, row-major.
 * r        pivots requested (1 <= r <= n).
 * eps_stop stop rule: the run ends at step j (rank = j) when the drawn pivot
 *          has residual d_s <= eps_stop * max_i H_ii, or when sum(d) <= 0.
 * replay_piv / replay_rank / window: optional (replay_piv == NULL disables).
 *          When given, each step compares the oracle's own draw with
 *          replay_piv[j] (and its own stop decision with replay_rank); a
 *          differing decision whose margin (as defined in wc_oracle.c) is
 *          <= window is accepted and the run continues with the replayed
 *          pivot; otherwise info->failed_step = j and the run stops.
 * piv      out, r entries; entries >= rank are -1.
 * F        out, n x r row-major: the partial Cholesky factor, F F^T ~ H;
 *          columns >= rank are zero.
 * dsum     optional out (NULL allowed), r + 1 entries: sum_i d_i before
 *          step j (dsum[j]), and after the last step (dsum[rank]).
 * dneg     optional out (NULL allowed): the most negative value of
 *          (d_i - F_ij^2) / H_ii met before the clamp to zero, over all steps
 *          and rows (0 when no residual ever went below zero).  The residual
 *          of a positive semidefinite matrix has a non-negative diagonal, so
 *          anything beyond rounding noise here is a defect.
 * Returns 0, or -1 on invalid arguments.
 */
int wco_rpcholesky(int32_t n, int32_t d, const double* K, double beta, int32_t r,
                   uint64_t seed, uint32_t unit, double eps_stop,
                   const int32_t* replay_piv, int32_t replay_rank, double window,
                   int32_t* piv, double* F, double* dsum, double* dneg,
                   wco_select_info* info);

/*
 * Nystrom weights on the coreset S = piv[0..rank)  [Methodik-2], acting on
 * [V | 1] so that the softmax normaliser is compressed with the values:
 *   C1 = h(K_S, K) [V | 1]            (rank x (dv+1)),  h(x,y) = exp(beta <x,y>)
 *   W  = h(K_S, K_S)^{-1} C1          (rank x (dv+1))
 * h(K_S,K_S) is factored here by a textbook Cholesky (it is symmetric
 * positive definite for distinct pivots), followed by forward and backward
 * substitution.  Returns 0, or -1 if the factorisation meets a non-positive
 * pivot (h(K_S,K_S) numerically singular).
 */
int wco_nystrom_weights(int32_t n, int32_t d, int32_t dv, const double* K, const double* V,
                        double beta, int32_t rank, const int32_t* piv, double* W);

/* C1 = h(K_S, K) [V | 1] alone (rank x (dv+1)); the first factor of the weights. */
void wco_coreset_values(int32_t n, int32_t d, int32_t dv, const double* K, const double* V,
                        double beta, int32_t rank, const int32_t* piv, double* C1);

/*
 * Coreset attention  [Abstract]:
 *   A = exp(beta Q K_S^T) W          (nq x (dv+1))
 *   out[q, c] = A[q, c] / A[q, dv]   c < dv
 * Ks is rank x d (the pivot keys), W is rank x (dv+1).
 */
void wco_coreset_attend(int32_t nq, int32_t d, int32_t dv, const double* Q, int32_t rank,
                        const double* Ks, const double* W, double beta, double* out);

/* Exact softmax attention, out = softmax(beta Q K^T) V (the ground truth). */
void wco_exact_attention(int32_t nq, int32_t nk, int32_t d, int32_t dv, const double* Q,
                         const double* K, const double* V, double beta, double* out);

#ifdef __cplusplus
}
#endif
#endif
