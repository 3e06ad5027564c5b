/*
 * oracle.h -- plain fp64 CPU oracle for parallel Newton evaluation of
 * nonlinear sequences.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library
 * and its Python binding) may include, link or call this code; only the
 * tests, the smoke check and the CPU-baseline leg of the benchmark do.  It
 * shares no code, header, table or helper with the CUDA path.
 *
 * Citations of the form "page §X" refer to the web article
 * "并行牛顿方法：加速非线性序列评估的计算革命" ("Parallel Newton methods: a
 * computing revolution for nonlinear sequence evaluation", jsqmd.com news
 * item 789890), section X.
 *
 * What it computes (all in double precision):
 *   - one cell step y = f_t(s_prev) for the three cells (tanh RNN, GRU,
 *     Euler-discretised drift) and its exact Jacobian df_t/ds;
 *   - sequential evaluation s_t = f_t(s_{t-1}), t = 1..T   (page §1.1);
 *   - the residual F_t(s) = s_t - f_t(s_{t-1}) with s_0 fixed  (page §1.2,
 *     reading: F's sign and indexing are not printed);
 *   - one fixed-point update s <- s - J~^{-1} F(s) with J~ = I - subdiag(A~_t)
 *     for the four Jacobian approximations (page §1.2, §2.2):
 *       jacobi: A~ = 0, picard: A~ = I, quasi: A~ = diag(df/ds),
 *       newton: A~ = df/ds;
 *   - the full iteration with the stop rule r^(i) = max|F(s^(i))| <= tol
 *     (page §5.3, residual monitoring; the norm and tie-break are a reading).
 *   - a serial affine recurrence s_t = A_t s_{t-1} + b_t, the object the
 *     parallel scan of page §2.1 evaluates.
 *
 * Parity status: every function here is pinned by the CPU tests (library
 * cells, finite differences, a dense linear solve of J~ delta = -F,
 * causality, closed forms).  The iteration COUNTS at the benchmark sizes
 * are pinned only through those pins of the update step; the page prints no
 * count for them.
 */
#ifndef PN_ORACLE_H
#define PN_ORACLE_H

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_TANH_RNN = 0, ORC_GRU = 1, ORC_EULER = 2 };
enum { ORC_JACOBI = 0, ORC_PICARD = 1, ORC_QUASI = 2, ORC_NEWTON = 3 };
enum {
  ORC_OK = 0,
  ORC_NOT_CONVERGED = 1,
  ORC_ERR_INVALID = -1,
  ORC_ERR_NOMEM = -2,
  ORC_ERR_NONFINITE = -4
};

/* Parameter packing (row-major, fp64):
 *   tanh RNN : W[D][D], U[D][d_in], b[D]          f(s) = tanh(W s + U x + b)
 *   GRU      : W_ih[3D][d_in], W_hh[3D][D], b_ih[3D], b_hh[3D]
 *              gate blocks in the order r, z, n (the PyTorch convention)
 *   Euler    : W[D][D]   (d_in must equal D; x_t is c_t)
 *              f(s) = s + eps * tanh(W s + c_t)                         */
long orc_param_count(int cell, int D, int d_in);

/* y = f_t(s_prev) for one step.  x_t has d_in entries. */
int orc_cell(int cell, int D, int d_in, const double* p, double eps,
             const double* x_t, const double* s_prev, double* y);

/* J = df_t/ds at s_prev, row-major D x D: J[j*D+k] = d y_j / d s_k. */
int orc_jacobian(int cell, int D, int d_in, const double* p, double eps,
                 const double* x_t, const double* s_prev, double* J);

/* A~ for the given mode at s_prev, row-major D x D. */
int orc_approx_jacobian(int cell, int mode, int D, int d_in, const double* p,
                        double eps, const double* x_t, const double* s_prev,
                        double* A);

/* s[b][t][:] = f_t(s[b][t-1][:]), with s0[b] before t = 0.
 * x: [B][T][d_in], s0: [B][D], s: [B][T][D].  nthreads <= 0 means 1. */
int orc_sequential(int cell, int D, int d_in, const double* p, double eps,
                   int T, int B, const double* x, const double* s0, double* s,
                   int nthreads);

/* F[b][t] = s[b][t] - f_t(s[b][t-1]) (s0 before t = 0); returns max |F|
 * through *rmax (NaN propagates). F may be NULL. */
int orc_residual(int cell, int D, int d_in, const double* p, double eps,
                 int T, int B, const double* x, const double* s0,
                 const double* s, double* F, double* rmax, int nthreads);

/* One update: s_next = s_cur + delta where J~ delta = -F(s_cur), solved by
 * the forward recurrence delta_t = A~_t delta_{t-1} - F_t, delta_0 = 0. */
int orc_update(int cell, int mode, int D, int d_in, const double* p,
               double eps, int T, int B, const double* x, const double* s0,
               const double* s_cur, double* s_next, int nthreads);

/* Full iteration from s^(0)_t = s0 for all t.  Stops at the first i with
 * r^(i) <= tol (status OK), or non-finite r^(i) (NONFINITE), or i ==
 * max_iters (NOT_CONVERGED).  s_out receives s^(i) for that i, *iters = i,
 * *resid = r^(i); history[k] = r^(k) for k <= i and k < hist_cap. */
int orc_iterate(int cell, int mode, int D, int d_in, const double* p,
                double eps, int T, int B, const double* x, const double* s0,
                int max_iters, double tol, double* s_out, int* iters,
                double* resid, double* history, int hist_cap, int nthreads);

/* s[t] = A[t] s[t-1] + b[t] for t = 0..T-1 with s_init before t = 0.
 * A: [T][D][D], b: [T][D], s: [T][D].  A serial loop. */
int orc_affine_recurrence(int D, int T, const double* A, const double* b,
                          const double* s_init, double* s);

#ifdef __cplusplus
}
#endif
#endif
