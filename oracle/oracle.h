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
 *     parallel scan of page §2.1 evaluates;
 *   - the page's refinements of the iteration: a banded Jacobian
 *     approximation (page §2.2.2), damping (page §4.3, §5.3), adaptive
 *     switching to a more exact approximation when the residual stalls
 *     (page §5.3), reduced-precision storage of the iterate (page §2.3) and
 *     a windowed solve (page §1.3.1, §2.3); the readings are stated at
 *     orc_iterate_ex.
 *
 * Parity status: every function here is pinned by the CPU tests (library
 * cells, finite differences, a dense linear solve of J~ delta = -F,
 * causality, closed forms, numpy's and PyTorch's float conversions).  The
 * iteration COUNTS at the benchmark sizes are pinned only through those pins
 * of the update step; the page prints no count for them.
 */
#ifndef PN_ORACLE_H
#define PN_ORACLE_H

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_TANH_RNN = 0, ORC_GRU = 1, ORC_EULER = 2 };
enum { ORC_JACOBI = 0, ORC_PICARD = 1, ORC_QUASI = 2, ORC_NEWTON = 3, ORC_BANDED = 4 };
/* formats the stored iterate can be rounded to (round to nearest, ties to even) */
enum { ORC_STORE_F64 = 0, ORC_STORE_F32 = 1, ORC_STORE_BF16 = 2, ORC_STORE_F16 = 3 };
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

/* ---- extensions of the iteration (the page's optimisation sections) ----
 *
 * Banded Jacobian approximation (page §2.2.2): A~ keeps the entries of
 * df_t/ds with |j - k| <= band and zeroes the rest.  band = 0 is the
 * diagonal (quasi-Newton); band >= D - 1 is the full Jacobian (Newton). */
int orc_banded_jacobian(int cell, int band, int D, int d_in, const double* p,
                        double eps, const double* x_t, const double* s_prev,
                        double* A);

/* Round n values in place to a storage format (ORC_STORE_*), to nearest
 * with ties to even, overflow to +-inf, gradual underflow (IEEE 754
 * binary32 / binary16; bfloat16 = binary32's exponent range with an
 * 8-bit significand).  ORC_STORE_F64 leaves the values unchanged. */
int orc_round_storage(int store, double* v, long n);

/* orc_update with a mode that may be ORC_BANDED (with its band) and a
 * damping factor lambda in (0, 1]: s_next = s_cur + lambda * delta, where
 * delta solves J~ delta = -F(s_cur) as in orc_update (page §4.3 and §5.3
 * name damping as the remedy for a stalled iteration). */
int orc_update_ex(int cell, int mode, int band, double damping, int D,
                  int d_in, const double* p, double eps, int T, int B,
                  const double* x, const double* s0, const double* s_cur,
                  double* s_next, int nthreads);

/* The full iteration with the page's optional refinements.  With
 * band = 0, damping = 1, adapt = 0, store = ORC_STORE_F64 and window <= 0
 * it is orc_iterate.
 *
 *   mode, band   starting approximation (ORC_JACOBI..ORC_BANDED).
 *   damping      lambda in (0, 1] applied to every update.
 *   adapt, stall adaptive switching (page §5.3: when the residual curve
 *                stalls, move to a more exact Jacobian approximation).
 *                Reading: after the residual r^(i) (i >= 1) is measured,
 *                if r^(i) > stall * r^(i-1) the mode moves one rung up the
 *                ladder jacobi/picard -> quasi -> banded (only when
 *                band >= 1) -> newton before update i is taken; newton
 *                stays newton.
 *   store,       reduced-precision iterate storage (page §2.3: states kept
 *   store_until  in a narrow format, arithmetic in a wider one).  The
 *                initial guess s^(0) and the first update s^(1) are rounded
 *                to the format before they are stored, and so is every later
 *                iterate s^(i+1) while the residual known when its update
 *                starts, r^(i-1), is above store_until (the page gives no
 *                switching rule; this one can be applied by an iteration
 *                that evaluates r^(i) and writes s^(i+1) in the same pass,
 *                before r^(i) is complete).  The residual and the update are
 *                computed in double from the stored values.
 *   window       windowed solve (page §1.3.1: the long sequence is split
 *                into blocks that fit in memory; page §2.3, chunks such as
 *                1024 steps).  Reading: t = 1..T is cut into consecutive
 *                windows of `window` steps (the last one ragged); each is
 *                solved in turn by the iteration above, from the start
 *                mode, with its initial state the last state of the
 *                previous window, until its own residual max-norm <= tol or
 *                max_iters.  window <= 0 or >= T: one window.
 *
 * Results: s_out [B][T][D]; *iters = iterations summed over windows;
 * *resid = the largest final window residual, which is the max-norm of F
 * over the whole sequence; status OK when every window converged,
 * NOT_CONVERGED when one ran out of iterations (the next windows still
 * run), NONFINITE when a residual is not finite (the windows after it keep
 * their initial guess).  history[] / modes_used[] hold, window after
 * window, each measured residual and the mode of the update that followed
 * it (-1 after a window's last residual), hist_cap entries at most;
 * window_iters[w] (may be NULL) each window's count. */
int orc_iterate_ex(int cell, int mode, int band, double damping, int adapt,
                   double stall, int store, double store_until, int window,
                   int D, int d_in, const double* p, double eps, int T, int B,
                   const double* x, const double* s0, int max_iters,
                   double tol, double* s_out, int* iters, double* resid,
                   double* history, int* modes_used, int hist_cap,
                   int* window_iters, int nthreads);

/* s[t] = A[t] s[t-1] + b[t] for t = 0..T-1 with s_init before t = 0.
 * A: [T][D][D], b: [T][D], s: [T][D].  A serial loop. */
int orc_affine_recurrence(int D, int T, const double* A, const double* b,
                          const double* s_init, double* s);

#ifdef __cplusplus
}
#endif
#endif
