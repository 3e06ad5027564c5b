/*
 * oracle.c -- plain fp64 CPU oracle (TEST INFRASTRUCTURE ONLY; see
 * oracle.h for the scope, the citation convention and the readings).
 *
 * Everything is written straight from the definitions: one step at a time,
 * full D x D Jacobians, serial loops over t.  Threads only split the batch
 * (independent sequences); no blocking, fusion or reordering of the
 * arithmetic within a sequence.
 */
#include "oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* parameters                                                          */
/* ------------------------------------------------------------------ */

long orc_param_count(int cell, int D, int d_in) {
  if (D <= 0 || d_in <= 0) return -1;
  switch (cell) {
    case ORC_TANH_RNN: return (long)D * D + (long)D * d_in + D;
    case ORC_GRU: return 3L * D * d_in + 3L * D * D + 3L * D + 3L * D;
    case ORC_EULER: return d_in == D ? (long)D * D : -1;
    default: return -1;
  }
}

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/* ------------------------------------------------------------------ */
/* cells: benchmark definitions; GRU in the PyTorch gate convention     */
/* ------------------------------------------------------------------ */

/* tanh RNN: y = tanh(W s + U x + b). */
static void tanh_rnn_cell(int D, int d_in, const double* p, const double* x,
                          const double* s, double* y) {
  const double* W = p;
  const double* U = p + (long)D * D;
  const double* bias = U + (long)D * d_in;
  for (int j = 0; j < D; ++j) {
    double z = bias[j];
    for (int k = 0; k < D; ++k) z += W[(long)j * D + k] * s[k];
    for (int k = 0; k < d_in; ++k) z += U[(long)j * d_in + k] * x[k];
    y[j] = tanh(z);
  }
}

/* GRU pieces at one step: r, z, n and hn = W_hn h + b_hn. */
static void gru_gates(int D, int d_in, const double* p, const double* x,
                      const double* h, double* r, double* z, double* n,
                      double* hn) {
  const double* W_ih = p;
  const double* W_hh = W_ih + 3L * D * d_in;
  const double* b_ih = W_hh + 3L * D * D;
  const double* b_hh = b_ih + 3L * D;
  for (int j = 0; j < D; ++j) {
    double ir = b_ih[j], iz = b_ih[D + j], in = b_ih[2 * D + j];
    for (int k = 0; k < d_in; ++k) {
      ir += W_ih[(long)j * d_in + k] * x[k];
      iz += W_ih[(long)(D + j) * d_in + k] * x[k];
      in += W_ih[(long)(2 * D + j) * d_in + k] * x[k];
    }
    double hr = b_hh[j], hz = b_hh[D + j], hnj = b_hh[2 * D + j];
    for (int k = 0; k < D; ++k) {
      hr += W_hh[(long)j * D + k] * h[k];
      hz += W_hh[(long)(D + j) * D + k] * h[k];
      hnj += W_hh[(long)(2 * D + j) * D + k] * h[k];
    }
    r[j] = sigmoid(ir + hr);
    z[j] = sigmoid(iz + hz);
    hn[j] = hnj;
    n[j] = tanh(in + r[j] * hnj);
  }
}

static int gru_cell(int D, int d_in, const double* p, const double* x,
                    const double* h, double* y) {
  double* tmp = (double*)malloc(sizeof(double) * 4 * (size_t)D);
  if (!tmp) return ORC_ERR_NOMEM;
  double *r = tmp, *z = tmp + D, *n = tmp + 2 * D, *hn = tmp + 3 * D;
  gru_gates(D, d_in, p, x, h, r, z, n, hn);
  for (int j = 0; j < D; ++j) y[j] = (1.0 - z[j]) * n[j] + z[j] * h[j];
  free(tmp);
  return ORC_OK;
}

/* Euler drift: y = s + eps * tanh(W s + c). */
static void euler_cell(int D, const double* p, double eps, const double* c,
                       const double* s, double* y) {
  const double* W = p;
  for (int j = 0; j < D; ++j) {
    double g = c[j];
    for (int k = 0; k < D; ++k) g += W[(long)j * D + k] * s[k];
    y[j] = s[j] + eps * tanh(g);
  }
}

int orc_cell(int cell, int D, int d_in, const double* p, double eps,
             const double* x_t, const double* s_prev, double* y) {
  if (orc_param_count(cell, D, d_in) < 0) return ORC_ERR_INVALID;
  switch (cell) {
    case ORC_TANH_RNN: tanh_rnn_cell(D, d_in, p, x_t, s_prev, y); return ORC_OK;
    case ORC_GRU: return gru_cell(D, d_in, p, x_t, s_prev, y);
    case ORC_EULER: euler_cell(D, p, eps, x_t, s_prev, y); return ORC_OK;
  }
  return ORC_ERR_INVALID;
}

/* ------------------------------------------------------------------ */
/* exact Jacobians df/ds                                               */
/* ------------------------------------------------------------------ */

int orc_jacobian(int cell, int D, int d_in, const double* p, double eps,
                 const double* x_t, const double* s_prev, double* J) {
  if (orc_param_count(cell, D, d_in) < 0) return ORC_ERR_INVALID;
  if (cell == ORC_TANH_RNN) {
    /* d tanh(W s + U x + b)_j / d s_k = (1 - y_j^2) W[j][k] */
    double* y = (double*)malloc(sizeof(double) * (size_t)D);
    if (!y) return ORC_ERR_NOMEM;
    tanh_rnn_cell(D, d_in, p, x_t, s_prev, y);
    for (int j = 0; j < D; ++j)
      for (int k = 0; k < D; ++k)
        J[(long)j * D + k] = (1.0 - y[j] * y[j]) * p[(long)j * D + k];
    free(y);
    return ORC_OK;
  }
  if (cell == ORC_EULER) {
    /* d (s + eps tanh(g))_j / d s_k = delta_jk + eps (1 - tanh(g_j)^2) W[j][k] */
    const double* W = p;
    for (int j = 0; j < D; ++j) {
      double g = x_t[j];
      for (int k = 0; k < D; ++k) g += W[(long)j * D + k] * s_prev[k];
      double th = tanh(g);
      for (int k = 0; k < D; ++k)
        J[(long)j * D + k] = (j == k ? 1.0 : 0.0) + eps * (1.0 - th * th) * W[(long)j * D + k];
    }
    return ORC_OK;
  }
  /* GRU: h' = (1-z) n + z h
   *   dh'_j/dh_k = z_j delta_jk + (h_j - n_j) dz_j/dh_k + (1 - z_j) dn_j/dh_k
   *   dz_j/dh_k  = z_j (1 - z_j) W_hz[j][k]
   *   dr_j/dh_k  = r_j (1 - r_j) W_hr[j][k]
   *   dn_j/dh_k  = (1 - n_j^2) (r_j W_hn[j][k] + hn_j dr_j/dh_k)          */
  double* tmp = (double*)malloc(sizeof(double) * 4 * (size_t)D);
  if (!tmp) return ORC_ERR_NOMEM;
  double *r = tmp, *z = tmp + D, *n = tmp + 2 * D, *hn = tmp + 3 * D;
  gru_gates(D, d_in, p, x_t, s_prev, r, z, n, hn);
  const double* W_hh = p + 3L * D * d_in;
  const double* W_hr = W_hh;
  const double* W_hz = W_hh + (long)D * D;
  const double* W_hn = W_hh + 2L * D * D;
  for (int j = 0; j < D; ++j) {
    for (int k = 0; k < D; ++k) {
      double dz = z[j] * (1.0 - z[j]) * W_hz[(long)j * D + k];
      double dr = r[j] * (1.0 - r[j]) * W_hr[(long)j * D + k];
      double dn = (1.0 - n[j] * n[j]) * (r[j] * W_hn[(long)j * D + k] + hn[j] * dr);
      J[(long)j * D + k] = (j == k ? z[j] : 0.0) + (s_prev[j] - n[j]) * dz + (1.0 - z[j]) * dn;
    }
  }
  free(tmp);
  return ORC_OK;
}

int orc_approx_jacobian(int cell, int mode, int D, int d_in, const double* p,
                        double eps, const double* x_t, const double* s_prev,
                        double* A) {
  if (orc_param_count(cell, D, d_in) < 0) return ORC_ERR_INVALID;
  long DD = (long)D * D;
  switch (mode) {
    case ORC_JACOBI: /* J~ = I: the dynamics Jacobian is dropped (page §1.2) */
      for (long e = 0; e < DD; ++e) A[e] = 0.0;
      return ORC_OK;
    case ORC_PICARD: /* dynamics Jacobian -> identity (page §2.2.3) */
      for (long e = 0; e < DD; ++e) A[e] = 0.0;
      for (int j = 0; j < D; ++j) A[(long)j * D + j] = 1.0;
      return ORC_OK;
    case ORC_QUASI: { /* keep only the diagonal (page §2.2.1) */
      int rc = orc_jacobian(cell, D, d_in, p, eps, x_t, s_prev, A);
      if (rc) return rc;
      for (int j = 0; j < D; ++j)
        for (int k = 0; k < D; ++k)
          if (j != k) A[(long)j * D + k] = 0.0;
      return ORC_OK;
    }
    case ORC_NEWTON: /* exact Jacobian (page §1.2) */
      return orc_jacobian(cell, D, d_in, p, eps, x_t, s_prev, A);
  }
  return ORC_ERR_INVALID;
}

/* ------------------------------------------------------------------ */
/* batch-parallel drivers (threads split b only)                        */
/* ------------------------------------------------------------------ */

typedef struct {
  int cell, mode, D, d_in, T;
  const double* p;
  double eps;
  const double* x;
  const double* s0;
  const double* s_in;  /* current iterate (residual / update) */
  double* out;         /* sequential states, F, or s_next */
  const double* F;     /* precomputed residual for the update, or NULL */
  int band;            /* half-bandwidth for ORC_BANDED */
  double damping;      /* lambda of s_next = s + lambda * delta (1 = undamped) */
  int b_begin, b_end;
  double rmax;
  int rc;
} orc_job;

typedef void* (*orc_worker)(void*);

static int run_jobs(orc_worker fn, orc_job* proto, int B, int nthreads,
                    double* rmax) {
  if (nthreads <= 0) nthreads = 1;
  if (nthreads > B) nthreads = B;
  orc_job* jobs = (orc_job*)calloc((size_t)nthreads, sizeof(orc_job));
  pthread_t* tids = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
  if (!jobs || !tids) {
    free(jobs);
    free(tids);
    return ORC_ERR_NOMEM;
  }
  for (int i = 0; i < nthreads; ++i) {
    jobs[i] = *proto;
    jobs[i].b_begin = (int)((long)B * i / nthreads);
    jobs[i].b_end = (int)((long)B * (i + 1) / nthreads);
    jobs[i].rmax = 0.0;
    jobs[i].rc = ORC_OK;
  }
  int rc = ORC_OK;
  if (nthreads == 1) {
    fn(&jobs[0]);
  } else {
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
      if (pthread_create(&tids[i], NULL, fn, &jobs[i]) != 0) break;
      ++started;
    }
    for (int i = 0; i < started; ++i) pthread_join(tids[i], NULL);
    for (int i = started; i < nthreads; ++i) fn(&jobs[i]);
  }
  double r = 0.0;
  for (int i = 0; i < nthreads; ++i) {
    if (jobs[i].rc != ORC_OK) rc = jobs[i].rc;
    /* max that lets NaN win */
    if (jobs[i].rmax != jobs[i].rmax || jobs[i].rmax > r) {
      if (r == r) r = jobs[i].rmax;
    }
  }
  if (rmax) *rmax = r;
  free(jobs);
  free(tids);
  return rc;
}

static void* sequential_worker(void* arg) {
  orc_job* j = (orc_job*)arg;
  int D = j->D, T = j->T, d_in = j->d_in;
  for (int b = j->b_begin; b < j->b_end; ++b) {
    const double* prev = j->s0 + (long)b * D;
    for (int t = 0; t < T; ++t) {
      double* cur = j->out + ((long)b * T + t) * D;
      int rc = orc_cell(j->cell, D, d_in, j->p, j->eps,
                        j->x + ((long)b * T + t) * d_in, prev, cur);
      if (rc) { j->rc = rc; return NULL; }
      prev = cur;
    }
  }
  return NULL;
}

int orc_sequential(int cell, int D, int d_in, const double* p, double eps,
                   int T, int B, const double* x, const double* s0, double* s,
                   int nthreads) {
  if (orc_param_count(cell, D, d_in) < 0 || T < 0 || B < 0) return ORC_ERR_INVALID;
  if (T == 0 || B == 0) return ORC_OK;
  orc_job proto = {0};
  proto.cell = cell; proto.D = D; proto.d_in = d_in; proto.T = T;
  proto.p = p; proto.eps = eps; proto.x = x; proto.s0 = s0; proto.out = s;
  return run_jobs(sequential_worker, &proto, B, nthreads, NULL);
}

/* F_t = s_t - f_t(s_{t-1}); also the max |F_t| of the job's sequences. */
static void* residual_worker(void* arg) {
  orc_job* j = (orc_job*)arg;
  int D = j->D, T = j->T, d_in = j->d_in;
  double* y = (double*)malloc(sizeof(double) * (size_t)D);
  if (!y) { j->rc = ORC_ERR_NOMEM; return NULL; }
  double r = 0.0;
  for (int b = j->b_begin; b < j->b_end; ++b) {
    const double* prev = j->s0 + (long)b * D;
    for (int t = 0; t < T; ++t) {
      const double* cur = j->s_in + ((long)b * T + t) * D;
      int rc = orc_cell(j->cell, D, d_in, j->p, j->eps,
                        j->x + ((long)b * T + t) * d_in, prev, y);
      if (rc) { j->rc = rc; free(y); return NULL; }
      for (int k = 0; k < D; ++k) {
        double F = cur[k] - y[k];
        if (j->out) j->out[((long)b * T + t) * D + k] = F;
        double a = fabs(F);
        if (a != a) r = a;           /* NaN sticks */
        else if (r == r && a > r) r = a;
      }
      prev = cur;
    }
  }
  j->rmax = r;
  free(y);
  return NULL;
}

int orc_residual(int cell, int D, int d_in, const double* p, double eps,
                 int T, int B, const double* x, const double* s0,
                 const double* s, double* F, double* rmax, int nthreads) {
  if (orc_param_count(cell, D, d_in) < 0 || T < 0 || B < 0) return ORC_ERR_INVALID;
  if (T == 0 || B == 0) { if (rmax) *rmax = 0.0; return ORC_OK; }
  orc_job proto = {0};
  proto.cell = cell; proto.D = D; proto.d_in = d_in; proto.T = T;
  proto.p = p; proto.eps = eps; proto.x = x; proto.s0 = s0;
  proto.s_in = s; proto.out = F;
  return run_jobs(residual_worker, &proto, B, nthreads, rmax);
}

/* One update for the job's sequences:
 *   F_t = s_t - f_t(s_{t-1})   (taken from j->F when the caller has it);
 *   A~_t at s_{t-1};
 *   delta_t = A~_t delta_{t-1} - F_t  (delta before t = 0 is 0; s0 is fixed)
 *   s_next_t = s_t + delta_t
 * For jacobi (A~ = 0) and picard (A~ = I) the product A~ delta is written
 * out as 0 and delta; quasi multiplies by the diagonal; newton by the full
 * matrix. */
static void* update_worker(void* arg) {
  orc_job* j = (orc_job*)arg;
  int D = j->D, T = j->T, d_in = j->d_in;
  double* buf = (double*)malloc(sizeof(double) * ((size_t)D * D + 4 * (size_t)D));
  if (!buf) { j->rc = ORC_ERR_NOMEM; return NULL; }
  double* A = buf;
  double* y = A + (long)D * D;
  double* dprev = y + D;
  double* dcur = dprev + D;
  double* Fv = dcur + D;
  for (int b = j->b_begin; b < j->b_end; ++b) {
    const double* prev = j->s0 + (long)b * D;
    for (int k = 0; k < D; ++k) dprev[k] = 0.0;
    for (int t = 0; t < T; ++t) {
      const double* xt = j->x + ((long)b * T + t) * d_in;
      const double* cur = j->s_in + ((long)b * T + t) * D;
      int rc = ORC_OK;
      if (j->F) {
        const double* Ft = j->F + ((long)b * T + t) * D;
        for (int r = 0; r < D; ++r) Fv[r] = Ft[r];
      } else {
        rc = orc_cell(j->cell, D, d_in, j->p, j->eps, xt, prev, y);
        for (int r = 0; r < D; ++r) Fv[r] = cur[r] - y[r];
      }
      if (!rc && (j->mode == ORC_QUASI || j->mode == ORC_NEWTON))
        rc = orc_approx_jacobian(j->cell, j->mode, D, d_in, j->p, j->eps, xt, prev, A);
      else if (!rc && j->mode == ORC_BANDED)
        rc = orc_banded_jacobian(j->cell, j->band, D, d_in, j->p, j->eps, xt, prev, A);
      if (rc) { j->rc = rc; free(buf); return NULL; }
      for (int r = 0; r < D; ++r) {
        double acc;
        if (j->mode == ORC_JACOBI) {
          acc = 0.0;
        } else if (j->mode == ORC_PICARD) {
          acc = dprev[r];
        } else if (j->mode == ORC_QUASI) {
          acc = A[(long)r * D + r] * dprev[r];
        } else { /* newton, and banded with its zeros outside the band */
          acc = 0.0;
          for (int k = 0; k < D; ++k) acc += A[(long)r * D + k] * dprev[k];
        }
        dcur[r] = acc - Fv[r];
      }
      double* nxt = j->out + ((long)b * T + t) * D;
      for (int r = 0; r < D; ++r) {
        /* the recurrence runs on the full delta; damping scales only the
           step taken (lambda * delta solves J~ v = -lambda F) */
        nxt[r] = cur[r] + j->damping * dcur[r];
        dprev[r] = dcur[r];
      }
      prev = cur;
    }
  }
  free(buf);
  return NULL;
}

int orc_update(int cell, int mode, int D, int d_in, const double* p,
               double eps, int T, int B, const double* x, const double* s0,
               const double* s_cur, double* s_next, int nthreads) {
  if (orc_param_count(cell, D, d_in) < 0 || T < 0 || B < 0) return ORC_ERR_INVALID;
  if (mode < ORC_JACOBI || mode > ORC_NEWTON) return ORC_ERR_INVALID;
  if (T == 0 || B == 0) return ORC_OK;
  orc_job proto = {0};
  proto.cell = cell; proto.mode = mode; proto.D = D; proto.d_in = d_in;
  proto.T = T; proto.p = p; proto.eps = eps; proto.x = x; proto.s0 = s0;
  proto.s_in = s_cur; proto.out = s_next; proto.damping = 1.0;
  return run_jobs(update_worker, &proto, B, nthreads, NULL);
}

static int iterate_block(int cell, int mode, int band, double damping,
                         int adapt, double stall, int store,
                         double store_until, int D, int d_in, const double* p,
                         double eps, int T, int B, const double* x,
                         const double* s0, int max_iters, double tol,
                         double* s_out, int* iters, double* resid,
                         double* history, int* modes, int hist_cap,
                         int nthreads);

/* The plain iteration is the general loop below (iterate_block) with every
 * refinement off: no band, no damping, no switching, double storage. */
int orc_iterate(int cell, int mode, int D, int d_in, const double* p,
                double eps, int T, int B, const double* x, const double* s0,
                int max_iters, double tol, double* s_out, int* iters,
                double* resid, double* history, int hist_cap, int nthreads) {
  if (orc_param_count(cell, D, d_in) < 0 || T < 0 || B < 0) return ORC_ERR_INVALID;
  if (mode < ORC_JACOBI || mode > ORC_NEWTON) return ORC_ERR_INVALID;
  if (max_iters < 0 || !(tol >= 0.0)) return ORC_ERR_INVALID;
  int it = 0;
  double r = 0.0;
  int st = iterate_block(cell, mode, 0, 1.0, 0, 0.0, ORC_STORE_F64, 0.0, D, d_in, p, eps, T, B, x, s0,
                         max_iters, tol, s_out, &it, &r, history, NULL, hist_cap < 0 ? 0 : hist_cap, nthreads);
  if (st == ORC_ERR_INVALID || st == ORC_ERR_NOMEM) return st;
  if (iters) *iters = it;
  if (resid) *resid = r;
  return st;
}

int orc_affine_recurrence(int D, int T, const double* A, const double* b,
                          const double* s_init, double* s) {
  if (D <= 0 || T < 0) return ORC_ERR_INVALID;
  const double* prev = s_init;
  for (int t = 0; t < T; ++t) {
    const double* At = A + (long)t * D * D;
    double* cur = s + (long)t * D;
    for (int r = 0; r < D; ++r) {
      double acc = b[(long)t * D + r];
      for (int k = 0; k < D; ++k) acc += At[(long)r * D + k] * prev[k];
      cur[r] = acc;
    }
    prev = cur;
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* extensions: banded Jacobian, storage rounding, damping, adaptive     */
/* switching, windowed solve (declarations and readings in oracle.h)    */
/* ------------------------------------------------------------------ */

int orc_banded_jacobian(int cell, int band, int D, int d_in, const double* p,
                        double eps, const double* x_t, const double* s_prev,
                        double* A) {
  if (band < 0) return ORC_ERR_INVALID;
  int rc = orc_jacobian(cell, D, d_in, p, eps, x_t, s_prev, A);
  if (rc) return rc;
  for (int j = 0; j < D; ++j)
    for (int k = 0; k < D; ++k)
      if (abs(j - k) > band) A[(long)j * D + k] = 0.0;
  return ORC_OK;
}

/* Nearest value of a binary format with `prec` significand bits (the
 * leading one included) and normal exponents emin..emax, ties to even.
 * Below 2^emin the spacing stays 2^(emin - prec + 1) (gradual underflow);
 * a rounded magnitude above the largest finite value becomes infinite. */
static double round_to_format(double v, int prec, int emin, int emax) {
  if (v == 0.0 || !isfinite(v)) return v;
  int e;
  (void)frexp(v, &e);            /* |v| in [2^(e-1), 2^e) */
  int lead = e - 1;              /* exponent of v's leading bit */
  if (lead < emin) lead = emin;
  /* scale so that one unit in the last place of the format is 1; the
     scaling by a power of two is exact, nearbyint rounds ties to even in
     the default rounding mode */
  double q = nearbyint(ldexp(v, prec - 1 - lead));
  double r = ldexp(q, lead - (prec - 1));
  double maxv = ldexp(2.0 - ldexp(1.0, 1 - prec), emax);
  if (fabs(r) > maxv) return copysign(INFINITY, v);
  return r;
}

int orc_round_storage(int store, double* v, long n) {
  int prec, emin, emax;
  switch (store) {
    case ORC_STORE_F64: return ORC_OK;
    case ORC_STORE_F32: prec = 24; emin = -126; emax = 127; break;
    case ORC_STORE_BF16: prec = 8; emin = -126; emax = 127; break;
    case ORC_STORE_F16: prec = 11; emin = -14; emax = 15; break;
    default: return ORC_ERR_INVALID;
  }
  for (long i = 0; i < n; ++i) v[i] = round_to_format(v[i], prec, emin, emax);
  return ORC_OK;
}

static int mode_valid(int mode, int band) {
  if (mode == ORC_BANDED) return band >= 0;
  return mode >= ORC_JACOBI && mode <= ORC_NEWTON;
}

int orc_update_ex(int cell, int mode, int band, double damping, int D,
                  int d_in, const double* p, double eps, int T, int B,
                  const double* x, const double* s0, const double* s_cur,
                  double* s_next, int nthreads) {
  if (orc_param_count(cell, D, d_in) < 0 || T < 0 || B < 0) return ORC_ERR_INVALID;
  if (!mode_valid(mode, band) || !(damping > 0.0 && damping <= 1.0)) return ORC_ERR_INVALID;
  if (T == 0 || B == 0) return ORC_OK;
  orc_job proto = {0};
  proto.cell = cell; proto.mode = mode; proto.D = D; proto.d_in = d_in;
  proto.T = T; proto.p = p; proto.eps = eps; proto.x = x; proto.s0 = s0;
  proto.s_in = s_cur; proto.out = s_next; proto.band = band; proto.damping = damping;
  return run_jobs(update_worker, &proto, B, nthreads, NULL);
}

/* One rung up the ladder of Jacobian approximations (adaptive switching). */
static int stronger_mode(int mode, int band) {
  switch (mode) {
    case ORC_JACOBI:
    case ORC_PICARD: return ORC_QUASI;
    case ORC_QUASI: return band >= 1 ? ORC_BANDED : ORC_NEWTON;
    default: return ORC_NEWTON;
  }
}

/* The iteration over one block of contiguous sequences [B][T]: orc_iterate
 * with the damping, adaptive switching and storage rounding of
 * orc_iterate_ex.  history / modes receive at most hist_cap entries. */
static int iterate_block(int cell, int mode, int band, double damping,
                         int adapt, double stall, int store,
                         double store_until, int D, int d_in, const double* p,
                         double eps, int T, int B, const double* x,
                         const double* s0, int max_iters, double tol,
                         double* s_out, int* iters, double* resid,
                         double* history, int* modes, int hist_cap,
                         int nthreads) {
  size_t n = (size_t)B * (size_t)T * (size_t)D;
  double* other = (double*)malloc(sizeof(double) * (n ? n : 1));
  double* F = (double*)malloc(sizeof(double) * (n ? n : 1));
  if (!other || !F) { free(other); free(F); return ORC_ERR_NOMEM; }
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < T; ++t)
      memcpy(s_out + ((size_t)b * T + t) * D, s0 + (size_t)b * D, sizeof(double) * (size_t)D);
  orc_round_storage(store, s_out, (long)n);   /* the initial guess is stored too */
  double* cur = s_out;
  double* nxt = other;
  int status = ORC_NOT_CONVERGED;
  int i = 0;
  double r = 0.0, r_prev = 0.0;
  /* the residual known when update i starts: r^(i-1), none (+inf) before update 0 */
  double r_known = INFINITY;
  for (;; ++i) {
    int rc = orc_residual(cell, D, d_in, p, eps, T, B, x, s0, cur, F, &r, nthreads);
    if (rc) { free(other); free(F); return rc; }
    if (i < hist_cap) {
      if (history) history[i] = r;
      if (modes) modes[i] = -1;
    }
    if (!isfinite(r)) { status = ORC_ERR_NONFINITE; break; }
    if (r <= tol) { status = ORC_OK; break; }
    if (i >= max_iters) { status = ORC_NOT_CONVERGED; break; }
    if (adapt && i >= 1 && r > stall * r_prev) mode = stronger_mode(mode, band);
    if (modes && i < hist_cap) modes[i] = mode;
    {
      orc_job proto = {0};
      proto.cell = cell; proto.mode = mode; proto.D = D; proto.d_in = d_in;
      proto.T = T; proto.p = p; proto.eps = eps; proto.x = x; proto.s0 = s0;
      proto.s_in = cur; proto.out = nxt; proto.F = F;
      proto.band = band; proto.damping = damping;
      rc = run_jobs(update_worker, &proto, B, nthreads, NULL);
    }
    if (rc) { free(other); free(F); return rc; }
    if (r_known > store_until) orc_round_storage(store, nxt, (long)n);
    double* tmp = cur; cur = nxt; nxt = tmp;
    r_prev = r;
    r_known = r;
  }
  if (cur != s_out) memcpy(s_out, cur, sizeof(double) * n);
  free(other);
  free(F);
  *iters = i;
  *resid = r;
  return status;
}

int orc_iterate_ex(int cell, int mode, int band, double damping, int adapt,
                   double stall, int store, double store_until, int window,
                   int D, int d_in, const double* p, double eps, int T, int B,
                   const double* x, const double* s0, int max_iters,
                   double tol, double* s_out, int* iters, double* resid,
                   double* history, int* modes_used, int hist_cap,
                   int* window_iters, int nthreads) {
  if (orc_param_count(cell, D, d_in) < 0 || T < 0 || B < 0) return ORC_ERR_INVALID;
  if (!mode_valid(mode, band) || !(damping > 0.0 && damping <= 1.0)) return ORC_ERR_INVALID;
  if (max_iters < 0 || !(tol >= 0.0) || (adapt && !(stall >= 0.0))) return ORC_ERR_INVALID;
  if (store < ORC_STORE_F64 || store > ORC_STORE_F16 || store_until != store_until) return ORC_ERR_INVALID;
  if (hist_cap < 0) hist_cap = 0;
  int Wn = (window <= 0 || window >= T) ? T : window;
  int nwin = T == 0 ? 0 : (T + Wn - 1) / Wn;
  size_t xw_n = (size_t)B * Wn * d_in, sw_n = (size_t)B * Wn * D, s0_n = (size_t)B * D;
  double* xw = (double*)malloc(sizeof(double) * (xw_n ? xw_n : 1));
  double* sw = (double*)malloc(sizeof(double) * (sw_n ? sw_n : 1));
  double* s0w = (double*)malloc(sizeof(double) * (s0_n ? s0_n : 1));
  if (!xw || !sw || !s0w) { free(xw); free(sw); free(s0w); return ORC_ERR_NOMEM; }
  int status = ORC_OK, total = 0, hpos = 0;
  double rmax = 0.0;
  for (int w = 0; w < nwin; ++w) {
    int t0 = w * Wn;
    int L = T - t0 < Wn ? T - t0 : Wn;
    for (int b = 0; b < B; ++b) {
      memcpy(xw + (size_t)b * L * d_in, x + ((size_t)b * T + t0) * d_in, sizeof(double) * (size_t)L * d_in);
      const double* init = w == 0 ? s0 + (size_t)b * D : s_out + ((size_t)b * T + t0 - 1) * D;
      memcpy(s0w + (size_t)b * D, init, sizeof(double) * (size_t)D);
    }
    if (status == ORC_ERR_NONFINITE) {
      /* an earlier window failed: this one keeps its initial guess */
      for (int b = 0; b < B; ++b)
        for (int t = 0; t < L; ++t)
          memcpy(s_out + ((size_t)b * T + t0 + t) * D, s0w + (size_t)b * D, sizeof(double) * (size_t)D);
      if (window_iters) window_iters[w] = 0;
      continue;
    }
    int it = 0;
    double r = 0.0;
    int st = iterate_block(cell, mode, band, damping, adapt, stall, store, store_until, D,
                           d_in, p, eps, L, B, xw, s0w, max_iters, tol, sw, &it, &r,
                           history ? history + hpos : NULL, modes_used ? modes_used + hpos : NULL,
                           hist_cap - hpos, nthreads);
    if (st == ORC_ERR_INVALID || st == ORC_ERR_NOMEM) { free(xw); free(sw); free(s0w); return st; }
    for (int b = 0; b < B; ++b)
      memcpy(s_out + ((size_t)b * T + t0) * D, sw + (size_t)b * L * D, sizeof(double) * (size_t)L * D);
    if (window_iters) window_iters[w] = it;
    hpos += (it + 1 < hist_cap - hpos) ? it + 1 : hist_cap - hpos;
    total += it;
    if (r != r) rmax = r;                 /* NaN sticks */
    else if (rmax == rmax && r > rmax) rmax = r;
    if (st == ORC_ERR_NONFINITE) status = ORC_ERR_NONFINITE;
    else if (st == ORC_NOT_CONVERGED && status == ORC_OK) status = ORC_NOT_CONVERGED;
  }
  free(xw);
  free(sw);
  free(s0w);
  *iters = total;
  *resid = rmax;
  return status;
}
