/*
 * pn.h -- C ABI of libpn: parallel Newton evaluation of nonlinear sequences
 * on one NVIDIA B200 (sm_100a).
 *
 * The problem (web article "并行牛顿方法：加速非线性序列评估的计算革命",
 * "Parallel Newton methods for nonlinear sequence evaluation", jsqmd.com news
 * item 789890; cited below as "page §X"):
 *   given s0 and f_1..f_T, compute every state s_t = f_t(s_{t-1})   (§1.1)
 * by the fixed-point iteration s^(i+1) = s^(i) - J~^{-1}(s^(i)) F(s^(i))
 * (§1.2), where F_t(s) = s_t - f_t(s_{t-1}) and J~ = I - subdiag(A~_t):
 *   PN_JACOBI  A~_t = 0                      (J~ ~ I, §1.2)
 *   PN_PICARD  A~_t = I                      (identity approximation, §2.2.3)
 *   PN_QUASI   A~_t = diag(df_t/ds)          (diagonal approximation, §2.2.1)
 *   PN_NEWTON  A~_t = df_t/ds, dense D x D   (exact Jacobian, §1.2)
 * Each iteration evaluates f_t and A~_t at all t in parallel and then solves
 * the linear recurrence s^(i+1)_t = A~_t s^(i+1)_{t-1} + (f_t(s^(i)_{t-1}) -
 * A~_t s^(i)_{t-1}) with a parallel scan (§2.1).  The loop stops at the first
 * i whose residual r^(i) = max_{b,t,d} |F_t(s^(i))| satisfies r^(i) <= tol,
 * or at i == max_iters (residual monitoring, §5.3; the infinity norm over the
 * whole batch and the "<=" tie-break are this library's reading).  The
 * initial guess is s^(0)_t = s0 for every t.
 *
 * Conventions for every entry point:
 *  - All tensors are row-major float32.  x is [B][T][d_in], s0 is [B][D],
 *    states is [B][T][D] (channels innermost).
 *  - "device" pointers must be CUDA device (or managed) memory of the device
 *    that was current at pn_create; "host" pointers are ordinary or pinned
 *    host memory.  The caller owns every pointer it passes; the library never
 *    frees or retains them past the call.
 *  - Work is ordered on the handle's stream (set at pn_create or with
 *    pn_set_stream).  Every evaluation entry point (pn_eval, pn_eval_host,
 *    pn_eval_host_many, pn_eval_windowed, pn_eval_static) synchronises that
 *    stream before returning, so every output is complete on return.
 *  - Errors are reported by the return code; pn_last_error gives the text.
 *    A handle is not thread-safe: one call at a time per handle.
 */
#ifndef PN_H
#define PN_H

#include <stddef.h>

#if defined(__GNUC__)
#define PN_API __attribute__((visibility("default")))
#else
#define PN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pn_ctx* pn_handle;

typedef enum {
  PN_OK = 0,              /* converged: r^(iters) <= tol                         */
  PN_NOT_CONVERGED = 1,   /* soft: iters == max_iters and r > tol; outputs valid */
  PN_ERR_INVALID = -1,    /* bad argument; nothing was launched                  */
  PN_ERR_NOMEM = -2,      /* device or pinned-host allocation failed             */
  PN_ERR_CUDA = -3,       /* a CUDA runtime call failed (text in pn_last_error)  */
  PN_ERR_NONFINITE = -4,  /* r^(i) was NaN or Inf; states hold that s^(i)        */
  PN_ERR_TIMEOUT = -5     /* a bounded device wait gave up; states are invalid   */
} pn_status;

typedef enum {
  PN_CELL_TANH_RNN = 0,   /* f_t(s) = tanh(W s + U x_t + b)                       */
  PN_CELL_GRU = 1,        /* GRU, gates r, z, n (PyTorch convention)              */
  PN_CELL_EULER_TANH = 2  /* f_t(s) = s + eps * tanh(W s + c_t), c_t = x_t, d_in=D */
} pn_cell;

typedef enum { PN_JACOBI = 0, PN_PICARD = 1, PN_QUASI = 2, PN_NEWTON = 3 } pn_mode;

typedef enum {
  /* Bound, in nanoseconds, on every device-side spin wait of the chunked scan
   * (default 1e9).  When it runs out the iteration stops with PN_ERR_TIMEOUT. */
  PN_OPT_WAIT_TIMEOUT_NS = 0,
  /* Test hook: the scan tile with this ticket number never publishes its
   * result, so its successors' bounded waits run out (-1 = off, default). */
  PN_OPT_DEBUG_STALL_TICKET = 1,
  /* 1 (default): the convergence loop runs on the device inside a CUDA graph
   * (conditional WHILE node); 0: the host launches one iteration at a time and
   * reads the stop decision back after each. */
  PN_OPT_DEVICE_LOOP = 2,
  /* 1 (default where available): the diagonal-mode kernels form the cell's
   * recurrent matvec on the tensor cores (3 TF32 passes, fp32-level accuracy;
   * D = 32, or D = 64 for the tanh RNN and Euler cells); 0: FP32 FMA. */
  PN_OPT_TENSOR_CORES = 3,
  /* PN_NEWTON with a banded Jacobian approximation (page §2.2.2, banded
   * structure of locally connected systems): k >= 0 keeps the entries of
   * df_t/ds with |row - col| <= k (k = 0 is the diagonal, as PN_QUASI;
   * k >= D - 1 the exact Jacobian); -1 (default) the exact Jacobian.  At
   * D <= 32 the in-chunk products run over the band only (4 + 2k columns
   * instead of D); the aggregates that cross chunks stay dense, since
   * products of banded matrices fill in. */
  PN_OPT_NEWTON_BAND = 4,
  /* Consecutive scan chunks one ticket of the Newton kernels at D <= 32
   * covers (a run: one aggregate per run in the look-back, the cell phase
   * evaluated twice per chunk when the run is longer than one): 0 (default)
   * chooses one run per resident warp where the work allows, n >= 1 fixes
   * it (capped at the chunks of a sequence).  Other kernels ignore it. */
  PN_OPT_RUN_LENGTH = 5,
  /* 1 (default): PN_NEWTON at D <= 8, when the problem's step inputs,
   * iterate, Jacobian coefficients and chunk aggregates fit in one SM's
   * shared memory (about B*T <= 3000 at D = 4 for the one-gate cells), runs
   * the whole solve -- projection, every iteration with its stop rule, the
   * result copy -- in one launch of one CTA, with the scan's chunk hand-off
   * in shared memory; 0: the multi-CTA kernels.  Used only with the device
   * loop and without adaptive switching. */
  PN_OPT_SMALL_SOLVE = 6
} pn_option;

/* Per-handle counters, cumulative since pn_create (or pn_reset_stats). */
typedef struct {
  long long iteration_launches;  /* fused iteration kernels launched           */
  long long iteration_ns;        /* their summed device durations (first CTA
                                    start to last CTA end, %globaltimer)       */
  long long evals;               /* completed evaluations: one per pn_eval or
                                    pn_eval_host call, per batch of
                                    pn_eval_host_many, per window of
                                    pn_eval_windowed                            */
} pn_stats;

/* Supported sizes: 1 <= D <= 256 for PN_JACOBI/PN_PICARD/PN_QUASI and
 * 1 <= D <= 64 for PN_NEWTON; d_in >= 1 (d_in == D for the Euler cell);
 * T >= 1, B >= 1, B*T*max(D,d_in)*4 bytes must fit in device memory. */
#define PN_MAX_D_DIAG 256
#define PN_MAX_D_NEWTON 64

/* Create a solver for one cell and one problem shape.
 *   params   host, float32, n_params entries, copied to the device (the caller
 *            keeps ownership).  Packing, row-major:
 *              tanh RNN : W[D][D], U[D][d_in], b[D]
 *              GRU      : W_ih[3D][d_in], W_hh[3D][D], b_ih[3D], b_hh[3D]
 *              Euler    : W[D][D]
 *   eps      Euler step (ignored by the other cells).
 *   cuda_stream  a cudaStream_t (NULL = the legacy default stream).
 * Allocates every work buffer for (D, d_in, T, B) up front.  On error *out is
 * set to NULL and the message is available from pn_last_error(NULL). */
PN_API pn_status pn_create(pn_handle* out, pn_cell cell, int D, int d_in, int T, int B,
                    const float* params, size_t n_params, float eps,
                    void* cuda_stream);

/* Evaluate all states.
 *   x       device [B][T][d_in]  (Euler: c_t, d_in == D)
 *   s0      device [B][D]
 *   mode    iteration, see pn_mode
 *   max_iters  >= 0; at most this many updates are applied
 *   tol     >= 0 and finite
 *   states  device [B][T][D], written with s^(iters); also used as one of
 *           the two iterate buffers while the call runs
 *   iters_out, resid_out  host; receive the iteration count and r^(iters)
 *           (either may be NULL)
 * Returns PN_OK, PN_NOT_CONVERGED, or an error (see pn_status). */
PN_API pn_status pn_eval(pn_handle h, const float* x, const float* s0, pn_mode mode,
                  int max_iters, float tol, float* states, int* iters_out,
                  float* resid_out);

/* pn_eval with HOST buffers: copies x and s0 to library-owned device buffers,
 * evaluates, and copies the states back into states_host, all on the handle's
 * stream (pinned host memory makes the copies asynchronous).  The device
 * buffers are allocated on the first call and reused. */
PN_API pn_status pn_eval_host(pn_handle h, const float* x_host, const float* s0_host,
                       pn_mode mode, int max_iters, float tol,
                       float* states_host, int* iters_out, float* resid_out);

/* pn_eval_host over n independent batches in a pipeline: batch k+1's inputs
 * are copied in while batch k is evaluated and batch k-1's states are copied
 * out, on two internal copy streams ordered against the handle's stream by
 * events, through two device staging slots (allocated on the first call,
 * 2 x (x, s0, states) of this handle's shapes).  x_host[k], s0_host[k] and
 * states_host[k] are batch k's host buffers (pinned memory lets the copies
 * overlap; states_host may repeat a buffer only for batches whose results
 * are not kept); iters_out[k] and resid_out[k] (arrays of n, either may be
 * NULL) receive each batch's count and final residual.  Every batch gives
 * the same result pn_eval_host gives for it.  Returns the first error, else
 * PN_NOT_CONVERGED if any batch did not converge, else PN_OK; the call is
 * complete (all copies done) on return. */
PN_API pn_status pn_eval_host_many(pn_handle h, int n, const float* const* x_host,
                                   const float* const* s0_host, pn_mode mode, int max_iters,
                                   float tol, float* const* states_host, int* iters_out,
                                   float* resid_out);

/* Windowed solve of a sequence longer than the handle (web article "并行牛顿
 * 方法：加速非线性序列评估的计算革命", §1.3.1, the long sequence split into
 * blocks that fit in memory, and §2.3, chunked computation).  Steps
 * t = 1..T_total are cut into consecutive windows of W = h's T steps; each
 * window is solved in turn by pn_eval's iteration, with the previous
 * window's last state as its s0 and its own stop rule (residual max-norm
 * over the window and the batch <= tol, or max_iters), so the result is the
 * windowed result of the oracle's orc_iterate_ex.
 *   h        handle; its T is the window length W
 *   tail     handle for the last window when W does not divide T_total: same
 *            cell, D, d_in, B, eps, device, stream and PARAMETERS as h (the
 *            parameters cannot be checked: the caller's responsibility),
 *            T = T_total mod W; must be NULL when W divides T_total
 *   T_total  >= 1
 *   x        device [B][T_total][d_in];  s0 device [B][D]
 *   states   device [B][T_total][D], written window by window
 *   iters_out     host; the iterations summed over the windows (may be NULL)
 *   resid_out     host; the largest final window residual, which is the
 *                 residual max-norm over the whole sequence (may be NULL)
 *   window_iters  host array of n_window_cap ints (may be NULL); receives
 *                 each window's count, in order, as far as it reaches
 * Each window's x slice and initial state are staged with strided device
 * copies into h's host-evaluation buffers (allocated on first use, as for
 * pn_eval_host), and its states are copied back, all on h's stream.
 * Returns PN_OK when every window converged; PN_NOT_CONVERGED when some
 * window used up max_iters (the windows after it still run); the first
 * error otherwise: PN_ERR_NONFINITE leaves the windows after the failing
 * one unwritten.  Afterwards pn_get_residual_history on h (or tail) reports
 * the last window that handle solved. */
PN_API pn_status pn_eval_windowed(pn_handle h, pn_handle tail, int T_total, const float* x,
                                  const float* s0, pn_mode mode, int max_iters, float tol,
                                  float* states, int* iters_out, float* resid_out,
                                  int* window_iters, int n_window_cap);

/* Copy min(n, iters+1, 65537) residuals r^(0..) of the handle's last
 * evaluation into the host array out (n >= 0 entries; may be NULL when
 * n == 0); *n_written (may be NULL) receives the count, 0 before the first
 * evaluation.  PN_ERR_INVALID for a NULL handle or a bad array. */
PN_API pn_status pn_get_residual_history(pn_handle h, float* out, int n, int* n_written);

/* Time the fused iteration kernel of `mode` alone: after a pn_eval on this
 * handle (its x, s0 and states must still be valid), run exactly n_launches
 * iterations on the handle's stream with no stop rule, bracketed by CUDA
 * events, and return the mean time per iteration in *avg_ms.  Kernels that
 * launch once per iteration are launched n_launches times back to back;
 * kernels that loop over iterations on the device (the quasi-Newton
 * tensor-core kernel of the one-gate cells) run one launch of n_launches
 * iterations, as in pn_eval.  The states buffer of that pn_eval is
 * overwritten with later iterates. */
PN_API pn_status pn_time_iterations(pn_handle h, pn_mode mode, int n_launches, float* avg_ms);

/* Fill *out (host) with the handle's counters; synchronises the handle's
 * stream first.  PN_ERR_INVALID for a NULL handle or out. */
PN_API pn_status pn_get_stats(pn_handle h, pn_stats* out);

/* Zero the handle's counters (after synchronising its stream). */
PN_API pn_status pn_reset_stats(pn_handle h);

/* Set one pn_option.  Values: PN_OPT_WAIT_TIMEOUT_NS >= 1000;
 * PN_OPT_DEBUG_STALL_TICKET -1 or a ticket >= 0; PN_OPT_NEWTON_BAND -1 or a
 * half-bandwidth >= 0; PN_OPT_RUN_LENGTH >= 0; PN_OPT_SMALL_SOLVE, PN_OPT_DEVICE_LOOP and
 * PN_OPT_TENSOR_CORES 0 or 1 (tensor cores, 3xTF32: the matvec kernels of the
 * diagonal modes, the Newton compositions at padded width 16, 32 and 64; 0 runs
 * the FP32 kernels; ignored where the shape has no tensor-core kernel;
 * switching re-selects the kernels after synchronising the stream).  Anything else: PN_ERR_INVALID, the handle unchanged. */
PN_API pn_status pn_set_option(pn_handle h, pn_option opt, long long value);

/* Adaptive switching (page §5.3: when the residual curve stalls, switch to
 * a more exact Jacobian approximation).  With stall >= 0, later evaluations
 * move one rung up the ladder jacobi/picard -> quasi -> newton (newton only
 * where this handle supports it) whenever r^(i) > stall * r^(i-1), i >= 1,
 * before update i is applied: iteration i runs again in the stronger mode.
 * With the device loop (PN_OPT_DEVICE_LOOP = 1, the default) the rule runs
 * on the device: a CUDA graph holds one conditional IF node per mode inside
 * its WHILE node, and the last CTA of each iteration turns on the node of the
 * mode the next iteration runs in.  With PN_OPT_DEVICE_LOOP = 0 the host
 * applies it, one launch per iteration.  stall < 0 switches it off
 * (default).  A NaN or infinite stall is PN_ERR_INVALID. */
PN_API pn_status pn_set_adaptive(pn_handle h, float stall);

/* The mode of each update of the handle's last evaluation (out[i] for update
 * i, i < iters), n entries at most; *n_written (may be NULL) receives the
 * count.  Empty unless that evaluation ran with adaptive switching. */
PN_API pn_status pn_get_mode_history(pn_handle h, int* out, int n, int* n_written);

/* Damping (page §4.3 and §5.3: a damping factor for an iteration that does
 * not converge): later evaluations store s^(i+1) = s^(i) + lambda * delta,
 * delta the undamped update, 0 < lambda <= 1 (1, the default, is undamped),
 * in every mode (PN_NEWTON with or without PN_OPT_NEWTON_BAND).  The scan
 * that solves for delta is unchanged; only the stored iterate moves lambda of
 * the way.  While lambda < 1, Picard and the GRU's quasi-Newton run on the
 * FP32 kernels instead of the tensor-core ones.  A lambda outside (0, 1] is
 * PN_ERR_INVALID, the handle unchanged. */
PN_API pn_status pn_set_damping(pn_handle h, float lambda);

/* Iterate storage formats for pn_set_storage. */
typedef enum { PN_STORE_F32 = 0, PN_STORE_BF16 = 1, PN_STORE_F16 = 2 } pn_store;

/* Reduced-precision iterate storage (page §2.3: intermediate states kept in
 * FP16, the key computation in FP32; page §4.2 and §4.3: lower the precision
 * of intermediate states).  With format PN_STORE_BF16 or PN_STORE_F16, later
 * evaluations store the iterate in that 16-bit format (round to nearest, ties
 * to even) while the residual known when an update starts, r^(i-1), is above
 * store_until -- the initial guess s^(0) and the first update s^(1) always --
 * and in float32 afterwards; every cell, Jacobian, residual and scan step
 * still computes in float32 from the stored values.  A narrow iterate takes
 * the first half of its float32 buffer, so each narrow iteration reads and
 * writes half the state bytes.  The result is returned as float32 whatever
 * its storage.  Stored narrow throughout (store_until = 0: every residual
 * is above it), the residual stalls at the format's resolution (about 2^-9
 * of max|s| for bfloat16, 2^-12 for float16), so store_until must sit above
 * that floor and tol may then go below it.
 * PN_STORE_F32 (default) stores float32 throughout.  While a narrow format
 * is set the evaluations run on the FP32-FMA kernels.  An unknown format or
 * a NaN store_until is PN_ERR_INVALID, the handle unchanged. */
PN_API pn_status pn_set_storage(pn_handle h, int format, float store_until);

/* Order the handle's later work on cuda_stream (a cudaStream_t; NULL = the
 * legacy default stream).  The caller keeps the stream alive while the handle
 * uses it and orders it against earlier work itself. */
PN_API pn_status pn_set_stream(pn_handle h, void* cuda_stream);

/* pn_eval without allocation, for the tanh RNN cell and the diagonal modes.
 * (An addition of this library; the paper has no counterpart.)
 *
 * For callers that cannot call cudaMalloc once they are running -- a loop with
 * its device memory budget fixed at start-up, code whose device memory belongs
 * to another framework's allocator, a plug-in that may not grow its footprint:
 * pn_create allocates its work buffers, this call does not.  All of its scratch
 * (second iterate buffer, projected inputs, packed weights, scan descriptors,
 * control block, residual history) lives in one fixed 24 MiB device array that
 * every device loading the library holds until the process exits.
 *   params  host, tanh RNN packing W[D][D], U[D][d_in], b[D] (n_params entries)
 *   x, s0, states, mode, max_iters, tol, iters_out, resid_out: as in pn_eval
 *           (device pointers, 16-byte aligned; mode jacobi, picard or quasi)
 *   cuda_stream  the stream the work is ordered on; the call synchronises it.
 * Limits: 1 <= D <= 64, d_in <= 1024, and the scratch of the shape must fit in
 * 24 MiB (about B*T*D <= 2.9 million at D = 64); larger shapes return
 * PN_ERR_INVALID with the needed size in pn_last_error(NULL), which also holds
 * the text of every other error of this call.
 * The first call on each device looks up the array's device address (with that
 * device current).  Every call clears the look-back flags it will use, reuses
 * the same array and leaves its contents behind: calls that overlap on the GPU
 * (other threads, other streams) race and corrupt each other.  The loop runs
 * from the host, one kernel launch per iteration, with the control block read
 * back after each. */
PN_API pn_status pn_eval_static(const float* params, size_t n_params, int D, int d_in, int T, int B,
                                const float* x, const float* s0, pn_mode mode, int max_iters, float tol,
                                float* states, int* iters_out, float* resid_out, void* cuda_stream);

/* Evaluate the activations the cell kernels use, element-wise, on device
 * arrays: which = 0 gives tanh(x), 1 gives 1 / (1 + exp(-x)).  x and y are
 * device float32 arrays of n elements (they may alias); the work is ordered
 * on cuda_stream and the call synchronises it.  For accuracy tests. */
PN_API pn_status pn_activation(int which, const float* x, float* y, long long n, void* cuda_stream);

/* Shape queries (for the binding); each returns -1 for a NULL handle.
 * which = 0..4: D, d_in, T, B, cell.  which = 5 + mode: 1 when that mode's
 * iteration kernel loops over the iterations on the device (one launch per
 * evaluation, between the projection and the result copy), 2 when one
 * single-CTA launch runs the whole evaluation (PN_OPT_SMALL_SOLVE), 0 when
 * pn_eval launches the iteration kernel once per iteration. */
PN_API int pn_dim(pn_handle h, int which);

/* Last error message of this handle; with h NULL, the calling thread's last
 * error that had no handle to go to (pn_create, pn_eval_static,
 * pn_activation, or any call given a NULL handle).  Never NULL; "" when there
 * was no error. */
PN_API const char* pn_last_error(pn_handle h);

/* Release every device and host resource of the handle (NULL is a no-op). */
PN_API void pn_destroy(pn_handle h);

/* Library version string. */
PN_API const char* pn_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PN_H */
