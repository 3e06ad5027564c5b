// pn_small.cuh -- the whole Newton solve of a small problem in one CTA.
//
// The iteration is the page's unified update with J~ = J ("Parallel Newton
// methods..." page, §1.2), or its banded approximation (§2.2.2):
//     s^(i+1)_t = A_t s^(i+1)_{t-1} + b_t,  A_t = df_t/ds(s^(i)_{t-1}),
//     b_t = f_t(s^(i)_{t-1}) - A_t s^(i)_{t-1},
// solved by the chunked affine scan of §2.1.  When every array of the problem
// fits in one SM's shared memory (D <= 8 and a few thousand steps), one CTA
// runs the input projection, the initial guess, every iteration with its stop
// rule, and the result copy in a single launch: no graph, no look-back through
// global memory, no grid barrier.  Each iteration is three block-wide phases:
//   1. one thread per (b, t, channel): y = f_t(s^(i)_{t-1}), the Jacobian's
//      coefficient vectors (A_t = diag(c0) + sum_q diag(c_q) W_q), b_t and
//      |F_t|; the block's max is r^(i), which decides the stop;
//   2. one thread per (32-step chunk, column j of [P | q]): the column of the
//      chunk's aggregate, the product of its A_t applied to e_j (P) or the
//      chunk's response to a zero entering state (q), held in registers step
//      after step -- the columns of an affine product evolve independently;
//   3. one thread per sequence folds the aggregates chunk after chunk into
//      each chunk's entering state (starting from s0); then one thread per
//      chunk applies s_t = A_t s_{t-1} + b_t step by step in registers and
//      stores s^(i+1) in place of s^(i) (damped: s^(i) + lambda (s - s^(i));
//      narrow storage: rounded to the 16-bit format while the residual known
//      at the update's start is above store_until).
// Per-step arrays are laid out chunk-interleaved (row m * ntiles + k for step
// m of chunk k), so the threads of neighbouring chunks touch neighbouring
// rows.  Padded channels (D < DP) are identity maps with zero input.
#pragma once

#include "pn_cells.cuh"

namespace pn {

template <int CELL, int DP>
struct SmallCfg {
  static constexpr int R = CellInfo<CELL>::R;
  static constexpr int NCS = R + 1;   // coefficient vectors per step: c0, c_1 .. c_R
  static constexpr int L = 32;        // steps per chunk
  static constexpr int NW = 8;        // warps
  static constexpr int NT = 32 * NW;
  static constexpr int WR = R * DP;   // row length of the transposed weights
  static_assert(DP == 4 || DP == 8, "DP in {4, 8}");
  // shared memory in floats: two weight copies, the block reduction, the s0 rows, then per step
  // (step inputs, the iterate, coefficients, b_t) and per chunk (aggregate, entering state)
  static constexpr size_t fixed_floats(int B) { return 2 * (size_t)DP * WR + NW + (size_t)B * DP; }
  // per-step arrays in chunk-interleaved rows: L rows per chunk (a ragged last chunk's rows past
  // T are allocated and never read); step inputs in natural order, B T rows
  static constexpr size_t smem_bytes(int B, int T) {
    const size_t nbt = (size_t)B * T;
    const size_t ntiles = (size_t)B * ((T + L - 1) / L);
    const size_t nrows = (size_t)L * ntiles;
    return 4 * (fixed_floats(B) + nbt * WR + nrows * (DP + NCS * DP + DP) + ntiles * (DP * DP + 2 * DP));
  }
};

// N consecutive floats of shared memory (16-byte aligned) into registers, 16 bytes at a time
template <int N>
__device__ __forceinline__ void lds_vec(const float* p, float (&v)[N]) {
  static_assert(N % 4 == 0, "whole float4s");
#pragma unroll
  for (int e = 0; e < N; e += 4) {
    const float4 t = *reinterpret_cast<const float4*>(p + e);
    v[e] = t.x;
    v[e + 1] = t.y;
    v[e + 2] = t.z;
    v[e + 3] = t.w;
  }
}

__device__ __forceinline__ float round_storage(float v, int fmt) {
  if (fmt == 1) return __bfloat162float(__float2bfloat16_rn(v));
  if (fmt == 2) return __half2float(__float2half_rn(v));
  return v;
}

// proj_w [R*D][d_in], proj_b [R*D]: the hoisted input projection (not read for the Euler cell)
template <int CELL, int DP>
__global__ void __launch_bounds__(SmallCfg<CELL, DP>::NT, 1)
    small_solve_kernel(const IterParams P, const float* __restrict__ proj_w, const float* __restrict__ proj_b) {
  using C = SmallCfg<CELL, DP>;
  constexpr int R = C::R;
  constexpr int NCS = C::NCS;
  constexpr int L = C::L;
  constexpr int NW = C::NW;
  constexpr int NT = C::NT;
  constexpr int WR = C::WR;
  extern __shared__ __align__(16) float smem_sm[];
  __shared__ int s_dec;
  __shared__ float s_r;

  const unsigned long long t_begin = globaltimer();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const Args A = *P.args;
  Ctrl* ctrl = P.ctrl;
  const int D = P.D, T = P.T, B = P.B, d_in = P.d_in;
  const int nch = (T + L - 1) / L;
  const int ntiles = B * nch;
  const int nbt = B * T;   // the problem fits one SM's shared memory: far below 2^31
  const int nrows = L * ntiles;   // chunk-interleaved rows (>= nbt: a ragged last chunk leaves gaps)
  const int band = A.newton_band;
  const bool banded = band >= 0 && band < D - 1;
  const float lambda = A.damping;
  const bool damped = lambda != 1.0f;
  const int sfmt = A.store_fmt;

  float* sWf = smem_sm;                                  // W_q[i][k] at k * WR + q * DP + i
  float* sWb = sWf + DP * WR;                            // the Jacobian's copy (band-masked)
  float* sRed = sWb + DP * WR;                           // [NW]
  float* sS0 = sRed + NW;                                // s0 [B][DP]
  float* sU = sS0 + B * DP;                              // step inputs [b T + t][WR]
  float* sS = sU + nbt * WR;                             // the iterate [row][DP], nrows rows
  float* sCf = sS + nrows * DP;                          // coefficients [row][NCS][DP]
  float* sBv = sCf + nrows * NCS * DP;                   // b_t [row][DP]
  float* sAgg = sBv + nrows * DP;                        // [P | q] per chunk: P row-major, then q
  float* sCar = sAgg + ntiles * (DP * DP + DP);          // entering state per chunk [ntiles][DP]
  // row of step t of sequence b: chunk-interleaved
  auto row_of = [&](int b, int t) { return (t % L) * ntiles + b * nch + t / L; };

  // ---- set-up: weights, s0 rows, the input projection, s^(0) = s0 --------------------------------
  for (int e = tid; e < DP * WR; e += NT) {
    const float w = __ldg(P.wt + e);
    sWf[e] = w;
    const int k = e / WR, i = e % DP;
    sWb[e] = (banded && abs(i - k) > band) ? 0.0f : w;
  }
  for (int e = tid; e < B * DP; e += NT) {
    const int b = e / DP, c = e % DP;
    sS0[e] = c < D ? __ldg(A.s0 + (size_t)b * D + c) : 0.0f;
  }
  for (int e = tid; e < nbt * WR; e += NT) {
    const int bt = e / WR;
    const int qc = e % WR, q = qc / DP, c = qc % DP;
    float v = 0.0f;
    if (c < D) {
      const float* xr = A.x + (size_t)bt * d_in;
      if constexpr (CELL == PN_CELL_EULER_TANH) {
        v = __ldg(xr + c);   // c_t = x_t (d_in = D)
      } else {
        const float* w = proj_w + (size_t)(q * D + c) * d_in;
        float acc = 0.0f;
        for (int k = 0; k < d_in; ++k) acc = fmaf(__ldg(w + k), __ldg(xr + k), acc);
        v = acc + __ldg(proj_b + q * D + c);
      }
    }
    sU[e] = v;
  }
  __syncthreads();
  for (int e = tid; e < nrows * DP; e += NT) {
    const int r = e / DP, c = e % DP;
    const int b = (r % ntiles) / nch;   // row -> chunk -> sequence
    sS[e] = round_storage(sS0[b * DP + c], sfmt);   // s^(0) in the storage format
  }
  const float* sWj = banded ? sWb : sWf;
  __syncthreads();

  float r_prev = 0.0f;   // r^(i-1)
  int i = 0;
  for (;; ++i) {
    // ---- 1. cell phase: one thread per (b, t, channel) -------------------------------------------
    unsigned rb = 0u;
    for (int e = tid; e < nbt * DP; e += NT) {
      const int bt = e / DP;
      const int ci = e % DP;
      const int b = bt / T, t = bt - b * T;
      const int row = row_of(b, t);
      const float* sp = (t == 0) ? sS0 + b * DP : sS + row_of(b, t - 1) * DP;   // s^(i)_{t-1}
      float z[R], zb[R];
#pragma unroll
      for (int q = 0; q < R; ++q) z[q] = zb[q] = 0.0f;
#pragma unroll
      for (int k = 0; k < DP; ++k) {
        const float sv = sp[k];
#pragma unroll
        for (int q = 0; q < R; ++q) {
          z[q] = fmaf(sWf[k * WR + q * DP + ci], sv, z[q]);
          zb[q] = fmaf(sWb[k * WR + q * DP + ci], sv, zb[q]);
        }
      }
      const float spi = sp[ci];
      const float sci = sS[row * DP + ci];
      const float* u = sU + bt * WR;
      float cf[NCS], bb, res;
      if constexpr (CELL == PN_CELL_TANH_RNN) {
        const float y = tanh_pn(z[0] + u[ci]);
        cf[0] = 0.0f;
        cf[1] = 1.0f - y * y;
        bb = y - cf[1] * zb[0];
        res = sci - y;
      } else if constexpr (CELL == PN_CELL_EULER_TANH) {
        const float gg = tanh_pn(z[0] + u[ci]);
        const float eg = P.eps * gg;
        cf[0] = 1.0f;
        cf[1] = P.eps * (1.0f - gg * gg);
        bb = eg - cf[1] * zb[0];
        res = (sci - spi) - eg;
      } else {
        const float bhn = ci < D ? __ldg(P.bhn + ci) : 0.0f;
        const float rr = sigmoidf_acc(u[ci] + z[0]);
        const float zz = sigmoidf_acc(u[DP + ci] + z[1]);
        const float hn = z[2] + bhn;
        const float nn = tanh_pn(u[2 * DP + ci] + rr * hn);
        const float y = nn + zz * (spi - nn);
        const float omz = 1.0f - zz;
        const float dn = omz * (1.0f - nn * nn);
        cf[0] = zz;
        cf[1] = dn * hn * rr * (1.0f - rr);   // W_hr
        cf[2] = (spi - nn) * zz * omz;        // W_hz
        cf[3] = dn * rr;                      // W_hn
        bb = y - (zz * spi + cf[1] * zb[0] + cf[2] * zb[1] + cf[3] * zb[2]);
        res = sci - y;
      }
      if (ci < D) {
        rb = max(rb, abs_bits(res));
      } else {   // padded channel: identity map
        cf[0] = 1.0f;
#pragma unroll
        for (int q = 1; q < NCS; ++q) cf[q] = 0.0f;
        bb = 0.0f;
      }
#pragma unroll
      for (int q = 0; q < NCS; ++q) sCf[(row * NCS + q) * DP + ci] = cf[q];
      sBv[row * DP + ci] = bb;
    }
    rb = warp_max_u32(rb);
    if (lane == 0) sRed[warp] = __uint_as_float(rb);
    __syncthreads();
    if (tid == 0) {
      unsigned v = 0u;
      for (int w = 0; w < NW; ++w) v = max(v, __float_as_uint(sRed[w]));
      const float r = __uint_as_float(v);
      if (i < kHistCap) P.hist[i] = r;
      int st = kRunning;
      if (!(r <= 3.402823466e38f)) st = PN_ERR_NONFINITE;
      else if (r <= A.tol) st = PN_OK;
      else if (i >= A.max_iters) st = PN_NOT_CONVERGED;
      s_dec = st;
      s_r = r;
    }
    __syncthreads();
    if (s_dec != kRunning) break;
    // s^(i+1) is stored narrow while r^(i-1), the residual known when this update starts, is above
    // store_until (s^(1) always, when a narrow format is set)
    const int fmt_new = (sfmt != 0 && (i == 0 || r_prev > A.store_until)) ? sfmt : 0;
    r_prev = s_r;

    // ---- 2. chunk aggregates, one thread per (chunk, column of [P | q]) --------------------------
    for (int e = tid; e < ntiles * (DP + 1); e += NT) {
      const int k = e / (DP + 1), j = e % (DP + 1);   // column j: P e_j for j < DP, q for j = DP
      const int t0 = (k % nch) * L;
      const int n = min(L, T - t0);
      float x[DP];
      {   // step 0: A_{t0} e_j, or b_{t0}
        const float* cf = sCf + (size_t)k * NCS * DP;
#pragma unroll
        for (int ii = 0; ii < DP; ++ii) {
          float v;
          if (j < DP) {
            v = (ii == j) ? cf[ii] : 0.0f;
#pragma unroll
            for (int q = 0; q < R; ++q) v = fmaf(cf[(1 + q) * DP + ii], sWj[j * WR + q * DP + ii], v);
          } else {
            v = sBv[k * DP + ii];
          }
          x[ii] = v;
        }
      }
      for (int m = 1; m < n; ++m) {
        const int row = m * ntiles + k;
        float cf[NCS * DP], bv[DP];
        lds_vec<NCS * DP>(sCf + (size_t)row * NCS * DP, cf);
        lds_vec<DP>(sBv + row * DP, bv);
        float y[DP];
#pragma unroll
        for (int ii = 0; ii < DP; ++ii) {
          float v = cf[ii] * x[ii];
          if (j == DP) v += bv[ii];
#pragma unroll
          for (int q = 0; q < R; ++q) {
            float acc = 0.0f;
#pragma unroll
            for (int kk = 0; kk < DP; ++kk) acc = fmaf(sWj[kk * WR + q * DP + ii], x[kk], acc);
            v = fmaf(cf[(1 + q) * DP + ii], acc, v);
          }
          y[ii] = v;
        }
#pragma unroll
        for (int ii = 0; ii < DP; ++ii) x[ii] = y[ii];
      }
      float* ag = sAgg + k * (DP * DP + DP);
#pragma unroll
      for (int ii = 0; ii < DP; ++ii) {
        if (j < DP) ag[ii * DP + j] = x[ii];
        else ag[DP * DP + ii] = x[ii];
      }
    }
    __syncthreads();

    // ---- 3a. entering state of every chunk: one thread per sequence, chunk after chunk -----------
    for (int b = tid; b < B; b += NT) {
      float carry[DP];
#pragma unroll
      for (int ii = 0; ii < DP; ++ii) carry[ii] = sS0[b * DP + ii];
      for (int c = 0; c < nch; ++c) {
        const int k = b * nch + c;
        float ag[DP * DP + DP];
        lds_vec<DP * DP + DP>(sAgg + k * (DP * DP + DP), ag);
        float nxt[DP];
#pragma unroll
        for (int ii = 0; ii < DP; ++ii) {
          sCar[k * DP + ii] = carry[ii];
          float v = ag[DP * DP + ii];
#pragma unroll
          for (int jj = 0; jj < DP; ++jj) v = fmaf(ag[ii * DP + jj], carry[jj], v);
          nxt[ii] = v;
        }
#pragma unroll
        for (int ii = 0; ii < DP; ++ii) carry[ii] = nxt[ii];
      }
    }
    __syncthreads();

    // ---- 3b. apply: s_t = A_t s_{t-1} + b_t within each chunk, one thread per chunk, stored in place
    for (int k = tid; k < ntiles; k += NT) {
      const int t0 = (k % nch) * L;
      const int n = min(L, T - t0);
      float s[DP];
#pragma unroll
      for (int ii = 0; ii < DP; ++ii) s[ii] = sCar[k * DP + ii];
      for (int m = 0; m < n; ++m) {
        const int row = m * ntiles + k;
        float cf[NCS * DP], bv[DP];
        lds_vec<NCS * DP>(sCf + (size_t)row * NCS * DP, cf);
        lds_vec<DP>(sBv + row * DP, bv);
        float v[DP];
#pragma unroll
        for (int ii = 0; ii < DP; ++ii) {
          float w = fmaf(cf[ii], s[ii], bv[ii]);
#pragma unroll
          for (int q = 0; q < R; ++q) {
            float acc = 0.0f;
#pragma unroll
            for (int kk = 0; kk < DP; ++kk) acc = fmaf(sWj[kk * WR + q * DP + ii], s[kk], acc);
            w = fmaf(cf[(1 + q) * DP + ii], acc, w);
          }
          v[ii] = w;
        }
        float* dst = sS + row * DP;
        float old[DP];   // s^(i)_t
        lds_vec<DP>(dst, old);
#pragma unroll
        for (int ii = 0; ii < DP; ii += 4) {
          float4 o;
          o.x = round_storage(damped ? fmaf(lambda, v[ii] - old[ii], old[ii]) : v[ii], fmt_new);
          o.y = round_storage(damped ? fmaf(lambda, v[ii + 1] - old[ii + 1], old[ii + 1]) : v[ii + 1], fmt_new);
          o.z = round_storage(damped ? fmaf(lambda, v[ii + 2] - old[ii + 2], old[ii + 2]) : v[ii + 2], fmt_new);
          o.w = round_storage(damped ? fmaf(lambda, v[ii + 3] - old[ii + 3], old[ii + 3]) : v[ii + 3], fmt_new);
          *reinterpret_cast<float4*>(dst + ii) = o;
        }
#pragma unroll
        for (int ii = 0; ii < DP; ++ii) s[ii] = v[ii];   // the scan runs undamped and unrounded
      }
    }
    __syncthreads();
  }

  // ---- the result s^(i), and the control block as the multi-CTA loop leaves it -------------------
  for (int e = tid; e < nbt * DP; e += NT) {
    const int bt = e / DP, c = e % DP;
    const int b = bt / T, t = bt - b * T;
    if (c < D) A.states[(size_t)bt * D + c] = sS[row_of(b, t) * DP + c];
  }
  if (tid == 0) {
    ctrl->iter = i;
    ctrl->status = s_dec;
    ctrl->error = 0;
    ctrl->final_iter = i;
    ctrl->final_resid = s_r;
    ctrl->timeout_ticket = -1;
    ctrl->resid_bits = 0u;
    ctrl->done = 0u;
    ctrl->fmt_in = 0;
    ctrl->fmt_out = 0;
    ctrl->final_fmt = 0;
    ctrl->cur_mode = PN_NEWTON;
    ctrl->retried = 0;
    ctrl->launches += (unsigned long long)(i + 1);
    const unsigned long long t1 = globaltimer();
    if (t1 > t_begin) ctrl->kernel_ns += t1 - t_begin;
    ctrl->t_start = ~0ull;
  }
}

}  // namespace pn
