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
//   2. one warp per 32-step chunk: the chunk's aggregate [P | q] (the product
//      of its A_t, and the chunk's response to a zero entering state);
//   3. one warp per sequence folds the aggregates chunk after chunk into each
//      chunk's entering state (starting from s0), then one warp per chunk
//      applies s_t = A_t s_{t-1} + b_t step by step and stores s^(i+1) in place
//      of s^(i) (damped: s^(i) + lambda (s - s^(i)); narrow storage: rounded
//      to the 16-bit format while the residual known at the update's start is
//      above store_until).
// Padded channels (D < DP) are identity maps with zero input.
#pragma once

#include "pn_cells.cuh"

namespace pn {

template <int CELL, int DP>
struct SmallCfg {
  static constexpr int R = CellInfo<CELL>::R;
  static constexpr int NCS = R + 1;   // coefficient vectors per step: c0, c_1 .. c_R
  static constexpr int L = 32;        // steps per chunk
  static constexpr int NW = 32;       // warps
  static constexpr int NT = 32 * NW;
  static constexpr int WR = R * DP;   // row length of the transposed weights
  static_assert(DP == 4 || DP == 8, "DP in {4, 8}");
  // shared memory in floats: two weight copies, per-warp chain buffers, the block reduction, the
  // s0 rows, then per step (step inputs, the iterate, coefficients, b_t) and per chunk (aggregate,
  // entering state)
  static constexpr size_t fixed_floats(int B) {
    return 2 * (size_t)DP * WR + (size_t)NW * (2 * DP * DP + 2 * DP) + NW + (size_t)B * DP;
  }
  static constexpr size_t smem_bytes(int B, int T) {
    const size_t nbt = (size_t)B * T;
    const size_t ntiles = (size_t)B * ((T + L - 1) / L);
    return 4 * (fixed_floats(B) + nbt * (WR + DP + NCS * DP + DP) + ntiles * (DP * DP + 2 * DP));
  }
};

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
  const size_t nbt = (size_t)B * T;
  const int band = A.newton_band;
  const bool banded = band >= 0 && band < D - 1;
  const float lambda = A.damping;
  const bool damped = lambda != 1.0f;
  const int sfmt = A.store_fmt;

  float* sWf = smem_sm;                                   // W_q[i][k] at k * WR + q * DP + i
  float* sWb = sWf + DP * WR;                             // the Jacobian's copy (band-masked)
  float* sWarp = sWb + DP * WR;                           // per warp: P [2][DP*DP], q [2][DP]
  float* sRed = sWarp + NW * (2 * DP * DP + 2 * DP);      // [NW]
  float* sS0 = sRed + NW;                                 // s0 [B][DP]
  float* sU = sS0 + (size_t)B * DP;                       // step inputs [B*T][WR]
  float* sS = sU + nbt * WR;                              // the iterate [B*T][DP]
  float* sCf = sS + nbt * DP;                             // coefficients [B*T][NCS][DP]
  float* sBv = sCf + nbt * NCS * DP;                      // b_t [B*T][DP]
  float* sAgg = sBv + nbt * DP;                           // [P | q] per chunk [ntiles][DP*DP + DP]
  float* sCar = sAgg + (size_t)ntiles * (DP * DP + DP);   // entering state per chunk [ntiles][DP]

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
  for (size_t e = tid; e < nbt * WR; e += NT) {
    const size_t bt = e / WR;
    const int qc = (int)(e % WR), q = qc / DP, c = qc % DP;
    float v = 0.0f;
    if (c < D) {
      const float* xr = A.x + bt * d_in;
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
  for (size_t e = tid; e < nbt * DP; e += NT) {
    const int b = (int)(e / DP / T), c = (int)(e % DP);
    sS[e] = round_storage(sS0[b * DP + c], sfmt);   // s^(0) in the storage format
  }
  const float* sWj = banded ? sWb : sWf;
  __syncthreads();

  float r_prev = 0.0f;   // r^(i-1)
  int i = 0;
  for (;; ++i) {
    // ---- 1. cell phase: one thread per (b, t, channel) -------------------------------------------
    unsigned rb = 0u;
    for (size_t e = tid; e < nbt * DP; e += NT) {
      const size_t bt = e / DP;
      const int ci = (int)(e % DP);
      const int t = (int)(bt % T), b = (int)(bt / T);
      const float* sp = (t == 0) ? sS0 + b * DP : sS + (bt - 1) * DP;   // s^(i)_{t-1}
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
      const float sci = sS[bt * DP + ci];
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
      for (int q = 0; q < NCS; ++q) sCf[(bt * NCS + q) * DP + ci] = cf[q];
      sBv[bt * DP + ci] = bb;
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

    // ---- 2. chunk aggregates [P | q]: one warp per chunk -----------------------------------------
    float* wP = sWarp + warp * (2 * DP * DP + 2 * DP);
    float* wQ = wP + 2 * DP * DP;
    for (int k = warp; k < ntiles; k += NW) {
      const int b = k / nch, t0 = (k % nch) * L;
      const int n = min(L, T - t0);
      const size_t bt0 = (size_t)b * T + t0;
      {
        const float* cf = sCf + bt0 * NCS * DP;
        for (int e = lane; e < DP * DP; e += 32) {
          const int ii = e / DP, j = e % DP;
          float v = (ii == j) ? cf[ii] : 0.0f;
#pragma unroll
          for (int q = 0; q < R; ++q) v = fmaf(cf[(1 + q) * DP + ii], sWj[j * WR + q * DP + ii], v);
          wP[e] = v;
        }
        if (lane < DP) wQ[lane] = sBv[bt0 * DP + lane];
      }
      __syncwarp();
      int cur = 0;
      for (int m = 1; m < n; ++m) {
        const float* cf = sCf + (bt0 + m) * NCS * DP;
        const float* Pk = wP + cur * DP * DP;
        float* Pn = wP + (cur ^ 1) * DP * DP;
        for (int e = lane; e < DP * DP; e += 32) {
          const int ii = e / DP, j = e % DP;
          float v = cf[ii] * Pk[e];
#pragma unroll
          for (int q = 0; q < R; ++q) {
            float acc = 0.0f;
#pragma unroll
            for (int kk = 0; kk < DP; ++kk) acc = fmaf(sWj[kk * WR + q * DP + ii], Pk[kk * DP + j], acc);
            v = fmaf(cf[(1 + q) * DP + ii], acc, v);
          }
          Pn[e] = v;
        }
        if (lane < DP) {
          const float* qk = wQ + cur * DP;
          float v = fmaf(cf[lane], qk[lane], sBv[(bt0 + m) * DP + lane]);
#pragma unroll
          for (int q = 0; q < R; ++q) {
            float acc = 0.0f;
#pragma unroll
            for (int kk = 0; kk < DP; ++kk) acc = fmaf(sWj[kk * WR + q * DP + lane], qk[kk], acc);
            v = fmaf(cf[(1 + q) * DP + lane], acc, v);
          }
          wQ[(cur ^ 1) * DP + lane] = v;
        }
        __syncwarp();
        cur ^= 1;
      }
      float* ag = sAgg + (size_t)k * (DP * DP + DP);
      for (int e = lane; e < DP * DP; e += 32) ag[e] = wP[cur * DP * DP + e];
      if (lane < DP) ag[DP * DP + lane] = wQ[cur * DP + lane];
      __syncwarp();
    }
    __syncthreads();

    // ---- 3a. entering state of every chunk: one warp per sequence, chunk after chunk -------------
    for (int b = warp; b < B; b += NW) {
      float carry = (lane < DP) ? sS0[b * DP + lane] : 0.0f;
      for (int c = 0; c < nch; ++c) {
        const int k = b * nch + c;
        if (lane < DP) sCar[k * DP + lane] = carry;
        const float* ag = sAgg + (size_t)k * (DP * DP + DP);
        float v = (lane < DP) ? ag[DP * DP + lane] : 0.0f;
#pragma unroll
        for (int j = 0; j < DP; ++j) {
          const float cj = __shfl_sync(0xffffffffu, carry, j);
          if (lane < DP) v = fmaf(ag[lane * DP + j], cj, v);
        }
        carry = v;
      }
    }
    __syncthreads();

    // ---- 3b. apply: s_t = A_t s_{t-1} + b_t within each chunk, stored in place -------------------
    for (int k = warp; k < ntiles; k += NW) {
      const int b = k / nch, t0 = (k % nch) * L;
      const int n = min(L, T - t0);
      const size_t bt0 = (size_t)b * T + t0;
      float sprev = (lane < DP) ? sCar[k * DP + lane] : 0.0f;
      for (int m = 0; m < n; ++m) {
        const float* cf = sCf + (bt0 + m) * NCS * DP;
        float acc[R];
#pragma unroll
        for (int q = 0; q < R; ++q) acc[q] = 0.0f;
#pragma unroll
        for (int kk = 0; kk < DP; ++kk) {
          const float sk = __shfl_sync(0xffffffffu, sprev, kk);
          if (lane < DP) {
#pragma unroll
            for (int q = 0; q < R; ++q) acc[q] = fmaf(sWj[kk * WR + q * DP + lane], sk, acc[q]);
          }
        }
        float v = 0.0f;
        if (lane < DP) {
          v = fmaf(cf[lane], sprev, sBv[(bt0 + m) * DP + lane]);
#pragma unroll
          for (int q = 0; q < R; ++q) v = fmaf(cf[(1 + q) * DP + lane], acc[q], v);
          float* dst = sS + (bt0 + m) * DP + lane;
          const float old = *dst;   // s^(i)_t
          *dst = round_storage(damped ? fmaf(lambda, v - old, old) : v, fmt_new);
        }
        sprev = v;
      }
    }
    __syncthreads();
  }

  // ---- the result s^(i), and the control block as the multi-CTA loop leaves it -------------------
  for (size_t e = tid; e < nbt * DP; e += NT) {
    const int c = (int)(e % DP);
    if (c < D) A.states[(e / DP) * D + c] = sS[e];
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
