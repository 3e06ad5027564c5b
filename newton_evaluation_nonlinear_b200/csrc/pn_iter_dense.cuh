// pn_iter_dense.cuh -- fused iteration kernel for full Newton (dense D x D).
//
// One launch performs one iteration of the page's unified update with the
// exact Jacobian J~ = J ("Parallel Newton methods..." page, §1.2):
//     s^(i+1)_t = A_t s^(i+1)_{t-1} + b_t,  A_t = df_t/ds(s^(i)_{t-1}),
//     b_t = f_t(s^(i)_{t-1}) - A_t s^(i)_{t-1},
// solved with the affine-map scan of §2.1 (combine (A,b) o (A',b') =
// (A'A, A'b + b'), (A,b) earlier) over D x D blocks.
//
// With a band k >= 0 (Args::newton_band) the kernel uses the banded
// approximation of §2.2.2 instead: A_t keeps the entries of df_t/ds with
// |row - col| <= k, and b_t = f_t(s^(i)_{t-1}) - A_t s^(i)_{t-1} takes the
// banded product.  k >= D - 1 is the exact Jacobian.
//
// With a damping factor lambda < 1 (Args::damping; page §4.3 and §5.3 name
// damping as the remedy for a stalled iteration) the stored iterate is
// s^(i) + lambda (s_full - s^(i)), where s_full is the undamped update the
// scan produces; the scan itself, its aggregates and its carried states stay
// undamped (lambda * delta solves J~ v = -lambda F).
//
// Every Jacobian of the three cells is a row-scaled sum of fixed matrices,
//     A_t = diag(c0_t) + sum_q diag(c_{q,t}) W_q,
// so the kernel evaluates the cell once, keeps the per-step coefficient
// vectors, and materialises A_t in shared memory.
//
// Persistent CTAs claim tiles = (sequence b, chunk of L steps) in ticket
// order; NT = L * DP threads.  Per tile:
//   1. stage s^(i) rows t0-1..t0+L-1; thread (m, i) computes the cell at step
//      m, channel i: y, coefficients, b_t (from W s_{t-1} of the same matvec)
//      and |F|;
//   2. build A_m for every step of the tile;
//   3. prefix chain [P_m | q_m] = A_m [P_{m-1} | q_{m-1}] + [0 | b_m],
//      [P_0 | q_0] = [A_0 | b_0], kept for every m (L x D x (D+1) floats);
//   4. decoupled look-back: publish [P_{L-1} | q_{L-1}], find the nearest
//      predecessor with a published state (32 per round trip), load the
//      aggregates in between into shared memory and apply them farthest first
//      (one D x D matvec each), publish this tile's end state;
//   5. s_t = P_m carry + q_m for every step in parallel.
#pragma once

#include "pn_cells.cuh"

namespace pn {

template <int CELL, int DP, int L>
struct DenseCfg {
  static constexpr int R = CellInfo<CELL>::R;
  static constexpr int NT = L * DP;
  static constexpr int SP = DP + 4;
  static constexpr int WCOLS = R * DP;
  static constexpr int NC = R + 1;       // coefficient vectors per step: c0 and one per W_q
  static constexpr int PQW = DP + 1;     // row width of [P | q]
  static constexpr int OFF_S = 0;
  static constexpr int OFF_W = OFF_S + (L + 1) * SP;                 // transposed [DP][R*DP]
  static constexpr int OFF_WR = OFF_W + DP * WCOLS;                  // row-major [R][DP][DP]
  static constexpr int OFF_COEF = OFF_WR + R * DP * DP;              // [L][NC][DP]
  static constexpr int OFF_A = OFF_COEF + L * NC * DP;               // [L][DP][DP]; look-back window later
  static constexpr int OFF_PQ = OFF_A + L * DP * DP;                 // [L][DP][PQW]
  static constexpr int OFF_CARRY = OFF_PQ + L * DP * PQW;            // 2 x DP
  static constexpr int OFF_RED = OFF_CARRY + 2 * DP;
  static constexpr int SMEM_FLOATS = OFF_RED + (NT + 31) / 32;
  static constexpr size_t SMEM_BYTES = (size_t)SMEM_FLOATS * sizeof(float);
  static constexpr int WCAP = (L * DP * DP) / (DP * PQW);            // aggregates per window batch
  static_assert(DP % 4 == 0, "DP must be a multiple of 4");
  static_assert(NT % 32 == 0 && NT <= 1024, "bad thread count");
  static_assert(OFF_W % 4 == 0 && OFF_WR % 4 == 0, "alignment");
  static_assert(WCAP >= 1, "look-back window must hold one aggregate");
};

template <int CELL, int DP, int L>
__global__ void __launch_bounds__(DenseCfg<CELL, DP, L>::NT) dense_iter_kernel(const IterParams P) {
  using C = DenseCfg<CELL, DP, L>;
  constexpr int R = C::R;
  constexpr int NC = C::NC;
  constexpr int PQW = C::PQW;

  extern __shared__ __align__(16) float smem[];
  float* sS = smem + C::OFF_S;
  float* sW = smem + C::OFF_W;
  float* sWr = smem + C::OFF_WR;
  float* sCoef = smem + C::OFF_COEF;
  float* sA = smem + C::OFF_A;
  float* sPQ = smem + C::OFF_PQ;
  float* sCarry = smem + C::OFF_CARRY;
  float* sRed = smem + C::OFF_RED;
  __shared__ int s_ticket, s_nagg, s_last;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  Ctrl* ctrl = P.ctrl;
  const Args A = *P.args;
  const int D = P.D, T = P.T, B = P.B;
  const int band = A.newton_band;
  const bool banded = band >= 0 && band < D - 1;
  const float lambda = A.damping;
  const bool damped = lambda != 1.0f;
  const size_t stride = (size_t)B;

  if (tid == 0) atomicMin(&ctrl->t_start, globaltimer());
  const unsigned epoch = *(volatile unsigned*)&ctrl->epoch;
  const int iter = *(volatile int*)&ctrl->iter;
  const float* __restrict__ src = (iter & 1) ? P.buf1 : A.states;
  float* __restrict__ dst = (iter & 1) ? A.states : P.buf1;
  const int2 fmt = iter_formats(ctrl, A);   // storage of s^(i) (x) and s^(i+1) (y)

  // thread (m, i): step m of the tile, channel i
  const int m = tid / DP;
  const int i = tid % DP;
  const float bhn_i = (CELL == PN_CELL_GRU && i < D) ? __ldg(P.bhn + i) : 0.0f;

  {
    const float4* w4 = reinterpret_cast<const float4*>(P.wt);
    float4* d4 = reinterpret_cast<float4*>(sW);
    for (int e = tid; e < DP * C::WCOLS / 4; e += C::NT) d4[e] = __ldg(w4 + e);
    const float4* r4 = reinterpret_cast<const float4*>(P.wt + (size_t)DP * C::WCOLS);
    float4* e4 = reinterpret_cast<float4*>(sWr);
    for (int e = tid; e < R * DP * DP / 4; e += C::NT) e4[e] = __ldg(r4 + e);
  }
  unsigned rbits = 0u;

  for (;;) {
    if (tid == 0) s_ticket = (int)atomicAdd(&ctrl->ticket[0], 1u);
    __syncthreads();
    const int k = s_ticket;
    if (k >= P.tiles_per_group) break;
    const int b = k % B;
    const int chunk = k / B;
    const int t0 = chunk * L;
    const int t = t0 + m;
    const bool ok = (t < T) && (i < D);

    // ---- 1. stage ----------------------------------------------------------
    float xv[R];
    {
      const float* xin = (CELL == PN_CELL_EULER_TANH) ? A.x : P.xin;
#pragma unroll
      for (int q = 0; q < R; ++q)
        xv[q] = ok ? __ldg(xin + ((size_t)b * T + t) * (R * D) + (size_t)q * D + i) : 0.0f;
    }
    for (int e = tid; e < (L + 1) * DP; e += C::NT) {
      const int r = e / DP;
      const int c = e % DP;
      const int tt = t0 - 1 + r;
      float v = 0.0f;
      if (c < D) {
        if (tt < 0) v = __ldg(A.s0 + (size_t)b * D + c);
        else if (tt < T) v = ld_state(src, ((size_t)b * T + tt) * D + c, fmt.x);
      }
      sS[r * C::SP + c] = v;
    }
    __syncthreads();

    // ---- 1b. cell at (m, i): matvec, coefficients, b_t, |F| ---------------
    {
      float acc[R];
#pragma unroll
      for (int q = 0; q < R; ++q) acc[q] = 0.0f;
#pragma unroll(DP <= 32 ? DP / 4 : 4)
      for (int kk = 0; kk < DP; kk += 4) {
        const float4 sv = *reinterpret_cast<const float4*>(sS + m * C::SP + kk);
#pragma unroll
        for (int q = 0; q < R; ++q) {
          acc[q] = fmaf(sW[(kk + 0) * C::WCOLS + q * DP + i], sv.x, acc[q]);
          acc[q] = fmaf(sW[(kk + 1) * C::WCOLS + q * DP + i], sv.y, acc[q]);
          acc[q] = fmaf(sW[(kk + 2) * C::WCOLS + q * DP + i], sv.z, acc[q]);
          acc[q] = fmaf(sW[(kk + 3) * C::WCOLS + q * DP + i], sv.w, acc[q]);
        }
      }
      const float sp = sS[m * C::SP + i];        // s^(i)_{t-1}, channel i
      const float sc = sS[(m + 1) * C::SP + i];  // s^(i)_t
      // the products W_q s restricted to the band, for b_t = f - A s (the full products
      // above serve the cell itself)
      float accb[R];
#pragma unroll
      for (int q = 0; q < R; ++q) accb[q] = acc[q];
      if (banded) {
        const int k_lo = max(0, i - band);
        const int k_hi = min(DP - 1, i + band);
#pragma unroll
        for (int q = 0; q < R; ++q) {
          float v = 0.0f;
          for (int kk = k_lo; kk <= k_hi; ++kk) v = fmaf(sWr[(q * DP + i) * DP + kk], sS[m * C::SP + kk], v);
          accb[q] = v;
        }
      }
      float coef[NC];
      float bb, res;
      if constexpr (CELL == PN_CELL_TANH_RNN) {
        // A = diag(1 - y^2) W
        const float y = tanh_pn(acc[0] + xv[0]);
        const float d = 1.0f - y * y;
        coef[0] = 0.0f;
        coef[1] = d;
        bb = y - d * accb[0];
        res = sc - y;
      } else if constexpr (CELL == PN_CELL_EULER_TANH) {
        // A = I + diag(eps (1 - g^2)) W
        const float gg = tanh_pn(acc[0] + xv[0]);
        const float eg = P.eps * gg;
        const float e = P.eps * (1.0f - gg * gg);
        coef[0] = 1.0f;
        coef[1] = e;
        bb = eg - e * accb[0];
        res = (sc - sp) - eg;
      } else {
        // A = diag(z) + diag(gam) W_hr + diag(alp) W_hz + diag(bet) W_hn
        const float r = sigmoidf_acc(xv[0] + acc[0]);
        const float z = sigmoidf_acc(xv[1] + acc[1]);
        const float hn = acc[2] + bhn_i;
        const float nn = tanh_pn(xv[2] + r * hn);
        const float y = nn + z * (sp - nn);
        const float omz = 1.0f - z;
        const float dn = omz * (1.0f - nn * nn);
        const float alp = (sp - nn) * z * omz;
        const float bet = dn * r;
        const float gam = dn * hn * r * (1.0f - r);
        coef[0] = z;
        coef[1] = gam;
        coef[2] = alp;
        coef[3] = bet;
        bb = y - (z * sp + gam * accb[0] + alp * accb[1] + bet * accb[2]);
        res = sc - y;
      }
      if (ok) {
        rbits = max(rbits, abs_bits(res));
      } else {
#pragma unroll
        for (int q = 0; q < NC; ++q) coef[q] = 0.0f;
        bb = 0.0f;
      }
#pragma unroll
      for (int q = 0; q < NC; ++q) sCoef[(m * NC + q) * DP + i] = coef[q];
      sPQ[(m * DP + i) * PQW + DP] = bb;   // q column starts as b_m
    }
    __syncthreads();

    // ---- 2. A_m = diag(c0) + sum_q diag(c_q) W_q for every step -------------
    for (int e = tid; e < L * DP * DP; e += C::NT) {
      const int mm = e / (DP * DP);
      const int ii = (e / DP) % DP;
      const int kk = e % DP;
      float v = (ii == kk) ? sCoef[(mm * NC + 0) * DP + ii] : 0.0f;
#pragma unroll
      for (int q = 0; q < R; ++q) v = fmaf(sCoef[(mm * NC + 1 + q) * DP + ii], sWr[(q * DP + ii) * DP + kk], v);
      if (banded && abs(ii - kk) > band) v = 0.0f;
      sA[e] = v;
      if (mm == 0) sPQ[ii * PQW + kk] = v;   // P_0 = A_0
    }
    __syncthreads();

    // ---- 3. prefix chain ---------------------------------------------------
    for (int mm = 1; mm < L; ++mm) {
      const float* Am = sA + mm * DP * DP;
      const float* prev = sPQ + (mm - 1) * DP * PQW;
      float* cur = sPQ + mm * DP * PQW;
      for (int e = tid; e < DP * PQW; e += C::NT) {
        const int ii = e / PQW;
        const int jj = e % PQW;
        float v = (jj == DP) ? cur[ii * PQW + DP] : 0.0f;
#pragma unroll(DP <= 16 ? DP : 16)
        for (int kk = 0; kk < DP; ++kk) v = fmaf(Am[ii * DP + kk], prev[kk * PQW + jj], v);
        cur[ii * PQW + jj] = v;
      }
      __syncthreads();
    }

    // ---- 4. decoupled look-back --------------------------------------------
    const float* last = sPQ + (L - 1) * DP * PQW;
    const bool stall = (A.stall_ticket == k);
    if (chunk > 0 && !stall) {
      float* ag = P.agg + (size_t)k * P.agg_stride;
      for (int e = tid; e < DP * PQW; e += C::NT) ag[e] = last[e];
      __threadfence();
    }
    __syncthreads();
    if (warp == 0) {
      if (chunk > 0 && !stall && lane == 0) st_release(P.flags + k, make_flag(epoch, kFlagAgg));
      const int n = lookback_find_prefix(P.flags, (size_t)k, stride, chunk, epoch, ctrl, A.timeout_ns);
      if (lane == 0) s_nagg = n;
    }
    __syncthreads();
    const int n_agg = s_nagg;
    if (n_agg < 0) break;   // gave up: the launch reports the error
    // starting state: the end state of the tile at distance n_agg + 1, or s0
    float* cur = sCarry;
    float* nxt = sCarry + DP;
    if (tid < DP) {
      float v = 0.0f;
      if (chunk - 1 - n_agg >= 0) v = __ldcg(P.pref + ((size_t)k - (size_t)(n_agg + 1) * stride) * P.pref_stride + tid);
      else if (tid < D) v = __ldg(A.s0 + (size_t)b * D + tid);
      cur[tid] = v;
    }
    __syncthreads();
    // apply the aggregates at distances n_agg .. 1, farthest first, in batches
    for (int hi = n_agg; hi >= 1; hi -= C::WCAP) {
      const int nb = min(C::WCAP, hi);   // distances hi, hi-1, ..., hi-nb+1
      for (int e = tid; e < nb * DP * PQW; e += C::NT) {
        const int w = e / (DP * PQW);
        const int off = e % (DP * PQW);
        sA[e] = __ldcg(P.agg + ((size_t)k - (size_t)(hi - w) * stride) * P.agg_stride + off);
      }
      __syncthreads();
      for (int w = 0; w < nb; ++w) {
        const float* ag = sA + w * DP * PQW;
        if (tid < DP) {
          float v = ag[tid * PQW + DP];
#pragma unroll(DP <= 16 ? DP : 16)
          for (int kk = 0; kk < DP; ++kk) v = fmaf(ag[tid * PQW + kk], cur[kk], v);
          nxt[tid] = v;
        }
        __syncthreads();
        float* tmp = cur; cur = nxt; nxt = tmp;
      }
    }
    if (tid < DP && !stall) {
      float v = last[tid * PQW + DP];
#pragma unroll(DP <= 16 ? DP : 16)
      for (int kk = 0; kk < DP; ++kk) v = fmaf(last[tid * PQW + kk], cur[kk], v);
      P.pref[(size_t)k * P.pref_stride + tid] = v;
      __threadfence();
    }
    __syncthreads();
    if (tid == 0 && !stall) st_release(P.flags + k, make_flag(epoch, kFlagPrefix));

    // ---- 5. s_t = P_m carry + q_m ------------------------------------------
    if (ok) {
      const float* row = sPQ + (m * DP + i) * PQW;
      float v = row[DP];
#pragma unroll(DP <= 16 ? DP : 16)
      for (int kk = 0; kk < DP; ++kk) v = fmaf(row[kk], cur[kk], v);
      if (damped) {
        const float sc = sS[(m + 1) * C::SP + i];   // s^(i)_t, staged in step 1
        v = fmaf(lambda, v - sc, sc);
      }
      st_state(dst, ((size_t)b * T + t) * D + i, v, fmt.y);
    }
  }

  rbits = warp_max_u32(rbits);
  if (lane == 0) sRed[warp] = __uint_as_float(rbits);
  __syncthreads();
  if (tid == 0) {
    unsigned v = 0u;
    for (int w = 0; w < (C::NT + 31) / 32; ++w) v = max(v, __float_as_uint(sRed[w]));
    if (v) atomicMax(&ctrl->resid_bits, v);
  }
  finish_launch(P, A, epoch, s_last);
}

}  // namespace pn
