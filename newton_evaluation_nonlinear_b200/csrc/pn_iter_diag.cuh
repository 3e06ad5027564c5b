// pn_iter_diag.cuh -- fused iteration kernel for the Jacobi, Picard and
// diagonal quasi-Newton modes.
//
// One launch performs one full iteration s^(i) -> s^(i+1) of the page's
// unified update s^(i+1) = s^(i) - J~^{-1} F(s^(i)) ("Parallel Newton
// methods..." page, §1.2), in the direct form
//     s^(i+1)_t = a_t s^(i+1)_{t-1} + b_t,   b_t = f_t(s^(i)_{t-1}) - a_t s^(i)_{t-1}
// with a_t = 0 (Jacobi), 1 (Picard, identity approximation, §2.2.3) or the
// diagonal of df_t/ds (quasi-Newton, §2.2.1), per channel.  Each channel is
// an independent scalar affine recurrence, scanned with the combine
// (a,b) o (a',b') = (a'a, a'b + b'), (a,b) the earlier element (§2.1).
//
// Persistent CTAs, each bound to one channel group g (so the group's
// transposed recurrent weights are staged in shared memory once per launch),
// claim tiles = (sequence b, chunk of L steps) of their group in ticket order.
// Per tile:
//   1. stage s^(i) rows t0-1 .. t0+L-1 (all channels) transposed, sT[k][t],
//      so a thread reads its TM consecutive steps of one channel as one
//      16-byte shared load; prefetch the step inputs into registers;
//   2. register-tiled matvec W s_{t-1}: TM steps x TN channels per thread;
//   3. cell + diagonal Jacobian, b_t, and |s^(i)_t - f_t(s^(i)_{t-1})|;
//   4. serial scan over the thread's TM steps, warp-shuffle scan across the
//      TS thread segments (plus a shared-memory pass when TS > 32);
//   5. decoupled look-back: publish the tile aggregate, find the nearest
//      predecessor with a published state (32 predecessors per round trip,
//      one lane each), fold in the aggregates in between, publish this tile's
//      own end state;
//   6. apply the carry and write s^(i+1).
// The CTA's running max of |F| goes to one atomicMax; the last CTA takes the
// stop decision.  A tile only ever waits on tiles with lower tickets, which are
// held by running CTAs (forward progress), and every wait is bounded in time.
#pragma once

#include "pn_cells.cuh"

namespace pn {

// PRE: the recurrent product W s_{t-1} of every step comes precomputed from the
// tensor cores (pn_wide_gemm.cuh) in IterParams::ypre, row b T + t - 1 for step t
// (step 0 forms W s0 itself); the CTA stages only its channel group's states.
template <int CELL, int MODE, int DP, int G, int TM, int TN, int TS, bool PRE = false>
struct DiagCfg {
  static constexpr int R = CellInfo<CELL>::R;
  static constexpr int L = TS * TM;           // steps per tile
  static constexpr int JG = G / TN;           // channel groups of TN per tile
  static constexpr int NT = TS * JG;          // threads per CTA
  static constexpr int LP = L + 4;            // row length of sT (time rows 0..L, padded)
  static constexpr int WCOLS = R * G;         // columns of the transposed weight slice
  static constexpr int TSW = TS < 32 ? TS : 32;
  static constexpr int WPG = TS / TSW;        // warps along t per channel group
  static constexpr int NQ = (G + 31) / 32;    // channels per lane in the look-back warp
  static constexpr int OFF_S = 0;
  static constexpr int OFF_W = OFF_S + DP * LP;
  static constexpr int OFF_AGG = OFF_W + (PRE ? 0 : DP * WCOLS);
  static constexpr int OFF_PART = OFF_AGG + 2 * G;
  static constexpr int OFF_CARRY = OFF_PART + 2 * JG * WPG * TN;
  static constexpr int OFF_RED = OFF_CARRY + G;
  static constexpr int SMEM_FLOATS = OFF_RED + NT / 32;
  static constexpr size_t SMEM_BYTES = (size_t)SMEM_FLOATS * sizeof(float);
  static_assert(DP % 4 == 0 && TM == 4, "DP multiple of 4, TM == 4");
  static_assert(G % TN == 0 && G <= DP, "bad group");
  static_assert(NT % 32 == 0 && NT <= 1024, "bad thread count");
  static_assert((TS & (TS - 1)) == 0 && (TS <= 32 || TS % 32 == 0), "TS must be a power of two");
  static_assert(TN == 1 || TN == 2 || TN == 4, "TN must be 1, 2 or 4");
  static_assert(OFF_W % 4 == 0 && LP % 4 == 0, "16-byte alignment of shared tiles");
  static_assert(!PRE || R == 1, "precomputed products: one-gate cells");
};

template <int CELL, int MODE, int DP, int G, int TM, int TN, int TS, bool PRE = false>
__global__ void __launch_bounds__(DiagCfg<CELL, MODE, DP, G, TM, TN, TS, PRE>::NT)
    diag_iter_kernel(const IterParams P) {
  using C = DiagCfg<CELL, MODE, DP, G, TM, TN, TS, PRE>;
  constexpr int R = C::R;
  constexpr int L = C::L;
  constexpr int LP = C::LP;
  constexpr bool kScan = (MODE != PN_JACOBI);
  constexpr bool kHasA = (MODE == PN_QUASI);

  extern __shared__ __align__(16) float smem[];
  float* sT = smem + C::OFF_S;
  float* sW = smem + C::OFF_W;
  float* sAgg = smem + C::OFF_AGG;
  float* sPart = smem + C::OFF_PART;
  float* sCarry = smem + C::OFF_CARRY;
  float* sRed = smem + C::OFF_RED;
  __shared__ int s_ticket, s_abort, s_last;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  Ctrl* ctrl = P.ctrl;
  const Args A = *P.args;
  const int D = P.D, T = P.T, B = P.B;
  const float lambda = A.damping;   // s^(i+1) = s^(i) + lambda * delta (1: undamped)
  const bool damped = lambda != 1.0f;
  const int g = (int)(blockIdx.x % (unsigned)P.ngroups);
  const size_t stride = (size_t)B * P.ngroups;   // flag distance between consecutive chunks

  if (tid == 0) atomicMin(&ctrl->t_start, globaltimer());
  const unsigned epoch = *(volatile unsigned*)&ctrl->epoch;
  const int iter = *(volatile int*)&ctrl->iter;
  const float* __restrict__ src = (iter & 1) ? P.buf1 : A.states;
  float* __restrict__ dst = (iter & 1) ? A.states : P.buf1;
  const int2 fmt = iter_formats(ctrl, A);   // storage of s^(i) (x) and s^(i+1) (y): 0 float32, else 16-bit

  const int tseg = tid % TS;
  const int jg = tid / TS;
  const int m0 = tseg * TM;          // first local step of this thread
  const int j0 = jg * TN;            // first channel within the group
  const int c0 = g * G + j0;         // first global channel
  const int cvalid = max(0, min(TN, D - c0));
  const bool vec_ok = ((D % TN) == 0);
  const bool dvec = (D % 4) == 0;

  // weights of this group, once per launch
  if constexpr (!PRE) {
    const float4* wsrc = reinterpret_cast<const float4*>(P.wt + (size_t)g * DP * C::WCOLS);
    float4* wdst = reinterpret_cast<float4*>(sW);
    for (int e = tid; e < DP * C::WCOLS / 4; e += C::NT) wdst[e] = __ldg(wsrc + e);
  }
  // s^(i+1) elements e .. e + cvalid - 1, in the storage format of the output
  auto store_out = [&](size_t e, const float (&o)[TN]) {
    if (fmt.y == 0) {
      store_n<TN>(dst + e, o, cvalid, vec_ok);
    } else {
#pragma unroll
      for (int n = 0; n < TN; ++n)
        if (n < cvalid) st_state(dst, e + n, o[n], fmt.y);
    }
  };
  float wd[TN][R];    // W_q[c][c] for this thread's channels (quasi mode)
  float bhn[TN];
  unsigned rbits = 0u;

  for (int tile_iter = 0;; ++tile_iter) {
    if (tid == 0) s_ticket = (int)atomicAdd(&ctrl->ticket[g], 1u);
    __syncthreads();   // also orders the previous tile's shared reads before restaging
    const int kg = s_ticket;
    if (kg >= P.tiles_per_group) break;
    const int b = kg % B;
    const int chunk = kg / B;
    const int t0 = chunk * L;
    const size_t k = (size_t)kg * P.ngroups + g;   // descriptor index of this tile

    // ---- 1a. prefetch the step inputs (u / gx / c) into registers --------
    float xv[TM][R][TN];
    {
      const float* xin = (CELL == PN_CELL_EULER_TANH) ? A.x : P.xin;
      const int xstride = R * D;
#pragma unroll
      for (int m = 0; m < TM; ++m) {
        const int t = t0 + m0 + m;
#pragma unroll
        for (int q = 0; q < R; ++q) {
          if (t < T && cvalid > 0) {
            load_n<TN>(xin + ((size_t)b * T + t) * xstride + (size_t)q * D + c0, xv[m][q], cvalid, vec_ok);
          } else {
#pragma unroll
            for (int n = 0; n < TN; ++n) xv[m][q][n] = 0.0f;
          }
        }
      }
    }

    // ---- 1b. stage s rows t0-1 .. t0+L-1 transposed: sT[k][r], time t0-1+r
    {
      constexpr int Q4 = PRE ? G / 4 : DP / 4;   // PRE: only this group's channels are read
      constexpr int RB = (L + 1 + 7) / 8;
      for (int e = tid; e < RB * Q4 * 8; e += C::NT) {
        const int rl = e & 7;
        const int c4 = (e >> 3) % Q4 + (PRE ? g * (G / 4) : 0);
        const int r = ((e >> 3) / Q4) * 8 + rl;
        if (r > L) continue;
        const int c = c4 * 4;
        const int t = t0 - 1 + r;
        const float* row = nullptr;
        if (t < 0) row = A.s0 + (size_t)b * D;
        else if (t < T) row = src + ((size_t)b * T + t) * D;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row != nullptr && c < D) {
          if (t >= 0 && fmt.x != 0) {   // narrow s^(i)
            const size_t e0 = ((size_t)b * T + t) * D + c;
            v.x = ld_state(src, e0, fmt.x);
            if (c + 1 < D) v.y = ld_state(src, e0 + 1, fmt.x);
            if (c + 2 < D) v.z = ld_state(src, e0 + 2, fmt.x);
            if (c + 3 < D) v.w = ld_state(src, e0 + 3, fmt.x);
          } else if (dvec) {
            v = __ldg(reinterpret_cast<const float4*>(row + c));
          } else {
            v.x = __ldg(row + c);
            if (c + 1 < D) v.y = __ldg(row + c + 1);
            if (c + 2 < D) v.z = __ldg(row + c + 2);
            if (c + 3 < D) v.w = __ldg(row + c + 3);
          }
        }
        sT[(c + 0) * LP + r] = v.x;
        sT[(c + 1) * LP + r] = v.y;
        sT[(c + 2) * LP + r] = v.z;
        sT[(c + 3) * LP + r] = v.w;
      }
    }
    if (tile_iter == 0) {
#pragma unroll
      for (int n = 0; n < TN; ++n) {
        const int c = c0 + n;
        const int cw = (n < cvalid) ? c : 0;
        const int jl = j0 + n;
#pragma unroll
        for (int q = 0; q < R; ++q) {
          if constexpr (PRE) wd[n][q] = (n < cvalid) ? __ldg(P.wdiag + q * DP + c) : 0.0f;
          else wd[n][q] = sW[cw * C::WCOLS + q * G + jl];
        }
        bhn[n] = (CELL == PN_CELL_GRU && n < cvalid) ? __ldg(P.bhn + c) : 0.0f;
      }
    }
    __syncthreads();

    // ---- 2. matvec: acc[m][q][n] = sum_k W_q[c0+n][k] * s_{t-1}[k] --------
    float acc[TM][R][TN];
#pragma unroll
    for (int m = 0; m < TM; ++m)
#pragma unroll
      for (int q = 0; q < R; ++q)
#pragma unroll
        for (int n = 0; n < TN; ++n) acc[m][q][n] = 0.0f;

    if constexpr (PRE) {
      // W s_{t-1} from the tensor cores' product; step 0 of a sequence: W s0, formed here
#pragma unroll
      for (int m = 0; m < TM; ++m) {
        const int t = t0 + m0 + m;
        if (t >= 1 && t < T && cvalid > 0) {
          load_n<TN>(P.ypre + ((size_t)b * T + t - 1) * D + c0, acc[m][0], cvalid, vec_ok);
        } else if (t == 0) {
          for (int kk = 0; kk < D; ++kk) {
            const float s0k = __ldg(A.s0 + (size_t)b * D + kk);
#pragma unroll
            for (int n = 0; n < TN; ++n)
              acc[m][0][n] = fmaf(__ldg(P.wt + ((size_t)g * DP + kk) * G + j0 + n), s0k, acc[m][0][n]);
          }
        }
      }
    }
#pragma unroll(DP <= 64 ? DP : 8)
    for (int kk = 0; kk < (PRE ? 0 : DP); ++kk) {
      const float4 sv = *reinterpret_cast<const float4*>(sT + kk * LP + m0);
      const float s4[4] = {sv.x, sv.y, sv.z, sv.w};
      const float* wrow = sW + kk * C::WCOLS + j0;
#pragma unroll
      for (int q = 0; q < R; ++q) {
        float w[TN];
        if constexpr (TN == 4) {
          const float4 w4 = *reinterpret_cast<const float4*>(wrow + q * G);
          w[0] = w4.x; w[1] = w4.y; w[2] = w4.z; w[3] = w4.w;
        } else if constexpr (TN == 2) {
          const float2 w2 = *reinterpret_cast<const float2*>(wrow + q * G);
          w[0] = w2.x; w[1] = w2.y;
        } else {
          w[0] = wrow[q * G];
        }
#pragma unroll
        for (int m = 0; m < TM; ++m)
#pragma unroll
          for (int n = 0; n < TN; ++n) acc[m][q][n] = fmaf(w[n], s4[m], acc[m][q][n]);
      }
    }

    // ---- 3. cell, diagonal Jacobian, affine coefficients, residual -------
    float av[TM][TN], bv[TM][TN];
#pragma unroll
    for (int n = 0; n < TN; ++n) {
      const bool cok = (n < cvalid);
      const int cw = cok ? c0 + n : 0;
#pragma unroll
      for (int m = 0; m < TM; ++m) {
        const int t = t0 + m0 + m;
        const bool ok = cok && (t < T);
        const float sp = sT[cw * LP + m0 + m];       // s^(i)_{t-1}
        const float sc = sT[cw * LP + m0 + m + 1];   // s^(i)_t
        float y, a, bb, res;
        if constexpr (CELL == PN_CELL_TANH_RNN) {
          y = tanh_pn(acc[m][0][n] + xv[m][0][n]);
          res = sc - y;
          a = (MODE == PN_QUASI) ? (1.0f - y * y) * wd[n][0] : (MODE == PN_PICARD ? 1.0f : 0.0f);
          bb = (MODE == PN_JACOBI) ? y : y - a * sp;
        } else if constexpr (CELL == PN_CELL_EULER_TANH) {
          const float gg = tanh_pn(acc[m][0][n] + xv[m][0][n]);
          const float eg = P.eps * gg;
          y = sp + eg;
          res = (sc - sp) - eg;
          if (MODE == PN_QUASI) {
            const float ed = P.eps * (1.0f - gg * gg) * wd[n][0];
            a = 1.0f + ed;
            bb = eg - ed * sp;
          } else if (MODE == PN_PICARD) {
            a = 1.0f;
            bb = eg;
          } else {
            a = 0.0f;
            bb = y;
          }
        } else {  // GRU
          const float r = sigmoidf_acc(xv[m][0][n] + acc[m][0][n]);
          const float z = sigmoidf_acc(xv[m][1][n] + acc[m][1][n]);
          const float hn = acc[m][2][n] + bhn[n];
          const float nn = tanh_pn(xv[m][2][n] + r * hn);
          y = nn + z * (sp - nn);
          res = sc - y;
          if (MODE == PN_QUASI) {
            const float omz = 1.0f - z;
            const float dn = omz * (1.0f - nn * nn);
            a = z + (sp - nn) * z * omz * wd[n][1] + dn * (r * wd[n][2] + hn * r * (1.0f - r) * wd[n][0]);
          } else {
            a = (MODE == PN_PICARD) ? 1.0f : 0.0f;
          }
          bb = (MODE == PN_JACOBI) ? y : y - a * sp;
        }
        if (ok) {
          rbits = max(rbits, abs_bits(res));
          av[m][n] = a;
          bv[m][n] = bb;
        } else {
          av[m][n] = 1.0f;   // identity element: padded steps and channels
          bv[m][n] = 0.0f;
        }
      }
    }

    if constexpr (!kScan) {
      // Jacobi: s^(i+1)_t = f_t(s^(i)_{t-1}); no recurrence to solve.
      if (cvalid > 0) {
#pragma unroll
        for (int m = 0; m < TM; ++m) {
          const int t = t0 + m0 + m;
          if (t < T) {
            float o[TN];
#pragma unroll
            for (int n = 0; n < TN; ++n) {
              o[n] = bv[m][n];
              if (damped && n < cvalid) {
                const float sc = sT[(c0 + n) * LP + m0 + m + 1];   // s^(i)_t
                o[n] = fmaf(lambda, o[n] - sc, sc);
              }
            }
            store_out(((size_t)b * T + t) * D + c0, o);
          }
        }
      }
    } else {
      // ---- 4. scan: thread-serial, then warp shuffle, then across warps --
      float IA[TN], IB[TN];
#pragma unroll
      for (int n = 0; n < TN; ++n) {
        float a_ = 1.0f, b_ = 0.0f;
#pragma unroll
        for (int m = 0; m < TM; ++m) {
          b_ = fmaf(av[m][n], b_, bv[m][n]);
          if (kHasA) a_ *= av[m][n];
        }
        IA[n] = a_;
        IB[n] = b_;
      }
      const int lt = tseg % C::TSW;
#pragma unroll
      for (int off = 1; off < C::TSW; off <<= 1) {
#pragma unroll
        for (int n = 0; n < TN; ++n) {
          const float ub = __shfl_up_sync(0xffffffffu, IB[n], off, C::TSW);
          float ua = 1.0f;
          if (kHasA) ua = __shfl_up_sync(0xffffffffu, IA[n], off, C::TSW);
          if (lt >= off) {
            IB[n] = fmaf(IA[n], ub, IB[n]);
            if (kHasA) IA[n] *= ua;
          }
        }
      }
      float EA[TN], EB[TN];   // exclusive prefix within the warp segment
#pragma unroll
      for (int n = 0; n < TN; ++n) {
        const float eb = __shfl_up_sync(0xffffffffu, IB[n], 1, C::TSW);
        float ea = 1.0f;
        if (kHasA) ea = __shfl_up_sync(0xffffffffu, IA[n], 1, C::TSW);
        EA[n] = (lt == 0) ? 1.0f : ea;
        EB[n] = (lt == 0) ? 0.0f : eb;
      }
      if constexpr (C::WPG > 1) {
        const int wg = tseg / C::TSW;
        if (lt == C::TSW - 1) {
#pragma unroll
          for (int n = 0; n < TN; ++n) {
            sPart[((jg * C::WPG + wg) * TN + n) * 2 + 0] = IA[n];
            sPart[((jg * C::WPG + wg) * TN + n) * 2 + 1] = IB[n];
          }
        }
        __syncthreads();
#pragma unroll
        for (int n = 0; n < TN; ++n) {
          float PA = 1.0f, PB = 0.0f;
          for (int w = 0; w < wg; ++w) {
            const float wa = sPart[((jg * C::WPG + w) * TN + n) * 2 + 0];
            const float wb = sPart[((jg * C::WPG + w) * TN + n) * 2 + 1];
            PB = fmaf(wa, PB, wb);
            PA *= wa;
          }
          EB[n] = fmaf(EA[n], PB, EB[n]);   // prepend the earlier warps
          EA[n] *= PA;
          IB[n] = fmaf(IA[n], PB, IB[n]);
          IA[n] *= PA;
        }
      }
      if (tseg == TS - 1) {
#pragma unroll
        for (int n = 0; n < TN; ++n) {
          sAgg[2 * (j0 + n) + 0] = IA[n];
          sAgg[2 * (j0 + n) + 1] = IB[n];
        }
      }
      __syncthreads();

      // ---- 5. decoupled look-back (warp 0) --------------------------------
      if (warp == 0) {
        const bool stall = (A.stall_ticket == (int)k);
        if (chunk > 0 && !stall) {
#pragma unroll
          for (int q = 0; q < C::NQ; ++q) {
            const int j = lane + 32 * q;
            if (j < G)
              reinterpret_cast<float2*>(P.agg + k * P.agg_stride)[j] = make_float2(sAgg[2 * j], sAgg[2 * j + 1]);
          }
          __threadfence();
          __syncwarp();
          if (lane == 0) st_release(P.flags + k, make_flag(epoch, kFlagAgg));
        }
        const int n_agg = lookback_find_prefix(P.flags, k, stride, chunk, epoch, ctrl, A.timeout_ns);
        if (n_agg >= 0) {
          float carry[C::NQ];
#pragma unroll
          for (int q = 0; q < C::NQ; ++q) {
            const int j = lane + 32 * q;
            float v = 0.0f;
            if (j < G) {
              if (chunk - 1 - n_agg >= 0) {
                v = __ldcg(P.pref + (k - (size_t)(n_agg + 1) * stride) * P.pref_stride + j);
              } else {
                const int c = g * G + j;
                v = (c < D) ? __ldg(A.s0 + (size_t)b * D + c) : 0.0f;
              }
              // fold in the aggregates, farthest first
#pragma unroll 4
              for (int d = n_agg; d >= 1; --d) {
                const float2 ab = __ldcg(reinterpret_cast<const float2*>(P.agg + (k - (size_t)d * stride) * P.agg_stride) + j);
                v = fmaf(ab.x, v, ab.y);
              }
            }
            carry[q] = v;
          }
          if (!stall) {
#pragma unroll
            for (int q = 0; q < C::NQ; ++q) {
              const int j = lane + 32 * q;
              if (j < G) P.pref[k * P.pref_stride + j] = fmaf(sAgg[2 * j], carry[q], sAgg[2 * j + 1]);
            }
            __threadfence();
            __syncwarp();
            if (lane == 0) st_release(P.flags + k, make_flag(epoch, kFlagPrefix));
          }
#pragma unroll
          for (int q = 0; q < C::NQ; ++q) {
            const int j = lane + 32 * q;
            if (j < G) sCarry[j] = carry[q];
          }
        }
        if (lane == 0) s_abort = (n_agg < 0) ? 1 : 0;
      }
      __syncthreads();

      // ---- 6. apply the carry, write s^(i+1) ------------------------------
      if (!s_abort && cvalid > 0) {
        float s[TN];
#pragma unroll
        for (int n = 0; n < TN; ++n) s[n] = fmaf(EA[n], sCarry[j0 + n], EB[n]);
#pragma unroll
        for (int m = 0; m < TM; ++m) {
          const int t = t0 + m0 + m;
          float o[TN];
#pragma unroll
          for (int n = 0; n < TN; ++n) {
            s[n] = fmaf(av[m][n], s[n], bv[m][n]);
            o[n] = s[n];
            if (damped && n < cvalid) {   // the stored iterate moves lambda of the way; the scan stays undamped
              const float sc = sT[(c0 + n) * LP + m0 + m + 1];
              o[n] = fmaf(lambda, o[n] - sc, sc);
            }
          }
          if (t < T) store_out(((size_t)b * T + t) * D + c0, o);
        }
      }
      if (s_abort) break;
    }
  }

  // ---- 7. one atomicMax per CTA, then the end-of-launch decision ----------
  rbits = warp_max_u32(rbits);
  if (lane == 0) sRed[warp] = __uint_as_float(rbits);
  __syncthreads();
  if (tid == 0) {
    unsigned v = 0u;
    for (int w = 0; w < C::NT / 32; ++w) v = max(v, __float_as_uint(sRed[w]));
    if (v) atomicMax(&ctrl->resid_bits, v);
  }
  finish_launch(P, A, epoch, s_last);
}

}  // namespace pn
