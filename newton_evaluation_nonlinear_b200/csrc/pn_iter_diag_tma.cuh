// pn_iter_diag_tma.cuh -- pipelined fused iteration kernel for the Jacobi,
// Picard and diagonal quasi-Newton modes (D a multiple of 4, 32 <= DP <= 256).
//
// Same iteration as pn_iter_diag.cuh (the page's unified update, §1.2, with
// a diagonal A~_t, §2.2.1/§2.2.3, solved by the chunked scan of §2.1), with
// the data movement split off into a producer warp:
//
//   producer warp : claims the next tile ticket of the CTA's channel group,
//                   waits until a shared-memory stage is free, and stages the
//                   tile's rows with bulk async copies (TMA, one copy per row
//                   into padded rows) completing on the stage's mbarrier:
//                     s^(i) rows t0-1 .. t0+L-1 (all D channels),
//                     step-input rows t0 .. t0+L-1 (this group's channels);
//   consumer warps: wait for the stage, run the register-tiled matvec and the
//                   cell, release the stage (so the producer refills it while
//                   they scan), scan, look back, and write s^(i+1).
//
// Consumer thread (tseg, jg) owns steps r = m*TS + tseg (m < TM) of channels
// c0 .. c0+TN-1: the TS lanes of a channel group hold TS consecutive steps, so
// a quarter warp reads 8 consecutive padded rows (conflict-free 16-byte
// shared loads), and the scan is a TS-lane shuffle scan per m followed by a
// serial combine over the TM segments.
#pragma once

#include "pn_cells.cuh"
#include "pn_tma.cuh"

namespace pn {

template <int CELL, int MODE, int DP, int G, int TM, int TN, int TS>
struct DiagTmaCfg {
  static constexpr int R = CellInfo<CELL>::R;
  static constexpr int L = TS * TM;
  static constexpr int JG = G / TN;
  static constexpr int NTC = TS * JG;             // consumer threads
  static constexpr int NCW = NTC / 32;            // consumer warps
  static constexpr int NT = NTC + 32;             // + one producer warp
  static constexpr int SP = DP + 4;               // padded s row (floats)
  static constexpr int XP = R * G + 4;            // padded step-input row (floats)
  static constexpr int WCOLS = R * G;
  static constexpr int STAGES = 2;
  static constexpr int NQ = (G + 31) / 32;
  static constexpr int STAGE_S = (L + 1) * SP;
  static constexpr int STAGE_X = L * XP;
  static constexpr int STAGE = ((STAGE_S + STAGE_X + 31) / 32) * 32;   // 128-byte aligned stages
  static constexpr int OFF_W = STAGES * STAGE;
  static constexpr int OFF_AGG = OFF_W + DP * WCOLS;
  static constexpr int OFF_CARRY = OFF_AGG + 2 * G;
  static constexpr int OFF_RED = OFF_CARRY + G;
  static constexpr int SMEM_FLOATS = OFF_RED + NT / 32;
  static constexpr size_t SMEM_BYTES = (size_t)SMEM_FLOATS * sizeof(float);
  static constexpr int MIN_BLOCKS = (SMEM_BYTES <= 110 * 1024) ? 2 : 1;
  static_assert(TS == 8 || TS == 16 || TS == 32, "TS lanes per channel group");
  static_assert(TM >= 1 && TN >= 1 && (TN == 1 || TN == 2 || TN == 4), "thread tile");
  static_assert(NTC % 32 == 0, "consumer threads");
  static_assert(DP % 4 == 0 && G % 4 == 0, "16-byte rows");
  static_assert((STAGE_S % 4) == 0 && (OFF_W % 4) == 0, "alignment");
};

template <int CELL, int MODE, int DP, int G, int TM, int TN, int TS>
__global__ void __launch_bounds__(DiagTmaCfg<CELL, MODE, DP, G, TM, TN, TS>::NT,
                                  DiagTmaCfg<CELL, MODE, DP, G, TM, TN, TS>::MIN_BLOCKS)
    diag_tma_kernel(const IterParams P) {
  using C = DiagTmaCfg<CELL, MODE, DP, G, TM, TN, TS>;
  constexpr int R = C::R;
  constexpr int L = C::L;
  constexpr int SP = C::SP;
  constexpr int XP = C::XP;
  constexpr int NTC = C::NTC;
  constexpr int STAGES = C::STAGES;
  constexpr bool kScan = (MODE != PN_JACOBI);
  constexpr bool kHasA = (MODE == PN_QUASI);

  extern __shared__ __align__(128) float smem_tma[];
  float* sW = smem_tma + C::OFF_W;
  float* sAgg = smem_tma + C::OFF_AGG;
  float* sCarry = smem_tma + C::OFF_CARRY;
  float* sRed = smem_tma + C::OFF_RED;
  __shared__ __align__(8) uint64_t s_full[STAGES];
  __shared__ __align__(8) uint64_t s_empty[STAGES];
  __shared__ int s_tk[STAGES];
  __shared__ int s_abort, s_last;
  __shared__ int s_go[2];   // ticket verdicts, double-buffered by tile parity

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  Ctrl* ctrl = P.ctrl;
  const Args A = *P.args;
  const int D = P.D, T = P.T, B = P.B;
  // damping: s^(i+1) = s^(i) + lambda * delta; the stage of s^(i) is released before the write-out,
  // so a damped write re-reads s^(i)_t (the scan itself stays undamped)
  const float lambda = A.damping;
  const bool damped = lambda != 1.0f;
  const int g = (int)(blockIdx.x % (unsigned)P.ngroups);
  const size_t stride = (size_t)B * P.ngroups;
  const int gw = min(G, D - g * G);   // channels of this group present in D (multiple of 4)

  if (tid == 0) {
    atomicMin(&ctrl->t_start, globaltimer());
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&s_full[s], 1u);
      mbar_init(&s_empty[s], (unsigned)C::NCW);
    }
    mbar_init_fence();
    s_abort = 0;
  }
  const unsigned epoch = *(volatile unsigned*)&ctrl->epoch;
  const int iter = *(volatile int*)&ctrl->iter;
  const float* __restrict__ src = (iter & 1) ? P.buf1 : A.states;
  float* __restrict__ dst = (iter & 1) ? A.states : P.buf1;

  // columns the copies never write: zero them once (s beyond D, inputs beyond gw)
  for (int s = 0; s < STAGES; ++s) {
    float* S = smem_tma + s * C::STAGE;
    float* X = S + C::STAGE_S;
    for (int e = tid; e < (L + 1) * (SP - D); e += C::NT) S[(e / (SP - D)) * SP + D + e % (SP - D)] = 0.0f;
    for (int e = tid; e < L * XP; e += C::NT) {
      const int col = e % XP;
      if (col >= R * G || (col % G) >= gw) X[e] = 0.0f;
    }
  }
  {
    const float4* wsrc = reinterpret_cast<const float4*>(P.wt + (size_t)g * DP * C::WCOLS);
    float4* wdst = reinterpret_cast<float4*>(sW);
    for (int e = tid; e < DP * C::WCOLS / 4; e += C::NT) wdst[e] = __ldg(wsrc + e);
  }
  __syncthreads();

  unsigned rbits = 0u;

  if (warp == C::NCW) {
    // ======================= producer warp =================================
    const float* xin = (CELL == PN_CELL_EULER_TANH) ? A.x : P.xin;
    int it = 0;
    bool ok = true;
    for (;; ++it) {
      const int stage = it % STAGES;
      const unsigned ph = (unsigned)(it / STAGES) & 1u;
      if (it >= STAGES && !mbar_wait(&s_empty[stage], ph ^ 1u, ctrl, A.timeout_ns)) { ok = false; break; }
      int kg = 0;
      if (lane == 0) kg = (int)atomicAdd(&ctrl->ticket[g], 1u);
      kg = __shfl_sync(0xffffffffu, kg, 0);
      if (kg >= P.tiles_per_group) {
        if (lane == 0) {
          s_tk[stage] = -1;
          mbar_arrive(&s_full[stage]);
        }
        ++it;
        break;
      }
      const int b = kg % B;
      const int t0 = (kg / B) * L;
      const int s_rows = min(L + 1, T - t0 + 1);   // rows r with t0-1+r < T (t = -1 is s0)
      const int x_rows = min(L, T - t0);
      const unsigned bytes = (unsigned)(s_rows * D + x_rows * R * gw) * 4u;
      float* S = smem_tma + stage * C::STAGE;
      float* X = S + C::STAGE_S;
      if (lane == 0) {
        s_tk[stage] = kg;
        mbar_arrive_expect_tx(&s_full[stage], bytes);
      }
      __syncwarp();
      for (int r = lane; r < s_rows; r += 32) {
        const int t = t0 - 1 + r;
        const float* row = (t < 0) ? A.s0 + (size_t)b * D : src + ((size_t)b * T + t) * D;
        bulk_copy_g2s(S + r * SP, row, (unsigned)D * 4u, &s_full[stage]);
      }
      for (int e = lane; e < x_rows * R; e += 32) {
        const int r = e / R;
        const int q = e % R;
        const float* row = xin + ((size_t)b * T + t0 + r) * (R * D) + (size_t)q * D + (size_t)g * G;
        bulk_copy_g2s(X + r * XP + q * G, row, (unsigned)gw * 4u, &s_full[stage]);
      }
    }
    // drain: every issued fill must land before the CTA may exit
    for (int j = max(0, it - STAGES); j < it; ++j)
      if (!mbar_drain(&s_full[j % STAGES], (unsigned)(j / STAGES) & 1u, A.timeout_ns) && lane == 0)
        raise_error(ctrl, (int)PN_ERR_TIMEOUT);
    (void)ok;
  } else {
    // ======================= consumer warps ================================
    const int tseg = tid % TS;
    const int jg = tid / TS;
    const int j0 = jg * TN;
    const int c0 = g * G + j0;
    const int cvalid = max(0, min(TN, D - c0));
    float wd[TN][R];
    float bhn[TN];
#pragma unroll
    for (int n = 0; n < TN; ++n) {
      const int cw = (n < cvalid) ? c0 + n : 0;
#pragma unroll
      for (int q = 0; q < R; ++q) wd[n][q] = sW[cw * C::WCOLS + q * G + j0 + n];
      bhn[n] = (CELL == PN_CELL_GRU && n < cvalid) ? __ldg(P.bhn + c0 + n) : 0.0f;
    }

    for (int it = 0;; ++it) {
      const int stage = it % STAGES;
      const unsigned ph = (unsigned)(it / STAGES) & 1u;
      // one thread polls the stage (bounded) and broadcasts the verdict, so
      // every consumer warp takes the same exit decision
      if (tid == 0) s_go[it & 1] = mbar_wait(&s_full[stage], ph, ctrl, A.timeout_ns) ? s_tk[stage] : -2;
      named_barrier(1, NTC);
      const int kg = s_go[it & 1];
      if (kg < 0) break;
      mbar_try_wait(&s_full[stage], ph);   // completed: gives this thread its own acquire of the copies
      const int b = kg % B;
      const int chunk = kg / B;
      const int t0 = chunk * L;
      const size_t k = (size_t)kg * P.ngroups + g;
      const float* S = smem_tma + stage * C::STAGE;
      const float* X = S + C::STAGE_S;

      // ---- matvec ----------------------------------------------------------
      float acc[TM][R][TN];
#pragma unroll
      for (int m = 0; m < TM; ++m)
#pragma unroll
        for (int q = 0; q < R; ++q)
#pragma unroll
          for (int n = 0; n < TN; ++n) acc[m][q][n] = 0.0f;
#pragma unroll(DP <= 64 ? DP / 4 : 4)
      for (int kk = 0; kk < DP; kk += 4) {
        float4 sv[TM];
#pragma unroll
        for (int m = 0; m < TM; ++m) sv[m] = *reinterpret_cast<const float4*>(S + (m * TS + tseg) * SP + kk);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float* wrow = sW + (kk + u) * C::WCOLS + j0;
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
            for (int m = 0; m < TM; ++m) {
              const float s = (u == 0) ? sv[m].x : (u == 1) ? sv[m].y : (u == 2) ? sv[m].z : sv[m].w;
#pragma unroll
              for (int n = 0; n < TN; ++n) acc[m][q][n] = fmaf(w[n], s, acc[m][q][n]);
            }
          }
        }
      }

      // ---- cell, diagonal Jacobian, affine coefficients, residual ----------
      float av[TM][TN], bv[TM][TN];
#pragma unroll
      for (int m = 0; m < TM; ++m) {
        const int r = m * TS + tseg;
        const int t = t0 + r;
        float xv[R][TN];
#pragma unroll
        for (int q = 0; q < R; ++q) {
          const float* xr = X + r * XP + q * G + j0;
          if constexpr (TN == 4) {
            const float4 v = *reinterpret_cast<const float4*>(xr);
            xv[q][0] = v.x; xv[q][1] = v.y; xv[q][2] = v.z; xv[q][3] = v.w;
          } else if constexpr (TN == 2) {
            const float2 v = *reinterpret_cast<const float2*>(xr);
            xv[q][0] = v.x; xv[q][1] = v.y;
          } else {
            xv[q][0] = xr[0];
          }
        }
#pragma unroll
        for (int n = 0; n < TN; ++n) {
          const bool cok = (n < cvalid);
          const int cw = cok ? c0 + n : 0;
          const bool ok = cok && (t < T);
          const float sp = S[r * SP + cw];         // s^(i)_{t-1}
          const float sc = S[(r + 1) * SP + cw];   // s^(i)_t
          float y, a, bb, res;
          if constexpr (CELL == PN_CELL_TANH_RNN) {
            y = tanh_pn(acc[m][0][n] + xv[0][n]);
            res = sc - y;
            a = (MODE == PN_QUASI) ? (1.0f - y * y) * wd[n][0] : (MODE == PN_PICARD ? 1.0f : 0.0f);
            bb = (MODE == PN_JACOBI) ? y : y - a * sp;
          } else if constexpr (CELL == PN_CELL_EULER_TANH) {
            const float gg = tanh_pn(acc[m][0][n] + xv[0][n]);
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
            const float rr = sigmoidf_acc(xv[0][n] + acc[m][0][n]);
            const float z = sigmoidf_acc(xv[1][n] + acc[m][1][n]);
            const float hn = acc[m][2][n] + bhn[n];
            const float nn = tanh_pn(xv[2][n] + rr * hn);
            y = nn + z * (sp - nn);
            res = sc - y;
            if (MODE == PN_QUASI) {
              const float omz = 1.0f - z;
              const float dn = omz * (1.0f - nn * nn);
              a = z + (sp - nn) * z * omz * wd[n][1] + dn * (rr * wd[n][2] + hn * rr * (1.0f - rr) * wd[n][0]);
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
            av[m][n] = 1.0f;   // identity: padded steps and channels
            bv[m][n] = 0.0f;
          }
        }
      }
      // every read of this stage is done: hand it back to the producer
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[stage]);

      if constexpr (!kScan) {
        if (cvalid > 0) {
#pragma unroll
          for (int m = 0; m < TM; ++m) {
            const int t = t0 + m * TS + tseg;
            if (t < T) {
              float o[TN];
#pragma unroll
              for (int n = 0; n < TN; ++n) {
                o[n] = bv[m][n];
                if (damped && n < cvalid) {
                  const float sc = __ldg(src + ((size_t)b * T + t) * D + c0 + n);
                  o[n] = fmaf(lambda, o[n] - sc, sc);
                }
              }
              store_n<TN>(dst + ((size_t)b * T + t) * D + c0, o, cvalid, (D % TN) == 0);
            }
          }
        }
      } else {
        // ---- scan: TS-lane shuffle scan per segment m, then over m ---------
        float PA[TN], PB[TN];
#pragma unroll
        for (int n = 0; n < TN; ++n) { PA[n] = 1.0f; PB[n] = 0.0f; }
#pragma unroll
        for (int m = 0; m < TM; ++m) {
#pragma unroll
          for (int n = 0; n < TN; ++n) {
            float a_ = av[m][n], b_ = bv[m][n];
#pragma unroll
            for (int off = 1; off < TS; off <<= 1) {
              const float ub = __shfl_up_sync(0xffffffffu, b_, off, TS);
              float ua = 1.0f;
              if (kHasA) ua = __shfl_up_sync(0xffffffffu, a_, off, TS);
              if (tseg >= off) {
                b_ = fmaf(a_, ub, b_);
                if (kHasA) a_ *= ua;
              }
            }
            const float tb = __shfl_sync(0xffffffffu, b_, TS - 1, TS);
            float ta = 1.0f;
            if (kHasA) ta = __shfl_sync(0xffffffffu, a_, TS - 1, TS);
            // inclusive prefix of this element within the tile: segments < m, then lanes <= tseg
            bv[m][n] = fmaf(a_, PB[n], b_);
            av[m][n] = kHasA ? a_ * PA[n] : 1.0f;
            PB[n] = fmaf(ta, PB[n], tb);
            if (kHasA) PA[n] *= ta;
          }
        }
        if (tseg == 0) {
#pragma unroll
          for (int n = 0; n < TN; ++n) {
            sAgg[2 * (j0 + n) + 0] = PA[n];
            sAgg[2 * (j0 + n) + 1] = PB[n];
          }
        }
        named_barrier(1, NTC);

        // ---- decoupled look-back (consumer warp 0) ---------------------------
        if (warp == 0) {
          const bool stall = (A.stall_ticket == (int)k);
          if (chunk > 0 && !stall) {
#pragma unroll
            for (int q = 0; q < C::NQ; ++q) {
              const int j = lane + 32 * q;
              if (j < G)
                reinterpret_cast<float2*>(P.agg + k * P.agg_stride)[j] = make_float2(sAgg[2 * j], sAgg[2 * j + 1]);
            }
            __syncwarp();
            if (lane == 0) {
              __threadfence();
              st_release(P.flags + k, make_flag(epoch, kFlagAgg));
            }
          }
          const int n_agg = lookback_find_prefix(P.flags, k, stride, chunk, epoch, ctrl, A.timeout_ns);
          __syncwarp();
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
#pragma unroll 4
                for (int d = n_agg; d >= 1; --d) {
                  const float2 ab =
                      __ldcg(reinterpret_cast<const float2*>(P.agg + (k - (size_t)d * stride) * P.agg_stride) + j);
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
              __syncwarp();
              if (lane == 0) {
                __threadfence();
                st_release(P.flags + k, make_flag(epoch, kFlagPrefix));
              }
            }
#pragma unroll
            for (int q = 0; q < C::NQ; ++q) {
              const int j = lane + 32 * q;
              if (j < G) sCarry[j] = carry[q];
            }
          }
          if (lane == 0) s_abort = (n_agg < 0) ? 1 : 0;
        }
        named_barrier(1, NTC);
        if (s_abort) break;

        // ---- apply the carry, write s^(i+1) ---------------------------------
        if (cvalid > 0) {
          float cr[TN];
#pragma unroll
          for (int n = 0; n < TN; ++n) cr[n] = sCarry[j0 + n];
#pragma unroll
          for (int m = 0; m < TM; ++m) {
            const int t = t0 + m * TS + tseg;
            float o[TN];
#pragma unroll
            for (int n = 0; n < TN; ++n) {
              o[n] = fmaf(av[m][n], cr[n], bv[m][n]);
              if (damped && n < cvalid && t < T) {
                const float sc = __ldg(src + ((size_t)b * T + t) * D + c0 + n);
                o[n] = fmaf(lambda, o[n] - sc, sc);
              }
            }
            if (t < T) store_n<TN>(dst + ((size_t)b * T + t) * D + c0, o, cvalid, (D % TN) == 0);
          }
        }
      }
    }
  }

  // ---- one atomicMax per CTA, then the end-of-launch decision --------------
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
