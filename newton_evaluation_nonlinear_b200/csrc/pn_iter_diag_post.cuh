// pn_iter_diag_post.cuh -- the Jacobi, Picard and diagonal quasi-Newton
// iteration of the wide one-gate cells (tanh RNN, Euler drift at D = 128,
// 256) once the tensor cores have formed every step's recurrent product.
//
// Same iteration as pn_iter_diag.cuh (the page's unified update, "Parallel
// Newton methods..." page §1.2, with a diagonal A~_t, §2.2.1 / §2.2.3, solved
// by the chunked scan of §2.1).  With Y = S W^T computed for every step by
// wide_gemm_kernel (row b T + t - 1 holds W s^(i)_{t-1} for step t), all that
// is left of an iteration is per channel: the cell, the diagonal Jacobian,
// the residual, and a scalar affine recurrence.  So one thread owns one
// channel of a tile (sequence b, chunk of L steps, group of G channels) and
// walks its L steps in order, the loads of U steps in flight ahead of the
// arithmetic; the tile's aggregate goes to the decoupled look-back, in which
// every thread folds its own channel; the carry then turns the in-register
// prefixes into the states.  Every global access is a row of G consecutive
// floats.  Step 0 of a sequence forms W s0 itself (from the dense weight copy,
// W[c][k] at k DP + c).
#pragma once

#include "pn_cells.cuh"

namespace pn {

template <int CELL, int MODE, int DP>
struct PostCfg {
  static constexpr int G = DP < 128 ? DP : 128;   // channels per tile, one thread each
  static constexpr int NT = G;
  static constexpr int L = 32;                    // steps per tile
  static constexpr int U = 8;                     // steps whose loads are issued together
  static_assert(CellInfo<CELL>::R == 1, "one-gate cells");
  static_assert(DP % G == 0 && G % 32 == 0 && L % U == 0, "tile shape");
};

template <int CELL, int MODE, int DP>
__global__ void __launch_bounds__(PostCfg<CELL, MODE, DP>::NT) diag_post_kernel(const IterParams P) {
  using C = PostCfg<CELL, MODE, DP>;
  constexpr int G = C::G;
  constexpr int L = C::L;
  constexpr int U = C::U;
  constexpr int NT = C::NT;
  constexpr bool kScan = (MODE != PN_JACOBI);
  constexpr bool kHasA = (MODE == PN_QUASI);
  __shared__ int s_ticket, s_nagg, s_last;
  __shared__ float sRed[NT / 32];

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  Ctrl* ctrl = P.ctrl;
  const Args A = *P.args;
  const int D = P.D, T = P.T, B = P.B;
  const float lambda = A.damping;   // s^(i+1) = s^(i) + lambda * delta
  const bool damped = lambda != 1.0f;
  const int g = (int)(blockIdx.x % (unsigned)P.ngroups);
  const size_t stride = (size_t)B * P.ngroups;   // descriptor distance between consecutive chunks

  if (tid == 0) atomicMin(&ctrl->t_start, globaltimer());
  const unsigned epoch = *(volatile unsigned*)&ctrl->epoch;
  const int iter = *(volatile int*)&ctrl->iter;
  const float* __restrict__ src = (iter & 1) ? P.buf1 : A.states;
  float* __restrict__ dst = (iter & 1) ? A.states : P.buf1;
  const float* __restrict__ xin = (CELL == PN_CELL_EULER_TANH) ? A.x : P.xin;   // [B][T][D]

  const int c = g * G + tid;   // this thread's channel
  const bool cok = c < D;
  const float wdc = (kHasA && cok) ? __ldg(P.wdiag + c) : 0.0f;
  unsigned rbits = 0u;

  for (;;) {
    __syncthreads();   // every thread has read the previous ticket and shared words
    if (tid == 0) s_ticket = (int)atomicAdd(&ctrl->ticket[g], 1u);
    __syncthreads();
    const int kg = s_ticket;
    if (kg >= P.tiles_per_group) break;
    const int b = kg % B;
    const int chunk = kg / B;
    const int t0 = chunk * L;
    const int n = min(L, T - t0);
    const size_t k = (size_t)kg * P.ngroups + g;   // descriptor index of this tile
    const size_t row0 = (size_t)b * T + t0;        // row of step t0

    // s^(i)_{t0-1} and, for the first chunk, W s0
    float sp0 = 0.0f, z0 = 0.0f;
    if (cok) {
      if (t0 == 0) {
        const float* s0 = A.s0 + (size_t)b * D;
        sp0 = __ldg(s0 + c);
        for (int kk = 0; kk < D; ++kk) z0 = fmaf(__ldg(P.wt + (size_t)kk * DP + c), __ldg(s0 + kk), z0);
      } else {
        sp0 = __ldg(src + (row0 - 1) * DP + c);
      }
    }
    // the cell, the diagonal Jacobian a_t, b_t = y_t - a_t s_{t-1} and F_t of a step from its loads:
    // (a, b, F)
    auto coef = [&](float z, float x, float sc, float sp) -> float3 {
      float a, bb, res;
      if constexpr (CELL == PN_CELL_TANH_RNN) {
        const float y = tanh_pn(z + x);
        res = sc - y;
        a = (MODE == PN_QUASI) ? (1.0f - y * y) * wdc : (MODE == PN_PICARD ? 1.0f : 0.0f);
        bb = (MODE == PN_JACOBI) ? y : y - a * sp;
      } else {
        const float gg = tanh_pn(z + x);
        const float eg = P.eps * gg;
        res = (sc - sp) - eg;
        if (MODE == PN_QUASI) {
          const float ed = P.eps * (1.0f - gg * gg) * wdc;
          a = 1.0f + ed;
          bb = eg - ed * sp;
        } else if (MODE == PN_PICARD) {
          a = 1.0f;
          bb = eg;
        } else {
          a = 0.0f;
          bb = sp + eg;
        }
      }
      return make_float3(a, bb, res);
    };
    // the loads of U steps from m0 on (all in flight together); rows are DP floats apart (the wide
    // path runs only with D == DP), so every address is a base plus an immediate offset
    const float* zrow = P.ypre + (row0 - 1) * DP + c;   // row of step t0 - 1 (never read for t = 0)
    const float* xrow = xin + row0 * DP + c;
    const float* srow = src + row0 * DP + c;
    auto load = [&](int m0, float (&zv)[U], float (&xv)[U], float (&sv)[U]) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int m = m0 + u;
        const bool ok = cok && m < n;
        zv[u] = (ok && (t0 + m) > 0) ? __ldg(zrow + m * DP) : z0;
        xv[u] = ok ? __ldg(xrow + m * DP) : 0.0f;
        sv[u] = ok ? __ldg(srow + m * DP) : 0.0f;
      }
    };

    // ---- the residual, the tile's aggregate and its in-tile prefixes (Jacobi: the states)
    float SA = 1.0f, SB = 0.0f;
    float pa[L], pb[L];
    {
      float sp = sp0;
#pragma unroll
      for (int m0 = 0; m0 < L; m0 += U) {
        float zv[U], xv[U], sv[U];
        load(m0, zv, xv, sv);
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int m = m0 + u;
          const bool ok = cok && m < n;
          const float3 f = coef(zv[u], xv[u], sv[u], sp);
          float a = f.x, bb = f.y;
          if (ok) {
            rbits = max(rbits, abs_bits(f.z));
            if constexpr (!kScan) dst[(row0 + m) * DP + c] = damped ? fmaf(lambda, bb - sv[u], sv[u]) : bb;
          } else {
            a = 1.0f;   // identity element: steps past T, channels past D
            bb = 0.0f;
          }
          SB = fmaf(a, SB, bb);
          if (kHasA) SA *= a;
          pa[m] = SA;
          pb[m] = SB;
          sp = sv[u];
        }
      }
    }
    if constexpr (!kScan) continue;

    // ---- decoupled look-back: this tile's aggregate, the nearest published state, the carry.
    // The barrier orders every thread's words before the releasing store (a cumulative release).
    // Every thread writes its channel's words; the barrier orders them before the one releasing
    // store of the flag (a release covers what precedes it in causality order).  Warp 0 acquires
    // the predecessors' flags; the barrier after it orders every thread's loads of their words.
    const bool stall = (A.stall_ticket == (int)k);
    if (chunk > 0 && !stall) reinterpret_cast<float2*>(P.agg + k * P.agg_stride)[tid] = make_float2(SA, SB);
    __syncthreads();
    if (warp == 0) {
      if (lane == 0 && chunk > 0 && !stall) st_release(P.flags + k, make_flag(epoch, kFlagAgg));
      const int na = lookback_find_prefix(P.flags, k, stride, chunk, epoch, ctrl, A.timeout_ns);
      if (lane == 0) s_nagg = na;
    }
    __syncthreads();
    const int n_agg = s_nagg;
    if (n_agg < 0) break;   // a wait gave up: the error is set, the launch winds down
    float carry;
    if (chunk - 1 - n_agg >= 0) carry = __ldcg(P.pref + (k - (size_t)(n_agg + 1) * stride) * P.pref_stride + tid);
    else carry = cok ? __ldg(A.s0 + (size_t)b * D + c) : 0.0f;
    // the aggregates n_agg .. 1 places back, farthest first, four loads in flight
    for (int d = n_agg; d >= 1; d -= 4) {
      float2 ab[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        ab[u] = (d - u >= 1) ? __ldcg(reinterpret_cast<const float2*>(P.agg + (k - (size_t)(d - u) * stride) * P.agg_stride) + tid)
                             : make_float2(1.0f, 0.0f);
#pragma unroll
      for (int u = 0; u < 4; ++u) carry = fmaf(ab[u].x, carry, ab[u].y);
    }
    if (!stall) P.pref[k * P.pref_stride + tid] = fmaf(SA, carry, SB);
    __syncthreads();
    if (tid == 0 && !stall) st_release(P.flags + k, make_flag(epoch, kFlagPrefix));

    // ---- the states of the tile: s_t = A_t carry + B_t, damped against s^(i)_t
    if (cok) {
#pragma unroll
      for (int m = 0; m < L; ++m) {
        if (m < n) {
          const float v = fmaf(pa[m], carry, pb[m]);
          float o = v;
          if (damped) {
            const float sc = __ldg(srow + m * DP);
            o = fmaf(lambda, v - sc, sc);
          }
          dst[(row0 + m) * DP + c] = o;
        }
      }
    }
  }

  // ---- one atomicMax per CTA, then the end-of-launch decision
  rbits = warp_max_u32(rbits);
  if (lane == 0) sRed[warp] = __uint_as_float(rbits);
  __syncthreads();
  if (tid == 0) {
    unsigned v = 0u;
    for (int w = 0; w < NT / 32; ++w) v = max(v, __float_as_uint(sRed[w]));
    if (v) atomicMax(&ctrl->resid_bits, v);
  }
  finish_launch(P, A, epoch, s_last);
}

}  // namespace pn
