// pn_iter_dense_warp.cuh -- fused Newton iteration with one warp per tile
// (dense or banded Jacobian, D <= 32), FP32.
//
// The iteration is the page's unified update with J~ = J ("Parallel Newton
// methods..." page, §1.2), or its banded approximation (§2.2.2):
//     s^(i+1)_t = A_t s^(i+1)_{t-1} + b_t,  A_t = df_t/ds(s^(i)_{t-1}),
//     b_t = f_t(s^(i)_{t-1}) - A_t s^(i)_{t-1},
// solved by the affine scan of §2.1 with the combine (A,b) o (A',b') =
// (A'A, A'b + b') over chunks of L steps and a decoupled look-back between
// chunks.  Every Jacobian of the three cells is a row-scaled sum of fixed
// matrices, A_t = diag(c0_t) + sum_q diag(c_{q,t}) W_q, so a step stores only
// its coefficient vectors, never A_t itself.
//
// One warp owns one tile (sequence b, steps t0 .. t0+L-1) from start to end,
// so the chain needs no block-wide barrier:
//   1. stage s^(i) rows t0-1 .. t0+L-1 and the step inputs in the warp's slice
//      of shared memory;
//   2. cell phase, lane = step: y = f_t(s_{t-1}), the coefficient vectors, b_t
//      and |F_t|, with W from shared memory (broadcast reads);
//   3. chain [P | q] <- A_m [P | q] + [0 | b_m], m = 1 .. L-1, from
//      [A_0 | b_0]: lane (rg, cg) holds rows 4 rg .. 4 rg + 3 and columns
//      cg CPL .. of P in registers and reads P_{m-1} back from shared memory
//      (one warp-synchronous exchange per step).  With a band k the inner
//      product runs only over the band's columns of W, 4 + 2k of them instead
//      of D: the banded mode costs less than the dense one.  q is a matvec
//      split over the column-group lanes and reduced with shuffles;
//   4. decoupled look-back: publish [P_L | q_L], find the nearest published
//      state, fold the aggregates in between (one matvec each), publish the
//      tile's end state P_L carry + q_L;
//   5. apply the carry sequentially, s_m = A_m s_{m-1} + b_m (a matvec per
//      step, D^2 instead of the D^3 of the chain), stage the states and write
//      them out (damped: s^(i) + lambda (s - s^(i))).
// Padded steps (t >= T) and channels (i >= D) are identity maps.
#pragma once

#include "pn_cells.cuh"

namespace pn {

template <int CELL, int DP, int NWARP>
struct DenseWarpCfg {
  static constexpr int R = CellInfo<CELL>::R;
  static constexpr int L = 32;                          // steps per chunk
  static constexpr int RPL = (DP == 4) ? 4 : 2;         // P rows per lane in the chain
  static constexpr int RG = DP / RPL;                   // row groups
  static constexpr int CG = (32 / RG < DP) ? 32 / RG : DP;   // column groups
  static constexpr int NA = RG * CG;                    // lanes active in the chain and the matvecs
  static constexpr int CPL = DP / CG;                   // P columns per lane = k-slice per lane
  static constexpr bool WREG = (R == 1);                // the chain keeps its W rows in registers
  static constexpr int SPP = 32 / DP;                   // cell phase: steps per pass (lane = channel)
  static constexpr int NCS = R + 1;                     // coefficient vectors per step: c0, c_1 .. c_R
  static constexpr int SP = DP + 4;                     // row stride of the staged s rows (16-byte rows)
  static constexpr int UP = R * DP + 1;                 // row stride of the staged step inputs
  // row stride of P: the lanes of one store phase (rows r0, r0 + RPL of neighbouring row groups)
  // land in disjoint banks (D = 16: 8 lanes x 16 bytes, row groups 48 words apart; D = 8: 32 lanes,
  // row groups 24 words apart); other widths keep D
  static constexpr int PS = (DP == 16) ? 24 : (DP == 8 ? 12 : DP);
  static constexpr int a4(int v) { return (v + 3) / 4 * 4; }
  // per-warp shared memory, in floats
  static constexpr int O_S = 0;                         // s^(i) rows t0-1 .. t0+L-1: [L+1][SP]
  static constexpr int O_U = a4(O_S + (L + 1) * SP);    // step inputs [L][UP]
  static constexpr int O_C = a4(O_U + L * UP);          // coefficients [L][NCS][DP]
  static constexpr int O_B = O_C + L * NCS * DP;        // b_m [L][DP]
  static constexpr int O_P = O_B + L * DP;              // P double buffer [2][DP][PS]
  static constexpr int O_Q = O_P + 2 * DP * PS;         // q double buffer [2][DP]
  static constexpr int O_O = O_U;                       // new states [L][DP], over the step inputs
                                                        // (consumed by the cell phase before)
  static constexpr int O_X = O_Q + 2 * DP;              // carry and fold scratch [2][DP]
  static constexpr int WARP_FLOATS = a4(O_X + 2 * DP);
  // per-CTA: W_q^T for the cell [DP][R*DP] (k-major rows: W_q[i][k] at k*R*DP + q*DP + i), the banded
  // copy used by the Jacobian (same layout), then the warps' slices
  static constexpr int C_WF = 0;
  static constexpr int C_WB = C_WF + DP * R * DP;
  static constexpr int C_WARPS = C_WB + DP * R * DP;
  static constexpr int C_RED = C_WARPS + NWARP * WARP_FLOATS;
  static constexpr int SMEM_FLOATS = C_RED + NWARP;
  static constexpr size_t SMEM_BYTES = (size_t)SMEM_FLOATS * sizeof(float);
  static constexpr int NT = 32 * NWARP;
  // two CTAs per SM where the shared memory allows (the register budget follows)
  static constexpr int MINB = (2 * (SMEM_BYTES + 1024) <= 228 * 1024) ? 2 : 1;
  static_assert(DP % 4 == 0 && DP <= 32, "DP in {4, 8, 16, 32}");
  static_assert(NA <= 32 && RG * RPL == DP && CG * CPL == DP, "lane grid");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

// N consecutive floats from shared memory (16-, 8- or 4-byte loads)
template <int N>
__device__ __forceinline__ void lds_n(const float* p, float (&v)[N]) {
  if constexpr (N % 4 == 0) {
#pragma unroll
    for (int e = 0; e < N; e += 4) {
      const float4 t = *reinterpret_cast<const float4*>(p + e);
      v[e] = t.x; v[e + 1] = t.y; v[e + 2] = t.z; v[e + 3] = t.w;
    }
  } else if constexpr (N == 2) {
    const float2 t = *reinterpret_cast<const float2*>(p);
    v[0] = t.x; v[1] = t.y;
  } else {
#pragma unroll
    for (int e = 0; e < N; ++e) v[e] = p[e];
  }
}

// The chain at D = 16 on the tensor cores (one-gate cells; banded: W is the band-masked copy, at the
// dense cost -- the tensor cores gain nothing from the zeros).  With Q = P^T the step
// P_m = (diag(c0) + diag(c1) W) P_{m-1} reads Q_m = Q_{m-1} diag(c0) + (Q_{m-1} W^T) diag(c1): a
// 16 x 16 x 16 product with the constant W^T as the B operand.  Q lives in the f32 accumulator
// layout of the m16n8k8 TF32 MMA (lane = 4 g + i holds rows g, g + 8 and columns 2 i, 2 i + 1 of
// each 8-column tile j), and that layout is also an A operand once the K index is relabelled: in
// K-step s, A column i stands for Q column 8 s + 2 i and column i + 4 for 8 s + 2 i + 1, and the B
// fragments hold W^T's rows in the same order.  So one step needs no data movement between lanes.
// Products are 3xTF32 (hi hi + hi lo + lo hi, hi the operand with its low 13 mantissa bits
// cleared), the two small passes in an accumulator of their own.
__device__ __forceinline__ uint32_t tf32_hi_bits(float x) { return __float_as_uint(x) & 0xFFFFE000u; }
__device__ __forceinline__ void mma_m16n8k8_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// One chain step on q = Q_{m-1} (q[j][e]: row g + 8 (e >> 1), column 8 j + 2 i + (e & 1)), with
// bh / bl the hi / lo B fragments (bh[s][j][h] = W[8 j + g][8 s + 2 i + h]) and c0 / c1 the
// scalings of this lane's columns (c[j][h] for column 8 j + 2 i + h).
__device__ __forceinline__ void chain_step_mma16(float (&q)[2][4], const uint32_t (&bh)[2][2][2],
                                                 const uint32_t (&bl)[2][2][2], const float (&c0)[2][2],
                                                 const float (&c1)[2][2]) {
  uint32_t ah[2][4], al[2][4];
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    const float v[4] = {q[s][0], q[s][2], q[s][1], q[s][3]};   // A rows g, g + 8 x columns i, i + 4
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      ah[s][e] = tf32_hi_bits(v[e]);
      al[s][e] = tf32_hi_bits(v[e] - __uint_as_float(ah[s][e]));
    }
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    float hh[4] = {0.0f, 0.0f, 0.0f, 0.0f}, lo[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      mma_m16n8k8_tf32(hh, ah[s], bh[s][j]);
      mma_m16n8k8_tf32(lo, ah[s], bl[s][j]);
      mma_m16n8k8_tf32(lo, al[s], bh[s][j]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) q[j][e] = fmaf(c1[j][e & 1], hh[e] + lo[e], c0[j][e & 1] * q[j][e]);
  }
}

template <int CELL, int DP, int NWARP>
__global__ void __launch_bounds__(32 * NWARP, DenseWarpCfg<CELL, DP, NWARP>::MINB) dense_warp_kernel(const IterParams P) {
  using C = DenseWarpCfg<CELL, DP, NWARP>;
  constexpr int R = C::R;
  constexpr int L = C::L;
  constexpr int NCS = C::NCS;
  constexpr int CG = C::CG;
  constexpr int CPL = C::CPL;
  constexpr int RPL = C::RPL;
  constexpr int SP = C::SP;
  constexpr int UP = C::UP;
  constexpr int PS = C::PS;
  constexpr int WR = R * DP;   // row length of the transposed weights

  extern __shared__ __align__(16) float smem_dw[];
  float* sWf = smem_dw + C::C_WF;
  float* sWb = smem_dw + C::C_WB;
  float* sRed = smem_dw + C::C_RED;
  __shared__ int s_last;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  float* ws = smem_dw + C::C_WARPS + warp * C::WARP_FLOATS;
  float* sS = ws + C::O_S;
  float* sU = ws + C::O_U;
  float* sC = ws + C::O_C;
  float* sB = ws + C::O_B;
  float* sP = ws + C::O_P;
  float* sQ = ws + C::O_Q;
  float* sO = ws + C::O_O;
  float* sX = ws + C::O_X;

  Ctrl* ctrl = P.ctrl;
  const Args A = *P.args;
  const int D = P.D, T = P.T, B = P.B;
  const int band = A.newton_band;
  const bool banded = band >= 0 && band < D - 1;
  const float lambda = A.damping;
  const bool damped = lambda != 1.0f;
  const size_t stride = (size_t)B;

  if (tid == 0) atomicMin(&ctrl->t_start, globaltimer());
  // iteration and look-back epoch of this launch's first iteration; with P.persist each further
  // iteration of the launch adds one to both (the grid barrier's last CTA advances the control block)
  const unsigned gen0 = *(volatile unsigned*)&ctrl->gen;
  const unsigned epoch0 = *(volatile unsigned*)&ctrl->epoch;
  const int iter0 = *(volatile int*)&ctrl->iter;
  const float* xin = (CELL == PN_CELL_EULER_TANH) ? A.x : P.xin;

  // weights: the cell's W_q^T, and the copy the Jacobian uses (band-masked when banded)
  for (int e = tid; e < DP * WR; e += C::NT) {
    const float w = __ldg(P.wt + e);   // W_q[i][k] at k * R * DP + q * DP + i
    sWf[e] = w;
    const int k = e / WR;
    const int i = e % DP;
    sWb[e] = (banded && abs(i - k) > band) ? 0.0f : w;
  }
  __syncthreads();
  const float* sWj = banded ? sWb : sWf;

  // chain / matvec lane grid: rows r0 .. r0 + RPL - 1, P columns (= k-slice) cg CPL .. cg CPL + CPL - 1
  const bool act = lane < C::NA;
  const int rg = act ? lane / CG : 0;
  const int cg = act ? lane % CG : 0;
  const int r0 = RPL * rg;
  const int j0 = cg * CPL;
  // band-limited k range of the chain's inner product for these rows
  const int klo = banded ? max(0, r0 - band) : 0;
  const int khi = banded ? min(DP - 1, r0 + RPL - 1 + band) : DP - 1;
  // cell phase: lane = channel ci of step group ms (SPP steps per pass)
  const int ci = lane % DP;
  const int ms = lane / DP;
  const float bhn_c = (CELL == PN_CELL_GRU && ci < D) ? __ldg(P.bhn + ci) : 0.0f;
  // the chain's W rows in registers (one-gate cells, band off): wreg[r][k] = W[r0 + r][k]
  float wreg[C::WREG ? RPL : 1][C::WREG ? DP : 1];
  if constexpr (C::WREG) {
#pragma unroll
    for (int r = 0; r < RPL; ++r)
#pragma unroll
      for (int kk = 0; kk < DP; ++kk) wreg[r][kk] = sWf[kk * WR + r0 + r];
  }
  unsigned rbits = 0u;
  bool aborted = false;
  // the D = 16 tensor-core chain (one-gate cells, dense or banded)
  constexpr bool kMmaChain = (DP == 16 && R == 1);
  static_assert(!kMmaChain || C::NA == 32, "every lane takes part in the chain");
  const bool mma_chain = kMmaChain && P.tc != 0;   // PN_OPT_TENSOR_CORES = 0: the FMA chain
  const int qg = lane >> 2, qi = lane & 3;   // the MMA fragments' row group and column pair

  // W_q[r0 + r][k] of the Jacobian (band-masked when banded), RPL consecutive rows
  auto wrows = [&](int kk, int q, float (&w)[RPL]) { lds_n<RPL>(sWj + kk * WR + q * DP + r0, w); };

  // y = W_q x for rows r0 .. r0 + RPL - 1.  With the W rows in registers (one gate, no band) every
  // lane forms the whole sum from x read by broadcast; otherwise the sum over the lane's k-slice,
  // with W from shared memory, is reduced over the column-group lanes.
  auto slice_matvec = [&](const float* x, float (&out)[R][RPL]) {
    if constexpr (C::WREG) {
      if (!banded) {
        float acc[RPL][4];   // four partial sums per row (k mod 4): a short dependent chain
#pragma unroll
        for (int r = 0; r < RPL; ++r)
#pragma unroll
          for (int u = 0; u < 4; ++u) acc[r][u] = 0.0f;
#pragma unroll
        for (int kk = 0; kk < DP; kk += 4) {
          const float4 x4 = *reinterpret_cast<const float4*>(x + kk);
          const float xv[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int r = 0; r < RPL; ++r) acc[r][u] = fmaf(wreg[r][kk + u], xv[u], acc[r][u]);
        }
#pragma unroll
        for (int r = 0; r < RPL; ++r) out[0][r] = (acc[r][0] + acc[r][1]) + (acc[r][2] + acc[r][3]);
        return;
      }
    }
    float xs[CPL];
    lds_n<CPL>(x + j0, xs);
#pragma unroll
    for (int q = 0; q < R; ++q)
#pragma unroll
      for (int r = 0; r < RPL; ++r) out[q][r] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < CPL; ++kk) {
#pragma unroll
      for (int q = 0; q < R; ++q) {
        float w[RPL];
        wrows(j0 + kk, q, w);
#pragma unroll
        for (int r = 0; r < RPL; ++r) out[q][r] = fmaf(w[r], xs[kk], out[q][r]);
      }
    }
#pragma unroll
    for (int off = 1; off < CG; off <<= 1)
#pragma unroll
      for (int q = 0; q < R; ++q)
#pragma unroll
        for (int r = 0; r < RPL; ++r) out[q][r] += __shfl_xor_sync(0xffffffffu, out[q][r], off);
  };
  // RPL consecutive floats at p + r0 (rows of a per-step vector), and their store
  auto ld_rows = [&](const float* p, float (&v)[RPL]) { lds_n<RPL>(p + r0, v); };
  auto st_rows = [&](float* p, const float (&v)[RPL]) {
    if constexpr (RPL == 4) *reinterpret_cast<float4*>(p + r0) = make_float4(v[0], v[1], v[2], v[3]);
    else *reinterpret_cast<float2*>(p + r0) = make_float2(v[0], v[1]);
  };

  unsigned epoch = epoch0;
  for (int round = 0;; ++round) {
  epoch = epoch0 + (unsigned)round;
  const int iter = iter0 + round;
  const float* __restrict__ src = (iter & 1) ? P.buf1 : A.states;
  float* __restrict__ dst = (iter & 1) ? A.states : P.buf1;
  const int2 fmt = iter_formats(ctrl, A);   // storage of s^(i) (x) and s^(i+1) (y)
  rbits = 0u;
  aborted = false;
  for (;;) {
    int k = 0;
    if (lane == 0) k = (int)atomicAdd(&ctrl->ticket[0], 1u);
    k = __shfl_sync(0xffffffffu, k, 0);
    if (k >= P.tiles_per_group || aborted) break;
    // a ticket is a run of P.run consecutive chunks of one sequence
    const int b = k % B;
    const int chunk = k / B;                      // run index (the look-back's chain position)
    const int c_first = chunk * P.run;
    const int c_end = min(c_first + P.run, (T + L - 1) / L);

    // ---- 1. stage s^(i) rows t0-1 .. t0+L-1 and the step inputs of one chunk -------------
    auto stage = [&](int t0) {
      __syncwarp();   // the previous chunk's readers are done with the slice
      for (int e = lane; e < (L + 1) * DP; e += 32) {
        const int r = e / DP, c = e % DP;
        const int tt = t0 - 1 + r;
        float v = 0.0f;
        if (c < D) {
          if (tt < 0) v = __ldg(A.s0 + (size_t)b * D + c);
          else if (tt < T) v = ld_state(src, ((size_t)b * T + tt) * D + c, fmt.x);
        }
        sS[r * SP + c] = v;
      }
      for (int e = lane; e < L * R * DP; e += 32) {
        const int m = e / (R * DP), qc = e % (R * DP);
        const int q = qc / DP, c = qc % DP;
        const int tt = t0 + m;
        sU[m * UP + qc] = (c < D && tt < T) ? __ldg(xin + ((size_t)b * T + tt) * (R * D) + (size_t)q * D + c) : 0.0f;
      }
      __syncwarp();
    };

    // ---- 2. cell phase, lane = channel ci of step m = pass SPP + ms: the coefficient vectors, b_m (and
    //         |F_m| on the first pass); the writes of a pass go to consecutive channels
    auto cell = [&](int t0, bool with_res) {
#pragma unroll 1
      for (int m = ms; m < L; m += C::SPP) {
        const bool tok = (t0 + m) < T;
        const float* sp = sS + m * SP;   // s^(i)_{t-1}: the same row for the lanes of a pass
        // W_q s: two partial sums per product (even and odd k) keep the dependent chain short
        float z[R], zb[R], z2[R][2], zb2[R][2];
#pragma unroll
        for (int q = 0; q < R; ++q) z2[q][0] = z2[q][1] = zb2[q][0] = zb2[q][1] = 0.0f;
#pragma unroll
        for (int kk = 0; kk < DP; kk += 4) {
          const float4 s4 = *reinterpret_cast<const float4*>(sp + kk);
          const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
#pragma unroll
            for (int q = 0; q < R; ++q) {
              z2[q][u & 1] = fmaf(sWf[(kk + u) * WR + q * DP + ci], sv[u], z2[q][u & 1]);
              if (banded) zb2[q][u & 1] = fmaf(sWb[(kk + u) * WR + q * DP + ci], sv[u], zb2[q][u & 1]);
            }
          }
        }
#pragma unroll
        for (int q = 0; q < R; ++q) {
          z[q] = z2[q][0] + z2[q][1];
          zb[q] = zb2[q][0] + zb2[q][1];
        }
        if (!banded) {
#pragma unroll
          for (int q = 0; q < R; ++q) zb[q] = z[q];
        }
        const float spi = sp[ci];
        const float sci = sS[(m + 1) * SP + ci];
        float cf[NCS], bb, res;
        if constexpr (CELL == PN_CELL_TANH_RNN) {
          const float y = tanh_pn(z[0] + sU[m * UP + ci]);
          cf[0] = 0.0f;
          cf[1] = 1.0f - y * y;
          bb = y - cf[1] * zb[0];
          res = sci - y;
        } else if constexpr (CELL == PN_CELL_EULER_TANH) {
          const float gg = tanh_pn(z[0] + sU[m * UP + ci]);
          const float eg = P.eps * gg;
          cf[0] = 1.0f;
          cf[1] = P.eps * (1.0f - gg * gg);
          bb = eg - cf[1] * zb[0];
          res = (sci - spi) - eg;
        } else {
          const float rr = sigmoidf_acc(sU[m * UP + ci] + z[0]);
          const float zz = sigmoidf_acc(sU[m * UP + DP + ci] + z[1]);
          const float hn = z[2] + bhn_c;
          const float nn = tanh_pn(sU[m * UP + 2 * DP + ci] + rr * hn);
          const float y = nn + zz * (spi - nn);
          const float omz = 1.0f - zz;
          const float dn = omz * (1.0f - nn * nn);
          cf[0] = zz;
          cf[1] = dn * hn * rr * (1.0f - rr);   // gamma: W_hr
          cf[2] = (spi - nn) * zz * omz;        // alpha: W_hz
          cf[3] = dn * rr;                      // beta:  W_hn
          // b_t = y - A s with the banded products of W_hr, W_hz, W_hn
          bb = y - (zz * spi + cf[1] * zb[0] + cf[2] * zb[1] + cf[3] * zb[2]);
          res = sci - y;
        }
        if (tok && ci < D) {
          if (with_res) rbits = max(rbits, abs_bits(res));
        } else {   // identity map
          cf[0] = 1.0f;
#pragma unroll
          for (int q = 1; q < NCS; ++q) cf[q] = 0.0f;
          bb = 0.0f;
        }
#pragma unroll
        for (int q = 0; q < NCS; ++q) sC[(m * NCS + q) * DP + ci] = cf[q];
        sB[m * DP + ci] = bb;
      }
      __syncwarp();
    };

    // ---- 3. chain [P | q] over the run, one chunk at a time --------------------------------
    // gs counts the run's composition steps: step 0 sets [P | q] = [A_0 | b_0], step gs > 0 composes
    // with A_m from buffer (gs - 1) & 1 into buffer gs & 1
    // the lane's P entries; the tensor-core chain keeps Q = P^T there instead (accumulator layout)
    float pold[RPL][CPL];
    float (&qt)[2][4] = *reinterpret_cast<float (*)[2][4]>(&pold[0][0]);
    static_assert(!kMmaChain || (RPL == 2 && CPL == 4), "Q fits the P registers");
    int gs = 0;
#pragma unroll 1
    for (int c = c_first; c < c_end; ++c) {
      const int t0 = c * L;
      stage(t0);
      cell(t0, true);
      uint32_t wbh[2][2][2], wbl[2][2][2];   // the tensor-core chain's W^T fragments, hi and lo
      if (kMmaChain && mma_chain) {
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
#pragma unroll
          for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float w = sWj[(8 * ks + 2 * qi + h) * WR + 8 * j + qg];   // W[8 j + g][8 s + 2 i + h]
              wbh[ks][j][h] = tf32_hi_bits(w);
              wbl[ks][j][h] = tf32_hi_bits(w - __uint_as_float(wbh[ks][j][h]));
            }
      }
#pragma unroll 1
      for (int m = 0; m < L; ++m, ++gs) {
        float c0[RPL], cq[R][RPL], bm[RPL];
        ld_rows(sC + (m * NCS) * DP, c0);
#pragma unroll
        for (int q = 0; q < R; ++q) ld_rows(sC + (m * NCS + 1 + q) * DP, cq[q]);
        ld_rows(sB + m * DP, bm);
        float* Pn = sP + (gs & 1) * DP * PS;
        float qn[RPL];
        if (kMmaChain && mma_chain) {
          // P on the tensor cores; q as below.  c0, c1 of this lane's Q columns 2 i, 2 i + 1, 8 + 2 i, 9 + 2 i
          const float* cv = sC + (m * NCS) * DP;
          const float2 u0 = *reinterpret_cast<const float2*>(cv + 2 * qi);
          const float2 u1 = *reinterpret_cast<const float2*>(cv + 8 + 2 * qi);
          const float2 v0 = *reinterpret_cast<const float2*>(cv + DP + 2 * qi);
          const float2 v1 = *reinterpret_cast<const float2*>(cv + DP + 8 + 2 * qi);
          const float sc0[2][2] = {{u0.x, u0.y}, {u1.x, u1.y}};
          const float sc1[2][2] = {{v0.x, v0.y}, {v1.x, v1.y}};
          if (gs == 0) {   // Q_0 = A_0^T: Q_0[n][r] = c0[r] [r == n] + c1[r] W[r][n]
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int n = qg + 8 * (e >> 1), r = 8 * j + 2 * qi + (e & 1);
                qt[j][e] = fmaf(sc1[j][e & 1], sWj[n * WR + r], (r == n) ? sc0[j][e & 1] : 0.0f);
              }
#pragma unroll
            for (int r = 0; r < RPL; ++r) qn[r] = bm[r];
          } else {
            chain_step_mma16(qt, wbh, wbl, sc0, sc1);
            const float* Qk = sQ + ((gs - 1) & 1) * DP;
            float qa[R][RPL], qo[RPL];
            slice_matvec(Qk, qa);
            ld_rows(Qk, qo);
#pragma unroll
            for (int r = 0; r < RPL; ++r) qn[r] = fmaf(cq[0][r], qa[0][r], fmaf(c0[r], qo[r], bm[r]));
          }
          if (cg == 0) st_rows(sQ + (gs & 1) * DP, qn);
          __syncwarp();
          continue;
        }
        if (gs == 0) {
#pragma unroll
          for (int r = 0; r < RPL; ++r) {
#pragma unroll
            for (int cc = 0; cc < CPL; ++cc) {
              const int i = r0 + r, j = j0 + cc;
              float v = (i == j) ? c0[r] : 0.0f;
#pragma unroll
              for (int q = 0; q < R; ++q) v = fmaf(cq[q][r], sWj[j * WR + q * DP + i], v);
              pold[r][cc] = v;
            }
            qn[r] = bm[r];
          }
        } else {
          const float* Pk = sP + ((gs - 1) & 1) * DP * PS;
          const float* Qk = sQ + ((gs - 1) & 1) * DP;
          float acc[R][RPL][CPL];
#pragma unroll
          for (int q = 0; q < R; ++q)
#pragma unroll
            for (int r = 0; r < RPL; ++r)
#pragma unroll
              for (int cc = 0; cc < CPL; ++cc) acc[q][r][cc] = 0.0f;
          bool done = false;
          if constexpr (C::WREG) {
            if (!banded) {
              // W rows from registers: per k, one load of this lane's P columns and RPL x CPL FMAs
#pragma unroll
              for (int kk = 0; kk < DP; ++kk) {
                float p[CPL];
                lds_n<CPL>(Pk + kk * PS + j0, p);
#pragma unroll
                for (int r = 0; r < RPL; ++r)
#pragma unroll
                  for (int cc = 0; cc < CPL; ++cc) acc[0][r][cc] = fmaf(wreg[r][kk], p[cc], acc[0][r][cc]);
              }
              done = true;
            }
          }
          if (!done && act) {
            // W rows from shared memory, over the band's k range only
#pragma unroll 4
            for (int kk = klo; kk <= khi; ++kk) {
              float p[CPL];
              lds_n<CPL>(Pk + kk * PS + j0, p);
#pragma unroll
              for (int q = 0; q < R; ++q) {
                float w[RPL];
                wrows(kk, q, w);
#pragma unroll
                for (int r = 0; r < RPL; ++r)
#pragma unroll
                  for (int cc = 0; cc < CPL; ++cc) acc[q][r][cc] = fmaf(w[r], p[cc], acc[q][r][cc]);
              }
            }
          }
          float qa[R][RPL];
          slice_matvec(Qk, qa);
          float qo[RPL];
          ld_rows(Qk, qo);
#pragma unroll
          for (int r = 0; r < RPL; ++r) {
#pragma unroll
            for (int cc = 0; cc < CPL; ++cc) {
              float v = c0[r] * pold[r][cc];
#pragma unroll
              for (int q = 0; q < R; ++q) v = fmaf(cq[q][r], acc[q][r][cc], v);
              pold[r][cc] = v;
            }
            float v = fmaf(c0[r], qo[r], bm[r]);
#pragma unroll
            for (int q = 0; q < R; ++q) v = fmaf(cq[q][r], qa[q][r], v);
            qn[r] = v;
          }
        }
        if (act) {
#pragma unroll
          for (int r = 0; r < RPL; ++r) {
            if constexpr (CPL % 4 == 0) {
#pragma unroll
              for (int cc = 0; cc < CPL; cc += 4)
                *reinterpret_cast<float4*>(Pn + (r0 + r) * PS + j0 + cc) =
                    make_float4(pold[r][cc], pold[r][cc + 1], pold[r][cc + 2], pold[r][cc + 3]);
            } else if constexpr (CPL == 2) {
              *reinterpret_cast<float2*>(Pn + (r0 + r) * PS + j0) = make_float2(pold[r][0], pold[r][1]);
            } else {
              Pn[(r0 + r) * PS + j0] = pold[r][0];
            }
          }
          if (cg == 0) st_rows(sQ + (gs & 1) * DP, qn);
        }
        __syncwarp();
      }
    }
    if (kMmaChain && mma_chain) {   // the tensor-core chain's aggregate into the shared-memory P
      float* Pw = sP + ((gs - 1) & 1) * DP * PS;
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) Pw[(8 * j + 2 * qi + (e & 1)) * PS + qg + 8 * (e >> 1)] = qt[j][e];
      __syncwarp();
    }
    const float* Pl = sP + ((gs - 1) & 1) * DP * PS;   // the run's aggregate [P | q]
    const float* Ql = sQ + ((gs - 1) & 1) * DP;

    // ---- 4. decoupled look-back over the runs of the sequence ---------------------------------
    const bool stall = (A.stall_ticket == k);
    if (chunk > 0 && !stall) {
      float* ag = P.agg + (size_t)k * P.agg_stride;
      for (int e = lane; e < DP * (DP + 1); e += 32) {
        const int i = e / (DP + 1), j = e % (DP + 1);
        ag[e] = (j == DP) ? Ql[i] : Pl[i * PS + j];
      }
      __threadfence();
      __syncwarp();
      if (lane == 0) st_release(P.flags + k, make_flag(epoch, kFlagAgg));
    }
    const int n_agg = lookback_find_prefix(P.flags, (size_t)k, stride, chunk, epoch, ctrl, A.timeout_ns);
    if (n_agg < 0) {
      aborted = true;
      break;
    }
    // starting state: the end state of the run n_agg + 1 back, or s0
    float* cur = sX;
    float* nxt = sX + DP;
    if (lane < DP) {
      float v = 0.0f;
      if (chunk - 1 - n_agg >= 0) v = __ldcg(P.pref + ((size_t)k - (size_t)(n_agg + 1) * stride) * P.pref_stride + lane);
      else if (lane < D) v = __ldg(A.s0 + (size_t)b * D + lane);
      cur[lane] = v;
    }
    __syncwarp();
    // fold the aggregates at distances n_agg .. 1, farthest first: carry <- P_d carry + q_d.  Each
    // lane's blocks of FB aggregates are loaded together, so a batch costs one L2 round trip.
    constexpr int FB = (CPL <= 4) ? 4 : 2;
    for (int d = n_agg; d >= 1; d -= FB) {
      float blk[FB][RPL][CPL], qd[FB][RPL];
#pragma unroll
      for (int u = 0; u < FB; ++u) {
        const bool use = act && (d - u >= 1);
        const float* ag = P.agg + ((size_t)k - (size_t)max(d - u, 1) * stride) * P.agg_stride;
#pragma unroll
        for (int r = 0; r < RPL; ++r) {
#pragma unroll
          for (int cc = 0; cc < CPL; ++cc) blk[u][r][cc] = use ? __ldcg(ag + (r0 + r) * (DP + 1) + j0 + cc) : 0.0f;
          qd[u][r] = use ? __ldcg(ag + (r0 + r) * (DP + 1) + DP) : 0.0f;
        }
      }
#pragma unroll
      for (int u = 0; u < FB; ++u) {
        if (d - u < 1) break;   // uniform across the warp
        float xs[CPL];
        lds_n<CPL>(cur + j0, xs);
        float part[RPL];
#pragma unroll
        for (int r = 0; r < RPL; ++r) {
          float v = 0.0f;
#pragma unroll
          for (int cc = 0; cc < CPL; ++cc) v = fmaf(blk[u][r][cc], xs[cc], v);
          part[r] = v;
        }
#pragma unroll
        for (int off = 1; off < CG; off <<= 1)
#pragma unroll
          for (int r = 0; r < RPL; ++r) part[r] += __shfl_xor_sync(0xffffffffu, part[r], off);
        if (act && cg == 0) {
#pragma unroll
          for (int r = 0; r < RPL; ++r) part[r] += qd[u][r];
          st_rows(nxt, part);
        }
        __syncwarp();
        float* tmp = cur;
        cur = nxt;
        nxt = tmp;
      }
    }
    // this run's end state P carry + q
    if (!stall) {
      float xs[CPL];
      lds_n<CPL>(cur + j0, xs);
      float part[RPL];
#pragma unroll
      for (int r = 0; r < RPL; ++r) {
        float v = 0.0f;
#pragma unroll
        for (int cc = 0; cc < CPL; ++cc) v = fmaf(Pl[(r0 + r) * PS + j0 + cc], xs[cc], v);
        part[r] = v;
      }
#pragma unroll
      for (int off = 1; off < CG; off <<= 1)
#pragma unroll
        for (int r = 0; r < RPL; ++r) part[r] += __shfl_xor_sync(0xffffffffu, part[r], off);
      if (act && cg == 0) {
#pragma unroll
        for (int r = 0; r < RPL; ++r) P.pref[(size_t)k * P.pref_stride + r0 + r] = part[r] + Ql[r0 + r];
      }
      __threadfence();
      __syncwarp();
      if (lane == 0) st_release(P.flags + k, make_flag(epoch, kFlagPrefix));
    }

    // ---- 5. apply the carry step by step over the run, chunk by chunk, write the states ------
    // (sX holds the running state across the chunks' restaging)
    {
      float sold[RPL];
      ld_rows(cur, sold);
      if (cur != sX) {
        if (act && cg == 0) st_rows(sX, sold);
        __syncwarp();
      }
#pragma unroll 1
      for (int c = c_first; c < c_end; ++c) {
        const int t0 = c * L;
        if (P.run > 1) {   // the first pass's coefficients belong to the run's last chunk
          stage(t0);
          cell(t0, false);
        }
        const float* xcur = sX;
#pragma unroll 1
        for (int m = 0; m < L; ++m) {
          float pa[R][RPL];
          slice_matvec(xcur, pa);
          float c0[RPL], cq[R][RPL], bm[RPL];
          ld_rows(sC + (m * NCS) * DP, c0);
#pragma unroll
          for (int q = 0; q < R; ++q) ld_rows(sC + (m * NCS + 1 + q) * DP, cq[q]);
          ld_rows(sB + m * DP, bm);
#pragma unroll
          for (int r = 0; r < RPL; ++r) {
            float v = fmaf(c0[r], sold[r], bm[r]);
#pragma unroll
            for (int q = 0; q < R; ++q) v = fmaf(cq[q][r], pa[q][r], v);
            sold[r] = v;
          }
          if (act && cg == 0) st_rows(sO + m * DP, sold);
          __syncwarp();
          xcur = sO + m * DP;
        }
        for (int e = lane; e < L * DP; e += 32) {
          const int m = e / DP, i = e % DP;
          const int tt = t0 + m;
          if (tt < T && i < D) {
            float v = sO[e];
            if (damped) {
              const float sc = sS[(m + 1) * SP + i];   // s^(i)_t
              v = fmaf(lambda, v - sc, sc);
            }
            st_state(dst, ((size_t)b * T + tt) * D + i, v, fmt.y);
          }
        }
        // the chunk's last state starts the next chunk
        if (act && cg == 0) st_rows(sX, sold);
        __syncwarp();
      }
    }
  }

  // ---- residual of this iteration; the next one (grid barrier) or the end of the launch
  rbits = warp_max_u32(rbits);
  if (lane == 0) sRed[warp] = __uint_as_float(rbits);
  __syncthreads();
  unsigned rmax = 0u;   // the CTA's residual maximum, on thread 0
  if (tid == 0) {
    for (int w = 0; w < NWARP; ++w) rmax = max(rmax, __float_as_uint(sRed[w]));
    if (rmax && !P.persist) atomicMax(&ctrl->resid_bits, rmax);
  }
  if (!P.persist) break;
  if (!finish_iteration(P, A, iter, epoch, s_last, (gen0 >> 1) + (unsigned)round, rmax)) break;
  }   // iterations
  if (!P.persist) finish_launch(P, A, epoch, s_last);
}

}  // namespace pn
