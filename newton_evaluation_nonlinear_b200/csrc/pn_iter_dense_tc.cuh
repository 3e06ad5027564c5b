// pn_iter_dense_tc.cuh -- fused Newton iteration with the batched D x D
// compositions on the tensor cores (tcgen05, 3xTF32), for the one-gate cells
// (tanh RNN, Euler drift) at padded widths DP = 32 and 64.
//
// The iteration is the page's unified update with J~ = J ("Parallel Newton
// methods..." page, §1.2) solved by the affine scan of §2.1, as in
// pn_iter_dense_warp.cuh; the page names the tensor cores as the hardware for
// the dense work (§5.2).  For these cells A_t = diag(c0_t) + diag(c1_t) W
// (tanh RNN: c0 = 0, c1 = 1 - y^2; Euler: c0 = 1, c1 = eps (1 - g^2)), so one
// composition step of the chunk aggregate,
//     [P | q] <- A_m [P | q] + [0 | b_m],
// is the product W P followed by a row scaling.  It runs transposed,
// (W P)^T = P^T W^T, as one M x DP x DP tcgen05.mma (M = 64 for DP = 32, 128
// for DP = 64) whose A operand holds P^T (row j = column j of P, row DP = q)
// and whose B operand is W, both in the K-major core-matrix layout.  The
// accumulator row j lands in TMEM lane j, so thread j reads column j of W P,
// scales it, keeps it in registers, and writes it back as row j of the next
// A operand: one product, one TMEM read and one shared-memory write per step,
// with no exchange between threads.  Products are 3xTF32 (P_hi W_hi + P_hi
// W_lo + P_lo W_hi), fp32-level accuracy; P_hi is the tensor core's
// truncation of the stored fp32 value and P_lo its exact remainder.
//
// Per tile of L steps of one sequence (one tile per CTA at a time):
//   1. stage s^(i) rows t0-1 .. t0+L-1 and the step inputs;
//   2. cell phase: the same MMA with the A operand the staged rows gives
//      W s_{t-1} for every step; thread m evaluates the cell of step m: the
//      coefficient vectors, b_m and |F_m|;
//   3. chain of L composition steps from P = I, q = 0;
//   4. decoupled look-back over the D x (D+1) aggregates (plain floats);
//   5. apply the carry sequentially in FP32, s_m = A_m s_{m-1} + b_m, stage
//      and write the states (damped: s^(i) + lambda (s - s^(i))).
// Padded steps (t >= T) and channels (i >= D) are identity maps.  The banded
// approximation runs on the FP32 kernels (the host does not select this one).
#pragma once

#include "pn_iter_diag_tc.cuh"

namespace pn {

template <int CELL, int DP>
struct DenseTcCfg {
  static_assert(CELL != PN_CELL_GRU, "one-gate cells only");
  static_assert(DP == 32 || DP == 64, "DP = 32 or 64");
  static constexpr int L = 32;                      // steps per tile
  static constexpr int M = (DP + 1 <= 64) ? 64 : 128;   // MMA M: rows of P^T and q^T (chain), or steps (cell)
  static constexpr int NT = 128;                    // four warps: one per TMEM lane quarter
  static constexpr int TCOLS = DP < 32 ? 32 : DP;   // TMEM columns (fp32 accumulator, N = DP)
  static constexpr int OP_BYTES = M * DP * 4;       // one A operand (hi or lo), K-major core matrices
  static constexpr int W_BYTES = DP * DP * 4;       // one B operand (W_hi or W_lo)
  static constexpr int SP = DP + 1;                 // row stride of staged s rows
  static constexpr int a128(int v) { return (v + 127) / 128 * 128; }
  static constexpr int OFF_AHI = 0;
  static constexpr int OFF_ALO = OFF_AHI + OP_BYTES;
  static constexpr int OFF_WHI = OFF_ALO + OP_BYTES;
  static constexpr int OFF_WLO = OFF_WHI + W_BYTES;
  static constexpr int OFF_WF = OFF_WLO + W_BYTES;              // fp32 W, [k][i] (W[i][k] at k DP + i)
  static constexpr int OFF_S = OFF_WF + DP * DP * 4;            // [L+1][SP]
  static constexpr int OFF_U = a128(OFF_S + (L + 1) * SP * 4);  // [L][DP]
  static constexpr int OFF_C = OFF_U + L * DP * 4;              // [L][2][DP]: c0, c1
  static constexpr int OFF_B = OFF_C + L * 2 * DP * 4;          // [L][DP]
  static constexpr int OFF_O = OFF_B + L * DP * 4;              // [L][DP]
  static constexpr int OFF_X = OFF_O + L * DP * 4;              // carry [2][DP]
  static constexpr int OFF_RED = OFF_X + 2 * DP * 4;
  static constexpr int SMEM_USED = OFF_RED + 4 * 4;
  static constexpr int SMEM_BYTES = SMEM_USED + 128;            // + slack to align the base to 128 bytes
  static constexpr uint32_t SBO = (DP / 4) * 128;               // stride between 8-row core-matrix groups
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

template <int CELL, int DP>
__global__ void __launch_bounds__(128, 1) dense_tc_kernel(const IterParams P) {
  using C = DenseTcCfg<CELL, DP>;
  constexpr int L = C::L;
  constexpr int M = C::M;
  constexpr int SP = C::SP;

  extern __shared__ __align__(128) unsigned char smem_dtc[];
  unsigned char* base = smem_dtc + ((128u - (smem_addr(smem_dtc) & 127u)) & 127u);
  unsigned char* sAhi = base + C::OFF_AHI;
  unsigned char* sAlo = base + C::OFF_ALO;
  unsigned char* sWhi = base + C::OFF_WHI;
  unsigned char* sWlo = base + C::OFF_WLO;
  float* sWf = reinterpret_cast<float*>(base + C::OFF_WF);
  float* sS = reinterpret_cast<float*>(base + C::OFF_S);
  float* sU = reinterpret_cast<float*>(base + C::OFF_U);
  float* sC = reinterpret_cast<float*>(base + C::OFF_C);
  float* sB = reinterpret_cast<float*>(base + C::OFF_B);
  float* sO = reinterpret_cast<float*>(base + C::OFF_O);
  float* sX = reinterpret_cast<float*>(base + C::OFF_X);
  float* sRed = reinterpret_cast<float*>(base + C::OFF_RED);
  __shared__ __align__(8) uint64_t bar_mma;
  __shared__ uint32_t s_tmem;
  __shared__ int s_ticket, s_nagg, s_last;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  Ctrl* ctrl = P.ctrl;
  const Args A = *P.args;
  const int D = P.D, T = P.T, B = P.B;
  const float lambda = A.damping;
  const bool damped = lambda != 1.0f;
  const size_t stride = (size_t)B;
  const long long tmo = A.timeout_ns;

  if (tid == 0) {
    atomicMin(&ctrl->t_start, globaltimer());
    mbar_init(&bar_mma, 1u);
    mbar_init_fence();
  }
  const unsigned epoch = *(volatile unsigned*)&ctrl->epoch;
  const int iter = *(volatile int*)&ctrl->iter;
  const float* __restrict__ src = (iter & 1) ? P.buf1 : A.states;
  float* __restrict__ dst = (iter & 1) ? A.states : P.buf1;
  const int2 fmt = iter_formats(ctrl, A);
  const float* xin = (CELL == PN_CELL_EULER_TANH) ? A.x : P.xin;

  // weights: W_hi, W_lo (host-split, K-major core matrices: row n = output channel, K = input),
  // and the fp32 W for the apply, [k][i]
  {
    const float4* w4 = reinterpret_cast<const float4*>(P.wt_tc);
    float4* h4 = reinterpret_cast<float4*>(sWhi);
    float4* l4 = reinterpret_cast<float4*>(sWlo);
    for (int e = tid; e < C::W_BYTES / 16; e += C::NT) {
      h4[e] = __ldg(w4 + e);
      l4[e] = __ldg(w4 + C::W_BYTES / 16 + e);
    }
    for (int e = tid; e < DP * DP; e += C::NT) sWf[e] = __ldg(P.wt + e);
    fence_async_smem();
  }
  if (warp == 0) {
    tmem_alloc(&s_tmem, (uint32_t)C::TCOLS);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  // the accumulator row this thread reads: M = 128, row = tid; M = 64, rows 16 w + l for lanes l < 16
  // of warp w (an M = 64 accumulator takes lanes 0-15 of each lane quarter)
  const int row = (M == 128) ? tid : ((lane < 16) ? 16 * warp + lane : -1);
  const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
  constexpr uint32_t idesc = umma_idesc_tf32(M, DP);
  const uint64_t a_hi = umma_smem_desc(smem_addr(sAhi), 128, C::SBO, 0);
  const uint64_t a_lo = umma_smem_desc(smem_addr(sAlo), 128, C::SBO, 0);
  const uint64_t w_hi = umma_smem_desc(smem_addr(sWhi), 128, C::SBO, 0);
  const uint64_t w_lo = umma_smem_desc(smem_addr(sWlo), 128, C::SBO, 0);
  unsigned phase = 0;
  unsigned rbits = 0u;

  // row r of both A operands from v[0 .. DP-1] (hi: the value; lo: its TF32 remainder)
  auto write_row = [&](int r, const float (&v)[DP]) {
#pragma unroll
    for (int k = 0; k < DP; k += 4) {
      const uint32_t off = kmajor_offset(r, k, DP);
      *reinterpret_cast<float4*>(sAhi + off) = make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
      *reinterpret_cast<float4*>(sAlo + off) =
          make_float4(tf32_tail(v[k]), tf32_tail(v[k + 1]), tf32_tail(v[k + 2]), tf32_tail(v[k + 3]));
    }
  };
  // D = A W^T on the tensor cores (3xTF32), then every thread has waited for it; false on a timeout
  auto product = [&]() -> bool {
    fence_async_smem();   // the generic writes of the A rows -> the tensor cores
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
#pragma unroll
      for (int kb = 0; kb < DP / 8; ++kb) {
        const uint64_t ko = (uint64_t)((kb * 256) >> 4);   // two core matrices along K per MMA
        umma_tf32(tmem, a_hi + ko, w_hi + ko, idesc, kb ? 1u : 0u);
        umma_tf32(tmem, a_hi + ko, w_lo + ko, idesc, 1u);
        umma_tf32(tmem, a_lo + ko, w_hi + ko, idesc, 1u);
      }
      umma_commit(&bar_mma);
    }
    const bool ok = mbar_wait(&bar_mma, phase, ctrl, tmo);
    phase ^= 1u;
    tc_fence_after();
    return __syncthreads_and(ok) != 0;   // one decision for the whole CTA
  };
  // this thread's accumulator row (DP columns)
  auto read_row = [&](float (&v)[DP]) {
#pragma unroll
    for (int c = 0; c < DP; c += 16) {
      float t[16];
      tmem_ld16(lane_base + (uint32_t)c, t);
#pragma unroll
      for (int u = 0; u < 16; ++u) v[c + u] = t[u];
    }
  };

  bool failed = false;
  for (;;) {
    if (tid == 0) s_ticket = (int)atomicAdd(&ctrl->ticket[0], 1u);
    __syncthreads();
    const int k = s_ticket;
    if (k >= P.tiles_per_group) break;
    const int b = k % B;
    const int chunk = k / B;
    const int t0 = chunk * L;

    // ---- 1. stage ------------------------------------------------------------------
    for (int e = tid; e < (L + 1) * DP; e += C::NT) {
      const int r = e / DP, c = e % DP;
      const int tt = t0 - 1 + r;
      float v = 0.0f;
      if (c < D) {
        if (tt < 0) v = __ldg(A.s0 + (size_t)b * D + c);
        else if (tt < T) v = ld_state(src, ((size_t)b * T + tt) * D + c, fmt.x);
      }
      sS[r * SP + c] = v;
    }
    for (int e = tid; e < L * DP; e += C::NT) {
      const int m = e / DP, c = e % DP;
      const int tt = t0 + m;
      sU[e] = (c < D && tt < T) ? __ldg(xin + ((size_t)b * T + tt) * D + c) : 0.0f;
    }
    __syncthreads();

    // ---- 2. cell phase: row m of the A operand = s_{t0+m-1}; D row m = W s_{t0+m-1} --------
    if (row >= 0 && row < L) {
      float v[DP];
#pragma unroll
      for (int c = 0; c < DP; ++c) v[c] = sS[row * SP + c];
      write_row(row, v);
    }
    if (!product()) { failed = true; break; }
    {
      float z[DP];
      read_row(z);
      if (row >= 0 && row < L) {
        const int m = row;
        const bool tok = (t0 + m) < T;
#pragma unroll
        for (int i = 0; i < DP; ++i) {
          const float spi = sS[m * SP + i];
          const float sci = sS[(m + 1) * SP + i];
          float c0, c1, bb, res;
          if constexpr (CELL == PN_CELL_TANH_RNN) {
            const float y = tanh_pn(z[i] + sU[m * DP + i]);
            c0 = 0.0f;
            c1 = 1.0f - y * y;
            bb = y - c1 * z[i];
            res = sci - y;
          } else {
            const float gg = tanh_pn(z[i] + sU[m * DP + i]);
            const float eg = P.eps * gg;
            c0 = 1.0f;
            c1 = P.eps * (1.0f - gg * gg);
            bb = eg - c1 * z[i];
            res = (sci - spi) - eg;
          }
          if (tok && i < D) {
            rbits = max(rbits, abs_bits(res));
          } else {
            c0 = 1.0f;
            c1 = 0.0f;
            bb = 0.0f;
          }
          sC[(m * 2 + 0) * DP + i] = c0;
          sC[(m * 2 + 1) * DP + i] = c1;
          sB[m * DP + i] = bb;
        }
      }
    }

    // ---- 3. chain from P = I, q = 0: row j < DP of P^T is e_j, row DP is q^T ------------
    float pcol[DP];   // this thread's column of P (row j = DP: q)
    if (row >= 0 && row <= DP) {
#pragma unroll
      for (int i = 0; i < DP; ++i) pcol[i] = (i == row) ? 1.0f : 0.0f;
      write_row(row, pcol);
    }
#pragma unroll 1
    for (int m = 0; m < L; ++m) {
      if (!product()) { failed = true; break; }
      float z[DP];
      read_row(z);
      if (row >= 0 && row <= DP) {
        const float* c0 = sC + (m * 2 + 0) * DP;
        const float* c1 = sC + (m * 2 + 1) * DP;
        const float* bm = sB + m * DP;
#pragma unroll
        for (int i = 0; i < DP; ++i) {
          float v = fmaf(c0[i], pcol[i], c1[i] * z[i]);
          if (row == DP) v += bm[i];
          pcol[i] = v;
        }
        write_row(row, pcol);
      }
    }
    if (failed) break;
    __syncthreads();   // the last A rows hold P_L^T and q_L^T

    // ---- 4. decoupled look-back ------------------------------------------------------
    // P_L[i][j] is row j, column i of the A operand (hi: the fp32 value); q_L[i] is row DP
    auto pl = [&](int i, int j) -> float {
      return *reinterpret_cast<const float*>(sAhi + kmajor_offset(j, i, DP));
    };
    const bool stall = (A.stall_ticket == k);
    if (chunk > 0 && !stall) {
      float* ag = P.agg + (size_t)k * P.agg_stride;
      for (int e = tid; e < DP * (DP + 1); e += C::NT) {
        const int i = e / (DP + 1), j = e % (DP + 1);
        ag[e] = pl(i, j);
      }
      __threadfence();
    }
    __syncthreads();
    if (warp == 0) {
      if (chunk > 0 && !stall && lane == 0) st_release(P.flags + k, make_flag(epoch, kFlagAgg));
      const int n = lookback_find_prefix(P.flags, (size_t)k, stride, chunk, epoch, ctrl, tmo);
      if (lane == 0) s_nagg = n;
    }
    __syncthreads();
    const int n_agg = s_nagg;
    if (n_agg < 0) { failed = true; break; }
    float* cur = sX;
    float* nxt = sX + DP;
    if (tid < DP) {
      float v = 0.0f;
      if (chunk - 1 - n_agg >= 0) v = __ldcg(P.pref + ((size_t)k - (size_t)(n_agg + 1) * stride) * P.pref_stride + tid);
      else if (tid < D) v = __ldg(A.s0 + (size_t)b * D + tid);
      cur[tid] = v;
    }
    __syncthreads();
    for (int d = n_agg; d >= 1; --d) {
      if (tid < DP) {
        const float* ag = P.agg + ((size_t)k - (size_t)d * stride) * P.agg_stride + (size_t)tid * (DP + 1);
        float v = __ldcg(ag + DP);
#pragma unroll 8
        for (int j = 0; j < DP; ++j) v = fmaf(__ldcg(ag + j), cur[j], v);
        nxt[tid] = v;
      }
      __syncthreads();
      float* tmp = cur; cur = nxt; nxt = tmp;
    }
    if (tid < DP && !stall) {
      float v = pl(tid, DP);
#pragma unroll 8
      for (int j = 0; j < DP; ++j) v = fmaf(pl(tid, j), cur[j], v);
      P.pref[(size_t)k * P.pref_stride + tid] = v;
      __threadfence();
    }
    __syncthreads();
    if (tid == 0 && !stall) st_release(P.flags + k, make_flag(epoch, kFlagPrefix));

    // ---- 5. apply the carry step by step (threads 0 .. DP-1), write the states --------
    if (tid < DP) {
      const int i = tid;
      float si = cur[i];
      const float* sprev = cur;
#pragma unroll 1
      for (int m = 0; m < L; ++m) {
        float acc = 0.0f;
#pragma unroll 8
        for (int kk = 0; kk < DP; ++kk) acc = fmaf(sWf[kk * DP + i], sprev[kk], acc);
        si = fmaf(sC[(m * 2 + 0) * DP + i], si, fmaf(sC[(m * 2 + 1) * DP + i], acc, sB[m * DP + i]));
        sO[m * DP + i] = si;
        named_barrier(1, DP);
        sprev = sO + m * DP;
      }
    }
    __syncthreads();
    for (int e = tid; e < L * DP; e += C::NT) {
      const int m = e / DP, i = e % DP;
      const int tt = t0 + m;
      if (tt < T && i < D) {
        float v = sO[e];
        if (damped) {
          const float sc = sS[(m + 1) * SP + i];
          v = fmaf(lambda, v - sc, sc);
        }
        st_state(dst, ((size_t)b * T + tt) * D + i, v, fmt.y);
      }
    }
  }

  rbits = warp_max_u32(rbits);
  if (lane == 0) sRed[warp] = __uint_as_float(rbits);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    tmem_dealloc(tmem, (uint32_t)C::TCOLS);
  if (tid == 0) {
    unsigned v = 0u;
    for (int w = 0; w < 4; ++w) v = max(v, __float_as_uint(sRed[w]));
    if (v) atomicMax(&ctrl->resid_bits, v);
  }
  (void)failed;
  finish_launch(P, A, epoch, s_last);
}

}  // namespace pn
