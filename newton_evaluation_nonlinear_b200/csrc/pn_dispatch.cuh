// pn_dispatch.cuh -- launch shapes of the fused iteration kernels.
//
// The padded state width DP is the smallest of 4, 8, ..., 256 that holds D;
// each (cell, DP) has one tile shape for the diagonal-family kernel (channel
// group G, TM steps x TN channels per thread, TS thread segments along t) and
// one for the dense Newton kernel (L steps x DP channels per CTA).
#pragma once

#include "pn_iter_dense.cuh"
#include "pn_iter_dense_tc.cuh"
#include "pn_iter_dense_warp.cuh"
#include "pn_iter_diag.cuh"
#include "pn_iter_diag_tc.cuh"
#include "pn_iter_diag_tct.cuh"
#include "pn_small.cuh"
#include "pn_iter_diag_post.cuh"
#include "pn_iter_diag_tma.cuh"
#include "pn_wide_gemm.cuh"

namespace pn {

// Which weight packing and look-back format a kernel uses.
enum KKind { kKindDiag = 0, kKindDiagTc = 1, kKindDense = 2, kKindDiagTct = 3, kKindDiagPost = 4 };

// Kernels whose look-back aggregates and states are tagged 64-bit words.
inline bool tagged_lookback(int kind) { return kind == kKindDiagTc || kind == kKindDiagTct; }

struct KInfo {
  const void* fn;   // __global__ function
  int nt;           // threads per CTA
  int L;            // steps per tile
  int G;            // channels per tile
  size_t smem;      // dynamic shared memory bytes
  int kind;         // KKind: which weight packing the kernel reads
  bool loops = false;   // can run every iteration in one launch (IterParams::persist, grid barrier)
  int tpc = 0;          // > 0: takes runs of several chunks per ticket, tpc tickets in flight per CTA
  const void* pre_fn = nullptr;   // launched before fn in every iteration (the tensor-core product Y = S W^T)
  int pre_nt = 0;
  size_t pre_smem = 0;
  bool coop = false;    // meets a grid barrier inside every launch: launched cooperatively
};

template <int CELL, int MODE, int DP, int G, int TM, int TN, int TS>
inline KInfo diag_kinfo() {
  using C = DiagCfg<CELL, MODE, DP, G, TM, TN, TS>;
  return KInfo{(const void*)&diag_iter_kernel<CELL, MODE, DP, G, TM, TN, TS>, C::NT, C::L, G,
               C::SMEM_BYTES, kKindDiag};
}

template <int CELL, int MODE, int DP>
inline KInfo diag_pick() {
  constexpr bool gru = (CELL == PN_CELL_GRU);
  if constexpr (DP == 4) return diag_kinfo<CELL, MODE, 4, 4, 4, 1, 64>();
  else if constexpr (DP == 8) return diag_kinfo<CELL, MODE, 8, 8, 4, 2, 64>();
  else if constexpr (DP == 16) return diag_kinfo<CELL, MODE, 16, 16, 4, 4, 64>();
  else if constexpr (DP == 32) {
    if constexpr (gru) return diag_kinfo<CELL, MODE, 32, 32, 4, 2, 16>();
    else return diag_kinfo<CELL, MODE, 32, 32, 4, 4, 32>();
  } else if constexpr (DP == 64) {
    if constexpr (gru) return diag_kinfo<CELL, MODE, 64, 64, 4, 2, 8>();
    else return diag_kinfo<CELL, MODE, 64, 64, 4, 4, 16>();
  } else if constexpr (DP == 128) {
    if constexpr (gru) return diag_kinfo<CELL, MODE, 128, 32, 4, 2, 16>();
    else return diag_kinfo<CELL, MODE, 128, 64, 4, 4, 16>();
  } else {
    if constexpr (gru) return diag_kinfo<CELL, MODE, 256, 32, 4, 2, 16>();
    else return diag_kinfo<CELL, MODE, 256, 64, 4, 4, 16>();
  }
}

template <int CELL, int MODE, int DP, int G, int TM, int TN, int TS>
inline KInfo diag_tma_kinfo() {
  using C = DiagTmaCfg<CELL, MODE, DP, G, TM, TN, TS>;
  return KInfo{(const void*)&diag_tma_kernel<CELL, MODE, DP, G, TM, TN, TS>, C::NT, C::L, G, C::SMEM_BYTES,
               kKindDiag};
}

// Pipelined (producer warp + bulk copies) variant, for D a multiple of 4 and DP >= 32.
template <int CELL, int MODE, int DP>
inline KInfo diag_tma_pick() {
  constexpr bool gru = (CELL == PN_CELL_GRU);
  if constexpr (DP == 32) {
    if constexpr (gru) return diag_tma_kinfo<CELL, MODE, 32, 32, 4, 2, 16>();
    else return diag_tma_kinfo<CELL, MODE, 32, 32, 4, 4, 32>();
  } else if constexpr (DP == 64) {
    if constexpr (gru) return diag_tma_kinfo<CELL, MODE, 64, 64, 4, 2, 8>();
    else return diag_tma_kinfo<CELL, MODE, 64, 64, 4, 4, 16>();
  } else if constexpr (DP == 128) {
    if constexpr (gru) return diag_tma_kinfo<CELL, MODE, 128, 32, 2, 2, 16>();
    else return diag_tma_kinfo<CELL, MODE, 128, 64, 2, 4, 16>();
  } else {
    if constexpr (gru) return diag_tma_kinfo<CELL, MODE, 256, 32, 2, 2, 16>();
    else return diag_tma_kinfo<CELL, MODE, 256, 64, 2, 4, 16>();
  }
}

// Tensor-core variant: D == DP in {32, 64}; the GRU's three gates fit only at D = 32.
template <int CELL, int MODE, int DP>
inline KInfo diag_tc_kinfo() {
  using C = DiagTcCfg<CELL, MODE, DP>;
  return KInfo{(const void*)&diag_tc_kernel<CELL, MODE, DP>, C::NT, C::L, DP, (size_t)C::SMEM_BYTES, kKindDiagTc,
               true};
}

// Channel-major tensor-core variant for the one-gate cells: D == DP in {32, 64}.
template <int CELL, int MODE, int DP>
inline KInfo diag_tct_kinfo() {
  using C = DiagTctCfg<CELL, MODE, DP>;
  return KInfo{(const void*)&diag_tct_kernel<CELL, MODE, DP>, C::NT, C::L, DP, (size_t)C::SMEM_BYTES, kKindDiagTct,
               true};
}

template <int CELL, int DP, int L>
inline KInfo dense_kinfo() {
  using C = DenseCfg<CELL, DP, L>;
  return KInfo{(const void*)&dense_iter_kernel<CELL, DP, L>, C::NT, L, DP, C::SMEM_BYTES, kKindDense};
}

// One warp per tile, FP32 chain (D <= 32); NW warps per CTA, sized so two CTAs fit on an SM where
// the per-warp staging allows it.
template <int CELL, int DP, int NW>
inline KInfo dense_warp_kinfo() {
  using C = DenseWarpCfg<CELL, DP, NW>;
  return KInfo{(const void*)&dense_warp_kernel<CELL, DP, NW>, C::NT, C::L, DP, C::SMEM_BYTES, kKindDense, true, NW};
}

template <int CELL, int DP>
inline KInfo dense_pick() {
  constexpr bool gru = (CELL == PN_CELL_GRU);
  if constexpr (DP == 4) return dense_warp_kinfo<CELL, 4, 8>();
  else if constexpr (DP == 8) return dense_warp_kinfo<CELL, 8, 8>();
  else if constexpr (DP == 16) {
    if constexpr (gru) return dense_warp_kinfo<CELL, 16, 4>();
    else return dense_warp_kinfo<CELL, 16, 7>();
  } else if constexpr (DP == 32) {
    if constexpr (gru) return dense_warp_kinfo<CELL, 32, 3>();
    else return dense_warp_kinfo<CELL, 32, 6>();
  } else {
    if constexpr (gru) return dense_kinfo<CELL, 64, 2>();
    else return dense_kinfo<CELL, 64, 4>();
  }
}

// Wide one-gate cells (DP = 128, 256): the recurrent product of every step on the tensor cores
// (wide_gemm_kernel), then the FP32 diagonal kernel reading it.
template <int CELL, int MODE, int DP>
inline KInfo diag_wide_kinfo() {
  using C = PostCfg<CELL, MODE, DP>;
  using W = WideGemmCfg<DP>;   // N = K = DP
  KInfo k{(const void*)&diag_post_kernel<CELL, MODE, DP>, C::NT, C::L, C::G, C::SMEM_BYTES, kKindDiagPost};
  k.pre_fn = (const void*)&wide_gemm_kernel<DP>;
  k.pre_nt = W::NT;
  k.pre_smem = (size_t)W::SMEM_BYTES;
  k.coop = true;   // the phases of the scan meet at grid barriers
  return k;
}

// Newton with the compositions on the tensor cores: one-gate cells, DP = 32 or 64.
template <int CELL, int DP>
inline KInfo dense_tc_kinfo() {
  using C = DenseTcCfg<CELL, DP>;
  return KInfo{(const void*)&dense_tc_kernel<CELL, DP>, C::NT, C::L, DP, (size_t)C::SMEM_BYTES, kKindDense};
}

// tma: use the pipelined variant where it exists (the caller checks D % 4 == 0);
// tc: use the tensor-core variant where it exists (diagonal modes: the caller checks D == DP; Newton:
// the caller checks that the band is off).
template <int CELL>
inline KInfo lookup_cell(int mode, int DP, bool tma, bool tc) {
  KInfo none{nullptr, 0, 0, 0, 0, 0};
  if constexpr (CELL != PN_CELL_GRU) {
    if (tc && mode == PN_NEWTON) {
      if (DP == 32) return dense_tc_kinfo<CELL, 32>();
      if (DP == 64) return dense_tc_kinfo<CELL, 64>();
    }
    if (tc && mode != PN_NEWTON && (DP == 128 || DP == 256)) {
#define PN_WIDE(MODE_)                                              \
  return DP == 128 ? diag_wide_kinfo<CELL, MODE_, 128>() : diag_wide_kinfo<CELL, MODE_, 256>();
      if (mode == PN_JACOBI) { PN_WIDE(PN_JACOBI) }
      if (mode == PN_PICARD) { PN_WIDE(PN_PICARD) }
      PN_WIDE(PN_QUASI)
#undef PN_WIDE
    }
  }
  if (tc && mode != PN_NEWTON) {
    if constexpr (CELL == PN_CELL_GRU) {
      // three gates per channel: the row-major kernel (D = 32)
      if (DP == 32) {
        if (mode == PN_JACOBI) return diag_tc_kinfo<CELL, PN_JACOBI, 32>();
        if (mode == PN_PICARD) return diag_tc_kinfo<CELL, PN_PICARD, 32>();
        return diag_tc_kinfo<CELL, PN_QUASI, 32>();
      }
    } else {
      // quasi-Newton: the channel-major kernel (sequential in-register scan); Jacobi and
      // Picard: the row-major one (half the tensor-core operand traffic, cheap scan)
      if (DP == 32) {
        if (mode == PN_JACOBI) return diag_tc_kinfo<CELL, PN_JACOBI, 32>();
        if (mode == PN_PICARD) return diag_tc_kinfo<CELL, PN_PICARD, 32>();
        return diag_tct_kinfo<CELL, PN_QUASI, 32>();
      }
      if (DP == 64) {
        if (mode == PN_JACOBI) return diag_tc_kinfo<CELL, PN_JACOBI, 64>();
        if (mode == PN_PICARD) return diag_tc_kinfo<CELL, PN_PICARD, 64>();
        return diag_tct_kinfo<CELL, PN_QUASI, 64>();
      }
    }
  }
#define PN_DIAG_CASES(MODE)                                                              \
  switch (DP) {                                                                          \
    case 4: return diag_pick<CELL, MODE, 4>();                                           \
    case 8: return diag_pick<CELL, MODE, 8>();                                           \
    case 16: return diag_pick<CELL, MODE, 16>();                                         \
    case 32: return tma ? diag_tma_pick<CELL, MODE, 32>() : diag_pick<CELL, MODE, 32>();     \
    case 64: return tma ? diag_tma_pick<CELL, MODE, 64>() : diag_pick<CELL, MODE, 64>();     \
    case 128: return tma ? diag_tma_pick<CELL, MODE, 128>() : diag_pick<CELL, MODE, 128>(); \
    case 256: return tma ? diag_tma_pick<CELL, MODE, 256>() : diag_pick<CELL, MODE, 256>(); \
    default: return none;                                                                \
  }
  switch (mode) {
    case PN_JACOBI: PN_DIAG_CASES(PN_JACOBI)
    case PN_PICARD: PN_DIAG_CASES(PN_PICARD)
    case PN_QUASI: PN_DIAG_CASES(PN_QUASI)
    case PN_NEWTON:
      switch (DP) {
        case 4: return dense_pick<CELL, 4>();
        case 8: return dense_pick<CELL, 8>();
        case 16: return dense_pick<CELL, 16>();
        case 32: return dense_pick<CELL, 32>();
        case 64: return dense_pick<CELL, 64>();
        default: return none;
      }
    default: return none;
  }
#undef PN_DIAG_CASES
}

// The single-CTA Newton solve (DP = 4, 8): its kernel (smem: set by the caller from small_smem_bytes).
template <int CELL>
inline KInfo small_cell(int DP) {
  if (DP == 4) return KInfo{(const void*)&small_solve_kernel<CELL, 4>, SmallCfg<CELL, 4>::NT, 32, 4, 0, kKindDense};
  if (DP == 8) return KInfo{(const void*)&small_solve_kernel<CELL, 8>, SmallCfg<CELL, 8>::NT, 32, 8, 0, kKindDense};
  return KInfo{nullptr, 0, 0, 0, 0, 0};
}
inline size_t small_smem_bytes(int cell, int DP, int B, int T) {
  auto pick = [&](auto cfg4, auto cfg8) -> size_t {
    return DP == 4 ? decltype(cfg4)::smem_bytes(B, T) : decltype(cfg8)::smem_bytes(B, T);
  };
  switch (cell) {
    case PN_CELL_TANH_RNN: return pick(SmallCfg<PN_CELL_TANH_RNN, 4>{}, SmallCfg<PN_CELL_TANH_RNN, 8>{});
    case PN_CELL_GRU: return pick(SmallCfg<PN_CELL_GRU, 4>{}, SmallCfg<PN_CELL_GRU, 8>{});
    default: return pick(SmallCfg<PN_CELL_EULER_TANH, 4>{}, SmallCfg<PN_CELL_EULER_TANH, 8>{});
  }
}

// Defined in one translation unit per cell (compiled in parallel).
KInfo lookup_tanh(int mode, int DP, bool tma, bool tc);
KInfo lookup_gru(int mode, int DP, bool tma, bool tc);
KInfo lookup_euler(int mode, int DP, bool tma, bool tc);
KInfo small_tanh(int DP);
KInfo small_gru(int DP);
KInfo small_euler(int DP);

inline KInfo lookup_small(int cell, int DP) {
  switch (cell) {
    case PN_CELL_TANH_RNN: return small_tanh(DP);
    case PN_CELL_GRU: return small_gru(DP);
    case PN_CELL_EULER_TANH: return small_euler(DP);
    default: return KInfo{nullptr, 0, 0, 0, 0, 0};
  }
}

inline KInfo lookup(int cell, int mode, int DP, bool tma, bool tc) {
  switch (cell) {
    case PN_CELL_TANH_RNN: return lookup_tanh(mode, DP, tma, tc);
    case PN_CELL_GRU: return lookup_gru(mode, DP, tma, tc);
    case PN_CELL_EULER_TANH: return lookup_euler(mode, DP, tma, tc);
    default: return KInfo{nullptr, 0, 0, 0, 0, 0};
  }
}

}  // namespace pn
