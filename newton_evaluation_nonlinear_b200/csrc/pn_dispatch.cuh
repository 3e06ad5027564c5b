// pn_dispatch.cuh -- launch shapes of the fused iteration kernels.
//
// The padded state width DP is the smallest of 4, 8, ..., 256 that holds D;
// each (cell, DP) has one tile shape for the diagonal-family kernel (channel
// group G, TM steps x TN channels per thread, TS thread segments along t) and
// one for the dense Newton kernel (L steps x DP channels per CTA).
#pragma once

#include "pn_iter_dense.cuh"
#include "pn_iter_diag.cuh"

namespace pn {

struct KInfo {
  const void* fn;   // __global__ function
  int nt;           // threads per CTA
  int L;            // steps per tile
  int G;            // channels per tile
  size_t smem;      // dynamic shared memory bytes
};

template <int CELL, int MODE, int DP, int G, int TM, int TN, int TS>
inline KInfo diag_kinfo() {
  using C = DiagCfg<CELL, MODE, DP, G, TM, TN, TS>;
  return KInfo{(const void*)&diag_iter_kernel<CELL, MODE, DP, G, TM, TN, TS>, C::NT, C::L, G,
               C::SMEM_BYTES};
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

template <int CELL, int DP, int L>
inline KInfo dense_kinfo() {
  using C = DenseCfg<CELL, DP, L>;
  return KInfo{(const void*)&dense_iter_kernel<CELL, DP, L>, C::NT, L, DP, C::SMEM_BYTES};
}

template <int CELL, int DP>
inline KInfo dense_pick() {
  if constexpr (DP == 4) return dense_kinfo<CELL, 4, 64>();
  else if constexpr (DP == 8) return dense_kinfo<CELL, 8, 32>();
  else if constexpr (DP == 16) return dense_kinfo<CELL, 16, 16>();
  else if constexpr (DP == 32) return dense_kinfo<CELL, 32, 8>();
  else {
    if constexpr (CELL == PN_CELL_GRU) return dense_kinfo<CELL, 64, 2>();
    else return dense_kinfo<CELL, 64, 4>();
  }
}

template <int CELL>
inline KInfo lookup_cell(int mode, int DP) {
  KInfo none{nullptr, 0, 0, 0, 0};
#define PN_DIAG_CASES(MODE)                                 \
  switch (DP) {                                             \
    case 4: return diag_pick<CELL, MODE, 4>();              \
    case 8: return diag_pick<CELL, MODE, 8>();              \
    case 16: return diag_pick<CELL, MODE, 16>();            \
    case 32: return diag_pick<CELL, MODE, 32>();            \
    case 64: return diag_pick<CELL, MODE, 64>();            \
    case 128: return diag_pick<CELL, MODE, 128>();          \
    case 256: return diag_pick<CELL, MODE, 256>();          \
    default: return none;                                   \
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

// Defined in one translation unit per cell (compiled in parallel).
KInfo lookup_tanh(int mode, int DP);
KInfo lookup_gru(int mode, int DP);
KInfo lookup_euler(int mode, int DP);

inline KInfo lookup(int cell, int mode, int DP) {
  switch (cell) {
    case PN_CELL_TANH_RNN: return lookup_tanh(mode, DP);
    case PN_CELL_GRU: return lookup_gru(mode, DP);
    case PN_CELL_EULER_TANH: return lookup_euler(mode, DP);
    default: return KInfo{nullptr, 0, 0, 0, 0};
  }
}

}  // namespace pn
