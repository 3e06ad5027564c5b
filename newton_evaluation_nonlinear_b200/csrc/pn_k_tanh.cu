// pn_k_tanh.cu -- fused iteration kernels instantiated for the tanh cell.
#include "pn_dispatch.cuh"

namespace pn {
KInfo lookup_tanh(int mode, int DP, bool tma, bool tc) { return lookup_cell<PN_CELL_TANH_RNN>(mode, DP, tma, tc); }
KInfo small_tanh(int DP) { return small_cell<PN_CELL_TANH_RNN>(DP); }
}  // namespace pn
