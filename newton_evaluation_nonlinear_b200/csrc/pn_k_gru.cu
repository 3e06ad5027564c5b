// pn_k_gru.cu -- fused iteration kernels instantiated for the gru cell.
#include "pn_dispatch.cuh"

namespace pn {
KInfo lookup_gru(int mode, int DP, bool tma, bool tc) { return lookup_cell<PN_CELL_GRU>(mode, DP, tma, tc); }
KInfo small_gru(int DP) { return small_cell<PN_CELL_GRU>(DP); }
}  // namespace pn
