// pn_k_euler.cu -- fused iteration kernels instantiated for the euler cell.
#include "pn_dispatch.cuh"

namespace pn {
KInfo lookup_euler(int mode, int DP, bool tma, bool tc) { return lookup_cell<PN_CELL_EULER_TANH>(mode, DP, tma, tc); }
KInfo small_euler(int DP) { return small_cell<PN_CELL_EULER_TANH>(DP); }
}  // namespace pn
