// pn_cells.cuh -- per-cell constants shared by the fused iteration kernels.
//
// The three cells (benchmark definitions; GRU in the PyTorch gate order):
//   tanh RNN : f_t(s) = tanh(W s + u_t),           u_t = U x_t + b (hoisted)
//   GRU      : r = sig(gx_r + W_hr h), z = sig(gx_z + W_hz h),
//              n = tanh(gx_n + r (W_hn h + b_hn)),  h' = (1-z) n + z h,
//              gx = W_ih x_t + b_ih + [b_hr; b_hz; 0]  (hoisted)
//   Euler    : f_t(s) = s + eps tanh(W s + c_t)
// R is the number of D x D recurrent weight blocks a channel needs.
#pragma once

#include "pn_common.cuh"

namespace pn {

template <int CELL>
struct CellInfo;
template <>
struct CellInfo<PN_CELL_TANH_RNN> {
  static constexpr int R = 1;
};
template <>
struct CellInfo<PN_CELL_GRU> {
  static constexpr int R = 3;  // gate blocks r, z, n of W_hh
};
template <>
struct CellInfo<PN_CELL_EULER_TANH> {
  static constexpr int R = 1;
};

// Vector load / store of N consecutive floats (N = 1, 2, 4) when aligned,
// element-wise with a bound otherwise.
template <int N>
__device__ __forceinline__ void load_n(const float* p, float (&v)[N], int valid, bool vec_ok) {
  if (N == 4 && vec_ok && valid >= 4) {
    float4 q = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
  } else if (N == 2 && vec_ok && valid >= 2) {
    float2 q = __ldg(reinterpret_cast<const float2*>(p));
    v[0] = q.x; v[1] = q.y;
  } else {
#pragma unroll
    for (int n = 0; n < N; ++n) v[n] = (n < valid) ? __ldg(p + n) : 0.0f;
  }
}

template <int N>
__device__ __forceinline__ void store_n(float* p, const float (&v)[N], int valid, bool vec_ok) {
  if (N == 4 && vec_ok && valid >= 4) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  } else if (N == 2 && vec_ok && valid >= 2) {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
  } else {
#pragma unroll
    for (int n = 0; n < N; ++n)
      if (n < valid) p[n] = v[n];
  }
}

}  // namespace pn
