// pn_aux.cuh -- kernels around the convergence loop: the input projection
// (hoisted out of the loop, since f_t depends on t only through x_t), the
// initial guess s^(0)_t = s0, and the final copy of the result.
#pragma once

#include "pn_common.cuh"

namespace pn {

// out[r][n] = sum_k in[r][k] * Wm[n][k] + bias[n] for r < M, n < N, k < K,
// where `in` is args->x ([M][K] with M = B*T).  64 x 64 output tile per CTA,
// 4 x 4 per thread, K staged through shared memory in slabs of 16.
constexpr int kProjTile = 64;
constexpr int kProjK = 16;
__global__ void __launch_bounds__(256) proj_kernel(const Args* __restrict__ args,
                                                   const float* __restrict__ Wm,
                                                   const float* __restrict__ bias,
                                                   float* __restrict__ out, int M, int N, int K) {
  __shared__ __align__(16) float sIn[kProjK][kProjTile + 4];
  __shared__ __align__(16) float sWm[kProjK][kProjTile + 4];
  const float* __restrict__ in = args->x;
  const int tid = threadIdx.x;
  const int tr = tid / 16;   // rows tr*4 .. tr*4+3
  const int tc = tid % 16;   // cols tc*4 .. tc*4+3
  const long r0 = (long)blockIdx.x * kProjTile;
  const int n0 = blockIdx.y * kProjTile;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[a][c] = 0.0f;
  for (int k0 = 0; k0 < K; k0 += kProjK) {
    for (int e = tid; e < kProjTile * kProjK; e += 256) {
      const int rr = e / kProjK, kk = e % kProjK;
      const long r = r0 + rr;
      const int k = k0 + kk;
      sIn[kk][rr] = (r < M && k < K) ? __ldg(in + r * K + k) : 0.0f;
      const int n = n0 + rr;
      sWm[kk][rr] = (n < N && k < K) ? __ldg(Wm + (long)n * K + k) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kProjK; ++kk) {
      const float4 a4 = *reinterpret_cast<const float4*>(&sIn[kk][tr * 4]);
      const float4 w4 = *reinterpret_cast<const float4*>(&sWm[kk][tc * 4]);
      const float av[4] = {a4.x, a4.y, a4.z, a4.w};
      const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(av[a], wv[c], acc[a][c]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const long r = r0 + tr * 4 + a;
    if (r >= M) continue;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int n = n0 + tc * 4 + c;
      if (n < N) out[r * N + n] = acc[a][c] + __ldg(bias + n);
    }
  }
}

// s^(0)_t = s0 for every t, and a fresh control block for the loop.  Each
// blockIdx.y takes whole sequences (b = blockIdx.y, + gridDim.y, ...), the x
// dimension strides over one sequence; 16-byte stores when D % 4 == 0.
__global__ void init_kernel(const Args* __restrict__ args, Ctrl* __restrict__ ctrl, int D, int T,
                            int B) {
  const size_t per_seq = (size_t)T * D;
  const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t nthr = (size_t)gridDim.x * blockDim.x;
  const int fmt = args->store_fmt;   // s^(0) is stored in the narrow format when one is set
  for (int b = blockIdx.y; b < B; b += gridDim.y) {
    const float* s0 = args->s0 + (size_t)b * D;
    float* st = args->states + (size_t)b * per_seq;
    if (fmt != 0) {
      for (size_t e = tid; e < per_seq; e += nthr) st_state(args->states, (size_t)b * per_seq + e, __ldg(s0 + e % (size_t)D), fmt);
    } else if ((D & 3) == 0) {
      const size_t D4 = (size_t)(D >> 2);
      const float4* s04 = reinterpret_cast<const float4*>(s0);
      float4* st4 = reinterpret_cast<float4*>(st);
      for (size_t e = tid; e < per_seq / 4; e += nthr) st4[e] = __ldg(s04 + e % D4);
    } else {
      for (size_t e = tid; e < per_seq; e += nthr) st[e] = __ldg(s0 + e % (size_t)D);
    }
  }
  if (blockIdx.y == 0 && blockIdx.x == 0 && threadIdx.x == 0) {
    ctrl->iter = 0;
    ctrl->status = kRunning;
    ctrl->error = 0;
    ctrl->final_iter = 0;
    ctrl->final_resid = 0.0f;
    ctrl->resid_bits = 0u;
    for (int g = 0; g < kMaxGroups; ++g) ctrl->ticket[g] = 0u;
    ctrl->done = 0u;
    ctrl->arrive = 0ull;
    ctrl->resid_loop[0] = 0u;
    ctrl->resid_loop[1] = 0u;
    ctrl->sync_count = 0u;
    ctrl->timeout_ticket = -1;
    ctrl->t_start = ~0ull;
    ctrl->fmt_in = fmt != 0;    // s^(0) and s^(1) are narrow when a narrow format is set
    ctrl->fmt_out = fmt != 0;
    ctrl->final_fmt = 0;
    ctrl->cur_mode = args->start_mode;
    ctrl->retried = 0;
  }
}

// The result is s^(final_iter), which lives in buffer (final_iter & 1), in
// float32 or (final_fmt) in the narrow storage format.  Pass 1 moves it into
// the caller's states buffer as float32: a copy from the work buffer, or a
// widening of the narrow copy in the work buffer.  Pass 0 runs first when a
// narrow format is set: a narrow result in the caller's buffer (the first half
// of it) is moved to the work buffer, so pass 1 never widens in place.
__global__ void finish_kernel(const Args* __restrict__ args, const Ctrl* __restrict__ ctrl,
                              float* __restrict__ buf1, size_t n, int pass) {
  const int fi = *(const volatile int*)&ctrl->final_iter;
  const int narrow = *(const volatile int*)&ctrl->final_fmt;
  const int fmt = args->store_fmt;
  const size_t g0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t gs = (size_t)gridDim.x * blockDim.x;
  if (pass == 0) {
    if (!narrow || (fi & 1)) return;
    const unsigned short* src = reinterpret_cast<const unsigned short*>(args->states);
    unsigned short* dst = reinterpret_cast<unsigned short*>(buf1);
    for (size_t e = g0; e < n; e += gs) dst[e] = src[e];
    return;
  }
  if (narrow) {
    for (size_t e = g0; e < n; e += gs) args->states[e] = ld_state(buf1, e, fmt);
    return;
  }
  if ((fi & 1) == 0) return;
  float* st = args->states;
  const size_t n4 = n / 4;
  const float4* s4 = reinterpret_cast<const float4*>(buf1);
  float4* d4 = reinterpret_cast<float4*>(st);
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n4;
       e += (size_t)gridDim.x * blockDim.x)
    d4[e] = __ldcs(s4 + e);
  for (size_t e = n4 * 4 + (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x)
    st[e] = buf1[e];
}

// y[e] = activation(x[e]) with the cells' device activations.
__global__ void activation_kernel(int which, const float* __restrict__ x, float* __restrict__ y, long long n) {
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x)
    y[e] = which == 0 ? tanh_pn(x[e]) : sigmoid_pn(x[e]);
}

}  // namespace pn
