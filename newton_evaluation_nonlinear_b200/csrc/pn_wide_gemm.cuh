// pn_wide_gemm.cuh -- a 3xTF32 tcgen05 GEMM Y = X W^T (+ bias) over all B*T
// rows, with W streamed from L2 in 32-column K chunks.  It forms the cell's
// recurrent product for wide states (D = 128, 256: X = the iterate, W = the
// recurrent weights) and the hoisted input projection (X = x, W = U or W_ih).
//
// At D = 256 one step's W s costs 2 D^2 = 131 kflop, so an iteration of the
// Euler workload (B = 32, T = 1024) is 4.3 GFLOP: about 60 us of the FP32 FMA
// peak against 15 us of HBM traffic, and W_hi + W_lo (512 KB) do not fit in
// shared memory.  Here the product runs as a plain GEMM on the tensor cores
// (rows r = b T + t of the iterate, Y[r][n] = sum_k S[r][k] W[n][k] =
// (W s_r)[n]) and the fused cell + Jacobian + scan kernel reads Y instead of
// forming W s itself ("Parallel Newton methods..." page, §5.2: tensor cores as
// the hardware lever; the iteration itself is §1.2 and §2.2).  Products are
// 3xTF32 as in the other tensor-core kernels: S W_hi + S W_lo + S_lo W_hi,
// with S read by the tensor core as its TF32 truncation and S_lo the exact
// remainder, formed in shared memory.
//
// Per CTA (persistent, static round-robin over 128-row tiles):
//   warp 0   producer: per (tile, K chunk) one TMA load of the S chunk
//            (128 rows x 32 floats) and of W_hi and W_lo (D rows x 32),
//            128-byte swizzled, into a stage of the ring;
//   warp 1   MMA issuer: 3 passes x 4 K-steps per chunk into one of two TMEM
//            accumulators (128 lanes x D columns); a commit frees the stage;
//   warps 2-3, 8-9  S_lo of each landed S chunk (element-wise: the swizzled
//            layout is the same for both);
//   warps 4-7  epilogue: thread = row, TMEM -> registers -> Y; for N a multiple
//            of 32 through a double-buffered 128 x 32 staging tile (128-byte
//            swizzled) and one TMA tensor store per 32 columns, so that Y is
//            written in whole lines (a warp's direct stores would touch 32
//            rows each).
// TMA loads never use cluster multicast.  Rows past B*T read as zero and are
// not stored.
#pragma once

#include "pn_iter_diag_tc.cuh"

namespace pn {

// N output columns (the rows of W), a multiple of 16 up to 256.
template <int N>
struct WideGemmCfg {
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "N: a multiple of 16, at most 256");
  static constexpr int BM = 128;                  // rows per tile
  static constexpr int KC = 32;                   // K chunk: one 128-byte swizzle row of fp32
  static constexpr int S_BYTES = BM * KC * 4;     // 16 KB
  static constexpr int W_BYTES = N * KC * 4;
  static constexpr int STAGE = 2 * S_BYTES + 2 * W_BYTES;   // S, S_lo, W_hi, W_lo
  static constexpr int NSTAGE = (200 * 1024) / STAGE < 4 ? (200 * 1024) / STAGE : 4;
  static constexpr int TCOLS = (2 * N <= 32) ? 32 : (2 * N <= 64) ? 64 : (2 * N <= 128) ? 128 : (2 * N <= 256) ? 256 : 512;
  static constexpr int NT = 320;                  // 10 warps: producer, MMA, 2 + 2 split, 4 epilogue
  static constexpr bool kStaged = (N % 32) == 0;  // epilogue through the staging tile and TMA stores
  static constexpr int OUT_BYTES = BM * 32 * 4;   // one staging buffer: 128 rows x 32 floats
  static constexpr int OFF_OUT = NSTAGE * STAGE;  // two staging buffers after the ring
  static constexpr int SMEM_BYTES = NSTAGE * STAGE + (kStaged ? 2 * OUT_BYTES : 0) + 1024;   // + alignment slack
  static_assert(NSTAGE >= 2, "two stages at least");
  static_assert(STAGE % 1024 == 0, "stages stay 1024-byte aligned");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

// 2-D TMA tensor store of one box from shared memory (coordinates >= 0); elements outside the
// array are not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int c0, int c1, const void* src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(map), "r"(c0), "r"(c1),
               "r"(smem_addr(src))
               : "memory");
}
// this thread's committed bulk stores, all but the most recent group, have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_but1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }

// 2-D TMA tensor load (coordinates: column c0, row c1), counted on bar.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_addr(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_addr(bar))
      : "memory");
}

// Y[r][n] = sum_k X[r][k] W[n][k] (+ bias[n]) for r < rows, n < N, k < K.  maps: [0] X of iterate
// buffer 0 and [1] of buffer 1 (the iteration's parity picks one; the input projection passes the
// same map twice), [2] W_hi, [3] W_lo, [4] Y (stores, 128 rows x 32 floats, 128-byte swizzled;
// used when N is a multiple of 32).  K need not be a multiple of 32 (the loads zero-fill).
template <int N>
__global__ void __launch_bounds__(WideGemmCfg<N>::NT, 1) wide_gemm_kernel(const CUtensorMap* __restrict__ maps, float* __restrict__ Y,
                                                           int rows, int K, const float* __restrict__ bias, Ctrl* ctrl,
                                                           const Args* __restrict__ args) {
  using C = WideGemmCfg<N>;
  constexpr int DP = N;
  constexpr int NS = C::NSTAGE;
  const int NKC = (K + C::KC - 1) / C::KC;
  extern __shared__ __align__(1024) unsigned char smem_wg[];
  unsigned char* ring = smem_wg + ((1024u - (smem_addr(smem_wg) & 1023u)) & 1023u);
  __shared__ __align__(8) uint64_t bar_full[NS], bar_lo[NS], bar_empty[NS], bar_acc[2], bar_accfree[2];
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ int s_loaded, s_issued;   // units whose loads / products were issued (for the drain)

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const long long tmo = args->timeout_ns;
  const int iter = *(volatile int*)&ctrl->iter;
  const CUtensorMap* mS = maps + ((iter & 1) ? 1 : 0);   // s^(i)
  const CUtensorMap* mWh = maps + 2;
  const CUtensorMap* mWl = maps + 3;
  const int ntiles = (rows + C::BM - 1) / C::BM;
  const int my_tiles = (ntiles > (int)blockIdx.x) ? (ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int units = my_tiles * NKC;

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar_full[s], 1u);
      mbar_init(&bar_lo[s], 4u);
      mbar_init(&bar_empty[s], 1u);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bar_acc[a], 1u);
      mbar_init(&bar_accfree[a], 4u);
    }
    mbar_init_fence();
    s_abort = 0;
    s_loaded = 0;
    s_issued = 0;
  }
  if (warp == 0) {
    tmem_alloc(&s_tmem, (uint32_t)C::TCOLS);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  auto sbuf = [&](int s) { return ring + s * C::STAGE; };                 // S chunk
  auto lbuf = [&](int s) { return ring + s * C::STAGE + C::S_BYTES; };    // S_lo
  auto hbuf = [&](int s) { return ring + s * C::STAGE + 2 * C::S_BYTES; };   // W_hi
  auto wlbuf = [&](int s) { return hbuf(s) + C::W_BYTES; };                  // W_lo

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      tmap_acquire(mS);
      tmap_acquire(mWh);
      tmap_acquire(mWl);
      asm volatile("fence.proxy.async.global;" ::: "memory");   // s^(i) written by the previous kernel
      for (int u = 0; u < units; ++u) {
        const int s = u % NS;
        if (u >= NS && !mbar_wait_flag(&bar_empty[s], (unsigned)((u / NS) - 1) & 1u, ctrl, tmo, &s_abort)) break;
        const int tile = (int)blockIdx.x + (u / NKC) * (int)gridDim.x;
        const int kc = u % NKC;
        mbar_arrive_expect_tx(&bar_full[s], (unsigned)(C::S_BYTES + 2 * C::W_BYTES));
        tma_load_2d(sbuf(s), mS, kc * C::KC, tile * C::BM, &bar_full[s]);
        tma_load_2d(hbuf(s), mWh, kc * C::KC, 0, &bar_full[s]);
        tma_load_2d(wlbuf(s), mWl, kc * C::KC, 0, &bar_full[s]);
        s_loaded = u + 1;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t idesc = umma_idesc_tf32(C::BM, DP);
    for (int u = 0; u < units; ++u) {
      const int s = u % NS;
      const int j = u / NKC;    // this CTA's tile number
      const int kc = u % NKC;
      const int acc = j & 1;
      if (kc == 0 && j >= 2 && !mbar_wait_flag(&bar_accfree[acc], (unsigned)((j >> 1) - 1) & 1u, ctrl, tmo, &s_abort))
        break;
      if (!mbar_wait_flag(&bar_lo[s], (unsigned)(u / NS) & 1u, ctrl, tmo, &s_abort)) break;
      tc_fence_after();
      if (lane == 0) {
        const uint64_t a_hi = umma_smem_desc(smem_addr(sbuf(s)), 16, 1024, 2);
        const uint64_t a_lo = umma_smem_desc(smem_addr(lbuf(s)), 16, 1024, 2);
        const uint64_t b_hi = umma_smem_desc(smem_addr(hbuf(s)), 16, 1024, 2);
        const uint64_t b_lo = umma_smem_desc(smem_addr(wlbuf(s)), 16, 1024, 2);
        const uint32_t d = tmem + (uint32_t)(acc * DP);
#pragma unroll
        for (int ks = 0; ks < C::KC / 8; ++ks) {
          const uint64_t ko = (uint64_t)((ks * 32) >> 4);   // 8 fp32 of K = 32 bytes along the swizzled row
          umma_tf32(d, a_hi + ko, b_hi + ko, idesc, (kc | ks) ? 1u : 0u);
          umma_tf32(d, a_hi + ko, b_lo + ko, idesc, 1u);
          umma_tf32(d, a_lo + ko, b_hi + ko, idesc, 1u);
        }
        umma_commit(&bar_empty[s]);                 // the stage is free once these products are done
        if (kc == NKC - 1) umma_commit(&bar_acc[acc]);   // the tile's accumulator is complete
        s_issued = u + 1;
      }
      __syncwarp();
    }
  } else if (warp < 4 || warp >= 8) {
    // ---------------- S_lo (warps 2, 3, 8, 9) ----------------
    const int t = (warp < 4) ? tid - 64 : tid - 192;   // 0 .. 127
    for (int u = 0; u < units; ++u) {
      const int s = u % NS;
      if (!mbar_wait_flag(&bar_full[s], (unsigned)(u / NS) & 1u, ctrl, tmo, &s_abort)) break;
      const float4* src = reinterpret_cast<const float4*>(sbuf(s));
      float4* dst = reinterpret_cast<float4*>(lbuf(s));
#pragma unroll 4
      for (int e = t; e < C::S_BYTES / 16; e += 128) {
        const float4 v = src[e];
        dst[e] = make_float4(tf32_tail(v.x), tf32_tail(v.y), tf32_tail(v.z), tf32_tail(v.w));
      }
      fence_async_smem();   // generic writes -> the tensor cores
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_lo[s]);
    }
  } else if constexpr (C::kStaged) {
    // ---------------- epilogue: thread = row, staged TMA stores ----------------
    const int q = warp & 3;   // TMEM lane quarter
    const int r = 32 * q + lane;   // row of the tile
    const bool issuer = (warp == 4 && lane == 0);
    const CUtensorMap* mY = maps + 4;
    if (issuer) tmap_acquire(mY);
    int nst = 0;   // staging buffers filled so far (buffer nst & 1 next)
    for (int j = 0; j < my_tiles; ++j) {
      const int acc = j & 1;
      // the four warps meet the staging barriers together: all go on, or all stop, here
      const bool ok = mbar_wait_flag(&bar_acc[acc], (unsigned)(j >> 1) & 1u, ctrl, tmo, &s_abort);
      if (!named_barrier_and(1, 128, ok)) break;
      tc_fence_after();
      const int tile = (int)blockIdx.x + j * (int)gridDim.x;
      const uint32_t base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * DP);
#pragma unroll 1
      for (int c = 0; c < DP; c += 32, ++nst) {
        unsigned char* ob = ring + C::OFF_OUT + (nst & 1) * C::OUT_BYTES;
        // the store that last read this buffer (two back) is done with it
        if (issuer && nst >= 2) bulk_wait_read_but1();
        named_barrier(1, 128);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float v[16];
          tmem_ld16(base + (uint32_t)(c + 16 * hh), v);
          if (bias) {
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] += __ldg(bias + c + 16 * hh + e);
          }
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<float4*>(ob + sw128_offset(r, 16 * hh + e)) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
        fence_async_smem();   // generic writes -> the tensor store (async proxy)
        named_barrier(1, 128);
        if (issuer) {
          tma_store_2d(mY, c, tile * C::BM, ob);
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_accfree[acc]);
    }
    if (issuer) bulk_wait_all();   // Y is in global memory (and the staging buffers read) before the CTA retires
    __syncwarp();
  } else {
    // ---------------- epilogue: thread = row ----------------
    const int q = warp & 3;   // TMEM lane quarter
    for (int j = 0; j < my_tiles; ++j) {
      const int acc = j & 1;
      if (!mbar_wait_flag(&bar_acc[acc], (unsigned)(j >> 1) & 1u, ctrl, tmo, &s_abort)) break;
      tc_fence_after();
      const int tile = (int)blockIdx.x + j * (int)gridDim.x;
      const int row = tile * C::BM + 32 * q + lane;
      float* yr = Y + (size_t)row * DP;
      const uint32_t base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(acc * DP);
#pragma unroll 1
      for (int c = 0; c < DP; c += 16) {
        float v[16];
        tmem_ld16(base + (uint32_t)c, v);
        if (bias) {
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] += __ldg(bias + c + e);
        }
        if (row < rows) {
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<float4*>(yr + c + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_accfree[acc]);
    }
  }

  // every issued copy and product completes before the CTA releases TMEM and exits
  if (warp == 0 && lane == 0) {
    const int n = s_loaded;
    for (int u = max(0, n - NS); u < n; ++u)
      if (!mbar_drain(&bar_full[u % NS], (unsigned)(u / NS) & 1u, tmo)) raise_error(ctrl, (int)PN_ERR_TIMEOUT);
  }
  if (warp == 1 && lane == 0) {
    const int n = s_issued;
    for (int u = max(0, n - NS); u < n; ++u)
      if (!mbar_drain(&bar_empty[u % NS], (unsigned)(u / NS) & 1u, tmo)) raise_error(ctrl, (int)PN_ERR_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    tmem_dealloc(tmem, (uint32_t)C::TCOLS);
}

}  // namespace pn
