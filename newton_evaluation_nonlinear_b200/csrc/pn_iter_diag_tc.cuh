// pn_iter_diag_tc.cuh -- fused iteration kernel for the Jacobi, Picard and
// diagonal quasi-Newton modes with the cell's recurrent matvec on the
// 5th-generation tensor cores (tcgen05, accumulators in TMEM).  D = 32 or 64.
//
// The iteration is the page's unified update ("Parallel Newton methods..."
// page, §1.2) with a diagonal A~_t (§2.2.1, §2.2.3), solved by the chunked
// scan of §2.1, exactly as in pn_iter_diag.cuh; what changes is how the
// matvec W s_{t-1} of all L = 128 steps of a tile is formed: as one
// 128 x N x D product Z = S W^T (S = the tile's s^(i) rows, N = R*D) on the
// tensor cores, split into three TF32 products
//     Z = S W + S W_lo + S_lo W,   x_lo = x - tf32(x),
// which keeps the products to about 2^-22 relative error (fp32 level) while
// the tensor pipe does the multiply-adds.
//
// Warp roles (one CTA per SM, 3 + D/4 warps):
//   warp 0     producer: claims tiles (ticket order) and stages the s rows
//              t0-1..t0+L-1 and the step inputs with ONE 2-D TMA tensor load
//              each.  The boxes are 4 columns wider than the tensors, so the
//              hardware zero-fills 16 bytes at the end of every row and the
//              rows land padded (conflict-free column reads);
//   warp 1     MMA issuer: one thread issues the 3 x D/8 tcgen05.mma of a
//              tile into one of two TMEM accumulators, commits to an mbarrier;
//   warp 2     look-back: finds the nearest predecessor with a published
//              state, folds the aggregates in between, publishes the tile's
//              end state and hands the carry to the epilogue;
//   warps 3..  epilogue, four row quarters x D/16 channel groups: one thread
//              per step row (TMEM lane) and 16 channels.  Reads Z from TMEM,
//              evaluates the cell, the diagonal Jacobian and |F|, scans along
//              the rows (warp shuffles, all 16 channels level by level, then
//              across the row quarters), publishes the tile aggregate,
//              prepares the next tile's tensor-core operands and parks the
//              in-tile prefixes in TMEM.  A tile's states are written one tile
//              later, when the look-back warp has had a whole tile of time to
//              deliver its carry.
#pragma once

#include <string.h>

#include "pn_cells.cuh"
#include "pn_tma.cuh"

namespace pn {

// --- tcgen05 helpers (inline PTX) ------------------------------------------

// Canonical K-major layout without swizzle ("interleaved" core matrices):
// a core matrix is 8 rows x 16 bytes stored contiguously; core matrices
// adjacent along K are 128 bytes apart (leading byte offset) and groups of 8
// rows are K/4 * 128 bytes apart (stride byte offset).
__host__ __device__ __forceinline__ uint32_t kmajor_offset(int row, int k, int K) {
  return (uint32_t)((row >> 3) * (K / 4) * 128 + (k >> 2) * 128 + (row & 7) * 16 + (k & 3) * 4);
}

// Shared-memory matrix descriptor (sm_100): start address >> 4 in bits 0-13,
// leading byte offset >> 4 in bits 16-29, stride byte offset >> 4 in bits
// 32-45, version 1 in bits 46-47, no swizzle (bits 61-63 = 0).
__device__ __forceinline__ uint64_t umma_smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}

// Instruction descriptor for kind::tf32: D fp32 (bit 4), A and B tf32 (code 2
// at bits 7 and 10), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t umma_idesc_tf32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_tf32(uint32_t dtmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(dtmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 16 consecutive fp32 columns of this warp's 32 TMEM lanes: thread i gets lane i.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}

// Store 16 fp32 columns into this warp's 32 TMEM lanes (thread i -> lane i).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// The tensor map was written to global memory by a host copy before this
// launch: order that write before the tensor-map proxy reads it.
__device__ __forceinline__ void tmap_acquire(const CUtensorMap* map) {
  asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(map) : "memory");
}

// 2-D TMA tensor load of one box at element coordinates (c0, c1) into this
// CTA's shared memory (128-byte aligned), counted on `bar`.  c0 is 0 here
// (16-byte aligned); c1 may be -1, where the hardware zero-fills the row.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_addr(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_addr(bar))
      : "memory");
}

// Round to the nearest TF32 value (10 explicit mantissa bits): the tensor
// core ignores the low 13 bits, so pre-rounded operands lose nothing more.
// The device form skips the inf/NaN guard: a non-finite iterate ends the
// solve as non-finite whatever its rounding.
__host__ __device__ __forceinline__ float tf32_round(float x) {
#ifdef __CUDA_ARCH__
  return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xFFFFE000u);
#else
  uint32_t u;
  memcpy(&u, &x, 4);
  if ((u & 0x7F800000u) != 0x7F800000u) u = (u + 0x1000u) & 0xFFFFE000u;
  float r;
  memcpy(&r, &u, 4);
  return r;
#endif
}

// Bounded mbarrier wait that never leaves the caller's control flow: on
// timeout / error it records the failure in *abort and returns false.
__device__ __forceinline__ bool mbar_wait_flag(uint64_t* bar, unsigned parity, Ctrl* ctrl, long long timeout_ns,
                                               volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  unsigned spins = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (((++spins) & 15u) == 0u) {
      if (*abort || ld_volatile(&ctrl->error)) {
        *abort = 1;
        return false;
      }
      if ((long long)(globaltimer() - t0) > timeout_ns) {
        atomicCAS(&ctrl->error, 0, (int)PN_ERR_TIMEOUT);
        *abort = 1;
        return false;
      }
    }
  }
}

template <int CELL, int MODE, int DP>
struct DiagTcCfg {
  static constexpr int R = CellInfo<CELL>::R;
  static constexpr int L = 128;                 // steps per tile = MMA M
  static constexpr int K = DP;                  // MMA K (input channels)
  static constexpr int N = R * DP;              // MMA N (output rows of W)
  static constexpr int TCOLS = N <= 64 ? 64 : (N <= 128 ? 128 : 256);   // TMEM columns per accumulator
  static constexpr int SCOLS = (MODE == PN_QUASI ? 2 : 1) * DP;        // stash columns per tile: [A |] B
  static constexpr int STASH0 = 2 * TCOLS;                              // first stash column
  static constexpr int USED_COLS = STASH0 + (MODE == PN_JACOBI ? 0 : 2 * SCOLS);
  static constexpr int ALLOC_COLS = USED_COLS <= 128 ? 128 : (USED_COLS <= 256 ? 256 : 512);
  static constexpr int CH = 16;                 // channels per epilogue thread
  static constexpr int NCG = DP / CH;           // channel groups
  static constexpr int NEW = 4 * NCG;           // epilogue warps: 4 row quarters x channel groups
  static constexpr int NTE = 32 * NEW;          // epilogue threads
  static constexpr int NT = 32 * (3 + NEW);
  static constexpr int SP = DP + 4;             // padded s row (floats) = TMA box width
  static constexpr int XP = R * DP + 4;         // padded step-input row (floats) = TMA box width
  static constexpr int NQ = (DP + 31) / 32;
  static constexpr uint32_t SBO_A = (K / 4) * 128;
  static constexpr uint32_t SBO_B = (K / 4) * 128;
  static constexpr int align(int v, int a) { return (v + a - 1) / a * a; }
  static constexpr int S_BYTES = (L + 1) * SP * 4;
  static constexpr int X_BYTES = L * XP * 4;
  static constexpr int A_BYTES = L * K * 4;
  static constexpr int B_BYTES = N * K * 4;
  static constexpr int OFF_S0 = 0;
  static constexpr int OFF_S1 = align(OFF_S0 + S_BYTES, 128);
  static constexpr int OFF_X = align(OFF_S1 + S_BYTES, 128);
  static constexpr int OFF_AH = align(OFF_X + X_BYTES, 128);
  static constexpr int OFF_AL = OFF_AH + A_BYTES;
  static constexpr int OFF_BH = OFF_AL + A_BYTES;
  static constexpr int OFF_BL = OFF_BH + B_BYTES;
  static constexpr int OFF_WD = OFF_BL + B_BYTES;                // R*DP floats: diagonals of W_q
  static constexpr int OFF_BHN = OFF_WD + R * DP * 4;            // DP floats
  static constexpr int OFF_TOT = OFF_BHN + DP * 4;               // [NCG][4 quarters][CH][2]
  static constexpr int OFF_AGG = OFF_TOT + NCG * 4 * CH * 2 * 4; // [2 slots][DP][2]
  static constexpr int OFF_CARRY = OFF_AGG + 2 * DP * 2 * 4;     // [2 slots][DP]
  static constexpr int OFF_RED = OFF_CARRY + 2 * DP * 4;         // NT/32 floats
  static constexpr int SMEM_USED = OFF_RED + (NT / 32) * 4;
  static constexpr int SMEM_BYTES = SMEM_USED + 128;             // + slack to align the base to 128 bytes
  static_assert(DP == 32 || DP == 64, "tensor-core path covers D = 32 and D = 64");
  static_assert(USED_COLS <= 512, "TMEM columns");
  static_assert(SP <= 256 && XP <= 256 && L + 1 <= 256, "TMA box extents");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

template <int CELL, int MODE, int DP>
__global__ void __launch_bounds__(DiagTcCfg<CELL, MODE, DP>::NT, 1) diag_tc_kernel(const IterParams P) {
  using C = DiagTcCfg<CELL, MODE, DP>;
  constexpr int R = C::R;
  constexpr int L = C::L;
  constexpr int K = C::K;
  constexpr int N = C::N;
  constexpr int SP = C::SP;
  constexpr int XP = C::XP;
  constexpr int CH = C::CH;
  constexpr int NTE = C::NTE;
  constexpr bool kScan = (MODE != PN_JACOBI);
  constexpr bool kHasA = (MODE == PN_QUASI);

  extern __shared__ __align__(128) unsigned char smem_tc[];
  // TMA destinations want 128-byte alignment: round the dynamic base up (the launch adds 128 bytes)
  unsigned char* smem_raw = smem_tc + ((128u - (smem_addr(smem_tc) & 127u)) & 127u);
  float* sS[2] = {reinterpret_cast<float*>(smem_raw + C::OFF_S0), reinterpret_cast<float*>(smem_raw + C::OFF_S1)};
  float* sX = reinterpret_cast<float*>(smem_raw + C::OFF_X);
  unsigned char* sAH = smem_raw + C::OFF_AH;
  unsigned char* sAL = smem_raw + C::OFF_AL;
  unsigned char* sBH = smem_raw + C::OFF_BH;
  unsigned char* sBL = smem_raw + C::OFF_BL;
  float* sWd = reinterpret_cast<float*>(smem_raw + C::OFF_WD);
  float* sBhn = reinterpret_cast<float*>(smem_raw + C::OFF_BHN);
  float* sTot = reinterpret_cast<float*>(smem_raw + C::OFF_TOT);
  float* sAgg = reinterpret_cast<float*>(smem_raw + C::OFF_AGG);
  float* sCarry = reinterpret_cast<float*>(smem_raw + C::OFF_CARRY);
  float* sRed = reinterpret_cast<float*>(smem_raw + C::OFF_RED);

  __shared__ __align__(8) uint64_t bar_sfull[2], bar_sempty[2], bar_xfull, bar_xempty, bar_afull,
      bar_mma[2], bar_tempty[2], bar_lb[2], bar_cfull[2], bar_cempty[2];
  __shared__ int s_tk[2];        // ticket staged in s stage 0/1 (-1: no more tiles)
  __shared__ int s_atk;          // ticket whose operands sit in the A buffers (-1: stop)
  __shared__ int s_lbtk[2];      // ticket handed to the look-back warp per slot (-1: stop)
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ int s_last;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  Ctrl* ctrl = P.ctrl;
  const Args A = *P.args;
  const int D = P.D, T = P.T, B = P.B;
  const size_t stride = (size_t)B;   // one channel group: consecutive chunks are B tickets apart
  const long long tmo = A.timeout_ns;

  if (tid == 0) {
    atomicMin(&ctrl->t_start, globaltimer());
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_sfull[s], 1u);
      mbar_init(&bar_sempty[s], (unsigned)C::NEW);
      mbar_init(&bar_mma[s], 1u);
      mbar_init(&bar_tempty[s], (unsigned)C::NEW);
      mbar_init(&bar_lb[s], 1u);
      mbar_init(&bar_cfull[s], 1u);
      mbar_init(&bar_cempty[s], (unsigned)C::NEW);
    }
    mbar_init(&bar_xfull, 1u);
    mbar_init(&bar_xempty, (unsigned)C::NEW);
    mbar_init(&bar_afull, (unsigned)C::NEW);
    mbar_init_fence();
    s_abort = 0;
  }
  const unsigned epoch = *(volatile unsigned*)&ctrl->epoch;
  const int iter = *(volatile int*)&ctrl->iter;
  float* __restrict__ dst = (iter & 1) ? A.states : P.buf1;

  // weights: W and W_lo in the K-major core-matrix layout (pre-packed), diagonals, b_hn
  {
    const float4* w4 = reinterpret_cast<const float4*>(P.wt);
    float4* d4 = reinterpret_cast<float4*>(sBH);   // sBH and sBL are contiguous
    for (int e = tid; e < 2 * C::B_BYTES / 16; e += C::NT) d4[e] = __ldg(w4 + e);
    for (int e = tid; e < R * DP; e += C::NT) sWd[e] = __ldg(P.wdiag + e);
    for (int e = tid; e < DP; e += C::NT) sBhn[e] = (CELL == PN_CELL_GRU) ? __ldg(P.bhn + e) : 0.0f;
    fence_async_smem();   // the tensor cores read sBH/sBL through the async proxy
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&s_tmem)),
                 "r"((uint32_t)C::ALLOC_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  unsigned rbits = 0u;

  if (warp == 0) {
    // =========================== producer ===================================
    const CUtensorMap* tm_s = P.tmaps + ((iter & 1) ? 1 : 0);   // rows of s^(i)
    const CUtensorMap* tm_x = P.tmaps + 2;                      // step inputs
    if (lane == 0) {
      tmap_acquire(tm_s);
      tmap_acquire(tm_x);
    }
    int it = 0;
    int x_issued = 0;
    for (;; ++it) {
      const int st = it & 1;
      if (it >= 2 && !mbar_wait_flag(&bar_sempty[st], (((unsigned)it >> 1) & 1u) ^ 1u, ctrl, tmo, &s_abort)) break;
      int kg = 0;
      if (lane == 0) kg = (int)atomicAdd(&ctrl->ticket[0], 1u);
      kg = __shfl_sync(0xffffffffu, kg, 0);
      if (kg >= P.tiles_per_group) {
        if (lane == 0) {
          s_tk[st] = -1;
          mbar_arrive(&bar_sfull[st]);
        }
        ++it;
        break;
      }
      const int row0 = (kg % B) * T + (kg / B) * L;   // global row of step t0
      if (lane == 0) {
        // rows t0-1 .. t0+L-1; for the first chunk of a sequence row t0-1 is replaced by s0
        // when the stage is split, rows past the end are zero-filled or unused
        s_tk[st] = kg;
        mbar_arrive_expect_tx(&bar_sfull[st], (unsigned)C::S_BYTES);
        tma_load_2d(sS[st], tm_s, 0, row0 - 1, &bar_sfull[st]);
      }
      // the single step-input buffer: wait until the previous tile's inputs were consumed
      if (it >= 1 && !mbar_wait_flag(&bar_xempty, ((unsigned)(it - 1)) & 1u, ctrl, tmo, &s_abort)) {
        ++it;
        break;
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar_xfull, (unsigned)C::X_BYTES);
        tma_load_2d(sX, tm_x, 0, row0, &bar_xfull);
      }
      __syncwarp();
      x_issued = it + 1;
    }
    // drain every fill this warp issued
    for (int j = max(0, it - 2); j < it; ++j)
      if (!mbar_drain(&bar_sfull[j & 1], ((unsigned)j >> 1) & 1u, tmo) && lane == 0)
        atomicCAS(&ctrl->error, 0, (int)PN_ERR_TIMEOUT);
    if (x_issued > 0 && !mbar_drain(&bar_xfull, ((unsigned)(x_issued - 1)) & 1u, tmo) && lane == 0)
      atomicCAS(&ctrl->error, 0, (int)PN_ERR_TIMEOUT);
  } else if (warp == 1) {
    // =========================== MMA issuer =================================
    constexpr uint32_t idesc = umma_idesc_tf32(L, N);
    int issued = 0;
    for (int it = 0;; ++it) {
      if (!mbar_wait_flag(&bar_afull, (unsigned)it & 1u, ctrl, tmo, &s_abort)) break;
      if (s_atk < 0) break;
      const int buf = it & 1;
      if (it >= 2 && !mbar_wait_flag(&bar_tempty[buf], (((unsigned)it >> 1) & 1u) ^ 1u, ctrl, tmo, &s_abort)) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t d = tmem + (uint32_t)(buf * C::TCOLS);
        const uint32_t ah = smem_addr(sAH), al = smem_addr(sAL), bh = smem_addr(sBH), bl = smem_addr(sBL);
#pragma unroll 1
        for (int pass = 0; pass < 3; ++pass) {
          const uint32_t a = (pass == 2) ? al : ah;
          const uint32_t bb = (pass == 1) ? bl : bh;
#pragma unroll
          for (int kb = 0; kb < K / 8; ++kb)
            umma_tf32(d, umma_smem_desc(a + kb * 256, 128, C::SBO_A), umma_smem_desc(bb + kb * 256, 128, C::SBO_B),
                      idesc, (pass > 0 || kb > 0) ? 1u : 0u);
        }
        umma_commit(&bar_mma[buf]);
      }
      __syncwarp();
      issued = it + 1;
    }
    // every issued product must have completed before TMEM is released
    for (int j = max(0, issued - 2); j < issued; ++j)
      if (!mbar_drain(&bar_mma[j & 1], ((unsigned)j >> 1) & 1u, tmo) && lane == 0)
        atomicCAS(&ctrl->error, 0, (int)PN_ERR_TIMEOUT);
  } else if (warp == 2) {
    // =========================== look-back ==================================
    if constexpr (kScan) {
      for (int it = 0;; ++it) {
        const int slot = it & 1;
        if (!mbar_wait_flag(&bar_lb[slot], ((unsigned)it >> 1) & 1u, ctrl, tmo, &s_abort)) break;
        const int kg = s_lbtk[slot];
        if (kg < 0) break;
        if (it >= 2 && !mbar_wait_flag(&bar_cempty[slot], (((unsigned)it >> 1) & 1u) ^ 1u, ctrl, tmo, &s_abort)) break;
        const int b = kg % B;
        const int chunk = kg / B;
        const size_t k = (size_t)kg;
        const bool stall = (A.stall_ticket == kg);
        const float* agg = sAgg + slot * DP * 2;
        const int n_agg = lookback_find_prefix(P.flags, k, stride, chunk, epoch, ctrl, tmo);
        __syncwarp();
        float carry[C::NQ];
#pragma unroll
        for (int q = 0; q < C::NQ; ++q) {
          const int j = lane + 32 * q;
          float v = 0.0f;
          if (n_agg >= 0 && j < DP) {
            if (chunk - 1 - n_agg >= 0) v = __ldcg(P.pref + (k - (size_t)(n_agg + 1) * stride) * P.pref_stride + j);
            else v = (j < D) ? __ldg(A.s0 + (size_t)b * D + j) : 0.0f;
#pragma unroll 4
            for (int d = n_agg; d >= 1; --d) {
              const float2 ab =
                  __ldcg(reinterpret_cast<const float2*>(P.agg + (k - (size_t)d * stride) * P.agg_stride) + j);
              v = fmaf(ab.x, v, ab.y);
            }
          }
          carry[q] = v;
        }
        if (n_agg >= 0 && !stall) {
#pragma unroll
          for (int q = 0; q < C::NQ; ++q) {
            const int j = lane + 32 * q;
            if (j < DP) P.pref[k * P.pref_stride + j] = fmaf(agg[2 * j], carry[q], agg[2 * j + 1]);
          }
          // the warp barrier orders the other lanes' stores before lane 0's release,
          // which is cumulative: a reader that acquires the flag sees all of them
          __syncwarp();
          if (lane == 0) st_release(P.flags + k, make_flag(epoch, kFlagPrefix));
        }
        if (n_agg < 0) s_abort = 1;
#pragma unroll
        for (int q = 0; q < C::NQ; ++q) {
          const int j = lane + 32 * q;
          if (j < DP) sCarry[slot * DP + j] = carry[q];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_cfull[slot]);
      }
    }
  } else {
    // =========================== epilogue ===================================
    const int e = warp - 3;                 // 0 .. NEW-1
    const int quarter = warp & 3;           // TMEM lane quarter this warp may access
    const int cg = e >> 2;                  // channel group
    const int row = quarter * 32 + lane;    // step row within the tile
    const int cbase = cg * CH;              // first channel of this thread
    const int te = tid - 96;                // 0 .. NTE-1 among the epilogue threads
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;

    // Operand split of stage S: tf32(S) and tf32(S - tf32(S)) in the K-major
    // core-matrix layout.  For the first chunk of a sequence the stage's row 0
    // (time -1) is s0, written into the stage here as well for the cell phase.
    auto split = [&](float* S, int kgs) {
      const bool first = (kgs / B) == 0;
      const float* s0row = A.s0 + (size_t)(kgs % B) * D;
      for (int c = te; c < L * (K / 4); c += NTE) {
        const int r = (c & 7) + 8 * ((c >> 3) / (K / 4));
        const int kq = (c >> 3) % (K / 4);
        float4 v;
        if (first && r == 0) {
          v = __ldg(reinterpret_cast<const float4*>(s0row) + kq);
          *reinterpret_cast<float4*>(S + kq * 4) = v;
        } else {
          v = *reinterpret_cast<const float4*>(S + r * SP + kq * 4);
        }
        const float4 hi = make_float4(tf32_round(v.x), tf32_round(v.y), tf32_round(v.z), tf32_round(v.w));
        const float4 lo = make_float4(tf32_round(v.x - hi.x), tf32_round(v.y - hi.y), tf32_round(v.z - hi.z),
                                      tf32_round(v.w - hi.w));
        const uint32_t off = kmajor_offset(r, kq * 4, K);
        *reinterpret_cast<float4*>(sAH + off) = hi;
        *reinterpret_cast<float4*>(sAL + off) = lo;
      }
      fence_async_smem();   // generic writes -> async proxy (tensor cores, next TMA fill)
    };

    // s^(i+1) of tile j from its parked prefixes and the carry of the look-back warp
    auto write_out = [&](int j, int kgj) {
      const int slot = j & 1;
      mbar_wait_flag(&bar_cfull[slot], ((unsigned)j >> 1) & 1u, ctrl, tmo, &s_abort);
      const float* cr = sCarry + slot * DP + cbase;
      const int bj = kgj % B;
      const int tj = (kgj / B) * L + row;
      const bool okj = (tj < T) && !s_abort;
      const uint32_t sbase = tmem + (uint32_t)(C::STASH0 + slot * C::SCOLS) + lane_off;
      float bb[16], aa[16];
      tmem_ld16(sbase + (uint32_t)((kHasA ? DP : 0) + cbase), bb);
      if constexpr (kHasA) tmem_ld16(sbase + (uint32_t)cbase, aa);
      if (okj) {
        float* o = dst + ((size_t)bj * T + tj) * D + cbase;
#pragma unroll
        for (int c4 = 0; c4 < CH; c4 += 4) {
          const float4 c = *reinterpret_cast<const float4*>(cr + c4);
          float4 v;
          if constexpr (kHasA) {
            v = make_float4(fmaf(aa[c4], c.x, bb[c4]), fmaf(aa[c4 + 1], c.y, bb[c4 + 1]),
                            fmaf(aa[c4 + 2], c.z, bb[c4 + 2]), fmaf(aa[c4 + 3], c.w, bb[c4 + 3]));
          } else {
            v = make_float4(c.x + bb[c4], c.y + bb[c4 + 1], c.z + bb[c4 + 2], c.w + bb[c4 + 3]);
          }
          *reinterpret_cast<float4*>(o + c4) = v;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_cempty[slot]);
    };

    // prologue: operands of the first tile
    {
      int kg0 = -1;
      if (mbar_wait_flag(&bar_sfull[0], 0u, ctrl, tmo, &s_abort)) kg0 = s_tk[0];
      if (kg0 >= 0) split(sS[0], kg0);
      __syncwarp();
      named_barrier(1, NTE);
      if (lane == 0) {
        if (te == 0) s_atk = s_abort ? -1 : kg0;
        mbar_arrive(&bar_afull);
      }
    }
    named_barrier(1, NTE);
    int kg = s_atk;   // written by te == 0 before the barrier
    int it = 0;
    int prev_kg = -1;
    for (; kg >= 0; ++it) {
      const int st = it & 1;
      const int buf = it & 1;
      const int b = kg % B;
      const int chunk = kg / B;
      const int t = chunk * L + row;
      const float* S = sS[st];

      // ---- Z from TMEM, then the cell --------------------------------------
      mbar_wait_flag(&bar_mma[buf], ((unsigned)it >> 1) & 1u, ctrl, tmo, &s_abort);
      tc_fence_after();
      float z[R][CH];
#pragma unroll
      for (int q = 0; q < R; ++q) tmem_ld16(tmem + (uint32_t)(buf * C::TCOLS) + lane_off + (uint32_t)(q * DP + cbase), z[q]);
      mbar_wait_flag(&bar_xfull, (unsigned)it & 1u, ctrl, tmo, &s_abort);
      const bool tok = (t < T);
      float av[CH], bv[CH];
#pragma unroll
      for (int c4 = 0; c4 < CH; c4 += 4) {
        const int c = cbase + c4;
        const float4 sp4 = *reinterpret_cast<const float4*>(S + row * SP + c);
        const float4 sc4 = *reinterpret_cast<const float4*>(S + (row + 1) * SP + c);
        float4 x4[R];
#pragma unroll
        for (int q = 0; q < R; ++q) x4[q] = *reinterpret_cast<const float4*>(sX + row * XP + q * DP + c);
        const float spv[4] = {sp4.x, sp4.y, sp4.z, sp4.w};
        const float scv[4] = {sc4.x, sc4.y, sc4.z, sc4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int cc = c + u;
          float xv[R];
#pragma unroll
          for (int q = 0; q < R; ++q) xv[q] = (u == 0) ? x4[q].x : (u == 1) ? x4[q].y : (u == 2) ? x4[q].z : x4[q].w;
          const float sp = spv[u], sc = scv[u];
          float y, a, bb, res;
          if constexpr (CELL == PN_CELL_TANH_RNN) {
            y = tanh_pn(z[0][c4 + u] + xv[0]);
            res = sc - y;
            a = (MODE == PN_QUASI) ? (1.0f - y * y) * sWd[cc] : (MODE == PN_PICARD ? 1.0f : 0.0f);
            bb = (MODE == PN_JACOBI) ? y : y - a * sp;
          } else if constexpr (CELL == PN_CELL_EULER_TANH) {
            const float gg = tanh_pn(z[0][c4 + u] + xv[0]);
            const float eg = P.eps * gg;
            y = sp + eg;
            res = (sc - sp) - eg;
            if (MODE == PN_QUASI) {
              const float ed = P.eps * (1.0f - gg * gg) * sWd[cc];
              a = 1.0f + ed;
              bb = eg - ed * sp;
            } else if (MODE == PN_PICARD) {
              a = 1.0f;
              bb = eg;
            } else {
              a = 0.0f;
              bb = y;
            }
          } else {
            const float rr = sigmoidf_acc(xv[0] + z[0][c4 + u]);
            const float zz = sigmoidf_acc(xv[1] + z[1][c4 + u]);
            const float hn = z[2][c4 + u] + sBhn[cc];
            const float nn = tanh_pn(xv[2] + rr * hn);
            y = nn + zz * (sp - nn);
            res = sc - y;
            if (MODE == PN_QUASI) {
              const float omz = 1.0f - zz;
              const float dn = omz * (1.0f - nn * nn);
              a = zz + (sp - nn) * zz * omz * sWd[DP + cc] +
                  dn * (rr * sWd[2 * DP + cc] + hn * rr * (1.0f - rr) * sWd[cc]);
            } else {
              a = (MODE == PN_PICARD) ? 1.0f : 0.0f;
            }
            bb = (MODE == PN_JACOBI) ? y : y - a * sp;
          }
          if (tok) {
            rbits = max(rbits, abs_bits(res));
            av[c4 + u] = a;
            bv[c4 + u] = bb;
          } else {
            av[c4 + u] = 1.0f;
            bv[c4 + u] = 0.0f;
          }
        }
      }
      // this tile's TMEM accumulator, step inputs and s stage are consumed
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar_tempty[buf]);
        mbar_arrive(&bar_xempty);
        mbar_arrive(&bar_sempty[st]);
      }

      // ---- operands of the next tile (the tensor cores work while we scan) --
      {
        int kn = -1;
        if (mbar_wait_flag(&bar_sfull[st ^ 1], (((unsigned)it + 1u) >> 1) & 1u, ctrl, tmo, &s_abort)) kn = s_tk[st ^ 1];
        if (kn >= 0 && !s_abort) split(sS[st ^ 1], kn);
        __syncwarp();
        named_barrier(1, NTE);   // every epilogue thread has written its part of the split
        if (lane == 0) {
          if (te == 0) s_atk = s_abort ? -1 : kn;   // also the loop's exit decision, read after the last barrier
          mbar_arrive(&bar_afull);
        }
      }
      // the previous tile's carry had this tile's cell phase to arrive: write it out now
      if constexpr (kScan) {
        if (it > 0) write_out(it - 1, prev_kg);
      }

      if constexpr (!kScan) {
        if (tok && !s_abort) {
          float* o = dst + ((size_t)b * T + t) * D + cbase;
#pragma unroll
          for (int c4 = 0; c4 < CH; c4 += 4)
            *reinterpret_cast<float4*>(o + c4) = make_float4(bv[c4], bv[c4 + 1], bv[c4 + 2], bv[c4 + 3]);
        }
      } else {
        // ---- scan along the rows: within the warp (a level at a time over all 16
        //      channels, so the shuffles of one level are independent), then across quarters
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
#pragma unroll
          for (int c = 0; c < CH; ++c) {
            const float ub = __shfl_up_sync(0xffffffffu, bv[c], off);
            if constexpr (kHasA) {
              const float ua = __shfl_up_sync(0xffffffffu, av[c], off);
              if (lane >= off) {
                bv[c] = fmaf(av[c], ub, bv[c]);
                av[c] *= ua;
              }
            } else {
              if (lane >= off) bv[c] += ub;
            }
          }
        }
        if (lane == 31) {
#pragma unroll
          for (int c = 0; c < CH; c += 2)
            *reinterpret_cast<float4*>(sTot + ((cg * 4 + quarter) * CH + c) * 2) =
                make_float4(kHasA ? av[c] : 1.0f, bv[c], kHasA ? av[c + 1] : 1.0f, bv[c + 1]);
        }
        named_barrier(1, NTE);
        if (quarter > 0) {
          // prefix of the earlier quarters: tot_{quarter-1} o ... o tot_0
          float PA[CH], PB[CH];
#pragma unroll
          for (int c = 0; c < CH; ++c) {
            PA[c] = 1.0f;
            PB[c] = 0.0f;
          }
          for (int qq = 0; qq < quarter; ++qq) {
            const float* tq = sTot + (cg * 4 + qq) * CH * 2;
#pragma unroll
            for (int c = 0; c < CH; c += 2) {
              const float4 w = *reinterpret_cast<const float4*>(tq + c * 2);
              PB[c] = fmaf(w.x, PB[c], w.y);
              PA[c] *= w.x;
              PB[c + 1] = fmaf(w.z, PB[c + 1], w.w);
              PA[c + 1] *= w.z;
            }
          }
#pragma unroll
          for (int c = 0; c < CH; ++c) {
            bv[c] = kHasA ? fmaf(av[c], PB[c], bv[c]) : bv[c] + PB[c];
            if (kHasA) av[c] *= PA[c];
          }
        }
        // the last row holds the tile aggregate
        const int slot = it & 1;
        if (quarter == 3 && lane == 31) {
#pragma unroll
          for (int c = 0; c < CH; c += 2)
            *reinterpret_cast<float4*>(sAgg + (slot * DP + cbase + c) * 2) =
                make_float4(kHasA ? av[c] : 1.0f, bv[c], kHasA ? av[c + 1] : 1.0f, bv[c + 1]);
        }
        named_barrier(1, NTE);
        if (e == 0) {   // publish the aggregate, then wake the look-back warp
          const bool stall = (A.stall_ticket == kg);
          const int ab = __shfl_sync(0xffffffffu, (int)s_abort, 0);   // one value for the whole warp
          if (chunk > 0 && !stall && !ab) {
#pragma unroll
            for (int q = 0; q < C::NQ; ++q) {
              const int j = lane + 32 * q;
              if (j < DP)
                reinterpret_cast<float2*>(P.agg + (size_t)kg * P.agg_stride)[j] =
                    *reinterpret_cast<const float2*>(sAgg + (slot * DP + j) * 2);
            }
            __syncwarp();   // lane 0's release is cumulative over the lanes' stores ordered before it
            if (lane == 0) st_release(P.flags + kg, make_flag(epoch, kFlagAgg));
          }
          __syncwarp();
          if (lane == 0) {
            s_lbtk[slot] = ab ? -1 : kg;
            mbar_arrive(&bar_lb[slot]);
          }
        }
        // ---- park this tile's in-tile prefixes in TMEM; written out next tile
        {
          const uint32_t sbase = tmem + (uint32_t)(C::STASH0 + slot * C::SCOLS) + lane_off;
          if constexpr (kHasA) tmem_st16(sbase + (uint32_t)cbase, av);
          tmem_st16(sbase + (uint32_t)((kHasA ? DP : 0) + cbase), bv);
          tmem_st_wait();
        }
        prev_kg = kg;
      }
      named_barrier(1, NTE);   // uniform exit decision (s_atk was set by te == 0 above)
      kg = s_atk;
    }
    if constexpr (kScan) {
      if (it > 0) write_out(it - 1, prev_kg);
      // stop the look-back warp: its next slot is the `it`-th
      if (e == 0 && lane == 0) {
        s_lbtk[it & 1] = -1;
        mbar_arrive(&bar_lb[it & 1]);
      }
    }
  }

  // ---- residual, TMEM release, end-of-launch decision ------------------------
  rbits = warp_max_u32(rbits);
  if (lane == 0) sRed[warp] = __uint_as_float(rbits);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)C::ALLOC_COLS)
                 : "memory");
  if (tid == 0) {
    unsigned v = 0u;
    for (int w = 0; w < C::NT / 32; ++w) v = max(v, __float_as_uint(sRed[w]));
    if (v) atomicMax(&ctrl->resid_bits, v);
  }
  finish_launch(P, A, epoch, s_last);
}

}  // namespace pn
