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
//     Z = S_hi W_hi + S_hi W_lo + S_lo W_hi,
// where the tensor core reads S as S_hi (it ignores the low 13 mantissa bits
// of an fp32 operand), S_lo = S - S_hi is formed in shared memory, and W_hi,
// W_lo come pre-split from the host.  The dropped S_lo W_lo term and the
// truncation of S_lo are below 2^-20 relative, about fp32 level.
//
// Data movement (all TMA, never multicast):
//   s^(i) rows t0-1 .. t0+L-1 of one sequence arrive in the tensor cores'
//   128-byte-swizzled K-major layout, one 32-float column half per load; the
//   epilogue reads them there directly (the swizzle keeps column reads
//   conflict-free).  Step t0-1 < 0 reads as zero and is replaced by s0.
//   Step inputs arrive as rows padded by 4 floats (box wider than the array).
//   New states leave through a padded-row staging buffer and one TMA tensor
//   store per tile; steps >= T are clipped by the store itself.
//
// Warp roles (one CTA per SM):
//   warp 0      producer: claims tiles (ticket order), issues the loads;
//   warp 1      MMA and store issuer: one thread issues the 3 x D/8
//               tcgen05.mma of a tile into one of two TMEM accumulators,
//               commits to an mbarrier, then issues the TMA store of the
//               newest finished output tile while the tensor cores work;
//   warps 2-3   look-back (scan modes), alternate tiles: publish the tile
//               aggregate, find the nearest predecessor with a published
//               state, fold the aggregates in between, hand the carry to the
//               epilogue, then publish the tile's end state;
//   the rest    epilogue, four row quarters x D/16 channel groups: one thread
//               per step row (TMEM lane) and 16 channels.  Reads Z from TMEM,
//               evaluates the cell, the diagonal Jacobian and |F|, forms the
//               next tile's S_lo, scans along the rows (warp shuffles a level
//               at a time over all 16 channels, then across the row quarters)
//               and parks the in-tile prefixes in TMEM.  A tile's states are
//               formed two tiles later, so the look-back has two tiles of time
//               to deliver its carry.
#pragma once

#include <string.h>

#include "pn_cells.cuh"
#include "pn_tma.cuh"

namespace pn {

// --- tcgen05 / TMA helpers (inline PTX) ------------------------------------

// Canonical K-major layout without swizzle ("interleaved" core matrices):
// a core matrix is 8 rows x 16 bytes stored contiguously; core matrices
// adjacent along K are 128 bytes apart (leading byte offset) and groups of 8
// rows are K/4 * 128 bytes apart (stride byte offset).  Used for W.
__host__ __device__ __forceinline__ uint32_t kmajor_offset(int row, int k, int K) {
  return (uint32_t)((row >> 3) * (K / 4) * 128 + (k >> 2) * 128 + (row & 7) * 16 + (k & 3) * 4);
}

// 128-byte-swizzled K-major layout of a 32-float column half (base 1024-byte
// aligned): row r occupies bytes [128 r, 128 r + 128) and its 16-byte chunk j
// sits at chunk position j ^ (r mod 8).  This is the layout a TMA load with
// 128-byte swizzle writes.  Used for S and S_lo.
__device__ __forceinline__ uint32_t sw128_offset(int r, int c) {
  return (uint32_t)(r * 128 + ((((c >> 2) ^ r) & 7) << 4) + (c & 3) * 4);
}

// Shared-memory matrix descriptor (sm_100): start address >> 4 in bits 0-13,
// leading byte offset >> 4 in bits 16-29, stride byte offset >> 4 in bits
// 32-45, version 1 in bits 46-47, layout in bits 61-63 (0: no swizzle,
// 2: 128-byte swizzle).
__device__ __forceinline__ uint64_t umma_smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46) | ((uint64_t)layout << 61);
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

// The tcgen05 instructions below are warp-aligned (.sync.aligned): every thread of the warp must
// execute them together, which inline asm does not tell the compiler, so each helper reconverges
// the warp first (the code before it may have diverged, e.g. in a spin-wait).
// Allocate `cols` TMEM columns for the CTA (one warp calls it; the base address lands in *dst).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t cols) {
  __syncwarp();
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst)), "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
  __syncwarp();
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}

// 16 consecutive fp32 columns of this warp's 32 TMEM lanes: thread i gets lane i.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  __syncwarp();
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
  __syncwarp();
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  __syncwarp();
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 32 consecutive fp32 columns of this warp's 32 TMEM lanes in one load (thread i gets lane i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  __syncwarp();
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}

// Store 32 fp32 columns into this warp's 32 TMEM lanes (thread i -> lane i): a[16] then b[16].
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&a)[16], const float (&b)[16]) {
  __syncwarp();
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(a[0])), "r"(__float_as_uint(a[1])), "r"(__float_as_uint(a[2])), "r"(__float_as_uint(a[3])),
      "r"(__float_as_uint(a[4])), "r"(__float_as_uint(a[5])), "r"(__float_as_uint(a[6])), "r"(__float_as_uint(a[7])),
      "r"(__float_as_uint(a[8])), "r"(__float_as_uint(a[9])), "r"(__float_as_uint(a[10])), "r"(__float_as_uint(a[11])),
      "r"(__float_as_uint(a[12])), "r"(__float_as_uint(a[13])), "r"(__float_as_uint(a[14])), "r"(__float_as_uint(a[15])),
      "r"(__float_as_uint(b[0])), "r"(__float_as_uint(b[1])), "r"(__float_as_uint(b[2])), "r"(__float_as_uint(b[3])),
      "r"(__float_as_uint(b[4])), "r"(__float_as_uint(b[5])), "r"(__float_as_uint(b[6])), "r"(__float_as_uint(b[7])),
      "r"(__float_as_uint(b[8])), "r"(__float_as_uint(b[9])), "r"(__float_as_uint(b[10])), "r"(__float_as_uint(b[11])),
      "r"(__float_as_uint(b[12])), "r"(__float_as_uint(b[13])), "r"(__float_as_uint(b[14])), "r"(__float_as_uint(b[15]))
      : "memory");
}

// The tensor map was written to global memory by a host copy before this
// launch: order that write before the tensor-map proxy reads it.
__device__ __forceinline__ void tmap_acquire(const CUtensorMap* map) {
  asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(map) : "memory");
}

// 3-D TMA tensor load of one box at element coordinates (column c0, step c1,
// sequence c2) into this CTA's shared memory, counted on `bar`.  c0 is a
// multiple of 32 (16-byte aligned); c1 may be -1 (that row reads as zero).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          smem_addr(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
      : "memory");
}

// L2 cache policies for the bulk tensor copies: data read every iteration (the
// step inputs) is kept in L2 ahead of data streamed once per iteration.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// tma_load_3d with an L2 cache policy (from createpolicy).
__device__ __forceinline__ void tma_load_3d_hint(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                                 uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_addr(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// 3-D TMA tensor store of one box from shared memory (coordinates >= 0);
// elements outside the array are not written.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, int c0, int c1, int c2, const void* src) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(map), "r"(c0),
               "r"(c1), "r"(c2), "r"(smem_addr(src))
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// this thread's committed bulk stores have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// ... and have completed their global writes
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Round to the nearest TF32 value (10 explicit mantissa bits), for the host
// split of W: W_hi = tf32(W), W_lo = tf32(W - W_hi).
__host__ __device__ __forceinline__ float tf32_round(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  if ((u & 0x7F800000u) != 0x7F800000u) u = (u + 0x1000u) & 0xFFFFE000u;
  float r;
  memcpy(&r, &u, 4);
  return r;
}

// The part of x below its TF32 truncation (exact in fp32).
__device__ __forceinline__ float tf32_tail(float x) { return x - __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }

// Bounded mbarrier wait that never leaves the caller's control flow: on
// timeout / error it records the failure in *abort and returns false.
// `site` (> 0) names the wait in the control block's timeout_ticket word (as -site) when it is
// the one that gives up, so a timeout report says which wait of which role ran out.
__device__ __forceinline__ bool mbar_wait_flag(uint64_t* bar, unsigned parity, Ctrl* ctrl, long long timeout_ns,
                                               volatile int* abort, int site = 0) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  unsigned spins = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    ++spins;
    // the CTA's own abort flag (shared memory) often; the grid's error word and the clock
    // rarely: thousands of waiting warps polling one global word make its L2 slice a hot spot
    if ((spins & 15u) == 0u && *abort) return false;
    if ((spins & 255u) == 0u) {
      if (ld_volatile(&ctrl->error)) {
        *abort = 1;
        return false;
      }
      if ((long long)(globaltimer() - t0) > timeout_ns) {
        if (raise_error(ctrl, (int)PN_ERR_TIMEOUT) && site > 0) ctrl->timeout_ticket = -site;
        *abort = 1;
        return false;
      }
    }
  }
}

// Launch tag of the self-validating look-back words: never 0, so memory that
// was only cleared never validates.
__device__ __forceinline__ unsigned lookback_tag(unsigned epoch) { return 0x80000000u | epoch; }

// Gives up a warp-wide spin: true (for all lanes) when another CTA reported an
// error or this wait ran past timeout_ns (then it reports PN_ERR_TIMEOUT).
__device__ __forceinline__ bool spin_give_up(unsigned& spins, unsigned long long t0, Ctrl* ctrl, long long timeout_ns) {
  int g = 0;
  if ((++spins & 15u) == 0u && (threadIdx.x & 31) == 0) {
    if (ld_volatile(&ctrl->error)) g = 1;
    else if ((long long)(globaltimer() - t0) > timeout_ns) {
      raise_error(ctrl, (int)PN_ERR_TIMEOUT);
      g = 1;
    }
  }
  return __shfl_sync(0xffffffffu, g, 0) != 0;
}

// A published state: the DP words of one tile, lane j holding channels
// j + 32 q.  Spins (bounded) until every word carries `tag`.
template <int DP, int NQ>
__device__ __forceinline__ bool ld_tagged_state(const unsigned long long* src, unsigned tag, float (&v)[NQ], Ctrl* ctrl,
                                                long long timeout_ns) {
  const int lane = threadIdx.x & 31;
  unsigned long long w[NQ];
  unsigned long long t0 = 0;
  unsigned spins = 0;
  while (true) {
    bool ok = true;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const int j = lane + 32 * q;
      w[q] = (j < DP) ? ld_word(src + j) : tag_word(0.0f, tag);
      ok = ok && word_tagged(w[q], tag);
    }
    if (__all_sync(0xffffffffu, ok)) break;
    if (spins == 0) t0 = globaltimer();
    if (spin_give_up(spins, t0, ctrl, timeout_ns)) return false;
  }
#pragma unroll
  for (int q = 0; q < NQ; ++q) v[q] = word_value(w[q]);
  return true;
}

// Aggregates of the tiles d0, d0-1, .., d0-3 places back (k - d * stride,
// those with d >= 1), loaded together; spins (bounded) until all validate.
template <int DP, int NQ>
__device__ __forceinline__ bool ld_tagged_aggs(const unsigned long long* aggw, size_t k, size_t stride, int d0,
                                               unsigned tag, float (&fa)[4][NQ], float (&fb)[4][NQ], Ctrl* ctrl,
                                               long long timeout_ns) {
  const int lane = threadIdx.x & 31;
  unsigned long long t0 = 0;
  unsigned spins = 0;
  while (true) {
    bool ok = true;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int d = d0 - u;
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const int j = lane + 32 * q;
        unsigned long long wa = tag_word(1.0f, tag), wb = tag_word(0.0f, tag);
        if (d >= 1 && j < DP) ld_word2(aggw + ((k - (size_t)d * stride) * DP + j) * 2, wa, wb);
        ok = ok && word_tagged(wa, tag) && word_tagged(wb, tag);
        fa[u][q] = word_value(wa);
        fb[u][q] = word_value(wb);
      }
    }
    if (__all_sync(0xffffffffu, ok)) return true;
    if (spins == 0) t0 = globaltimer();
    if (spin_give_up(spins, t0, ctrl, timeout_ns)) return false;
  }
}

template <int CELL, int MODE, int DP>
struct DiagTcCfg {
  static constexpr int R = CellInfo<CELL>::R;
  static constexpr bool kScan = (MODE != PN_JACOBI);
  static constexpr int L = 128;                 // steps per tile = MMA M
  static constexpr int K = DP;                  // MMA K (input channels)
  static constexpr int N = R * DP;              // MMA N (output rows of W)
  static constexpr int NKH = DP / 32;           // 32-float column halves of S (one swizzle atom wide)
  static constexpr int TCOLS = N <= 64 ? 64 : (N <= 128 ? 128 : 256);   // TMEM columns per accumulator
  static constexpr int SCOLS = (MODE == PN_QUASI ? 2 : 1) * DP;        // stash columns per tile: [A |] B
  static constexpr int NSLOT = 3;               // tiles between their scan and their write-out, + 1
  static constexpr int DEFER = NSLOT - 1;       // a tile's states are formed DEFER tiles later
  static constexpr int NLB = kScan ? 2 : 0;     // look-back warps, alternating tiles
  static constexpr int STASH0 = 2 * TCOLS;      // first stash column
  static constexpr int USED_COLS = STASH0 + (kScan ? NSLOT * SCOLS : 0);
  static constexpr int ALLOC_COLS = USED_COLS <= 128 ? 128 : (USED_COLS <= 256 ? 256 : 512);
  static constexpr int CH = 16;                 // channels per epilogue thread
  static constexpr int NCG = DP / CH;           // channel groups
  static constexpr int NEW = 4 * NCG;           // epilogue warps: 4 row quarters x channel groups
  static constexpr int NTE = 32 * NEW;          // epilogue threads
  static constexpr int WE0 = 2 + NLB;           // first epilogue warp
  static constexpr int OUT_LAG = kScan ? DEFER : 0;   // output tile j is staged in epilogue tile j + OUT_LAG
  static constexpr int NT = 32 * (WE0 + NEW);
  static constexpr int SP = DP + 4;             // padded output row (floats) = store box width
  static constexpr int XP = R * DP + 4;         // padded step-input row (floats) = load box width
  static constexpr int NQ = (DP + 31) / 32;
  static constexpr int align(int v, int a) { return (v + a - 1) / a * a; }
  static constexpr int SH_LOAD = (L + 1) * 128;                  // bytes of one S column-half load
  static constexpr int SH_BYTES = align(SH_LOAD, 1024);          // S column-half buffer
  static constexpr int LO_BYTES = L * 128;                       // S_lo column-half buffer
  static constexpr int X_BYTES = L * XP * 4;
  static constexpr int O_BYTES = L * SP * 4;
  static constexpr int B_BYTES = N * K * 4;
  static constexpr int TOT_FLOATS = NCG * 4 * CH * 2;            // one buffer of quarter totals
  static constexpr int OFF_S = 0;                                // [2 stages][NKH][SH_BYTES]
  static constexpr int OFF_LO = OFF_S + 2 * NKH * SH_BYTES;      // [NKH][LO_BYTES]
  static constexpr int OFF_X = OFF_LO + NKH * LO_BYTES;
  static constexpr int OFF_O = align(OFF_X + X_BYTES, 128);
  static constexpr int OFF_BH = align(OFF_O + O_BYTES, 128);
  static constexpr int OFF_BL = OFF_BH + B_BYTES;
  static constexpr int OFF_WD = OFF_BL + B_BYTES;                // R*DP floats: diagonals of W_q
  static constexpr int OFF_BHN = OFF_WD + R * DP * 4;            // DP floats
  static constexpr int OFF_TOT = OFF_BHN + DP * 4;               // [2][NCG][4 quarters][CH][2]
  static constexpr int OFF_AGG = OFF_TOT + 2 * TOT_FLOATS * 4;   // [NSLOT][DP][2]
  static constexpr int OFF_CARRY = OFF_AGG + NSLOT * DP * 2 * 4; // [NSLOT][DP]
  static constexpr int OFF_RED = OFF_CARRY + NSLOT * DP * 4;     // NT/32 floats
  static constexpr int SMEM_USED = OFF_RED + (NT / 32) * 4;
  static constexpr int SMEM_BYTES = SMEM_USED + 1024;            // + slack to align the base to 1024 bytes
  static_assert(DP == 32 || DP == 64, "tensor-core path covers D = 32 and D = 64");
  static_assert(USED_COLS <= 512, "TMEM columns");
  static_assert(SP <= 256 && XP <= 256 && L + 1 <= 256, "TMA box extents");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(DEFER == 2, "the epilogue keeps the tickets of the last two tiles");
};

template <int CELL, int MODE, int DP>
__global__ void __launch_bounds__(DiagTcCfg<CELL, MODE, DP>::NT, 1) diag_tc_kernel(const IterParams P) {
  using C = DiagTcCfg<CELL, MODE, DP>;
  constexpr int R = C::R;
  constexpr int L = C::L;
  constexpr int K = C::K;
  constexpr int N = C::N;
  constexpr int NKH = C::NKH;
  constexpr int SP = C::SP;
  constexpr int XP = C::XP;
  constexpr int CH = C::CH;
  constexpr int NTE = C::NTE;
  constexpr int NSLOT = C::NSLOT;
  constexpr bool kScan = C::kScan;
  constexpr bool kHasA = (MODE == PN_QUASI);

  extern __shared__ __align__(1024) unsigned char smem_tc[];
  // 128-byte swizzled TMA destinations want 1024-byte alignment: round the base up (the launch adds 1 KB)
  unsigned char* smem_raw = smem_tc + ((1024u - (smem_addr(smem_tc) & 1023u)) & 1023u);
  unsigned char* sS = smem_raw + C::OFF_S;       // stage st, half h at sS + (st * NKH + h) * SH_BYTES
  unsigned char* sLo = smem_raw + C::OFF_LO;     // half h at sLo + h * LO_BYTES
  float* sX = reinterpret_cast<float*>(smem_raw + C::OFF_X);
  float* sO = reinterpret_cast<float*>(smem_raw + C::OFF_O);
  unsigned char* sBH = smem_raw + C::OFF_BH;
  unsigned char* sBL = smem_raw + C::OFF_BL;
  float* sWd = reinterpret_cast<float*>(smem_raw + C::OFF_WD);
  float* sBhn = reinterpret_cast<float*>(smem_raw + C::OFF_BHN);
  float* sTot = reinterpret_cast<float*>(smem_raw + C::OFF_TOT);
  float* sAgg = reinterpret_cast<float*>(smem_raw + C::OFF_AGG);
  float* sCarry = reinterpret_cast<float*>(smem_raw + C::OFF_CARRY);
  float* sRed = reinterpret_cast<float*>(smem_raw + C::OFF_RED);

  __shared__ __align__(8) uint64_t bar_sfull[2], bar_sempty[2], bar_xfull, bar_xempty, bar_afull, bar_mma[2],
      bar_tempty[2], bar_ofull, bar_oempty, bar_lb[NSLOT], bar_cfull[NSLOT], bar_cempty[NSLOT];
  __shared__ int s_tk[2];        // ticket staged in s stage 0/1 (-1: no more tiles)
  __shared__ int s_atk[2];       // ticket of tile i's operands, by the parity of i (-1: stop)
  __shared__ int s_otk[2];       // ticket of output tile j, by the parity of j (-1: stop, -2: skip)
  __shared__ int s_lbtk[NSLOT];  // ticket handed to the look-back per slot (-1: stop)
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ int s_last;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  Ctrl* ctrl = P.ctrl;
  const Args A = *P.args;
  const int D = P.D, T = P.T, B = P.B;
  const float lambda = A.damping;
  const size_t stride = (size_t)B;   // one channel group: consecutive chunks are B tickets apart
  const long long tmo = A.timeout_ns;

  auto init_barriers = [&]() {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_sfull[s], 1u);
      mbar_init(&bar_sempty[s], (unsigned)C::NEW);
      mbar_init(&bar_mma[s], 1u);
      mbar_init(&bar_tempty[s], (unsigned)C::NEW);
    }
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&bar_lb[s], (unsigned)C::NCG);
      mbar_init(&bar_cfull[s], 1u);
      mbar_init(&bar_cempty[s], (unsigned)C::NEW);
    }
    mbar_init(&bar_xfull, 1u);
    mbar_init(&bar_xempty, (unsigned)C::NEW);
    mbar_init(&bar_afull, (unsigned)C::NEW);
    mbar_init(&bar_ofull, (unsigned)C::NEW);
    mbar_init(&bar_oempty, 1u);
    mbar_init_fence();
  };
  auto inval_barriers = [&]() {
    for (int s = 0; s < 2; ++s) {
      mbar_inval(&bar_sfull[s]);
      mbar_inval(&bar_sempty[s]);
      mbar_inval(&bar_mma[s]);
      mbar_inval(&bar_tempty[s]);
    }
    for (int s = 0; s < NSLOT; ++s) {
      mbar_inval(&bar_lb[s]);
      mbar_inval(&bar_cfull[s]);
      mbar_inval(&bar_cempty[s]);
    }
    mbar_inval(&bar_xfull);
    mbar_inval(&bar_xempty);
    mbar_inval(&bar_afull);
    mbar_inval(&bar_ofull);
    mbar_inval(&bar_oempty);
  };
  // iteration and look-back epoch of this launch's first iteration; with P.persist each further
  // iteration of the launch (one round of the loop below, after the grid barrier) adds one to both
  const unsigned gen0 = *(volatile unsigned*)&ctrl->gen;
  const unsigned epoch0 = *(volatile unsigned*)&ctrl->epoch;
  const int iter0 = *(volatile int*)&ctrl->iter;
  unsigned epoch = epoch0;
  uint32_t tmem = 0u;
  for (int round = 0;; ++round) {
  if (tid == 0) {
    if (round == 0) {
      atomicMin(&ctrl->t_start, globaltimer());
      init_barriers();   // later rounds: re-initialised at the end of the previous one
    }
    s_abort = 0;
  }
  epoch = epoch0 + (unsigned)round;
  const int iter = iter0 + round;
  if (tid == 0) {
    // The first tile of every CTA has a static ticket (blockIdx.x < tiles: the grid is never
    // larger) and is fetched right away, overlapping the weight load and TMEM set-up below.
    const CUtensorMap* tm_s = P.tmaps + ((iter & 1) ? 1 : 0);
    const CUtensorMap* tm_x = P.tmaps + 2;
    tmap_acquire(tm_s);
    tmap_acquire(tm_x);
    // the last round's states (other CTAs' stores, ordered before the grid barrier) are read by
    // the tensor-copy loads below
    asm volatile("fence.proxy.async.global;" ::: "memory");
    const int kg = (int)blockIdx.x;
    if (kg < P.tiles_per_group) {
      const int b = kg % B;
      const int t0 = (kg / B) * L;
      s_tk[0] = kg;
      mbar_arrive_expect_tx(&bar_sfull[0], (unsigned)(NKH * C::SH_LOAD));
#pragma unroll
      for (int h = 0; h < NKH; ++h) tma_load_3d(sS + h * C::SH_BYTES, tm_s, 32 * h, t0 - 1, b, &bar_sfull[0]);
      mbar_arrive_expect_tx(&bar_xfull, (unsigned)C::X_BYTES);
      tma_load_3d(sX, tm_x, 0, t0, b, &bar_xfull);
    } else {
      s_tk[0] = -1;
      mbar_arrive(&bar_sfull[0]);
    }
  }

  // weights: W_hi and W_lo in the K-major core-matrix layout (pre-packed), diagonals, b_hn
  if (round == 0) {
    const float4* w4 = reinterpret_cast<const float4*>(P.wt);
    float4* d4 = reinterpret_cast<float4*>(sBH);   // sBH and sBL are contiguous
    for (int e = tid; e < 2 * C::B_BYTES / 16; e += C::NT) d4[e] = __ldg(w4 + e);
    for (int e = tid; e < R * DP; e += C::NT) sWd[e] = __ldg(P.wdiag + e);
    for (int e = tid; e < DP; e += C::NT) sBhn[e] = (CELL == PN_CELL_GRU) ? __ldg(P.bhn + e) : 0.0f;
    fence_async_smem();   // the tensor cores read sBH/sBL through the async proxy
  }
  if (warp == 0 && round == 0) {
    tmem_alloc(&s_tmem, (uint32_t)C::ALLOC_COLS);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  tmem = s_tmem;

  unsigned rbits = 0u;

  if (warp == 0) {
    // =========================== producer ===================================
    const CUtensorMap* tm_s = P.tmaps + ((iter & 1) ? 1 : 0);   // s^(i)
    const CUtensorMap* tm_x = P.tmaps + 2;                      // step inputs
    // tile 0 was issued before the block-wide sync (static ticket blockIdx.x)
    const bool none = (int)blockIdx.x >= P.tiles_per_group;
    int it = 1;
    int x_issued = none ? 0 : 1;
    for (; !none; ++it) {
      const int st = it & 1;
      if (it >= 2 && !mbar_wait_flag(&bar_sempty[st], (((unsigned)it >> 1) & 1u) ^ 1u, ctrl, tmo, &s_abort)) break;
      int kg = 0;
      if (lane == 0) kg = (int)(gridDim.x + atomicAdd(&ctrl->ticket[0], 1u));
      kg = __shfl_sync(0xffffffffu, kg, 0);
      if (kg >= P.tiles_per_group) {
        if (lane == 0) {
          s_tk[st] = -1;
          mbar_arrive(&bar_sfull[st]);
        }
        ++it;
        break;
      }
      const int b = kg % B;
      const int t0 = (kg / B) * L;
      if (lane == 0) {
        // steps t0-1 .. t0+L-1 (step -1 reads as zero and is replaced by s0 in the split)
        s_tk[st] = kg;
        mbar_arrive_expect_tx(&bar_sfull[st], (unsigned)(NKH * C::SH_LOAD));
#pragma unroll
        for (int h = 0; h < NKH; ++h) tma_load_3d(sS + (st * NKH + h) * C::SH_BYTES, tm_s, 32 * h, t0 - 1, b, &bar_sfull[st]);
      }
      // the single step-input buffer: wait until the previous tile's inputs were consumed
      if (it >= 1 && !mbar_wait_flag(&bar_xempty, ((unsigned)(it - 1)) & 1u, ctrl, tmo, &s_abort)) {
        ++it;
        break;
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar_xfull, (unsigned)C::X_BYTES);
        tma_load_3d(sX, tm_x, 0, t0, b, &bar_xfull);
      }
      __syncwarp();
      x_issued = it + 1;
    }
    // drain every fill this warp issued
    for (int j = max(0, it - 2); j < it; ++j)
      if (!mbar_drain(&bar_sfull[j & 1], ((unsigned)j >> 1) & 1u, tmo) && lane == 0)
        raise_error(ctrl, (int)PN_ERR_TIMEOUT);
    if (x_issued > 0 && !mbar_drain(&bar_xfull, ((unsigned)(x_issued - 1)) & 1u, tmo) && lane == 0)
      raise_error(ctrl, (int)PN_ERR_TIMEOUT);
  } else if (warp == 1) {
    // ======================= MMA and store issuer ============================
    constexpr uint32_t idesc = umma_idesc_tf32(L, N);
    constexpr uint32_t SBO_B = (K / 4) * 128;
    const uint64_t a_base0 = umma_smem_desc(smem_addr(sS), 16, 1024, 2);
    const uint64_t a_lo = umma_smem_desc(smem_addr(sLo), 16, 1024, 2);
    const uint64_t b_base = umma_smem_desc(smem_addr(sBH), 128, SBO_B, 0);   // W_lo follows W_hi
    const CUtensorMap* tm_o = P.tmaps + ((iter & 1) ? 3 : 4);   // s^(i+1) goes to the other buffer
    if (lane == 0) tmap_acquire(tm_o);
    int nstored = 0;   // output tiles taken so far
    // output tile j: wait until it is staged, store it, release the staging buffer.
    // Returns false at the stop marker or when the wait gave up.
    auto store_tile = [&](int j) -> bool {
      if (!mbar_wait_flag(&bar_ofull, (unsigned)j & 1u, ctrl, tmo, &s_abort)) return false;
      const int kgj = s_otk[j & 1];
      if (kgj == -1) return false;
      if (lane == 0) {
        if (kgj >= 0) {
          tma_store_3d(tm_o, 0, (kgj / B) * L, kgj % B, sO);
          bulk_commit();
          bulk_wait_read();
        }
        mbar_arrive(&bar_oempty);
      }
      __syncwarp();
      nstored = j + 1;
      return true;
    };
    int issued = 0;
    for (int it = 0;; ++it) {
      if (!mbar_wait_flag(&bar_afull, (unsigned)it & 1u, ctrl, tmo, &s_abort)) break;
      if (s_atk[it & 1] < 0) break;
      const int buf = it & 1;
      if (it >= 2 && !mbar_wait_flag(&bar_tempty[buf], (((unsigned)it >> 1) & 1u) ^ 1u, ctrl, tmo, &s_abort)) break;
      tc_fence_after();
      if (lane == 0) {
        // descriptors differ only in the start-address field: base + compile-time offsets
        const uint32_t d = tmem + (uint32_t)(buf * C::TCOLS);
        const uint64_t a_hi = a_base0 + (uint64_t)(((it & 1) * NKH * C::SH_BYTES) >> 4);
#pragma unroll
        for (int pass = 0; pass < 3; ++pass) {
          // pass 0: S_hi W_hi, pass 1: S_hi W_lo, pass 2: S_lo W_hi
#pragma unroll
          for (int kb = 0; kb < K / 8; ++kb) {
            const int h = kb >> 2;   // column half; 4 K-steps of 32 bytes per 128-byte swizzled row
            const uint64_t ad = (pass == 2) ? a_lo + (uint64_t)((h * C::LO_BYTES + (kb & 3) * 32) >> 4)
                                            : a_hi + (uint64_t)((h * C::SH_BYTES + (kb & 3) * 32) >> 4);
            const uint64_t bd = b_base + (uint64_t)(((pass == 1 ? C::B_BYTES : 0) + kb * 256) >> 4);
            umma_tf32(d, ad, bd, idesc, (pass > 0 || kb > 0) ? 1u : 0u);
          }
        }
        umma_commit(&bar_mma[buf]);
      }
      __syncwarp();
      issued = it + 1;
      // the output tile staged in epilogue tile it-1 (after it released the operands of tile it)
      const int j = it - 1 - C::OUT_LAG;
      if (j >= 0 && !store_tile(j)) break;
    }
    // every issued product must have completed before TMEM is released
    for (int j = max(0, issued - 2); j < issued; ++j)
      if (!mbar_drain(&bar_mma[j & 1], ((unsigned)j >> 1) & 1u, tmo) && lane == 0)
        raise_error(ctrl, (int)PN_ERR_TIMEOUT);
    // the remaining output tiles, up to the stop marker
    for (int j = nstored;; ++j)
      if (!store_tile(j)) break;
    // the stored states are in global memory, ordered before this CTA's part of the grid barrier
    if (lane == 0) {
      bulk_wait_all();
      asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    __syncwarp();
    if (lane == 0) bulk_wait_all();   // the states are in global memory before the CTA retires
  } else if (warp < C::WE0) {
    // =========================== look-back ==================================
    // warp 2 + j takes tiles j, j + NLB, j + 2 NLB, ... of this CTA.  Aggregates
    // and states are published as self-validating words (value + launch tag);
    // the flags only tell a reader where to look, so no fences are needed.
    if constexpr (kScan) {
      unsigned long long* aggw = reinterpret_cast<unsigned long long*>(P.agg);    // [tile][DP] x {A, B}
      unsigned long long* prefw = reinterpret_cast<unsigned long long*>(P.pref);  // [tile][DP]
      const unsigned tag = lookback_tag(epoch);
      for (int it = warp - 2;; it += C::NLB) {
        const int slot = it % NSLOT;
        const unsigned ph = (unsigned)(it / NSLOT) & 1u;
        if (!mbar_wait_flag(&bar_lb[slot], ph, ctrl, tmo, &s_abort)) break;
        const int kg = s_lbtk[slot];
        if (kg < 0) break;
        const int b = kg % B;
        const int chunk = kg / B;
        const size_t k = (size_t)kg;
        const bool stall = (A.stall_ticket == kg);
        float2 ag[C::NQ];
#pragma unroll
        for (int q = 0; q < C::NQ; ++q) {
          const int j = lane + 32 * q;
          ag[q] = (j < DP) ? *reinterpret_cast<const float2*>(sAgg + (slot * DP + j) * 2) : make_float2(1.0f, 0.0f);
        }
        // 1. the tile aggregate, for successors that reach this tile before its state (the
        //    first chunk too: a successor may start from s0 before that chunk's state is out)
        if (!stall) {
#pragma unroll
          for (int q = 0; q < C::NQ; ++q) {
            const int j = lane + 32 * q;
            if (j < DP) st_word2(aggw + (k * DP + j) * 2, tag_word(ag[q].x, tag), tag_word(ag[q].y, tag));
          }
          __syncwarp();
          if (lane == 0) st_relaxed(P.flags + k, make_flag(epoch, kFlagAgg));
        }
        // 2. the carry: nearest published state, then the aggregates in between
        int n_agg = lookback_nearest_state(P.flags, k, stride, chunk, epoch, ctrl, tmo);
        float carry[C::NQ];
#pragma unroll
        for (int q = 0; q < C::NQ; ++q) carry[q] = 0.0f;
        if (n_agg >= 0) {
          if (chunk - 1 - n_agg >= 0) {
            if (!ld_tagged_state<DP, C::NQ>(prefw + (k - (size_t)(n_agg + 1) * stride) * DP, tag, carry, ctrl, tmo))
              n_agg = -1;
          } else {
#pragma unroll
            for (int q = 0; q < C::NQ; ++q) {
              const int j = lane + 32 * q;
              carry[q] = (j < D) ? __ldg(A.s0 + (size_t)b * D + j) : 0.0f;
            }
          }
        }
        for (int d0 = n_agg; d0 >= 1; d0 -= 4) {   // oldest aggregate first, four loads in flight
          float fa[4][C::NQ], fb[4][C::NQ];
          if (!ld_tagged_aggs<DP, C::NQ>(aggw, k, stride, d0, tag, fa, fb, ctrl, tmo)) {
            n_agg = -1;
            break;
          }
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (d0 - u >= 1) {
#pragma unroll
              for (int q = 0; q < C::NQ; ++q) carry[q] = fmaf(fa[u][q], carry[q], fb[u][q]);
            }
        }
        if (n_agg < 0) s_abort = 1;
        // 3. hand the carry to the epilogue (its slot is free once tile it - NSLOT was formed)
        if (it >= NSLOT && !mbar_wait_flag(&bar_cempty[slot], ph ^ 1u, ctrl, tmo, &s_abort)) break;
#pragma unroll
        for (int q = 0; q < C::NQ; ++q) {
          const int j = lane + 32 * q;
          if (j < DP) sCarry[slot * DP + j] = carry[q];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_cfull[slot]);
        // 4. the tile's end state
        if (n_agg >= 0 && !stall) {
#pragma unroll
          for (int q = 0; q < C::NQ; ++q) {
            const int j = lane + 32 * q;
            if (j < DP) st_word(prefw + k * DP + j, tag_word(fmaf(ag[q].x, carry[q], ag[q].y), tag));
          }
          __syncwarp();
          if (lane == 0) st_relaxed(P.flags + k, make_flag(epoch, kFlagPrefix));
        }
      }
    }
  } else {
    // =========================== epilogue ===================================
    const int e = warp - C::WE0;            // 0 .. NEW-1
    const int quarter = warp & 3;           // TMEM lane quarter this warp may access
    const int cg = e >> 2;                  // channel group
    const int row = quarter * 32 + lane;    // step row within the tile
    const int cbase = cg * CH;              // first channel of this thread
    const int te = tid - 32 * C::WE0;       // 0 .. NTE-1 among the epilogue threads
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int hh = cbase >> 5;              // column half of this thread's channels
    const int cw = cbase & 31;              // first column within that half

    // S_lo of stage `stg` (rows 0..L-1), in the same swizzled layout.  For the first
    // chunk of a sequence, row 0 (step -1, loaded as zero) becomes s0 first.
    auto split = [&](int stg, int kgs) {
      const bool first = (kgs / B) == 0;
      const float* s0row = A.s0 + (size_t)(kgs % B) * D;
      for (int u = te; u < NKH * L * 8; u += NTE) {
        const int q = u & 7;             // 16-byte chunk within the 128-byte row
        const int r = (u >> 3) % L;
        const int h = (u >> 3) / L;
        const uint32_t off = sw128_offset(r, 4 * q);
        unsigned char* srow = sS + (stg * NKH + h) * C::SH_BYTES;
        float4 v;
        if (first && r == 0) {
          v = __ldg(reinterpret_cast<const float4*>(s0row + 32 * h) + q);
          *reinterpret_cast<float4*>(srow + off) = v;
        } else {
          v = *reinterpret_cast<const float4*>(srow + off);
        }
        *reinterpret_cast<float4*>(sLo + h * C::LO_BYTES + off) =
            make_float4(tf32_tail(v.x), tf32_tail(v.y), tf32_tail(v.z), tf32_tail(v.w));
      }
      fence_async_smem();   // generic writes -> async proxy (tensor cores)
    };

    // hand the staged rows of output tile j (ticket kgj) to the store issuer
    auto publish_out = [&](int j, int kgj) {
      fence_async_smem();   // this thread's staging writes -> async proxy (the TMA store)
      __syncwarp();
      if (lane == 0) {
        if (te == 0) s_otk[j & 1] = s_abort ? -2 : kgj;
        mbar_arrive(&bar_ofull);
      }
    };

    // s^(i+1) of tile j from its parked prefixes and the carry of the look-back
    auto write_out = [&](int j, int kgj) {
      const int slot = j % NSLOT;
      mbar_wait_flag(&bar_cfull[slot], (unsigned)(j / NSLOT) & 1u, ctrl, tmo, &s_abort);
      if (j >= 1) mbar_wait_flag(&bar_oempty, (unsigned)(j - 1) & 1u, ctrl, tmo, &s_abort);   // staging free
      const float* cr = sCarry + slot * DP + cbase;
      const uint32_t sbase = tmem + (uint32_t)(C::STASH0 + slot * C::SCOLS) + lane_off;
      float bb[16], aa[16];
      tmem_ld16(sbase + (uint32_t)((kHasA ? DP : 0) + cbase), bb);
      if constexpr (kHasA) tmem_ld16(sbase + (uint32_t)cbase, aa);
      float* o = sO + row * SP + cbase;
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
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_cempty[slot]);
      publish_out(j, kgj);
    };

    // prologue: operands of the first tile
    {
      int kg0 = -1;
      if (mbar_wait_flag(&bar_sfull[0], 0u, ctrl, tmo, &s_abort)) kg0 = s_tk[0];
      if (kg0 >= 0) split(0, kg0);
      __syncwarp();
      if (lane == 0) {
        if (te == 0) s_atk[0] = s_abort ? -1 : kg0;
        mbar_arrive(&bar_afull);
      }
    }
    named_barrier(1, NTE);
    int kg = s_atk[0];   // written by te == 0 before the barrier
    int it = 0;
    int kg_m1 = -1, kg_m2 = -1;   // tickets of tiles it-1 and it-2
    for (; kg >= 0; ++it) {
      const int st = it & 1;
      const int buf = it & 1;
      const int chunk = kg / B;
      const int t = chunk * L + row;
      const unsigned char* Sst = sS + st * NKH * C::SH_BYTES + hh * C::SH_BYTES;

      // ---- Z from TMEM, then the cell --------------------------------------
      mbar_wait_flag(&bar_mma[buf], ((unsigned)it >> 1) & 1u, ctrl, tmo, &s_abort);
      tc_fence_after();
      float z[R][CH];
#pragma unroll
      for (int q = 0; q < R; ++q)
        tmem_ld16(tmem + (uint32_t)(buf * C::TCOLS) + lane_off + (uint32_t)(q * DP + cbase), z[q]);
      mbar_wait_flag(&bar_xfull, (unsigned)it & 1u, ctrl, tmo, &s_abort);
      const bool tok = (t < T);
      float av[CH], bv[CH];
#pragma unroll
      for (int c4 = 0; c4 < CH; c4 += 4) {
        const int c = cbase + c4;
        const float4 sp4 = *reinterpret_cast<const float4*>(Sst + sw128_offset(row, cw + c4));
        const float4 sc4 = *reinterpret_cast<const float4*>(Sst + sw128_offset(row + 1, cw + c4));
        float4 x4[R];
#pragma unroll
        for (int q = 0; q < R; ++q) x4[q] = *reinterpret_cast<const float4*>(sX + row * XP + q * DP + c);
        float4 wd4[R];
#pragma unroll
        for (int q = 0; q < R; ++q) wd4[q] = *reinterpret_cast<const float4*>(sWd + q * DP + c);
        const float4 bhn4 = *reinterpret_cast<const float4*>(sBhn + c);
        const float spv[4] = {sp4.x, sp4.y, sp4.z, sp4.w};
        const float scv[4] = {sc4.x, sc4.y, sc4.z, sc4.w};
        const float bhv[4] = {bhn4.x, bhn4.y, bhn4.z, bhn4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float xv[R], wd[R];
#pragma unroll
          for (int q = 0; q < R; ++q) {
            xv[q] = (u == 0) ? x4[q].x : (u == 1) ? x4[q].y : (u == 2) ? x4[q].z : x4[q].w;
            wd[q] = (u == 0) ? wd4[q].x : (u == 1) ? wd4[q].y : (u == 2) ? wd4[q].z : wd4[q].w;
          }
          const float sp = spv[u], sc = scv[u];
          float y, a, bb, res;
          if constexpr (CELL == PN_CELL_TANH_RNN) {
            y = tanh_pn(z[0][c4 + u] + xv[0]);
            res = sc - y;
            a = (MODE == PN_QUASI) ? (1.0f - y * y) * wd[0] : (MODE == PN_PICARD ? 1.0f : 0.0f);
            bb = (MODE == PN_JACOBI) ? y : y - a * sp;
          } else if constexpr (CELL == PN_CELL_EULER_TANH) {
            const float gg = tanh_pn(z[0][c4 + u] + xv[0]);
            const float eg = P.eps * gg;
            y = sp + eg;
            res = (sc - sp) - eg;
            if (MODE == PN_QUASI) {
              const float ed = P.eps * (1.0f - gg * gg) * wd[0];
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
            const float hn = z[2][c4 + u] + bhv[u];
            const float nn = tanh_pn(xv[2] + rr * hn);
            y = nn + zz * (sp - nn);
            res = sc - y;
            if (MODE == PN_QUASI) {
              const float omz = 1.0f - zz;
              const float dn = omz * (1.0f - nn * nn);
              a = zz + (sp - nn) * zz * omz * wd[1] + dn * (rr * wd[2] + hn * rr * (1.0f - rr) * wd[0]);
            } else {
              a = (MODE == PN_PICARD) ? 1.0f : 0.0f;
            }
            bb = (MODE == PN_JACOBI) ? y : y - a * sp;
          }
          if (tok) {
            rbits = max(rbits, abs_bits(res));
            av[c4 + u] = a;
            bv[c4 + u] = bb;
            // damping (Jacobi only here: the host routes damped Picard and GRU quasi-Newton to the
            // FP32 kernels, whose write-out still has s^(i)_t at hand)
            if (MODE == PN_JACOBI && lambda != 1.0f) bv[c4 + u] = fmaf(lambda, bb - sc, sc);
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
        if (kn >= 0 && !s_abort) split(st ^ 1, kn);
        __syncwarp();
        if (lane == 0) {
          // the ticket of tile it+1 is also the loop's exit decision, read after the next barrier
          if (te == 0) s_atk[(it + 1) & 1] = s_abort ? -1 : kn;
          mbar_arrive(&bar_afull);
        }
      }

      if constexpr (!kScan) {
        // s^(i+1) = f(s^(i)) row by row: stage it for the store issuer
        if (it >= 1) mbar_wait_flag(&bar_oempty, (unsigned)(it - 1) & 1u, ctrl, tmo, &s_abort);
        float* o = sO + row * SP + cbase;
#pragma unroll
        for (int c4 = 0; c4 < CH; c4 += 4)
          *reinterpret_cast<float4*>(o + c4) = make_float4(bv[c4], bv[c4 + 1], bv[c4 + 2], bv[c4 + 3]);
        publish_out(it, kg);
        named_barrier(1, NTE);
        kg = s_atk[(it + 1) & 1];
      } else {
        // the states of tile it-2: its carry had two tiles of time to arrive
        if (it >= C::DEFER) write_out(it - C::DEFER, kg_m2);

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
        float* tot = sTot + (it & 1) * C::TOT_FLOATS;
        if (lane == 31) {
#pragma unroll
          for (int c = 0; c < CH; c += 2)
            *reinterpret_cast<float4*>(tot + ((cg * 4 + quarter) * CH + c) * 2) =
                make_float4(kHasA ? av[c] : 1.0f, bv[c], kHasA ? av[c + 1] : 1.0f, bv[c + 1]);
        }
        named_barrier(1, NTE);   // quarter totals, and the ticket of tile it+1
        const int kg_next = s_atk[(it + 1) & 1];
        if (quarter > 0) {
          // prefix of the earlier quarters: tot_{quarter-1} o ... o tot_0
          float PA[CH], PB[CH];
#pragma unroll
          for (int c = 0; c < CH; ++c) {
            PA[c] = 1.0f;
            PB[c] = 0.0f;
          }
          for (int qq = 0; qq < quarter; ++qq) {
            const float* tq = tot + (cg * 4 + qq) * CH * 2;
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
        // the last row holds the tile aggregate: hand it to the look-back
        const int slot = it % NSLOT;
        if (quarter == 3 && lane == 31) {
#pragma unroll
          for (int c = 0; c < CH; c += 2)
            *reinterpret_cast<float4*>(sAgg + (slot * DP + cbase + c) * 2) =
                make_float4(kHasA ? av[c] : 1.0f, bv[c], kHasA ? av[c + 1] : 1.0f, bv[c + 1]);
          if (cg == 0) s_lbtk[slot] = s_abort ? -1 : kg;
          mbar_arrive(&bar_lb[slot]);
        }
        // ---- park this tile's in-tile prefixes in TMEM; formed two tiles later
        {
          const uint32_t sbase = tmem + (uint32_t)(C::STASH0 + slot * C::SCOLS) + lane_off;
          if constexpr (kHasA) tmem_st16(sbase + (uint32_t)cbase, av);
          tmem_st16(sbase + (uint32_t)((kHasA ? DP : 0) + cbase), bv);
          tmem_st_wait();
        }
        kg_m2 = kg_m1;
        kg_m1 = kg;
        kg = kg_next;
      }
    }
    if constexpr (kScan) {
      if (it >= 2) write_out(it - 2, kg_m2);
      if (it >= 1) write_out(it - 1, kg_m1);
      // stop the look-back warps: their next tiles are it .. it + NLB - 1
      if (quarter == 3 && lane == 31) {
        for (int j = it; j < it + C::NLB; ++j) {
          if (cg == 0) s_lbtk[j % NSLOT] = -1;
          mbar_arrive(&bar_lb[j % NSLOT]);
        }
      }
    }
    // stop the store issuer once it has taken the last tile (a warp arrives on
    // bar_ofull again only after the previous phase completed)
    if (it >= 1) mbar_wait_flag(&bar_oempty, (unsigned)(it - 1) & 1u, ctrl, tmo, &s_abort);
    __syncwarp();
    if (lane == 0) {
      if (te == 0) s_otk[it & 1] = -1;
      mbar_arrive(&bar_ofull);
    }
  }

  // ---- residual of this iteration; the next one (grid barrier) or the end of the launch
  rbits = warp_max_u32(rbits);
  if (lane == 0) sRed[warp] = __uint_as_float(rbits);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  unsigned rmax = 0u;   // the CTA's residual maximum, on thread 0
  if (tid == 0) {
    for (int w = 0; w < C::NT / 32; ++w) rmax = max(rmax, __float_as_uint(sRed[w]));
    if (rmax && !P.persist) atomicMax(&ctrl->resid_bits, rmax);
  }
  if (!P.persist) break;
  // fresh barriers for the next round (every operation on the old ones has completed)
  if (tid == 0) {
    inval_barriers();
    init_barriers();
  }
  if (!finish_iteration(P, A, iter, epoch, s_last, (gen0 >> 1) + (unsigned)round, rmax)) break;
  }   // rounds

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    tmem_dealloc(tmem, (uint32_t)C::ALLOC_COLS);
  if (!P.persist) finish_launch(P, A, epoch, s_last);
}

}  // namespace pn
