// pn_iter_diag_tct.cuh -- tensor-core iteration kernel with a channel-major
// accumulator, for the one-gate cells (tanh RNN, Euler drift) at D = 32, 64,
// in the Jacobi, Picard and diagonal quasi-Newton modes.
//
// Same iteration as pn_iter_diag_tc.cuh (the page's unified update, "Parallel
// Newton methods..." page §1.2, with a diagonal A~_t, §2.2.1 / §2.2.3, solved
// by the chunked scan of §2.1), with the roles of the two MMA operands
// swapped: Z = W S^T, so a TMEM lane holds one channel and its columns hold
// consecutive steps.  The MMAs are M = 64: an M = 64 accumulator takes 16
// lanes of each 32-lane quarter (row m at lane 32 (m / 16) + m mod 16), and a
// second one sits beside it at lane offset 16, so the 128 lanes hold two
// halves.  Each half holds 64 / D bands of D channels, and each (half, band)
// pair is one step segment: RS = D L / 128 consecutive steps of all D
// channels.  Segment (h, j)'s MMA reads its steps of S as the B operand and a
// 64-row window of a banded copy of W as the A operand, whose nonzero rows are
// exactly band j (for D = 64 the window is W itself, with no zero rows).
// Products are 3xTF32 as in the row-major kernel: S_hi W_hi + S_hi W_lo +
// S_lo W_hi, with S_hi the tensor core's truncation.
//
// Each epilogue thread owns one lane (channel c of one segment: the two lane
// halves of a warp hold two different segments) and 16
// consecutive steps: it evaluates the cell, the Jacobian diagonal and the
// residual, and scans those steps sequentially in registers -- no shuffles.
// The 8 sixteen-step pieces of a channel are combined through shared memory;
// the piece prefix (PA, PB) stays in registers, the in-piece prefixes are
// parked in TMEM, and the states are formed three tiles later from the carry
// of the look-back warps and stored to global memory by the epilogue threads
// themselves (each warp store instruction covers two 64-byte row segments).
//
// With P.persist = 1 the kernel runs the whole fixed-point loop in one launch:
// after each iteration the CTAs meet at a bounded grid barrier whose last
// arrival applies the stop rule, then the next iteration starts with the
// weights, TMEM and barrier memory of the CTA kept (no launch gap, no set-up).
//
// The step inputs are double-buffered with the S stages and released with
// them, so both are fetched two tiles ahead of their use.
//
// Warp roles (one CTA per SM): 0 producer (tickets and TMA loads); 1 MMA issuer;
// 2-3 look-back (scan modes, alternate tiles); the rest epilogue (4 TMEM lane
// quarters x RS / 16 step groups).  The epilogue forms the next tile's S_lo
// right after the current tile's cell phase, so the tensor cores compute the
// next tile's products while the epilogue finishes the current one.
#pragma once

#include "pn_iter_diag_tc.cuh"

namespace pn {

// The carry into tile k: the published state n_agg + 1 places back (unless
// `from_s0`: the chain starts at s0, which the caller put in `carry`) folded
// with the aggregates n_agg .. 1 places back, oldest first.  Each round trip
// loads up to FB aggregates, the first one the state as well; a round spins
// (bounded) until all its words carry `tag`.  Returns false when a wait gave up.
template <int DP, int NQ, int FB>
__device__ __forceinline__ bool lookback_fold(const unsigned long long* aggw, const unsigned long long* prefw, size_t k,
                                              size_t stride, int n_agg, bool from_s0, unsigned tag, float (&carry)[NQ],
                                              Ctrl* ctrl, long long timeout_ns) {
  const int lane = threadIdx.x & 31;
  bool need_state = !from_s0;
  const unsigned long long* src = prefw + (k - (size_t)(n_agg + 1) * stride) * DP;
  for (int d0 = n_agg; need_state || d0 >= 1; d0 -= FB) {
    unsigned long long ws[NQ], wa[FB][NQ], wb[FB][NQ];
    unsigned long long t0 = 0;
    unsigned spins = 0;
    while (true) {
      bool ok = true;
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        const int j = lane + 32 * q;
        ws[q] = (need_state && j < DP) ? ld_word(src + j) : tag_word(0.0f, tag);
#pragma unroll
        for (int u = 0; u < FB; ++u) {
          const int d = d0 - u;
          wa[u][q] = tag_word(1.0f, tag);
          wb[u][q] = tag_word(0.0f, tag);
          if (d >= 1 && j < DP) ld_word2(aggw + ((k - (size_t)d * stride) * DP + j) * 2, wa[u][q], wb[u][q]);
        }
      }
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        ok = ok && word_tagged(ws[q], tag);
#pragma unroll
        for (int u = 0; u < FB; ++u) ok = ok && word_tagged(wa[u][q], tag) && word_tagged(wb[u][q], tag);
      }
      if (__all_sync(0xffffffffu, ok)) break;
      if (spins == 0) t0 = globaltimer();
      if (spin_give_up(spins, t0, ctrl, timeout_ns)) return false;
    }
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      if (need_state) carry[q] = word_value(ws[q]);
#pragma unroll
      for (int u = 0; u < FB; ++u) carry[q] = fmaf(word_value(wa[u][q]), carry[q], word_value(wb[u][q]));
    }
    need_state = false;
  }
  return true;
}

// 32 TMEM columns of this warp's lanes from a[16], b[16] in the order
// [a 0-7 | b 0-7 | a 8-15 | b 8-15], so that each half can be read back alone.
__device__ __forceinline__ void tmem_st32_split8(uint32_t taddr, const float (&a)[16], const float (&b)[16]) {
  float lo[16], hi[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    lo[i] = a[i];
    lo[8 + i] = b[i];
    hi[i] = a[8 + i];
    hi[8 + i] = b[8 + i];
  }
  tmem_st32(taddr, lo, hi);
}

template <int CELL, int MODE, int DP>
struct DiagTctCfg {
  static_assert(CELL != PN_CELL_GRU, "one-gate cells only");
  static_assert(DP == 32 || DP == 64, "D = 32 or 64");
  static constexpr bool kScan = (MODE != PN_JACOBI);
  static constexpr int L = 128;                  // steps per tile
  static constexpr int K = DP;                   // MMA K (input channels)
  static constexpr int MT = 64;                  // MMA M: one accumulator half (16 lanes of each lane quarter)
  static constexpr int NB = MT / DP;             // channel bands per accumulator half (1 for D = 64, 2 for D = 32)
  static constexpr int NSEG = 2 * NB;            // step segments: 2 halves x NB bands = 128 / D
  static constexpr int RS = L / NSEG;            // steps per segment = MMA N
  static constexpr int NRG = RS / 16;            // 16-step groups per segment
  static constexpr int NPC = NSEG * NRG;         // pieces per channel (L / 16)
  static constexpr int NKH = DP / 32;            // 32-float column halves of S
  static constexpr int SCOLS = (MODE == PN_QUASI ? 2 : 1) * RS;   // stash columns per tile: per 16-step
                                                                     // group, [A (16) |] B (16)
  static constexpr int NSLOT = 3;                // TMEM stash slots (and look-back carry slots)
  static constexpr int DEFER = NSLOT;            // a tile's states are formed 3 tiles later, just before
                                                 // that tile's prefixes take over its stash slot
  static constexpr int NAG = NSLOT + 1;          // slots of the aggregate hand-off to the look-back
  static constexpr int NLB = kScan ? 2 : 0;      // look-back warps, alternating tiles
  static constexpr int FB = 4;                   // aggregates per look-back round trip (4 measured fastest of 2-8)
  static constexpr int STASH0 = 2 * RS;          // accumulators: 2 x RS columns
  static constexpr int USED_COLS = STASH0 + (kScan ? NSLOT * SCOLS : 0);
  static constexpr int ALLOC_COLS =
      USED_COLS <= 32 ? 32 : USED_COLS <= 64 ? 64 : USED_COLS <= 128 ? 128 : USED_COLS <= 256 ? 256 : 512;
  static constexpr int NEW = 4 * NRG;            // epilogue warps
  static constexpr int NTE = 32 * NEW;
  static constexpr int WE0 = 2 + NLB;            // first epilogue warp
  static constexpr int NT = 32 * (WE0 + NEW);
  static constexpr int NQ = DP / 32;             // channels per look-back lane
  static constexpr int NLASTW = 4 / NB;          // epilogue warps holding the last piece of a channel
  static constexpr int WROWS = 3 * MT - DP;      // banded W: Z(64-D) W_hi Z(64-D) W_lo Z(64-D)
  static constexpr int align(int v, int a) { return (v + a - 1) / a * a; }
  static constexpr int SH_LOAD = (L + 1) * 128;
  static constexpr int SH_BYTES = align(SH_LOAD, 1024);
  static constexpr int LO_BYTES = L * 128;
  static constexpr int X_BYTES = L * DP * 4;
  static constexpr int W_BYTES = WROWS * DP * 4;
  static constexpr uint32_t SBO_W = (K / 4) * 128;
  static constexpr int OFF_S = 0;                                 // [2 stages][NKH][SH_BYTES]
  static constexpr int OFF_LO = OFF_S + 2 * NKH * SH_BYTES;       // [NKH][LO_BYTES]
  static constexpr int OFF_X = OFF_LO + NKH * LO_BYTES;           // [2 stages][L][DP]
  static constexpr int OFF_W = align(OFF_X + 2 * X_BYTES, 128);
  static constexpr int OFF_WD = OFF_W + W_BYTES;                  // DP floats
  static constexpr int OFF_TOT = OFF_WD + DP * 4;                 // [2][NPC][DP] float2
  static constexpr int OFF_AGG = OFF_TOT + 2 * NPC * DP * 8;      // [NAG][DP] float2
  static constexpr int OFF_CARRY = OFF_AGG + NAG * DP * 8;        // [NSLOT][DP]
  static constexpr int OFF_RED = OFF_CARRY + NSLOT * DP * 4;      // NT/32 floats
  static constexpr int SMEM_USED = OFF_RED + (NT / 32) * 4;
  static constexpr int SMEM_BYTES = SMEM_USED + 1024;             // + slack to align the base to 1024 bytes
  // first row of band j's 64-row window of the banded W (W_hi or W_lo at window rows j D .. j D + D - 1)
  static constexpr int win_hi(int j) { return (MT - DP) - j * DP; }
  static constexpr int win_lo(int j) { return (2 * MT - DP) - j * DP; }
  static_assert(USED_COLS <= 512, "TMEM columns");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

template <int CELL, int MODE, int DP>
__global__ void __launch_bounds__(DiagTctCfg<CELL, MODE, DP>::NT, 1) diag_tct_kernel(const IterParams P) {
  using C = DiagTctCfg<CELL, MODE, DP>;
  constexpr int L = C::L;
  constexpr int K = C::K;
  constexpr int NKH = C::NKH;
  constexpr int RS = C::RS;
  constexpr int NTE = C::NTE;
  constexpr int NSLOT = C::NSLOT;
  constexpr bool kScan = C::kScan;
  constexpr bool kHasA = (MODE == PN_QUASI);

  extern __shared__ __align__(1024) unsigned char smem_tct[];
  unsigned char* smem_raw = smem_tct + ((1024u - (smem_addr(smem_tct) & 1023u)) & 1023u);
  unsigned char* sS = smem_raw + C::OFF_S;       // stage st, half h at sS + (st * NKH + h) * SH_BYTES
  unsigned char* sLo = smem_raw + C::OFF_LO;     // half h at sLo + h * LO_BYTES
  const float* sX = reinterpret_cast<const float*>(smem_raw + C::OFF_X);
  unsigned char* sW = smem_raw + C::OFF_W;
  float* sWd = reinterpret_cast<float*>(smem_raw + C::OFF_WD);
  float* sTot = reinterpret_cast<float*>(smem_raw + C::OFF_TOT);
  float* sAgg = reinterpret_cast<float*>(smem_raw + C::OFF_AGG);
  float* sCarry = reinterpret_cast<float*>(smem_raw + C::OFF_CARRY);
  float* sRed = reinterpret_cast<float*>(smem_raw + C::OFF_RED);

  __shared__ __align__(8) uint64_t bar_sfull[2], bar_sempty[2], bar_xfull[2], bar_afull, bar_mma[2], bar_tempty[2],
      bar_lb[C::NAG], bar_cfull[NSLOT], bar_cempty[NSLOT];
  __shared__ int s_tk[2];        // ticket staged in s stage 0/1 (-1: no more tiles)
  __shared__ int s_atk[2];       // ticket of tile i's operands, by the parity of i (-1: stop)
  __shared__ int s_lbtk[C::NAG];  // ticket handed to the look-back per slot (-1: stop)
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ int s_last;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  Ctrl* ctrl = P.ctrl;
  const Args A = *P.args;
  const int D = P.D, T = P.T, B = P.B;
  const size_t stride = (size_t)B;   // consecutive chunks of a sequence are B tickets apart
  // Damping, s^(i+1) = s^(i) + lambda * delta: the parked prefixes (A_t, B_t), from which a state is
  // formed as A_t carry + B_t, are stored as (lambda A_t, lambda B_t + (1 - lambda) s^(i)_t); the scan,
  // the piece totals and the look-back stay undamped.
  const float lambda = A.damping;
  const bool damped = lambda != 1.0f;
  const long long tmo = A.timeout_ns;

  auto init_barriers = [&]() {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_sfull[s], 1u);
      mbar_init(&bar_xfull[s], 1u);
      mbar_init(&bar_sempty[s], (unsigned)C::NEW);
      mbar_init(&bar_mma[s], 1u);
      mbar_init(&bar_tempty[s], (unsigned)C::NEW);
    }
    for (int s = 0; s < C::NAG; ++s) mbar_init(&bar_lb[s], (unsigned)C::NLASTW);
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&bar_cfull[s], 1u);
      mbar_init(&bar_cempty[s], (unsigned)C::NEW);
    }
    mbar_init(&bar_afull, (unsigned)C::NEW);
    mbar_init_fence();
  };
  auto inval_barriers = [&]() {
    uint64_t* bars[] = {&bar_sfull[0], &bar_sfull[1], &bar_sempty[0], &bar_sempty[1], &bar_mma[0], &bar_mma[1],
                        &bar_tempty[0], &bar_tempty[1], &bar_xfull[0], &bar_xfull[1], &bar_afull};
    for (uint64_t* bb : bars) mbar_inval(bb);
    for (int s = 0; s < C::NAG; ++s) mbar_inval(&bar_lb[s]);
    for (int s = 0; s < NSLOT; ++s) {
      mbar_inval(&bar_cfull[s]);
      mbar_inval(&bar_cempty[s]);
    }
  };
  // iteration and look-back epoch of this launch's first iteration; each further
  // iteration of a looping launch adds one to both
  const unsigned gen0 = *(volatile unsigned*)&ctrl->gen;
  const unsigned epoch0 = *(volatile unsigned*)&ctrl->epoch;
  const int iter0 = *(volatile int*)&ctrl->iter;
  const bool has_tile0 = (int)blockIdx.x < P.tiles_per_group;
  unsigned epoch = epoch0;
  for (int round = 0;; ++round) {
  if (tid == 0) {
    if (round == 0) {
      atomicMin(&ctrl->t_start, globaltimer());
      init_barriers();   // later iterations: re-initialised at the end of the previous one
    }
    s_abort = 0;
  }
  epoch = epoch0 + (unsigned)round;
  const int iter = iter0 + round;
  if (tid == 0) {
    // The first tile of every CTA has a static ticket (blockIdx.x < tiles: the grid is never
    // larger) and is fetched right away, overlapping the remaining set-up.
    const CUtensorMap* tm_s = P.tmaps + ((iter & 1) ? 1 : 0);
    const CUtensorMap* tm_x = P.tmaps + 2;
    tmap_acquire(tm_s);
    tmap_acquire(tm_x);
    // the last iteration's states (other CTAs' generic stores, ordered before the grid barrier)
    // are read by this thread's tensor-copy loads, here and for every later tile of the iteration
    asm volatile("fence.proxy.async.global;" ::: "memory");
    const int kg = (int)blockIdx.x;
    if (kg < P.tiles_per_group) {
      const int b = kg % B;
      const int t0 = (kg / B) * L;
      s_tk[0] = kg;
      mbar_arrive_expect_tx(&bar_sfull[0], (unsigned)(NKH * C::SH_LOAD));
#pragma unroll
      for (int h = 0; h < NKH; ++h)
        tma_load_3d_hint(sS + h * C::SH_BYTES, tm_s, 32 * h, t0 - 1, b, &bar_sfull[0], l2_policy_evict_first());
      if (round == 0) {   // later iterations: fetched before the grid barrier
        mbar_arrive_expect_tx(&bar_xfull[0], (unsigned)C::X_BYTES);
        tma_load_3d_hint(smem_raw + C::OFF_X, tm_x, 0, t0, b, &bar_xfull[0], l2_policy_evict_last());
      }
    } else {
      s_tk[0] = -1;
      mbar_arrive(&bar_sfull[0]);
    }
  }
  float* __restrict__ dst = (iter & 1) ? A.states : P.buf1;

  if (round == 0) {
    // banded W (hi and lo in the K-major core-matrix layout): the zero bands are written here,
    // only the W_hi and W_lo row blocks (pre-packed by the host at their band offsets) are loaded
    const float4* w4 = reinterpret_cast<const float4*>(P.wt);
    float4* d4 = reinterpret_cast<float4*>(sW);
    constexpr int ROW16 = DP / 4;                 // float4s per row of the K-major layout (on average)
    constexpr int HI0 = (C::MT - DP) * ROW16, HI1 = C::MT * ROW16;            // W_hi rows, in float4 units
    constexpr int LO0 = (2 * C::MT - DP) * ROW16, LO1 = 2 * C::MT * ROW16;    // W_lo rows
    for (int e = tid; e < C::W_BYTES / 16; e += C::NT) {
      const bool wrow = (e >= HI0 && e < HI1) || (e >= LO0 && e < LO1);
      d4[e] = wrow ? __ldg(w4 + e) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
    for (int e = tid; e < DP; e += C::NT) sWd[e] = __ldg(P.wdiag + e);
    fence_async_smem();   // the tensor cores read sW through the async proxy
    if (warp == 0) {
      tmem_alloc(&s_tmem, (uint32_t)C::ALLOC_COLS);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  unsigned rbits = 0u;

  if (warp == 0) {
    // =========================== producer ===================================
    const CUtensorMap* tm_s = P.tmaps + ((iter & 1) ? 1 : 0);   // s^(i)
    const CUtensorMap* tm_x = P.tmaps + 2;                      // step inputs
    // the step inputs are read by every iteration: kept in L2 ahead of the iterates, read once each
    const uint64_t pol_keep = l2_policy_evict_last();
    const uint64_t pol_stream = l2_policy_evict_first();
    // tile 0 was issued before the block-wide sync (static ticket blockIdx.x)
    const bool none = (int)blockIdx.x >= P.tiles_per_group;
    int it = 1;
    int n_loaded = none ? 0 : 1;   // stages with their S and step-input loads issued
    for (; !none; ++it) {
      const int st = it & 1;
      // stage st (S and step inputs) is free once tile it-2's cell phase is done; the ticket is
      // claimed only then, so a CTA holds no ticket it cannot start loading
      if (it >= 2 && !mbar_wait_flag(&bar_sempty[st], (((unsigned)it >> 1) & 1u) ^ 1u, ctrl, tmo, &s_abort, 102)) break;
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
        for (int h = 0; h < NKH; ++h)
          tma_load_3d_hint(sS + (st * NKH + h) * C::SH_BYTES, tm_s, 32 * h, t0 - 1, b, &bar_sfull[st], pol_stream);
        mbar_arrive_expect_tx(&bar_xfull[st], (unsigned)C::X_BYTES);
        tma_load_3d_hint(smem_raw + C::OFF_X + st * C::X_BYTES, tm_x, 0, t0, b, &bar_xfull[st], pol_keep);
      }
      __syncwarp();
      n_loaded = it + 1;
    }
    // the last two stages' loads (and the stop marker, which has no step-input load) complete
    // before the CTA moves on
    for (int j = max(0, it - 2); j < it; ++j)
      if (!mbar_drain(&bar_sfull[j & 1], ((unsigned)j >> 1) & 1u, tmo) && lane == 0)
        raise_error(ctrl, (int)PN_ERR_TIMEOUT);
    for (int j = max(0, n_loaded - 2); j < n_loaded; ++j)
      if (!mbar_drain(&bar_xfull[j & 1], ((unsigned)j >> 1) & 1u, tmo) && lane == 0)
        raise_error(ctrl, (int)PN_ERR_TIMEOUT);
  } else if (warp == 1) {
    // =========================== MMA issuer =================================
    constexpr uint32_t idesc = umma_idesc_tf32(C::MT, RS);
    // Descriptors differ between MMAs only in the start address (bits 0-13, address >> 4;
    // shared addresses stay below 2^18 so the field never carries): precompute the bases
    // and add compile-time offsets in the fully unrolled issue loop.
    const uint64_t a_base = umma_smem_desc(smem_addr(sW), 128, C::SBO_W, 0);
    const uint64_t b_base0 = umma_smem_desc(smem_addr(sS), 16, 1024, 2);
    const uint64_t b_lo = umma_smem_desc(smem_addr(sLo), 16, 1024, 2);
    // products of stage `it` for passes p0 .. p1-1 (pass 0: W_hi S_hi, 1: W_lo S_hi, 2: W_hi S_lo)
    auto issue = [&](int it, int p0, int p1) {
      const int buf = it & 1;
      const uint32_t d = tmem + (uint32_t)(buf * RS);
      const uint64_t b_hi = b_base0 + (uint64_t)(((it & 1) * NKH * C::SH_BYTES) >> 4);
#pragma unroll
      for (int pass = 0; pass < 3; ++pass) {
        if (pass < p0 || pass >= p1) continue;
#pragma unroll
        for (int kb = 0; kb < K / 8; ++kb) {
          const int h = kb >> 2;   // column half of S; 4 K-steps of 32 bytes per 128-byte swizzled row
#pragma unroll
          for (int g = 0; g < C::NSEG; ++g) {
            // segment g = accumulator half g / NB (lane offset 16), band g % NB; the first
            // product of each half overwrites it (its other bands receive zeros)
            const int band = g % C::NB;
            const int ws = (pass == 1) ? C::win_lo(band) : C::win_hi(band);
            const uint64_t ad = a_base + (uint64_t)(((ws / 8) * C::SBO_W + kb * 256) >> 4);
            const uint64_t bd = (pass == 2 ? b_lo + (uint64_t)((h * C::LO_BYTES + g * RS * 128 + (kb & 3) * 32) >> 4)
                                           : b_hi + (uint64_t)((h * C::SH_BYTES + g * RS * 128 + (kb & 3) * 32) >> 4));
            umma_tf32(d + ((uint32_t)(16 * (g / C::NB)) << 16), ad, bd, idesc, (pass | kb | band) ? 1u : 0u);
          }
        }
      }
    };
    // The two S_hi passes need only the loaded stage (the tensor core truncates S itself), so
    // they are issued as soon as it lands and run under the epilogue's cell phase of the
    // previous tile; only the S_lo pass waits for the split.  A sequence's first chunk is the
    // exception: its row 0 (step -1) becomes s0 in the split, so all its passes wait.
    int issued = 0;
    for (int it = 0;; ++it) {
      const int buf = it & 1;
      if (!mbar_wait_flag(&bar_sfull[it & 1], ((unsigned)it >> 1) & 1u, ctrl, tmo, &s_abort, 103)) break;
      const int kn = s_tk[it & 1];
      bool early = false;
      if (kn >= 0 && kn / B != 0) {
        if (it >= 2 && !mbar_wait_flag(&bar_tempty[buf], (((unsigned)it >> 1) & 1u) ^ 1u, ctrl, tmo, &s_abort, 104)) break;
        tc_fence_after();
        if (lane == 0) issue(it, 0, 2);
        __syncwarp();
        early = true;
      }
      const bool ok = mbar_wait_flag(&bar_afull, (unsigned)it & 1u, ctrl, tmo, &s_abort, 105);
      if (!ok || s_atk[it & 1] < 0) {
        if (early) {   // let the issued products complete before the accumulator is released
          if (lane == 0) umma_commit(&bar_mma[buf]);
          __syncwarp();
          issued = it + 1;
        }
        break;
      }
      if (!early && it >= 2 && !mbar_wait_flag(&bar_tempty[buf], (((unsigned)it >> 1) & 1u) ^ 1u, ctrl, tmo, &s_abort, 106))
        break;
      tc_fence_after();
      if (lane == 0) {
        issue(it, early ? 2 : 0, 3);
        umma_commit(&bar_mma[buf]);
      }
      __syncwarp();
      issued = it + 1;
    }
    for (int j = max(0, issued - 2); j < issued; ++j)
      if (!mbar_drain(&bar_mma[j & 1], ((unsigned)j >> 1) & 1u, tmo) && lane == 0)
        raise_error(ctrl, (int)PN_ERR_TIMEOUT);
  } else if (warp < C::WE0) {
    // =========================== look-back ==================================
    // warp 2 + j takes tiles j, j + NLB, ...; self-validating words, flags as hints
    if constexpr (kScan) {
      unsigned long long* aggw = reinterpret_cast<unsigned long long*>(P.agg);    // [tile][DP] x {A, B}
      unsigned long long* prefw = reinterpret_cast<unsigned long long*>(P.pref);  // [tile][DP]
      const unsigned tag = lookback_tag(epoch);
      for (int it = warp - 2;; it += C::NLB) {
        const int aslot = it % C::NAG;   // aggregate hand-off slot
        const int slot = it % NSLOT;     // carry slot
        const unsigned ph = (unsigned)(it / NSLOT) & 1u;
        if (!mbar_wait_flag(&bar_lb[aslot], (unsigned)(it / C::NAG) & 1u, ctrl, tmo, &s_abort, 107)) break;
        const int kg = s_lbtk[aslot];
        if (kg < 0) break;
        const int b = kg % B;
        const int chunk = kg / B;
        const size_t k = (size_t)kg;
        const bool stall = (A.stall_ticket == kg);
        float2 ag[C::NQ];
#pragma unroll
        for (int q = 0; q < C::NQ; ++q)
          ag[q] = *reinterpret_cast<const float2*>(sAgg + (aslot * DP + lane + 32 * q) * 2);
        // 1. the tile aggregate (the first chunk too: a successor may start from s0)
        if (!stall) {
#pragma unroll
          for (int q = 0; q < C::NQ; ++q)
            st_word2(aggw + (k * DP + lane + 32 * q) * 2, tag_word(ag[q].x, tag), tag_word(ag[q].y, tag));
          __syncwarp();
          if (lane == 0) st_relaxed(P.flags + k, make_flag(epoch, kFlagAgg));
        }
        // 2. the carry: nearest published state, then the aggregates in between
        int n_agg = lookback_nearest_state(P.flags, k, stride, chunk, epoch, ctrl, tmo);
        float carry[C::NQ];
#pragma unroll
        for (int q = 0; q < C::NQ; ++q) carry[q] = 0.0f;
        if (n_agg >= 0) {
          const bool from_s0 = chunk - 1 - n_agg < 0;
          if (from_s0) {
#pragma unroll
            for (int q = 0; q < C::NQ; ++q) {
              const int j = lane + 32 * q;
              carry[q] = (j < D) ? __ldg(A.s0 + (size_t)b * D + j) : 0.0f;
            }
          }
          if (!lookback_fold<DP, C::NQ, C::FB>(aggw, prefw, k, stride, n_agg, from_s0, tag, carry, ctrl, tmo)) n_agg = -1;
        }
        if (n_agg < 0) s_abort = 1;
        // 3. hand the carry to the epilogue (its slot is free once tile it - NSLOT was formed)
        if (it >= NSLOT && !mbar_wait_flag(&bar_cempty[slot], ph ^ 1u, ctrl, tmo, &s_abort, 108)) break;
#pragma unroll
        for (int q = 0; q < C::NQ; ++q) sCarry[slot * DP + lane + 32 * q] = carry[q];
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_cfull[slot]);
        // 4. the tile's end state
        if (n_agg >= 0 && !stall) {
#pragma unroll
          for (int q = 0; q < C::NQ; ++q)
            st_word(prefw + k * DP + lane + 32 * q, tag_word(fmaf(ag[q].x, carry[q], ag[q].y), tag));
          __syncwarp();
          if (lane == 0) st_relaxed(P.flags + k, make_flag(epoch, kFlagPrefix));
        }
      }
    }
  } else {
    // =========================== epilogue ===================================
    const int e = warp - C::WE0;            // 0 .. NEW-1
    const int quarter = warp & 3;           // TMEM lane quarter this warp may access
    const int rg = e >> 2;                  // 16-step group within the segment
    // TMEM lane quarter * 32 + lane = row m of accumulator half `half`
    const int m = 16 * quarter + (lane & 15);
    const int half = lane >> 4;
    const int c = m % DP;                   // channel
    const int g = half * C::NB + m / DP;    // step segment (differs between the lane halves)
    const int row0 = g * RS + 16 * rg;      // first step (tile row) of this thread
    const int piece = g * C::NRG + rg;
    // the warps holding the last piece (last step group of the last band of half 1)
    const bool lastw = (rg == C::NRG - 1) && ((16 * quarter) / DP == C::NB - 1);
    const int te = tid - 32 * C::WE0;       // 0 .. NTE-1 among the epilogue threads
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int hc = c >> 5;                  // column half of channel c in S
    const int cc = c & 31;                  // its column within the half
    const float wdc = sWd[c];

    // S_lo of stage `stg` (rows 0..L-1), swizzled like S.  For the first chunk of a
    // sequence, row 0 (step -1, loaded as zero) becomes s0 first.
    auto split = [&](int stg, int kgs) {
      constexpr int NU = NKH * L * 8 / NTE;   // 16-byte chunks per thread
      static_assert(NU * NTE == NKH * L * 8, "split covers the stage exactly");
      const bool first = (kgs / B) == 0;
      float4 v[NU];
#pragma unroll
      for (int k = 0; k < NU; ++k) {   // all loads first
        const int u = te + k * NTE;
        const int h = (u >> 3) / L;
        v[k] = *reinterpret_cast<const float4*>(sS + (stg * NKH + h) * C::SH_BYTES + sw128_offset((u >> 3) % L, 4 * (u & 7)));
      }
#pragma unroll
      for (int k = 0; k < NU; ++k) {
        const int u = te + k * NTE;
        const int r = (u >> 3) % L;
        const int h = (u >> 3) / L;
        const uint32_t off = sw128_offset(r, 4 * (u & 7));
        if (first && r == 0) {
          v[k] = __ldg(reinterpret_cast<const float4*>(A.s0 + (size_t)(kgs % B) * D + 32 * h) + (u & 7));
          *reinterpret_cast<float4*>(sS + (stg * NKH + h) * C::SH_BYTES + off) = v[k];
        }
        *reinterpret_cast<float4*>(sLo + h * C::LO_BYTES + off) =
            make_float4(tf32_tail(v[k].x), tf32_tail(v[k].y), tf32_tail(v[k].z), tf32_tail(v[k].w));
      }
      fence_async_smem();   // generic writes -> the tensor cores (async proxy)
    };

    // operands of the tile after `itn - 1`: wait for its stage, split it, publish its ticket
    // (the exit decision, read by everyone after the next named barrier) and wake the MMA warp
    auto prepare = [&](int itn) {
      const int stg = itn & 1;
      int kn = -1;
      if (mbar_wait_flag(&bar_sfull[stg], ((unsigned)itn >> 1) & 1u, ctrl, tmo, &s_abort, 109)) kn = s_tk[stg];
      if (kn >= 0 && !s_abort) split(stg, kn);
      __syncwarp();
      if (lane == 0) {
        if (te == 0) s_atk[itn & 1] = s_abort ? -1 : kn;
        mbar_arrive(&bar_afull);
      }
    };

    // s^(i+1) of tile j (ticket kj): piece carry from the look-back carry, then the parked
    // prefixes (the stash holds [A 0-7 | B 0-7 | A 8-15 | B 8-15] per 16 steps; B only for
    // Picard), stored eight steps at a time.  The rows are D = DP floats apart (the kernel runs
    // only with D == DP); steps past T are not stored.
    auto stage_out = [&](int j, float pa, float pb, int kj) {
      const int slot = j % NSLOT;
      mbar_wait_flag(&bar_cfull[slot], (unsigned)(j / NSLOT) & 1u, ctrl, tmo, &s_abort, 110);
      const float carry = sCarry[slot * DP + c];
      // Picard parks only B: its damped A_t = lambda enters here
      const float cp = kHasA ? fmaf(pa, carry, pb) : (carry + pb) * lambda;
      const uint32_t sbase = tmem + (uint32_t)(C::STASH0 + slot * C::SCOLS + (kHasA ? 32 : 16) * rg) + lane_off;
      const int tj = (kj / B) * L + row0;   // this thread's first step of tile j
      float* o = dst + ((size_t)(kj % B) * T + tj) * DP + c;
      const bool fullj = tj + 16 <= T;
#pragma unroll
      for (int h8 = 0; h8 < (kHasA ? 2 : 1); ++h8) {
        float v[16];   // quasi: A then B of steps 8 h8 .. 8 h8 + 7; Picard: B of all 16 steps
        tmem_ld16(sbase + (uint32_t)(16 * h8), v);
#pragma unroll
        for (int i = 0; i < (kHasA ? 8 : 16); ++i) {
          const int ii = (kHasA ? 8 * h8 : 0) + i;
          if (fullj || tj + ii < T) o[(size_t)ii * DP] = kHasA ? fmaf(v[i], cp, v[8 + i]) : cp + v[i];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_cempty[slot]);
    };

    // The loop's exit decision is one thread's reading of the next stage's ticket,
    // published before a named barrier, so every epilogue thread takes the same path.
    prepare(0);
    named_barrier(1, NTE);
    int kg = s_atk[0];
    int it = 0;
    int kg_m1 = -1, kg_m2 = -1, kg_m3 = -1;  // tickets of tiles it-1, it-2, it-3
    float pa1 = 1.0f, pb1 = 0.0f, pa2 = 1.0f, pb2 = 0.0f, pa3 = 1.0f, pb3 = 0.0f;   // their piece prefixes
    for (; kg >= 0; ++it) {
      const int st = it & 1;
      const int buf = it & 1;
      const int b = kg % B;
      const int t0 = (kg / B) * L;

      // ---- Z of this thread's channel and 16 steps, then cell + sequential scan
      mbar_wait_flag(&bar_mma[buf], ((unsigned)it >> 1) & 1u, ctrl, tmo, &s_abort, 111);
      tc_fence_after();
      float z[16];
      tmem_ld16(tmem + (uint32_t)(buf * RS + 16 * rg) + lane_off, z);
      mbar_wait_flag(&bar_xfull[st], ((unsigned)it >> 1) & 1u, ctrl, tmo, &s_abort, 112);
      // rows row0 .. row0 + 16 of the swizzled stage (row0 is a multiple of 16, so the swizzle
      // phase of row row0 + i is i mod 8): byte offset = 128 (row0 + i) + (cq ^ (i mod 8)) 16 + (cc mod 4) 4
      const unsigned char* Sh = sS + (st * NKH + hc) * C::SH_BYTES + row0 * 128 + (cc & 3) * 4;
      const uint32_t cq16 = (uint32_t)(cc >> 2) << 4;
      // step t0 + row0 - 1; for the first step of a sequence that is s0 (the stage's row 0
      // holds s0 only for the tensor cores)
      float sp = (t0 + row0 == 0) ? __ldg(A.s0 + (size_t)b * D + c) : *reinterpret_cast<const float*>(Sh + cq16);
      const bool full = (t0 + row0 + 16 <= T);   // no step of this thread lies past the sequence end
      const float* xr = sX + st * (L * DP) + row0 * DP + c;
      float SA = 1.0f, SB = 0.0f;
      float av[16], bv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = row0 + i;
        const float sc = *reinterpret_cast<const float*>(Sh + (i + 1) * 128 + (cq16 ^ (uint32_t)(((i + 1) & 7) << 4)));
        const float xv = xr[i * DP];
        float y, a, bb, res;
        if constexpr (CELL == PN_CELL_TANH_RNN) {
          y = tanh_pn(z[i] + xv);
          res = sc - y;
          a = (MODE == PN_QUASI) ? (1.0f - y * y) * wdc : (MODE == PN_PICARD ? 1.0f : 0.0f);
          bb = (MODE == PN_JACOBI) ? y : y - a * sp;
        } else {
          const float gg = tanh_pn(z[i] + xv);
          const float eg = P.eps * gg;
          y = sp + eg;
          res = (sc - sp) - eg;
          if (MODE == PN_QUASI) {
            const float ed = P.eps * (1.0f - gg * gg) * wdc;
            a = 1.0f + ed;
            bb = eg - ed * sp;
          } else if (MODE == PN_PICARD) {
            a = 1.0f;
            bb = eg;
          } else {
            a = 0.0f;
            bb = y;
          }
        }
        if (full || t0 + r < T) {
          rbits = max(rbits, abs_bits(res));
        } else {
          a = 1.0f;
          bb = 0.0f;
        }
        if constexpr (kHasA) {
          SB = fmaf(a, SB, bb);
          SA *= a;
        } else {
          SB += bb;   // Picard: a = 1; Jacobi: SB unused
        }
        av[i] = SA;
        bv[i] = (MODE == PN_JACOBI) ? bb : SB;
        if (damped) {
          av[i] *= lambda;
          bv[i] = fmaf(lambda, bv[i], (1.0f - lambda) * sc);
        }
        sp = sc;
      }
      // this tile's TMEM accumulator and its stage (S and step inputs) are consumed
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar_tempty[buf]);
        mbar_arrive(&bar_sempty[st]);
      }
      // the next tile's operands (S_lo is free: this tile's products are done)
      prepare(it + 1);


      if constexpr (!kScan) {
        if (!s_abort) {
          float* o = dst + ((size_t)b * T + t0 + row0) * D + c;
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (t0 + row0 + i < T) o[(size_t)i * D] = bv[i];
        }
        named_barrier(1, NTE);   // the ticket of tile it+1
        kg = s_atk[(it + 1) & 1];
      } else {
        // ---- combine the 8 pieces of each channel
        float* tot = sTot + (it & 1) * C::NPC * DP * 2;
        *reinterpret_cast<float2*>(tot + (piece * DP + c) * 2) = make_float2(SA, SB);
        named_barrier(1, NTE);   // piece totals, and the ticket of tile it+1
        const int kg_next = s_atk[(it + 1) & 1];
        float PA = 1.0f, PB = 0.0f;   // prefix of the earlier pieces
        {
          float2 w[C::NPC - 1];   // all loads in flight together
#pragma unroll
          for (int p = 0; p < C::NPC - 1; ++p) w[p] = *reinterpret_cast<const float2*>(tot + (p * DP + c) * 2);
#pragma unroll
          for (int p = 0; p < C::NPC - 1; ++p)
            if (p < piece) {
              PB = kHasA ? fmaf(w[p].x, PB, w[p].y) : PB + w[p].y;
              if (kHasA) PA *= w[p].x;
            }
        }
        // the last piece's inclusive prefix is the tile aggregate: hand it to the look-back
        const int aslot = it % C::NAG;
        if (lastw) {
          if (piece == C::NPC - 1)
            *reinterpret_cast<float2*>(sAgg + (aslot * DP + c) * 2) =
                kHasA ? make_float2(SA * PA, fmaf(SA, PB, SB)) : make_float2(1.0f, PB + SB);
          __syncwarp();
          if (lane == 0) {
            if (c == 0) s_lbtk[aslot] = s_abort ? -1 : kg;
            mbar_arrive(&bar_lb[aslot]);
          }
        }
        // the states of tile it-3 (its carry had three tiles of time to arrive); this frees the
        // stash slot this tile's prefixes take
        if (it >= C::DEFER) stage_out(it - C::DEFER, pa3, pb3, kg_m3);
        // ---- park the in-piece prefixes in TMEM
        {
          const uint32_t sbase =
              tmem + (uint32_t)(C::STASH0 + (it % NSLOT) * C::SCOLS + (kHasA ? 32 : 16) * rg) + lane_off;
          if constexpr (kHasA) tmem_st32_split8(sbase, av, bv);
          else tmem_st16(sbase, bv);
          tmem_st_wait();
        }
        pa3 = pa2;
        pb3 = pb2;
        pa2 = pa1;
        pb2 = pb1;
        pa1 = PA;
        pb1 = PB;
        kg_m3 = kg_m2;
        kg_m2 = kg_m1;
        kg_m1 = kg;
        kg = kg_next;
      }
    }
    if constexpr (kScan) {
      // the last three tiles' states (a loop, not unrolled: one copy of the write-out code
      // serves it, which keeps the epilogue's code smaller)
#pragma unroll 1
      for (int j = 0; j < C::DEFER; ++j) {
        const int tj = it + j - C::DEFER;
        const int kj = (j == 0) ? kg_m3 : (j == 1 ? kg_m2 : kg_m1);
        const float pa = (j == 0) ? pa3 : (j == 1 ? pa2 : pa1);
        const float pb = (j == 0) ? pb3 : (j == 1 ? pb2 : pb1);
        if (tj >= 0) stage_out(tj, pa, pb, kj);
      }
      // the next iteration reads these states with tensor copies (async proxy) after the grid barrier
      asm volatile("fence.proxy.async.global;" ::: "memory");
      // stop the look-back warps: their next tiles are it .. it + NLB - 1
      if (lastw && lane == 0) {
        for (int j = it; j < it + C::NLB; ++j) {
          if (c == 0) s_lbtk[j % C::NAG] = -1;
          mbar_arrive(&bar_lb[j % C::NAG]);
        }
      }
    }
  }

  // ---- residual of this iteration; next iteration or end of the launch ------
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
  // Set-up of the next iteration ahead of the grid barrier: fresh barriers (every operation on
  // the old ones has completed) and the first tile's step inputs, which every iteration reads.
  if (tid == 0) {
    inval_barriers();
    init_barriers();
    if (has_tile0) {
      const int kg = (int)blockIdx.x;
      mbar_arrive_expect_tx(&bar_xfull[0], (unsigned)C::X_BYTES);
      tma_load_3d_hint(smem_raw + C::OFF_X, P.tmaps + 2, 0, (kg / B) * L, kg % B, &bar_xfull[0],
                       l2_policy_evict_last());
    }
  }
  if (!finish_iteration(P, A, iter, epoch, s_last, (gen0 >> 1) + (unsigned)round, rmax)) {
    // no next iteration: the prefetched step inputs land before the CTA exits
    if (tid == 0 && has_tile0 && !mbar_drain(&bar_xfull[0], 0u, tmo)) raise_error(ctrl, (int)PN_ERR_TIMEOUT);
    break;
  }
  }   // iterations

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    tmem_dealloc(s_tmem, (uint32_t)C::ALLOC_COLS);
  if (!P.persist) finish_launch(P, A, epoch, s_last);
}

}  // namespace pn
