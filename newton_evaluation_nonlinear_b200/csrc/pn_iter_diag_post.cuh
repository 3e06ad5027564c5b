// pn_iter_diag_post.cuh -- the Jacobi, Picard and diagonal quasi-Newton
// iteration of the wide one-gate cells (tanh RNN, Euler drift at D = 128,
// 256) once the tensor cores have formed every step's recurrent product.
//
// Same iteration as pn_iter_diag.cuh (the page's unified update, "Parallel
// Newton methods..." page §1.2, with a diagonal A~_t, §2.2.1 / §2.2.3, solved
// as the chunked scan of §2.1).  With Y = S W^T computed for every step by
// wide_gemm_kernel (row b T + t - 1 holds W s^(i)_{t-1} for step t), all that
// is left of an iteration is per channel: the cell, the diagonal Jacobian,
// the residual, and a scalar affine recurrence s_t = a_t s_{t-1} + b_t.
//
// A tile is (sequence b, chunk of L steps, group of G channels); two threads
// own one channel of a tile, each half of its steps.  The scan runs in three
// phases over all tiles, with a bounded grid barrier between them (the launch
// is cooperative), so that no tile ever waits on another's result:
//   1. each thread walks its half of a tile's steps and composes them into an
//      aggregate (A, B); the pair combines its halves through shared memory
//      and stores the tile's aggregate and its first half's;
//   2. per (sequence, channel group), one thread per channel folds the tile
//      aggregates of the chunks in order from s0 and stores each tile's carry
//      (the state just before the tile);
//   3. each thread walks its half again from its carry (the second half's is
//      the first half's aggregate applied to the tile's) and stores s^(i+1).
// Jacobi needs no scan: phase 1 stores its states and the launch ends there.
// A producer warp streams every tile's rows (Y, step inputs, s^(i)) into a
// two-stage shared-memory ring with three TMA tensor loads, phase 3's first
// tiles during the barriers (they read nothing phases 1 and 2 write).  Step 0
// of a sequence forms W s0 itself (from the dense weight copy, W[c][k] at
// k DP + c).
#pragma once

#include "pn_iter_diag_tc.cuh"

namespace pn {

template <int CELL, int MODE, int DP>
struct PostCfg {
  static constexpr int G = DP < 128 ? DP : 128;   // channels per tile
  static constexpr int NH = 2;                    // threads per channel (halves of the steps)
  static constexpr int NTC = NH * G;              // consumer threads
  static constexpr int NCW = NTC / 32;            // consumer warps
  static constexpr int NT = NTC + 32;             // + one producer warp
  static constexpr int L = 32;                    // steps per tile
  static constexpr int LH = L / NH;               // steps per thread
  static constexpr int NS = 2;                    // shared-memory stages
  static constexpr int FB = 16;                   // aggregates loaded together in phase 2
  static constexpr int STAGE_FLOATS = (3 * L + 1) * G;   // rows: Y [L], x [L], s^(i) [L + 1]
  static constexpr size_t SMEM_BYTES = (size_t)NS * STAGE_FLOATS * 4 + 128;   // + slack to align the stages
  static_assert(CellInfo<CELL>::R == 1, "one-gate cells");
  static_assert(DP % G == 0 && G % 32 == 0 && L % NH == 0, "tile shape");
  static_assert((G * 4) % 16 == 0 && (STAGE_FLOATS * 4) % 128 == 0, "TMA boxes: 16-byte rows, 128-byte aligned");
};

// Bounded barrier of all CTAs of a cooperative launch (all threads call it).  The generation is
// read before arriving: it changes only once every CTA has arrived, and the last one resets the
// count before it releases the next generation.  `arrive` = false makes this CTA wait without
// arriving (a test hook: the others then run out their wait).  Returns false, on every thread,
// when the wait gave up (the error is raised).
__device__ __forceinline__ bool grid_sync(Ctrl* c, long long timeout_ns, bool arrive, int& flag_smem) {
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned g = *(volatile unsigned*)&c->sync_gen;
    int ok = 1;
    __threadfence();
    if (arrive && atomicAdd(&c->sync_count, 1u) == gridDim.x - 1) {
      c->sync_count = 0u;
      __threadfence();
      st_release(&c->sync_gen, g + 1u);
    } else {
      const unsigned long long t0 = globaltimer();
      unsigned spins = 0;
      while (ld_acquire(&c->sync_gen) == g) {
        if (((++spins) & 15u) == 0u && (ld_volatile(&c->error) || (long long)(globaltimer() - t0) > timeout_ns)) {
          raise_error(c, (int)PN_ERR_TIMEOUT);
          ok = 0;
          break;
        }
        if (spins > 64u) __nanosleep(64);
      }
    }
    flag_smem = ok;
  }
  __syncthreads();
  return flag_smem != 0;
}

template <int CELL, int MODE, int DP>
__global__ void __launch_bounds__(PostCfg<CELL, MODE, DP>::NT, 2) diag_post_kernel(const IterParams P) {
  using C = PostCfg<CELL, MODE, DP>;
  constexpr int G = C::G;
  constexpr int L = C::L;
  constexpr int NS = C::NS;
  constexpr int NT = C::NT;
  constexpr bool kScan = (MODE != PN_JACOBI);
  constexpr bool kHasA = (MODE == PN_QUASI);
  // undamped Euler Picard forms its states from Y and the step inputs alone (b_t = eps g_t, the
  // residual was taken in phase 1), so phase 3 does not load s^(i)
  constexpr bool kEulerPicard = (CELL == PN_CELL_EULER_TANH && MODE == PN_PICARD);
  extern __shared__ __align__(128) unsigned char smem_post_raw[];
  float* smem_post = reinterpret_cast<float*>(smem_post_raw + ((128u - (smem_addr(smem_post_raw) & 127u)) & 127u));
  __shared__ __align__(8) uint64_t bar_full[NS], bar_empty[NS];
  __shared__ int s_last, s_sync;
  __shared__ float sRed[NT / 32];
  __shared__ float2 sHalf[2 * C::NTC];   // phase 1: the halves' aggregates, by unit parity
  __shared__ volatile int s_stop;        // phase 1: a consumer warp's wait gave up

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  Ctrl* ctrl = P.ctrl;
  const Args A = *P.args;
  const int D = P.D, T = P.T, B = P.B;
  const int ng = P.ngroups;
  const int nchunks = P.nchunks;
  const int ntiles = ng * B * nchunks;   // tile j = (chunk B + b) ng + g
  const float lambda = A.damping;        // s^(i+1) = s^(i) + lambda * delta
  const bool damped = lambda != 1.0f;
  const long long tmo = A.timeout_ns;

  if (tid == 0) {
    atomicMin(&ctrl->t_start, globaltimer());
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar_full[s], 1u);
      mbar_init(&bar_empty[s], (unsigned)C::NCW);
    }
    mbar_init_fence();
    s_stop = 0;
  }
  __syncthreads();
  const unsigned epoch = *(volatile unsigned*)&ctrl->epoch;
  const int iter = *(volatile int*)&ctrl->iter;
  float* __restrict__ dst = (iter & 1) ? A.states : P.buf1;   // s^(i+1); s^(i) and the inputs come by TMA
  unsigned rbits = 0u;

  // this CTA's tiles, blockIdx.x + r gridDim.x: phase 1 takes them as units 0 .. n1-1, phase 3 as
  // units n1 .. 2 n1 - 1; unit u fills stage u % NS
  const int n1 = (ntiles > (int)blockIdx.x) ? (ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int nunits = kScan ? 2 * n1 : n1;
  struct Tile {
    int g, b, t0, n;
    size_t row0;   // row b T + t0 of step t0
  };
  auto tile_of = [&](int u) -> Tile {
    const int j = (int)blockIdx.x + (u % max(n1, 1)) * (int)gridDim.x;
    Tile t;
    t.g = j % ng;
    const int kg = j / ng;
    t.b = kg % B;
    t.t0 = (kg / B) * L;
    t.n = min(L, T - t.t0);
    t.row0 = (size_t)t.b * T + t.t0;
    return t;
  };
  auto tile_index = [&](int u) { return (int)blockIdx.x + (u % max(n1, 1)) * (int)gridDim.x; };
  const bool stall = A.stall_ticket >= 0 && A.stall_ticket < ntiles && (A.stall_ticket % (int)gridDim.x) == (int)blockIdx.x;

  // the cell, the diagonal Jacobian a_t, b_t = y_t - a_t s_{t-1} and F_t of a step: (a, b, F)
  auto coef = [&](float z, float x, float sc, float sp, float wdc) -> float3 {
    float a, bb, res;
    if constexpr (CELL == PN_CELL_TANH_RNN) {
      const float y = tanh_pn(z + x);
      res = sc - y;
      a = (MODE == PN_QUASI) ? (1.0f - y * y) * wdc : (MODE == PN_PICARD ? 1.0f : 0.0f);
      bb = (MODE == PN_JACOBI) ? y : y - a * sp;
    } else {
      const float gg = tanh_pn(z + x);
      const float eg = P.eps * gg;
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
        bb = sp + eg;
      }
    }
    return make_float3(a, bb, res);
  };

  // ---- producer: unit u is three tensor loads into stage u % NS, each G channels of one sequence:
  // Y of steps t0 .. t0+L-1, the step inputs of the same steps, and s^(i) of steps t0-1 .. t0+L-1
  // (steps outside 0 .. T-1 read as zero and are not used).  All streamed with the evict-first
  // hint: marking phase 1's tiles to stay in L2 for phase 3 measured slower.  Returns false
  // (warp-uniform) when the wait for the stage gave up.
  const bool producer = (warp == C::NCW);
  const CUtensorMap* mY = P.tmaps;
  const CUtensorMap* mX = P.tmaps + 1;
  const CUtensorMap* mS = P.tmaps + ((iter & 1) ? 3 : 2);
  if (producer && lane == 0) {
    tmap_acquire(mY);
    tmap_acquire(mX);
    tmap_acquire(mS);
    asm volatile("fence.proxy.async.global;" ::: "memory");   // s^(i) written by an earlier kernel
  }
  int issued = 0;
  auto issue = [&](int u) -> bool {
    const int s = u % NS;
    int ok = 1;
    if (lane == 0) {
      if (u >= NS) ok = mbar_wait(&bar_empty[s], (unsigned)((u / NS) - 1) & 1u, ctrl, tmo) ? 1 : 0;
      if (ok) {
        const Tile t = tile_of(u);
        const uint64_t pol = l2_policy_evict_first();
        float* st = smem_post + (size_t)s * C::STAGE_FLOATS;
        const int col = t.g * G;
        const bool with_s = !(kEulerPicard && !damped && u >= n1);
        mbar_arrive_expect_tx(&bar_full[s], (unsigned)((with_s ? C::STAGE_FLOATS : 2 * L * G) * 4));
        tma_load_3d_hint(st, mY, col, t.t0 - 1, t.b, &bar_full[s], pol);
        tma_load_3d_hint(st + L * G, mX, col, t.t0, t.b, &bar_full[s], pol);
        if (with_s) tma_load_3d_hint(st + 2 * L * G, mS, col, t.t0 - 1, t.b, &bar_full[s], pol);
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok) issued = u + 1;
    return ok != 0;
  };

  // ---- consumers: thread (h, cl) owns channel g G + cl and steps h LH .. h LH + LH - 1 of a tile.
  // One walk over its steps of unit u from the unit's stage.  Phase 1 (apply = false): the residual
  // and the aggregate (A, B) of the steps, returned; Jacobi stores its states here.  Phase 3
  // (apply = true): the states from the carry s, stored.  Returns false (warp-uniform) without
  // touching the stage when the wait for it gave up.
  const int h = tid / G;
  const int cl = tid % G;
  auto walk = [&](int u, bool apply, float s, float2& agg) -> bool {
    const Tile t = tile_of(u);
    const int st = u % NS;
    const int c = t.g * G + cl;
    const bool cok = c < D;
    const int m0 = h * C::LH;
    const float wdc = (kHasA && cok) ? __ldg(P.wdiag + c) : 0.0f;
    // W s0 for the first step of a sequence (before the wait: its loads overlap the copies)
    float z0 = 0.0f, s0c = 0.0f;
    if (t.t0 == 0 && m0 == 0 && cok) {
      const float* s0 = A.s0 + (size_t)t.b * D;
      s0c = __ldg(s0 + c);
      for (int kk = 0; kk < D; ++kk) z0 = fmaf(__ldg(P.wt + (size_t)kk * DP + c), __ldg(s0 + kk), z0);
    }
    int ok = 1;
    if (lane == 0) ok = mbar_wait(&bar_full[st], (unsigned)(u / NS) & 1u, ctrl, tmo) ? 1 : 0;
    if (!__shfl_sync(0xffffffffu, ok, 0)) return false;
    const float* sY = smem_post + (size_t)st * C::STAGE_FLOATS + m0 * G + cl;   // row m0 of Y
    const float* sX = sY + L * G;
    const float* sS = sY + 2 * L * G;                                            // row m0: step t0 + m0 - 1
    float* orow = dst + (t.row0 + m0) * DP + c;
    float sp = (t.t0 + m0 == 0) ? s0c : ((kEulerPicard && apply && !damped) ? 0.0f : sS[0]);
    float SA = 1.0f, SB = 0.0f;
    const bool no_s = kEulerPicard && apply && !damped;   // phase 3 loaded no s^(i) (see the producer)
    auto step = [&](int i) {
      const float z = (t.t0 + m0 + i > 0) ? sY[i * G] : z0;
      const float sc = no_s ? 0.0f : sS[(i + 1) * G];
      const float3 f = coef(z, sX[i * G], sc, sp, wdc);
      sp = sc;
      if (!apply) {
        rbits = max(rbits, abs_bits(f.z));
        if constexpr (!kScan) {
          orow[(size_t)i * DP] = damped ? fmaf(lambda, f.y - sc, sc) : f.y;
        } else {
          SB = fmaf(f.x, SB, f.y);
          if (kHasA) SA *= f.x;
        }
      } else {
        s = fmaf(f.x, s, f.y);
        orow[(size_t)i * DP] = damped ? fmaf(lambda, s - sc, sc) : s;
      }
    };
    if (cok) {
      if (m0 + C::LH <= t.n) {   // every step of the half lies before T: no guards
#pragma unroll
        for (int i = 0; i < C::LH; ++i) step(i);
      } else {
        for (int i = 0; i < C::LH && m0 + i < t.n; ++i) step(i);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bar_empty[st]);   // this warp has read the stage
    agg = make_float2(SA, SB);
    return true;
  };

  // ---- phase 1: aggregates (Jacobi: the states); the two halves of a channel meet in sHalf,
  // double-buffered by the unit's parity so that the next unit's writes never meet this one's reads
  bool go = true;
  if (producer) {
    for (int u = 0; u < n1 && go; ++u) go = issue(u);
    // phase 3 reads nothing phases 1 and 2 write: its first stages are fetched now (their stages are
    // freed by phase-1 tiles, which the consumers finish before the barrier)
    if (kScan)
      for (int u = n1; u < min(nunits, n1 + NS) && go; ++u) go = issue(u);
  } else {
    for (int u = 0; u < n1 && go; ++u) {
      float2 ag = make_float2(1.0f, 0.0f);
      go = walk(u, false, 0.0f, ag);
      if (!kScan) continue;
      // every consumer warp meets the barrier, also one whose wait gave up; all of them then leave
      // together if any did
      if (!go) s_stop = 1;
      sHalf[(u & 1) * C::NTC + tid] = ag;
      named_barrier(1, C::NTC);
      go = (s_stop == 0);
      if (!go) break;
      float2* out = reinterpret_cast<float2*>(P.agg + (size_t)tile_index(u) * P.agg_stride);
      if (h == 0) {   // the tile: second half after the first
        const float2 a1 = sHalf[(u & 1) * C::NTC + G + cl];
        out[cl] = make_float2(a1.x * ag.x, fmaf(a1.x, ag.y, a1.y));
      } else {        // the first half's, for the second half's carry in phase 3
        out[G + cl] = sHalf[(u & 1) * C::NTC + cl];
      }
    }
  }
  if constexpr (kScan) {
    // ---- phase 2: the carry into every tile, per (sequence, channel group), chunks in order
    bool ok = grid_sync(ctrl, tmo, !stall, s_sync);
    if (ok && !producer && h == 0) {
      for (int q = blockIdx.x; q < B * ng; q += gridDim.x) {
        const int b = q / ng;
        const int g = q % ng;
        const int c = g * G + cl;
        float carry = (c < D) ? __ldg(A.s0 + (size_t)b * D + c) : 0.0f;
        for (int k0 = 0; k0 < nchunks; k0 += C::FB) {
          float2 ab[C::FB];
#pragma unroll
          for (int v = 0; v < C::FB; ++v) {
            const size_t j = (size_t)((k0 + v) * B + b) * ng + g;
            ab[v] = (k0 + v < nchunks) ? __ldcg(reinterpret_cast<const float2*>(P.agg + j * P.agg_stride) + cl)
                                       : make_float2(1.0f, 0.0f);
          }
#pragma unroll
          for (int v = 0; v < C::FB; ++v) {
            const size_t j = (size_t)((k0 + v) * B + b) * ng + g;
            if (k0 + v < nchunks) P.pref[j * P.pref_stride + cl] = carry;
            carry = fmaf(ab[v].x, carry, ab[v].y);
          }
        }
      }
    }
    if (ok) ok = grid_sync(ctrl, tmo, true, s_sync);
    // ---- phase 3: the states
    if (ok && producer) {
      for (int u = n1 + NS; u < nunits && go; ++u) go = issue(u);
    } else if (ok) {
      for (int u = n1; u < nunits && go; ++u) {
        const size_t j = (size_t)tile_index(u);
        float carry = __ldcg(P.pref + j * P.pref_stride + cl);
        if (h == 1) {
          const float2 a0 = __ldcg(reinterpret_cast<const float2*>(P.agg + j * P.agg_stride) + G + cl);
          carry = fmaf(a0.x, carry, a0.y);
        }
        float2 unused;
        go = walk(u, true, carry, unused);
      }
    }
  }
  // every issued copy lands before the CTA moves on
  if (producer && lane == 0)
    for (int u = max(0, issued - NS); u < issued; ++u)
      if (!mbar_drain(&bar_full[u % NS], (unsigned)(u / NS) & 1u, tmo)) raise_error(ctrl, (int)PN_ERR_TIMEOUT);
  __syncwarp();

  // ---- one atomicMax per CTA, then the end-of-launch decision
  rbits = warp_max_u32(rbits);
  if (lane == 0) sRed[warp] = __uint_as_float(rbits);
  __syncthreads();
  if (tid == 0) {
    unsigned v = 0u;
    for (int w = 0; w < NT / 32; ++w) v = max(v, __float_as_uint(sRed[w]));
    if (v) atomicMax(&ctrl->resid_bits, v);
  }
  finish_launch(P, A, epoch, s_last);
}

}  // namespace pn
