// pn_common.cuh -- shared device-side definitions of libpn (sm_100a).
//
// Control block, kernel parameter blocks, memory-ordering helpers for the
// single-pass chunked scan with decoupled look-back, and bounded waits.
#pragma once

#include <cuda.h>   // CUtensorMap (type only)
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pn.h"

namespace pn {

constexpr int kRunning = 100;          // ctrl.status while a loop is in flight
constexpr int kHistCap = 65537;        // residual history entries kept per handle
constexpr unsigned kFlagAgg = 1u;      // tile published its aggregate
constexpr unsigned kFlagPrefix = 2u;   // tile published its inclusive prefix (a state)
constexpr int kMaxGroups = 8;          // channel groups of the diagonal-family kernels (D / G)
constexpr int kTcMaps = 5;             // TMA tensor maps of the tensor-core kernels
constexpr int kWideMaps = 9;           // TMA tensor maps of the wide product and its per-channel kernel
constexpr int kProjMaps = 5;           // TMA tensor maps of the input projection

// Device control block: one per handle, in device memory.
struct Ctrl {
  // read at launch or iteration start, written by one thread
  int iter;            // index i of the iterate s^(i) the next launch evaluates
  int status;          // kRunning, or the final pn_status of the loop
  int final_iter;      // iteration count of the result
  float final_resid;   // r^(final_iter)
  unsigned epoch;      // launch sequence number; tags the look-back flags
  int timeout_ticket;  // ticket whose wait gave up (diagnostics), -1 if none
  unsigned long long t_start;    // min %globaltimer at CTA entry, current launch
  unsigned long long kernel_ns;  // summed launch durations
  unsigned long long launches;   // iterations run by the fused iteration kernels
  // reduced-precision storage: 1 when s^(iter) (fmt_in) / s^(iter+1) (fmt_out) is stored in the
  // narrow format Args::store_fmt, 0 for float32; final_fmt is fmt_in of the result s^(final_iter)
  int fmt_in;
  int fmt_out;
  int final_fmt;
  // adaptive switching on the device: the mode the current iteration runs in, and whether this
  // iteration is already the re-run of a stalled one
  int cur_mode;
  int retried;
  // The words below are hot and each sits in a 128-byte line of its own, so that
  // the ticket atomics do not queue behind the polls of the error word.
  alignas(128) int error;        // sticky device error (PN_ERR_TIMEOUT), 0 if none; polled by waiting warps
  alignas(128) unsigned ticket[kMaxGroups];  // tile tickets handed out per channel group, current launch
  alignas(128) unsigned resid_bits;  // running max of |F| for the current launch (float bits)
  unsigned done;       // CTAs finished in the current launch
  unsigned gen;        // grid barrier of the looping kernels: (iterations completed << 1) | (another follows)
  // Arrivals at the grid barrier of the looping kernels, with the stop rule's inputs packed in
  // (kArrive* below), and their residual maxima by iteration parity.
  alignas(128) unsigned long long arrive;
  unsigned resid_loop[2];
  // plain grid barrier inside one cooperative launch (the phases of the wide per-channel kernel)
  alignas(128) unsigned sync_count;
  unsigned sync_gen;
};

// Fields of Ctrl::arrive, each a count of CTAs (at most 2^20 - 1): arrived, with a residual
// above tol (or NaN), with a non-finite residual; the top field counts raised errors.
constexpr unsigned long long kArriveOne = 1ull;
constexpr unsigned long long kArriveHot = 1ull << 20;
constexpr unsigned long long kArriveBad = 1ull << 40;
constexpr unsigned long long kArriveErr = 1ull << 60;
constexpr unsigned long long kArriveMask = (1ull << 20) - 1ull;

// Sets the sticky device error unless one is set already; the first raise also counts itself in
// Ctrl::arrive, so the grid barrier's last arrival learns of it from the value its own atomic
// returns (the raising CTA arrives only after the raise).  Returns whether this call set it.
__device__ __forceinline__ bool raise_error(Ctrl* c, int code) {
  if (atomicCAS(&c->error, 0, code) != 0) return false;
  atomicAdd(&c->arrive, kArriveErr);
  return true;
}

// Per-call arguments, written by the host before each evaluation.
struct Args {
  const float* x;      // caller x [B][T][d_in]
  const float* s0;     // caller s0 [B][D]
  float* states;       // caller states [B][T][D] (iterate buffer 0)
  float tol;
  int max_iters;
  long long timeout_ns;
  int stall_ticket;    // -1 = off
  int use_cond;        // 1 inside the device loop graph
  int newton_band;     // Newton mode: < 0 the exact Jacobian; k >= 0 its entries with |row - col| <= k only
  float damping;       // lambda of s^(i+1) = s^(i) + lambda * delta (1 = undamped)
  int store_fmt;       // iterate storage: 0 float32, 1 bfloat16, 2 float16 (PN_STORE_*)
  float store_until;   // narrow storage while the residual known at an update's start is above this
  int adapt;           // 1: adaptive switching decided on the device (graph with one IF node per mode)
  float stall;         // switch when r^(i) > stall * r^(i-1)
  int mode_ok;         // bit m set when mode m has a kernel (the ladder skips the others)
  int start_mode;      // the evaluation's first mode
};

// Fixed per-handle parameters of the fused iteration kernels.
struct IterParams {
  const float* wt;     // recurrent weights, pre-packed per group: [ngroups][DP][R*G]
  const float* wt_tc;  // W_q rows split for the tensor cores: [W_hi; W_lo], K-major core-matrix layout
  const float* ypre;   // wide states: W s^(i)_r for every row r = b T + t, from the tensor cores
  const float* wdiag;  // diagonal entries per gate: [R][DP] (quasi mode)
  const float* bhn;    // GRU b_hn [DP] (zero-padded); unused otherwise
  const float* xin;    // per-step cell input: u [B][T][D] (tanh), gx [B][T][3D] (GRU); NULL for Euler
  float* buf1;         // iterate buffer 1 [B][T][D]
  unsigned* flags;     // look-back flags, one per tile
  float* agg;          // look-back aggregates, agg_stride floats per tile
  float* pref;         // look-back inclusive prefixes (states), pref_stride floats per tile
  Ctrl* ctrl;
  Args* args;
  float* hist;         // residual history [kHistCap]
  const CUtensorMap* tmaps;  // tensor-core kernels: [0]/[1] s^(i) loads from iterate buffer 0 (states) / 1,
                             // [2] step-input loads, [3]/[4] state stores into buffer 0 / 1
  float eps;           // Euler step
  int D, d_in, T, B;
  int ngroups, nchunks;
  int tiles_per_group;  // B * nchunks: tickets of one channel group
  int agg_stride, pref_stride;
  int persist;          // looping kernels: 1 = run iterations until the stop rule, 0 = one iteration
  int run;              // chunks of L steps per ticket (a run; 1 for the kernels that take single chunks)
  int tc;               // 1: the Newton kernel's D = 16 chunk chain on the tensor cores (PN_OPT_TENSOR_CORES)
  cudaGraphConditionalHandle cond;
  cudaGraphConditionalHandle mode_cond[4];   // adaptive graph: the IF node of each mode
  int* mode_hist;       // adaptive: the mode of each kept update [kHistCap]
};

// ---------------------------------------------------------------------------
// memory ordering
// ---------------------------------------------------------------------------
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned ld_relaxed(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// With a preceding relaxed load that observed a release store, this fence
// makes the later loads of this thread see what the releasing thread wrote.
__device__ __forceinline__ void fence_acquire_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void st_relaxed(unsigned* p, unsigned v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_volatile(const int* p) { return *(const volatile int*)p; }

// Self-validating look-back words: a float value in the low 32 bits and the
// launch epoch in the high 32 bits of one aligned 64-bit word.  A 64-bit
// access is single-copy atomic, so a reader that sees the expected epoch sees
// the value written with it; no fence is needed on either side.
__device__ __forceinline__ unsigned long long tag_word(float v, unsigned tag) {
  return ((unsigned long long)tag << 32) | (unsigned long long)__float_as_uint(v);
}
__device__ __forceinline__ float word_value(unsigned long long w) { return __uint_as_float((unsigned)w); }
__device__ __forceinline__ bool word_tagged(unsigned long long w, unsigned tag) { return (unsigned)(w >> 32) == tag; }
__device__ __forceinline__ void st_word(unsigned long long* p, unsigned long long w) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ void st_word2(unsigned long long* p, unsigned long long w0, unsigned long long w1) {
  asm volatile("st.relaxed.gpu.global.v2.u64 [%0], {%1, %2};" ::"l"(p), "l"(w0), "l"(w1) : "memory");
}
__device__ __forceinline__ unsigned long long ld_word(const unsigned long long* p) {
  unsigned long long w;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
  return w;
}
__device__ __forceinline__ void ld_word2(const unsigned long long* p, unsigned long long& w0, unsigned long long& w1) {
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(w0), "=l"(w1) : "l"(p) : "memory");
}
__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Look-back, phase A (called by all 32 lanes of one warp).
// The tile at chunk `chunk` of a scan chain looks at its predecessors
// chunk-1, chunk-2, ... (flag index k - d*stride for distance d) 32 at a time,
// one lane per predecessor, until it finds the nearest one that has published
// its inclusive prefix; chunk -1 counts as a published prefix (the state s0).
// It waits (bounded) until every predecessor nearer than that one has at least
// published its aggregate.  Returns the number of aggregate-only tiles between
// this tile and that prefix, or -1 when it gave up (timeout, or another CTA's
// error).  Flags are polled with relaxed loads; with `acquire`, one fence
// after the final poll gives the caller's subsequent loads of the aggregates
// and the prefix acquire semantics (flags published with a release store).
// Without it the flags are hints and the caller validates the data itself.
__device__ __forceinline__ int lookback_find_prefix(const unsigned* flags, size_t k, size_t stride,
                                                    int chunk, unsigned epoch, Ctrl* ctrl,
                                                    long long timeout_ns, bool acquire = true) {
  const int lane = threadIdx.x & 31;
  int n_agg = 0;
  int base = chunk - 1;   // nearest chunk of this window
  const unsigned long long t0 = globaltimer();
  unsigned spins = 0;
  while (true) {
    const int p = base - lane;
    bool valid = true, pfx = true;
    if (p >= 0) {
      const unsigned f = ld_relaxed(flags + (k - (size_t)(chunk - p) * stride));
      valid = ((f >> 2) == epoch) && (f & 3u);
      pfx = valid && ((f & 3u) == kFlagPrefix);
    }
    const unsigned pm = __ballot_sync(0xffffffffu, pfx);
    const unsigned vm = __ballot_sync(0xffffffffu, valid);
    const int nearest = pm ? (__ffs(pm) - 1) : 32;
    const unsigned need = (nearest >= 31) ? 0xffffffffu : ((2u << nearest) - 1u);
    if ((vm & need) == need) {
      if (nearest < 32) {
        if (acquire) fence_acquire_gpu();
        return n_agg + nearest;
      }
      n_agg += 32;
      base -= 32;
      continue;
    }
    ++spins;
    if ((spins & 15u) == 0u) {
      int give_up = 0;
      if (lane == 0) {
        if (ld_volatile(&ctrl->error)) give_up = 1;
        else if ((long long)(globaltimer() - t0) > timeout_ns) {
          if (raise_error(ctrl, (int)PN_ERR_TIMEOUT)) ctrl->timeout_ticket = (int)k;
          give_up = 1;
        }
      }
      if (__shfl_sync(0xffffffffu, give_up, 0)) return -1;
    }
    if (spins > 64u) __nanosleep(32);
  }
}

// Look-back for self-validating data (called by all 32 lanes of one warp):
// the distance to the nearest predecessor whose flag says it published its
// state, as the number n of tiles in between (chunk -1 = s0 counts as
// published).  Unlike lookback_find_prefix it does not wait for the flags of
// the n tiles in between: the caller waits on their tagged aggregate words
// directly, which saves a round trip.  The window moves on only when all of
// its 32 tiles have at least flagged an aggregate.  Returns -1 when it gave up.
__device__ __forceinline__ int lookback_nearest_state(const unsigned* flags, size_t k, size_t stride, int chunk,
                                                      unsigned epoch, Ctrl* ctrl, long long timeout_ns) {
  const int lane = threadIdx.x & 31;
  int n_agg = 0;
  int base = chunk - 1;
  const unsigned long long t0 = globaltimer();
  unsigned spins = 0;
  while (true) {
    const int p = base - lane;
    bool valid = true, pfx = true;
    if (p >= 0) {
      const unsigned f = ld_relaxed(flags + (k - (size_t)(chunk - p) * stride));
      valid = ((f >> 2) == epoch) && (f & 3u);
      pfx = valid && ((f & 3u) == kFlagPrefix);
    }
    const unsigned pm = __ballot_sync(0xffffffffu, pfx);
    if (pm) return n_agg + (__ffs(pm) - 1);
    if (__ballot_sync(0xffffffffu, valid) == 0xffffffffu) {
      n_agg += 32;
      base -= 32;
      continue;
    }
    ++spins;
    if ((spins & 15u) == 0u) {
      int give_up = 0;
      if (lane == 0) {
        if (ld_volatile(&ctrl->error)) give_up = 1;
        else if ((long long)(globaltimer() - t0) > timeout_ns) {
          if (raise_error(ctrl, (int)PN_ERR_TIMEOUT)) ctrl->timeout_ticket = (int)k;
          give_up = 1;
        }
      }
      if (__shfl_sync(0xffffffffu, give_up, 0)) return -1;
    }
    if (spins > 64u) __nanosleep(32);
  }
}

// Iterate storage: element idx of an iterate buffer in format fmt (0 float32, 1 bfloat16, 2 float16).
// A narrow iterate occupies the first half of its float32 buffer.  Stores round to nearest, ties to
// even (float16: overflow to infinity, gradual underflow).
__device__ __forceinline__ float ld_state(const void* base, size_t idx, int fmt) {
  if (fmt == 0) return __ldg(reinterpret_cast<const float*>(base) + idx);
  const unsigned short h = __ldg(reinterpret_cast<const unsigned short*>(base) + idx);
  return fmt == 1 ? __uint_as_float((unsigned)h << 16) : __half2float(__ushort_as_half(h));
}
__device__ __forceinline__ void st_state(void* base, size_t idx, float v, int fmt) {
  if (fmt == 0) reinterpret_cast<float*>(base)[idx] = v;
  else if (fmt == 1) reinterpret_cast<__nv_bfloat16*>(base)[idx] = __float2bfloat16_rn(v);
  else reinterpret_cast<__half*>(base)[idx] = __float2half_rn(v);
}
// The storage formats of the iteration a launch runs: of its input s^(i) and its output s^(i+1).
__device__ __forceinline__ int2 iter_formats(const Ctrl* c, const Args& A) {
  const int fi = *(const volatile int*)&c->fmt_in;
  const int fo = *(const volatile int*)&c->fmt_out;
  return make_int2(fi ? A.store_fmt : 0, fo ? A.store_fmt : 0);
}

__device__ __forceinline__ unsigned make_flag(unsigned epoch, unsigned state) {
  return (epoch << 2) | state;
}

// |F| values are >= 0, so their float bits order like unsigned integers, and
// NaN (0x7fc00000 and up) compares above +Inf: an integer max propagates NaN.
__device__ __forceinline__ unsigned abs_bits(float v) { return __float_as_uint(fabsf(v)); }

__device__ __forceinline__ unsigned warp_max_u32(unsigned v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Activations from the exponential identities, on the SFU's approximate base-2
// exponential and reciprocal (ex2.approx / rcp.approx, both within 2 ulp):
//   tanh(v) = 1 - 2 / (exp(2v) + 1),   sigmoid(v) = 1 / (1 + exp(-v)).
// Absolute error below 4e-7 over all finite v (the identity loses relative
// accuracy only where |tanh v| is tiny, never absolute accuracy); saturates
// to +-1 / 0 / 1 for large |v|.  A GPU test bounds it against CUDA's tanhf.
__device__ __forceinline__ float ex2_approx(float v) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ float rcp_approx(float v) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ float tanh_pn(float v) {
  const float e = ex2_approx(v * 2.8853900817779268f);   // 2 / ln 2
  return fmaf(-2.0f, rcp_approx(e + 1.0f), 1.0f);
}
__device__ __forceinline__ float sigmoid_pn(float v) {
  return rcp_approx(1.0f + ex2_approx(v * -1.4426950408889634f));   // -1 / ln 2
}
__device__ __forceinline__ float sigmoidf_acc(float v) { return sigmoid_pn(v); }

// ---------------------------------------------------------------------------
// end-of-launch bookkeeping, run by the last CTA to finish
// ---------------------------------------------------------------------------
// Every CTA calls this once, after all of its global writes.  The last CTA
// takes the stop decision for iterate i = ctrl->iter:
//   non-finite r -> PN_ERR_NONFINITE; r <= tol -> PN_OK;
//   i == max_iters -> PN_NOT_CONVERGED; otherwise continue with i+1.
__device__ __forceinline__ void finish_launch(const IterParams& P, const Args& A,
                                              unsigned epoch, int& is_last_smem) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    unsigned prev = atomicAdd(&P.ctrl->done, 1u);
    is_last_smem = (prev == gridDim.x - 1) ? 1 : 0;
  }
  __syncthreads();
  if (!is_last_smem || threadIdx.x != 0) return;
  __threadfence();
  Ctrl* c = P.ctrl;
  const int i = c->iter;
  const float r = __uint_as_float(atomicAdd(&c->resid_bits, 0u));
  const int err = ld_volatile(&c->error);
  if (i < kHistCap) P.hist[i] = r;
  int st = kRunning;
  if (err) st = err;
  else if (!(r <= 3.402823466e38f)) st = PN_ERR_NONFINITE;
  else if (r <= A.tol) st = PN_OK;
  else if (i >= A.max_iters) st = PN_NOT_CONVERGED;
  // adaptive switching (page §5.3): a stall, r^(i) > stall * r^(i-1), re-runs iteration i in the
  // next stronger mode -- the same rule as the host loop, applied here by the last CTA
  bool rerun = false;
  if (st == kRunning && A.adapt && A.use_cond && i >= 1 && !c->retried && i - 1 < kHistCap &&
      r > A.stall * P.hist[i - 1]) {
    const int mode = c->cur_mode;
    int next = (mode == PN_JACOBI || mode == PN_PICARD) ? PN_QUASI : PN_NEWTON;
    if (!((A.mode_ok >> next) & 1)) next = mode;
    if (next != mode) {
      c->cur_mode = next;
      c->retried = 1;
      rerun = true;
      for (int m = 0; m < 4; ++m) cudaGraphSetConditional(P.mode_cond[m], m == next ? 1u : 0u);
    }
  }
  if (st != kRunning) {
    c->status = st;
    c->final_iter = i;
    c->final_resid = r;
    c->final_fmt = c->fmt_in;
    if (A.use_cond) cudaGraphSetConditional(P.cond, 0u);
  } else if (!rerun) {
    if (A.adapt && i < kHistCap) P.mode_hist[i] = c->cur_mode;   // the mode of the kept update i
    c->retried = 0;
    c->iter = i + 1;
    // s^(i+2) is stored narrow while r^(i), the residual known when update i+1 starts, is above the bar
    c->fmt_in = c->fmt_out;
    c->fmt_out = (A.store_fmt != 0 && r > A.store_until) ? 1 : 0;
  }
  c->resid_bits = 0u;
#pragma unroll
  for (int g = 0; g < kMaxGroups; ++g) c->ticket[g] = 0u;
  c->done = 0u;
  c->epoch = epoch + 1u;
  const unsigned long long t1 = globaltimer();
  const unsigned long long t0 = c->t_start;
  if (t1 > t0) c->kernel_ns += t1 - t0;
  c->launches += 1ull;
  c->t_start = ~0ull;
  __threadfence();
}

// Grid barrier between the iterations of a looping kernel.  Every CTA calls
// it (all threads) after its part of the iteration and after all of its global
// writes; `rbits` is the CTA's residual maximum (float bits, read on thread 0).
// The last CTA to arrive applies the stop rule of finish_launch (iteration
// `iter`, look-back epoch `epoch`) and publishes the next generation of
// ctrl->gen together with the decision in its low bit, so the other CTAs learn
// both from the one word they wait on.  `gen_count` is the number of
// iterations this handle completed before this one.  Returns, for every thread
// of the CTA, whether another iteration follows (its iteration and epoch are
// one more).
//
// The decision needs no read after the arrival: each CTA adds to ctrl->arrive
// its arrival, whether its residual is above tol (or NaN) and whether it is
// non-finite, and every error raised counted itself there too, so the value
// the last arrival's atomic returns holds the whole rule (r <= tol exactly when
// no CTA's maximum is above it).  The residual value itself, for the history
// and the result, is read by the last CTA after the release, from the word of
// this iteration's parity, which it then clears for iteration iter + 2.
__device__ __forceinline__ bool finish_iteration(const IterParams& P, const Args& A, int iter, unsigned epoch,
                                                 int& flag_smem, unsigned gen_count, unsigned rbits) {
  __syncthreads();
  if (threadIdx.x == 0) {
    Ctrl* c = P.ctrl;
    unsigned* rw = &c->resid_loop[iter & 1];
    if (rbits) atomicMax(rw, rbits);
    unsigned long long mine = kArriveOne;
    if (__uint_as_float(rbits) > A.tol || rbits > 0x7f800000u) mine += kArriveHot;
    if (rbits >= 0x7f800000u) mine += kArriveBad;
    __threadfence();
    const unsigned long long prev = atomicAdd(&c->arrive, mine);
    int go = 0;
    if ((prev & kArriveMask) == (unsigned long long)(gridDim.x - 1)) {
      const unsigned long long tot = prev + mine;
      __threadfence();
      int st = kRunning;
      if (tot >> 60) {
        st = ld_volatile(&c->error);
        if (!st) st = PN_ERR_TIMEOUT;
      } else if ((tot >> 40) & kArriveMask) {
        st = PN_ERR_NONFINITE;
      } else if (((tot >> 20) & kArriveMask) == 0ull) {
        st = PN_OK;
      } else if (iter >= A.max_iters) {
        st = PN_NOT_CONVERGED;
      }
      c->launches += 1ull;
      if (st != kRunning) {
        c->status = st;
        c->final_iter = iter;
        c->final_fmt = c->fmt_in;
        const unsigned long long t1 = globaltimer();
        const unsigned long long t0 = c->t_start;
        if (t1 > t0) c->kernel_ns += t1 - t0;
        c->t_start = ~0ull;
      } else {
        c->iter = iter + 1;
        c->fmt_in = c->fmt_out;
        // narrow storage (not run by the looping kernels today) needs the value before the release
        c->fmt_out = (A.store_fmt != 0 && __uint_as_float(atomicAdd(rw, 0u)) > A.store_until) ? 1 : 0;
        go = 1;
      }
#pragma unroll
      for (int g = 0; g < kMaxGroups; ++g) c->ticket[g] = 0u;
      c->arrive = 0ull;
      c->epoch = epoch + 1u;
      __threadfence();
      st_release(&c->gen, ((gen_count + 1u) << 1) | (unsigned)go);
      // off the other CTAs' path: the residual of this iteration (every CTA folded its maximum
      // in before arriving), and its word cleared for iteration iter + 2
      const float r = __uint_as_float(atomicExch(rw, 0u));
      if (iter < kHistCap) P.hist[iter] = r;
      if (st != kRunning) c->final_resid = r;
    } else {
      const unsigned long long t0 = globaltimer();
      unsigned spins = 0;
      unsigned g;
      while (((g = ld_acquire(&c->gen)) >> 1) == (gen_count & 0x7fffffffu)) {
        if (((++spins) & 15u) == 0u && (long long)(globaltimer() - t0) > A.timeout_ns) {
          raise_error(c, (int)PN_ERR_TIMEOUT);
          break;
        }
        if (spins > 64u) __nanosleep(64);
      }
      go = ((g >> 1) != (gen_count & 0x7fffffffu)) && (g & 1u);
    }
    flag_smem = go;
  }
  __syncthreads();
  return flag_smem != 0;
}

}  // namespace pn
